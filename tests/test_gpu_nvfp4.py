"""NVFP4 linear layer on the GPU (block-scaled FP4 tensor-core MMAs) through
the C ABI against the fp64 oracle's decode of the same codes and scales.

Inputs are quantised by the input generator, so both sides multiply exactly
the same values: the GPU's only error is fp32 accumulation (and the bf16
rounding of a bf16 output)."""

import numpy as np
import pytest
import torch

import oracle as O
from synth.block_inputs import _normal, quantize_nvfp4
from tests._util import rel_l2
from tests.gpu_common import lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _operand(seed, name, rows, K, block, std):
    x = _normal(seed, 0, name, (rows, K), std)
    codes, sf, s = quantize_nvfp4(x, block)
    ref = O.dequant_nvfp4(codes.numpy(), sf.view(torch.uint8).numpy(), s.numpy())
    return codes, sf, s, ref


def _packed(ig4, sf):
    rows, k16 = sf.shape
    out = torch.empty(ig4.ig4_nvfp4_scale_bytes(rows, 16 * k16), dtype=torch.uint8, device="cuda")
    ig4.ig4_nvfp4_pack_scales(sf.view(torch.uint8).cuda(), out)
    return out


@pytest.mark.parametrize("M,N,K,out_dtype", [(128, 128, 256, torch.float32),
                                             (300, 384, 1024, torch.float32),
                                             (1000, 1024, 4608, torch.bfloat16),
                                             (77, 256, 12288, torch.float32),
                                             (128, 75776, 256, torch.float32),    # 256-wide tiles
                                             (4608, 4608, 512, torch.float32),    # CTA pairs
                                             (4600, 4608, 768, torch.bfloat16)])  # pairs, ragged M
def test_nvfp4_linear(ig4, M, N, K, out_dtype):
    a_codes, a_sf, a_s, a_ref = _operand(1, "a", M, K, 16, 1.0)        # activations: 16-blocks
    w_codes, w_sf, w_s, w_ref = _operand(2, "w", N, K, 64, 1.0 / np.sqrt(K))  # weights: 64-blocks
    bias = torch.from_numpy(_normal(3, 0, "bias", (N,), 0.1))
    out = torch.empty(M, N, dtype=out_dtype, device="cuda")
    ig4.ig4_nvfp4_linear(a_codes.cuda(), _packed(ig4, a_sf), a_s.cuda(), w_codes.cuda(),
                         _packed(ig4, w_sf), w_s.cuda(), bias.cuda(), out)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    got = out.cpu().double().numpy()
    ref = a_ref @ w_ref.T + bias.double().numpy()
    e = rel_l2(got, ref)
    print(f"nvfp4 linear {M}x{N}x{K}: relL2={e:.3e}")
    if out_dtype == torch.float32:
        assert e <= 2e-6
    else:
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref ** 2)))


def test_nvfp4_argument_errors(ig4):
    z = torch.zeros(12800, dtype=torch.uint8, device="cuda")
    f = torch.zeros(256, dtype=torch.float32, device="cuda")
    out = torch.empty(4, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(ig4.Ig4Error) as e:  # K = 200 is not a multiple of 256
        ig4.ig4_nvfp4_linear(z[:400].view(4, 100), z, f, z[:12800].view(128, 100), z, f, None, out)
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG
