"""MX8 activation quantiser on the GPU (E4M3 codes with a UE8M0 scale per 32
elements, the form the FP8 block's out- and down-projections consume)
through the C ABI against the oracle's quantize_mx8_activations: scale bytes
bit-exact, codes equal up to the sign of zero.  The block-scaled GEMM that
consumes MX8 is covered by the FP8 block and stack tests."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_common import lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _unpack_scales(packed: np.ndarray, M: int, K: int) -> np.ndarray:
    """[M, K/32] scale bytes from the tensor cores' chunk order."""
    r = np.arange(M)[:, None]
    b = np.arange(K // 32)[None, :]
    off = ((r >> 7) * (K >> 7) + (b >> 2)) * 512 + 16 * (r & 31) + 4 * ((r & 127) >> 5) + (b & 3)
    return packed[off]


@pytest.mark.parametrize("M,K", [(1, 128), (37, 384), (130, 4608), (300, 12288)])
def test_quantize_mx8_matches_oracle(ig4, M, K):
    g = torch.Generator().manual_seed(M * 7 + K)
    mag = torch.exp(torch.empty(M, K // 32, 1).uniform_(-12.0, 12.0, generator=g))
    x = (torch.randn(M, K // 32, 32, generator=g) * mag).reshape(M, K)
    x[0, :32] = 0.0                                   # an all-zero block
    if M > 2:
        x[2, 32:64] = 448.0 * 2.0 ** -20              # a block exactly at a power of two
    xb = x.to(torch.bfloat16)
    codes = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sf = torch.zeros(ig4.ig4_mx8_scale_bytes(M, K), dtype=torch.uint8, device="cuda")
    ig4.ig4_quantize_mx8(M, K, xb.cuda(), codes, sf)
    torch.cuda.synchronize()
    ref_codes, ref_sc = O.quantize_mx8_activations(xb.float().numpy())
    got_sc = _unpack_scales(sf.cpu().numpy(), M, K)
    assert np.array_equal(got_sc, ref_sc)
    dec = O.e4m3_decode_table()
    assert np.array_equal(dec[codes.cpu().numpy()], dec[ref_codes])


def test_quantize_mx8_rejects_bad_shapes(ig4):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((4, 256), dtype=torch.uint8, device="cuda")
    sf = torch.empty(512 * 2, dtype=torch.uint8, device="cuda")
    for M, K in [(0, 256), (4, 96), (4, 200)]:
        with pytest.raises(ig4.Ig4Error):
            ig4.ig4_quantize_mx8(M, K, x, codes, sf)
    assert ig4.ig4_mx8_scale_bytes(4, 100) == 0
    assert ig4.ig4_mx8_scale_bytes(130, 256) == 2 * 2 * 512
