"""Text conditioning projection (llm_cond_norm + llm_cond_proj) on the GPU
through the C ABI against the fp64 oracle: in full at the pages' width
(53248 features -> 4608) for a 512-token caption, on sampled rows for 2048
tokens, at reduced width with a ragged token count, bf16 and E4M3 weights."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle.inputs import to_f64, weight_f64
from synth import make_text_cond_inputs
from tests._util import max_abs_over_rms, rel_l2
from tests.gpu_common import lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _run(ig4, inp, D, wdt):
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    M, K = inp["raw"].shape
    out = torch.empty(M, D, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ig4.ig4_text_cond_workspace_size(M, K, wdt), dtype=torch.uint8, device="cuda")
    ig4.ig4_text_cond_project(dev["raw"], dev["g_norm"], 1e-6, dev["w_proj"], dev["s_proj"],
                              dev["b_proj"], out, ws)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return to_f64(out.cpu())


def _ref(inp, rows=None):
    raw = to_f64(inp["raw"])
    if rows is not None:
        raw = raw[rows]
    return O.text_cond_projection(raw, to_f64(inp["g_norm"]), weight_f64(inp["w_proj"], inp["s_proj"]),
                                  to_f64(inp["b_proj"]))


@pytest.mark.parametrize("M,K,D,wdt", [(300, 1024, 512, "bf16"), (300, 1024, 512, "e4m3"),
                                       (512, 53248, 4608, "bf16"), (512, 53248, 4608, "e4m3")])
def test_text_cond_full(ig4, M, K, D, wdt):
    inp = make_text_cond_inputs(M, K, D, wdt, seed=2, stress=True)
    got = _run(ig4, inp, D, wdt)
    ref = _ref(inp)
    e, m = rel_l2(got, ref), max_abs_over_rms(got, ref)
    print(f"text cond {M}x{K}->{D} {wdt}: relL2={e:.3e} maxabs/rms={m:.3e}")
    if wdt == "bf16":
        assert e <= 1e-2 and m <= 5e-2
    else:
        assert e <= 3e-2


def test_text_cond_2048_tokens_sampled(ig4):
    M, K, D = 2048, 53248, 4608
    inp = make_text_cond_inputs(M, K, D, "bf16", seed=3, stress=True)
    got = _run(ig4, inp, D, "bf16")
    rows = np.random.default_rng(0).choice(M, 48, replace=False)
    rows = np.concatenate([rows, [0, M - 1]])
    ref = _ref(inp, rows)
    e, m = rel_l2(got[rows], ref), max_abs_over_rms(got[rows], ref)
    print(f"text cond 2048 tokens sampled: relL2={e:.3e} maxabs/rms={m:.3e}")
    assert e <= 1e-2 and m <= 5e-2


def test_text_cond_argument_errors(ig4):
    inp = make_text_cond_inputs(8, 1000, 256, "bf16", seed=1)  # K_raw not a multiple of 128
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    out = torch.empty(8, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_text_cond_project(dev["raw"], dev["g_norm"], 1e-6, dev["w_proj"], None,
                                  dev["b_proj"], out, ws)
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG
