"""ig4_block_forward_noalloc: the block forward for callers that cannot
allocate device memory (runtimes that plan all device memory ahead and forbid
allocation while executing, real-time loops that cannot pay for cudaMalloc,
hosts whose own allocator owns the GPU).  It runs the same kernels as
ig4_block_forward on the library's static scratch array instead of a caller
workspace, so its output must be bit-identical to ig4_block_forward's.

Checked here, through the C ABI:
  * calls in a row on different problems and weight formats (bf16, E4M3,
    NVFP4 Mixed), each reading a scratch array that the previous call left
    filled with another layout's data, each equal to ig4_block_forward;
  * a problem at the scratch limit (the 1024-wide block at 4094 tokens),
    equal to ig4_block_forward and within the block tolerance of the oracle
    on sampled rows;
  * one token more is refused with IG4_ERR_WORKSPACE and launches nothing.

Kept in a file of its own that pytest collects last.
"""

import ctypes

import pytest
import torch

import oracle as O
from oracle.inputs import block_weights_f64, to_f64
from synth import CONFIGS, make_block_activations, make_block_weights
from tests.gpu_common import check_output, lib, run_block, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def _call_noalloc(ig4, cfg, wd, x, y, temb):
    c = ig4.config_from(cfg)
    pos = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w,
                                  device=x.device)
    return ig4.library().ig4_block_forward_noalloc(
        ctypes.byref(c), ctypes.byref(ig4.block_weights(wd)), ctypes.c_void_p(x.data_ptr()),
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(pos.data_ptr()),
        ctypes.c_void_p(temb.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _noalloc(ig4, cfg, wd, x, temb):
    y = torch.empty_like(x)
    st = _call_noalloc(ig4, cfg, wd, x, y, temb)
    assert st == ig4.IG4_OK, ig4.ig4_status_string(st)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return y


def _weights(ig4, cfg, seed):
    wd = to_dev(make_block_weights(cfg, seed=seed, stress=True))
    if cfg.w_dtype == "nvfp4_mixed":
        wd = ig4.nvfp4_pack_block_scales(wd)
    return wd


SMALL = CONFIGS["tiny"]
CALLS = [
    (SMALL, 21),
    (SMALL.with_(name="b2_bf16", B=2, T_text=5, grid_h=7, grid_w=9, D=512, H=2, I=384,
                 x_dtype="bf16"), 22),
    (SMALL.with_(name="tiny_fp8", w_dtype="e4m3"), 23),
    (CONFIGS["small_nvfp4"], 24),
    (SMALL.with_(name="b2_fp8", B=2, T_text=5, grid_h=7, grid_w=9, D=512, H=2, I=384,
                 x_dtype="bf16", w_dtype="e4m3"), 25),
    (SMALL.with_(name="tiny_bf16_again"), 26),
]


def test_noalloc_equals_workspace_entry_point_calls_in_a_row(cuda_device):
    ig4 = lib()
    for cfg, seed in CALLS:
        acts = make_block_activations(cfg, seed=seed)
        wd = _weights(ig4, cfg, seed)
        x = acts["x"].cuda()
        temb = acts["temb"].cuda()
        y_ws = run_block(ig4, cfg, wd, x, temb)
        y = _noalloc(ig4, cfg, wd, x, temb)
        y2 = _noalloc(ig4, cfg, wd, x, temb)
        print(f"{cfg.name}: noalloc == workspace: {torch.equal(y, y_ws)}")
        assert torch.equal(y, y_ws), cfg.name
        assert torch.equal(y2, y_ws), cfg.name


# 1024-wide block at 4094 tokens: the largest bf16-weight problem of this
# width whose workspace fits in the scratch array
AT_LIMIT = SMALL.with_(name="limit_1024", T_text=254, grid_h=60, grid_w=64, x_dtype="bf16")


def test_noalloc_at_the_scratch_limit(cuda_device):
    ig4 = lib()
    cfg = AT_LIMIT
    c = ig4.config_from(cfg)
    need = ig4.ig4_workspace_size(c)
    assert need <= ig4.IG4_NOALLOC_SCRATCH_BYTES
    assert need > ig4.IG4_NOALLOC_SCRATCH_BYTES - (1 << 20)
    acts = make_block_activations(cfg, seed=27)
    wts = make_block_weights(cfg, seed=27, stress=True)
    wd = to_dev(wts)
    x = acts["x"].cuda()
    temb = acts["temb"].cuda()
    y = _noalloc(ig4, cfg, wd, x, temb)
    assert torch.equal(y, run_block(ig4, cfg, wd, x, temb))
    rows = sample_rows(cfg, n=48)
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    x64 = to_f64(acts["x"])
    y_ref = O.block_forward_rows(x64, to_f64(acts["temb"]), pos, block_weights_f64(wts), cfg.H,
                                 rows, cfg.rope_theta, cfg.sections, cfg.eps)
    got = y.float().cpu().double().numpy().reshape(cfg.M, cfg.D)[rows]
    check_output(got, y_ref, x64.reshape(cfg.M, cfg.D)[rows], False, True, cfg.name)


def test_noalloc_refuses_problems_larger_than_its_scratch(cuda_device):
    ig4 = lib()
    cfg = AT_LIMIT.with_(name="over_limit", T_text=AT_LIMIT.T_text + 1)
    c = ig4.config_from(cfg)
    assert ig4.ig4_workspace_size(c) > ig4.IG4_NOALLOC_SCRATCH_BYTES
    acts = make_block_activations(cfg, seed=28)
    wd = to_dev(make_block_weights(cfg, seed=28))
    x = acts["x"].cuda()
    y = torch.full_like(x, 7.0)
    st = _call_noalloc(ig4, cfg, wd, x, y, acts["temb"].cuda())
    assert st == ig4.IG4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    assert bool((y == 7.0).all())  # nothing was launched
