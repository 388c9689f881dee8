"""ig4_block_forward_noalloc: the block forward for callers that cannot
allocate device memory (runtimes that plan all device memory ahead and forbid
allocation while executing, real-time loops that cannot pay for cudaMalloc,
hosts whose own allocator owns the GPU).  It runs the same kernels as
ig4_block_forward on the library's static scratch array instead of a caller
workspace; this file checks, through the C ABI, that two calls in a row (the
second on a different problem, with the first call's data left in the
scratch) match ig4_block_forward within the block tolerance, and that a
problem larger than the scratch is refused before anything is launched.

Kept in a file of its own that pytest collects last.
"""

import ctypes

import numpy as np
import pytest
import torch

from synth import CONFIGS, make_block_activations, make_block_weights
from tests._util import max_abs_over_rms, rel_l2
from tests.gpu_common import lib, run_block, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(ig4, cfg, wd, x, temb):
    c = ig4.config_from(cfg)
    pos = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w,
                                  device=x.device)
    y = torch.empty_like(x)
    lib_ = ig4.library()
    st = lib_.ig4_block_forward_noalloc(ctypes.byref(c), ctypes.byref(ig4.block_weights(wd)),
                                        ctypes.c_void_p(x.data_ptr()),
                                        ctypes.c_void_p(y.data_ptr()),
                                        ctypes.c_void_p(pos.data_ptr()),
                                        ctypes.c_void_p(temb.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ig4.IG4_OK, ig4.ig4_status_string(st)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return y


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row(cuda_device):
    ig4 = lib()
    calls = [
        (CONFIGS["tiny"], 21),
        (CONFIGS["tiny"].with_(name="b2_bf16", B=2, T_text=5, grid_h=7, grid_w=9, D=512, H=2,
                               I=384, x_dtype="bf16"), 22),
    ]
    for cfg, seed in calls:
        acts = make_block_activations(cfg, seed=seed)
        wd = to_dev(make_block_weights(cfg, seed=seed, stress=True))
        x = acts["x"].cuda()
        temb = acts["temb"].cuda()
        y_ws = run_block(ig4, cfg, wd, x, temb).double().cpu().numpy()
        y = _noalloc(ig4, cfg, wd, x, temb).double().cpu().numpy()
        e = rel_l2(y, y_ws)
        m = max_abs_over_rms(y, y_ws)
        print(f"{cfg.name}: noalloc vs workspace relL2={e:.3e} maxabs/rms={m:.3e}")
        assert e <= 1e-2 and m <= 5e-2
        assert np.all(np.isfinite(y))


def test_noalloc_refuses_problems_larger_than_its_scratch(cuda_device):
    ig4 = lib()
    cfg = CONFIGS["512px"]
    c = ig4.config_from(cfg)
    assert ig4.ig4_workspace_size(c) > ig4.IG4_NOALLOC_SCRATCH_BYTES
    # Only pointer values are inspected before the size check refuses the call.
    fake = {name: type("T", (), {"data_ptr": (lambda self, a=(1 << 40) + i * (1 << 20): a)})()
            for i, (name, _) in enumerate(ig4.BlockWeights._fields_)}
    st = ig4.library().ig4_block_forward_noalloc(
        ctypes.byref(c), ctypes.byref(ig4.block_weights(fake)), ctypes.c_void_p(1 << 41),
        ctypes.c_void_p(1 << 42), ctypes.c_void_p(1 << 43), ctypes.c_void_p(1 << 44), None)
    assert st == ig4.IG4_ERR_WORKSPACE
