"""The C-ABI library on the host: it loads, exports every entry point the
header declares, computes the position table exactly, and rejects bad
arguments before launching anything (so none of this needs a GPU)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ig4():
    from stream_diffusion_transformer_fwd_b200.build import build
    build()
    from stream_diffusion_transformer_fwd_b200 import ig4 as m
    return m


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "ig4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ig4_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_are_exported(ig4):
    declared = _declared_symbols()
    assert len(declared) >= 15
    lib = ig4.library()
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(ig4.EXPORTED) == declared


def test_status_strings_and_version(ig4):
    assert ig4.ig4_abi_version() == 2
    for code, name in enumerate(["IG4_OK", "IG4_ERR_INVALID_ARG", "IG4_ERR_UNSUPPORTED",
                                 "IG4_ERR_WORKSPACE", "IG4_ERR_CUDA", "IG4_ERR_TIMEOUT"]):
        assert ig4.ig4_status_string(code) == name
    assert ig4.ig4_status_string(99) == "IG4_ERR_UNKNOWN"


def test_struct_layouts_match_header(ig4, tmp_path):
    """ctypes mirrors of the header's structs have the C compiler's layout."""
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "ig4.h"\n'
        'int main(void) { printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(ig4_config),'
        ' offsetof(ig4_config, rope_theta), offsetof(ig4_config, eps), sizeof(ig4_block_weights),'
        ' sizeof(ig4_stack_weights), offsetof(ig4_stack_weights, w_in)); return 0; }\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals == [ctypes.sizeof(ig4.Config), ig4.Config.rope_theta.offset,
                    ig4.Config.eps.offset, ctypes.sizeof(ig4.BlockWeights),
                    ctypes.sizeof(ig4.StackWeights), ig4.StackWeights.w_in.offset]


@pytest.mark.parametrize("args", [(3, 1, 2, 3), (1, 2, 1, 2), (0, 1, 2, 2), (4, 1, 0, 0),
                                  (512, 1, 64, 64), (2048, 1, 128, 22), (32, 1, 8, 8)])
def test_host_positions_bit_exact(ig4, args):
    got = ig4.ig4_mrope_positions(*args).numpy()
    assert got.dtype == np.int32
    assert np.array_equal(got.astype(np.int64), O.mrope_positions(*args))


def test_positions_reject_bad_sizes(ig4):
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_mrope_positions(0, 1, 0, 0)
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG
    lib = ig4.library()
    assert lib.ig4_mrope_positions(-1, 1, 2, 2, ctypes.c_void_p(16), 0, None) == 1
    assert lib.ig4_mrope_positions(1, 1, 2, 2, None, 0, None) == 1


def _cfg(ig4, **kw):
    base = dict(B=1, T_text=32, grid_t=1, grid_h=8, grid_w=8, D=1024, H=4, I=2816,
                x_dtype="f32", w_dtype="bf16")
    base.update(kw)
    return ig4.make_config(**base)


def test_workspace_size(ig4):
    small = ig4.ig4_workspace_size(_cfg(ig4))
    big = ig4.ig4_workspace_size(_cfg(ig4, grid_h=16, grid_w=16))
    fp8 = ig4.ig4_workspace_size(_cfg(ig4, w_dtype="e4m3"))
    assert 0 < small < big and fp8 > small
    assert small % 256 == 0
    # invalid or unsupported configs report 0
    assert ig4.ig4_workspace_size(_cfg(ig4, head_dim=128)) == 0
    assert ig4.ig4_workspace_size(_cfg(ig4, D=1000)) == 0
    assert ig4.ig4_workspace_size(_cfg(ig4, sections=(24, 20, 21))) == 0
    assert ig4.ig4_workspace_size(_cfg(ig4, B=0)) == 0
    assert ig4.ig4_stack_workspace_size(_cfg(ig4, x_dtype="bf16")) > small
    assert ig4.ig4_stack_workspace_size(_cfg(ig4, x_dtype="f32")) == 0


class _Fake:
    """Stand-in for a device tensor: only its address is ever looked at."""

    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _weights(ig4, base=1 << 40, misalign=None):
    w = {}
    for i, (name, _) in enumerate(ig4.BlockWeights._fields_):
        w[name] = _Fake(base + i * (1 << 20) + (8 if name == misalign else 0))
    return ig4.block_weights(w)


def _call_block(ig4, cfg, bw, ws_bytes, x_in=1 << 41, x_out=1 << 42, ws=1 << 43):
    lib = ig4.library()
    return lib.ig4_block_forward(ctypes.byref(cfg), ctypes.byref(bw), ctypes.c_void_p(x_in),
                                 ctypes.c_void_p(x_out), ctypes.c_void_p(1 << 44),
                                 ctypes.c_void_p(1 << 45), ctypes.c_void_p(ws), ws_bytes, None)


def test_block_forward_validation_returns_before_launch(ig4):
    cfg = _cfg(ig4)
    need = ig4.ig4_workspace_size(cfg)
    bw = _weights(ig4)
    assert _call_block(ig4, cfg, bw, need - 1) == ig4.IG4_ERR_WORKSPACE
    assert _call_block(ig4, cfg, bw, need, ws=(1 << 43) + 128) == ig4.IG4_ERR_WORKSPACE
    assert _call_block(ig4, cfg, _weights(ig4, misalign="w_qkv"), need) == ig4.IG4_ERR_INVALID_ARG
    assert _call_block(ig4, cfg, bw, need, x_out=(1 << 41) + 64) == ig4.IG4_ERR_INVALID_ARG
    assert _call_block(ig4, _cfg(ig4, head_dim=128), bw, need) == ig4.IG4_ERR_UNSUPPORTED
    assert _call_block(ig4, _cfg(ig4, I=2800), bw, need) == ig4.IG4_ERR_UNSUPPORTED
    assert _call_block(ig4, _cfg(ig4, x_dtype=7), bw, need) == ig4.IG4_ERR_INVALID_ARG
    # E4M3 weights need their scales
    w = {name: _Fake((1 << 40) + i * (1 << 20)) for i, (name, _) in
         enumerate(ig4.BlockWeights._fields_) if not name.startswith("s_")}
    cfg8 = _cfg(ig4, w_dtype="e4m3")
    assert _call_block(ig4, cfg8, ig4.block_weights(w), ig4.ig4_workspace_size(cfg8)) == \
        ig4.IG4_ERR_INVALID_ARG


def test_op_validation_returns_before_launch(ig4):
    lib = ig4.library()
    p = ctypes.c_void_p(1 << 40)
    # GEMM shapes the tiles do not cover
    assert lib.ig4_gated_residual_linear(1, 8, 200, 64, p, 1, None, p, 1, None, p, 200, p, p, 1,
                                         None) == ig4.IG4_ERR_UNSUPPORTED
    assert lib.ig4_swiglu(8, 100, 64, p, 1, None, p, p, 1, None, None, p, None) == \
        ig4.IG4_ERR_UNSUPPORTED
    # E4M3 weights with bf16 activations are not a supported pairing
    assert lib.ig4_swiglu(8, 128, 128, p, 1, None, p, p, 2, p, p, p, None) == \
        ig4.IG4_ERR_UNSUPPORTED
    assert lib.ig4_joint_attention(1, 1, 10, p, p, p, 4, p, None) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_quantize_rows(4, 20000, p, p, p, None) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_selftest_timeout(0, None) == ig4.IG4_ERR_INVALID_ARG
    mhz = ctypes.c_double(0.0)
    assert lib.ig4_sm_clock_mhz(0, None, ctypes.byref(mhz)) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_sm_clock_mhz(100001, None, ctypes.byref(mhz)) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_sm_clock_mhz(20, None, None) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_adaln_modulation(9, 512, 8, p, p, 1, None, None, p, None) == \
        ig4.IG4_ERR_INVALID_ARG


def test_nvfp4_mixed_config_rules(ig4):
    """NVFP4 Mixed block configs: accepted with I % 256 == 0 and more than 128
    tokens; the workspace adds a bf16 h2 buffer and the packed scales."""
    def ws(T, gh, I, wd):
        return ig4.ig4_workspace_size(ig4.make_config(1, T, 1, gh, gh, D=1024, H=4, I=I,
                                                      w_dtype=wd))
    assert ws(64, 12, 2816, "nvfp4_mixed") > ws(64, 12, 2816, "e4m3") > 0
    assert ws(16, 8, 2816, "nvfp4_mixed") == 0      # 80 tokens
    assert ws(16, 8, 2816, "e4m3") > 0
    assert ws(64, 12, 2944, "nvfp4_mixed") == 0     # I = 23 x 128
    assert ws(64, 12, 2944, "e4m3") > 0


def test_nvfp4_validation_returns_before_launch(ig4):
    lib = ig4.library()
    p = ctypes.c_void_p(1 << 40)
    q = ctypes.c_void_p((1 << 40) + 8)  # not 16-byte aligned
    assert lib.ig4_nvfp4_quantize(4, 96, p, p, p, p, None) == ig4.IG4_ERR_INVALID_ARG  # K % 64
    assert lib.ig4_nvfp4_quantize(4, 128, q, p, p, p, None) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_nvfp4_quantize(0, 128, p, p, p, p, None) == ig4.IG4_ERR_INVALID_ARG
    assert lib.ig4_nvfp4_linear(8, 100, 256, p, p, p, p, p, p, None, p, 0, None) == \
        ig4.IG4_ERR_INVALID_ARG  # N % 128
    assert lib.ig4_nvfp4_linear(8, 128, 200, p, p, p, p, p, p, None, p, 0, None) == \
        ig4.IG4_ERR_INVALID_ARG  # K % 256
    assert ig4.ig4_nvfp4_scale_bytes(100, 100) == 0
    assert ig4.ig4_nvfp4_scale_bytes(129, 128) == 2 * 2 * 512
    # an NVFP4 Mixed block needs the FFN weights' packed scales
    cfg = ig4.make_config(1, 64, 1, 12, 12, D=1024, H=4, I=2816, w_dtype="nvfp4_mixed")
    need = ig4.ig4_workspace_size(cfg)
    w = {name: _Fake((1 << 40) + i * (1 << 20)) for i, (name, _) in
         enumerate(ig4.BlockWeights._fields_) if name != "sf_up"}
    assert _call_block(ig4, cfg, ig4.block_weights(w), need) == ig4.IG4_ERR_INVALID_ARG
