"""Python binding of libig4 (include/ig4.h): an sm_100a implementation of the
Ideogram 4 single-stream DiT block forward and the 34-block stack.

Argument marshalling only: every step of the block runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current CUDA stream.  The
functions carry the C entry points' names; each raises Ig4Error on a status
other than IG4_OK.  Importing the package fails loudly if the shared library
is missing (build it with ``python -m stream_diffusion_transformer_fwd_b200.build``).
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libig4.so")

IG4_OK, IG4_ERR_INVALID_ARG, IG4_ERR_UNSUPPORTED, IG4_ERR_WORKSPACE, IG4_ERR_CUDA, \
    IG4_ERR_TIMEOUT = range(6)
IG4_F32, IG4_BF16, IG4_E4M3, IG4_NVFP4_MIXED = 0, 1, 2, 3
IG4_ABI_VERSION = 2  # the include/ig4.h revision this binding marshals for
IG4_BLOCK_TRACE_EVENTS = 12
IG4_NOALLOC_SCRATCH_BYTES = 64 << 20

_DTYPE_CODE = {torch.float32: IG4_F32, torch.bfloat16: IG4_BF16, torch.float8_e4m3fn: IG4_E4M3}
_CODE_NAME = {IG4_F32: "f32", IG4_BF16: "bf16", IG4_E4M3: "e4m3", IG4_NVFP4_MIXED: "nvfp4_mixed"}
_NAME_CODE = {v: k for k, v in _CODE_NAME.items()}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m stream_diffusion_transformer_fwd_b200.build`"
        " (there is no fallback implementation)")
_lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float


class Ig4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.ig4_status_string(status).decode()}")


class Config(ctypes.Structure):
    _fields_ = [("B", _i), ("T_text", _i), ("grid_t", _i), ("grid_h", _i), ("grid_w", _i),
                ("D", _i), ("H", _i), ("head_dim", _i), ("I", _i), ("adaln_dim", _i),
                ("rope_theta", ctypes.c_double), ("sections", _i * 3), ("eps", _f),
                ("x_dtype", _i), ("w_dtype", _i)]


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("w_ada", "w_qkv", "w_o", "w_gate", "w_up", "w_down",
                                   "s_ada", "s_qkv", "s_o", "s_gate", "s_up", "s_down",
                                   "b_ada", "g_q", "g_k", "sf_gate", "sf_up", "sf_down")]


class StackWeights(ctypes.Structure):
    _fields_ = [("n_blocks", _i), ("latent_ch", _i), ("blocks", ctypes.POINTER(BlockWeights)),
                ("w_in", _vp), ("s_in", _vp), ("b_in", _vp),
                ("w_f", _vp), ("s_f", _vp), ("b_f", _vp),
                ("w_out", _vp), ("s_out", _vp), ("b_out", _vp)]


def _sig(name, args, res=_i):
    fn = getattr(_lib, name)
    fn.argtypes = args
    fn.restype = res
    return fn


_lib.ig4_status_string.argtypes = [_i]
_lib.ig4_status_string.restype = ctypes.c_char_p
_sig("ig4_abi_version", [])
if _lib.ig4_abi_version() != IG4_ABI_VERSION:
    raise ImportError(f"{LIB_PATH} has ABI revision {_lib.ig4_abi_version()}, this binding expects "
                      f"{IG4_ABI_VERSION}: rebuild it")
_sig("ig4_mrope_positions", [_i, _i, _i, _i, _vp, _i, _vp])
_sig("ig4_rope_table", [_i, _vp, ctypes.c_double, ctypes.POINTER(_i), _vp, _vp, _vp])
_sig("ig4_adaln_modulation", [_i, _i, _i, _vp, _vp, _i, _vp, _vp, _vp, _vp])
_sig("ig4_norm_modulate", [_i, _i, _i, _vp, _i, _vp, _vp, _i, _f, _vp, _i, _vp, _vp])
_sig("ig4_qkv_project", [_i, _i, _i, _i, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _f, _vp, _vp,
                         _vp, _vp, _vp, _i, _vp])
_sig("ig4_joint_attention", [_i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp])
_sig("ig4_joint_attention_workspace_size", [_i, _i, _i], ctypes.c_size_t)
_sig("ig4_joint_attention_ws", [_i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp, ctypes.c_size_t, _vp])
_sig("ig4_gated_residual_linear", [_i, _i, _i, _i, _vp, _i, _vp, _vp, _i, _vp, _vp, _i, _vp,
                                   _vp, _i, _vp])
_sig("ig4_swiglu", [_i, _i, _i, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp])
_sig("ig4_quantize_rows", [_i, _i, _vp, _vp, _vp, _vp])
_sig("ig4_quantize_mx8", [_i, _i, _vp, _vp, _vp, _vp])
_sig("ig4_mx8_scale_bytes", [_i, _i], ctypes.c_size_t)
_sig("ig4_workspace_size", [ctypes.POINTER(Config)], ctypes.c_size_t)
_sig("ig4_block_forward", [ctypes.POINTER(Config), ctypes.POINTER(BlockWeights), _vp, _vp, _vp,
                           _vp, _vp, ctypes.c_size_t, _vp])
_sig("ig4_block_forward_traced", [ctypes.POINTER(Config), ctypes.POINTER(BlockWeights), _vp, _vp,
                                  _vp, _vp, _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_vp), _i])
_sig("ig4_block_forward_noalloc", [ctypes.POINTER(Config), ctypes.POINTER(BlockWeights), _vp,
                                   _vp, _vp, _vp, _vp])
_sig("ig4_stack_workspace_size", [ctypes.POINTER(Config), _i], ctypes.c_size_t)
_sig("ig4_stack_forward", [ctypes.POINTER(Config), ctypes.POINTER(StackWeights), _vp, _vp, _vp,
                           _vp, _vp, _vp, ctypes.c_size_t, _vp])
_sig("ig4_stack_forward_tapped", [ctypes.POINTER(Config), ctypes.POINTER(StackWeights), _vp, _vp,
                                  _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_i),
                                  ctypes.POINTER(_vp), _i])
_sig("ig4_nvfp4_scale_bytes", [_i, _i], ctypes.c_size_t)
_sig("ig4_nvfp4_pack_scales", [_i, _i, _vp, _vp, _vp])
_sig("ig4_nvfp4_linear", [_i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp])
_sig("ig4_nvfp4_quantize", [_i, _i, _vp, _vp, _vp, _vp, _vp])
_sig("ig4_text_cond_workspace_size", [_i, _i, _i], ctypes.c_size_t)
_sig("ig4_text_cond_project", [_i, _i, _i, _vp, _vp, _f, _vp, _vp, _i, _vp, _vp, _vp,
                               ctypes.c_size_t, _vp])
_sig("ig4_flow_schedule", [_i, ctypes.c_double, ctypes.c_double, _i, _i,
                           ctypes.POINTER(ctypes.c_double)])
_sig("ig4_guidance_schedule", [_i, _i, _f, _f, ctypes.POINTER(_f)])
_sig("ig4_cfg_euler", [ctypes.c_longlong, _vp, _vp, _f, _f, _vp, _vp, _vp, _vp])
_sig("ig4_denoise_workspace_size", [ctypes.POINTER(Config), _i], ctypes.c_size_t)
_sig("ig4_denoise_step", [ctypes.POINTER(Config), ctypes.POINTER(StackWeights),
                          ctypes.POINTER(StackWeights), _vp, _vp, _vp, _vp, _vp, _vp, _f, _f, _f,
                          _vp, ctypes.c_size_t, _vp])
_sig("ig4_tp_workspace_size", [ctypes.POINTER(Config), _i], ctypes.c_size_t)
_sig("ig4_block_tp_attention", [ctypes.POINTER(Config), _i, _i, ctypes.POINTER(BlockWeights), _vp,
                                _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp])
_sig("ig4_block_tp_mlp", [ctypes.POINTER(Config), _i, _i, ctypes.POINTER(BlockWeights), _vp, _vp,
                          _vp, ctypes.c_size_t, _vp])
_sig("ig4_tp_reduce", [ctypes.c_longlong, _i, ctypes.POINTER(_vp), _vp, _i, _vp])
_sig("ig4_sp_image_range", [ctypes.POINTER(Config), _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)])
_sig("ig4_sp_positions", [ctypes.POINTER(Config), _i, _i, _vp, _i, _vp])
_sig("ig4_sp_workspace_size", [ctypes.POINTER(Config), _i, _i], ctypes.c_size_t)
_sig("ig4_sp_exchange_bytes", [ctypes.POINTER(Config), _i, _i, _i, _i], ctypes.c_size_t)
_sig("ig4_block_sp_pre", [ctypes.POINTER(Config), _i, _i, ctypes.POINTER(BlockWeights), _vp, _vp,
                          _vp, _vp, _vp, ctypes.c_size_t, _vp])
_sig("ig4_block_sp_attention", [ctypes.POINTER(Config), _i, _i, _vp, _vp, _vp, ctypes.c_size_t,
                                _vp])
_sig("ig4_block_sp_post", [ctypes.POINTER(Config), _i, _i, ctypes.POINTER(BlockWeights), _vp, _vp,
                           _vp, _vp, ctypes.c_size_t, _vp])
_sig("ig4_last_device_error", [_vp])
_sig("ig4_selftest_timeout", [_i, _vp])
_sig("ig4_sm_clock_mhz", [_i, _vp, ctypes.POINTER(ctypes.c_double)])

EXPORTED = ("ig4_status_string", "ig4_abi_version", "ig4_mrope_positions", "ig4_rope_table",
            "ig4_adaln_modulation", "ig4_norm_modulate", "ig4_qkv_project",
            "ig4_joint_attention", "ig4_joint_attention_workspace_size", "ig4_joint_attention_ws",
            "ig4_gated_residual_linear", "ig4_swiglu",
            "ig4_quantize_rows", "ig4_quantize_mx8", "ig4_mx8_scale_bytes", "ig4_workspace_size",
            "ig4_block_forward",
            "ig4_block_forward_traced", "ig4_block_forward_noalloc", "ig4_stack_workspace_size",
            "ig4_stack_forward", "ig4_stack_forward_tapped", "ig4_nvfp4_scale_bytes", "ig4_nvfp4_pack_scales",
            "ig4_nvfp4_linear", "ig4_nvfp4_quantize", "ig4_text_cond_workspace_size", "ig4_text_cond_project",
            "ig4_flow_schedule", "ig4_guidance_schedule", "ig4_cfg_euler",
            "ig4_denoise_workspace_size", "ig4_denoise_step", "ig4_tp_workspace_size",
            "ig4_block_tp_attention", "ig4_block_tp_mlp", "ig4_tp_reduce", "ig4_sp_image_range",
            "ig4_sp_positions", "ig4_sp_workspace_size", "ig4_sp_exchange_bytes",
            "ig4_block_sp_pre", "ig4_block_sp_attention", "ig4_block_sp_post",
            "ig4_last_device_error", "ig4_selftest_timeout", "ig4_sm_clock_mhz")


def library():
    """The loaded ctypes library (for tests that call entry points directly)."""
    return _lib


# ------------------------------------------------------------------ helpers

def _check(status: int, where: str):
    if status != IG4_OK:
        raise Ig4Error(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(0)


def dtype_code(t: torch.Tensor) -> int:
    return _DTYPE_CODE[t.dtype]


def make_config(B, T_text, grid_t, grid_h, grid_w, D=4608, H=18, head_dim=256, I=12288,
                adaln_dim=512, rope_theta=5.0e6, sections=(24, 20, 20), eps=1e-6,
                x_dtype="bf16", w_dtype="bf16") -> Config:
    c = Config()
    c.B, c.T_text, c.grid_t, c.grid_h, c.grid_w = B, T_text, grid_t, grid_h, grid_w
    c.D, c.H, c.head_dim, c.I, c.adaln_dim = D, H, head_dim, I, adaln_dim
    c.rope_theta = rope_theta
    c.sections = (_i * 3)(*sections)
    c.eps = eps
    c.x_dtype = _NAME_CODE[x_dtype] if isinstance(x_dtype, str) else x_dtype
    c.w_dtype = _NAME_CODE[w_dtype] if isinstance(w_dtype, str) else w_dtype
    return c


def config_from(cfg) -> Config:
    """Config from any object with the ig4_config field names (e.g. synth.Config)."""
    return make_config(cfg.B, cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w, cfg.D, cfg.H,
                       cfg.head_dim, cfg.I, cfg.adaln_dim, cfg.rope_theta, tuple(cfg.sections),
                       cfg.eps, cfg.x_dtype, cfg.w_dtype)


def nvfp4_pack_block_scales(w: dict, stream=None) -> dict:
    """For NVFP4-mixed block weights on the device: adds sf_gate / sf_up /
    sf_down, the packed block scales (ig4_nvfp4_pack_scales) of the row-major
    scales sfr_gate / sfr_up / sfr_down."""
    out = dict(w)
    for name in ("gate", "up", "down"):
        rows = w["sfr_" + name]
        packed = torch.empty(ig4_nvfp4_scale_bytes(rows.shape[0], 16 * rows.shape[1]),
                             dtype=torch.uint8, device=rows.device)
        ig4_nvfp4_pack_scales(rows, packed, stream)
        out["sf_" + name] = packed
    return out


def block_weights(w: dict) -> BlockWeights:
    """BlockWeights from a dict of device tensors (keys as in ig4_block_weights)."""
    bw = BlockWeights()
    for name, _ in BlockWeights._fields_:
        t = w.get(name)
        setattr(bw, name, None if t is None else t.data_ptr())
    return bw


# --------------------------------------------------------------- entry points

def ig4_status_string(status: int) -> str:
    return _lib.ig4_status_string(status).decode()


def ig4_abi_version() -> int:
    return _lib.ig4_abi_version()


def ig4_mrope_positions(T_text, grid_t, grid_h, grid_w, out: torch.Tensor | None = None,
                        device=None, stream=None) -> torch.Tensor:
    """int32 [3, L] position table, on `device` (default: host)."""
    L = T_text + grid_t * grid_h * grid_w
    if out is None:
        out = torch.empty((3, L), dtype=torch.int32,
                          device=device if device is not None else "cpu")
    on_dev = 1 if out.is_cuda else 0
    _check(_lib.ig4_mrope_positions(T_text, grid_t, grid_h, grid_w, _ptr(out), on_dev,
                                    _stream(stream) if on_dev else None), "ig4_mrope_positions")
    return out


def ig4_rope_table(pos, rope_theta, sections, cos_out, sin_out, stream=None):
    L = pos.shape[1]
    sec = (_i * 3)(*sections)
    _check(_lib.ig4_rope_table(L, _ptr(pos), rope_theta, sec, _ptr(cos_out), _ptr(sin_out),
                               _stream(stream)), "ig4_rope_table")


def ig4_adaln_modulation(temb, w, w_scale, bias, mod_out, stream=None):
    B, A = temb.shape
    N = w.shape[0]
    _check(_lib.ig4_adaln_modulation(B, A, N, _ptr(temb), _ptr(w), dtype_code(w), _ptr(w_scale),
                                     _ptr(bias), _ptr(mod_out), _stream(stream)),
           "ig4_adaln_modulation")


def ig4_norm_modulate(B, L, D, x, shift, scale, mod_stride, eps, h_out, h_scale_out=None,
                      stream=None):
    _check(_lib.ig4_norm_modulate(B, L, D, _ptr(x), dtype_code(x), _ptr(shift), _ptr(scale),
                                  mod_stride, eps, _ptr(h_out), dtype_code(h_out),
                                  _ptr(h_scale_out), _stream(stream)), "ig4_norm_modulate")


def ig4_qkv_project(B, L, D, H, h, h_scale, w_qkv, w_scale, g_q, g_k, eps, rope_cos, rope_sin,
                    q_out, k_out, vt_out, vt_ld, stream=None):
    _check(_lib.ig4_qkv_project(B, L, D, H, _ptr(h), dtype_code(h), _ptr(h_scale), _ptr(w_qkv),
                                dtype_code(w_qkv), _ptr(w_scale), _ptr(g_q), _ptr(g_k), eps,
                                _ptr(rope_cos), _ptr(rope_sin), _ptr(q_out), _ptr(k_out),
                                _ptr(vt_out), vt_ld, _stream(stream)), "ig4_qkv_project")


def ig4_joint_attention(B, H, L, q, k, vt, vt_ld, o_out, stream=None):
    _check(_lib.ig4_joint_attention(B, H, L, _ptr(q), _ptr(k), _ptr(vt), vt_ld, _ptr(o_out),
                                    _stream(stream)), "ig4_joint_attention")


def ig4_joint_attention_workspace_size(B: int, H: int, L: int) -> int:
    return int(_lib.ig4_joint_attention_workspace_size(B, H, L))


def ig4_joint_attention_ws(B, H, L, q, k, vt, vt_ld, o_out, workspace, stream=None):
    """ig4_joint_attention on the balanced persistent grid (workspace from
    ig4_joint_attention_workspace_size; may be empty)."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_joint_attention_ws(B, H, L, _ptr(q), _ptr(k), _ptr(vt), vt_ld, _ptr(o_out),
                                       _ptr(workspace) if ws_bytes else None, ws_bytes,
                                       _stream(stream)), "ig4_joint_attention_ws")


def ig4_gated_residual_linear(B, L, N, K, a, a_scale, w, w_scale, gate, gate_stride, x_res,
                              x_out, stream=None):
    _check(_lib.ig4_gated_residual_linear(B, L, N, K, _ptr(a), dtype_code(a), _ptr(a_scale),
                                          _ptr(w), dtype_code(w), _ptr(w_scale), _ptr(gate),
                                          gate_stride, _ptr(x_res), _ptr(x_out),
                                          dtype_code(x_out), _stream(stream)),
           "ig4_gated_residual_linear")


def ig4_swiglu(M, I, K, h, h_scale, w_gate, w_up, s_gate, s_up, u_out, stream=None):
    _check(_lib.ig4_swiglu(M, I, K, _ptr(h), dtype_code(h), _ptr(h_scale), _ptr(w_gate),
                           _ptr(w_up), dtype_code(w_gate), _ptr(s_gate), _ptr(s_up), _ptr(u_out),
                           _stream(stream)), "ig4_swiglu")


def ig4_quantize_rows(M, K, x, q_out, scale_out, stream=None):
    _check(_lib.ig4_quantize_rows(M, K, _ptr(x), _ptr(q_out), _ptr(scale_out), _stream(stream)),
           "ig4_quantize_rows")


def ig4_quantize_mx8(M, K, x, codes_out, sf_out, stream=None):
    _check(_lib.ig4_quantize_mx8(M, K, _ptr(x), _ptr(codes_out), _ptr(sf_out), _stream(stream)),
           "ig4_quantize_mx8")


def ig4_mx8_scale_bytes(M, K) -> int:
    return int(_lib.ig4_mx8_scale_bytes(M, K))


def ig4_workspace_size(cfg: Config) -> int:
    return int(_lib.ig4_workspace_size(ctypes.byref(cfg)))


def ig4_block_forward(cfg: Config, weights: BlockWeights, x_in, x_out, pos, temb, workspace,
                      events=None, stream=None):
    """x_out = block(x_in).  `events`: optional list of IG4_BLOCK_TRACE_EVENTS
    torch.cuda.Event(enable_timing=True) (or None: that boundary is not recorded)
    recorded around each kernel."""
    ws_bytes = workspace.numel() * workspace.element_size()
    if events is None:
        st = _lib.ig4_block_forward(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x_in),
                                    _ptr(x_out), _ptr(pos), _ptr(temb), _ptr(workspace),
                                    ws_bytes, _stream(stream))
        _check(st, "ig4_block_forward")
        return
    for e in events:  # make sure each event owns a CUDA handle
        if e is not None:
            e.record(stream) if stream is not None else e.record()
    arr = (_vp * len(events))(*[None if e is None else e.cuda_event for e in events])
    st = _lib.ig4_block_forward_traced(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x_in),
                                       _ptr(x_out), _ptr(pos), _ptr(temb), _ptr(workspace),
                                       ws_bytes, _stream(stream), arr, len(events))
    _check(st, "ig4_block_forward_traced")


def ig4_block_forward_noalloc(cfg: Config, weights: BlockWeights, x_in, x_out, pos, temb,
                              stream=None):
    """x_out = block(x_in) with the library's static scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/ig4.h)."""
    _check(_lib.ig4_block_forward_noalloc(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x_in),
                                          _ptr(x_out), _ptr(pos), _ptr(temb), _stream(stream)),
           "ig4_block_forward_noalloc")


def ig4_stack_workspace_size(cfg: Config, latent_ch: int = 128) -> int:
    return int(_lib.ig4_stack_workspace_size(ctypes.byref(cfg), latent_ch))


def stack_weights(blocks: list, w_in, s_in, b_in, w_f, s_f, b_f, w_out, s_out, b_out,
                  latent_ch=128) -> StackWeights:
    arr = (BlockWeights * max(1, len(blocks)))(*blocks)
    sw = StackWeights()
    sw.n_blocks = len(blocks)
    sw.latent_ch = latent_ch
    sw.blocks = ctypes.cast(arr, ctypes.POINTER(BlockWeights))
    sw._keep = arr  # keep the host array alive with the struct
    for name, t in (("w_in", w_in), ("s_in", s_in), ("b_in", b_in), ("w_f", w_f), ("s_f", s_f),
                    ("b_f", b_f), ("w_out", w_out), ("s_out", s_out), ("b_out", b_out)):
        setattr(sw, name, None if t is None else t.data_ptr())
    return sw


def ig4_stack_forward(cfg: Config, sw: StackWeights, x_latent, text, out_latent, pos, temb,
                      workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_stack_forward(ctypes.byref(cfg), ctypes.byref(sw), _ptr(x_latent),
                                  _ptr(text), _ptr(out_latent), _ptr(pos), _ptr(temb),
                                  _ptr(workspace), ws_bytes, _stream(stream)),
           "ig4_stack_forward")


def ig4_stack_forward_tapped(cfg: Config, sw: StackWeights, x_latent, text, out_latent, pos,
                             temb, workspace, taps: dict, stream=None):
    """ig4_stack_forward that copies the bf16 sequence [B, L, D] entering block i
    into taps[i] (a device tensor) for each key i (i == n_blocks: after the last block)."""
    ws_bytes = workspace.numel() * workspace.element_size()
    idx = list(taps)
    blocks = (_i * max(1, len(idx)))(*idx)
    outs = (_vp * max(1, len(idx)))(*[taps[i].data_ptr() for i in idx])
    _check(_lib.ig4_stack_forward_tapped(ctypes.byref(cfg), ctypes.byref(sw), _ptr(x_latent),
                                         _ptr(text), _ptr(out_latent), _ptr(pos), _ptr(temb),
                                         _ptr(workspace), ws_bytes, _stream(stream), blocks, outs,
                                         len(idx)), "ig4_stack_forward_tapped")


def ig4_nvfp4_scale_bytes(rows: int, K: int) -> int:
    return int(_lib.ig4_nvfp4_scale_bytes(rows, K))


def ig4_nvfp4_pack_scales(sf_rows, sf_packed, stream=None):
    """Row-major UE4M3 scales [rows, K/16] (uint8 or float8_e4m3fn) -> packed order."""
    rows, k16 = sf_rows.shape
    _check(_lib.ig4_nvfp4_pack_scales(rows, 16 * k16, _ptr(sf_rows), _ptr(sf_packed),
                                      _stream(stream)), "ig4_nvfp4_pack_scales")


def ig4_nvfp4_linear(a_codes, a_sf, a_scale, w_codes, w_sf, w_scale, bias, out, stream=None):
    """out = a_scale[:, None] * w_scale[None] * (A W^T) (+ bias); codes [rows, K/2] uint8."""
    M, K = a_codes.shape[0], 2 * a_codes.shape[1]
    N = w_codes.shape[0]
    _check(_lib.ig4_nvfp4_linear(M, N, K, _ptr(a_codes), _ptr(a_sf), _ptr(a_scale), _ptr(w_codes),
                                 _ptr(w_sf), _ptr(w_scale), _ptr(bias), _ptr(out),
                                 dtype_code(out), _stream(stream)), "ig4_nvfp4_linear")


def ig4_nvfp4_quantize(x, codes, sf_packed, row_scale, stream=None):
    """bf16 activations x [M, K] -> NVFP4 codes [M, K/2] uint8, packed block
    scales (ig4_nvfp4_scale_bytes(M, K) bytes) and fp32 row scales [M]."""
    M, K = x.shape
    _check(_lib.ig4_nvfp4_quantize(M, K, _ptr(x), _ptr(codes), _ptr(sf_packed), _ptr(row_scale),
                                   _stream(stream)), "ig4_nvfp4_quantize")


def ig4_text_cond_workspace_size(M: int, K_raw: int, w_dtype: str = "bf16") -> int:
    return int(_lib.ig4_text_cond_workspace_size(M, K_raw, _NAME_CODE[w_dtype]))


def ig4_text_cond_project(raw, g_norm, eps: float, w_proj, w_scale, b_proj, text_out, workspace,
                          stream=None):
    """text_out = RMSNorm(raw) * g_norm @ w_proj^T + b_proj (raw fp32 [M, K_raw])."""
    K_raw = raw.shape[-1]
    M = raw.numel() // K_raw
    D = w_proj.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_text_cond_project(M, K_raw, D, _ptr(raw), _ptr(g_norm), eps, _ptr(w_proj),
                                      _ptr(w_scale), dtype_code(w_proj), _ptr(b_proj),
                                      _ptr(text_out), _ptr(workspace), ws_bytes,
                                      _stream(stream)), "ig4_text_cond_project")


def ig4_flow_schedule(num_steps: int, mu_base: float, std: float, height_px: int,
                      width_px: int) -> list:
    """The num_steps + 1 sampler times t_0 = 1 > ... > t_N = 0 (host)."""
    out = (ctypes.c_double * (num_steps + 1))() if num_steps >= 0 else None
    _check(_lib.ig4_flow_schedule(num_steps, mu_base, std, height_px, width_px, out),
           "ig4_flow_schedule")
    return list(out)


def ig4_guidance_schedule(num_steps: int, n_polish: int, gw_main: float = 7.0,
                          gw_polish: float = 3.0) -> list:
    """Guidance weight of each step (host)."""
    out = (_f * max(1, num_steps))()
    _check(_lib.ig4_guidance_schedule(num_steps, n_polish, gw_main, gw_polish, out),
           "ig4_guidance_schedule")
    return list(out)[:num_steps]


def ig4_cfg_euler(v_cond, v_uncond, gw: float, dt: float, z_in, z_out=None, z16_out=None,
                  stream=None):
    _check(_lib.ig4_cfg_euler(z_in.numel(), _ptr(v_cond), _ptr(v_uncond), gw, dt, _ptr(z_in),
                              _ptr(z_out), _ptr(z16_out), _stream(stream)), "ig4_cfg_euler")


def ig4_denoise_workspace_size(cfg: Config, latent_ch: int = 128) -> int:
    return int(_lib.ig4_denoise_workspace_size(ctypes.byref(cfg), latent_ch))


def ig4_denoise_step(cfg: Config, cond: StackWeights, uncond: StackWeights, z, text, pos_cond,
                     pos_uncond, temb_cond, temb_uncond, t_cur: float, t_next: float, gw: float,
                     workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_denoise_step(ctypes.byref(cfg), ctypes.byref(cond), ctypes.byref(uncond),
                                 _ptr(z), _ptr(text), _ptr(pos_cond), _ptr(pos_uncond),
                                 _ptr(temb_cond), _ptr(temb_uncond), t_cur, t_next, gw,
                                 _ptr(workspace), ws_bytes, _stream(stream)), "ig4_denoise_step")


def ig4_last_device_error(stream=None) -> int:
    """Status of the device error word (synchronises the stream); does not raise."""
    return _lib.ig4_last_device_error(_stream(stream))


def ig4_selftest_timeout(wait_us: int, stream=None):
    _check(_lib.ig4_selftest_timeout(wait_us, _stream(stream)), "ig4_selftest_timeout")


def ig4_sm_clock_mhz(window_us: int = 20, stream=None) -> float:
    """SM clock (MHz) read by a kernel queued on the stream (synchronises it)."""
    v = ctypes.c_double(0.0)
    _check(_lib.ig4_sm_clock_mhz(window_us, _stream(stream), ctypes.byref(v)), "ig4_sm_clock_mhz")
    return v.value


# ------------------------------------------------------- multi-GPU layouts

def ig4_tp_workspace_size(cfg: Config, tp_size: int) -> int:
    return int(_lib.ig4_tp_workspace_size(ctypes.byref(cfg), tp_size))


def ig4_block_tp_attention(cfg: Config, tp_rank: int, tp_size: int, w: BlockWeights, x_in, pos,
                           temb, partial, workspace, stream=None):
    """partial (fp32 [B*L, D]) = [rank 0] x + gate_msa * (o_r W_o,r^T) of this head shard."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_block_tp_attention(ctypes.byref(cfg), tp_rank, tp_size, ctypes.byref(w),
                                       _ptr(x_in), _ptr(pos), _ptr(temb), _ptr(partial),
                                       _ptr(workspace), ws_bytes, _stream(stream)),
           "ig4_block_tp_attention")


def ig4_block_tp_mlp(cfg: Config, tp_rank: int, tp_size: int, w: BlockWeights, x1, partial,
                     workspace, stream=None):
    """partial = [rank 0] x1 + gate_mlp * (u_r W_down,r^T) of this FFN shard."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_block_tp_mlp(ctypes.byref(cfg), tp_rank, tp_size, ctypes.byref(w), _ptr(x1),
                                 _ptr(partial), _ptr(workspace), ws_bytes, _stream(stream)),
           "ig4_block_tp_mlp")


def ig4_tp_reduce(srcs: list, out, stream=None):
    """out = sum of the fp32 tensors in srcs (device-accessible), in list order."""
    arr = (_vp * len(srcs))(*[t.data_ptr() for t in srcs])
    _check(_lib.ig4_tp_reduce(out.numel(), len(srcs), arr, _ptr(out), dtype_code(out),
                              _stream(stream)), "ig4_tp_reduce")


def ig4_sp_image_range(cfg: Config, sp_size: int, sp_rank: int) -> tuple:
    off, cnt = _i(), _i()
    _check(_lib.ig4_sp_image_range(ctypes.byref(cfg), sp_size, sp_rank, ctypes.byref(off),
                                   ctypes.byref(cnt)), "ig4_sp_image_range")
    return off.value, cnt.value


def ig4_sp_positions(cfg: Config, sp_size: int, sp_rank: int, device=None, stream=None):
    """int32 [3, T + N_r] positions of rank sp_rank's local tokens."""
    _, cnt = ig4_sp_image_range(cfg, sp_size, sp_rank)
    out = torch.empty((3, cfg.T_text + cnt), dtype=torch.int32,
                      device=device if device is not None else "cpu")
    on_dev = 1 if out.is_cuda else 0
    _check(_lib.ig4_sp_positions(ctypes.byref(cfg), sp_size, sp_rank, _ptr(out), on_dev,
                                 _stream(stream) if on_dev else None), "ig4_sp_positions")
    return out


def ig4_sp_workspace_size(cfg: Config, sp_size: int, sp_rank: int) -> int:
    return int(_lib.ig4_sp_workspace_size(ctypes.byref(cfg), sp_size, sp_rank))


def ig4_sp_exchange_bytes(cfg: Config, sp_size: int, phase: int, src_rank: int,
                          dst_rank: int) -> int:
    return int(_lib.ig4_sp_exchange_bytes(ctypes.byref(cfg), sp_size, phase, src_rank, dst_rank))


def ig4_block_sp_pre(cfg: Config, sp_rank: int, sp_size: int, w: BlockWeights, x_local,
                     pos_local, temb, send, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_block_sp_pre(ctypes.byref(cfg), sp_rank, sp_size, ctypes.byref(w),
                                 _ptr(x_local), _ptr(pos_local), _ptr(temb), _ptr(send),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "ig4_block_sp_pre")


def ig4_block_sp_attention(cfg: Config, sp_rank: int, sp_size: int, recv, send_o, workspace,
                           stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_block_sp_attention(ctypes.byref(cfg), sp_rank, sp_size, _ptr(recv),
                                       _ptr(send_o), _ptr(workspace), ws_bytes, _stream(stream)),
           "ig4_block_sp_attention")


def ig4_block_sp_post(cfg: Config, sp_rank: int, sp_size: int, w: BlockWeights, x_local,
                      x_out_local, recv_o, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.ig4_block_sp_post(ctypes.byref(cfg), sp_rank, sp_size, ctypes.byref(w),
                                  _ptr(x_local), _ptr(x_out_local), _ptr(recv_o), _ptr(workspace),
                                  ws_bytes, _stream(stream)), "ig4_block_sp_post")
