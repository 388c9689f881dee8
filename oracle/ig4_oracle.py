"""fp64 CPU oracle of one Ideogram 4 single-stream DiT block and of the stack.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never
imports, links or runs anything under ``oracle/``, and this module imports
nothing from the product.

What it computes is the plain definition of the block, in float64 numpy,
written step by step in the order the source describes it.  The source is the
Ideogram 4.0 technical survey page ("Ideogram 4.0", section "模型架构"):
  * the DiT backbone: 34 single-stream layers, one self-attention over the
    joint sequence [text tokens | image latent tokens];
  * inside one Ideogram4TransformerBlock: self-attention with QK-RMSNorm and
    3D multimodal RoPE (text: 1D position broadcast to the 3 axes; image:
    (t, h, w) coordinates), mrope_section = (24, 20, 20), rope_theta = 5e6;
    a SwiGLU MLP with a SiLU gate; AdaLN from the timestep embedding giving
    per-block shift/scale/gate that modulate the attention and MLP paths;
  * the "Model spec" table: emb_dim 4608, 18 heads, intermediate 12288,
    adaln_dim 512, latent channels 32 x 2^2 = 128.
The release precision (FP8 E4M3 weights) comes from the SimpleTuner quickstart
page ("Ideogram 4 快速开始", section "硬件和精度").

Readings the pages leave open (each fixed here, listed with reasons in the
design notes): 6-way AdaLN (shift, scale, gate) x (attn, mlp) with a bias;
(1 + scale) on the normed input and a plain (no tanh) gate; weightless RMSNorm
with eps 1e-6 before attention and MLP; per-head QK-RMSNorm over head_dim with
learned weights g_q, g_k shared across heads; norm before rotary; the 64
frequency pairs rotate the first 128 dims of each head as rotate-half pairs
(j, j+64); contiguous frequency sections t:[0,24) h:[24,44) w:[44,64);
inv_freq[j] = theta^(-2j/128); image token (t, i, j) sits at position
(T+t, T+i, T+j) after T text tokens; attention scale 1/sqrt(head_dim), no mask;
no biases on QKV / out / gate / up / down; SwiGLU = silu(W_g h) * (W_u h).

Every function here is pinned by tests in ``tests/test_oracle_*.py`` against
closed forms, invariants and brute force.
"""

from __future__ import annotations

import numpy as np

# Ideogram 4.0 survey page, "Model spec" table.
ROPE_THETA = 5.0e6
MROPE_SECTION = (24, 20, 20)
ROTARY_DIM = 2 * sum(MROPE_SECTION)  # 128: 64 frequency pairs
EPS = 1e-6


# ---------------------------------------------------------------------------
# elementwise helpers
# ---------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) (the SwiGLU gate and the AdaLN input)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def rms_norm(x: np.ndarray, eps: float = EPS, weight: np.ndarray | None = None) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) [* weight].

    Used weightless as the pre-norm of the attention and MLP paths (AdaLN
    supplies the affine part) and with a learned weight as the per-head
    QK-RMSNorm (survey page, "单 block 内部": "QK-RMSNorm").
    """
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x * r
    if weight is not None:
        y = y * np.asarray(weight, dtype=np.float64)
    return y


# ---------------------------------------------------------------------------
# 3D multimodal RoPE
# ---------------------------------------------------------------------------

def mrope_positions(T_text: int, grid_t: int, grid_h: int, grid_w: int) -> np.ndarray:
    """Integer (t, h, w) position of every token of [text | image], shape [3, L].

    Survey page, "单 block 内部" and "条件注入方式": text tokens come first and
    use a 1D position broadcast to the 3 axes, so text token l sits at
    (l, l, l); image latent tokens use (temporal, height, width) coordinates.
    Reading: the image grid is laid out row-major over (t, i, j) and every
    image coordinate is offset by the text length T, so image token (t, i, j)
    sits at (T + t, T + i, T + j).
    """
    if min(T_text, grid_t, grid_h, grid_w) < 0:
        raise ValueError("negative size")
    n_img = grid_t * grid_h * grid_w
    L = T_text + n_img
    pos = np.zeros((3, L), dtype=np.int64)
    for l in range(T_text):
        pos[0, l] = l
        pos[1, l] = l
        pos[2, l] = l
    n = T_text
    for t in range(grid_t):
        for i in range(grid_h):
            for j in range(grid_w):
                pos[0, n] = T_text + t
                pos[1, n] = T_text + i
                pos[2, n] = T_text + j
                n += 1
    return pos


def rope_inv_freq(theta: float = ROPE_THETA, rotary_dim: int = ROTARY_DIM) -> np.ndarray:
    """inv_freq[j] = theta^(-2j / rotary_dim), j = 0 .. rotary_dim/2 - 1."""
    j = np.arange(rotary_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * j / float(rotary_dim))


def mrope_axis_of_pair(sections=MROPE_SECTION) -> np.ndarray:
    """Axis (0 = t, 1 = h, 2 = w) that drives each frequency pair.

    mrope_section = (24, 20, 20) splits the 64 pairs into contiguous chunks:
    pairs [0,24) follow t, [24,44) follow h, [44,64) follow w.
    """
    axis = []
    for a, n in enumerate(sections):
        axis.extend([a] * int(n))
    return np.asarray(axis, dtype=np.int64)


def mrope_angles(pos: np.ndarray, theta: float = ROPE_THETA, sections=MROPE_SECTION) -> np.ndarray:
    """Rotation angle of every (token, pair): ang[l, j] = pos[axis(j), l] * inv_freq[j]."""
    pos = np.asarray(pos)
    n_pairs = int(sum(sections))
    inv_freq = rope_inv_freq(theta, 2 * n_pairs)
    axis = mrope_axis_of_pair(sections)
    L = pos.shape[1]
    ang = np.zeros((L, n_pairs), dtype=np.float64)
    for j in range(n_pairs):
        ang[:, j] = pos[axis[j], :].astype(np.float64) * inv_freq[j]
    return ang


def apply_mrope(x: np.ndarray, pos: np.ndarray, theta: float = ROPE_THETA,
                sections=MROPE_SECTION) -> np.ndarray:
    """Rotate the first 2*sum(sections) dims of each head vector.

    x has shape [..., L, head_dim] (token axis second to last).  Pair j joins
    dims j and j + 64 of the rotary slice (rotate-half layout):
        a' = a cos - b sin,   b' = b cos + a sin.
    Dims from 128 to head_dim pass through unchanged.
    """
    x = np.asarray(x, dtype=np.float64)
    n_pairs = int(sum(sections))
    ang = mrope_angles(pos, theta, sections)  # [L, n_pairs]
    c = np.cos(ang)
    s = np.sin(ang)
    out = x.copy()
    a = x[..., :, 0:n_pairs]
    b = x[..., :, n_pairs:2 * n_pairs]
    out[..., :, 0:n_pairs] = a * c - b * s
    out[..., :, n_pairs:2 * n_pairs] = b * c + a * s
    return out


# ---------------------------------------------------------------------------
# AdaLN, attention, MLP
# ---------------------------------------------------------------------------

ADALN_CHUNKS = ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp")


def adaln_modulation(temb: np.ndarray, w_ada: np.ndarray, b_ada: np.ndarray, n_chunks: int = 6):
    """AdaLN projection of the timestep embedding.

    Survey page, "单 block 内部": AdaLN turns the flow-matching timestep
    embedding (adaln_dim 512) into per-block modulation of the attention and
    MLP residual paths.  Reading: mod = SiLU(temb) W_ada^T + b_ada, split into
    n_chunks vectors of width D in the order of ADALN_CHUNKS (6 for a block,
    (shift, scale) for the final layer).  Returns a list of [B, D] arrays.
    """
    c = silu(temb)
    mod = c @ np.asarray(w_ada, dtype=np.float64).T + np.asarray(b_ada, dtype=np.float64)
    D = mod.shape[-1] // n_chunks
    return [mod[:, i * D:(i + 1) * D] for i in range(n_chunks)]


def modulate(x: np.ndarray, shift: np.ndarray, scale: np.ndarray, eps: float = EPS) -> np.ndarray:
    """Pre-norm + modulation: RMSNorm(x) * (1 + scale) + shift, per sample.

    x is [B, L, D]; shift and scale are [B, D] and apply to every token of the
    sample, text and image alike.
    """
    return rms_norm(x, eps) * (1.0 + scale[:, None, :]) + shift[:, None, :]


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    """exp(s - max) / sum over `axis`."""
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def joint_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Full bidirectional attention over the joint [text | image] sequence.

    q, k, v: [B, H, L, dh].  o = softmax(q k^T / sqrt(dh)) v, no mask (the
    survey page: one self-attention over the single sequence, no separate
    text / image branches).  Returns [B, H, L, dh].
    """
    dh = q.shape[-1]
    s = np.matmul(q, np.swapaxes(k, -1, -2)) / np.sqrt(float(dh))
    p = softmax(s, axis=-1)
    return np.matmul(p, v)


def split_heads(t: np.ndarray, H: int) -> np.ndarray:
    """[B, L, H*dh] -> [B, H, L, dh] (column n = head * dh + d)."""
    B, L, N = t.shape
    return t.reshape(B, L, H, N // H).transpose(0, 2, 1, 3)


def merge_heads(t: np.ndarray) -> np.ndarray:
    """[B, H, L, dh] -> [B, L, H*dh]."""
    B, H, L, dh = t.shape
    return t.transpose(0, 2, 1, 3).reshape(B, L, H * dh)


def swiglu(h: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray) -> np.ndarray:
    """SwiGLU hidden state u = silu(h W_g^T) * (h W_u^T) (survey page: SwiGLU, SiLU gate)."""
    return silu(h @ w_gate.T) * (h @ w_up.T)


# ---------------------------------------------------------------------------
# FP8 E4M3 weights
# ---------------------------------------------------------------------------

def e4m3_decode_table() -> np.ndarray:
    """Value of each of the 256 FP8 E4M3 ("fn") codes, float64.

    Sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0
    is subnormal: (m / 8) * 2^-6.  There is no infinity; S.1111.111 is NaN, so
    the largest finite magnitude is 1.75 * 2^8 = 448.
    """
    table = np.zeros(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if (code >> 7) & 1 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            table[code] = np.nan
        elif e == 0:
            table[code] = sign * (m / 8.0) * 2.0 ** (-6)
        else:
            table[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return table


_E4M3 = None


def dequant_e4m3(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """W[n, k] = decode(q[n, k]) * scale[n] (per-output-channel fp32 scale)."""
    global _E4M3
    if _E4M3 is None:
        _E4M3 = e4m3_decode_table()
    q = np.asarray(q, dtype=np.uint8)
    return _E4M3[q] * np.asarray(scale, dtype=np.float64)[:, None]


# ---------------------------------------------------------------------------
# the block
# ---------------------------------------------------------------------------

BLOCK_WEIGHT_NAMES = ("w_ada", "b_ada", "w_qkv", "g_q", "g_k", "w_o", "w_gate", "w_up", "w_down")


def block_forward(x, temb, pos, W, H, theta=ROPE_THETA, sections=MROPE_SECTION, eps=EPS,
                  return_intermediates=False, ffn_nvfp4=False):
    """One Ideogram4TransformerBlock forward, float64.

    x: [B, L, D] residual stream ([text | image] tokens); temb: [B, adaln_dim];
    pos: [3, L] integer MRoPE positions; W: dict of float64 weights
      w_ada [6D, A], b_ada [6D], w_qkv [3D, D], g_q [dh], g_k [dh],
      w_o [D, D], w_gate [I, D], w_up [I, D], w_down [D, I]   ([out, in]).
    Steps, in the order of the survey page's block description:
      1 AdaLN: (shift, scale, gate) for attention and for the MLP;
      2 h = RMSNorm(x) (1 + scale_msa) + shift_msa;
      3 q, k, v = split(h W_qkv^T) into heads of dh = D / H;
      4 per-head QK-RMSNorm with g_q, g_k;
      5 3D MRoPE on q and k;
      6 o = softmax(q k^T / sqrt(dh)) v over all L tokens;
      7 x1 = x + gate_msa * (o W_o^T);
      8 h2 = RMSNorm(x1) (1 + scale_mlp) + shift_mlp;
        y = x1 + gate_mlp * (silu(h2 W_g^T) * (h2 W_u^T)) W_d^T.
    ffn_nvfp4: the FFN linears consume NVFP4 activations, as the NVFP4-mixed
    checkpoint runs them (deployment article, section "2.2 NVFP4 Mixed":
    FFN linears in NVFP4, attention projections and the time embedding in
    FP8): h2 and u are replaced by nvfp4_activation_values of themselves;
    the weights in W are the dequantised ones.
    """
    x = np.asarray(x, dtype=np.float64)
    B, L, D = x.shape
    dh = D // H
    shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp, gate_mlp = adaln_modulation(
        temb, W["w_ada"], W["b_ada"], 6)

    h = modulate(x, shift_msa, scale_msa, eps)
    qkv = h @ W["w_qkv"].T
    q = split_heads(qkv[:, :, 0:D], H)
    k = split_heads(qkv[:, :, D:2 * D], H)
    v = split_heads(qkv[:, :, 2 * D:3 * D], H)
    q = rms_norm(q, eps, W["g_q"])
    k = rms_norm(k, eps, W["g_k"])
    q = apply_mrope(q, pos, theta, sections)
    k = apply_mrope(k, pos, theta, sections)
    o = merge_heads(joint_attention(q, k, v))
    x1 = x + gate_msa[:, None, :] * (o @ W["w_o"].T)

    h2 = modulate(x1, shift_mlp, scale_mlp, eps)
    u = swiglu(nvfp4_activation_values(h2) if ffn_nvfp4 else h2, W["w_gate"], W["w_up"])
    y = x1 + gate_mlp[:, None, :] * ((nvfp4_activation_values(u) if ffn_nvfp4 else u) @ W["w_down"].T)
    if not return_intermediates:
        return y
    mod = np.concatenate([shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp, gate_mlp], axis=1)
    return y, dict(mod=mod, h=h, q=q, k=k, v=v, o=o, x1=x1, h2=h2, u=u)


def block_forward_rows(x, temb, pos, W, H, rows, theta=ROPE_THETA, sections=MROPE_SECTION,
                       eps=EPS, ffn_nvfp4=False):
    """The same block, evaluated only for the output tokens in `rows`.

    rows: integer array of flat token indices into B*L.  Every step except
    attention acts on one token at a time, and attention needs k and v of all
    tokens of the sample but q only of the selected token, so this evaluates
    exactly the rows of block_forward's result at a fraction of its cost
    (used for outputs sampled from full-size problems).  Returns [len(rows), D].
    """
    x = np.asarray(x, dtype=np.float64)
    B, L, D = x.shape
    dh = D // H
    rows = np.asarray(rows, dtype=np.int64)
    shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp, gate_mlp = adaln_modulation(
        temb, W["w_ada"], W["b_ada"], 6)
    w_q = W["w_qkv"][0:D]
    w_k = W["w_qkv"][D:2 * D]
    w_v = W["w_qkv"][2 * D:3 * D]
    out = np.zeros((len(rows), D), dtype=np.float64)
    for b in np.unique(rows // L):
        sel = rows[rows // L == b]
        ls = sel % L
        h = modulate(x[b:b + 1], shift_msa[b:b + 1], scale_msa[b:b + 1], eps)[0]  # [L, D]
        k = split_heads((h @ w_k.T)[None], H)  # [1, H, L, dh]
        v = split_heads((h @ w_v.T)[None], H)
        q = split_heads((h[ls] @ w_q.T)[None], H)  # [1, H, n, dh]
        k = apply_mrope(rms_norm(k, eps, W["g_k"]), pos, theta, sections)
        q = apply_mrope(rms_norm(q, eps, W["g_q"]), pos[:, ls], theta, sections)
        s = np.matmul(q, np.swapaxes(k, -1, -2)) / np.sqrt(float(dh))
        o = merge_heads(np.matmul(softmax(s, axis=-1), v))[0]  # [n, D]
        x1 = x[b, ls] + gate_msa[b][None, :] * (o @ W["w_o"].T)
        h2 = rms_norm(x1, eps) * (1.0 + scale_mlp[b][None, :]) + shift_mlp[b][None, :]
        if ffn_nvfp4:
            u = swiglu(nvfp4_activation_values(h2), W["w_gate"], W["w_up"])
            y = x1 + gate_mlp[b][None, :] * (nvfp4_activation_values(u) @ W["w_down"].T)
        else:
            y = x1 + gate_mlp[b][None, :] * (swiglu(h2, W["w_gate"], W["w_up"]) @ W["w_down"].T)
        for n, r in enumerate(sel):
            out[np.nonzero(rows == r)[0]] = y[n]
    return out


# ---------------------------------------------------------------------------
# the stack (one denoiser step)
# ---------------------------------------------------------------------------

def stack_forward(x_latent, text, temb, pos, block_weights, n_blocks, w_in, b_in, w_f, b_f,
                  w_out, b_out, H, theta=ROPE_THETA, sections=MROPE_SECTION, eps=EPS,
                  ffn_nvfp4=False, stream_bf16=False):
    """34-block DiT forward of one denoiser step, float64.

    Survey page: the DiT is 34 single-stream layers over [text | image]; image
    latents carry 128 channels (32 VAE channels x 2x2 patch) and a 1024 px image
    is a 64 x 64 token grid; text enters as a prefix of the sequence.
    Readings: the latent enters through a linear 128 -> D with bias; the text
    prefix arrives already projected to width D; after the last block a
    weightless RMSNorm with a 2-way AdaLN (shift, scale) from the same timestep
    embedding, then a linear D -> 128 with bias on the image tokens only.

    x_latent: [B, N, C]; text: [B, T, D]; block_weights: callable i -> dict as
    for block_forward (weights are built one block at a time, so they need not
    all be held at once).  ffn_nvfp4: every block's FFN takes NVFP4
    activations (see block_forward).  stream_bf16: the sequence [text | image]
    is rounded to bf16 where it is stored, after the in-projection and after
    every block (the storage precision of a bf16 residual stream; NVFP4's
    rounding decisions in the next block depend on it).  Returns [B, N, C].
    """
    T = np.asarray(text).shape[1]
    store = bf16_round if stream_bf16 else (lambda a: a)
    s = store(stack_input(x_latent, text, w_in, b_in))
    for i in range(n_blocks):
        s = store(block_forward(s, temb, pos, block_weights(i), H, theta, sections, eps,
                                ffn_nvfp4=ffn_nvfp4))
    return final_layer(s, temb, T, w_f, b_f, w_out, b_out, eps)


def stack_input(x_latent, text, w_in, b_in) -> np.ndarray:
    """The sequence entering the first block: [text | x_latent W_in^T + b_in].

    x_latent [B, N, C] (C = 128 latent channels), text [B, T, D] (already at
    the transformer's width) -> [B, T + N, D], text tokens first (survey page,
    "条件注入方式": the text tokens form the prefix of the one sequence).
    """
    x_latent = np.asarray(x_latent, dtype=np.float64)
    text = np.asarray(text, dtype=np.float64)
    img = x_latent @ np.asarray(w_in, dtype=np.float64).T + np.asarray(b_in, dtype=np.float64)
    return np.concatenate([text, img], axis=1)


def final_layer(s, temb, T, w_f, b_f, w_out, b_out, eps=EPS) -> np.ndarray:
    """After the last block: weightless RMSNorm with a 2-way AdaLN (shift,
    scale) from the timestep embedding, then the linear D -> C with bias on the
    image tokens (the T text tokens are dropped).  s [B, L, D] -> [B, L - T, C]."""
    s = np.asarray(s, dtype=np.float64)
    shift_f, scale_f = adaln_modulation(temb, w_f, b_f, 2)
    s_f = modulate(s, shift_f, scale_f, eps)
    return s_f[:, T:, :] @ np.asarray(w_out, dtype=np.float64).T + np.asarray(b_out, dtype=np.float64)


def e2m1_decode_table() -> np.ndarray:
    """Value of each of the 16 FP4 E2M1 codes, float64.

    E2M1 (the float4_e2m1fn format the SGLang / ComfyUI NVFP4 weights use):
    bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa; exponent 0 is
    subnormal (value = mantissa * 0.5); no infinities or NaNs.
    """
    out = np.empty(16, dtype=np.float64)
    for code in range(16):
        sign = -1.0 if code & 8 else 1.0
        e = (code >> 1) & 3
        m = code & 1
        mag = m * 0.5 if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
        out[code] = sign * mag
    return out


def dequant_nvfp4(packed, sf, s) -> np.ndarray:
    """NVFP4 weight -> float64: W[n, k] = s[n] * decode_e4m3(sf[n, k // 16]) *
    decode_e2m1(code[n, k]), code[n, 2i] in the low nibble of packed[n, i].

    Source: "不用再充会员！Ideogram 4.0 NF4 免费本地部署" (the ComfyUI / ROCm
    deployment article), section "2.2 NVFP4 Mixed": 4-bit floating-point
    weights sharing an FP8 E4M3 scale per block of 64 (the page calls the
    element format E2M3, which does not fit in 4 bits; the float4_e2m1fn type
    it names elsewhere is E2M1, used here), FFN linears in NVFP4 and the
    attention projections kept in FP8.  Stored here per 16-element sub-block,
    the block the tensor cores apply, each 64-block's scale repeated; plus a
    per-output-channel fp32 scale (reading: without it the block scales of
    N(0, 1/4608) weights fall into E4M3's subnormal range).
    """
    packed = np.asarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    codes = np.empty((N, 2 * packed.shape[1]), dtype=np.uint8)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    vals = e2m1_decode_table()[codes]
    sbv = e4m3_decode_table()[np.asarray(sf, dtype=np.uint8)]
    return np.asarray(s, dtype=np.float64)[:, None] * np.repeat(sbv, 16, axis=1) * vals


def bf16_round(x) -> np.ndarray:
    """Nearest bfloat16 value of each element (round to nearest, ties to an
    even last mantissa bit), returned as float64.  bfloat16 is float32 with
    the low 16 significand bits dropped; float64 inputs go through float32
    first (the precision the block's activations are computed in)."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    bits = f.view(np.uint32).astype(np.uint64)
    low = bits & 0xFFFF
    keep = bits >> 16
    up = (low > 0x8000) | ((low == 0x8000) & ((keep & 1) == 1))
    out = ((keep + up.astype(np.uint64)) << 16).astype(np.uint32)
    return out.view(np.float32).astype(np.float64)


def _nearest_code(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the value of the ascending `grid` nearest to each a >= 0,
    ties to the even index, saturating at the last entry."""
    a = np.minimum(a, grid[-1])
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    tie_pick = np.where(lo % 2 == 0, lo, hi)
    return np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, tie_pick))


def e4m3_encode(v) -> np.ndarray:
    """FP8 E4M3 code of each value: round to nearest (ties to the even code),
    saturating at +-448; sign bit set for negative values."""
    v = np.asarray(v, dtype=np.float64)
    grid = e4m3_decode_table()[:127]           # codes 0x00..0x7E, ascending
    code = _nearest_code(np.abs(v), grid).astype(np.uint8)
    return code | ((v < 0).astype(np.uint8) << 7)


def e2m1_encode(v) -> np.ndarray:
    """FP4 E2M1 code (0..15) of each value: nearest of {0, .5, 1, 1.5, 2, 3,
    4, 6}, ties to the even code, saturating at +-6; sign bit (bit 3) set for
    negative values that do not round to zero."""
    v = np.asarray(v, dtype=np.float64)
    grid = e2m1_decode_table()[:8]
    code = _nearest_code(np.abs(v), grid).astype(np.uint8)
    return code | (((v < 0) & (code > 0)).astype(np.uint8) << 3)


NVFP4_BLOCK = 16           # elements per block scale (the tensor cores' block)
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def quantize_nvfp4_activations(x):
    """Activation rows -> NVFP4: (codes uint8 [M, K] in 0..15, block-scale
    E4M3 codes uint8 [M, K/16], row scales float32 [M]).

    The recipe (the weights' NVFP4 layout of the deployment article, section
    "2.2 NVFP4 Mixed", applied to the activations the FFN linears consume,
    with 16-element blocks):
      s[m]      = amax_k |x[m, k]| / (6 * 448), or 1 for an all-zero row;
      sc[m, b]  = RNE_E4M3(amax over block b of |x[m, :]| / (6 * s[m]));
      code[m,k] = RNE_E2M1(x[m, k] * (1 / (s[m] * sc[m, k / 16]))), or 0 where
                  that product is 0.
    Every step is a float32 operation (the precision the quantising kernel
    takes the same decisions in): each product and quotient is rounded to
    float32 before the next step.
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    assert K % NVFP4_BLOCK == 0
    ax = np.abs(x)
    amax = ax.max(axis=1)
    s = np.where(amax > 0, amax / np.float32(E2M1_MAX * E4M3_MAX), np.float32(1)).astype(np.float32)
    bam = ax.reshape(M, K // NVFP4_BLOCK, NVFP4_BLOCK).max(axis=2)
    t = (np.float32(E2M1_MAX) * s).astype(np.float32)
    bs = (bam / t[:, None]).astype(np.float32)
    sc = e4m3_encode(bs)
    scv = e4m3_decode_table()[sc].astype(np.float32)
    d = (s[:, None] * scv).astype(np.float32)
    inv = np.where(d > 0, np.float32(1) / np.where(d > 0, d, np.float32(1)), np.float32(0)).astype(np.float32)
    q = (x * np.repeat(inv, NVFP4_BLOCK, axis=1)).astype(np.float32)
    return e2m1_encode(q), sc, s


MX8_BLOCK = 32            # elements per scale of the FP8 block's MX8 activations


def quantize_mx8_activations(x):
    """Activation rows -> MX8: (E4M3 codes uint8 [M, K], scale bytes uint8
    [M, K/32]) with x[m, k] ~= 2^(scale[m, k/32] - 127) * e4m3(code[m, k]).

    The FP8 block's out- and down-projections take their activations in this
    form (the release weights are FP8 E4M3, "Ideogram 4 快速开始", section on
    hardware and precision; sharing a power-of-two scale per 32 elements is
    the implementation's reading, not the pages').  Per block of 32
    consecutive elements of a row:
      amax = max |x|;
      e    = ceil(log2(float32(amax / 448))), at least -126; 0 for amax = 0;
      code = RNE_E4M3(x * 2^-e), saturating at +-448;
      scale byte = e + 127.
    The quotient amax / 448 is rounded to float32 (the precision the
    quantising kernel takes the decision in); x * 2^-e is exact.
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    assert K % MX8_BLOCK == 0
    blocks = x.reshape(M, K // MX8_BLOCK, MX8_BLOCK).astype(np.float64)
    amax = np.abs(x).reshape(M, K // MX8_BLOCK, MX8_BLOCK).max(axis=2)
    v = (amax / np.float32(E4M3_MAX)).astype(np.float32).astype(np.float64)
    e = np.zeros(amax.shape, dtype=np.int64)
    nz = v > 0
    mant, ex = np.frexp(v[nz])                 # v = mant * 2^ex, mant in [0.5, 1)
    e[nz] = np.where(mant == 0.5, ex - 1, ex)  # ceil(log2 v)
    e = np.where(amax > 0, np.maximum(e, -126), 0)
    codes = e4m3_encode(blocks * np.ldexp(1.0, -e)[..., None]).reshape(M, K)
    return codes, (e + 127).astype(np.uint8)


def mx8_values(codes, scales) -> np.ndarray:
    """float64 values of MX8 codes and scale bytes."""
    codes = np.asarray(codes, dtype=np.uint8)
    M, K = codes.shape
    vals = e4m3_decode_table()[codes].reshape(M, K // MX8_BLOCK, MX8_BLOCK)
    return (vals * np.ldexp(1.0, np.asarray(scales, dtype=np.int64) - 127)[..., None]).reshape(M, K)


def nvfp4_activation_values(x) -> np.ndarray:
    """float64 values of the NVFP4 quantisation of bf16 activations:
    s[m] * decode_E4M3(sc[m, k / 16]) * decode_E2M1(code[m, k]), taken of the
    bf16 rounding of x (the precision the block stores activations in)."""
    xb = bf16_round(x)
    shape = xb.shape
    rows = xb.reshape(-1, shape[-1])
    codes, sc, s = quantize_nvfp4_activations(rows)
    vals = e2m1_decode_table()[codes] * np.repeat(e4m3_decode_table()[sc], NVFP4_BLOCK, axis=1)
    return (s.astype(np.float64)[:, None] * vals).reshape(shape)


# ---------------------------------------------------------------------------
# text conditioning projection (the step before the stack)
# ---------------------------------------------------------------------------

TEXT_RAW_LAYERS = 13     # hidden states of 13 text-encoder layers, concatenated
TEXT_RAW_WIDTH = 4096    # per layer: 13 * 4096 = 53248 fp32 features per token


def text_cond_projection(raw, g_norm, w_proj, b_proj, eps: float = EPS) -> np.ndarray:
    """Projected text conditioning the stack consumes as its text prefix.

    "Ideogram 4 快速开始" (SimpleTuner quickstart), section "Text embed cache":
    the text encoder output concatenates the hidden states of 13 layers
    (13 * 4096 = 53248 fp32 values per token); the transformer's frozen
    llm_cond_norm and llm_cond_proj layers project these raw features to the
    conditioning tensor the transformer consumes (a bf16 cache of ~4.5 MiB for
    a 512-token caption, i.e. 4608 values per token).
    Readings: llm_cond_norm is one RMSNorm over the whole concatenated
    feature with a learned weight (eps 1e-6); llm_cond_proj is a linear layer
    53248 -> D with a bias.

    raw: [..., K_raw]; g_norm: [K_raw]; w_proj: [D, K_raw]; b_proj: [D].
    """
    h = rms_norm(np.asarray(raw, dtype=np.float64), eps, np.asarray(g_norm, dtype=np.float64))
    return h @ np.asarray(w_proj, dtype=np.float64).T + np.asarray(b_proj, dtype=np.float64)


# ---------------------------------------------------------------------------
# algorithmic work (closed forms used by the measurement code)
# ---------------------------------------------------------------------------

def block_flops(B, L, D, I, adaln_dim=512):
    """2 flops per multiply-add: GEMMs B L (8 D^2 + 6 D I), attention 4 B L^2 D, AdaLN 12 B A D."""
    gemm = B * L * (8 * D * D + 6 * D * I)
    attn = 4 * B * L * L * D
    ada = 12 * B * adaln_dim * D
    return gemm, attn, ada
