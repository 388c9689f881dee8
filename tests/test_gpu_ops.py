"""Per-kernel parity through the C-ABI: each entry point against the oracle's
matching step, on the same stored inputs, at sizes that span several tiles
and a ragged tail."""

import numpy as np
import pytest
import torch

import oracle as O
from tests._util import BF16_U, f64, randn, rel_l2
from tests.gpu_common import lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _e4m3(name, shape, std):
    from synth import quantize_e4m3_per_channel
    w = randn(name, shape, std, dtype=torch.float32).numpy()
    return quantize_e4m3_per_channel(w)


def _wf64(q, s):
    return O.dequant_e4m3(q.view(torch.uint8).numpy(), s.numpy())


# ------------------------------------------------------------- positions / rope

@pytest.mark.parametrize("args", [(3, 1, 2, 3), (1, 2, 1, 2), (0, 1, 5, 7), (512, 1, 64, 64),
                                  (2048, 1, 128, 128), (2048, 1, 128, 22), (32, 1, 8, 8)])
def test_positions_device_bit_exact(ig4, args):
    pos = ig4.ig4_mrope_positions(*args, device="cuda")
    torch.cuda.synchronize()
    assert np.array_equal(pos.cpu().numpy().astype(np.int64), O.mrope_positions(*args))


@pytest.mark.parametrize("args", [(32, 1, 8, 8), (2048, 1, 128, 22), (0, 1, 3, 3)])
def test_rope_table(ig4, args):
    pos = ig4.ig4_mrope_positions(*args, device="cuda")
    L = pos.shape[1]
    c = torch.empty((L, 64), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    ig4.ig4_rope_table(pos, 5e6, (24, 20, 20), c, s)
    torch.cuda.synchronize()
    ang = O.mrope_angles(O.mrope_positions(*args))
    ref_c = np.cos(ang).astype(np.float32)
    ref_s = np.sin(ang).astype(np.float32)
    # fp64 angles and sincos rounded once to fp32: at most one fp32 ulp apart
    assert np.max(np.abs(c.cpu().numpy() - ref_c)) <= 1.2e-7
    assert np.max(np.abs(s.cpu().numpy() - ref_s)) <= 1.2e-7
    # position 0 of a text token turns nothing (the uninitialised-table regression)
    if args[0] > 0:
        assert np.all(c.cpu().numpy()[0] == 1.0) and np.all(s.cpu().numpy()[0] == 0.0)


# ------------------------------------------------------------------ AdaLN

@pytest.mark.parametrize("wdt", ["bf16", "e4m3"])
def test_adaln(ig4, wdt):
    B, A, N = 2, 512, 6 * 1024
    temb = randn("temb", (B, A), dtype=torch.float32)
    bias = randn("b_ada", (N,), 0.1, dtype=torch.float32)
    if wdt == "bf16":
        w = randn("w_ada", (N, A), 0.02)
        s = None
        wf = f64(w)
    else:
        w, s = _e4m3("w_ada", (N, A), 0.02)
        wf = _wf64(w, s)
    mod = torch.empty((B, N), dtype=torch.float32, device="cuda")
    ig4.ig4_adaln_modulation(temb.cuda(), w.cuda(), None if s is None else s.cuda(),
                             bias.cuda(), mod)
    torch.cuda.synchronize()
    ref = np.concatenate(O.adaln_modulation(f64(temb), wf, f64(bias), 6), axis=1)
    assert rel_l2(mod.cpu().numpy(), ref) <= 2e-6


# ----------------------------------------------------------- norm + modulate

@pytest.mark.parametrize("xdt,D,out", [("f32", 1024, "bf16"), ("bf16", 4608, "bf16"),
                                        ("bf16", 4608, "e4m3"), ("bf16", 512, "bf16")])
def test_norm_modulate(ig4, xdt, D, out):
    B, L = 2, 37
    xt = torch.float32 if xdt == "f32" else torch.bfloat16
    x = randn("x", (B, L, D), dtype=xt) * 3.0
    mod = randn("mod", (B, 6 * D), 0.3, dtype=torch.float32)
    shift, scale = mod[:, 3 * D:4 * D], mod[:, 4 * D:5 * D]
    md = mod.cuda()
    if out == "bf16":
        h = torch.empty((B * L, D), dtype=torch.bfloat16, device="cuda")
        hs = None
    else:
        h = torch.empty((B * L, D), dtype=torch.float8_e4m3fn, device="cuda")
        hs = torch.empty((B * L,), dtype=torch.float32, device="cuda")
    ig4.ig4_norm_modulate(B, L, D, x.cuda(), md[:, 3 * D:], md[:, 4 * D:], 6 * D, 1e-6, h, hs)
    torch.cuda.synchronize()
    ref = O.modulate(f64(x), f64(shift), f64(scale)).reshape(B * L, D)
    if out == "bf16":
        got = f64(h.cpu())
        err = np.abs(got - ref)
        assert np.all(err <= BF16_U * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref ** 2)))
    else:
        got = O.dequant_e4m3(h.cpu().view(torch.uint8).numpy(), hs.cpu().numpy())
        amax = np.abs(ref).max(axis=1)
        assert np.allclose(hs.cpu().numpy(), amax / 448.0, rtol=1e-5)
        err = np.abs(got - ref)
        assert np.all(err <= 2.0 ** -4 * np.abs(ref) + (amax / 448.0)[:, None] * 2.0 ** -9 + 1e-6)


@pytest.mark.parametrize("M,K", [(5, 12288), (130, 4608), (3, 128)])
def test_quantize_rows(ig4, M, K):
    x = randn("xq", (M, K)) * 2.0
    x[1 % M] = 0.0
    q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    ig4.ig4_quantize_rows(M, K, x.cuda(), q, s)
    torch.cuda.synchronize()
    xf = f64(x)
    amax = np.abs(xf).max(axis=1)
    exp_s = np.where(amax > 0, amax / 448.0, 1.0)
    assert np.allclose(s.cpu().numpy(), exp_s, rtol=1e-6)
    got = O.dequant_e4m3(q.cpu().view(torch.uint8).numpy(), s.cpu().numpy())
    assert np.all(np.abs(got - xf) <= 2.0 ** -4 * np.abs(xf) + exp_s[:, None] * 2.0 ** -9 + 1e-7)
    assert np.all(got[1 % M] == 0.0)


# -------------------------------------------------------------- GEMM + residual

@pytest.mark.parametrize("B,L,N,K,xdt,wdt", [
    (1, 96, 256, 64, "f32", "bf16"),        # one tile, one k-block, ragged M
    (2, 150, 512, 1024, "f32", "bf16"),     # ragged tail across the batch boundary
    (1, 1000, 768, 4608, "bf16", "bf16"),   # many tiles, long K
    (2, 150, 512, 1024, "f32", "e4m3"),
    (1, 300, 1024, 2816, "bf16", "e4m3"),
    (1, 200, 384, 512, "f32", "bf16"),      # 128-wide single-CTA tiles
    (1, 200, 640, 512, "f32", "bf16"),      # 128-wide tiles
    (1, 4608, 4608, 256, "f32", "bf16"),    # the block's out-projection shape (240-wide pair
                                            # tiles, the last of 20 column tiles 48 wide)
    (1, 4608, 4608, 512, "f32", "e4m3"),    # the same with E4M3 operands
    (2, 2304, 4608, 128, "bf16", "bf16"),   # 240-wide tiles, batch boundary, bf16 stream
    (1, 1100, 4608, 256, "bf16", "bf16"),   # 192-wide pair tiles, ragged last pair tile
    (1, 1152, 4608, 256, "f32", "e4m3"),    # 192-wide pair tiles, E4M3 (512px shape)
    (1, 4864, 4608, 512, "bf16", "bf16"),   # 256-wide pair tiles (2048x352 shape)
    (2, 100, 384, 512, "f32", "e4m3"),      # E4M3, batch boundary inside a tile
])
def test_gated_residual_linear(ig4, B, L, N, K, xdt, wdt):
    M = B * L
    xt = torch.float32 if xdt == "f32" else torch.bfloat16
    x = randn("xr", (M, N), dtype=xt)
    gate = randn("gate", (B, 3 * N), 0.5, dtype=torch.float32)
    if wdt == "bf16":
        a = randn("a", (M, K))
        w = randn("w", (N, K), 1.0 / np.sqrt(K))
        a_s = w_s = None
        af, wf = f64(a), f64(w)
    else:
        a, a_s = _e4m3("a", (M, K), 1.0)
        w, w_s = _e4m3("w", (N, K), 1.0 / np.sqrt(K))
        af, wf = _wf64(a, a_s), _wf64(w, w_s)
    out = torch.empty_like(x, device="cuda")
    g = gate.cuda()
    ig4.ig4_gated_residual_linear(B, L, N, K, a.cuda(), None if a_s is None else a_s.cuda(),
                                  w.cuda(), None if w_s is None else w_s.cuda(), g[:, N:],
                                  3 * N, x.cuda(), out)
    torch.cuda.synchronize()
    bidx = np.arange(M) // L
    upd = f64(gate)[bidx, N:2 * N] * (af @ wf.T)
    ref = f64(x) + upd
    got = f64(out.cpu())
    if xdt == "f32":
        # fp32 accumulation of exact bf16 / E4M3 products, fp32 output
        assert rel_l2(got - f64(x), upd) <= 2e-5
    else:
        err = np.abs(got - ref)
        assert np.all(err <= BF16_U * np.abs(ref) + 1e-4 * np.sqrt(np.mean(upd ** 2)))


def test_gated_residual_in_place(ig4):
    B, L, N, K = 1, 200, 256, 256
    x = randn("xi", (B * L, N), dtype=torch.float32).cuda()
    x0 = x.clone()
    a = randn("ai", (B * L, K)).cuda()
    w = randn("wi", (N, K), 1.0 / 16).cuda()
    gate = torch.ones((B, N), dtype=torch.float32, device="cuda")
    ig4.ig4_gated_residual_linear(B, L, N, K, a, None, w, None, gate, N, x, x)
    torch.cuda.synchronize()
    ref = f64(x0.cpu()) + f64(a.cpu()) @ f64(w.cpu()).T
    assert rel_l2(f64(x.cpu()), ref) <= 1e-5


# ---------------------------------------------------------------------- SwiGLU

@pytest.mark.parametrize("M,I,K,wdt", [(96, 128, 64, "bf16"), (300, 768, 1024, "bf16"),
                                       (1000, 2816, 1024, "bf16"), (300, 768, 1024, "e4m3")])
def test_swiglu(ig4, M, I, K, wdt):
    if wdt == "bf16":
        h = randn("h", (M, K))
        wg = randn("wg", (I, K), 1.0 / np.sqrt(K))
        wu = randn("wu", (I, K), 1.0 / np.sqrt(K))
        hs = sg = su = None
        hf, wgf, wuf = f64(h), f64(wg), f64(wu)
    else:
        h, hs = _e4m3("h", (M, K), 1.0)
        wg, sg = _e4m3("wg", (I, K), 1.0 / np.sqrt(K))
        wu, su = _e4m3("wu", (I, K), 1.0 / np.sqrt(K))
        hf, wgf, wuf = _wf64(h, hs), _wf64(wg, sg), _wf64(wu, su)
    u = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    cu = (lambda t: None if t is None else t.cuda())
    ig4.ig4_swiglu(M, I, K, h.cuda(), cu(hs), wg.cuda(), wu.cuda(), cu(sg), cu(su), u)
    torch.cuda.synchronize()
    ref = O.swiglu(hf, wgf, wuf)
    got = f64(u.cpu())
    err = np.abs(got - ref)
    assert np.all(err <= BF16_U * np.abs(ref) + 2e-3 * np.sqrt(np.mean(ref ** 2)))


# ------------------------------------------------------ QKV + QK-norm + MRoPE

@pytest.mark.parametrize("B,T,gh,gw,H,wdt", [(1, 32, 8, 8, 4, "bf16"), (2, 5, 7, 9, 2, "bf16"),
                                             (1, 40, 10, 10, 2, "e4m3")])
def test_qkv_project(ig4, B, T, gh, gw, H, wdt):
    D = 256 * H
    L = T + gh * gw
    M = B * L
    pos = ig4.ig4_mrope_positions(T, 1, gh, gw, device="cuda")
    cs = torch.empty((L, 64), dtype=torch.float32, device="cuda")
    sn = torch.empty_like(cs)
    ig4.ig4_rope_table(pos, 5e6, (24, 20, 20), cs, sn)
    g_q = 1.0 + randn("gq", (256,), 0.2, dtype=torch.float32)
    g_k = 1.0 + randn("gk", (256,), 0.2, dtype=torch.float32)
    if wdt == "bf16":
        h = randn("hq", (M, D))
        w = randn("wqkv", (3 * D, D), 1.0 / np.sqrt(D))
        hs = ws = None
        hf, wf = f64(h), f64(w)
    else:
        h, hs = _e4m3("hq", (M, D), 1.0)
        w, ws = _e4m3("wqkv", (3 * D, D), 1.0 / np.sqrt(D))
        hf, wf = _wf64(h, hs), _wf64(w, ws)
    vt_ld = (L + 7) // 8 * 8
    q = torch.empty((B, H, L, 256), dtype=torch.bfloat16, device="cuda")
    k = torch.empty_like(q)
    vt = torch.zeros((B, H, 256, vt_ld), dtype=torch.bfloat16, device="cuda")
    cu = (lambda t: None if t is None else t.cuda())
    ig4.ig4_qkv_project(B, L, D, H, h.cuda(), cu(hs), w.cuda(), cu(ws), g_q.cuda(), g_k.cuda(),
                        1e-6, cs, sn, q, k, vt, vt_ld)
    torch.cuda.synchronize()
    qkv = (hf @ wf.T).reshape(B, L, 3 * D)
    pos_np = O.mrope_positions(T, 1, gh, gw)
    q_ref = O.apply_mrope(O.rms_norm(O.split_heads(qkv[:, :, :D], H), 1e-6, f64(g_q)), pos_np)
    k_ref = O.apply_mrope(O.rms_norm(O.split_heads(qkv[:, :, D:2 * D], H), 1e-6, f64(g_k)),
                          pos_np)
    v_ref = O.split_heads(qkv[:, :, 2 * D:], H)
    for got, ref in ((f64(q.cpu()), q_ref), (f64(k.cpu()), k_ref),
                     (f64(vt.cpu())[..., :L].transpose(0, 1, 3, 2), v_ref)):
        err = np.abs(got - ref)
        assert np.all(err <= BF16_U * np.abs(ref) + 1e-3 * np.sqrt(np.mean(ref ** 2)))


# ------------------------------------------------------------------ attention

@pytest.mark.parametrize("B,H,L,qscale", [(1, 1, 1, 1.0), (2, 2, 7, 1.0), (1, 2, 64, 1.0),
                                          (2, 1, 65, 1.0), (1, 2, 200, 1.0), (2, 2, 1152, 1.0),
                                          (1, 2, 1152, 6.0), (1, 1, 333, 12.0)])
def test_joint_attention(ig4, B, H, L, qscale):
    q = randn("aq", (B, H, L, 256)) * qscale
    k = randn("ak", (B, H, L, 256))
    v = randn("av", (B, H, L, 256))
    vt_ld = (L + 7) // 8 * 8
    vt = torch.zeros((B, H, 256, vt_ld), dtype=torch.bfloat16)
    vt[..., :L] = v.transpose(2, 3)
    o = torch.empty((B * L, H * 256), dtype=torch.bfloat16, device="cuda")
    ig4.ig4_joint_attention(B, H, L, q.cuda(), k.cuda(), vt.cuda(), vt_ld, o)
    torch.cuda.synchronize()
    ref = O.merge_heads(O.joint_attention(f64(q), f64(k), f64(v))).reshape(B * L, H * 256)
    got = f64(o.cpu())
    # P is rounded to bf16 before the PV product and o once on output
    assert rel_l2(got, ref) <= 1e-2
    assert np.max(np.abs(got - ref)) <= 2e-2 * np.max(np.abs(ref)) + 1e-3


# an output only 16-byte aligned takes 16-byte stores instead of 32-byte
# ones: the same values, bit for bit (with and without the workspace grid)
@pytest.mark.parametrize("B,H,L,use_ws", [(1, 3, 300, True), (1, 2, 200, False),
                                          (1, 18, 1152, True)])
def test_joint_attention_output_16_byte_aligned(ig4, B, H, L, use_ws):
    q = randn("gq", (B, H, L, 256)).cuda()
    k = randn("gk", (B, H, L, 256)).cuda()
    vt_ld = (L + 7) // 8 * 8
    vt = torch.zeros((B, H, 256, vt_ld), dtype=torch.bfloat16)
    vt[..., :L] = randn("gv", (B, H, L, 256)).transpose(2, 3)
    vt = vt.cuda()
    n = B * L * H * 256
    o = torch.empty((B * L, H * 256), dtype=torch.bfloat16, device="cuda")
    buf = torch.empty(n + 16, dtype=torch.bfloat16, device="cuda")
    o16 = buf[8:8 + n].view(B * L, H * 256)
    assert o.data_ptr() % 32 == 0 and o16.data_ptr() % 32 == 16
    if use_ws:
        ws = torch.empty(ig4.ig4_joint_attention_workspace_size(B, H, L), dtype=torch.uint8,
                         device="cuda")
        ig4.ig4_joint_attention_ws(B, H, L, q, k, vt, vt_ld, o, ws)
        ig4.ig4_joint_attention_ws(B, H, L, q, k, vt, vt_ld, o16, ws)
    else:
        ig4.ig4_joint_attention(B, H, L, q, k, vt, vt_ld, o)
        ig4.ig4_joint_attention(B, H, L, q, k, vt, vt_ld, o16)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    assert torch.equal(o, o16)


# the balanced persistent grid: more (b, h, query tile) items than SMs, so
# key-tile ranges split items between CTAs (partial O merged afterwards);
# ragged tails; a single item spread over many CTAs; one item per CTA
@pytest.mark.parametrize("B,H,L,qscale", [(1, 18, 1152, 1.0), (2, 5, 2000, 1.0),
                                          (1, 37, 640, 8.0), (1, 1, 2560, 1.0),
                                          (1, 3, 129, 1.0), (3, 2, 100, 1.0)])
def test_joint_attention_balanced_grid(ig4, B, H, L, qscale):
    q = randn("bq", (B, H, L, 256)) * qscale
    k = randn("bk", (B, H, L, 256))
    v = randn("bv", (B, H, L, 256))
    vt_ld = (L + 7) // 8 * 8
    vt = torch.zeros((B, H, 256, vt_ld), dtype=torch.bfloat16)
    vt[..., :L] = v.transpose(2, 3)
    ws = torch.empty(ig4.ig4_joint_attention_workspace_size(B, H, L), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty((B * L, H * 256), dtype=torch.bfloat16, device="cuda")
    qd, kd, vd = q.cuda(), k.cuda(), vt.cuda()
    ig4.ig4_joint_attention_ws(B, H, L, qd, kd, vd, vt_ld, o, ws)
    o2 = torch.empty_like(o)
    ig4.ig4_joint_attention_ws(B, H, L, qd, kd, vd, vt_ld, o2, ws)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    assert torch.equal(o, o2)  # the merge order is fixed
    ref = O.merge_heads(O.joint_attention(f64(q), f64(k), f64(v))).reshape(B * L, H * 256)
    got = f64(o.cpu())
    assert rel_l2(got, ref) <= 1e-2
    assert np.max(np.abs(got - ref)) <= 2e-2 * np.max(np.abs(ref)) + 1e-3
