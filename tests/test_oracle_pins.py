"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test fixes one step of the block with a closed form, an invariant the
definition implies, brute force on a tiny input, a hand-written table, or an
independent library routine, chosen so that a plausible slip (a dropped term,
a swapped sign or index, a wrong chunk order, a transposed operand) fails.
"""

import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _read_positions():
    cases = []
    cur = None
    for line in open(os.path.join(GOLDEN, "mrope_positions.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == "case":
            cur = {"args": tuple(int(v) for v in parts[1:]), "rows": {}}
            cases.append(cur)
        else:
            cur["rows"][parts[0]] = [int(v) for v in parts[1:]]
    return cases


# --------------------------------------------------------------------- positions

@pytest.mark.parametrize("case", _read_positions(), ids=lambda c: "T%d_g%dx%dx%d" % c["args"])
def test_positions_match_hand_written_tables(case):
    pos = O.mrope_positions(*case["args"])
    expect = np.array([case["rows"]["t"], case["rows"]["h"], case["rows"]["w"]])
    assert pos.shape == expect.shape
    assert np.array_equal(pos, expect)


@pytest.mark.parametrize("T,gh,gw", [(512, 64, 64), (2048, 128, 22), (32, 8, 8), (0, 5, 7)])
def test_positions_bounds_and_structure(T, gh, gw):
    pos = O.mrope_positions(T, 1, gh, gw)
    L = T + gh * gw
    assert pos.shape == (3, L)
    assert np.array_equal(pos[:, :T], np.tile(np.arange(T), (3, 1)))
    img = pos[:, T:]
    assert np.all(img[0] == T)
    assert img[1].min() == T and img[1].max() == T + gh - 1
    assert img[2].min() == T and img[2].max() == T + gw - 1
    assert pos.max() == (T + max(gh, gw) - 1 if gh * gw else T - 1)
    # every grid cell appears exactly once
    cells = set(zip(img[1].tolist(), img[2].tolist()))
    assert len(cells) == gh * gw


# --------------------------------------------------------------- rotary tables

def test_inv_freq_closed_forms():
    f = O.rope_inv_freq(5e6, 128)
    assert f.shape == (64,)
    assert f[0] == 1.0
    assert f[32] == pytest.approx(1.0 / np.sqrt(5e6), rel=1e-14)
    assert f[63] == pytest.approx(5e6 ** (-63.0 / 64.0), rel=1e-14)
    ratio = f[1:] / f[:-1]
    assert np.allclose(ratio, 5e6 ** (-1.0 / 64.0), rtol=1e-13)


def test_axis_sections():
    a = O.mrope_axis_of_pair((24, 20, 20))
    assert a.shape == (64,)
    assert np.array_equal(np.bincount(a), [24, 20, 20])
    assert np.all(np.diff(a) >= 0)
    assert a[23] == 0 and a[24] == 1 and a[43] == 1 and a[44] == 2


# -------------------------------------------------------------------- rotary

def _rand_heads(L, dh=256, lead=(1, 2)):
    return RNG.standard_normal(lead + (L, dh))


def test_rope_position_zero_is_identity():
    x = _rand_heads(5)
    pos = np.zeros((3, 5), dtype=np.int64)
    assert np.array_equal(O.apply_mrope(x, pos), x)


def test_rope_preserves_pair_norms_and_passes_tail():
    x = _rand_heads(40)
    pos = O.mrope_positions(8, 1, 4, 8)
    y = O.apply_mrope(x, pos)
    n0 = x[..., :64] ** 2 + x[..., 64:128] ** 2
    n1 = y[..., :64] ** 2 + y[..., 64:128] ** 2
    assert np.allclose(n0, n1, rtol=1e-12, atol=1e-12)
    assert np.array_equal(y[..., 128:], x[..., 128:])


def test_rope_text_tokens_are_textbook_1d_rope():
    """All three axes equal l: pair j of token l turns by l * theta^(-2j/128), written
    as the complex product (a + i b) * exp(i angle) of the RoFormer definition."""
    L = 9
    x = _rand_heads(L)
    pos = O.mrope_positions(L, 1, 0, 0)
    y = O.apply_mrope(x, pos)
    j = np.arange(64)
    omega = 5e6 ** (-2.0 * j / 128.0)
    for l in range(L):
        z = (x[..., l, :64] + 1j * x[..., l, 64:128]) * np.exp(1j * l * omega)
        assert np.allclose(y[..., l, :64], z.real, atol=1e-12)
        assert np.allclose(y[..., l, 64:128], z.imag, atol=1e-12)


def test_rope_relative_position_property():
    """q.k after rotation depends only on the position difference on each axis."""
    q = RNG.standard_normal(256)
    k = RNG.standard_normal(256)
    p = np.array([[3, 7], [11, 2], [5, 9]])  # [3 axes, 2 tokens]
    for c in (0, 1, 17, 1000):
        pc = p + c
        qq = O.apply_mrope(q[None, :], pc[:, :1])[0]
        kk = O.apply_mrope(k[None, :], pc[:, 1:])[0]
        if c == 0:
            ref = qq @ kk
        assert qq @ kk == pytest.approx(ref, rel=1e-10, abs=1e-10)


def test_rope_sections_drive_the_right_pairs():
    """Moving a token along one axis only turns that axis's frequency pairs."""
    x = _rand_heads(1, lead=())
    base = np.array([[4], [4], [4]])
    sl = {0: slice(0, 24), 1: slice(24, 44), 2: slice(44, 64)}
    y0 = O.apply_mrope(x, base)
    for ax in range(3):
        p = base.copy()
        p[ax, 0] += 3
        y = O.apply_mrope(x, p)
        changed = ~np.isclose(y[0, :64], y0[0, :64], rtol=0, atol=1e-14)
        expect = np.zeros(64, bool)
        expect[sl[ax]] = True
        assert np.array_equal(changed, expect), ax


# ---------------------------------------------------------------------- norms

def test_rms_norm_unit_rms_and_weight():
    x = RNG.standard_normal((3, 7, 256)) * 5.0
    y = O.rms_norm(x, 1e-6)
    ms = np.mean(x * x, axis=-1)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)
    assert np.allclose(O.rms_norm(3.0 * x), y, rtol=1e-6)
    g = RNG.standard_normal(256)
    assert np.allclose(O.rms_norm(x, 1e-6, g), y * g, rtol=1e-14)
    assert np.all(O.rms_norm(np.zeros((2, 8))) == 0.0)


def test_silu_values():
    assert O.silu(np.array(0.0)) == 0.0
    assert O.silu(np.array(1.0)) == pytest.approx(1.0 / (1.0 + np.exp(-1.0)), rel=1e-15)
    assert O.silu(np.array(40.0)) == pytest.approx(40.0, rel=1e-15)
    assert abs(O.silu(np.array(-800.0))) < 1e-300


def test_adaln_chunk_order_and_silu_input():
    D, A, B = 8, 4, 2
    b = np.concatenate([np.full(D, i + 1.0) for i in range(6)])
    chunks = O.adaln_modulation(np.zeros((B, A)), np.ones((6 * D, A)), b, 6)
    assert len(chunks) == 6
    for i, c in enumerate(chunks):
        assert np.all(c == i + 1.0), O.ADALN_CHUNKS[i]
    temb = RNG.standard_normal((B, A))
    w = RNG.standard_normal((6 * D, A))
    ref = np.array([[sum(temb[bb, a] / (1 + np.exp(-temb[bb, a])) * w[n, a] for a in range(A))
                     for n in range(6 * D)] for bb in range(B)])
    got = np.concatenate(O.adaln_modulation(temb, w, np.zeros(6 * D), 6), axis=1)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------ attention

def test_softmax_rows_sum_to_one():
    p = O.softmax(RNG.standard_normal((4, 5, 33)) * 30.0)
    assert np.allclose(p.sum(-1), 1.0, rtol=1e-14)
    assert np.all(p >= 0)


def test_attention_brute_force_tiny():
    B, H, L, dh = 1, 2, 6, 8
    q, k, v = (RNG.standard_normal((B, H, L, dh)) for _ in range(3))
    o = O.joint_attention(q, k, v)
    for h in range(H):
        for i in range(L):
            w = [np.exp(sum(q[0, h, i, d] * k[0, h, j, d] for d in range(dh)) / np.sqrt(dh))
                 for j in range(L)]
            z = sum(w)
            for d in range(dh):
                ref = sum(w[j] * v[0, h, j, d] for j in range(L)) / z
                assert o[0, h, i, d] == pytest.approx(ref, rel=1e-12, abs=1e-12)


def test_attention_special_cases():
    q, k, v = (RNG.standard_normal((1, 1, 1, 16)) for _ in range(3))
    assert np.allclose(O.joint_attention(q, k, v), v, rtol=1e-15)
    q = RNG.standard_normal((1, 3, 7, 16))
    k = np.broadcast_to(RNG.standard_normal((1, 3, 1, 16)), (1, 3, 7, 16))
    v = RNG.standard_normal((1, 3, 7, 16))
    o = O.joint_attention(q, k, v)
    assert np.allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), rtol=1e-12)


def test_matmul_step_against_triple_loop():
    a = RNG.standard_normal((8, 16))
    w = RNG.standard_normal((8, 16))  # [out, in] like every weight here
    y = a @ w.T
    for i in range(8):
        for n in range(8):
            assert y[i, n] == pytest.approx(sum(a[i, kk] * w[n, kk] for kk in range(16)), rel=1e-13)


# ------------------------------------------------------------------------ E4M3

def test_e4m3_table_against_library_conversion():
    table = O.e4m3_decode_table()
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float32).double().numpy()
    nan = np.isnan(table)
    assert np.array_equal(nan, np.isnan(lib))
    assert np.array_equal(table[~nan], lib[~nan])
    assert np.nanmax(table) == 448.0 and nan.sum() == 2


def test_e4m3_table_hand_values():
    table = O.e4m3_decode_table()
    for line in open(os.path.join(GOLDEN, "e4m3_codes.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        got = table[int(code, 16)]
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and np.signbit(got) == val.startswith("-")


def test_e4m3_dequant_round_trip_error_bound():
    from synth import quantize_e4m3_per_channel
    w = (RNG.standard_normal((16, 64)) * np.linspace(0.01, 3.0, 16)[:, None]).astype(np.float32)
    q, s = quantize_e4m3_per_channel(w)
    wd = O.dequant_e4m3(q.view(torch.uint8).numpy(), s.numpy())
    # E4M3 keeps 3 mantissa bits: rounding error <= 2^-4 relative, or half the
    # subnormal step 2^-10 * s absolute near zero.
    err = np.abs(wd - w)
    bound = np.maximum(np.abs(w) * 2.0 ** -4, s.numpy()[:, None].astype(np.float64) * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-6))
    assert np.allclose(np.abs(wd).max(axis=1), s.numpy() * 448.0, rtol=1e-6)
