"""Pins of the oracle's NVFP4 activation quantiser and of its NVFP4 FFN block.

* the E4M3 encoder against PyTorch's float8_e4m3fn conversion (an independent
  library routine) on every midpoint between neighbouring codes and on random
  values, and its saturation at 448;
* the E2M1 encoder on every code value, every midpoint (ties to even) and
  saturation;
* the bf16 rounding against PyTorch's float32 -> bfloat16 conversion;
* the quantiser: rows built from exactly representable values come back
  exactly; a row whose blocks differ by 2^12 in magnitude keeps the small
  block (a wrong block size would flush it); each element is the nearest
  point of its block's grid (or saturated); an all-zero row;
* the NVFP4 FFN of the block: with the MLP gate at zero the output is x1
  exactly; otherwise its FFN branch stays within NVFP4's error of the
  unquantised one and differs from it.
"""

import numpy as np
import torch

import oracle as O


def test_e4m3_encode_matches_torch_on_midpoints_and_random():
    grid = O.e4m3_decode_table()[:127]
    mids = 0.5 * (grid[1:] + grid[:-1])
    rng = np.random.default_rng(5)
    rand = np.exp(rng.uniform(np.log(1e-4), np.log(440.0), 20000))
    vals = np.concatenate([grid, mids, rand, -rand]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(vals.astype(np.float64))
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    assert list(O.e4m3_encode([448.0, 470.0, 1e6, -1e6])) == [0x7E, 0x7E, 0x7E, 0xFE]


def test_e2m1_encode_codes_midpoints_saturation():
    t = O.e2m1_decode_table()
    for code in range(16):
        if code == 8:  # -0 encodes as +0
            continue
        assert O.e2m1_encode([t[code]])[0] == code
    mags = t[:8]
    mids = 0.5 * (mags[1:] + mags[:-1])
    got = O.e2m1_encode(mids)
    # each midpoint between codes c and c + 1 goes to the even one of the two
    assert list(got) == [c if c % 2 == 0 else c + 1 for c in range(7)]
    assert list(O.e2m1_encode([6.5, 100.0, -7.0, -0.2])) == [7, 7, 15, 0]


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(50000) * np.exp(rng.uniform(-20, 20, 50000))).astype(np.float32)
    # ties: float32 values exactly half-way between bf16 neighbours
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy().astype(np.float64)
    assert np.array_equal(O.bf16_round(x), ref)


def test_quantizer_exact_on_representable_rows():
    # x = c * e2m1 values with c = 448 * 2^-5: s = 2^-5, every block holding a
    # 6 gets scale 448, so d = c and the codes are the values themselves
    t = O.e2m1_decode_table()
    rng = np.random.default_rng(7)
    c = 448.0 * 2.0 ** -5
    codes = rng.integers(0, 16, size=(4, 64))
    codes[:, ::16] = 7  # a 6 in every block
    x = (c * t[codes]).astype(np.float32)
    got_codes, sc, s = O.quantize_nvfp4_activations(x)
    assert np.all(s == np.float32(2.0 ** -5))
    assert np.all(sc == 0x7E)
    assert np.array_equal(O.e2m1_decode_table()[got_codes], t[codes])
    assert np.array_equal(O.nvfp4_activation_values(x), x.astype(np.float64))


def test_quantizer_block_size_is_16():
    x = np.zeros((1, 48), dtype=np.float32)
    x[0, :16] = np.linspace(-1000.0, 1000.0, 16)
    x[0, 16:32] = np.linspace(-0.25, 0.25, 16)      # 2^12 smaller than block 0
    x[0, 32:] = np.linspace(0.0, 3.0, 16)
    v = O.nvfp4_activation_values(x)[0]
    for b in range(3):
        blk = slice(16 * b, 16 * b + 16)
        amax = np.abs(x[0, blk]).max()
        # error of each element at most half the largest grid step (2) of its
        # block's grid, whose top value 6 sits at about amax
        assert np.max(np.abs(v[blk] - x[0, blk])) <= amax / 6.0 * 1.07 + 1e-12
        assert np.any(v[blk] != 0)


def test_quantizer_picks_nearest_grid_point():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 256)).astype(np.float32) * np.exp(rng.uniform(-3, 3, (16, 1))).astype(np.float32)
    codes, sc, s = O.quantize_nvfp4_activations(x)
    d = (s[:, None] * O.e4m3_decode_table()[sc].astype(np.float32)).astype(np.float32)
    dd = np.repeat(d, 16, axis=1).astype(np.float64)
    grid = np.concatenate([-O.e2m1_decode_table()[:8][::-1], O.e2m1_decode_table()[1:8]])
    got = O.e2m1_decode_table()[codes] * dd
    err = np.abs(got - x)
    best = np.min(np.abs(x[..., None] - grid[None, None, :] * dd[..., None]), axis=-1)
    assert np.all(err <= best + 1e-6 * np.abs(x) + 1e-30)
    # block scales never exceed 448 and the largest block of each row is near it
    assert O.e4m3_decode_table()[sc].max() <= 448.0
    assert np.all(O.e4m3_decode_table()[sc].max(axis=1) >= 416.0)


def test_quantizer_zero_row():
    codes, sc, s = O.quantize_nvfp4_activations(np.zeros((2, 32), dtype=np.float32))
    assert np.all(codes == 0) and np.all(sc == 0) and np.all(s == 1.0)


def _tiny_block(seed=3, B=1, L=24, D=256, H=1, I=256, A=16):
    rng = np.random.default_rng(seed)
    W = dict(w_ada=rng.standard_normal((6 * D, A)) * 0.02, b_ada=np.zeros(6 * D),
             w_qkv=rng.standard_normal((3 * D, D)) / np.sqrt(D), g_q=np.ones(D // H),
             g_k=np.ones(D // H), w_o=rng.standard_normal((D, D)) / np.sqrt(D),
             w_gate=rng.standard_normal((I, D)) / np.sqrt(D),
             w_up=rng.standard_normal((I, D)) / np.sqrt(D),
             w_down=rng.standard_normal((D, I)) / np.sqrt(I))
    x = rng.standard_normal((B, L, D))
    temb = rng.standard_normal((B, A))
    pos = O.mrope_positions(8, 1, 4, 4)
    return x, temb, pos, W, H


def test_nvfp4_ffn_block_zero_gate_is_x1():
    x, temb, pos, W, H = _tiny_block()
    D = x.shape[-1]
    W["b_ada"][5 * D:] = 0.0
    W["w_ada"][5 * D:] = 0.0  # gate_mlp = 0
    y, im = O.block_forward(x, temb, pos, W, H, return_intermediates=True, ffn_nvfp4=True)
    assert np.array_equal(y, im["x1"])


def test_nvfp4_ffn_block_within_quantisation_error():
    x, temb, pos, W, H = _tiny_block()
    D = x.shape[-1]
    W["b_ada"][5 * D:] = 1.0  # gate_mlp about 1: the FFN branch is visible
    y_ref, im = O.block_forward(x, temb, pos, W, H, return_intermediates=True)
    y_q = O.block_forward(x, temb, pos, W, H, ffn_nvfp4=True)
    d_ref = y_ref - im["x1"]
    d_q = y_q - im["x1"]
    e = np.linalg.norm(d_q - d_ref) / np.linalg.norm(d_ref)
    # two NVFP4 roundings (h2 and u), about 9% relative each
    assert 0.02 < e < 0.3
    rows = np.array([0, 5, 17, 23])
    y_rows = O.block_forward_rows(x, temb, pos, W, H, rows, ffn_nvfp4=True)
    assert np.allclose(y_rows, y_q.reshape(-1, D)[rows], rtol=0, atol=1e-10)


def test_nvfp4_stack_is_the_blocks_composed():
    x, temb, pos, W, H = _tiny_block()
    B, L, D = x.shape
    T = 8
    rng = np.random.default_rng(4)
    C = 16
    lat = rng.standard_normal((B, L - T, C))
    text = x[:, :T]
    w_in, b_in = rng.standard_normal((D, C)) / 4, rng.standard_normal(D) * 0.1
    w_f, b_f = rng.standard_normal((2 * D, temb.shape[1])) * 0.02, np.zeros(2 * D)
    w_out, b_out = rng.standard_normal((C, D)) / 16, np.zeros(C)
    got = O.stack_forward(lat, text, temb, pos, lambda i: W, 2, w_in, b_in, w_f, b_f, w_out,
                          b_out, H, ffn_nvfp4=True)
    s = np.concatenate([text, lat @ w_in.T + b_in], axis=1)
    for _ in range(2):
        s = O.block_forward(s, temb, pos, W, H, ffn_nvfp4=True)
    sh, sc = O.adaln_modulation(temb, w_f, b_f, 2)
    ref = O.modulate(s, sh, sc)[:, T:] @ w_out.T + b_out
    assert np.array_equal(got, ref)
    plain = O.stack_forward(lat, text, temb, pos, lambda i: W, 2, w_in, b_in, w_f, b_f, w_out,
                            b_out, H)
    assert not np.array_equal(got, plain)
    # a bf16-stored stream: rounded after the in-projection and after each block
    got16 = O.stack_forward(lat, text, temb, pos, lambda i: W, 2, w_in, b_in, w_f, b_f, w_out,
                            b_out, H, ffn_nvfp4=True, stream_bf16=True)
    s = O.bf16_round(np.concatenate([text, lat @ w_in.T + b_in], axis=1))
    for _ in range(2):
        s = O.bf16_round(O.block_forward(s, temb, pos, W, H, ffn_nvfp4=True))
    ref16 = O.modulate(s, sh, sc)[:, T:] @ w_out.T + b_out
    assert np.array_equal(got16, ref16)
    assert 0 < np.linalg.norm(got16 - got) / np.linalg.norm(got) < 0.2
