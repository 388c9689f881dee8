"""Pins of the oracle's NVFP4 decoding: the 16 E2M1 codes written out by hand,
their ordering and sign symmetry, the decode of a constructed weight (codes,
block scales, channel scale chosen by hand), and a round trip of the input
generator's quantiser within E2M1's half-step."""

import os

import numpy as np
import torch

import oracle as O
from synth.block_inputs import quantize_nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_codes.txt")


def test_e2m1_codes_match_hand_table():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    table = O.e2m1_decode_table()
    assert len(rows) == 16
    for code, val in rows:
        assert table[int(code)] == float(val)
        assert np.signbit(table[int(code)]) == val.startswith("-")
    assert np.all(np.diff(table[:8]) > 0)
    assert np.array_equal(table[8:], -table[:8])


def test_dequant_constructed_weight():
    # one row, K = 32: codes 0..15 then 15..0; block scales 1.0 (0x38) and 2.0 (0x40); s = 0.5
    codes = np.concatenate([np.arange(16), np.arange(16)[::-1]]).astype(np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]
    sf = np.array([[0x38, 0x40]], dtype=np.uint8)
    s = np.array([0.5])
    got = O.dequant_nvfp4(packed, sf, s)[0]
    t = O.e2m1_decode_table()
    ref = np.concatenate([0.5 * 1.0 * t[np.arange(16)], 0.5 * 2.0 * t[np.arange(16)[::-1]]])
    assert np.array_equal(got, ref)


def test_generator_round_trip_within_half_step():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((16, 256)) / 16).astype(np.float32)
    packed, sf, s = quantize_nvfp4(w, block=64)
    deq = O.dequant_nvfp4(packed.numpy(), sf.view(torch.uint8).numpy(), s.numpy())
    # each 64-block shares one scale: its 4 sub-block scales are equal
    sfu = sf.view(torch.uint8).numpy().reshape(16, 4, 4)
    assert np.all(sfu == sfu[:, :, :1])
    # |W - deq| <= half the E2M1 step at that magnitude (largest step 2, at 4..6) times the
    # block's scale, plus the E4M3 rounding of the scale (relative 2^-4) on the block's max
    step = s.numpy()[:, None] * np.repeat(O.e4m3_decode_table()[sf.view(torch.uint8).numpy()], 16,
                                          axis=1)
    assert np.all(np.abs(w - deq) <= 1.0 * step + 1e-7)
    rel = np.linalg.norm(w - deq) / np.linalg.norm(w)
    assert 0.02 < rel < 0.15  # 4-bit: a few percent of error, not zero, not garbage
