"""Pins of the oracle's MX8 activation quantiser (E4M3 codes with a UE8M0
scale per 32 elements, the form the FP8 block feeds its out- and
down-projections).

* hand-worked blocks: the scale byte of a block whose amax is 448 (2^0),
  just above 448 (2^1), 3 (2^-7) and zero (byte 127, codes 0);
* rows built from values exactly representable at their block's scale come
  back exactly;
* the scale is the smallest power of two that fits the block: the largest
  magnitude lands in (224, 448] after scaling;
* every element is the nearest point of its block's grid (RNE within
  E4M3's spacing), checked against PyTorch's float8_e4m3fn conversion of
  the scaled values (an independent library routine);
* blocks are independent: a row whose blocks differ by 2^20 in magnitude
  keeps the small block (a wrong block size or a row-wide scale would
  flush it).
"""

import numpy as np
import torch

import oracle as O


def test_hand_worked_blocks():
    x = np.zeros((4, 32), dtype=np.float32)
    x[0, 0] = 448.0
    x[1, 5] = np.nextafter(np.float32(448.0), np.float32(1e9))
    x[2, :2] = [-3.0, 2.5]
    codes, sc = O.quantize_mx8_activations(x)
    assert list(sc[:, 0]) == [127, 128, 120, 127]
    vals = O.mx8_values(codes, sc)
    assert vals[0, 0] == 448.0
    assert vals[1, 5] == 448.0                      # 448 + ulp rounds back to 448 at scale 2
    assert vals[2, 0] == -3.0 and vals[2, 1] == 2.5
    assert np.all(codes[3] == 0)


def test_representable_rows_are_exact():
    rng = np.random.default_rng(1)
    grid = O.e4m3_decode_table()[:127]
    M, K = 6, 256
    e = rng.integers(-30, 30, size=(M, K // 32))
    v = rng.choice(grid, size=(M, K)) * rng.choice([-1.0, 1.0], size=(M, K))
    v = v.reshape(M, K // 32, 32)
    v[:, :, 0] = 448.0                               # pin the block's scale to 2^e
    x = (v * np.ldexp(1.0, e)[..., None]).reshape(M, K).astype(np.float32)
    codes, sc = O.quantize_mx8_activations(x)
    assert np.array_equal(sc.astype(np.int64) - 127, e)
    assert np.array_equal(O.mx8_values(codes, sc), x.astype(np.float64))


def test_scale_is_minimal_and_elements_nearest():
    rng = np.random.default_rng(2)
    M, K = 16, 512
    mag = np.exp(rng.uniform(np.log(1e-6), np.log(1e6), size=(M, K // 32, 1)))
    x = (rng.standard_normal((M, K // 32, 32)) * mag).reshape(M, K).astype(np.float32)
    codes, sc = O.quantize_mx8_activations(x)
    e = sc.astype(np.int64) - 127
    scaled = x.reshape(M, K // 32, 32).astype(np.float64) * np.ldexp(1.0, -e)[..., None]
    top = np.abs(scaled).max(axis=2)
    assert np.all(top <= 448.0) and np.all(top > 224.0)
    ref = torch.from_numpy(scaled.reshape(M, K).astype(np.float32)).to(torch.float8_e4m3fn)
    ref = ref.view(torch.uint8).numpy()
    dec = O.e4m3_decode_table()
    assert np.array_equal(dec[codes], dec[ref])


def test_blocks_are_independent():
    x = np.ones((1, 64), dtype=np.float32)
    x[0, :32] *= 2.0 ** 20
    x[0, 40] = 0.75
    codes, sc = O.quantize_mx8_activations(x)
    vals = O.mx8_values(codes, sc)
    assert vals[0, 40] == 0.75 and vals[0, 41] == 1.0
    assert sc[0, 0] - sc[0, 1] == 20
