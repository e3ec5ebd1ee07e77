"""Oracle pins: FP4 (E2M1) descriptor compression ([P5] "COBS 阅读笔记" §5.5, "量化：对存储的
特征向量做 FP4"; Algorithm 2 steps 7-8).

The page fixes the format (2 exponent bits, 1 mantissa bit, one fp32 scale per scaled
eigenvector, bf16 block mean) and the byte count (r = 4, D = 128: 1024 bf16 bytes become
272 FP4 bytes per block).  The scale rule (absmax / 6) and the rounding (nearest, ties to
the zero-mantissa value) are this build's reading.
"""
import numpy as np

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_grid_values_round_trip_exactly():
    rng = np.random.default_rng(0)
    s = np.float32(0.37)
    vals = rng.choice(np.concatenate([GRID, -GRID]), size=128)
    vals[0] = 6.0                                    # absmax fixes the scale to s
    x = (vals * s).astype(np.float32)
    codes, scale = oracle.fp4_quantize(x[None])
    assert np.float32(scale[0]) == np.float32(np.float32(6.0 * s) / np.float32(6.0))
    back = oracle.fp4_dequantize(codes, scale)[0]
    assert np.array_equal(back, vals * np.float64(scale[0]))


def test_ties_go_to_the_even_code_and_absmax_to_six():
    # scale 1 (absmax 6): the midpoints of the E2M1 grid and where they must land
    x = np.zeros(16, np.float32)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    x[0] = 6.0
    x[1:8] = mids
    x[8:15] = [-m for m in mids]
    codes, scale = oracle.fp4_quantize(x[None])
    assert scale[0] == 1.0
    back = oracle.fp4_dequantize(codes, scale)[0]
    assert back[0] == 6.0
    assert list(back[1:8]) == want
    assert list(back[8:15]) == [-w for w in want]


def test_error_is_at_most_half_the_local_grid_step():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    codes, scale = oracle.fp4_quantize(x)
    back = oracle.fp4_dequantize(codes, scale)
    a = np.abs(x / scale[:, None].astype(np.float64))
    half_step = np.where(a <= 2.0, 0.25, np.where(a <= 4.0, 0.5, 1.0))
    err = np.abs(back - x) / scale[:, None]
    assert (err <= half_step + 1e-6).all()
    # every vector's largest element is represented as +-6 * scale
    i = np.abs(x).argmax(axis=1)
    assert np.allclose(np.abs(back[np.arange(64), i]), 6.0 * scale)


def test_zero_vector_and_packing():
    x = np.zeros((2, 8), np.float32)
    x[1, 3] = -1.5
    codes, scale = oracle.fp4_quantize(x)
    assert scale[0] == 0.0 and (codes[0] == 0).all()
    assert scale[1] == np.float32(0.25)
    # element 3 = -1.5 / 0.25 = -6 -> sign bit 8 | index 7, odd element in the high nibble
    assert codes[1, 1] == (0x8 | 0x7) << 4
    assert (oracle.fp4_dequantize(codes, scale)[1] == x[1]).all()


def test_byte_accounting_matches_the_page():
    # [P5] §5.5: rank-4 factors of D = 128 take 1024 bytes in bf16 and 272 bytes in FP4
    # (4 vectors x (128 four-bit codes + one fp32 scale))
    rank, D = 4, 128
    codes, scale = oracle.fp4_quantize(np.ones((rank, D), np.float32))
    assert rank * D * 2 == 1024
    assert codes.nbytes + scale.nbytes == 272
