"""Pins of the W8A8 oracle (oracle/w8a8_oracle.py) against things other than itself: a
float64 matmul of the dequantized operands, exact integer products, the locality of the
128x128 weight-block scales and the quantizer's bound. No GPU."""
import numpy as np

from oracle import norm_oracle as no
from oracle import w8a8_oracle as wo


def test_weight_blocks_are_independent_and_bounded():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((300, 384))
    w[5, 7] = 40.0                       # a spike in block (0, 0) only
    codes, scales = wo.quantize_weight_blocks(w)
    assert scales.shape == (3, 3)
    assert scales[0, 0] == np.float32(np.float32(40.0) / np.float32(127))
    for bn in range(3):
        for bk in range(3):
            blk = w[128 * bn:min(128 * bn + 128, 300), 128 * bk:128 * bk + 128]
            a = np.float32(np.abs(blk).max())
            assert scales[bn, bk] == np.float32(a / np.float32(127))
            c = codes[128 * bn:min(128 * bn + 128, 300), 128 * bk:128 * bk + 128]
            assert np.abs(c).max() == 127
            err = np.abs(c.astype(np.float64) * np.float64(scales[bn, bk]) - blk)
            assert np.all(err <= 0.5 * scales[bn, bk] * (1 + 1e-6) + 1e-6 * a)
    # the spike leaves the other blocks of its rows and columns untouched
    assert scales[0, 1] < 1.0 and scales[1, 0] < 1.0


def test_linear_equals_dequantized_matmul():
    rng = np.random.default_rng(2)
    M, K, N = 37, 512, 200
    x8 = rng.integers(-127, 128, (M, K)).astype(np.int8)
    s_x = rng.uniform(0.001, 0.1, M).astype(np.float32)
    w8 = rng.integers(-127, 128, (N, K)).astype(np.int8)
    s_w = rng.uniform(0.001, 0.1, ((N + 127) // 128, K // 128)).astype(np.float32)
    bias = rng.standard_normal(N)
    # dequantize with the block scales expanded over their blocks, then one float matmul
    xd = x8.astype(np.float64) * s_x.astype(np.float64)[:, None]
    wd = w8.astype(np.float64) * np.repeat(np.repeat(s_w.astype(np.float64), 128, 0)[:N], 128, 1)
    ref = xd @ wd.T + bias[None, :]
    y, t = wo.w8a8_linear(x8, s_x, w8, s_w, bias)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.all(t >= np.abs(y - bias[None, :]) * (1 - 1e-12))


def test_unit_scales_give_the_exact_integer_product():
    rng = np.random.default_rng(3)
    x8 = rng.integers(-127, 128, (9, 256)).astype(np.int8)
    w8 = rng.integers(-127, 128, (130, 256)).astype(np.int8)
    y, _ = wo.w8a8_linear(x8, np.ones(9, np.float32), w8, np.ones((2, 2), np.float32))
    exact = x8.astype(np.int64) @ w8.astype(np.int64).T
    assert np.array_equal(y, exact.astype(np.float64))
    # one K block per scale: doubling the second block's scale adds exactly that block again
    s_w = np.array([[1.0, 2.0], [1.0, 2.0]], np.float32)
    y2, _ = wo.w8a8_linear(x8, np.ones(9, np.float32), w8, s_w)
    second = x8[:, 128:].astype(np.int64) @ w8[:, 128:].astype(np.int64).T
    assert np.array_equal(y2, (exact + second).astype(np.float64))


def test_quantized_layer_approximates_the_float_layer():
    rng = np.random.default_rng(4)
    M, K, N = 64, 1024, 256
    x = rng.standard_normal((M, K))
    w = rng.standard_normal((N, K)) * 0.05
    _, xb = no.norm_forward(x, no.NO_NORM, 0.0)
    x8, s_x = no.quant_rows_int8(xb)
    w8, s_w = wo.quantize_weight_blocks(w)
    y, _ = wo.w8a8_linear(x8, s_x, w8, s_w)
    ref = xb @ w.T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.02, rel          # 8-bit operands: about 1% relative error
