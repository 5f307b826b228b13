"""Pins of the fused-normalization oracle (oracle/norm_oracle.py) against things other than
itself: closed forms worked by hand, torch's float64 layer_norm / rms_norm, invariances of
the definitions, and the quantizer's error bound. No GPU."""
import math

import numpy as np
import pytest
import torch

from oracle import norm_oracle as no
from oracle import round_bf16


def test_layer_norm_closed_form():
    # x = [1, 2, 3, 4]: mean 2.5, biased variance 1.25, so y = (x - 2.5) / sqrt(1.25)
    y = no.normalize_rows(np.array([[1.0, 2.0, 3.0, 4.0]]), no.LAYER_NORM, 0.0)
    r = math.sqrt(1.25)
    np.testing.assert_allclose(y[0], [-1.5 / r, -0.5 / r, 0.5 / r, 1.5 / r], rtol=0, atol=1e-15)
    # affine: gamma scales first, beta shifts after
    y2 = no.normalize_rows(np.array([[1.0, 2.0, 3.0, 4.0]]), no.LAYER_NORM, 0.0,
                           gamma=[2, 2, 2, 2], beta=[1, 1, 1, 1])
    np.testing.assert_allclose(y2[0], [1 - 3 / r, 1 - 1 / r, 1 + 1 / r, 1 + 3 / r], atol=1e-15)


def test_rms_norm_closed_form():
    # x = [3, 4]: mean square 12.5
    y = no.normalize_rows(np.array([[3.0, 4.0]]), no.RMS_NORM, 0.0, gamma=[1.0, 0.5])
    np.testing.assert_allclose(y[0], [3 / math.sqrt(12.5), 0.5 * 4 / math.sqrt(12.5)], atol=1e-15)
    # eps enters under the root: x = [1, 1], eps = 3 -> 1 / sqrt(1 + 3) = 0.5
    y = no.normalize_rows(np.array([[1.0, 1.0]]), no.RMS_NORM, 3.0)
    np.testing.assert_allclose(y[0], [0.5, 0.5], atol=1e-15)


def test_constant_row_layer_norm_is_zero_and_eps_matters():
    y = no.normalize_rows(np.full((1, 8), 3.25), no.LAYER_NORM, 1e-6)
    assert np.all(y == 0.0)
    # x = [0, 2]: variance 1; with eps = 3, y = +-1 / 2
    y = no.normalize_rows(np.array([[0.0, 2.0]]), no.LAYER_NORM, 3.0)
    np.testing.assert_allclose(y[0], [-0.5, 0.5], atol=1e-15)


@pytest.mark.parametrize("K", [64, 1536, 5120])
def test_against_torch_float64(K):
    g = torch.Generator().manual_seed(K)
    x = torch.randn(7, K, generator=g, dtype=torch.float64) * 3 + 0.5
    gamma = torch.randn(K, generator=g, dtype=torch.float64)
    beta = torch.randn(K, generator=g, dtype=torch.float64)
    ref = torch.nn.functional.layer_norm(x, (K,), gamma, beta, eps=1e-6).numpy()
    got = no.normalize_rows(x.numpy(), no.LAYER_NORM, 1e-6, gamma.numpy(), beta.numpy())
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    ref = torch.nn.functional.rms_norm(x, (K,), gamma, eps=1e-6).numpy()
    got = no.normalize_rows(x.numpy(), no.RMS_NORM, 1e-6, gamma.numpy())
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_invariances():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 96))
    base = no.normalize_rows(x, no.LAYER_NORM, 0.0)
    np.testing.assert_allclose(no.normalize_rows(x + 7.0, no.LAYER_NORM, 0.0), base, atol=1e-12)
    np.testing.assert_allclose(no.normalize_rows(5.0 * x, no.LAYER_NORM, 0.0), base, atol=1e-12)
    rbase = no.normalize_rows(x, no.RMS_NORM, 0.0)
    np.testing.assert_allclose(no.normalize_rows(0.25 * x, no.RMS_NORM, 0.0), rbase, atol=1e-12)
    # unit mean and variance of a LayerNorm row
    np.testing.assert_allclose(base.mean(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose((base ** 2).mean(axis=1), 1.0, atol=1e-12)


def test_modulation_groups_rows_by_sample():
    y = np.ones((4, 3))
    scale = np.array([[0.0, 1.0, -0.5], [2.0, 0.0, 0.0]])
    shift = np.array([[0.0, 0.0, 1.0], [-1.0, 3.0, 0.0]])
    out = no.modulate_rows(y, scale, shift, rows_per_sample=2)
    np.testing.assert_array_equal(out[0], [1.0, 2.0, 1.5])
    np.testing.assert_array_equal(out[1], [1.0, 2.0, 1.5])
    np.testing.assert_array_equal(out[2], [2.0, 4.0, 1.0])
    np.testing.assert_array_equal(out[3], [2.0, 4.0, 1.0])
    # zero modulation is the identity
    np.testing.assert_array_equal(no.modulate_rows(y * 3, np.zeros((2, 3)), np.zeros((2, 3)), 2), y * 3)


def test_norm_forward_rounds_to_bf16():
    rng = np.random.default_rng(4)
    x = round_bf16(rng.standard_normal((3, 128)))
    y, yb = no.norm_forward(x, no.LAYER_NORM, 1e-6)
    np.testing.assert_array_equal(yb, round_bf16(y))
    assert np.max(np.abs(yb - y) / np.maximum(np.abs(y), 1e-30)) <= 2.0 ** -8


def test_row_quantizer_bound_and_special_cases():
    rng = np.random.default_rng(5)
    yb = round_bf16(rng.standard_normal((16, 256)) * rng.uniform(0.01, 50, (16, 1)))
    codes, scales = no.quant_rows_int8(yb)
    for r in range(16):
        a = np.max(np.abs(yb[r]))
        assert np.max(np.abs(codes[r])) == 127
        assert scales[r] == np.float32(np.float32(a) / np.float32(127))
        err = np.abs(codes[r].astype(np.float64) * np.float64(scales[r]) - yb[r])
        assert np.all(err <= 0.5 * scales[r] * (1 + 1e-6) + 1e-6 * a)
    codes, scales = no.quant_rows_int8(np.zeros((1, 8)))
    assert scales[0] == 1.0 and not codes.any()
    # ties go to even: a row with amax 127 has inv = 1, so 2.5 -> 2 and 3.5 -> 4
    codes, scales = no.quant_rows_int8(np.array([[127.0, 2.5, 3.5, -2.5]]))
    np.testing.assert_array_equal(codes[0], [127, 2, 4, -2])
