"""CPU oracle for the fused normalization + modulation + INT8 activation quantization.

TEST INFRASTRUCTURE ONLY. Only the tests and the CPU legs of ``bench.py`` may import this
module; the product path never calls it, and it shares no code with the CUDA path.

What it computes (float64, whole rows with numpy reductions as the only library steps):

* LayerNorm and RMSNorm over the channels of each token row, the AdaLN modulation
  y * (1 + scale) + shift, and the bf16 rounding of the result: news.qq.com TurboDiffusion
  article, section 第四把钥匙 (LayerNorm and RMSNorm rewritten and fused with their
  neighbours so that data crosses memory fewer times).
* The per-token INT8 quantization of the normalized row for the 8-bit linear layers: same
  article, section 第三把钥匙 (activations quantized to INT8 on the fly; weights in 128x128
  blocks). Reading: one scale per token row, with the block quantizer of the attention's
  INT8 step applied to the row.

Pins: ``tests/test_norm_oracle_pins.py`` (closed forms on small rows, torch's layer_norm /
rms_norm in float64, invariances, the quantizer's bound and exhaustive small cases).
"""
from __future__ import annotations

import numpy as np

from .sagesla_oracle import quant_int8_block, round_bf16

LAYER_NORM = 0
RMS_NORM = 1
NO_NORM = 2        # the row itself (per-token quantization of any activation row)


def normalize_rows(x, kind: int, eps: float, gamma=None, beta=None):
    """Real-valued normalization of each row of x [M, K] (float64 result, no rounding)."""
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if kind == LAYER_NORM:
        mu = x.sum(axis=-1, keepdims=True) / K
        d = x - mu
        var = (d * d).sum(axis=-1, keepdims=True) / K
        y = d / np.sqrt(var + eps)
        if gamma is not None:
            y = y * np.asarray(gamma, dtype=np.float64)
        if beta is not None:
            y = y + np.asarray(beta, dtype=np.float64)
        return y
    if kind == RMS_NORM:
        ms = (x * x).sum(axis=-1, keepdims=True) / K
        y = x / np.sqrt(ms + eps)
        if gamma is not None:
            y = y * np.asarray(gamma, dtype=np.float64)
        return y
    if kind == NO_NORM:
        return x.copy()
    raise ValueError(f"unknown normalization kind {kind}")


def modulate_rows(y, scale, shift, rows_per_sample: int):
    """AdaLN modulation: row r belongs to sample r // rows_per_sample;
    y <- y * (1 + scale[b]) + shift[b] (scale, shift [B, K])."""
    y = np.asarray(y, dtype=np.float64)
    b = np.arange(y.shape[0]) // rows_per_sample
    out = y
    if scale is not None:
        out = out * (1.0 + np.asarray(scale, dtype=np.float64)[b])
    if shift is not None:
        out = out + np.asarray(shift, dtype=np.float64)[b]
    return out


def norm_forward(x, kind: int, eps: float, gamma=None, beta=None, scale=None, shift=None,
                 rows_per_sample: int = 1):
    """The fused operation: returns (y_real float64, y_bf16 as float64 values)."""
    y = normalize_rows(x, kind, eps, gamma, beta)
    if scale is not None or shift is not None:
        y = modulate_rows(y, scale, shift, rows_per_sample)
    return y, round_bf16(y)


def quant_rows_int8(y_bf16):
    """Per-row INT8 codes and scales of bf16-valued rows (the block quantizer on each row)."""
    y = np.asarray(y_bf16, dtype=np.float64)
    codes = np.empty(y.shape, dtype=np.int8)
    scales = np.empty(y.shape[0], dtype=np.float32)
    for r in range(y.shape[0]):
        codes[r], scales[r] = quant_int8_block(y[r])
    return codes, scales
