"""CPU oracle for the W8A8 linear layer (INT8 GEMM with 128x128 block-scaled weights and
per-token activation scales).

TEST INFRASTRUCTURE ONLY. Only the tests and the CPU legs of ``bench.py`` may import this
module; the product path never calls it, and it shares no code with the CUDA path.

news.qq.com TurboDiffusion article, section 第三把钥匙: weights and activations both in 8-bit
integers so that the whole linear layer runs in the integer domain on the INT8 tensor cores;
the weights are quantized block-wise with 128x128 blocks, one scale per block; the
activations are quantized dynamically. Reading: one scale per token row for the activations
(the per-token codes of the fused normalization).

What it computes: the block quantizer of the attention's INT8 step on every 128x128 weight
block, and Y = s_x[m] * sum over K blocks of s_w[n/128][kb] * (exact integer block dot
product), in float64 with int64 block products (numpy matmul on int64 is the library step).

Pins: ``tests/test_w8a8_oracle_pins.py`` (dequantized float64 matmul, exact integer cases,
block-locality of the scales, the quantizer bound).
"""
from __future__ import annotations

import numpy as np

from .sagesla_oracle import quant_int8_block

WBLOCK = 128


def quantize_weight_blocks(w):
    """W [N, K] (bf16 values as float64), K a multiple of 128 -> (codes int8 [N, K],
    scales float32 [ceil(N/128), K/128])."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % WBLOCK == 0, "K must be a multiple of 128"
    nbn, nbk = (N + WBLOCK - 1) // WBLOCK, K // WBLOCK
    codes = np.empty((N, K), dtype=np.int8)
    scales = np.empty((nbn, nbk), dtype=np.float32)
    for bn in range(nbn):
        r0, r1 = bn * WBLOCK, min((bn + 1) * WBLOCK, N)
        for bk in range(nbk):
            c0, c1 = bk * WBLOCK, (bk + 1) * WBLOCK
            codes[r0:r1, c0:c1], scales[bn, bk] = quant_int8_block(w[r0:r1, c0:c1])
    return codes, scales


def block_partials(x8, w8):
    """Exact integer partial sums S[bk][m][n] = sum over block bk of x8[m, k] * w8[n, k]."""
    x = np.asarray(x8, dtype=np.int64)
    w = np.asarray(w8, dtype=np.int64)
    K = x.shape[1]
    return np.stack([x[:, c:c + WBLOCK] @ w[:, c:c + WBLOCK].T for c in range(0, K, WBLOCK)])


def w8a8_linear(x8, s_x, w8, s_w, bias=None):
    """Y [M, N] in float64 and the term size T (for the tolerance)."""
    S = block_partials(x8, w8).astype(np.float64)           # [nbk, M, N]
    N = w8.shape[0]
    bn = np.arange(N) // WBLOCK
    sw = np.asarray(s_w, dtype=np.float64)[bn].T             # [nbk, N]
    sx = np.asarray(s_x, dtype=np.float64)[:, None]
    y = sx * np.einsum("bmn,bn->mn", S, sw)
    t = np.abs(sx) * np.einsum("bmn,bn->mn", np.abs(S), np.abs(sw))
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
        t = t + np.abs(np.asarray(bias, dtype=np.float64))[None, :]
    return y, t
