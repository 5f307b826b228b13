"""CPU oracle for the SLA backward: gradients of the unquantized sparse-linear attention.

TEST INFRASTRUCTURE ONLY. Only the tests and the CPU legs of ``bench.py`` may import this
module; the product path never calls it, and it shares no code with the CUDA path.

What it computes (float64, plain numpy): the layer fine-tuned is SLA without the
8-bit quantization (news.qq.com TurboDiffusion article, section 从训练到部署: full attention
is replaced by SLA and fine-tuned; SageSLA, SLA plus low-bit quantization, replaces it only
at inference). The block selection of the forward is held fixed. For one (b, h) with kept
lists ``kept[i]`` and the output gradient dO:

* sparse branch, per query block i over the tokens u of its kept blocks:
  L = logsumexp(s), P = exp(s - L), O_s = P V, D = rowsum(dO * O_s), dP = dO V^T,
  dS = P (dP - D), dQ = dS K / sqrt(d), dK += dS^T Q / sqrt(d), dV += P^T dO;
* linear branch, per query block i with G_i the sum of H_j over the blocks it does not keep:
  a = phi(q), num = a G_i[:, :d], den = a G_i[:, d], O_l = num / den,
  dnum = dO / den, dden = -(dO . O_l) / den, da = G_i[:, :d] dnum + G_i[:, d] dden,
  dq += a * (da - a . da) (a . da = num . dnum + den dden = 0: O_l does not change when a is
  scaled), dG_i = a^T [dnum | dden]; then dH_j = sum of dG_i over the query
  blocks that do not keep j, and per key token u of block j with b = phi(k_u):
  db = dH_j[:, :d] v_u + dH_j[:, d], dk_u += b * (db - b . db), dv_u += dH_j[:, :d]^T b.

Each gradient comes with its magnitude: the same sums with every term taken in absolute
value, which scales the tolerance of the GPU comparison (2^-5 of it, plus 1e-6 of the
largest gradient).

Pins: ``tests/test_sla_backward_oracle_pins.py`` (central finite differences of the forward,
float64 autograd of an independent torch forward, dense attention gradients from torch's
scaled_dot_product_attention when every block is kept).
"""
from __future__ import annotations

import math

import numpy as np

from .sagesla_oracle import block_rows, key_block_states, n_blocks, phi


def _kept_tokens(kept_blocks, n: int) -> np.ndarray:
    """Token indices of the given key blocks, in ascending block order."""
    return np.concatenate([np.arange(block_rows(int(j), n).start, block_rows(int(j), n).stop)
                           for j in sorted(int(x) for x in kept_blocks)])


def sla_forward_head(q, k, v, kept):
    """Unquantized SLA forward of one head with a fixed block selection.

    Returns (O [N, D], state) where state holds what the backward reuses."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    n, d = q.shape
    nb = n_blocks(n)
    scale = 1.0 / math.sqrt(d)
    h_blocks = key_block_states(k, v)                 # [nb, d, d+1]
    o_s = np.zeros((n, d))
    o_l = np.zeros((n, d))
    lse = np.zeros(n)
    g_list = [None] * nb
    for i in range(nb):
        rows = block_rows(i, n)
        toks = _kept_tokens(kept[i], n)
        s = (q[rows] @ k[toks].T) * scale
        mx = s.max(axis=1, keepdims=True)
        lse[rows] = (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True)))[:, 0]
        p = np.exp(s - lse[rows][:, None])
        o_s[rows] = p @ v[toks]
        comp = np.setdiff1d(np.arange(nb), np.asarray(kept[i], dtype=np.int64))
        if comp.size:
            g = h_blocks[comp].sum(axis=0)
            g_list[i] = g
            a = phi(q[rows])
            o_l[rows] = (a @ g[:, :d]) / (a @ g[:, d])[:, None]
    return o_s + o_l, {"o_s": o_s, "o_l": o_l, "lse": lse, "g": g_list, "h": h_blocks}


def sla_backward_head(q, k, v, kept, d_out):
    """Gradients (dq, dk, dv) of one head and their magnitudes (mq, mk, mv)."""
    q, k, v, d_out = (np.asarray(x, dtype=np.float64) for x in (q, k, v, d_out))
    n, d = q.shape
    nb = n_blocks(n)
    scale = 1.0 / math.sqrt(d)
    _, st = sla_forward_head(q, k, v, kept)
    dq, dk, dv = np.zeros((n, d)), np.zeros((n, d)), np.zeros((n, d))
    mq, mk, mv = np.zeros((n, d)), np.zeros((n, d)), np.zeros((n, d))
    # ---- sparse branch
    for i in range(nb):
        rows = block_rows(i, n)
        toks = _kept_tokens(kept[i], n)
        s = (q[rows] @ k[toks].T) * scale
        p = np.exp(s - st["lse"][rows][:, None])
        dd = (d_out[rows] * st["o_s"][rows]).sum(axis=1)
        dp = d_out[rows] @ v[toks].T
        ds = p * (dp - dd[:, None])
        dq[rows] += ds @ k[toks] * scale
        mq[rows] += np.abs(ds) @ np.abs(k[toks]) * scale
        dk[toks] += ds.T @ q[rows] * scale
        mk[toks] += np.abs(ds).T @ np.abs(q[rows]) * scale
        dv[toks] += p.T @ d_out[rows]
        mv[toks] += p.T @ np.abs(d_out[rows])
    # ---- linear branch, query side
    d_g = np.zeros((nb, d, d + 1))
    m_g = np.zeros((nb, d, d + 1))
    for i in range(nb):
        g = st["g"][i]
        if g is None:
            continue
        rows = block_rows(i, n)
        a = phi(q[rows])
        num = a @ g[:, :d]
        den = a @ g[:, d]
        o_l = num / den[:, None]
        dnum = d_out[rows] / den[:, None]
        dden = -(d_out[rows] * o_l).sum(axis=1) / den
        da = dnum @ g[:, :d].T + dden[:, None] * g[:, d][None, :]
        mda = np.abs(dnum) @ np.abs(g[:, :d]).T + np.abs(dden)[:, None] * np.abs(g[:, d])[None, :]
        dq[rows] += a * (da - (a * da).sum(axis=1, keepdims=True))
        mq[rows] += a * (mda + (a * mda).sum(axis=1, keepdims=True))
        d_g[i, :, :d] = a.T @ dnum
        d_g[i, :, d] = a.T @ dden
        m_g[i, :, :d] = a.T @ np.abs(dnum)
        m_g[i, :, d] = a.T @ np.abs(dden)
    # ---- complement transpose: dH_j = sum of dG_i over the query blocks not keeping j
    d_h = np.zeros((nb, d, d + 1))
    m_h = np.zeros((nb, d, d + 1))
    for i in range(nb):
        if st["g"][i] is None:
            continue
        comp = np.setdiff1d(np.arange(nb), np.asarray(kept[i], dtype=np.int64))
        d_h[comp] += d_g[i]
        m_h[comp] += m_g[i]
    # ---- linear branch, key side
    pk = phi(k)
    for j in range(nb):
        rows = block_rows(j, n)
        b = pk[rows]
        db = v[rows] @ d_h[j, :, :d].T + d_h[j, :, d][None, :]
        mdb = np.abs(v[rows]) @ m_h[j, :, :d].T + m_h[j, :, d][None, :]
        dk[rows] += b * (db - (b * db).sum(axis=1, keepdims=True))
        mk[rows] += b * (mdb + (b * mdb).sum(axis=1, keepdims=True))
        dv[rows] += b @ d_h[j, :, :d]
        mv[rows] += b @ m_h[j, :, :d]
    return (dq, dk, dv), (mq, mk, mv)


def sla_backward(q, k, v, kept, d_out):
    """Gradients on [B, H, N, D] arrays; ``kept[b][h][i]`` the kept key blocks of query
    block i. Returns ((dq, dk, dv), (mq, mk, mv))."""
    q = np.asarray(q, dtype=np.float64)
    bsz, heads = q.shape[:2]
    grads = [np.zeros(q.shape) for _ in range(3)]
    mags = [np.zeros(q.shape) for _ in range(3)]
    for b in range(bsz):
        for h in range(heads):
            g, m = sla_backward_head(q[b, h], k[b, h], v[b, h], kept[b][h], d_out[b, h])
            for x, y in zip(grads, g):
                x[b, h] = y
            for x, y in zip(mags, m):
                x[b, h] = y
    return tuple(grads), tuple(mags)
