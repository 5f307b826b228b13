"""Pins of the SLA backward oracle (oracle/sla_backward_oracle.py) against things other than
its own formulas: central finite differences of the forward, float64 autograd of a torch
forward written here from the definition (masked softmax + normalized linear attention on
the complement), and torch's scaled_dot_product_attention gradients when every block is
kept. No GPU."""
import math

import numpy as np
import pytest
import torch

from oracle import sagesla_oracle as orc
from oracle import sla_backward_oracle as sbo


def _inputs(n, seed, kept_per_row=2):
    rng = np.random.default_rng(seed)
    d = 128
    q = rng.standard_normal((n, d))
    k = rng.standard_normal((n, d)) + 0.5 * rng.standard_normal(d)[None, :]
    v = rng.standard_normal((n, d))
    d_out = rng.standard_normal((n, d))
    nb = orc.n_blocks(n)
    kept = [np.sort(rng.choice(nb, size=min(kept_per_row, nb), replace=False)) for _ in range(nb)]
    return q, k, v, d_out, kept


def _torch_sla(q, k, v, kept):
    """SLA forward from its definition, for autograd (float64 tensors)."""
    n, d = q.shape
    nb = orc.n_blocks(n)
    blk = torch.arange(n) // 64
    keep = torch.zeros(nb, nb, dtype=torch.bool)
    for i in range(nb):
        keep[i, torch.as_tensor(np.asarray(kept[i], dtype=np.int64))] = True
    tok_keep = keep[blk][:, blk]                      # [query token, key token]
    s = (q @ k.T) / math.sqrt(d)
    o_s = torch.softmax(s.masked_fill(~tok_keep, float("-inf")), dim=1) @ v
    w = torch.softmax(q, dim=1) @ torch.softmax(k, dim=1).T      # phi(q_t) . phi(k_u)
    w = w * (~tok_keep)
    den = w.sum(dim=1, keepdim=True)
    o_l = torch.where(den > 0, (w @ v) / torch.where(den > 0, den, torch.ones_like(den)),
                      torch.zeros_like(den))
    return o_s + o_l


@pytest.mark.parametrize("n,seed,kept_per_row", [(200, 1, 2), (130, 2, 1), (256, 3, 3)])
def test_matches_autograd_of_the_definition(n, seed, kept_per_row):
    q, k, v, d_out, kept = _inputs(n, seed, kept_per_row)
    (dq, dk, dv), _ = sbo.sla_backward_head(q, k, v, kept, d_out)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = _torch_sla(tq, tk, tv, kept)
    np.testing.assert_allclose(out.detach().numpy(), sbo.sla_forward_head(q, k, v, kept)[0],
                               rtol=1e-11, atol=1e-12)
    out.backward(torch.tensor(d_out))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        ref = ref.numpy()
        np.testing.assert_allclose(mine, ref, rtol=1e-9, atol=1e-11 * np.abs(ref).max())


def test_central_differences():
    n = 150
    q, k, v, d_out, kept = _inputs(n, 5, 2)
    (dq, dk, dv), _ = sbo.sla_backward_head(q, k, v, kept, d_out)
    rng = np.random.default_rng(9)
    loss = lambda q_, k_, v_: float((sbo.sla_forward_head(q_, k_, v_, kept)[0] * d_out).sum())
    h = 1e-5
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        e = rng.standard_normal((n, 128))
        args = {"q": q, "k": k, "v": v}
        plus = dict(args, **{name: args[name] + h * e})
        minus = dict(args, **{name: args[name] - h * e})
        fd = (loss(plus["q"], plus["k"], plus["v"]) - loss(minus["q"], minus["k"], minus["v"])) / (2 * h)
        an = float((grad * e).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_every_block_kept_is_dense_attention():
    n = 192
    q, k, v, d_out, _ = _inputs(n, 7)
    nb = orc.n_blocks(n)
    kept = [np.arange(nb) for _ in range(nb)]
    (dq, dk, dv), _ = sbo.sla_backward_head(q, k, v, kept, d_out)
    tq, tk, tv = (torch.tensor(x[None, None], requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(torch.tensor(d_out[None, None]))
    for mine, ref in ((dq, tq.grad[0, 0]), (dk, tk.grad[0, 0]), (dv, tv.grad[0, 0])):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-9, atol=1e-12)


def test_magnitudes_bound_the_gradients():
    q, k, v, d_out, kept = _inputs(200, 11, 2)
    (dq, dk, dv), (mq, mk, mv) = sbo.sla_backward_head(q, k, v, kept, d_out)
    for g, m in ((dq, mq), (dk, mk), (dv, mv)):
        assert np.all(np.abs(g) <= m * (1 + 1e-12) + 1e-15)
        assert np.all(m > 0)


def test_query_side_projection_vanishes():
    """O_l is homogeneous of degree 0 in phi(q_t), so phi(q_t) . d phi(q_t) = 0 (Euler)."""
    n = 160
    q, k, v, d_out, kept = _inputs(n, 13, 1)
    _, st = sbo.sla_forward_head(q, k, v, kept)
    d = q.shape[1]
    for i in range(orc.n_blocks(n)):
        g = st["g"][i]
        if g is None:
            continue
        rows = orc.block_rows(i, n)
        a = orc.phi(q[rows])
        num, den = a @ g[:, :d], a @ g[:, d]
        dnum = d_out[rows] / den[:, None]
        dden = -(d_out[rows] * (num / den[:, None])).sum(axis=1) / den
        da = dnum @ g[:, :d].T + dden[:, None] * g[:, d][None, :]
        proj = (a * da).sum(axis=1)
        assert np.all(np.abs(proj) <= 1e-12 * (np.abs(a) @ np.abs(da).T).diagonal())


def test_d_is_rowsum_of_p_times_dp():
    """D = rowsum(dO * O_s) equals rowsum(P * dP) with dP = dO V^T (O_s = P V), the form the
    GPU's log-sum-exp pass accumulates; checked on the oracle's forward state, per query block
    over its kept tokens."""
    n = 200
    q, k, v, d_out, kept = _inputs(n, 17, 2)
    _, st = sbo.sla_forward_head(q, k, v, kept)
    for i in range(orc.n_blocks(n)):
        rows = orc.block_rows(i, n)
        toks = np.concatenate([np.arange(orc.block_rows(int(j), n).start,
                                         orc.block_rows(int(j), n).stop)
                               for j in sorted(int(x) for x in kept[i])])
        s = (q[rows] @ k[toks].T) / math.sqrt(q.shape[1])
        p = np.exp(s - st["lse"][rows][:, None])
        d_def = (d_out[rows] * st["o_s"][rows]).sum(axis=1)
        d_alt = (p * (d_out[rows] @ v[toks].T)).sum(axis=1)
        np.testing.assert_allclose(d_alt, d_def, rtol=1e-12, atol=1e-12 * np.abs(d_def).max())
