"""GPU parity of the SLA backward (through the C ABI) against the float64 CPU oracle
(oracle/sla_backward_oracle.py), element by element, on the GPU's own block selection (read
back from the workspace; the selection itself is checked against the oracle's Top-K by the
forward's parity tests). Tolerance: |g - ref| <= 2^-5 * magnitude + 1e-6 *
max|ref|, the magnitude being the oracle's sum of absolute terms of the element."""
import numpy as np
import pytest
import torch

import sparse_bit_attention_b200 as sba
from oracle import sagesla_oracle as orc
from oracle import sla_backward_oracle as sbo
from sparse_bit_attention_b200 import inputs

pytestmark = pytest.mark.gpu

REL = 2.0 ** -5
ABS = 1e-6


def _make(B, H, N, seed):
    q, k, v = inputs.make_random(B, H, N, seed, k_offset_std=1.0)
    g = torch.Generator().manual_seed(seed + 1000)
    d_out = torch.randn(B, H, N, 128, generator=g).to(torch.bfloat16)
    return q, k, v, d_out


def _gpu(q, k, v, d_out, ratio, grad_dtype=torch.float32):
    dev = torch.device("cuda:0")
    B, H, N, D = q.shape
    need = sba.sagesla_sla_backward_workspace_size(B, H, N, D, ratio)
    ws = sba.alloc_workspace(need, dev)
    grads = sba.sagesla_sla_backward(q.to(dev), k.to(dev), v.to(dev), d_out.to(dev), ratio,
                                     grad_dtype=grad_dtype, workspace=ws)
    st = sba.sagesla_stream_status(None, ws)
    assert st == 0, sba.sagesla_status_string(st)
    lay = sba.sagesla_get_workspace_layout(B, H, N, D, ratio)
    nb, kk = lay["nb"], lay["k"]
    kept = ws[lay["kept"]: lay["kept"] + B * H * nb * kk * 4].view(torch.int32)
    kept = kept.view(B * H, nb, kk).cpu().numpy()
    return [g.float().cpu().numpy() for g in grads], kept


def _check(q, k, v, d_out, ratio, grad_dtype=torch.float32):
    B, H, N, _ = q.shape
    (gq, gk, gv), kept = _gpu(q, k, v, d_out, ratio, grad_dtype)
    lists = [[list(kept[b * H + h, i]) for i in range(kept.shape[1])] for b in range(B)
             for h in range(H)]
    lists = [lists[b * H:(b + 1) * H] for b in range(B)]
    f64 = lambda x: inputs.as_float64(x)
    (rq, rk, rv), (mq, mk, mv) = sbo.sla_backward(f64(q), f64(k), f64(v), lists, f64(d_out))
    for name, g, r, m in (("dq", gq, rq, mq), ("dk", gk, rk, mk), ("dv", gv, rv, mv)):
        assert np.isfinite(g).all(), name
        tol = REL * m + ABS * np.abs(r).max()
        if grad_dtype == torch.bfloat16:
            tol = tol + np.abs(r) * 2.0 ** -8
        excess = np.abs(g - r) - tol
        assert excess.max() <= 0, (name, float(excess.max()), float(np.abs(g - r).max()),
                                   float(np.abs(r).max()))
    return (gq, gk, gv), kept


@pytest.mark.parametrize("B,H,N,ratio,seed", [
    (1, 2, 1024, 0.25, 1),      # whole blocks
    (1, 1, 1000, 0.1, 2),       # ragged tail block (40 tokens)
    (2, 1, 200, 0.5, 3),        # batch, 4 blocks, tail of 8
    (1, 2, 4096, 0.1, 4),       # 64 blocks, k = 7
    (1, 1, 130, 0.4, 5),        # three blocks, a 2-token tail
])
def test_backward_matches_oracle(B, H, N, ratio, seed):
    _check(*_make(B, H, N, seed), ratio)


def test_every_block_kept_is_dense_attention():
    """r = 1: no linear branch; the sparse branch is dense attention."""
    _check(*_make(1, 1, 640, 6), 1.0)


def test_single_block_sequence():
    _check(*_make(1, 2, 48, 7), 0.5)


def test_bf16_gradients_are_the_rounded_f32_gradients():
    q, k, v, d_out = _make(1, 2, 700, 8)
    (f32q, f32k, f32v), _ = _gpu(q, k, v, d_out, 0.2)
    (bq, bk, bv), _ = _gpu(q, k, v, d_out, 0.2, torch.bfloat16)
    for a, b in ((f32q, bq), (f32k, bk), (f32v, bv)):
        np.testing.assert_array_equal(torch.from_numpy(a).to(torch.bfloat16).float().numpy(), b)


def test_strided_views():
    """Non-contiguous inputs and outputs (a [B, N, H, D] storage viewed as [B, H, N, D])."""
    B, H, N = 1, 3, 300
    q, k, v, d_out = _make(B, H, N, 9)
    dev = torch.device("cuda:0")
    views = [x.transpose(1, 2).contiguous().transpose(1, 2).to(dev) for x in (q, k, v, d_out)]
    outs = [torch.empty(B, N, H, 128, device=dev).transpose(1, 2) for _ in range(3)]
    need = sba.sagesla_sla_backward_workspace_size(B, H, N, 128, 0.3)
    ws = sba.alloc_workspace(need, dev)
    sba.sagesla_sla_backward(*views, 0.3, dq=outs[0], dk=outs[1], dv=outs[2], workspace=ws)
    assert sba.sagesla_stream_status(None, ws) == 0
    (gq, gk, gv), _ = _gpu(q, k, v, d_out, 0.3)
    for a, b in zip((gq, gk, gv), outs):
        np.testing.assert_array_equal(a, b.cpu().numpy())
