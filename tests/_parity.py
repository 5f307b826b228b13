"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI binding, read
its intermediates back from the workspace, and compare with the CPU oracle on the same seeded
inputs (the oracle evaluated on the GPU's validated block mask, so that rows whose Top-K is
ambiguous within the margin compare like with like)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import inputs

OUT_TOL = 2e-3          # max |out_gpu - out_oracle|, fp32 output
MARGIN = orc.AMBIGUOUS_MARGIN

# Linear branch tolerance, per element: the GPU rounds four operands to bf16 on the way to
# O_l (phi(k), H_j, G_i, phi(q); relative 2^-9 each), and every term of the numerator and of
# the denominator is positive in phi, so to first order
#   |O_l,gpu - O_l| <= 4 * 2^-9 * (A + |O_l|),  A = the linear branch of |V| (same weights),
# plus the fp32 sums (about 2^-12 relative over a few thousand terms) and an absolute floor.
# With V ~ N(0, 1) (the benchmark workloads) O_l is a few 1e-3 and the plain output gate
# OUT_TOL covers it; inputs whose O_l is of order one add this bound to the output gate.
LIN_REL = 4 * 2.0 ** -9 + 2.0 ** -12
LIN_ABS = 1e-6

# The two parts of the last compare_head result (output, sparse-branch output), for messages.
LAST_ERRS = {}


def _ws_slice(ws: torch.Tensor, off: int, count: int, dtype: torch.dtype) -> torch.Tensor:
    nbytes = count * torch.empty((), dtype=dtype).element_size()
    return ws[off: off + nbytes].view(dtype)


def gpu_run(q, k, v, ratio, out_dtype=torch.float32, extras=True, device="cuda:0",
            quant=True, pv_fp8=True):
    """Forward on the GPU. Returns a dict of CPU tensors: out, kept [BH,nb,k], mask words,
    scores, sparse (sparse-branch output) and the raw workspace tensor (on the device)."""
    dev = torch.device(device)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    B, H, N, D = q.shape
    lay = sba.sagesla_get_workspace_layout(B, H, N, D, ratio, quant=quant, pv_fp8=pv_fp8)
    ws = sba.alloc_workspace(lay["total_bytes"], dev)
    nb, kk, W = lay["nb"], lay["k"], lay["mask_words"]
    res = {"layout": lay, "ws": ws}
    kw = {}
    if extras:
        kw = dict(kept_idx_out=torch.empty(B * H * nb * kk, dtype=torch.int32, device=dev),
                  mask_out=torch.empty(B * H * nb * W, dtype=torch.int32, device=dev),
                  scores_out=torch.empty(B * H * nb * nb, dtype=torch.float32, device=dev),
                  sparse_out=torch.empty(B * H * N * D, dtype=torch.float32, device=dev))
    out = sba.sagesla_forward(qd, kd, vd, ratio, out_dtype=out_dtype, workspace=ws,
                              quant=quant, pv_fp8=pv_fp8, **kw)
    status = sba.sagesla_stream_status(None, ws)
    assert status == 0, sba.sagesla_status_string(status)
    res["out"] = out.float().cpu()
    if extras:
        res["kept"] = kw["kept_idx_out"].view(B * H, nb, kk).cpu().numpy()
        res["mask"] = kw["mask_out"].view(B * H, nb, W).cpu().numpy().view(np.uint32)
        res["scores"] = kw["scores_out"].view(B * H, nb, nb).cpu().numpy()
        res["sparse"] = kw["sparse_out"].view(B, H, N, D).cpu()
    return res


def workspace_codes(res, bh: int):
    """Quantization intermediates of head bh from the workspace (CPU numpy)."""
    lay, ws = res["layout"], res["ws"]
    n_pad, nb = lay["n_pad"], lay["nb"]
    nbq = n_pad // 64
    q8 = _ws_slice(ws, lay["q8"] + bh * n_pad * 128, n_pad * 128, torch.int8).view(n_pad, 128)
    k8 = _ws_slice(ws, lay["k8"] + bh * n_pad * 128, n_pad * 128, torch.int8).view(n_pad, 128)
    v8 = _ws_slice(ws, lay["v8"] + bh * n_pad * 128, n_pad * 128, torch.uint8).view(n_pad, 128)
    sq = _ws_slice(ws, lay["sq"] + bh * nbq * 4, nbq, torch.float32)
    sk = _ws_slice(ws, lay["sk"] + bh * nbq * 4, nbq, torch.float32)
    s_v = _ws_slice(ws, lay["s_v"] + bh * 128 * 4, 128, torch.float32)
    mu = _ws_slice(ws, lay["mu"] + bh * 128 * 4, 128, torch.float32)
    res_np = {n: t.cpu().numpy() for n, t in
              dict(q8=q8, k8=k8, v8=v8, sq=sq, sk=sk, s_v=s_v, mu=mu).items()}
    # K8 rows are stored key-interleaved inside each 64-key block: key r at row 2(r%32)+r//32
    r = np.arange(64)
    perm = 2 * (r % 32) + r // 32
    k8s = res_np["k8"].reshape(-1, 64, 128)
    res_np["k8"] = k8s[:, perm, :].reshape(-1, 128)
    return res_np


def kept_sets_from_mask(mask_words: np.ndarray, nb: int) -> list:
    bits = np.unpackbits(mask_words.view(np.uint8).reshape(mask_words.shape[0], -1),
                         axis=1, bitorder="little")[:, :nb]
    return [np.flatnonzero(bits[i]) for i in range(mask_words.shape[0])]


def check_mask(prep, gpu_kept: list) -> int:
    """Bit-exact on rows whose oracle margin exceeds 1e-4; elsewhere the GPU set must be a
    valid Top-K within the margin. Returns the number of ambiguous rows."""
    ambiguous = 0
    for i in range(prep.nb):
        g = np.asarray(gpu_kept[i])
        assert g.size == prep.k, (i, g.size, prep.k)
        if prep.margin[i] > MARGIN:
            assert np.array_equal(g, prep.selected[i]), (i, g, prep.selected[i], prep.margin[i])
            continue
        ambiguous += 1
        s = prep.scores[i]
        tol = MARGIN * np.max(np.abs(s))
        desc = np.sort(s)[::-1]
        skth = desc[prep.k - 1]
        snext = desc[prep.k] if prep.k < prep.nb else -np.inf
        excluded = np.setdiff1d(np.arange(prep.nb), g)
        assert np.all(s[g] >= skth - tol), i
        assert excluded.size == 0 or np.all(s[excluded] <= snext + tol), i
    return ambiguous


def compare_head(q, k, v, ratio, res, b: int, h: int, rows=None, check_codes=True,
                 linear_tol=False, quant=True, pv_fp8=True):
    """Oracle vs GPU for one head: codes (bit-exact), mask, and the output of the query blocks
    in ``rows`` (default all). Returns (max abs error, ambiguous rows): the largest amount by
    which an element exceeds its allowance (ambiguous P codes and the row-sum window; with
    ``linear_tol`` also the linear branch's bf16 bound) before the OUT_TOL gate."""
    B, H, N, D = q.shape
    bh = b * H + h
    qh, kh, vh = (inputs.as_float64(x[b, h]) for x in (q, k, v))
    nb = res["layout"]["nb"]
    gpu_kept = [res["kept"][bh, i] for i in range(nb)]
    prep, out = orc.forward_head(qh, kh, vh, ratio, rows=rows, kept_override=gpu_kept,
                                 quant=quant, pv_fp8=pv_fp8)
    check_codes = check_codes and quant      # quant off: the oracle forms no codes
    ambiguous = check_mask(prep, gpu_kept)
    # the mask words and the kept lists agree
    assert all(np.array_equal(a, bb) for a, bb in
               zip(kept_sets_from_mask(res["mask"][bh], nb), gpu_kept))
    if check_codes:
        wc = workspace_codes(res, bh)
        np.testing.assert_array_equal(wc["mu"], prep.mu.astype(np.float32))
        np.testing.assert_array_equal(wc["s_v"], prep.s_v)
        np.testing.assert_array_equal(wc["sq"][:nb], prep.sq)
        np.testing.assert_array_equal(wc["sk"][:nb], prep.sk)
        np.testing.assert_array_equal(wc["q8"][:N], prep.q8)
        np.testing.assert_array_equal(wc["k8"][:N], prep.k8)
        np.testing.assert_array_equal(wc["v8"][:N], orc.e4m3_code(prep.v8))
        assert not wc["q8"][N:].any() and not wc["k8"][N:].any() and not wc["v8"][N:].any()
    # err: max over elements of |gpu - oracle| minus the bound of what ambiguous P codes
    # (values within the exp2 approximation error of an e4m3 midpoint) could change
    LAST_ERRS.clear()
    h_abs = orc.key_block_states(kh, np.abs(vh)) if linear_tol else None
    err = 0.0
    for i, r in out.items():
        sl = orc.block_rows(i, N)
        g = res["out"][b, h, sl].double().numpy()
        assert np.isfinite(g).all(), f"non-finite output in block {i}"
        allow = r["o_s_ambig"]
        if linear_tol:
            mag = orc.linear_block_row(prep, i, qh, h_abs)
            allow = allow + LIN_REL * (mag + np.abs(r["o_l"])) + LIN_ABS
        e_out = float(np.max(np.abs(g - r["o"]) - allow))
        LAST_ERRS["out"] = max(LAST_ERRS.get("out", -np.inf), e_out)
        err = max(err, e_out)
        if "sparse" in res:
            gs = res["sparse"][b, h, sl].double().numpy()
            assert np.isfinite(gs).all(), f"non-finite sparse-branch output in block {i}"
            e_sp = float(np.max(np.abs(gs - r["o_s"]) - r["o_s_ambig"]))
            LAST_ERRS["sparse"] = max(LAST_ERRS.get("sparse", -np.inf), e_sp)
            err = max(err, e_sp)
    return err, ambiguous
