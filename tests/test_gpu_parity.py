"""GPU parity: the CUDA path (through the C-ABI) against the CPU oracle on the same seeded
inputs. Codes and scales bit-exact, block masks bit-exact on rows with a clear margin,
outputs within 2e-3 (max abs, fp32 output)."""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import inputs
from _parity import OUT_TOL, compare_head, gpu_run

pytestmark = pytest.mark.gpu


def _all_heads(q, k, v, ratio, res, rows=None, check_codes=True):
    B, H = q.shape[:2]
    worst, amb = 0.0, 0
    for b in range(B):
        for h in range(H):
            e, a = compare_head(q, k, v, ratio, res, b, h, rows=rows, check_codes=check_codes)
            worst, amb = max(worst, e), amb + a
    return worst, amb


@pytest.mark.parametrize("ratio", [0.1, 1.0])
def test_tiny_workload(ratio):
    q, k, v = inputs.make_qkv("tiny")
    res = gpu_run(q, k, v, ratio)
    err, amb = _all_heads(q, k, v, ratio, res)
    assert err <= OUT_TOL, err


@pytest.mark.parametrize("n,ratio,seed", [
    (1000, 0.1, 11),    # ragged last block (40 tokens)
    (1088, 0.25, 12),   # odd block count: the last pair has one block
    (1025, 0.2, 13),    # last block holds a single token
    (64, 0.1, 14),      # one block: dense, empty linear branch
    (33, 0.5, 15),      # one partial block
    (4096, 0.05, 16),   # 64 blocks, k = 4
    (2048, 0.5, 17),    # wide kept sets
])
def test_shapes_and_tails(n, ratio, seed):
    q, k, v = inputs.make_random(1, 2, n, seed, k_offset_std=1.0)
    res = gpu_run(q, k, v, ratio)
    err, _ = _all_heads(q, k, v, ratio, res)
    assert err <= OUT_TOL, err


def test_batch_heads_and_strided_views():
    """B=2, H=3 given as [B, N, H, D] storage (non-contiguous head stride)."""
    q, k, v = inputs.make_random(2, 3, 700, 21, k_offset_std=0.5)
    qs, ks, vs = (x.transpose(1, 2).contiguous().transpose(1, 2) for x in (q, k, v))
    assert not qs.is_contiguous()
    res = gpu_run(qs, ks, vs, 0.3)
    err, _ = _all_heads(q, k, v, 0.3, res)
    assert err <= OUT_TOL, err
    res2 = gpu_run(q.contiguous(), k.contiguous(), v.contiguous(), 0.3, extras=False)
    assert torch.equal(res["out"], res2["out"])


def test_bf16_output_is_rounded_fp32_output():
    q, k, v = inputs.make_random(1, 2, 1024, 22)
    a = gpu_run(q, k, v, 0.1, extras=False)
    b = gpu_run(q, k, v, 0.1, out_dtype=torch.bfloat16, extras=False)
    assert torch.equal(a["out"].to(torch.bfloat16).float(), b["out"])


def test_scores_output():
    q, k, v = inputs.make_random(1, 2, 1500, 23)
    res = gpu_run(q, k, v, 0.1)
    for h in range(2):
        qb = orc.pooled_means(inputs.as_float64(q[0, h]))
        kb = orc.pooled_means(inputs.as_float64(k[0, h]))
        ref = orc.block_scores(qb, kb)
        np.testing.assert_allclose(res["scores"][h], ref, rtol=0, atol=1e-5 * np.abs(ref).max())


def test_host_entry_point_matches_device_entry_point():
    q, k, v = inputs.make_random(1, 2, 1024, 24)
    dev = gpu_run(q, k, v, 0.1, extras=False)["out"]
    out = torch.empty(q.shape, dtype=torch.float32).pin_memory()
    sba.sagesla_forward_host(q.contiguous().pin_memory(), k.contiguous().pin_memory(),
                             v.contiguous().pin_memory(), out, 0.1)
    assert torch.equal(out, dev)


@pytest.mark.parametrize("B,H,out_dtype", [(1, 11, torch.float32), (2, 5, torch.bfloat16)])
def test_host_entry_point_chunks_heads(B, H, out_dtype):
    """The host entry point pipelines copies and forwards over chunks of heads (the last
    chunk may be short); its output equals the device entry point's."""
    q, k, v = inputs.make_random(B, H, 700, 33 + H, k_offset_std=0.5)
    dev = gpu_run(q, k, v, 0.2, out_dtype=out_dtype, extras=False)["out"]
    out = torch.empty(q.shape, dtype=out_dtype).pin_memory()
    sba.sagesla_forward_host(q.contiguous().pin_memory(), k.contiguous().pin_memory(),
                             v.contiguous().pin_memory(), out, 0.2)
    assert torch.equal(out.float(), dev)


def test_repeatable():
    q, k, v = inputs.make_random(1, 2, 2048, 25)
    a = gpu_run(q, k, v, 0.1, extras=False)["out"]
    b = gpu_run(q, k, v, 0.1, extras=False)["out"]
    assert torch.equal(a, b)


@pytest.mark.parametrize("n,seed", [(1025, 26), (4096, 27), (700, 28)])
def test_dense_mode(n, seed):
    """r = 1 keeps every key block: no selection, no linear branch, the attention kernel walks
    the blocks in order (odd block counts leave a single-block last pair)."""
    q, k, v = inputs.make_random(1, 2, n, seed, k_offset_std=1.0)
    res = gpu_run(q, k, v, 1.0)
    nb = res["layout"]["nb"]
    assert res["layout"]["k"] == nb
    assert (res["kept"] == np.arange(nb, dtype=np.int32)[None, None, :]).all()
    err, _ = _all_heads(q, k, v, 1.0, res)
    assert err <= OUT_TOL, err
    # without the optional outputs the lists are never written; the output is the same
    plain = gpu_run(q, k, v, 1.0, extras=False)
    assert torch.equal(plain["out"], res["out"])


@pytest.mark.parametrize("nb,ratio,seed", [
    (200, 0.1, 41),     # 7 chunks of 32 key blocks per lane row
    (700, 0.15, 42),    # 22 chunks
    (1000, 0.05, 43),   # 32 chunks, the bucket's full width
    (1400, 0.1, 44),    # 44 chunks
    (1900, 0.1, 45),    # 60 chunks
])
def test_selection_for_every_row_length_bucket(nb, ratio, seed):
    """Rows of each register-resident size of the warp selection: kept lists and masks against
    the oracle's Top-K, codes bit-exact, sampled query blocks against the oracle output."""
    n = nb * 64 - 17
    q, k, v = inputs.make_random(1, 1, n, seed, k_offset_std=1.0)
    res = gpu_run(q, k, v, ratio)
    assert res["layout"]["nb"] == nb
    err, _ = compare_head(q, k, v, ratio, res, 0, 0, rows=_sampled_rows(nb, seed, count=2))
    assert err <= OUT_TOL, err


@pytest.mark.parametrize("n", [4096, 700 * 64, 2050 * 64])
def test_equal_scores_keep_the_lowest_blocks(n):
    """Constant K makes every score of a row equal: the selection keeps blocks 0..k-1."""
    q, _, v = inputs.make_random(1, 1, n, 31)
    k = torch.full_like(q, 0.5)
    res = gpu_run(q, k, v, 0.05)
    nb, kk = res["layout"]["nb"], res["layout"]["k"]
    assert (res["kept"][0] == np.arange(kk, dtype=np.int32)[None, :]).all()
    err, _ = compare_head(q, k, v, 0.05, res, 0, 0, rows=_sampled_rows(nb, 31, count=2))
    assert err <= OUT_TOL, err


def test_long_rows_block_topk():
    """More than 2048 key blocks per row: the selection takes the one-CTA-per-row path."""
    q, k, v = inputs.make_random(1, 1, 2050 * 64 - 10, 29, k_offset_std=0.5)
    res = gpu_run(q, k, v, 0.02, extras=True)
    nb = res["layout"]["nb"]
    assert nb == 2050
    err, _ = compare_head(q, k, v, 0.02, res, 0, 0, rows=_sampled_rows(nb, 29, count=4))
    assert err <= OUT_TOL, err


def test_dense_mode_full_size_sampled():
    """r = 1 on the Wan2.1-1.3B-480P shape (512 kept blocks per query block), sampled rows."""
    q, k, v = inputs.make_qkv("wan21_1p3b_480p", heads=2)
    res = gpu_run(q, k, v, 1.0)
    nb = res["layout"]["nb"]
    for h in range(2):
        err, _ = compare_head(q, k, v, 1.0, res, 0, h, rows=_sampled_rows(nb, 30 + h, count=3))
        assert err <= OUT_TOL, (h, err)


def _sampled_rows(nb, seed, count=6):
    rng = np.random.default_rng(seed)
    return sorted(set([0, 1, nb - 2, nb - 1] + list(rng.integers(0, nb, count))))


@pytest.mark.parametrize("name", ["wan21_1p3b_480p", "wan21_14b_480p", "wan21_14b_720p"])
def test_full_size_workloads_sampled(name):
    """Full-size run in the benchmark's launch configuration; the oracle checks sampled
    heads and query blocks (first, last and random), codes of those heads bit-exact."""
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.make_qkv(name)
    res = gpu_run(q, k, v, w.topk_ratios[0])
    nb = res["layout"]["nb"]
    for h in sorted({0, w.H - 1}):
        err, _ = compare_head(q, k, v, w.topk_ratios[0], res, 0, h, rows=_sampled_rows(nb, h))
        assert err <= OUT_TOL, (h, err)


_LOCALITY = {}


@pytest.mark.parametrize("ratio", [0.05, 0.1, 0.15])
def test_locality_workload_sampled(ratio):
    if not _LOCALITY:
        _LOCALITY["qkv"] = inputs.make_qkv("locality_14b_720p")
    q, k, v = _LOCALITY["qkv"]
    res = gpu_run(q, k, v, ratio)
    nb = res["layout"]["nb"]
    err, _ = compare_head(q, k, v, ratio, res, 0, 7, rows=_sampled_rows(nb, 7))
    assert err <= OUT_TOL, err
