"""GPU parity of the 16-bit operand modes of sagesla_options against the oracle:
quant = 1, pv_fp8 = 0 (INT8 Q.K^T, bf16 P times the raw V) and quant = 0, pv_fp8 = 0 (the
unquantized SLA forward). The block selection, the codes and the linear branch are those of
the default mode; the sparse branch is compared with the oracle's real-P.V loop within
2e-3 + 2^-8 times the same weights applied to |v| (P rounded to bf16)."""
import numpy as np
import pytest
import torch

import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import inputs
from _parity import LAST_ERRS, OUT_TOL, compare_head, gpu_run

pytestmark = pytest.mark.gpu

MODES = [(True, False), (False, False)]


def _all_heads(q, k, v, ratio, res, quant, pv_fp8, rows=None):
    worst = 0.0
    for h in range(q.shape[1]):
        err, _ = compare_head(q, k, v, ratio, res, 0, h, rows=rows, quant=quant, pv_fp8=pv_fp8)
        assert err <= OUT_TOL, (h, err, dict(LAST_ERRS))
        worst = max(worst, err)
    return worst


@pytest.mark.parametrize("quant,pv_fp8", MODES)
@pytest.mark.parametrize("ratio", [0.1, 1.0])
def test_tiny_workload(quant, pv_fp8, ratio):
    q, k, v = inputs.make_qkv("tiny")
    res = gpu_run(q, k, v, ratio, quant=quant, pv_fp8=pv_fp8)
    _all_heads(q, k, v, ratio, res, quant, pv_fp8)


@pytest.mark.parametrize("quant,pv_fp8", MODES)
@pytest.mark.parametrize("n,ratio,seed", [(1000, 0.2, 71), (1088, 0.25, 72), (33, 0.5, 73)])
def test_tails(quant, pv_fp8, n, ratio, seed):
    q, k, v = inputs.make_random(1, 2, n, seed, k_offset_std=1.0)
    res = gpu_run(q, k, v, ratio, quant=quant, pv_fp8=pv_fp8)
    _all_heads(q, k, v, ratio, res, quant, pv_fp8)


@pytest.mark.parametrize("quant,pv_fp8", MODES)
def test_full_size_sampled(quant, pv_fp8):
    """The Wan2.1-1.3B-480P sequence length, two heads, sampled query blocks."""
    q, k, v = inputs.make_qkv("wan21_1p3b_480p", heads=2)
    res = gpu_run(q, k, v, 0.1, quant=quant, pv_fp8=pv_fp8)
    nb = res["layout"]["nb"]
    rows = sorted({0, 1, 100, 311, nb - 2, nb - 1})
    _all_heads(q, k, v, 0.1, res, quant, pv_fp8, rows=rows)


def test_modes_share_selection_and_differ_in_the_sparse_branch():
    """Same kept lists in every mode; the outputs differ (by the quantization) but stay close."""
    q, k, v = inputs.make_random(1, 2, 2048, 74)
    outs = [gpu_run(q, k, v, 0.1, quant=qm, pv_fp8=pm) for qm, pm in [(True, True)] + MODES]
    for r in outs[1:]:
        assert np.array_equal(r["kept"], outs[0]["kept"])
        d = (r["out"] - outs[0]["out"]).abs().max().item()
        assert 0 < d < 0.1, d


def test_unsupported_mode_is_rejected():
    q, k, v = (x.cuda() for x in inputs.make_random(1, 1, 128, 75))
    with pytest.raises(sba.SageslaError):
        sba.sagesla_forward(q, k, v, 0.5, quant=False, pv_fp8=True)
