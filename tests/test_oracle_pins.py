"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a library routine, a brute-force evaluation on tiny
inputs, an exact-arithmetic computation, a closed form, an invariant of the definition, or a
fixture under tests/golden/ with its citation. Together they are chosen so that a dropped
term, a wrong sign or index, or a transposed operand anywhere in the oracle fails one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as orc
from sparse_bit_attention_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_head(n, seed, scale=1.0, k_offset=0.0):
    q, k, v = inputs.make_random(1, 1, n, seed, k_offset_std=k_offset, scale=scale)
    return inputs.as_float64(q[0, 0]), inputs.as_float64(k[0, 0]), inputs.as_float64(v[0, 0])


def _sdpa64(q, k, v, mask=None):
    """Dense softmax attention in float64 through torch's library routine."""
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)[0, 0].numpy()


# ---------------------------------------------------------------- number formats

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
        rng.standard_normal(2000) * 1e-39,               # bf16 subnormal range
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 0.0]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.round_bf16(x.astype(np.float64)), ref)


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.uniform(-463.0, 463.0, 20000),
        rng.uniform(-0.02, 0.02, 20000),                 # subnormal and low normal range
        orc.e4m3_decode(np.arange(0, 126)) * 1.0,       # grid points
        (orc.e4m3_decode(np.arange(0, 125)) + orc.e4m3_decode(np.arange(1, 126))) / 2,  # ties
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn)
    got = orc.round_e4m3(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref.to(torch.float64).numpy())
    np.testing.assert_array_equal(orc.e4m3_code(got), ref.view(torch.uint8).numpy())


def test_e4m3_golden_points():
    path = os.path.join(GOLDEN, "e4m3_points.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    for xin, xout, code in rows:
        got = orc.round_e4m3(np.array([float(xin)]))
        assert got[0] == float(xout), (xin, got)
        assert int(orc.e4m3_code(got)[0]) == int(code, 16), (xin, code)


def test_e4m3_decode_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = orc.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])
    # every finite pattern survives decode -> encode (the zero pattern 0x80 is -0.0)
    np.testing.assert_array_equal(orc.e4m3_code(got[fin]), codes[fin])


def test_int8_quantizer_round_trip_bound():
    rng = np.random.default_rng(3)
    for trial in range(50):
        x = (rng.standard_normal((64, 128)) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        codes, s = orc.quant_int8_block(x)
        assert codes.dtype == np.int8 and np.abs(codes.astype(int)).max() == 127
        err = np.abs(x.astype(np.float64) - float(s) * codes.astype(np.float64))
        # half a step, plus the binary32 rounding of inv, of x*inv and of s
        assert err.max() <= float(s) * (0.5 + 1e-5)
    codes, s = orc.quant_int8_block(np.zeros((64, 128), np.float32))
    assert s == 1.0 and not codes.any()


def test_int8_quantizer_closed_form():
    # integers with max 127: inv = 1 exactly, so the codes are the integers themselves
    x = np.tile(np.arange(-127, 128, dtype=np.float32)[:128], (64, 1))
    codes, s = orc.quant_int8_block(x)
    assert s == 1.0
    np.testing.assert_array_equal(codes.astype(np.float32), x)


def test_v_fp8_quantizer_bound():
    q, k, v = _rand_head(300, 4)
    vals, s_v = orc.quant_v_fp8(v)
    assert np.abs(vals).max() == 448.0
    rec = vals * s_v.astype(np.float64)[None, :]
    # e4m3 relative step 2^-3 for normals -> error <= 2^-4 relative (+ subnormal floor)
    bound = np.abs(v) * 2.0 ** -4 + (2.0 ** -10) * s_v[None, :] + 1e-7 * np.abs(v)
    assert np.all(np.abs(rec - v) <= bound)


def test_smoothing_mean_exact_arithmetic():
    q, k, v = _rand_head(777, 5, k_offset=1.5)
    mu = orc.smoothing_mean(k)
    for c in range(0, 128, 9):
        exact = sum(Fraction(float(x)) for x in k[:, c]) / k.shape[0]
        assert mu[c] == orc.round_bf16(np.array([float(exact)]))[0]
        # the bf16 value is the nearest one to the exact mean
        assert abs(Fraction(float(mu[c])) - exact) <= abs(Fraction(float(mu[c])) * 2 ** -8) + Fraction(1, 2 ** 140)


# ---------------------------------------------------------------- blocks, Top-K

def test_topk_counts_golden():
    path = os.path.join(GOLDEN, "topk_counts.txt")
    for line in open(path):
        if not line.strip() or line.startswith("#"):
            continue
        n, nb, r, k = line.split()
        assert orc.n_blocks(int(n)) == int(nb)
        assert orc.topk_count(float(r), int(nb)) == int(k), line


def test_topk_matches_bruteforce_sort_with_ties():
    rng = np.random.default_rng(6)
    for trial in range(200):
        nb = int(rng.integers(1, 40))
        k = int(rng.integers(1, nb + 1))
        s = rng.integers(-5, 5, nb).astype(np.float64)          # many ties
        brute = sorted(sorted(range(nb), key=lambda j: (-s[j], j))[:k])
        assert list(orc.select_topk(s, k)) == brute


def test_pooled_means_and_scores_bruteforce():
    q, k, v = _rand_head(150, 7)                   # 3 blocks, last one 22 tokens
    qb = orc.pooled_means(q)
    assert qb.shape == (3, 128)
    np.testing.assert_allclose(qb[2], np.array([sum(q[t, c] for t in range(128, 150)) / 22
                                                for c in range(128)]), rtol=0, atol=1e-15)
    s = orc.block_scores(qb, orc.pooled_means(k))
    i, j = 2, 1
    brute = sum(qb[i, c] * orc.pooled_means(k)[j, c] for c in range(128)) / math.sqrt(128)
    assert abs(s[i, j] - brute) < 1e-15


def test_margin_definition():
    s = np.array([3.0, 1.0, 2.0, 2.0 - 1e-6])
    assert orc.row_margin(s, 2) == pytest.approx((2.0 - (2.0 - 1e-6)) / 3.0)
    assert orc.row_margin(s, 4) == math.inf


# ---------------------------------------------------------------- the two branches

@pytest.mark.parametrize("n", [256, 200, 64, 37])
def test_dense_limit_equals_softmax_attention(n):
    """r = 1 with quantization off: the complement is empty and the sparse branch is exact
    softmax attention over all keys."""
    q, k, v = _rand_head(n, 8)
    prep, out = orc.forward_head(q, k, v, 1.0, quant=False)
    o = np.concatenate([out[i]["o"] for i in range(prep.nb)])
    assert all(not out[i]["o_l"].any() for i in range(prep.nb))
    np.testing.assert_allclose(o, _sdpa64(q, k, v), rtol=0, atol=1e-10)


def test_sparse_branch_equals_block_masked_attention():
    """Quantization off, r < 1: the online block loop equals softmax attention restricted
    to the kept blocks (a boolean block mask given to the library routine)."""
    n = 300
    q, k, v = _rand_head(n, 9)
    prep, out = orc.forward_head(q, k, v, 0.4, quant=False)
    mask = np.zeros((n, n), dtype=bool)
    for i in range(prep.nb):
        for j in prep.kept[i]:
            mask[orc.block_rows(i, n), orc.block_rows(int(j), n)] = True
    ref = _sdpa64(q, k, v, mask)
    o_s = np.concatenate([out[i]["o_s"] for i in range(prep.nb)])
    np.testing.assert_allclose(o_s, ref, rtol=0, atol=1e-10)
    # the kept sets really are the top scores
    for i in range(prep.nb):
        brute = sorted(sorted(range(prep.nb), key=lambda j: (-prep.scores[i, j], j))[:prep.k])
        assert list(prep.kept[i]) == brute


def test_linear_branch_block_form_equals_per_token_definition():
    n = 200
    q, k, v = _rand_head(n, 10)
    prep, out = orc.forward_head(q, k, v, 0.3, quant=True)
    for i in range(prep.nb):
        brute = orc.linear_block_row_bruteforce(prep, i, q, k, v)
        np.testing.assert_allclose(out[i]["o_l"], brute, rtol=0, atol=1e-12)


def test_smoothing_is_a_row_constant_shift():
    n = 256
    q, k, v = _rand_head(n, 11, k_offset=2.0)
    _, a = orc.forward_head(q, k, v, 0.5, quant=False)
    _, b = orc.forward_head(q, k, v, 0.5, quant=False, smooth_in_quant_off=True)
    for i in a:
        np.testing.assert_allclose(a[i]["o"], b[i]["o"], rtol=0, atol=1e-12)


def test_constant_v():
    n = 256
    q, k, _ = _rand_head(n, 12)
    c = np.linspace(-2.0, 2.0, 128)
    v = np.tile(orc.round_bf16(c), (n, 1))
    prep, out = orc.forward_head(q, k, v, 0.25, quant=False)
    for i in out:
        np.testing.assert_allclose(out[i]["o"], 2 * v[: out[i]["o"].shape[0]], atol=1e-12)
    prep, out = orc.forward_head(q, k, v, 0.25, quant=True)
    for i in out:
        vv = v[: out[i]["o"].shape[0]]
        np.testing.assert_allclose(out[i]["o_l"], vv, atol=1e-12)
        # sparse branch: each P entry is off by at most 2^-4 relative after e4m3 rounding
        assert np.all(np.abs(out[i]["o_s"] - vv) <= np.abs(vv) * 2.0 ** -4 + 1e-6)


def test_single_block_is_dense_attention():
    q, k, v = _rand_head(50, 13)
    prep, out = orc.forward_head(q, k, v, 0.1, quant=False)
    assert prep.nb == 1 and prep.k == 1
    assert not out[0]["o_l"].any()
    np.testing.assert_allclose(out[0]["o"], _sdpa64(q, k, v), atol=1e-10)


def test_quantized_scores_are_integer_exact():
    n = 128
    q, k, v = _rand_head(n, 14, k_offset=1.0)
    prep = orc.prepare_head(q, k, v, 1.0)
    for t, u in [(0, 0), (5, 77), (63, 127), (100, 3)]:
        brute = sum(int(prep.q8[t, c]) * int(prep.k8[u, c]) for c in range(128))
        assert float(prep.q8[t].astype(np.float64) @ prep.k8[u].astype(np.float64)) == brute
    # K smoothing: codes dequantize to k - mu within half a step
    ks = k - prep.mu[None, :]
    for j in range(prep.nb):
        r = orc.block_rows(j, n)
        assert np.abs(ks[r] - float(prep.sk[j]) * prep.k8[r]).max() <= float(prep.sk[j]) * 0.5001


def test_quantized_forward_is_close_to_exact():
    """Quantization is a small perturbation: INT8/FP8 output within a few 1e-2 of the
    quantization-off output on the tiny workload's distribution."""
    q, k, v = _rand_head(512, 15, k_offset=math.sqrt(2.0))
    _, a = orc.forward_head(q, k, v, 0.25, quant=True)
    _, b = orc.forward_head(q, k, v, 0.25, quant=False)
    err = max(np.abs(a[i]["o"] - b[i]["o"]).max() for i in a)
    assert 1e-4 < err < 0.08


def _golden_two_blocks():
    rows, cur, s_v = {}, None, None
    for line in open(os.path.join(GOLDEN, "p8_two_blocks.txt")):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "s_v":
            s_v = np.array([float(x) for x in f[1:]])
        elif f[0] == "row":
            cur = rows.setdefault(f[1], {"blocks": []})
        elif f[0] == "block":
            cur["blocks"].append([])
        elif f[0] == "key":
            cur["blocks"][-1].append((float(f[1]), int(f[2])))
        elif f[0] == "expect_l":
            cur["l"] = float(f[1])
        elif f[0] == "expect_o":
            cur["o"] = np.array([float(x) for x in f[1:]])
    return rows, s_v


def test_online_loop_golden_two_blocks():
    """The hand-derived two-block rows of tests/golden/p8_two_blocks.txt: codes against the
    running maximum of each block, the row sum of the unquantized p, the 1/448 and s_v
    scales. Row A fails if codes are taken against the final maximum or l sums the codes;
    row B fails if codes are taken against each block's own maximum."""
    rows, s_v = _golden_two_blocks()
    for name, r in rows.items():
        blocks = []
        for keys in r["blocks"]:
            s = np.array([[lg for lg, _ in keys]])
            v8 = np.zeros((len(keys), s_v.size))
            for u, (_, ch) in enumerate(keys):
                v8[u, ch] = 1.0
            blocks.append((s, v8))
        o, l, amb, lw = orc.online_softmax_p8(blocks)
        assert abs(l[0] - r["l"]) <= 1e-13, (name, l)
        np.testing.assert_allclose(orc.sparse_output(o, l, s_v)[0], r["o"], rtol=0, atol=1e-13)
        assert not amb.any(), name          # no code of the example is near a midpoint
        assert 0 < lw[0] / l[0] < 1e-5


def _binary32_codes(s_blocks, sq, sk_list, eps, rng):
    """An independent binary32 evaluation of the P codes (the way a kernel forms them): the
    exponent in base 2 with the factor 448 folded in, from a float32 constant, a float32 running
    maximum and one fused rounding, then 2^x with a random relative error of up to eps."""
    L = np.float32(np.float32(1.4426950408889634) * np.float32(1.0 / math.sqrt(128.0)))
    lg448 = np.float32(math.log2(448.0))
    m32 = np.full(s_blocks[0].shape[0], -np.inf, dtype=np.float32)
    out = []
    for s_int, sk in zip(s_blocks, sk_list):
        c = np.float32(np.float32(np.float32(sq) * L) * np.float32(sk))
        mx = (s_int.max(axis=1).astype(np.float32) * c).astype(np.float32)
        m32 = np.maximum(m32, mx)
        neg = (lg448 - m32).astype(np.float32)
        x = (s_int.astype(np.float64) * np.float64(c) + neg.astype(np.float64)[:, None]).astype(np.float32)
        y = np.exp2(x.astype(np.float64)) * (1.0 + rng.uniform(-eps, eps, x.shape))
        out.append(orc.round_e4m3(y))
    return out


@pytest.mark.parametrize("scale,offset", [(1.0, 0), (30.0, 0), (30.0, 190000)])
def test_p_code_window_covers_a_binary32_evaluation(scale, offset):
    """Wherever a binary32 evaluation (written here, not in the oracle) picks another e4m3 code
    than the oracle's exact e4m3(448 p), the oracle's window marks that code ambiguous; and the
    window is narrow (few codes ambiguous). Three blocks in sequence, so that the running
    maximum moves; ordinary logits, large logits, and large logits close to each other (many
    codes near the top of the grid computed from large binary32 operands)."""
    rng = np.random.default_rng(16)
    flagged = total = differ = 0
    for trial in range(30):
        sq = np.float32(rng.uniform(0.005, 0.05) * scale)
        sks = [np.float32(rng.uniform(0.005, 0.05)) for _ in range(3)]
        spread = 3000 if offset else 127 * 127 * 12
        s_ints = [offset + rng.integers(-spread, spread, size=(64, 64)) for _ in range(3)]
        ref_codes = _binary32_codes(s_ints, sq, sks, 2.0 ** -21, rng)
        m = np.full(64, -np.inf)
        for s_int, sk, code32 in zip(s_ints, sks, ref_codes):
            s = s_int * (float(sq) * float(sk)) / math.sqrt(128.0)
            m = np.maximum(m, s.max(axis=1))
            y = 448.0 * np.exp(s - m[:, None])
            amb = orc.e4m3_ambiguity(y, orc.p_code_window(s, m))
            differs = code32 != orc.round_e4m3(y)
            assert not np.any(differs & (amb == 0))
            flagged += int((amb > 0).sum())
            differ += int(differs.sum())
            total += amb.size
    assert flagged < 2e-2 * total
    if offset:
        assert differ > 0        # the case does move codes: the window is exercised


def test_e4m3_ambiguity_bound():
    """Zero away from midpoints; exactly one grid step at a midpoint."""
    grid = orc.e4m3_decode(np.arange(0, 127))
    mids = (grid[:-1] + grid[1:]) / 2
    amb = orc.e4m3_ambiguity(mids, 1e-6)
    np.testing.assert_allclose(amb, np.diff(grid))
    off = orc.e4m3_ambiguity(grid[1:], 1e-6)     # on the grid: unambiguous
    assert not off.any()


def test_int8_logits_with_real_pv_equal_block_masked_attention_of_dequantized_q_k():
    """INT8 Q.K^T with real P and V: the sparse branch equals softmax attention over
    the kept blocks with the dequantized Q8 * sq and K8 * sk (the logits are the same numbers)
    and the raw V, through the library routine."""
    n = 300
    q, k, v = _rand_head(n, 17, k_offset=1.0)
    prep, out = orc.forward_head(q, k, v, 0.4, quant=True, pv_fp8=False)
    qd = np.zeros_like(q)
    kd = np.zeros_like(k)
    for j in range(prep.nb):
        r = orc.block_rows(j, n)
        qd[r] = prep.q8[r] * float(prep.sq[j])
        kd[r] = prep.k8[r] * float(prep.sk[j])
    mask = np.zeros((n, n), dtype=bool)
    for i in range(prep.nb):
        for j in prep.kept[i]:
            mask[orc.block_rows(i, n), orc.block_rows(int(j), n)] = True
    ref = _sdpa64(qd, kd, v, mask)
    o_s = np.concatenate([out[i]["o_s"] for i in range(prep.nb)])
    np.testing.assert_allclose(o_s, ref, rtol=0, atol=1e-10)


def test_real_pv_allowance_is_the_branch_of_abs_v():
    """The bf16-P allowance of the real-P.V modes is BF16_PV_REL times the same weights applied
    to |v|: with V >= 0 it equals BF16_PV_REL times the output itself."""
    q, k, v = _rand_head(200, 18)
    v = np.abs(v)
    for quant in (False, True):
        _, out = orc.forward_head(q, k, v, 0.5, quant=quant, pv_fp8=False)
        for r in out.values():
            np.testing.assert_allclose(r["o_s_ambig"], orc.BF16_PV_REL * r["o_s"], rtol=1e-12)
