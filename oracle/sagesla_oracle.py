"""CPU oracle for the SageSLA attention forward.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module. The
product path (the C-ABI library and its Python binding) never calls it, and this module
shares no code, table or constant generator with the CUDA path.

What it computes, in float64 with plain loops over blocks (numpy matmul is the only library
primitive used for a step), following the pages step by step:

* Block scores and Top-K: news.qq.com TurboDiffusion article, section 第一把钥匙 (score the
  pairs, keep the Top-K ratio 0.1 of connections, skip the rest); section 从训练到部署
  (ratio 0.1-0.15); tiemojia.cn article section 2.2.1 (``sla_topk`` default 0.1).
  Mean pooling over 64-token blocks is the reading taken for "quickly score".
* Low-bit quantization: same article, section 第一把钥匙 (8-bit integers, a quarter of the
  data) and section 第三把钥匙 (per-block shared scales; outliers smoothed by a transform
  before quantization). Reading: INT8 per-block scales for Q and mean-smoothed K, FP8 e4m3
  per-channel scales for V, FP8 P with the fixed scale 1/448.
* Linear branch: dgmzs.com.cn README translation, section 方法论 ("Sparse-Linear
  Attention"), bonega.ai article section "SLA: Sparse-Linear Attention" (near-linear cost).
  Reading: normalized linear attention with phi = softmax over the head dimension, over the
  key blocks that the sparse branch skips, summed with the sparse branch.

Pins: every function here is pinned by a test in ``tests/test_oracle_pins.py`` against
something other than itself (a library routine, brute force on tiny inputs, a closed form or
an invariant). Parity with the authors' own kernel is unpinned: the pages hold no code and
no numeric example for it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

D_HEAD = 128
BLOCK = 64
E4M3_MAX = 448.0
INT8_MAX = 127.0
AMBIGUOUS_MARGIN = 1e-4


# --------------------------------------------------------------------------------------
# Number formats, written from their public definitions (IEEE-754 binary32, bfloat16,
# OCP 8-bit floating point e4m3 "fn").
# --------------------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """Round real values (float64) to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits; its smallest subnormal step is 2**-133. Values whose
    rounded magnitude exceeds the largest finite bfloat16 become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    nz = np.isfinite(x) & (x != 0.0)
    ax = np.abs(x[nz])
    _, e = np.frexp(ax)                      # ax = f * 2**e with f in [0.5, 1)
    q_exp = np.maximum(e - 8, -133)          # quantum of an 8-significant-bit grid
    quantum = np.ldexp(1.0, q_exp)
    r = np.rint(ax / quantum) * quantum      # division by a power of two is exact
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(r > bf16_max, np.inf, r)
    out[nz] = np.copysign(r, x[nz])
    return out


def round_e4m3(x) -> np.ndarray:
    """Round to the OCP e4m3 grid, ties to even, then saturate magnitudes above 448.

    e4m3: exponent bias 7, 3 mantissa bits; normals from 2**-6, subnormal step 2**-9,
    largest finite value 1.75 * 2**8 = 448 (the all-ones pattern is NaN). "satfinite"
    clamps a result beyond 448 to 448 instead of producing NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    _, e = np.frexp(np.where(ax > 0, ax, 1.0))
    unbiased = e - 1                          # ax = 2**unbiased * [1, 2)
    q_exp = np.maximum(unbiased - 3, -9)      # 3 mantissa bits; subnormal step 2**-9
    quantum = np.ldexp(1.0, q_exp)
    r = np.rint(ax / quantum) * quantum
    r = np.minimum(r, E4M3_MAX)
    r = np.where(ax > 0, r, 0.0)
    return np.copysign(r, x)


def e4m3_code(values) -> np.ndarray:
    """Bit pattern (uint8) of values that already lie on the e4m3 grid."""
    v = np.asarray(values, dtype=np.float64)
    sign = np.signbit(v).astype(np.int64)
    a = np.abs(v)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    unbiased = e - 1
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, unbiased + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, unbiased) * 8.0 - 8.0, a / 2.0 ** -9)
    mant = np.where(a > 0, mant, 0.0)
    return ((sign << 7) | (exp_field << 3) | mant.astype(np.int64)).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 bit pattern (NaN for 0x7F and 0xFF)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp_field = (c >> 3) & 0xF
    mant = c & 0x7
    val = np.where(exp_field == 0,
                   mant * 2.0 ** -9,
                   (1.0 + mant / 8.0) * np.ldexp(1.0, exp_field - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def f32(x) -> np.ndarray:
    """IEEE binary32 rounding of a value (numpy float32 arithmetic is IEEE, ties to even)."""
    return np.asarray(x, dtype=np.float32)


# --------------------------------------------------------------------------------------
# Blocks, pooling, scores, Top-K
# --------------------------------------------------------------------------------------

def n_blocks(n_tokens: int) -> int:
    return (n_tokens + BLOCK - 1) // BLOCK


def block_rows(j: int, n_tokens: int) -> slice:
    return slice(BLOCK * j, min(BLOCK * j + BLOCK, n_tokens))


def topk_count(topk_ratio: float, nb: int) -> int:
    """k = clamp(ceil(r * nb - 1e-9), 1, nb) in double precision."""
    k = math.ceil(float(topk_ratio) * nb - 1e-9)
    return max(1, min(nb, k))


def pooled_means(x: np.ndarray) -> np.ndarray:
    """Mean of each 64-token block over its real tokens -> [nb, D] float64."""
    n = x.shape[0]
    nb = n_blocks(n)
    out = np.empty((nb, x.shape[1]), dtype=np.float64)
    for j in range(nb):
        out[j] = x[block_rows(j, n)].mean(axis=0)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """s_ij = qbar_i . kbar_j / sqrt(D)."""
    return (qbar @ kbar.T) / math.sqrt(qbar.shape[1])


def select_topk(scores_row: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, equal scores taken lowest index first; ascending.

    Threshold form: take every index whose score is above the k-th largest value, then fill
    the remaining places with the lowest indices whose score equals it.
    """
    nb = scores_row.shape[0]
    if k >= nb:
        return np.arange(nb)
    kth = np.partition(scores_row, nb - k)[nb - k]        # k-th largest value
    above = np.flatnonzero(scores_row > kth)
    equal = np.flatnonzero(scores_row == kth)
    chosen = np.concatenate([above, equal[: k - above.size]])
    return np.sort(chosen)


def row_margin(scores_row: np.ndarray, k: int) -> float:
    """(s_(k) - s_(k+1)) / max|s|; +inf when there is no (k+1)-th score or max|s| = 0."""
    nb = scores_row.shape[0]
    denom = float(np.max(np.abs(scores_row)))
    if k >= nb or denom == 0.0:
        return math.inf
    desc = np.sort(scores_row)[::-1]
    return float(desc[k - 1] - desc[k]) / denom


# --------------------------------------------------------------------------------------
# Smoothing and quantization
# --------------------------------------------------------------------------------------

def smoothing_mean(k_head: np.ndarray) -> np.ndarray:
    """mu_c = bf16_rne(exact column sum / N), the division done once in double."""
    n = k_head.shape[0]
    sums = np.array([math.fsum(k_head[:, c]) for c in range(k_head.shape[1])])
    return round_bf16(sums / n)


def quant_int8_block(x_block) -> tuple[np.ndarray, np.float32]:
    """Per-block INT8: inv = fl32(127/a), code = clamp(rne(fl32(x*inv)), -127, 127),
    scale = fl32(a/127); a = 0 gives scale 1 and zero codes."""
    xb = f32(x_block)
    a = np.float32(np.max(np.abs(xb))) if xb.size else np.float32(0.0)
    if a == 0:
        return np.zeros(xb.shape, dtype=np.int8), np.float32(1.0)
    inv = np.float32(INT8_MAX) / a
    codes = np.clip(np.rint(xb * inv), -INT8_MAX, INT8_MAX).astype(np.int8)
    return codes, np.float32(a / np.float32(INT8_MAX))


def quant_v_fp8(v_head: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-channel e4m3: inv_c = fl32(448/a_c), code = e4m3(fl32(v*inv_c)),
    s_v = fl32(a_c/448); a_c = 0 gives s_v = 1 and zero codes.
    Returns (decoded code values in [-448, 448] as float64, s_v as float32)."""
    vf = f32(v_head)
    a = np.max(np.abs(vf), axis=0).astype(np.float32)
    safe = np.where(a > 0, a, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    scaled = (vf * inv[None, :]).astype(np.float32)
    vals = round_e4m3(scaled.astype(np.float64))
    vals = np.where(a[None, :] > 0, vals, 0.0)
    s_v = np.where(a > 0, (a / np.float32(E4M3_MAX)).astype(np.float32), np.float32(1.0))
    return vals, s_v.astype(np.float32)


# --------------------------------------------------------------------------------------
# The two branches
# --------------------------------------------------------------------------------------

# The P tile holds e4m3(448 p) with p = e^{S - m'} (m' the running maximum after the block):
# the oracle takes that code exactly, from the float64 value of 448 p. A kernel evaluates
# 448 p in binary32 and through an approximate base-2 exponential, so where 448 p lies very
# close to a rounding boundary of the e4m3 grid it may take the neighbouring code. The bound
# on how far the kernel's value may sit from 448 p is a property of a binary32 evaluation of
# the exponent, independent of any particular kernel:
#   x = S c + (log2 448 - m)      c = sq sk log2(e) / sqrt(128),  m = m' log2(e).
# The factor of c common to all blocks of a row (sq log2(e) / sqrt(128)) is rounded at most
# four times; that common relative error scales every exponent of the row alike, so it moves
# x by at most 4u |S c - m|. Each block's c takes one more rounding (u |S c|), the block
# maximum times c one and the running maximum is one of those (2u |m|), the difference with
# log2 448 two (u (2 log2 448 + |m|)) and the fused multiply-add one (u |x|). With u = 2^-24:
#   |x - x_exact| <= u (5 |S c - m| + |S c| + 3 |m| + 27)     (base-2 units),
# and the exponential itself adds a relative error eps_exp. In natural-log units (s = S c
# ln 2, the logit; m' the running maximum) the relative distance of the kernel's value from
# 448 p is therefore at most
#   w = 2^-21 (|s - m'| + (|s| + 3 |m'|) / 4 + 3) + eps_exp,
# a factor of two or more above each term (2^-21 = 8u). A code is *ambiguous* when
# 448 p (1 - w) and 448 p (1 + w) round to different e4m3 values; the oracle reports, per
# output element, how much choosing the other code could change it, and how much the row sum l
# can move when every p carries its window.
EXP2_REL_ERR = 2.0 ** -20        # eps_exp: the kernel's 2^x (a few units in the last place)


def p_code_window(s: np.ndarray, m_new: np.ndarray, exp_rel_err: float = EXP2_REL_ERR):
    """Relative window w around 448 p for logits s [nq, nk] and running maxima m_new [nq]."""
    m = m_new[:, None]
    return 2.0 ** -21 * (np.abs(s - m) + (np.abs(s) + 3.0 * np.abs(m)) / 4.0 + 3.0) + exp_rel_err


def e4m3_ambiguity(y: np.ndarray, rel) -> np.ndarray:
    """|code change| (as a value) when y, perturbed by up to rel relative (a scalar or an
    array shaped like y), can round to the neighbouring e4m3 value instead; 0 where the
    rounding is unambiguous."""
    lo = round_e4m3(y * (1.0 - rel))
    hi = round_e4m3(y * (1.0 + rel))
    r = round_e4m3(y)
    return np.maximum(np.abs(hi - r), np.abs(r - lo))


def online_softmax_p8(blocks, exp_rel_err: float = EXP2_REL_ERR):
    """The online loop of the sparse branch with the P tile in e4m3.

    ``blocks``: the kept key blocks in ascending order, each a pair (s, v8) of the logits
    s [nq, nk] (float64, natural-log units) and the decoded V codes v8 [nk, D] of its keys.
    For each block: m' = max(m, rowmax s); alpha = e^{m - m'} (0 while m = -inf);
    p = e^{s - m'}; l <- alpha l + sum p (unquantized p); o <- alpha o + e4m3(448 p) . v8;
    m <- m'. Returns (o [nq, D], l [nq], amb [nq, D], lw [nq]): amb bounds the change of o
    from ambiguous codes (sum of the alternative code's distance times |v8|), and lw = the
    same recurrence as l with every p weighted by its window w, so that lw / l bounds the
    relative error of a row sum formed from values within their windows."""
    nq = blocks[0][0].shape[0]
    d = blocks[0][1].shape[1]
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    lw = np.zeros(nq)
    o = np.zeros((nq, d))
    amb = np.zeros((nq, d))
    for s, v8 in blocks:
        m_new = np.maximum(m, s.max(axis=1))
        alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
        p = np.exp(s - m_new[:, None])
        w = p_code_window(s, m_new, exp_rel_err)
        y = E4M3_MAX * p
        l = alpha * l + p.sum(axis=1)
        lw = alpha * lw + (p * w).sum(axis=1)
        o = alpha[:, None] * o + round_e4m3(y) @ v8
        amb = alpha[:, None] * amb + e4m3_ambiguity(y, w) @ np.abs(v8)
        m = m_new
    return o, l, amb, lw


def online_softmax_real(blocks):
    """The online loop with real P and V (the 16-bit operand modes): for each kept block in
    ascending order, with logits s [nq, nk] and value rows v [nk, D]: m' = max(m, rowmax s),
    alpha = e^{m - m'}, p = e^{s - m'}, l <- alpha l + sum p, o <- alpha o + p . v. Returns
    (o, l, mag) with mag the same recurrence over p . |v| (so that mag / l is the output of
    the same weights applied to |v|, the size of the terms each output element sums)."""
    nq = blocks[0][0].shape[0]
    d = blocks[0][1].shape[1]
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    o = np.zeros((nq, d))
    mag = np.zeros((nq, d))
    for s, v in blocks:
        m_new = np.maximum(m, s.max(axis=1))
        alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
        p = np.exp(s - m_new[:, None])
        l = alpha * l + p.sum(axis=1)
        o = alpha[:, None] * o + p @ v
        mag = alpha[:, None] * mag + p @ np.abs(v)
        m = m_new
    return o, l, mag


# Tolerance of the sparse branch when P (and V) enter the P.V product in bf16: P rounded to
# bf16 (relative 2^-9 per term), fp32 accumulation; twice the unit roundoff times the size of
# the terms.
BF16_PV_REL = 2.0 ** -8


def sparse_output(o: np.ndarray, l: np.ndarray, s_v: np.ndarray) -> np.ndarray:
    """O_s = o s_v / (448 l): the P codes carry the scale 1/448, the V codes s_v per channel."""
    return o * (np.asarray(s_v, dtype=np.float64)[None, :] / (E4M3_MAX * l[:, None]))


def phi(x: np.ndarray) -> np.ndarray:
    """Softmax over the last (head) dimension."""
    z = np.exp(x - x.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


@dataclass
class HeadPrep:
    """Per-(b,h) quantities shared by all query blocks."""
    n: int
    nb: int
    k: int
    qbar: np.ndarray
    kbar: np.ndarray
    scores: np.ndarray
    kept: list                          # blocks the branches use (selected, or the override)
    margin: np.ndarray
    selected: list | None = None        # the oracle's own Top-K selection
    mu: np.ndarray | None = None
    q8: np.ndarray | None = None       # int8 codes [N, D]
    sq: np.ndarray | None = None       # float32 [nb]
    k8: np.ndarray | None = None
    sk: np.ndarray | None = None
    v8: np.ndarray | None = None       # decoded e4m3 values [N, D]
    s_v: np.ndarray | None = None      # float32 [D]
    h_blocks: np.ndarray | None = field(default=None, repr=False)  # [nb, D, D+1]


def prepare_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, topk_ratio: float,
                 quant: bool = True, kept_override=None) -> HeadPrep:
    """Everything of one head that does not depend on the query block being evaluated.

    ``kept_override`` replaces the Top-K selection (used to evaluate the branches on a block
    mask chosen elsewhere, e.g. on an ambiguous row)."""
    n = q.shape[0]
    nb = n_blocks(n)
    kk = topk_count(topk_ratio, nb)
    qbar, kbar = pooled_means(q), pooled_means(k)
    scores = block_scores(qbar, kbar)
    kept = [select_topk(scores[i], kk) for i in range(nb)]
    selected = kept
    if kept_override is not None:
        kept = [np.asarray(kept_override[i], dtype=np.int64) for i in range(nb)]
    margin = np.array([row_margin(scores[i], kk) for i in range(nb)])
    prep = HeadPrep(n=n, nb=nb, k=kk, qbar=qbar, kbar=kbar, scores=scores, kept=kept,
                    margin=margin, selected=selected)
    if quant:
        prep.mu = smoothing_mean(k)
        ks = (f32(k) - f32(prep.mu)[None, :]).astype(np.float32)
        prep.q8 = np.zeros(q.shape, dtype=np.int8)
        prep.k8 = np.zeros(k.shape, dtype=np.int8)
        prep.sq = np.zeros(nb, dtype=np.float32)
        prep.sk = np.zeros(nb, dtype=np.float32)
        for j in range(nb):
            rows = block_rows(j, n)
            prep.q8[rows], prep.sq[j] = quant_int8_block(q[rows])
            prep.k8[rows], prep.sk[j] = quant_int8_block(ks[rows])
        prep.v8, prep.s_v = quant_v_fp8(v)
    return prep


def key_block_states(k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """H_j = sum over the real tokens u of block j of phi(k_u)^T [v_u | 1] -> [nb, D, D+1]."""
    n = k.shape[0]
    nb = n_blocks(n)
    pk = phi(k)
    h = np.zeros((nb, k.shape[1], v.shape[1] + 1), dtype=np.float64)
    for j in range(nb):
        rows = block_rows(j, n)
        h[j, :, : v.shape[1]] = pk[rows].T @ v[rows]
        h[j, :, v.shape[1]] = pk[rows].sum(axis=0)
    return h


def sparse_block_row(prep: HeadPrep, i: int, q, k, v, quant: bool = True,
                     smooth_in_quant_off: bool = False, return_ambiguity: bool = False,
                     pv_fp8: bool = True):
    """Sparse branch for the real query tokens of block i: online softmax over kept(i) in
    ascending order, running max updated per key block (no lazy rescale).

    ``quant``: logits from the INT8 codes of the smoothed, block-scaled Q and K, or from the
    real Q and K. ``pv_fp8`` (with ``quant``): P and V as e4m3 codes, or real P and V.
    With ``return_ambiguity`` also returns, per output element, the allowance a kernel needs:
    ambiguous P codes and the window of the row sum (e4m3 P.V), or the bf16 rounding of P
    (real P.V: BF16_PV_REL times the output of the same weights applied to |v|)."""
    n = prep.n
    qrows = block_rows(i, n)
    inv_sqrt_d = 1.0 / math.sqrt(q.shape[1])
    if quant:
        logits = []
        for j in prep.kept[i]:
            krows = block_rows(int(j), n)
            s_int = prep.q8[qrows].astype(np.float64) @ prep.k8[krows].astype(np.float64).T
            logits.append((s_int * (float(prep.sq[i]) * float(prep.sk[j])) * inv_sqrt_d, krows))
        if pv_fp8:
            o, l, amb, lw = online_softmax_p8([(s_, prep.v8[kr]) for s_, kr in logits])
            o_s = sparse_output(o, l, prep.s_v)
            if return_ambiguity:
                return o_s, sparse_output(amb, l, prep.s_v) + np.abs(o_s) * (lw / l)[:, None]
            return o_s
        o, l, mag = online_softmax_real([(s_, v[kr]) for s_, kr in logits])
    else:
        k_used = k - smoothing_mean(k)[None, :] if smooth_in_quant_off else k
        blocks = []
        for j in prep.kept[i]:
            krows = block_rows(int(j), n)
            blocks.append(((q[qrows] @ k_used[krows].T) * inv_sqrt_d, v[krows]))
        o, l, mag = online_softmax_real(blocks)
    if return_ambiguity:
        return o / l[:, None], BF16_PV_REL * mag / l[:, None]
    return o / l[:, None]


def linear_block_row(prep: HeadPrep, i: int, q, h_blocks: np.ndarray) -> np.ndarray:
    """Linear branch for block i: phi(q_t) G_i[:, :D] / phi(q_t) G_i[:, D], G_i the sum of
    H_j over the key blocks not kept by i; zero when every block is kept."""
    qrows = block_rows(i, prep.n)
    d = q.shape[1]
    comp = np.setdiff1d(np.arange(prep.nb), prep.kept[i])
    if comp.size == 0:
        return np.zeros((qrows.stop - qrows.start, d))
    g = h_blocks[comp].sum(axis=0)                   # [D, D+1]
    pq = phi(q[qrows])
    num = pq @ g[:, :d]
    den = pq @ g[:, d]
    return num / den[:, None]


def linear_block_row_bruteforce(prep: HeadPrep, i: int, q, k, v) -> np.ndarray:
    """Linear branch by its per-token definition (slow; for pins on tiny inputs)."""
    n = prep.n
    qrows = block_rows(i, n)
    comp = np.setdiff1d(np.arange(prep.nb), prep.kept[i])
    out = np.zeros((qrows.stop - qrows.start, q.shape[1]))
    if comp.size == 0:
        return out
    toks = np.concatenate([np.arange(block_rows(int(j), n).start, block_rows(int(j), n).stop)
                           for j in comp])
    for a, t in enumerate(range(qrows.start, qrows.stop)):
        pq = phi(q[t])
        num = np.zeros(q.shape[1])
        den = 0.0
        for u in toks:
            w = float(pq @ phi(k[u]))
            num += w * v[u]
            den += w
        out[a] = num / den
    return out


# --------------------------------------------------------------------------------------
# Whole forward
# --------------------------------------------------------------------------------------

def forward_head(q, k, v, topk_ratio: float, quant: bool = True, rows=None,
                 kept_override=None, smooth_in_quant_off: bool = False, pv_fp8: bool = True):
    """SageSLA forward for one (b,h). q, k, v: float64 [N, D] holding bf16 values.

    ``rows``: query blocks to evaluate (default all). Returns (prep, out) where out maps a
    block index to a dict with 'o_s', 'o_l' and 'o' ([n_i, D] float64)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    prep = prepare_head(q, k, v, topk_ratio, quant=quant, kept_override=kept_override)
    h_blocks = key_block_states(k, v)
    prep.h_blocks = h_blocks
    if rows is None:
        rows = range(prep.nb)
    out = {}
    for i in rows:
        o_s, amb = sparse_block_row(prep, i, q, k, v, quant=quant,
                                    smooth_in_quant_off=smooth_in_quant_off,
                                    return_ambiguity=True, pv_fp8=pv_fp8)
        o_l = linear_block_row(prep, i, q, h_blocks)
        out[i] = {"o_s": o_s, "o_l": o_l, "o": o_s + o_l, "o_s_ambig": amb}
    return prep, out


def forward(q, k, v, topk_ratio: float, quant: bool = True, kept_override=None):
    """Full forward on [B, H, N, D] arrays (float64 bf16 values) -> (O [B,H,N,D], preps)."""
    q = np.asarray(q, dtype=np.float64)
    b_, h_, n, d = q.shape
    o = np.zeros((b_, h_, n, d))
    preps = {}
    for b in range(b_):
        for h in range(h_):
            ko = None if kept_override is None else kept_override[b][h]
            prep, out = forward_head(q[b, h], k[b, h], v[b, h], topk_ratio, quant=quant,
                                     kept_override=ko)
            for i, r in out.items():
                o[b, h, block_rows(i, n)] = r["o"]
            preps[(b, h)] = prep
    return o, preps
