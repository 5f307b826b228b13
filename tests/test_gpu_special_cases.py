"""GPU parity on inputs that press on single steps of the forward: the linear branch with V of
non-zero channel mean (so that its output is far above the output gate's resolution), the
quantizers' zero cases (an all-zero Q block, a K block equal to the smoothing mean, a zero V
channel), and large logits that stretch the exponent range of the online softmax."""
import numpy as np
import pytest
import torch

import oracle as orc
from sparse_bit_attention_b200 import inputs
from _parity import LAST_ERRS, LIN_ABS, LIN_REL, OUT_TOL, compare_head, gpu_run

pytestmark = pytest.mark.gpu


def _check_linear_branch(q, k, v, ratio, res, b, h, rows):
    B, H, N, D = q.shape
    bh = b * H + h
    qh, kh, vh = (inputs.as_float64(x[b, h]) for x in (q, k, v))
    nb = res["layout"]["nb"]
    kept = [res["kept"][bh, i] for i in range(nb)]
    prep = orc.prepare_head(qh, kh, vh, ratio, quant=False, kept_override=kept)
    hs = orc.key_block_states(kh, vh)
    hs_abs = orc.key_block_states(kh, np.abs(vh))
    worst = 0.0
    for i in rows:
        sl = orc.block_rows(i, N)
        ref = orc.linear_block_row(prep, i, qh, hs)
        mag = orc.linear_block_row(prep, i, qh, hs_abs)
        gpu = (res["out"][b, h, sl].double() - res["sparse"][b, h, sl].double()).numpy()
        tol = LIN_REL * (mag + np.abs(ref)) + LIN_ABS
        excess = np.abs(gpu - ref) - tol
        assert np.all(excess <= 0), (i, float(excess.max()))
        worst = max(worst, float(np.max(np.abs(gpu - ref))))
    return worst


@pytest.mark.parametrize("n,ratio,seed", [
    (1024, 0.1, 51),     # the tiny shape
    (1000, 0.2, 52),     # ragged last block
    (2500, 0.05, 53),    # short rows of kept blocks, large complements
])
def test_linear_branch_with_channel_mean(n, ratio, seed):
    """V = mu_c + N(0, 1) with mu_c of order one: O_l is about mu_c, three orders of
    magnitude above the output gate, and is checked on its own against the oracle."""
    q, k, v = inputs.make_random(1, 2, n, seed, k_offset_std=1.0, v_mean_std=1.5)
    res = gpu_run(q, k, v, ratio)
    nb = res["layout"]["nb"]
    for h in range(2):
        _check_linear_branch(q, k, v, ratio, res, 0, h, range(nb))
        err, _ = compare_head(q, k, v, ratio, res, 0, h, linear_tol=True)
        assert err <= OUT_TOL, (err, LAST_ERRS)


def test_linear_branch_with_channel_mean_full_size_sampled():
    """The Wan2.1-1.3B-480P sequence length (512 blocks, 460 of them in each complement),
    two heads, V with channel means; sampled query blocks."""
    q, k, v = inputs.make_random(1, 2, 32760, 54, v_mean_std=1.5)
    res = gpu_run(q, k, v, 0.1)
    nb = res["layout"]["nb"]
    rows = sorted({0, 1, nb - 2, nb - 1, 97, 250, 401})
    for h in range(2):
        _check_linear_branch(q, k, v, 0.1, res, 0, h, rows)
        err, _ = compare_head(q, k, v, 0.1, res, 0, h, rows=rows, linear_tol=True)
        assert err <= OUT_TOL, (err, LAST_ERRS)


def test_zero_query_block():
    """An all-zero Q block: INT8 scale 1 and zero codes, every logit of its rows 0 (uniform
    attention over its kept blocks), all its block scores 0 (ties: the lowest blocks kept),
    phi(q) uniform."""
    q, k, v = inputs.make_random(1, 2, 1024, 55, k_offset_std=1.0)
    q[:, :, 64 * 5: 64 * 6] = 0
    res = gpu_run(q, k, v, 0.25)
    for h in range(2):
        assert list(res["kept"][h, 5]) == list(range(res["layout"]["k"]))
        err, _ = compare_head(q, k, v, 0.25, res, 0, h)
        assert err <= OUT_TOL, (err, LAST_ERRS)


def test_key_block_equal_to_the_smoothing_mean():
    """A K block whose rows equal the channel mean exactly: after smoothing it is zero, so its
    INT8 scale is 1 and its codes 0. The other blocks come in pairs mean +- r with values on a
    coarse grid, so that the channel mean over all tokens is exactly the block's value."""
    rng = np.random.default_rng(56)
    n = 1024
    c = (rng.integers(-8, 8, 128) / 4.0)                    # the channel means, bf16-exact
    half = (n - 64) // 2
    r = rng.integers(-16, 17, (2, half, 128)) / 8.0         # offsets on a 1/8 grid
    kk = np.empty((2, n, 128))
    kk[:, 3 * 64: 4 * 64] = c
    others = np.concatenate([c + r, c - r], axis=1)          # pairs average to c exactly
    kk[:, np.r_[0: 3 * 64, 4 * 64: n]] = others
    k = torch.from_numpy(kk[None]).to(torch.bfloat16)
    assert torch.equal(k.double(), torch.from_numpy(kk[None]))
    q, _, v = inputs.make_random(1, 2, n, 56)
    res = gpu_run(q, k, v, 0.3)
    for h in range(2):
        prep = orc.prepare_head(inputs.as_float64(q[0, h]), kk[h], inputs.as_float64(v[0, h]), 0.3)
        assert prep.sk[3] == 1.0 and not prep.k8[3 * 64: 4 * 64].any()
        err, _ = compare_head(q, k, v, 0.3, res, 0, h)
        assert err <= OUT_TOL, (err, LAST_ERRS)


def test_zero_v_channel():
    """A V channel that is zero everywhere: its FP8 scale is 1 and its codes 0, and both
    branches give exactly 0 in that channel."""
    q, k, v = inputs.make_random(1, 2, 1000, 57, k_offset_std=1.0)
    v[..., 17] = 0
    v[..., 100] = 0
    res = gpu_run(q, k, v, 0.2)
    assert not res["out"][..., 17].any() and not res["out"][..., 100].any()
    for h in range(2):
        err, _ = compare_head(q, k, v, 0.2, res, 0, h)
        assert err <= OUT_TOL, (err, LAST_ERRS)


@pytest.mark.parametrize("qk_scale", [20.0, 50.0])
def test_large_logits(qk_scale):
    """Q and K multiplied by 20 or 50 (logits of standard deviation 400 or 2500): the softmax
    is nearly one-hot and the running maximum is large, which widens the binary32 window of
    the P codes and stretches phi. V stays N(0, 1)."""
    q, k, v = inputs.make_random(1, 2, 1000, 58, qk_scale=qk_scale)
    res = gpu_run(q, k, v, 0.2)
    nb = res["layout"]["nb"]
    for h in range(2):
        _check_linear_branch(q, k, v, 0.2, res, 0, h, range(nb))
        err, _ = compare_head(q, k, v, 0.2, res, 0, h, linear_tol=True)
        assert err <= OUT_TOL, (err, LAST_ERRS)
