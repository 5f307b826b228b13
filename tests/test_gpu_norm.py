"""GPU parity of the fused normalization (sagesla_norm_quant, through the C ABI) against the
CPU oracle: the bf16 output within one bf16 ulp of the real-number result, the INT8 codes
and row scales bit-exact as functions of the kernel's own bf16 row, and the codes within
half a step (plus the bf16 rounding) of the real-number result."""
import numpy as np
import pytest
import torch

import sparse_bit_attention_b200 as sba
from oracle import norm_oracle as no
from oracle import quant_int8_block, round_bf16

pytestmark = pytest.mark.gpu


def _bf16(t):
    return t.float().double().cpu().numpy()


def _ulp_bf16(v):
    a = np.abs(v)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    return np.ldexp(1.0, np.maximum(e - 8, -133))


def _term_size(xr, kind, eps, gamma, beta, scale, shift, R):
    """Magnitude of the terms summed in the last fp32 steps (affine, modulation): the fp32
    result's absolute error scales with it when those terms cancel."""
    m = np.abs(no.normalize_rows(xr, kind, eps))
    if gamma is not None:
        m = m * np.abs(gamma)
    if beta is not None:
        m = m + np.abs(beta)
    b = np.arange(xr.shape[0]) // max(R, 1)
    if scale is not None:
        m = m * np.abs(1.0 + scale[b])
    if shift is not None:
        m = m + np.abs(shift[b])
    return m


def _check(x, kind, eps, gamma=None, beta=None, scale=None, shift=None, R=0, codes=True):
    dev = torch.device("cuda:0")
    xd = x.to(dev)
    args = [None if v is None else v.to(dev).contiguous() for v in (gamma, beta, scale, shift)]
    y, c, cs = sba.sagesla_norm_quant(xd, kind, eps, *args, rows_per_sample=R,
                                      want_y=True, want_codes=codes)
    torch.cuda.synchronize()
    xr = _bf16(x)
    ref, ref_b = no.norm_forward(xr, kind, eps, *[None if v is None else _bf16(v) for v in
                                                  (gamma, beta, scale, shift)],
                                 rows_per_sample=max(R, 1))
    yg = _bf16(y)
    assert np.isfinite(yg).all()
    # within one bf16 ulp of the real result rounded to bf16, plus the fp32 rounding of terms
    # that cancel in the affine / modulation steps (and equal to it almost always)
    terms = _term_size(xr, kind, eps, *[None if v is None else _bf16(v) for v in
                                         (gamma, beta, scale, shift)], R)
    diff = np.abs(yg - ref_b)
    tol = _ulp_bf16(ref) + 4e-7 * terms
    assert np.all(diff <= tol), float(np.max(diff - tol))
    assert np.mean(yg == ref_b) > 0.99
    if codes:
        cg = c.cpu().numpy()
        sg = cs.cpu().numpy()
        for r in range(x.shape[0]):
            want_c, want_s = quant_int8_block(yg[r])      # the quantizer on the GPU's own row
            np.testing.assert_array_equal(cg[r], want_c)
            assert sg[r] == want_s
            err = np.abs(cg[r].astype(np.float64) * float(sg[r]) - ref[r])
            assert np.all(err <= 0.5 * float(sg[r]) * (1 + 1e-6) + 2 * _ulp_bf16(ref[r]) +
                          4e-7 * terms[r])
    return y


def _x(M, K, seed, spread=1.0, offset=0.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g) * spread + offset
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("M,K", [(300, 5120), (257, 1536), (64, 8), (33, 16384), (100, 1032),
                                 (37, 8192), (29, 8200), (5, 16)])
def test_layer_norm_with_modulation_and_codes(M, K):
    """K <= 8192 runs the one-warp-per-row kernel (8192: its largest shared-memory footprint),
    larger K the one-CTA-per-row kernel (8200: the first width past the boundary)."""
    g = torch.Generator().manual_seed(K)
    x = _x(M, K, M + K, spread=2.0, offset=0.3)
    R = max(1, M // 3)
    B = (M + R - 1) // R
    scale = (torch.randn(B, K, generator=g) * 0.2).to(torch.bfloat16)
    shift = (torch.randn(B, K, generator=g) * 0.5).to(torch.bfloat16)
    _check(x, sba.SAGESLA_LAYER_NORM, 1e-6, scale=scale, shift=shift, R=R)


def test_layer_norm_affine_and_rms_norm():
    g = torch.Generator().manual_seed(7)
    x = _x(129, 2048, 7, spread=4.0)
    gamma = (torch.randn(2048, generator=g)).to(torch.bfloat16)
    beta = (torch.randn(2048, generator=g)).to(torch.bfloat16)
    _check(x, sba.SAGESLA_LAYER_NORM, 1e-5, gamma=gamma, beta=beta)
    _check(x, sba.SAGESLA_RMS_NORM, 1e-6, gamma=gamma)
    _check(x, sba.SAGESLA_RMS_NORM, 1e-6, codes=False)


def test_strided_rows_and_special_rows():
    x = torch.zeros(6, 1024, dtype=torch.bfloat16)
    x[1] = 1.5                                   # constant row: LayerNorm gives zeros
    x[2, 5] = 3.0                                # one spike
    x[3] = _x(1, 1024, 3)[0] * 1e-3              # tiny values
    x[4] = _x(1, 1024, 4)[0] * 1e4               # large values
    x[5] = _x(1, 1024, 5)[0]
    y = _check(x, sba.SAGESLA_LAYER_NORM, 1e-6)
    assert torch.equal(y[1].float().cpu(), torch.zeros(1024))
    # the same rows inside a wider buffer (row stride 1536)
    wide = torch.zeros(6, 1536, dtype=torch.bfloat16)
    wide[:, :1024] = x
    y2, c2, s2 = sba.sagesla_norm_quant(wide.cuda()[:, :1024], sba.SAGESLA_LAYER_NORM, 1e-6,
                                        want_codes=True)
    assert torch.equal(y2.cpu(), y.cpu())


def test_wan_shape_sampled_rows():
    """Wan2.1-14B hidden size on a 720P token count (75600 x 5120), with per-sample AdaLN
    modulation; the oracle checks sampled rows."""
    M, K = 75600, 5120
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16)
    scale = (torch.randn(1, K, generator=g) * 0.2).to(torch.bfloat16)
    shift = (torch.randn(1, K, generator=g) * 0.5).to(torch.bfloat16)
    y, c, cs = sba.sagesla_norm_quant(x.cuda(), sba.SAGESLA_LAYER_NORM, 1e-6, None, None,
                                      scale.cuda(), shift.cuda(), rows_per_sample=M,
                                      want_codes=True)
    torch.cuda.synchronize()
    rows = [0, 1, 4097, M // 2, M - 2, M - 1]
    ref, ref_b = no.norm_forward(_bf16(x[rows]), no.LAYER_NORM, 1e-6, scale=_bf16(scale),
                                 shift=_bf16(shift), rows_per_sample=len(rows))
    yg = _bf16(y[rows])
    terms = _term_size(_bf16(x[rows]), no.LAYER_NORM, 1e-6, None, None, _bf16(scale),
                       _bf16(shift), len(rows))
    assert np.all(np.abs(yg - ref_b) <= _ulp_bf16(ref) + 4e-7 * terms)
    cg, sg = c[rows].cpu().numpy(), cs[rows].cpu().numpy()
    for i in range(len(rows)):
        want_c, want_s = quant_int8_block(yg[i])
        np.testing.assert_array_equal(cg[i], want_c)
        assert sg[i] == want_s
