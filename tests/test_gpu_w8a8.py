"""GPU parity of the W8A8 linear layer (through the C ABI) against the CPU oracle: weight
codes and block scales bit-exact; the GEMM within 1e-5 of the size of its block terms (plus a
bf16 ulp for bf16 output). The GEMM is fed the oracle's own codes, so it is checked alone."""
import numpy as np
import pytest
import torch

import sparse_bit_attention_b200 as sba
from oracle import norm_oracle as no
from oracle import w8a8_oracle as wo

pytestmark = pytest.mark.gpu


def _ulp_bf16(v):
    a = np.abs(v)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    return np.ldexp(1.0, np.maximum(e - 8, -133))


def _operands(M, K, N, seed, w_std=0.05):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * w_std).to(torch.bfloat16)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    return x, w, bias


@pytest.mark.parametrize("N,K", [(300, 384), (128, 128), (5120, 1536), (8, 256)])
def test_weight_quantizer_bit_exact(N, K):
    _, w, _ = _operands(1, K, N, N + K)
    w8, ws = sba.sagesla_w8a8_quantize_weight(w.cuda())
    torch.cuda.synchronize()
    ref_c, ref_s = wo.quantize_weight_blocks(w.double().numpy())
    np.testing.assert_array_equal(w8.cpu().numpy(), ref_c)
    np.testing.assert_array_equal(ws.cpu().numpy(), ref_s)


def _gemm_check(M, K, N, seed, out_dtype, with_bias, rows=None):
    x, w, bias = _operands(M, K, N, seed)
    _, xb = no.norm_forward(x.double().numpy(), no.NO_NORM, 0.0)
    x8, s_x = no.quant_rows_int8(xb)
    w8, s_w = wo.quantize_weight_blocks(w.double().numpy())
    dev = torch.device("cuda:0")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y = sba.sagesla_w8a8_gemm(torch.from_numpy(x8).to(dev), torch.from_numpy(s_x).to(dev),
                              torch.from_numpy(w8).to(dev), torch.from_numpy(s_w).to(dev),
                              bias.to(dev) if with_bias else None, out_dtype=out_dtype,
                              status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = list(range(M)) if rows is None else rows
    ref, t = wo.w8a8_linear(x8[rows], s_x[rows], w8, s_w,
                            bias.double().numpy() if with_bias else None)
    got = y[rows].double().cpu().numpy()
    assert np.isfinite(got).all()
    tol = 1e-5 * t + (_ulp_bf16(ref) if out_dtype == torch.bfloat16 else 0.0) + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= tol), float(np.max(err - tol))
    return y


@pytest.mark.parametrize("M,K,N", [(300, 512, 256), (129, 1536, 384), (1000, 256, 8),
                                   (64, 5120, 5120)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_matches_oracle(M, K, N, out_dtype):
    _gemm_check(M, K, N, M + K + N, out_dtype, with_bias=(N != 8))


def test_gemm_wan_shape_sampled_rows():
    """The 14B-720P token rows through a 5120 x 5120 projection, sampled rows checked."""
    M = 75600
    rows = [0, 1, 127, 128, 37799, 75470, 75599]
    _gemm_check(M, 5120, 5120, 7, torch.bfloat16, with_bias=True, rows=rows)


def test_quantized_layer_tracks_the_bf16_layer():
    """End to end on the GPU (per-token codes from sagesla_norm_quant, block-quantized
    weights): within the 8-bit error of the plain bf16 layer."""
    x, w, bias = _operands(512, 1024, 512, 9)
    dev = torch.device("cuda:0")
    _, x8, s_x = sba.sagesla_norm_quant(x.to(dev), sba.SAGESLA_NO_NORM, 0.0, want_y=False,
                                        want_codes=True)
    w8, s_w = sba.sagesla_w8a8_quantize_weight(w.to(dev))
    y = sba.sagesla_w8a8_gemm(x8, s_x, w8, s_w, bias.to(dev), out_dtype=torch.float32)
    ref = x.double() @ w.double().T + bias.double()
    rel = (y.double().cpu() - ref).norm() / ref.norm()
    assert rel < 0.02, float(rel)
