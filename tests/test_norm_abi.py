"""The fused-normalization entry point through the C ABI on the CPU: argument validation
happens before any CUDA call (a valid call reaches the device check and, without a GPU,
returns SAGESLA_ERR_NO_DEVICE)."""
import ctypes

import pytest
import torch

from sparse_bit_attention_b200 import binding
from sparse_bit_attention_b200.build import build

INVALID, UNSUPPORTED, NO_DEVICE = 1, 2, 7
BASE = 1 << 32          # fake, well-aligned device addresses (never dereferenced on the host)


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def _args(**kw):
    a = dict(x=BASE, M=4, K=64, x_stride=64, kind=0, eps=1e-6, gamma=None, beta=None,
             scale=None, shift=None, rows_per_sample=0, y=BASE + (1 << 20), y_stride=64,
             codes=None, codes_stride=64, code_scale=None)
    a.update(kw)
    return binding.SageslaNormArgs(*[a[n] for n, _ in binding.SageslaNormArgs._fields_])


def _call(lib, **kw):
    return lib.sagesla_norm_quant(ctypes.byref(_args(**kw)), None)


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="the fake addresses would be launched on a GPU")
def test_valid_arguments_reach_the_device_check(lib):
    assert _call(lib) == NO_DEVICE
    assert _call(lib, y=None, codes=BASE + (2 << 20), code_scale=BASE + (3 << 20)) == NO_DEVICE


@pytest.mark.parametrize("kw,expect", [
    (dict(K=12, x_stride=16, y_stride=16), UNSUPPORTED),        # K not a multiple of 8
    (dict(K=16392, x_stride=16392, y_stride=16392), UNSUPPORTED),  # K above 16384
    (dict(K=0), INVALID),
    (dict(M=0), INVALID),
    (dict(kind=3), INVALID),
    (dict(kind=2, gamma=BASE + (4 << 20)), INVALID),              # no weight without a norm
    (dict(eps=-1.0), INVALID),
    (dict(eps=float("nan")), INVALID),
    (dict(kind=1, beta=BASE + (4 << 20)), INVALID),              # beta is LayerNorm only
    (dict(y=None), INVALID),                                     # no output
    (dict(codes=BASE + (2 << 20)), INVALID),                     # codes without scales
    (dict(code_scale=BASE + (3 << 20)), INVALID),                # scales without codes
    (dict(scale=BASE + (4 << 20)), INVALID),                     # modulation without R
    (dict(x_stride=60), INVALID),                                # stride below K
    (dict(x_stride=68), INVALID),                                # rows not 16-byte aligned
    (dict(x=BASE + 8), INVALID),                                 # base not 16-byte aligned
    (dict(gamma=BASE + (4 << 20) + 2), INVALID),
    (dict(y=BASE + 64), INVALID),                                # output overlaps the input
])
def test_bad_arguments_are_rejected_before_launch(lib, kw, expect):
    assert _call(lib, **kw) == expect


def test_null_argument_block(lib):
    assert lib.sagesla_norm_quant(None, None) == INVALID


W8 = (
    dict(x8=BASE, x_scale=BASE + (1 << 20), M=256, K=512, w8=BASE + (2 << 20),
         w_scale=BASE + (3 << 20), N=256, bias=None, y=BASE + (4 << 20), y_dtype=0,
         y_stride=256, status=None)
)
_W8_ORDER = ["x8", "x_scale", "M", "K", "w8", "w_scale", "N", "bias", "y", "y_dtype",
             "y_stride", "status"]


def _gemm(lib, **kw):
    a = dict(W8)
    a.update(kw)
    return lib.sagesla_w8a8_gemm(*[a[n] for n in _W8_ORDER], None)


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="the fake addresses would be launched on a GPU")
def test_w8a8_valid_arguments_reach_the_device_check(lib):
    assert _gemm(lib) == NO_DEVICE
    assert lib.sagesla_w8a8_quantize_weight(BASE, 256, 512, 512, BASE + (2 << 20),
                                            BASE + (3 << 20), None) == NO_DEVICE


@pytest.mark.parametrize("kw,expect", [
    (dict(K=500), UNSUPPORTED),             # K not a multiple of 128
    (dict(N=250, y_stride=256), UNSUPPORTED),  # N not a multiple of 8
    (dict(M=0), INVALID),
    (dict(y_dtype=5), INVALID),
    (dict(y_stride=255), INVALID),          # stride below N
    (dict(y_dtype=1, y_stride=258), INVALID),  # f32 rows not 16-byte aligned
    (dict(x8=BASE + 8), INVALID),
    (dict(bias=BASE + (5 << 20) + 2), INVALID),
    (dict(y=BASE + 64), INVALID),           # output overlaps x8
    (dict(x_scale=None), INVALID),
])
def test_w8a8_bad_arguments_are_rejected_before_launch(lib, kw, expect):
    assert _gemm(lib, **kw) == expect


def test_w8a8_weight_quantizer_validation(lib):
    assert lib.sagesla_w8a8_quantize_weight(BASE, 256, 500, 504, BASE + (2 << 20),
                                            BASE + (3 << 20), None) == UNSUPPORTED
    assert lib.sagesla_w8a8_quantize_weight(BASE, 256, 512, 510, BASE + (2 << 20),
                                            BASE + (3 << 20), None) == INVALID
    assert lib.sagesla_w8a8_quantize_weight(None, 256, 512, 512, BASE + (2 << 20),
                                            BASE + (3 << 20), None) == INVALID
