"""The SLA backward entry point through the C ABI on the CPU: workspace sizing and argument
validation happen before any CUDA call (a valid call reaches the device check and, without a
GPU, returns SAGESLA_ERR_NO_DEVICE)."""
import ctypes

import pytest
import torch

from sparse_bit_attention_b200 import binding
from sparse_bit_attention_b200.build import build

INVALID, UNSUPPORTED, WORKSPACE, NO_DEVICE = 1, 2, 3, 7
BASE = 1 << 32          # fake, well-aligned device addresses (never dereferenced on the host)
B, H, N = 1, 2, 1000
SPAN = B * H * N * 128 * 4


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def _view(addr, dtype=binding.SAGESLA_BF16, **kw):
    v = dict(data=addr, dtype=dtype, B=B, H=H, N=N, D=128, stride_b=H * N * 128,
             stride_h=N * 128, stride_n=128)
    v.update(kw)
    return binding.SageslaTensor(*[v[n] for n, _ in binding.SageslaTensor._fields_])


def _call(lib, ratio=0.1, block=64, ws_bytes=None, ws=None, **over):
    t = {name: _view(BASE + i * SPAN) for i, name in enumerate(("q", "k", "v", "do"))}
    for i, name in enumerate(("dq", "dk", "dv")):
        t[name] = _view(BASE + (4 + i) * SPAN, binding.SAGESLA_F32)
    t.update(over)
    need = lib.sagesla_sla_backward_workspace_size(B, H, N, 128, ratio, block) or 1
    ws = BASE + 8 * SPAN if ws is None else ws
    return lib.sagesla_sla_backward(
        *[ctypes.byref(t[n]) for n in ("q", "k", "v", "do")], ratio, block,
        *[ctypes.byref(t[n]) for n in ("dq", "dk", "dv")], ctypes.c_void_p(ws),
        need if ws_bytes is None else ws_bytes, None)


def test_workspace_holds_the_forward_layout(lib):
    fwd = lib.sagesla_workspace_size(B, H, N, 128, 0.1, 64)
    bwd = lib.sagesla_sla_backward_workspace_size(B, H, N, 128, 0.1, 64)
    assert bwd > fwd > 0
    assert lib.sagesla_sla_backward_workspace_size(B, H, N, 64, 0.1, 64) == 0     # D != 128
    assert lib.sagesla_sla_backward_workspace_size(B, H, N, 128, 0.1, 32) == 0    # block != 64
    assert lib.sagesla_sla_backward_workspace_size(B, H, N, 128, 0.0, 64) == 0    # ratio
    # every block kept: no linear-branch regions
    dense = lib.sagesla_sla_backward_workspace_size(B, H, N, 128, 1.0, 64)
    assert fwd < dense < bwd


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="the fake addresses would be launched on a GPU")
def test_valid_arguments_reach_the_device_check(lib):
    assert _call(lib) == NO_DEVICE
    bf = {n: _view(BASE + (4 + i) * SPAN) for i, n in enumerate(("dq", "dk", "dv"))}
    assert _call(lib, **bf) == NO_DEVICE                          # bf16 gradients
    assert _call(lib, ratio=1.0) == NO_DEVICE


@pytest.mark.parametrize("case,expect", [
    ("q_f32", UNSUPPORTED), ("do_f32", UNSUPPORTED), ("mixed_grad_dtypes", UNSUPPORTED),
    ("block32", UNSUPPORTED), ("ratio0", INVALID), ("ratio_gt1", INVALID),
    ("shape_mismatch", INVALID), ("grad_shape_mismatch", INVALID), ("misaligned_row", INVALID),
    ("dq_overlaps_q", INVALID), ("dk_overlaps_dv", INVALID), ("grad_in_workspace", INVALID),
    ("small_workspace", WORKSPACE), ("unaligned_workspace", WORKSPACE), ("null_grad", INVALID),
])
def test_invalid_arguments(lib, case, expect):
    over, kw = {}, {}
    if case == "q_f32":
        over["q"] = _view(BASE, binding.SAGESLA_F32)
    elif case == "do_f32":
        over["do"] = _view(BASE + 3 * SPAN, binding.SAGESLA_F32)
    elif case == "mixed_grad_dtypes":
        over["dv"] = _view(BASE + 6 * SPAN, binding.SAGESLA_BF16)
    elif case == "block32":
        kw["block"] = 32
    elif case == "ratio0":
        kw["ratio"] = 0.0
    elif case == "ratio_gt1":
        kw["ratio"] = 1.5
    elif case == "shape_mismatch":
        over["v"] = _view(BASE + 2 * SPAN, N=N - 1)
    elif case == "grad_shape_mismatch":
        over["dk"] = _view(BASE + 5 * SPAN, binding.SAGESLA_F32, H=H - 1)
    elif case == "misaligned_row":
        over["k"] = _view(BASE + SPAN, stride_n=132)
    elif case == "dq_overlaps_q":
        over["dq"] = _view(BASE + 256, binding.SAGESLA_F32)
    elif case == "dk_overlaps_dv":
        over["dk"] = _view(BASE + 6 * SPAN + 512, binding.SAGESLA_F32)
    elif case == "grad_in_workspace":
        over["dv"] = _view(BASE + 8 * SPAN + 1024, binding.SAGESLA_F32)
    elif case == "small_workspace":
        kw["ws_bytes"] = 4096
    elif case == "unaligned_workspace":
        kw["ws"] = BASE + 8 * SPAN + 16
    elif case == "null_grad":
        over["dq"] = _view(0, binding.SAGESLA_F32)
    assert _call(lib, **kw, **over) == expect
