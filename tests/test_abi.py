"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest
import torch

import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import binding
from sparse_bit_attention_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build()
    return binding.load_library()


def _header_functions():
    text = open(os.path.join(ROOT, "include", "sagesla.h")).read()
    return sorted(set(re.findall(r"\b(sagesla_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    lib = binding.load_library()
    declared = _header_functions()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(binding.exported_symbols()) == declared


def test_topk_count_matches_definition():
    assert sba.sagesla_topk_count(1024, 0.1) == 2
    assert sba.sagesla_topk_count(75600, 0.1) == 119
    assert sba.sagesla_topk_count(75600, 0.05) == 60
    assert sba.sagesla_topk_count(75600, 0.15) == 178
    assert sba.sagesla_topk_count(640, 0.3) == 3
    assert sba.sagesla_topk_count(10, 1.0) == 1
    assert sba.sagesla_topk_count(1024, 0.0) == -1
    assert sba.sagesla_topk_count(1024, 1.5) == -1
    assert sba.sagesla_topk_count(1024, float("nan")) == -1
    assert sba.sagesla_topk_count(1024, 0.1, block=128) == -1


def test_workspace_layout_is_consistent():
    for (B, H, N, r) in [(1, 2, 1024, 0.1), (1, 40, 75600, 0.1), (2, 3, 1025, 1.0), (1, 1, 1, 0.5)]:
        lay = sba.sagesla_get_workspace_layout(B, H, N, 128, r)
        nb = (N + 63) // 64
        assert lay["nb"] == nb and lay["k"] == sba.sagesla_topk_count(N, r)
        assert lay["n_pad"] == 128 * ((nb + 1) // 2)
        offs = sorted(lay[f] for f in binding._LAYOUT_FIELDS)
        assert offs[0] == 0 and all(o % 256 == 0 for o in offs)
        assert len(set(offs)) == len(offs)
        assert lay["total_bytes"] >= offs[-1]
        assert sba.sagesla_workspace_size(B, H, N, 128, r) == lay["total_bytes"]
    with pytest.raises(sba.SageslaError) as e:
        sba.sagesla_get_workspace_layout(1, 1, 100, 64, 0.1)
    assert e.value.status == 2
    assert sba.sagesla_workspace_size(1, 1, 100, 128, 0.1, 32) == 0


def _t(shape=(1, 2, 256, 128), dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def _call(q, k, v, out, ratio=0.1, block=64, ws_bytes=None, ws_ptr=None):
    lib = binding.load_library()
    vq, vk, vv, vo = (binding._view(x) for x in (q, k, v, out))
    B, H, N, D = q.shape
    need = lib.sagesla_workspace_size(B, H, N, D, ratio, block)
    buf = torch.zeros(need + 512, dtype=torch.uint8)
    ptr = ws_ptr if ws_ptr is not None else (buf.data_ptr() + 255) // 256 * 256
    return lib.sagesla_forward(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), ratio, block,
                               ctypes.byref(vo), ctypes.c_void_p(ptr),
                               need if ws_bytes is None else ws_bytes, None)


def test_validation_rejects_bad_arguments_before_launch():
    q, k, v = _t(), _t(), _t()
    out = _t(dtype=torch.float32)
    # well-formed call on a machine without an sm_100 device: NO_DEVICE, nothing launched
    st = _call(q, k, v, out)
    assert st in (0, 7)
    if st == 0:
        pytest.skip("a B200 is present; the no-device path is not reachable here")
    assert _call(q, k, v, out, ratio=0.0) == 1
    assert _call(q, k, v, out, ratio=1.01) == 1
    assert _call(q, k, v, out, block=128) == 2
    assert _call(_t((1, 2, 256, 64)), _t((1, 2, 256, 64)), _t((1, 2, 256, 64)),
                 _t((1, 2, 256, 64), torch.float32)) == 2
    # an output dtype code the library does not know
    lib = binding.load_library()
    vq, vo = binding._view(q), binding._view(out)
    vo.dtype = 7
    ws = torch.zeros(lib.sagesla_workspace_size(1, 2, 256, 128, 0.1, 64) + 512, dtype=torch.uint8)
    assert lib.sagesla_forward(ctypes.byref(vq), ctypes.byref(vq), ctypes.byref(vq), 0.1, 64,
                               ctypes.byref(vo), ctypes.c_void_p((ws.data_ptr() + 255) // 256 * 256),
                               ws.numel() - 512, None) == 2
    assert _call(q, _t((1, 2, 255, 128)), v, out) == 1              # shape mismatch
    assert _call(q, k, v, out, ws_bytes=16) == 3                     # workspace too small
    assert _call(q, k, v, out, ws_ptr=0) == 3                        # no workspace
    # misaligned rows: stride_n of 120 + 8 elements = 256 B ok; data offset by 2 B is not
    qm = torch.zeros(1 * 2 * 256 * 128 + 8, dtype=torch.bfloat16)[1:1 + 2 * 256 * 128].view(1, 2, 256, 128)
    assert _call(qm, k, v, out) == 1
    # output aliasing an input
    assert _call(q, k, v, q) == 1
    # null tensor
    assert lib.sagesla_forward(None, ctypes.byref(vq), ctypes.byref(vq), 0.1, 64,
                               ctypes.byref(vq), None, 0, None) == 1


def test_status_strings():
    for s in range(10):
        assert sba.sagesla_status_string(s) != "unknown status"
        assert s in binding.STATUS_NAMES
    assert sba.sagesla_status_string(99) == "unknown status"


def test_host_entry_rejects_bad_arguments():
    lib = binding.load_library()
    q = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    o = torch.zeros(1, 1, 64, 128)
    assert lib.sagesla_forward_host(None, None, None, 1, 1, 64, 128, 0.1, 64, None, 1, None, 0,
                                    None) == 1
    p = ctypes.c_void_p(q.data_ptr())
    assert lib.sagesla_forward_host(p, p, p, 1, 1, 64, 64, 0.1, 64, ctypes.c_void_p(o.data_ptr()),
                                    1, None, 0, None) == 2
    assert lib.sagesla_forward_host(p, p, p, 1, 1, 64, 128, 0.1, 64, ctypes.c_void_p(o.data_ptr()),
                                    1, None, 0, None) == 3


def test_operand_modes_workspace_and_validation():
    """The 16-bit modes add bf16 copies of their operands to the workspace (Q and K for
    quant = 0, V for pv_fp8 = 0); bf16 Q.K^T with e4m3 P.V is not a mode."""
    B, H, N = 1, 3, 1000
    base = sba.sagesla_workspace_size(B, H, N, 128, 0.2)
    n_pad = sba.sagesla_get_workspace_layout(B, H, N, 128, 0.2)["n_pad"]
    copy = B * H * n_pad * 256
    lay_v = sba.sagesla_get_workspace_layout(B, H, N, 128, 0.2, pv_fp8=False)
    lay_qkv = sba.sagesla_get_workspace_layout(B, H, N, 128, 0.2, quant=False, pv_fp8=False)
    assert lay_v["qb"] == 0 and lay_v["kb"] == 0 and lay_v["vb"] >= base
    assert lay_v["total_bytes"] >= base + copy
    assert min(lay_qkv["qb"], lay_qkv["kb"], lay_qkv["vb"]) >= base
    assert lay_qkv["total_bytes"] >= base + 3 * copy
    assert all(lay_qkv[f] % 256 == 0 for f in ("qb", "kb", "vb"))
    assert sba.sagesla_workspace_size(B, H, N, 128, 0.2, quant=False, pv_fp8=False) == lay_qkv["total_bytes"]
    lib = binding.load_library()
    opt = binding._options(quant=False, pv_fp8=True)
    assert lib.sagesla_workspace_size_ex(B, H, N, 128, 0.2, 64, ctypes.byref(opt)) == 0
    lay = binding.SageslaWorkspaceLayout()
    assert lib.sagesla_get_workspace_layout_ex(B, H, N, 128, 0.2, 64, ctypes.byref(opt),
                                               ctypes.byref(lay)) == 2     # UNSUPPORTED
    opt = binding._options()
    opt.quant = 3
    assert lib.sagesla_get_workspace_layout_ex(B, H, N, 128, 0.2, 64, ctypes.byref(opt),
                                               ctypes.byref(lay)) == 1     # INVALID_ARG


def test_options_init_defaults():
    opt = binding.SageslaOptions()
    opt.debug_skip_tile = 7
    binding.load_library().sagesla_options_init(ctypes.byref(opt))
    assert opt.quant == 1 and opt.pv_fp8 == 1 and opt.debug_skip_tile == 0
    assert not opt.kept_idx_out and not opt.stage_events
