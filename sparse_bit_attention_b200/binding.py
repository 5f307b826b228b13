"""Thin ctypes binding of libsagesla.so: the same entry points as include/sagesla.h.

Argument marshalling only — every step of the forward runs in the library's CUDA kernels.
PyTorch provides device memory and streams. There is no fallback: if the library is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsagesla.so")
# the bounds-checking build of the same sources (SAGESLA_CHECKS=1)
LIB_CHECKS_PATH = os.path.join(_PKG, "libsagesla_checks.so")

SAGESLA_BF16 = 0
SAGESLA_F32 = 1
BLOCK = 64
HEAD_DIM = 128

STATUS_NAMES = {
    0: "SAGESLA_OK", 1: "SAGESLA_ERR_INVALID_ARG", 2: "SAGESLA_ERR_UNSUPPORTED",
    3: "SAGESLA_ERR_WORKSPACE", 4: "SAGESLA_ERR_CUDA", 5: "SAGESLA_ERR_TIMEOUT",
    6: "SAGESLA_ERR_DEVICE_CHECK", 7: "SAGESLA_ERR_NO_DEVICE", 8: "SAGESLA_ERR_BOUNDS",
    9: "SAGESLA_ERR_CANARY",
}


class SageslaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} "
                         f"({sagesla_status_string(status)})")


class SageslaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64),
                ("D", ctypes.c_int64), ("stride_b", ctypes.c_int64),
                ("stride_h", ctypes.c_int64), ("stride_n", ctypes.c_int64)]


N_STAGES = 7
STAGE_NAMES = ["stats", "finalize", "quant", "scores", "topk", "complement_gemm", "attention"]


class SageslaOptions(ctypes.Structure):
    _fields_ = [("kept_idx_out", ctypes.c_void_p), ("mask_out", ctypes.c_void_p),
                ("scores_out", ctypes.c_void_p), ("sparse_out", ctypes.c_void_p),
                ("stage_events", ctypes.POINTER(ctypes.c_void_p)),
                ("debug_spin_limit_us", ctypes.c_uint32), ("debug_skip_tile", ctypes.c_int32),
                ("quant", ctypes.c_int32), ("pv_fp8", ctypes.c_int32),
                ("debug_checks", ctypes.c_int32), ("debug_plant", ctypes.c_int32)]


def _options(quant: bool = True, pv_fp8: bool = True) -> SageslaOptions:
    opt = SageslaOptions()
    load_library().sagesla_options_init(ctypes.byref(opt))
    opt.quant = 1 if quant else 0
    opt.pv_fp8 = 1 if pv_fp8 else 0
    return opt


_LAYOUT_FIELDS = ["status", "q8", "k8", "v8", "sq", "sk", "s_v", "inv_v", "mu", "qbar", "kbar",
                  "ksum_part", "vmax_part", "scores", "kept", "mask", "amask", "hflat", "gsum"]


# bf16 operand copies of the 16-bit modes (offset 0 when absent)
_MODE_LAYOUT_FIELDS = ["qb", "kb", "vb"]


class SageslaWorkspaceLayout(ctypes.Structure):
    _fields_ = ([("total_bytes", ctypes.c_size_t)] +
                [(n, ctypes.c_int64) for n in
                 ("nb", "k", "n_pad", "mask_words", "nb_k_pad", "nb_m_pad")] +
                [(n, ctypes.c_size_t) for n in _LAYOUT_FIELDS + _MODE_LAYOUT_FIELDS])


SAGESLA_LAYER_NORM = 0
SAGESLA_RMS_NORM = 1
SAGESLA_NO_NORM = 2
W8A8_BLOCK = 128


class SageslaNormArgs(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("M", ctypes.c_int64), ("K", ctypes.c_int64),
                ("x_stride", ctypes.c_int64), ("kind", ctypes.c_int32), ("eps", ctypes.c_float),
                ("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("shift", ctypes.c_void_p), ("rows_per_sample", ctypes.c_int64),
                ("y", ctypes.c_void_p), ("y_stride", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("codes_stride", ctypes.c_int64), ("code_scale", ctypes.c_void_p)]


# Every symbol the header declares, with its signature.
_SIGNATURES = {
    "sagesla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sagesla_topk_count": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_double, ctypes.c_int]),
    "sagesla_workspace_size": (ctypes.c_size_t, [ctypes.c_int64] * 4 + [ctypes.c_double, ctypes.c_int]),
    "sagesla_get_workspace_layout": (ctypes.c_int, [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int, ctypes.POINTER(SageslaWorkspaceLayout)]),
    "sagesla_options_init": (None, [ctypes.c_void_p]),
    "sagesla_build_checks": (ctypes.c_int, []),
    "sagesla_workspace_size_ex": (ctypes.c_size_t, [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p]),
    "sagesla_get_workspace_layout_ex": (ctypes.c_int, [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.POINTER(SageslaWorkspaceLayout)]),
    "sagesla_forward": (ctypes.c_int, [ctypes.POINTER(SageslaTensor)] * 3 + [
        ctypes.c_double, ctypes.c_int, ctypes.POINTER(SageslaTensor), ctypes.c_void_p,
        ctypes.c_size_t, ctypes.c_void_p]),
    "sagesla_forward_ex": (ctypes.c_int, [ctypes.POINTER(SageslaTensor)] * 3 + [
        ctypes.c_double, ctypes.c_int, ctypes.POINTER(SageslaTensor), ctypes.c_void_p,
        ctypes.c_size_t, ctypes.c_void_p, ctypes.POINTER(SageslaOptions)]),
    "sagesla_host_workspace_size": (ctypes.c_size_t, [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_int32]),
    "sagesla_forward_host": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
        ctypes.c_size_t, ctypes.c_void_p]),
    "sagesla_stream_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "sagesla_forward_no_alloc": (ctypes.c_int, [ctypes.POINTER(SageslaTensor)] * 3 + [
        ctypes.c_double, ctypes.c_int, ctypes.POINTER(SageslaTensor), ctypes.c_void_p]),
    "sagesla_norm_quant": (ctypes.c_int, [ctypes.POINTER(SageslaNormArgs), ctypes.c_void_p]),
    "sagesla_w8a8_quantize_weight": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                    ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_void_p]),
    "sagesla_sla_backward_workspace_size": (ctypes.c_size_t, [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int]),
    "sagesla_sla_backward": (ctypes.c_int, [ctypes.POINTER(SageslaTensor)] * 4 + [
        ctypes.c_double, ctypes.c_int] + [ctypes.POINTER(SageslaTensor)] * 3 + [
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "sagesla_w8a8_gemm": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                         ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_void_p]),
}

NO_ALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


def _open(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m sparse_bit_attention_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libsagesla.so (built by ``python -m sparse_bit_attention_b200.build``); every
    call of this module goes to it (see ``using_library`` for another build)."""
    global _lib
    if _lib is None:
        _lib = _open(path)
    return _lib


_checks_lib = None


def load_checks_library() -> ctypes.CDLL:
    """Loads the bounds-checking build libsagesla_checks.so (``python -m
    sparse_bit_attention_b200.build --checks``) beside the normal one."""
    global _checks_lib
    if _checks_lib is None:
        _checks_lib = _open(LIB_CHECKS_PATH)
    return _checks_lib


@contextlib.contextmanager
def using_library(lib: ctypes.CDLL):
    """Routes this module's calls to ``lib`` (e.g. the checking build) inside the block."""
    global _lib
    prev = load_library()
    _lib = lib
    try:
        yield lib
    finally:
        _lib = prev


def exported_symbols() -> list[str]:
    return list(_SIGNATURES)


def _check(status: int, where: str):
    if status != 0:
        raise SageslaError(status, where)


def _view(t: torch.Tensor) -> SageslaTensor:
    if t.dim() != 4:
        raise ValueError("expected a [B, H, N, D] tensor")
    if t.stride(3) != 1:
        raise ValueError("the head dimension must be contiguous")
    dt = {torch.bfloat16: SAGESLA_BF16, torch.float32: SAGESLA_F32}.get(t.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {t.dtype}")
    B, H, N, D = t.shape
    return SageslaTensor(t.data_ptr(), dt, B, H, N, D, t.stride(0), t.stride(1), t.stride(2))


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def sagesla_status_string(status: int) -> str:
    return load_library().sagesla_status_string(int(status)).decode()


def sagesla_topk_count(N: int, topk_ratio: float, block: int = BLOCK) -> int:
    return int(load_library().sagesla_topk_count(N, float(topk_ratio), block))


def sagesla_workspace_size(B: int, H: int, N: int, D: int = HEAD_DIM, topk_ratio: float = 0.1,
                           block: int = BLOCK, quant: bool = True, pv_fp8: bool = True) -> int:
    if quant and pv_fp8:
        return int(load_library().sagesla_workspace_size(B, H, N, D, float(topk_ratio), block))
    opt = _options(quant, pv_fp8)
    return int(load_library().sagesla_workspace_size_ex(B, H, N, D, float(topk_ratio), block,
                                                        ctypes.byref(opt)))


def sagesla_get_workspace_layout(B: int, H: int, N: int, D: int = HEAD_DIM,
                                 topk_ratio: float = 0.1, block: int = BLOCK,
                                 quant: bool = True, pv_fp8: bool = True) -> dict:
    lay = SageslaWorkspaceLayout()
    opt = _options(quant, pv_fp8)
    _check(load_library().sagesla_get_workspace_layout_ex(B, H, N, D, float(topk_ratio), block,
                                                          ctypes.byref(opt), ctypes.byref(lay)),
           "sagesla_get_workspace_layout_ex")
    return {name: getattr(lay, name) for name, _ in SageslaWorkspaceLayout._fields_}


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A device byte buffer for the workspace (the caching allocator returns 512-byte-aligned
    blocks, above the library's 256-byte requirement)."""
    ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")
    assert ws.data_ptr() % 256 == 0
    return ws


def sagesla_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, topk_ratio: float = 0.1,
                    block: int = BLOCK, out: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None,
                    out_dtype: torch.dtype = torch.float32, kept_idx_out=None, mask_out=None,
                    scores_out=None, sparse_out=None, stage_events=None,
                    debug_spin_limit_us: int = 0, debug_skip_tile: bool = False,
                    quant: bool = True, pv_fp8: bool = True, debug_checks: bool = False,
                    debug_plant: int = 0) -> torch.Tensor:
    """SageSLA forward on device tensors q, k, v (bf16 [B, H, N, 128]); returns ``out``.

    ``stage_events``: optional list of N_STAGES + 1 torch.cuda.Event(enable_timing=True)
    recorded around each kernel of the forward on the launching stream.
    ``debug_spin_limit_us`` / ``debug_skip_tile``: the failure-path test hooks of
    sagesla_options (0 / False in normal use). ``quant`` / ``pv_fp8``: the operand mode
    (INT8 Q.K^T / e4m3 P.V by default; False selects bf16). ``debug_checks``: workspace
    canaries written before and verified after the call (the result lands in the status word:
    ``sagesla_stream_status``); ``debug_plant``: host-side fault injection of the failure-path
    tests (1: a damaged canary, 2: an out-of-range kept index, checking build only)."""
    lib = load_library()
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    B, H, N, D = q.shape
    need = sagesla_workspace_size(B, H, N, D, topk_ratio, block, quant, pv_fp8)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    extra = (kept_idx_out, mask_out, scores_out, sparse_out)
    args = (ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), float(topk_ratio), int(block),
            ctypes.byref(vo), ctypes.c_void_p(workspace.data_ptr()),
            workspace.numel() * workspace.element_size(), ctypes.c_void_p(_stream_ptr(stream)))
    if (any(x is not None for x in extra) or stage_events is not None or debug_spin_limit_us
            or debug_skip_tile or not quant or not pv_fp8 or debug_checks or debug_plant):
        opt = _options(quant, pv_fp8)
        opt.debug_checks = 1 if debug_checks else 0
        opt.debug_plant = int(debug_plant)
        for name, x in zip(("kept_idx_out", "mask_out", "scores_out", "sparse_out"), extra):
            if x is not None:
                setattr(opt, name, x.data_ptr())
        opt.debug_spin_limit_us = int(debug_spin_limit_us)
        opt.debug_skip_tile = 1 if debug_skip_tile else 0
        if stage_events is not None:
            if len(stage_events) != N_STAGES + 1:
                raise ValueError(f"stage_events needs {N_STAGES + 1} events")
            for e in stage_events:          # torch creates the CUDA event on first record
                if e.cuda_event == 0:
                    e.record()
            handles = (ctypes.c_void_p * (N_STAGES + 1))(*[e.cuda_event for e in stage_events])
            opt.stage_events = ctypes.cast(handles, ctypes.POINTER(ctypes.c_void_p))
        _check(lib.sagesla_forward_ex(*args, ctypes.byref(opt)), "sagesla_forward_ex")
    else:
        _check(lib.sagesla_forward(*args), "sagesla_forward")
    return out


def sagesla_host_workspace_size(B: int, H: int, N: int, D: int = HEAD_DIM,
                                topk_ratio: float = 0.1, block: int = BLOCK,
                                out_dtype: int = SAGESLA_F32) -> int:
    return int(load_library().sagesla_host_workspace_size(B, H, N, D, float(topk_ratio), block,
                                                          int(out_dtype)))


def sagesla_forward_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                         out_host: torch.Tensor, topk_ratio: float = 0.1, block: int = BLOCK,
                         workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Forward on contiguous CPU tensors (pinned memory gives asynchronous copies): copies in,
    runs, copies out and synchronizes the stream."""
    lib = load_library()
    for t in (q_host, k_host, v_host, out_host):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors")
    B, H, N, D = q_host.shape
    odt = SAGESLA_F32 if out_host.dtype == torch.float32 else SAGESLA_BF16
    need = sagesla_host_workspace_size(B, H, N, D, topk_ratio, block, odt)
    if workspace is None:
        workspace = alloc_workspace(need)
    _check(lib.sagesla_forward_host(
        ctypes.c_void_p(q_host.data_ptr()), ctypes.c_void_p(k_host.data_ptr()),
        ctypes.c_void_p(v_host.data_ptr()), B, H, N, D, float(topk_ratio), int(block),
        ctypes.c_void_p(out_host.data_ptr()), odt, ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel(), ctypes.c_void_p(_stream_ptr(stream))), "sagesla_forward_host")
    return out_host


def sagesla_sla_backward_workspace_size(B: int, H: int, N: int, D: int = HEAD_DIM,
                                        topk_ratio: float = 0.1, block: int = BLOCK) -> int:
    return int(load_library().sagesla_sla_backward_workspace_size(B, H, N, D, float(topk_ratio),
                                                                  block))


def sagesla_sla_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, d_out: torch.Tensor,
                         topk_ratio: float = 0.1, block: int = BLOCK, dq=None, dk=None, dv=None,
                         grad_dtype: torch.dtype = torch.float32,
                         workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq, dk, dv) of sum(O * d_out) for the unquantized SLA forward (the block
    selection held fixed); q, k, v, d_out bf16 [B, H, N, 128] on the device."""
    lib = load_library()
    B, H, N, D = q.shape
    dq = torch.empty(q.shape, dtype=grad_dtype, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=dq.dtype, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=dq.dtype, device=q.device) if dv is None else dv
    need = sagesla_sla_backward_workspace_size(B, H, N, D, topk_ratio, block)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    views = [_view(x) for x in (q, k, v, d_out, dq, dk, dv)]
    _check(lib.sagesla_sla_backward(
        *[ctypes.byref(x) for x in views[:4]], float(topk_ratio), int(block),
        *[ctypes.byref(x) for x in views[4:]], ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), ctypes.c_void_p(_stream_ptr(stream))),
        "sagesla_sla_backward")
    return dq, dk, dv


def sagesla_stream_status(stream=None, workspace: torch.Tensor | None = None) -> int:
    """Synchronizes the stream and returns (and clears) the workspace's device status word."""
    wp = None if workspace is None else ctypes.c_void_p(workspace.data_ptr())
    return int(load_library().sagesla_stream_status(ctypes.c_void_p(_stream_ptr(stream)), wp))


def sagesla_forward_no_alloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                             topk_ratio: float = 0.1, block: int = BLOCK, stream=None) -> torch.Tensor:
    """Forward for callers that cannot allocate device memory: the library's built-in scratch
    area replaces the workspace (problems needing more than NO_ALLOC_SCRATCH_BYTES raise).
    Calls whose GPU work overlaps race on that shared area."""
    lib = load_library()
    vq, vk, vv, vo = _view(q), _view(k), _view(v), _view(out)
    _check(lib.sagesla_forward_no_alloc(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv),
                                        float(topk_ratio), int(block), ctypes.byref(vo),
                                        ctypes.c_void_p(_stream_ptr(stream))),
           "sagesla_forward_no_alloc")
    return out


def _ptr(t):
    return None if t is None else t.data_ptr()


def sagesla_norm_quant(x: torch.Tensor, kind: int = SAGESLA_LAYER_NORM, eps: float = 1e-6,
                       gamma=None, beta=None, scale=None, shift=None, rows_per_sample: int = 0,
                       want_y: bool = True, want_codes: bool = False, stream=None):
    """Fused LayerNorm / RMSNorm (+ modulation) of the rows of a bf16 [M, K] device tensor
    (last dimension contiguous). Returns (y bf16 [M, K] or None, codes int8 [M, K] or None,
    code_scale float32 [M] or None)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with contiguous rows")
    M, K = x.shape
    y = torch.empty((M, K), dtype=torch.bfloat16, device=x.device) if want_y else None
    codes = torch.empty((M, K), dtype=torch.int8, device=x.device) if want_codes else None
    cs = torch.empty((M,), dtype=torch.float32, device=x.device) if want_codes else None
    for v in (gamma, beta, scale, shift):
        if v is not None and (v.dtype != torch.bfloat16 or not v.is_contiguous()):
            raise ValueError("gamma, beta, scale, shift must be contiguous bf16 tensors")
    args = SageslaNormArgs(x.data_ptr(), M, K, x.stride(0), kind, eps, _ptr(gamma), _ptr(beta),
                           _ptr(scale), _ptr(shift), rows_per_sample, _ptr(y), K, _ptr(codes), K,
                           _ptr(cs))
    _check(load_library().sagesla_norm_quant(ctypes.byref(args),
                                             ctypes.c_void_p(_stream_ptr(stream))),
           "sagesla_norm_quant")
    return y, codes, cs


def sagesla_w8a8_quantize_weight(w: torch.Tensor, stream=None):
    """Block-wise (128 x 128) INT8 quantization of a bf16 [N, K] weight (rows contiguous).
    Returns (w8 int8 [N, K], w_scale float32 [ceil(N/128), K/128])."""
    if w.dtype != torch.bfloat16 or w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a bf16 [N, K] tensor with contiguous rows")
    N, K = w.shape
    w8 = torch.empty((N, K), dtype=torch.int8, device=w.device)
    ws = torch.empty(((N + W8A8_BLOCK - 1) // W8A8_BLOCK, K // W8A8_BLOCK), dtype=torch.float32,
                     device=w.device)
    _check(load_library().sagesla_w8a8_quantize_weight(
        ctypes.c_void_p(w.data_ptr()), N, K, w.stride(0), ctypes.c_void_p(w8.data_ptr()),
        ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(_stream_ptr(stream))),
        "sagesla_w8a8_quantize_weight")
    return w8, ws


def sagesla_w8a8_gemm(x8: torch.Tensor, x_scale: torch.Tensor, w8: torch.Tensor,
                      w_scale: torch.Tensor, bias=None, out_dtype=torch.bfloat16, out=None,
                      status=None, stream=None):
    """y[m, n] = x_scale[m] * sum_bk w_scale[n/128, bk] * (x8[m, block bk] . w8[n, block bk])
    (+ bias[n]) on the INT8 tensor cores; x8 [M, K] and w8 [N, K] contiguous int8."""
    M, K = x8.shape
    N = w8.shape[0]
    for t, dt in ((x8, torch.int8), (w8, torch.int8), (x_scale, torch.float32),
                  (w_scale, torch.float32)):
        if t.dtype != dt or not t.is_contiguous():
            raise ValueError("x8, w8 (int8) and x_scale, w_scale (float32) must be contiguous")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 vector")
    y_dtype = SAGESLA_F32 if out_dtype == torch.float32 else SAGESLA_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x8.device)
    _check(load_library().sagesla_w8a8_gemm(
        ctypes.c_void_p(x8.data_ptr()), ctypes.c_void_p(x_scale.data_ptr()), M, K,
        ctypes.c_void_p(w8.data_ptr()), ctypes.c_void_p(w_scale.data_ptr()), N,
        ctypes.c_void_p(_ptr(bias)), ctypes.c_void_p(out.data_ptr()), y_dtype, out.stride(0),
        ctypes.c_void_p(_ptr(status)), ctypes.c_void_p(_stream_ptr(stream))), "sagesla_w8a8_gemm")
    return out
