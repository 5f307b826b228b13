"""B200-native SageSLA attention: a C-ABI CUDA library (libsagesla.so, sm_100a) and its thin
Python binding. The forward (block scores, Top-K, INT8/FP8 sparse attention, linear branch),
the SLA backward, the fused norm + per-token INT8 quantizer and the W8A8 GEMM. See
include/sagesla.h for the ABI."""
from .binding import (  # noqa: F401
    SAGESLA_BF16, SAGESLA_F32, SageslaError, alloc_workspace, load_library,
    sagesla_forward, sagesla_forward_host, sagesla_forward_no_alloc, sagesla_get_workspace_layout,
    sagesla_host_workspace_size, sagesla_status_string, sagesla_stream_status,
    sagesla_topk_count, sagesla_workspace_size, SAGESLA_LAYER_NORM, SAGESLA_RMS_NORM,
    sagesla_norm_quant, SAGESLA_NO_NORM, sagesla_w8a8_quantize_weight, sagesla_w8a8_gemm,
    sagesla_sla_backward, sagesla_sla_backward_workspace_size,
)
