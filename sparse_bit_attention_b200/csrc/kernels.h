// Host-side launch interface shared by the translation units of the library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sagesla.h"

namespace sagesla {

// A [B,H,N,128] bf16/f32 view passed by value to kernels.
struct TensorArg {
  const void* data;
  int64_t stride_b, stride_h, stride_n;
  int32_t H;
};

struct ForwardPlan {
  int64_t B, H, N, BH;
  int64_t nb;          // key/query blocks per head
  int64_t k;           // kept blocks per query block
  int64_t n_pairs;     // ceil(nb / 2)
  int64_t n_pad;       // 128 * n_pairs token rows per head in the code buffers
  int64_t mask_words;  // ceil(nb / 32)
  int64_t scores_ld;   // row stride of the block scores: nb rounded up to a multiple of 4
  int64_t nb_k_pad;    // nb rounded up to 64 (K extent of the complement-sum GEMM)
  int64_t nb_m_pad;    // nb rounded up to 128 (M extent of the complement-sum GEMM)
  int32_t n_last;      // tokens in the last block
  bool linear_empty;   // k == nb: every block kept, the linear branch is zero
  sagesla_workspace_layout lay;
};

// Fills plan from the problem size; returns false for invalid arguments.
bool make_plan(int64_t B, int64_t H, int64_t N, double topk_ratio, ForwardPlan* plan);

// Resolves cuTensorMapEncodeTiled through the runtime (no link-time libcuda dependency).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, const void* base, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);

// Kernel launchers (defined next to their kernels); each returns the launch error.
cudaError_t launch_stats(const ForwardPlan& p, TensorArg k, TensorArg v, char* ws,
                         cudaStream_t stream);
cudaError_t launch_finalize(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_quant(const ForwardPlan& p, TensorArg q, TensorArg k, TensorArg v, char* ws,
                         cudaStream_t stream);
cudaError_t launch_scores(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_topk(const ForwardPlan& p, char* ws, cudaStream_t stream);
// SAGESLA_OK when the current device is a compute-capability-10.0 part (B200), else
// SAGESLA_ERR_NO_DEVICE.
sagesla_status require_b200();

cudaError_t launch_fill_all_kept(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_complement_gemm(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_attention(const ForwardPlan& p, TensorArg q, void* out, int32_t out_dtype,
                             int64_t out_sb, int64_t out_sh, int64_t out_sn, float* sparse_out,
                             char* ws, cudaStream_t stream);
cudaError_t launch_scale_scores(const ForwardPlan& p, const char* ws, float* scores_out,
                                cudaStream_t stream);

}  // namespace sagesla
