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

constexpr int kMaxCanaries = 32;

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
  bool quant;          // INT8 Q.K^T (else bf16 Q.K^T from packed bf16 copies)
  bool pv_fp8;         // e4m3 P.V (else bf16 P and raw bf16 V)
  sagesla_workspace_layout lay;
  // canary of each workspace region: 16 bytes at the region's end rounded up to 16
  int32_t n_canary;
  uint64_t canary[kMaxCanaries];
};

// Fills plan from the problem size and operand mode; returns false for invalid arguments.
bool make_plan(int64_t B, int64_t H, int64_t N, double topk_ratio, ForwardPlan* plan,
               bool quant = true, bool pv_fp8 = true);

// Resolves cuTensorMapEncodeTiled through the runtime (no link-time libcuda dependency).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, const void* base, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);

// Same for a tiled map of any rank (dims[0] contiguous; strides in bytes of dims 1..rank-1).
bool encode_tmap_nd(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                    const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                    CUtensorMapSwizzle swizzle);

// Workspace of the SLA backward: the forward's layout followed by these regions.
struct BackwardLayout {
  size_t qn, kn, vn, dn;            // packed bf16 Q, K, V, dO [BH][n_pad][128]
  size_t lse, dd;                   // [BH][n_pad] f32
  size_t tcount, toff, tlist;       // query blocks keeping each key block: counts [BH][nb],
                                    // offsets [BH][nb + 1], indices [BH][nb * k]
  size_t lin_q, lin_k, lin_v;       // linear-branch gradients [BH][n_pad][128] f32
  size_t amask_t;                   // transposed complement mask [BH][nb_m_pad][nb_m_pad] bf16
  size_t dg, dh;                    // [BH][nb_m_pad][129 * 128] bf16
  size_t total;
};
bool make_backward_layout(const ForwardPlan& p, BackwardLayout* bl);

// Gradient outputs of the backward (one dtype for all three; strides in elements).
struct GradOut {
  void* dq; void* dk; void* dv;
  int64_t dq_s[3], dk_s[3], dv_s[3];
  int32_t dtype;
};
cudaError_t launch_sla_backward(const ForwardPlan& p, const BackwardLayout& bl, TensorArg q,
                                TensorArg k, TensorArg v, TensorArg d_out, const GradOut& g,
                                char* ws, cudaStream_t stream);
// C[BH][M][16512] = A[BH][M][K] . B[BH][K][16512] (bf16, M a multiple of 128, K of 64).
cudaError_t launch_mask_gemm(const void* a, const void* b, void* c, int64_t BH, int64_t M,
                             int64_t K, int* status, cudaStream_t stream);

// Kernel launchers (defined next to their kernels); each returns the launch error.
cudaError_t launch_stats(const ForwardPlan& p, TensorArg k, TensorArg v, char* ws,
                         cudaStream_t stream);
cudaError_t launch_finalize(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_quant(const ForwardPlan& p, TensorArg q, TensorArg k, TensorArg v, char* ws,
                         cudaStream_t stream);
// bf16 copies of Q and K (quant off) and V (pv_fp8 off) into the workspace.
cudaError_t launch_pack_bf16(const ForwardPlan& p, TensorArg q, TensorArg k, TensorArg v,
                             char* ws, cudaStream_t stream);
cudaError_t launch_scores(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_topk(const ForwardPlan& p, char* ws, cudaStream_t stream);
// SAGESLA_OK when the current device is a compute-capability-10.0 part (B200), else
// SAGESLA_ERR_NO_DEVICE.
sagesla_status require_b200();

cudaError_t launch_fill_all_kept(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_complement_gemm(const ForwardPlan& p, char* ws, cudaStream_t stream);
// Failure-path test hooks of the attention kernel (zero in normal use).
struct AttnTestHooks {
  uint32_t spin_limit_us;   // > 0: limit of every wait instead of kSpinLimitNs
  int32_t skip_tile;        // 1: the first CTA never loads its first K tile pair
};
cudaError_t launch_attention(const ForwardPlan& p, TensorArg q, void* out, int32_t out_dtype,
                             int64_t out_sb, int64_t out_sh, int64_t out_sn, float* sparse_out,
                             char* ws, const AttnTestHooks& hooks, cudaStream_t stream);
// Dense mode (every key block kept, INT8 / e4m3 operands): M=128 tiles over all key blocks.
cudaError_t launch_attention_dense(const ForwardPlan& p, TensorArg q, void* out, int32_t out_dtype,
                                   int64_t out_sb, int64_t out_sh, int64_t out_sn,
                                   float* sparse_out, char* ws, const AttnTestHooks& hooks,
                                   cudaStream_t stream);
// debug_checks: write the canary pattern after every workspace region / verify it (a damaged
// canary records SAGESLA_ERR_CANARY in the status word).
cudaError_t launch_canary_fill(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_canary_verify(const ForwardPlan& p, char* ws, cudaStream_t stream);
cudaError_t launch_scale_scores(const ForwardPlan& p, const char* ws, float* scores_out,
                                cudaStream_t stream);

}  // namespace sagesla
