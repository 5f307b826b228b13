// Block scores and Top-K selection of the SageSLA forward.
//
// The news.qq.com TurboDiffusion article, section 第一把钥匙, describes SLA as first scoring
// how strongly each pair is related, then keeping only the most important fraction (Top-K
// ratio 0.1) and skipping the rest. Here a pair is (query block i, key block j) of 64 tokens
// and its score is the dot product of the pooled block means.
//
//  k_scores  fp32 FFMA tiles of qbar . kbar^T -> raw dot products [head][nb][nb]. FFMA, not a
//            low-precision tensor-core product, keeps the ranking accurate to ~1e-7 relative.
//  k_topk    one CTA per (query block, head): radix selection of the k-th largest score on
//            order-preserving 32-bit keys, then an ordered compaction that takes every larger
//            score and the lowest-index equal ones. Writes the kept list (ascending), the
//            bitmask and the bf16 complement mask row (1 = not kept) of the linear branch.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kScoreTile = 64;

__global__ void __launch_bounds__(256)
k_scores(int nb, const float* __restrict__ qbar, const float* __restrict__ kbar,
         float* __restrict__ scores) {
  extern __shared__ float score_smem[];
  float (*qs)[kHeadDim + 1] = reinterpret_cast<float (*)[kHeadDim + 1]>(score_smem);
  float (*ks)[kHeadDim + 1] = reinterpret_cast<float (*)[kHeadDim + 1]>(score_smem + kScoreTile * (kHeadDim + 1));
  const int64_t bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  const int t = threadIdx.x;
  for (int e = t; e < kScoreTile * kHeadDim; e += 256) {
    const int r = e / kHeadDim, c = e % kHeadDim;
    qs[r][c] = (i0 + r < nb) ? qbar[(bh * nb + i0 + r) * kHeadDim + c] : 0.f;
    ks[r][c] = (j0 + r < nb) ? kbar[(bh * nb + j0 + r) * kHeadDim + c] : 0.f;
  }
  __syncthreads();
  const int ty = t >> 4, tx = t & 15;   // 4 rows (i = ty + 16a) x 4 columns (j = tx + 16b)
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
  for (int c = 0; c < kHeadDim; ++c) {
    float qa[4], kb[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) qa[a] = qs[ty + 16 * a][c];
#pragma unroll
    for (int b = 0; b < 4; ++b) kb[b] = ks[tx + 16 * b][c];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qa[a], kb[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
      if (i < nb && j < nb) scores[(bh * nb + i) * nb + j] = acc[a][b];
    }
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 is mapped like +0.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTopkThreads = 256;

// Block-wide exclusive prefix sum of one int per thread (256 threads); returns the total.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int& excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int wt = warp_tot[w];
    if (w < warp) before += wt;
    total += wt;
  }
  excl = before + incl - v;
  return total;
}

__global__ void __launch_bounds__(kTopkThreads)
k_topk(int nb, int k, int mask_words, int nb_k_pad, const float* __restrict__ scores,
       int32_t* __restrict__ kept, uint32_t* __restrict__ mask, __nv_bfloat16* __restrict__ amask,
       int nb_m_pad) {
  extern __shared__ uint32_t keys[];          // [nb]
  __shared__ int hist[256];
  __shared__ int warp_tot[8];
  __shared__ uint32_t sel_prefix;
  __shared__ int sel_remaining;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int t = threadIdx.x;
  __nv_bfloat16* arow = amask + (bh * nb_m_pad + i) * static_cast<int64_t>(nb_k_pad);
  const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);

  if (i >= nb) {   // padding rows of the complement mask
    for (int j = t; j < nb_k_pad; j += kTopkThreads) arow[j] = zero;
    return;
  }
  const float* srow = scores + (bh * nb + i) * static_cast<int64_t>(nb);
  for (int j = t; j < nb; j += kTopkThreads) keys[j] = order_key(srow[j]);
  if (t == 0) { sel_prefix = 0u; sel_remaining = k; }
  __syncthreads();

  // Radix select, most significant byte first: find the k-th largest key T.
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[t] = 0;
    __syncthreads();
    const uint32_t prefix = sel_prefix;
    const uint32_t hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int j = t; j < nb; j += kTopkThreads) {
      const uint32_t key = keys[j];
      if ((key & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(key >> shift) & 0xFF], 1);
    }
    __syncthreads();
    // count of candidates in bins strictly above bin (255 - t) ... computed as a suffix sum
    const int bin = 255 - t;                   // thread t owns bin 255 - t (descending)
    const int c = hist[bin];
    int excl;
    block_excl_scan(c, warp_tot, excl);        // excl = candidates in bins above `bin`
    const int rem = sel_remaining;
    __syncthreads();
    if (excl < rem && excl + c >= rem) {       // exactly one thread
      sel_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
      sel_remaining = rem - excl;
    }
    __syncthreads();
  }
  const uint32_t T = sel_prefix;
  const int take_equal = sel_remaining;        // equal keys to take, lowest index first

  // Ordered compaction over j in chunks of 256.
  uint32_t* mrow = mask + (bh * nb + i) * static_cast<int64_t>(mask_words);
  int32_t* krow = kept + (bh * nb + i) * static_cast<int64_t>(k);
  int equal_base = 0, kept_base = 0;
  const int lane = t & 31;
#pragma unroll 1
  for (int j0 = 0; j0 < nb_k_pad; j0 += kTopkThreads) {
    const int j = j0 + t;
    const uint32_t key = j < nb ? keys[j] : 0u;
    const int is_eq = (j < nb && key == T) ? 1 : 0;
    int eq_excl;
    const int eq_tot = block_excl_scan(is_eq, warp_tot, eq_excl);
    const bool sel = j < nb && (key > T || (is_eq && equal_base + eq_excl < take_equal));
    const uint32_t word = __ballot_sync(0xffffffffu, sel);
    if (lane == 0 && (j >> 5) < mask_words) mrow[j >> 5] = word;
    int k_excl;
    const int k_tot = block_excl_scan(sel ? 1 : 0, warp_tot, k_excl);
    if (sel && kept_base + k_excl < k) krow[kept_base + k_excl] = j;
    if (j < nb_k_pad) arow[j] = (j < nb && !sel) ? one : zero;
    equal_base += eq_tot;
    kept_base += k_tot;
  }
}

// Every key block kept (k == nb): kept lists 0..nb-1 and full masks. Written only when a
// caller asks for them; the attention kernel then walks the key blocks in order without a list.
__global__ void k_fill_all_kept(int nb, int mask_words, int32_t* __restrict__ kept,
                                uint32_t* __restrict__ mask) {
  const int64_t row = blockIdx.x;
  for (int j = threadIdx.x; j < nb; j += blockDim.x) kept[row * nb + j] = j;
  for (int w = threadIdx.x; w < mask_words; w += blockDim.x) {
    const int rem = nb - 32 * w;
    mask[row * mask_words + w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
  }
}

__global__ void k_scale_scores(int64_t n, const float* __restrict__ src, float* __restrict__ dst) {
  const int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (e < n) dst[e] = src[e] * 0.08838834764831845f;   // 1/sqrt(128)
}

}  // namespace

cudaError_t launch_scores(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  const unsigned nt = static_cast<unsigned>((p.nb + kScoreTile - 1) / kScoreTile);
  dim3 grid(nt, nt, static_cast<unsigned>(p.BH));
  constexpr int smem = 2 * kScoreTile * (kHeadDim + 1) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_scores, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k_scores<<<grid, 256, smem, stream>>>(static_cast<int>(p.nb),
                                     reinterpret_cast<const float*>(ws + L.qbar),
                                     reinterpret_cast<const float*>(ws + L.kbar),
                                     reinterpret_cast<float*>(ws + L.scores));
  return cudaGetLastError();
}

cudaError_t launch_topk(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  const size_t smem = static_cast<size_t>(p.nb) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(static_cast<unsigned>(p.nb_m_pad), static_cast<unsigned>(p.BH));
  k_topk<<<grid, kTopkThreads, smem, stream>>>(
      static_cast<int>(p.nb), static_cast<int>(p.k), static_cast<int>(p.mask_words),
      static_cast<int>(p.nb_k_pad), reinterpret_cast<const float*>(ws + L.scores),
      reinterpret_cast<int32_t*>(ws + L.kept), reinterpret_cast<uint32_t*>(ws + L.mask),
      reinterpret_cast<__nv_bfloat16*>(ws + L.amask), static_cast<int>(p.nb_m_pad));
  return cudaGetLastError();
}

cudaError_t launch_fill_all_kept(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  k_fill_all_kept<<<static_cast<unsigned>(p.BH * p.nb), 256, 0, stream>>>(
      static_cast<int>(p.nb), static_cast<int>(p.mask_words),
      reinterpret_cast<int32_t*>(ws + p.lay.kept), reinterpret_cast<uint32_t*>(ws + p.lay.mask));
  return cudaGetLastError();
}

cudaError_t launch_scale_scores(const ForwardPlan& p, const char* ws, float* scores_out,
                                cudaStream_t stream) {
  const int64_t n = p.BH * p.nb * p.nb;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
  k_scale_scores<<<blocks, 256, 0, stream>>>(n, reinterpret_cast<const float*>(ws + p.lay.scores),
                                             scores_out);
  return cudaGetLastError();
}

}  // namespace sagesla
