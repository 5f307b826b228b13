// Block scores and Top-K selection of the SageSLA forward.
//
// The news.qq.com TurboDiffusion article, section 第一把钥匙, describes SLA as first scoring
// how strongly each pair is related, then keeping only the most important fraction (Top-K
// ratio 0.1) and skipping the rest. Here a pair is (query block i, key block j) of 64 tokens
// and its score is the dot product of the pooled block means.
//
//  k_scores  fp32 FMA tiles (128 x 128, 8 x 8 per thread, packed f32x2) of qbar . kbar^T -> raw dot products
//            [head][nb][nb], each a sum over the 128 channels in ascending order. FFMA, not a
//            low-precision tensor-core product, keeps the ranking accurate to ~1e-7 relative.
//  k_topk_warp  one warp per (query block, head) for rows of up to 2048 key blocks: bisection
//            for the k-th largest order-preserving 32-bit key with the row in registers, then
//            an ordered compaction that takes every larger score and the lowest-index equal
//            ones. Writes the kept list (ascending), the bitmask and the bf16 complement mask
//            row (1 = not kept) of the linear branch.
//  k_topk    the same selection for longer rows, one CTA per row (radix select by bytes).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kScoreTile = 128;            // 128 x 128 scores per CTA, 8 x 8 per thread
constexpr int kScoreChunk = 32;            // channels staged in shared memory at a time

__device__ __forceinline__ unsigned long long pk2(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void up2(unsigned long long v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Thread (ty, tx) of 16 x 16 computes the 8 x 8 scores of rows i0 + 8ty + a (a < 8) and
// columns j0 + 4tx + 64h + u (h < 2, u < 4) with packed f32x2 FMAs. Per channel it reads its
// rows and columns as 128-bit shared loads (6 shared-memory wavefronts per warp for 32 packed
// FMAs, so the FMA pipe sets the pace) and it stores 16-byte column groups, a warp covering
// 256 contiguous bytes of a row (rows are ld floats apart, ld a multiple of 4). Each score is
// one FMA chain over the channels in ascending order.
__global__ void __launch_bounds__(256)
k_scores(int nb, int ld, const float* __restrict__ qbar, const float* __restrict__ kbar,
         float* __restrict__ scores) {
  __shared__ __align__(16) float qs[kScoreChunk][kScoreTile];
  __shared__ __align__(16) float ks[kScoreChunk][kScoreTile];
  const int64_t bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  const int t = threadIdx.x;
  const int ty = t >> 4, tx = t & 15;
  unsigned long long acc[8][4];   // [row a][column pair: 2h + u/2]
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0ull;
  const float* qh = qbar + bh * nb * static_cast<int64_t>(kHeadDim);
  const float* kh = kbar + bh * nb * static_cast<int64_t>(kHeadDim);
#pragma unroll 1
  for (int c0 = 0; c0 < kHeadDim; c0 += kScoreChunk) {
    __syncthreads();
    // 128 rows x 8 float4 chunks per operand; consecutive threads take consecutive rows
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = t + 256 * it;
      const int r = e & 127, cq = e >> 7;
      float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), kv = qv;
      if (i0 + r < nb) qv = __ldg(reinterpret_cast<const float4*>(qh + (i0 + r) * kHeadDim + c0) + cq);
      if (j0 + r < nb) kv = __ldg(reinterpret_cast<const float4*>(kh + (j0 + r) * kHeadDim + c0) + cq);
      qs[4 * cq + 0][r] = qv.x; qs[4 * cq + 1][r] = qv.y; qs[4 * cq + 2][r] = qv.z; qs[4 * cq + 3][r] = qv.w;
      ks[4 * cq + 0][r] = kv.x; ks[4 * cq + 1][r] = kv.y; ks[4 * cq + 2][r] = kv.z; ks[4 * cq + 3][r] = kv.w;
    }
    __syncthreads();
#pragma unroll 2
    for (int c = 0; c < kScoreChunk; ++c) {
      const float4 q0 = *reinterpret_cast<const float4*>(&qs[c][8 * ty]);
      const float4 q1 = *reinterpret_cast<const float4*>(&qs[c][8 * ty + 4]);
      const ulonglong2 k0 = *reinterpret_cast<const ulonglong2*>(&ks[c][4 * tx]);
      const ulonglong2 k1 = *reinterpret_cast<const ulonglong2*>(&ks[c][4 * tx + 64]);
      const float qa[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      const unsigned long long kb[4] = {k0.x, k0.y, k1.x, k1.y};
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const unsigned long long q2 = pk2(qa[a], qa[a]);
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fma2(q2, kb[b], acc[a][b]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = i0 + 8 * ty + a;
    if (i >= nb) continue;
    float* srow = scores + (bh * nb + i) * static_cast<int64_t>(ld);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = j0 + 4 * tx + 64 * h;
      if (j >= ld) continue;
      float4 v;
      up2(acc[a][2 * h], v.x, v.y);
      up2(acc[a][2 * h + 1], v.z, v.w);
      *reinterpret_cast<float4*>(srow + j) = v;
    }
  }
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 is mapped like +0.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose key is k (inverse of order_key on keys of finite floats).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
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
k_topk(int nb, int ld, int k, int mask_words, int nb_k_pad, const float* __restrict__ scores,
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
  const float* srow = scores + (bh * nb + i) * static_cast<int64_t>(ld);
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

// One warp per (query block, head) row for rows of at most 32*M key blocks: the row's keys
// stay in registers (key j = 32m + lane in key[m]); the k-th largest key T is found by
// bisection on the 32-bit key space with warp-wide counts of the keys >= the midpoint, over
// all keys until at most 32 remain between the bounds, then over those alone; the row is
// then compacted in ascending j, taking every key above T and the lowest-index keys
// equal to T. Same selection as k_topk, without block-wide synchronization.
template <int M>
__global__ void __launch_bounds__(128, M <= 24 ? 8 : (M <= 40 ? 6 : 4))
k_topk_warp(int nb, int ld, int k, int mask_words, int nb_k_pad, const float* __restrict__ scores,
            int32_t* __restrict__ kept, uint32_t* __restrict__ mask,
            __nv_bfloat16* __restrict__ amask, int nb_m_pad) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int64_t bh = blockIdx.y;
  if (i >= nb_m_pad) return;
  __nv_bfloat16* arow = amask + (bh * nb_m_pad + i) * static_cast<int64_t>(nb_k_pad);
  const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
  if (i >= nb) {   // padding rows of the complement mask
    for (int j = lane; j < nb_k_pad; j += 32) arow[j] = zero;
    return;
  }
  const float* srow = scores + (bh * nb + i) * static_cast<int64_t>(ld);
  uint32_t key[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int j = 32 * m + lane;
    key[m] = j < nb ? order_key(__ldg(srow + j)) : 0u;   // 0 is below every real key
  }
  // Invariants: count(key >= lo) = cnt_lo >= k, count(key > hi) = cnt_above < k. The bracket
  // starts at the row's smallest and largest keys and is split at the midpoint of the two
  // scores (about half the splits of halving the key range, for score rows of ordinary
  // spread), or of the keys where the scores' midpoint does not split it.
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (32 * m + lane < nb) { kmin = min(kmin, key[m]); kmax = max(kmax, key[m]); }
  uint32_t lo = __reduce_min_sync(0xffffffffu, kmin), hi = __reduce_max_sync(0xffffffffu, kmax);
  int cnt_lo = nb, cnt_above = 0;
  while (lo < hi && cnt_lo - cnt_above > 32) {
    uint32_t mid = order_key(0.5f * key_value(lo) + 0.5f * key_value(hi));
    if (mid <= lo || mid > hi) mid = lo + ((hi - lo) >> 1) + 1u;
    int c = 0;
#pragma unroll
    for (int m = 0; m < M; ++m) c += key[m] >= mid ? 1 : 0;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= k) { lo = mid; cnt_lo = c; } else { hi = mid - 1u; cnt_above = c; }
  }
  if (lo < hi) {
    // At most 32 keys lie in [lo, hi]: gather them one per lane and finish the bisection on
    // them alone (count(key >= mid) = cnt_above + candidates >= mid).
    __shared__ uint32_t cand[4][32];
    uint32_t* cw = cand[threadIdx.x >> 5];
    int n_cand = 0;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const bool in = key[m] >= lo && key[m] <= hi;
      const uint32_t bits = __ballot_sync(0xffffffffu, in);
      if (in) cw[n_cand + __popc(bits & ((1u << lane) - 1u))] = key[m];
      n_cand += __popc(bits);
    }
    __syncwarp();
    const bool has = lane < n_cand;
    const uint32_t ck = has ? cw[lane] : 0u;
    while (lo < hi) {   // cnt_above stays the count above the gathered range
      const uint32_t mid = lo + ((hi - lo) >> 1) + 1u;
      const int c = cnt_above + __popc(__ballot_sync(0xffffffffu, has && ck >= mid));
      if (c >= k) lo = mid; else hi = mid - 1u;
    }
  }
  const uint32_t T = lo;
  int gt = 0;
#pragma unroll
  for (int m = 0; m < M; ++m) gt += key[m] > T ? 1 : 0;
  const int take_equal = k - __reduce_add_sync(0xffffffffu, gt);
  int32_t* krow = kept + (bh * nb + i) * static_cast<int64_t>(k);
  uint32_t* mrow = mask + (bh * nb + i) * static_cast<int64_t>(mask_words);
  const uint32_t below = (1u << lane) - 1u;
  int eq_base = 0, kept_base = 0;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int j = 32 * m + lane;
    const bool eq = j < nb && key[m] == T;
    const uint32_t eq_bits = __ballot_sync(0xffffffffu, eq);
    const bool sel = j < nb && (key[m] > T || (eq && eq_base + __popc(eq_bits & below) < take_equal));
    const uint32_t sel_bits = __ballot_sync(0xffffffffu, sel);
    if (sel) krow[kept_base + __popc(sel_bits & below)] = j;
    if (lane == 0 && m < mask_words) mrow[m] = sel_bits;
    if (j < nb_k_pad) arow[j] = (j < nb && !sel) ? one : zero;
    eq_base += __popc(eq_bits);
    kept_base += __popc(sel_bits);
  }
  for (int j = 32 * M + lane; j < nb_k_pad; j += 32) arow[j] = zero;
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

// dst[row][j] = src[row][j] / sqrt(128) for the nb real columns of each row (src rows are ld apart).
__global__ void k_scale_scores(int64_t n, int nb, int ld, const float* __restrict__ src,
                               float* __restrict__ dst) {
  const int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (e < n) dst[e] = src[(e / nb) * ld + e % nb] * 0.08838834764831845f;
}

}  // namespace

cudaError_t launch_scores(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  const unsigned nt = static_cast<unsigned>((p.nb + kScoreTile - 1) / kScoreTile);
  dim3 grid(nt, nt, static_cast<unsigned>(p.BH));
  k_scores<<<grid, 256, 0, stream>>>(static_cast<int>(p.nb), static_cast<int>(p.scores_ld),
                                     reinterpret_cast<const float*>(ws + L.qbar),
                                     reinterpret_cast<const float*>(ws + L.kbar),
                                     reinterpret_cast<float*>(ws + L.scores));
  return cudaGetLastError();
}

template <int M>
static cudaError_t launch_topk_warp(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  dim3 grid(static_cast<unsigned>((p.nb_m_pad + 3) / 4), static_cast<unsigned>(p.BH));
  k_topk_warp<M><<<grid, 128, 0, stream>>>(
      static_cast<int>(p.nb), static_cast<int>(p.scores_ld), static_cast<int>(p.k), static_cast<int>(p.mask_words),
      static_cast<int>(p.nb_k_pad), reinterpret_cast<const float*>(ws + L.scores),
      reinterpret_cast<int32_t*>(ws + L.kept), reinterpret_cast<uint32_t*>(ws + L.mask),
      reinterpret_cast<__nv_bfloat16*>(ws + L.amask), static_cast<int>(p.nb_m_pad));
  return cudaGetLastError();
}

cudaError_t launch_topk(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const int64_t chunks = (p.nb + 31) / 32;   // register-resident rows up to 2048 key blocks
  if (chunks <= 4) return launch_topk_warp<4>(p, ws, stream);
  if (chunks <= 8) return launch_topk_warp<8>(p, ws, stream);
  if (chunks <= 16) return launch_topk_warp<16>(p, ws, stream);
  if (chunks <= 24) return launch_topk_warp<24>(p, ws, stream);
  if (chunks <= 32) return launch_topk_warp<32>(p, ws, stream);
  if (chunks <= 40) return launch_topk_warp<40>(p, ws, stream);
  if (chunks <= 48) return launch_topk_warp<48>(p, ws, stream);
  if (chunks <= 64) return launch_topk_warp<64>(p, ws, stream);
  const auto& L = p.lay;
  const size_t smem = static_cast<size_t>(p.nb) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(static_cast<unsigned>(p.nb_m_pad), static_cast<unsigned>(p.BH));
  k_topk<<<grid, kTopkThreads, smem, stream>>>(
      static_cast<int>(p.nb), static_cast<int>(p.scores_ld), static_cast<int>(p.k), static_cast<int>(p.mask_words),
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
  k_scale_scores<<<blocks, 256, 0, stream>>>(n, static_cast<int>(p.nb), static_cast<int>(p.scores_ld),
                                             reinterpret_cast<const float*>(ws + p.lay.scores),
                                             scores_out);
  return cudaGetLastError();
}

}  // namespace sagesla
