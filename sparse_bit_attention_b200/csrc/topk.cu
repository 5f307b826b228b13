// Block scores and Top-K selection of the SageSLA forward.
//
// The news.qq.com TurboDiffusion article, section 第一把钥匙, describes SLA as first scoring
// how strongly each pair is related, then keeping only the most important fraction (Top-K
// ratio 0.1) and skipping the rest. Here a pair is (query block i, key block j) of 64 tokens
// and its score is the dot product of the pooled block means.
//
//  k_scores  qbar . kbar^T -> raw dot products [head][nb][nb] on the tensor cores (tcgen05
//            kind::tf32, 128 x 128 tiles) as three TF32 products of exact hi / lo splits
//            (3xTF32): about 2^-20 relative per product, where one TF32 product (2^-11) could
//            reorder blocks well outside the selection's tie margin.
//  k_topk_warp  one warp per (query block, head) row for rows of up to 2048 key blocks,
//            persistent over the rows with the next row's scores loaded during the current
//            selection: bisection for the k-th largest order-preserving 32-bit key with the row
//            in registers down to at most 32 candidates, a warp bitonic sort of those, then an
//            ordered compaction that takes every larger score and the lowest-index equal
//            ones. Writes the kept list (ascending), the bitmask and the bf16 complement mask
//            row (1 = not kept) of the linear branch.
//  k_topk    the same selection for longer rows, one CTA per row (radix select by bytes).
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kScoreTile = 128;                          // 128 x 128 scores per CTA (M = N = 128)
constexpr int kScoreChunk = 32;                          // channels per stage: one 128-byte fp32 row
constexpr int kScorePart = kScoreTile * kScoreChunk * 4; // 16 KB: one operand part of a stage
constexpr int kScoreSmem = 4 * kScorePart + 1024;        // A hi / lo, B hi / lo, alignment slack
constexpr uint32_t kFmtTF32 = 2;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// x = hi + lo exactly, hi with the low 13 mantissa bits cleared (a TF32 value), so that the
// tensor core reads hi without loss and lo (|lo| < 2^-10 |x|) to 2^-11 of itself.
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
  lo = x - hi;
}

// One CTA computes the 128 x 128 raw dot products qbar[i] . kbar[j] of rows i0.. and columns
// j0.. of one head on the tensor cores in three TF32 products (3xTF32): with a = a_hi + a_lo
// and b = b_hi + b_lo split exactly, a.b = a_lo.b_hi + a_hi.b_lo + a_hi.b_hi up to the
// dropped a_lo.b_lo and the TF32 reading of the lo parts, about 2^-20 of |a||b| per product:
// far inside the 1e-4 relative margin within which the Top-K selection counts as a tie.
// Channels are staged 32 at a time (a 128-byte row per block, 128-byte swizzle, K-major),
// each stage split into hi and lo parts by the 128 threads; thread 0 issues the 12 MMAs of a
// stage (4 K-steps of 8 channels x 3 products) into one fp32 TMEM accumulator of 128 columns.
// The global loads of stage c+1 are in flight while the MMAs of stage c run. Rows or columns
// past nb read as zero; columns up to ld (the padded row length) are written.
__global__ void __launch_bounds__(128)
k_scores(int nb, int ld, const float* __restrict__ qbar, const float* __restrict__ kbar,
         float* __restrict__ scores, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* a_hi = smem;
  uint8_t* a_lo = smem + kScorePart;
  uint8_t* b_hi = smem + 2 * kScorePart;
  uint8_t* b_lo = smem + 3 * kScorePart;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int64_t bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kScoreTile);
    tmem_relinquish();
  }
  if (t == 0) {
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const float* qh = qbar + bh * nb * static_cast<int64_t>(kHeadDim);
  const float* kh = kbar + bh * nb * static_cast<int64_t>(kHeadDim);
  constexpr uint32_t idesc = make_idesc(kFmtF32, kFmtTF32, kFmtTF32, 0, 0, kScoreTile, kScoreTile);
  bool ok = true;
#pragma unroll 1
  for (int c = 0; c < kHeadDim / kScoreChunk; ++c) {
    // 128 rows x 8 chunks of 16 bytes per operand; a warp reads 4 whole 128-byte rows
    float4 qv[8], kv[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int e = t + 128 * it, r = e >> 3, ch = e & 7;
      qv[it] = make_float4(0.f, 0.f, 0.f, 0.f);
      kv[it] = qv[it];
      if (i0 + r < nb)
        qv[it] = __ldg(reinterpret_cast<const float4*>(qh + (i0 + r) * kHeadDim + c * kScoreChunk) + ch);
      if (j0 + r < nb)
        kv[it] = __ldg(reinterpret_cast<const float4*>(kh + (j0 + r) * kHeadDim + c * kScoreChunk) + ch);
    }
    // the MMAs of the previous stage read the buffers about to be overwritten
    if (c > 0) ok = mbar_wait(&mma_bar, (c - 1) & 1, status);
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int e = t + 128 * it, r = e >> 3, ch = e & 7;
      const uint32_t off = sw128_offset(r, ch);
      float4 h, l;
      split_tf32(qv[it].x, h.x, l.x); split_tf32(qv[it].y, h.y, l.y);
      split_tf32(qv[it].z, h.z, l.z); split_tf32(qv[it].w, h.w, l.w);
      *reinterpret_cast<float4*>(a_hi + off) = h;
      *reinterpret_cast<float4*>(a_lo + off) = l;
      split_tf32(kv[it].x, h.x, l.x); split_tf32(kv[it].y, h.y, l.y);
      split_tf32(kv[it].z, h.z, l.z); split_tf32(kv[it].w, h.w, l.w);
      *reinterpret_cast<float4*>(b_hi + off) = h;
      *reinterpret_cast<float4*>(b_lo + off) = l;
    }
    fence_proxy_async_smem();
    if (__syncthreads_or(!ok)) {          // a timed-out wait: every thread leaves here
      ok = false;
      break;
    }
    if (t == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kScoreChunk / 8; ++ks) {
        // K-step of 8 fp32 = 32 bytes inside the swizzled 128-byte rows; 8-row groups 1 KB apart
        const uint64_t dah = make_sdesc(smem_u32(a_hi) + 32 * ks, 16, 1024, kLayoutSW128);
        const uint64_t dal = make_sdesc(smem_u32(a_lo) + 32 * ks, 16, 1024, kLayoutSW128);
        const uint64_t dbh = make_sdesc(smem_u32(b_hi) + 32 * ks, 16, 1024, kLayoutSW128);
        const uint64_t dbl = make_sdesc(smem_u32(b_lo) + 32 * ks, 16, 1024, kLayoutSW128);
        mma_tf32(tmem, dal, dbh, idesc, (c | ks) != 0);      // small terms first
        mma_tf32(tmem, dah, dbl, idesc, 1);
        mma_tf32(tmem, dah, dbh, idesc, 1);
      }
      mma_commit(&mma_bar);
    }
  }
  if (ok) ok = mbar_wait(&mma_bar, (kHeadDim / kScoreChunk - 1) & 1, status);
  ok = !__syncthreads_or(!ok);
  tc_fence_after();
  if (ok) {
    // warp w reads TMEM lanes 32w..32w+31 = rows; each thread stores 32 columns per load
    const int i = i0 + 32 * warp + lane;
    float* srow = scores + (bh * nb + i) * static_cast<int64_t>(ld);
#pragma unroll 1
    for (int cb = 0; cb < kScoreTile / 32; ++cb) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * cb, v);
      tmem_ld_wait();
      if (i < nb) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = j0 + 32 * cb + 4 * q;
          if (j < ld)
            *reinterpret_cast<float4*>(srow + j) =
                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kScoreTile);
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
       int nb_m_pad, int* status) {
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
    else if (kChecks && sel) record_error(status, SAGESLA_ERR_BOUNDS);
    if (j < nb_k_pad) arow[j] = (j < nb && !sel) ? one : zero;
    equal_base += eq_tot;
    kept_base += k_tot;
  }
}

// Bitonic sort of one key per lane into descending order across lanes 0..31 (15
// compare-exchange stages: in stage (size, step) the lower lane of each pair keeps the larger
// key inside blocks of `size` lanes that end up descending, the smaller one otherwise).
__device__ __forceinline__ uint32_t warp_sort_desc(uint32_t v, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int step = size >> 1; step > 0; step >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, v, step);
      const bool desc_block = (lane & size) == 0;
      const bool lower = (lane & step) == 0;
      v = (lower == desc_block) ? max(v, o) : min(v, o);
    }
  }
  return v;
}

// Selection of one row whose order-preserving keys sit in registers, key[m] of lane l being
// block j = 32m + l (0 for j >= nb, below every real key).
template <int M>
__device__ __forceinline__ void topk_row(const uint32_t (&key)[M], int lane, uint32_t* cw, int nb,
                                         int k, int mask_words, int nb_k_pad, int32_t* krow,
                                         uint32_t* mrow, __nv_bfloat16* arow, int* status) {
  const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
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
  // T = the k-th largest key; n_gt / n_ge = how many keys are above / at least T
  uint32_t T = lo;
  int n_gt = cnt_above, n_ge = cnt_lo;
  if (lo < hi) {
    // At most 32 keys lie in [lo, hi]: gather them one per lane, sort them, and read T off
    // as the (k - cnt_above)-th largest of them.
    int n_cand = 0;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const bool in = key[m] >= lo && key[m] <= hi;
      const uint32_t bits = __ballot_sync(0xffffffffu, in);
      if (in) cw[n_cand + __popc(bits & ((1u << lane) - 1u))] = key[m];
      n_cand += __popc(bits);
    }
    __syncwarp();
    const uint32_t sorted = warp_sort_desc(lane < n_cand ? cw[lane] : 0u, lane);
    __syncwarp();                          // cw is rewritten by the warp's next row
    T = __shfl_sync(0xffffffffu, sorted, k - cnt_above - 1);
    n_gt = cnt_above + __popc(__ballot_sync(0xffffffffu, sorted > T));
    n_ge = cnt_above + __popc(__ballot_sync(0xffffffffu, sorted >= T));
  }
  const uint32_t below = (1u << lane) - 1u;
  int kept_base = 0;
  if (n_ge == k) {
    // no tie at T to split: exactly the keys >= T are kept (T > 0, so never a padding slot)
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int j = 32 * m + lane;
      const bool sel = key[m] >= T;
      const uint32_t sel_bits = __ballot_sync(0xffffffffu, sel);
      if (sel && in_range(kept_base + __popc(sel_bits & below), k, status))
        krow[kept_base + __popc(sel_bits & below)] = j;
      if (lane == 0 && m < mask_words) mrow[m] = sel_bits;
      if (j < nb_k_pad) arow[j] = (j < nb && !sel) ? one : zero;
      kept_base += __popc(sel_bits);
    }
  } else {
    // keys equal to T: the lowest-index ones, up to k - n_gt of them
    const int take_equal = k - n_gt;
    int eq_base = 0;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int j = 32 * m + lane;
      const bool eq = j < nb && key[m] == T;
      const uint32_t eq_bits = __ballot_sync(0xffffffffu, eq);
      const bool sel = j < nb && (key[m] > T || (eq && eq_base + __popc(eq_bits & below) < take_equal));
      const uint32_t sel_bits = __ballot_sync(0xffffffffu, sel);
      if (sel && in_range(kept_base + __popc(sel_bits & below), k, status))
        krow[kept_base + __popc(sel_bits & below)] = j;
      if (lane == 0 && m < mask_words) mrow[m] = sel_bits;
      if (j < nb_k_pad) arow[j] = (j < nb && !sel) ? one : zero;
      eq_base += __popc(eq_bits);
      kept_base += __popc(sel_bits);
    }
  }
  for (int j = 32 * M + lane; j < nb_k_pad; j += 32) arow[j] = zero;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Rows of up to 32*M key blocks, one warp per row, persistent: warp w of the grid takes rows
// w, w + (warps in the grid), ... of all heads (padding rows i >= nb only clear their
// complement-mask row). The scores of the warp's next row are copied into its shared-memory
// row buffer (cp.async) while the current row is selected, so the DRAM latency of a row
// load overlaps the selection of the previous one.
template <int M>
__global__ void __launch_bounds__(128, M <= 8 ? 8 : (M <= 16 ? 6 : (M <= 48 ? 4 : 3)))
k_topk_warp(int nb, int ld, int k, int mask_words, int nb_k_pad, const float* __restrict__ scores,
            int32_t* __restrict__ kept, uint32_t* __restrict__ mask,
            __nv_bfloat16* __restrict__ amask, int nb_m_pad, int64_t n_rows, int* status) {
  __shared__ uint32_t cand[4][32];
  __shared__ __align__(16) float rowbuf[4][32 * M];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* cw = cand[warp];
  float* rb = rowbuf[warp];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 4;
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  // the nb real scores of a row as 16-byte chunks (rows are ld >= 4 * chunks floats apart)
  const int chunks = (nb + 3) >> 2;
  auto prefetch_row = [&](int64_t rw) {
    const int64_t bh = rw / nb_m_pad;
    const int i = static_cast<int>(rw - bh * nb_m_pad);
    if (i >= nb) return;
    const float* srow = scores + (bh * nb + i) * static_cast<int64_t>(ld);
    for (int c = lane; c < chunks; c += 32) cp_async16(rb + 4 * c, srow + 4 * c);
    cp_async_commit();
  };
  int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  if (row < n_rows) prefetch_row(row);
  for (; row < n_rows; row += stride) {
    const int64_t bh = row / nb_m_pad;
    const int i = static_cast<int>(row - bh * nb_m_pad);
    __nv_bfloat16* arow = amask + (bh * nb_m_pad + i) * static_cast<int64_t>(nb_k_pad);
    if (i >= nb) {   // padding rows of the complement mask (nothing was copied for them)
      for (int j = lane; j < nb_k_pad; j += 32) arow[j] = zero;
      if (row + stride < n_rows) prefetch_row(row + stride);
      continue;
    }
    cp_async_wait_all();
    __syncwarp();
    uint32_t key[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int j = 32 * m + lane;
      key[m] = j < nb ? order_key(rb[j]) : 0u;   // 0 is below every real key
    }
    __syncwarp();                              // the row buffer is refilled next
    if (row + stride < n_rows) prefetch_row(row + stride);
    topk_row<M>(key, lane, cw, nb, k, mask_words, nb_k_pad,
                kept + (bh * nb + i) * static_cast<int64_t>(k),
                mask + (bh * nb + i) * static_cast<int64_t>(mask_words), arow, status);
  }
  cp_async_wait_all();
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
  const cudaError_t attr =
      cudaFuncSetAttribute(k_scores, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem);
  if (attr != cudaSuccess) return attr;
  dim3 grid(static_cast<unsigned>((p.scores_ld + kScoreTile - 1) / kScoreTile),
            static_cast<unsigned>((p.nb + kScoreTile - 1) / kScoreTile), static_cast<unsigned>(p.BH));
  k_scores<<<grid, 128, kScoreSmem, stream>>>(static_cast<int>(p.nb), static_cast<int>(p.scores_ld),
                                              reinterpret_cast<const float*>(ws + L.qbar),
                                              reinterpret_cast<const float*>(ws + L.kbar),
                                              reinterpret_cast<float*>(ws + L.scores),
                                              reinterpret_cast<int*>(ws + L.status));
  return cudaGetLastError();
}

template <int M>
static cudaError_t launch_topk_warp(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
      (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_topk_warp<M>, 128, 0)) !=
          cudaSuccess)
    return e;
  const int64_t n_rows = p.BH * p.nb_m_pad;
  const int64_t resident = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>((n_rows + 3) / 4, resident));
  k_topk_warp<M><<<grid, 128, 0, stream>>>(
      static_cast<int>(p.nb), static_cast<int>(p.scores_ld), static_cast<int>(p.k), static_cast<int>(p.mask_words),
      static_cast<int>(p.nb_k_pad), reinterpret_cast<const float*>(ws + L.scores),
      reinterpret_cast<int32_t*>(ws + L.kept), reinterpret_cast<uint32_t*>(ws + L.mask),
      reinterpret_cast<__nv_bfloat16*>(ws + L.amask), static_cast<int>(p.nb_m_pad), n_rows,
      reinterpret_cast<int*>(ws + L.status));
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
      reinterpret_cast<__nv_bfloat16*>(ws + L.amask), static_cast<int>(p.nb_m_pad),
      reinterpret_cast<int*>(ws + L.status));
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
