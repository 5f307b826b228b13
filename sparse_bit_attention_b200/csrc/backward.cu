// SLA backward: gradients of the unquantized sparse-linear attention with the block
// selection of the forward held fixed.
//
// Method: news.qq.com TurboDiffusion article, section 从训练到部署 — the full attention layers
// are replaced by SLA and fine-tuned, and only at inference is SLA swapped for SageSLA (SLA
// plus low-bit quantization); the sparse and linear branches follow the "Sparse-Linear
// Attention" method named in the dgmzs.com.cn README translation, section 方法论. With
// s = q.k/sqrt(128), for a query token t of block i and the tokens u of its kept blocks:
//     L_t = log sum_u e^{s_tu},  P = e^{s - L},  O_s = P V,  D_t = dO_t . O_s,t,
//     dS = P (dO V^T - D),  dQ = dS K / sqrt(128),  dK = dS^T Q / sqrt(128),  dV = P^T dO;
// and for the linear branch (a = phi(q), G_i the sum of the key-block states H_j over the
// blocks i does not keep, num = a G_i[:, :128], den = a G_i[:, 128], O_l = num / den):
//     dnum = dO / den,  dden = -(dO . O_l) / den,  da = G_i[:, :128] dnum + G_i[:, 128] dden,
//     dq += a * da (the softmax Jacobian's projection a . da vanishes: O_l is unchanged when a
//     is scaled),  dG_i = a^T [dnum | dden],  dH_j = sum of dG_i over the blocks not keeping j,
//     db = dH_j[:, :128] v + dH_j[:, 128],  dk += b * (db - b . db),  dv += dH_j[:, :128]^T b,
//     with b = phi(k).
//
// B200 mapping. The forward's prologue supplies the kept lists, the complement mask and G_i.
// Q, K, V and dO are packed into zero-padded [head][row][128] bf16 copies; every 64-row tile is
// loaded by TMA in the key-interleaved order (row 2i + h of the tile holds token 32h + i) that
// makes the 16x64b TMEM fragment of an M=64 result hold 32 consecutive tokens per thread, so
// the P and dS operands written back by the threads are 64 contiguous bytes after one pair
// exchange. The sparse branch runs on tcgen05 BF16 MMAs (fp32 accumulators in TMEM):
//   k_bwd_lse     per query block: the scores again (online softmax), giving the base-2
//                 log-sum-exp L and D = rowsum(dO * O_s), taken as rowsum(P * dO V^T)
//   k_bwd_dq      per query block over its kept blocks: S, dP, dS, dQ (role warps: softmax,
//                 S / dP / dQ issuers, TMA producer); adds the linear dq
//   k_bwd_dkv     per key block over the query blocks that keep it (compressed per-head lists
//                 built from the kept bitmask): S^T, dP^T, dV, dK (role warps, a two-stage
//                 Q / dO ring); adds the linear dk, dv
// The linear branch: k_bwd_lin_query and k_bwd_lin_key put their products over channels on
// tcgen05 (the column-128 and rank-one terms on the CUDA cores), around one complement GEMM
// (dH = (1 - M)^T dG, the forward's GEMM on the transposed mask).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {


// 2^x by the MUFU approximation (subnormal results flushed to zero): the probabilities here
// are compared with a tolerance of 2^-5 of each gradient's magnitude
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kScale = 0.08838834764831845f;   // 1 / sqrt(128)
constexpr uint32_t kTile = 64 * 128 * 2;         // one 64-row bf16 tile (two 8 KB d-chunks)
constexpr uint32_t kPTile = 64 * 64 * 2;         // a 64 x 64 bf16 operand (one 128-byte atom)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Token of position p of a key-interleaved 64-row tile.
__device__ __forceinline__ int tile_token(int p) { return (p >> 1) + 32 * (p & 1); }

// 16x64b TMEM fragment of an M=64 result: warp w, lane t hold row 16w + t/4 + 8(t&1) and the
// columns kh + 2e (e = 0..31), kh = (t >> 1) & 1.
__device__ __forceinline__ int frag_row(int warp, int lane) {
  return 16 * warp + (lane >> 2) + 8 * (lane & 1);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// This thread's 32 values (columns kh + 2e of a row, i.e. the tile positions of tokens
// 32kh + e) as bf16 into a 64 x 64 K-major SW128 operand tile in tile-position order: after
// an exchange with lane ^ 2 (same row, other kh), the thread holds positions 32kh .. 32kh+31
// and stores them as four 16-byte chunks.
__device__ __forceinline__ void store_row_operand(uint8_t* tile, int row, int kh,
                                                  const float (&x)[32]) {
  uint32_t send[8], mine[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    // kh = 0 keeps e = 0..15 and sends 16..31; kh = 1 keeps 16..31 and sends 0..15
    send[u] = kh ? pack_bf16x2(x[2 * u], x[2 * u + 1]) : pack_bf16x2(x[16 + 2 * u], x[17 + 2 * u]);
    mine[u] = kh ? pack_bf16x2(x[16 + 2 * u], x[17 + 2 * u]) : pack_bf16x2(x[2 * u], x[2 * u + 1]);
  }
  uint32_t recv[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) recv[u] = __shfl_xor_sync(0xffffffffu, send[u], 2);
  // position 2e' + h holds token 32h + e'; the thread covers e' = 16kh .. 16kh + 15. The
  // kh = 0 thread owns tokens e (h = 0), the kh = 1 thread tokens 32 + e (h = 1).
  uint32_t w[16];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint32_t lo_m = mine[u] & 0xFFFFu, hi_m = mine[u] >> 16;
    const uint32_t lo_r = recv[u] & 0xFFFFu, hi_r = recv[u] >> 16;
    // words for e' = 16kh + 2u and 16kh + 2u + 1: (h=0 value, h=1 value)
    w[2 * u] = kh ? (lo_r | (lo_m << 16)) : (lo_m | (lo_r << 16));
    w[2 * u + 1] = kh ? (hi_r | (hi_m << 16)) : (hi_m | (hi_r << 16));
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, 4 * kh + c)) =
        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

// ------------------------------------------------------------------ packing and lists

// Q, K, V, dO rows -> zero-padded [head][n_pad][128] bf16 copies (one thread per 16 bytes).
__global__ void k_bwd_pack(TensorArg q, TensorArg k, TensorArg v, TensorArg d_out, int N,
                           int n_pad, int64_t total, uint4* __restrict__ qp, uint4* __restrict__ kp,
                           uint4* __restrict__ vp, uint4* __restrict__ dp) {
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= total) return;
  const int chunk = static_cast<int>(idx & 15);
  const int64_t row = idx >> 4;
  const int64_t bh = row / n_pad;
  const int n = static_cast<int>(row - bh * n_pad);
  uint4 z = make_uint4(0, 0, 0, 0);
  uint4 a = z, b = z, c = z, d = z;
  if (n < N) {
    auto ld = [&](const TensorArg& t) {
      const int64_t bb = bh / t.H, hh = bh % t.H;
      const uint16_t* base = static_cast<const uint16_t*>(t.data) + bb * t.stride_b +
                             hh * t.stride_h + static_cast<int64_t>(n) * t.stride_n;
      return __ldg(reinterpret_cast<const uint4*>(base) + chunk);
    };
    a = ld(q); b = ld(k); c = ld(v); d = ld(d_out);
  }
  qp[idx] = a; kp[idx] = b; vp[idx] = c; dp[idx] = d;
}

// Query blocks that keep each key block, as one compressed list per head: tcount[head][j]
// query blocks keep key block j; their indices, ascending, are tlist[head][toff[head][j] ..],
// nb * k entries per head in all. Three passes: counts (one warp per (head, j) reading the kept
// bitmask column j), an exclusive scan per head, and the fill.
__global__ void k_bwd_list_count(int nb, int mask_words, int64_t BH, const uint32_t* __restrict__ mask,
                                 int32_t* __restrict__ tcount) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  if (w >= BH * nb) return;
  const int64_t bh = w / nb;
  const int j = static_cast<int>(w - bh * nb);
  const uint32_t* mcol = mask + bh * nb * static_cast<int64_t>(mask_words) + (j >> 5);
  int count = 0;
  for (int i0 = 0; i0 < nb; i0 += 32) {
    const int i = i0 + lane;
    const bool kept = i < nb && ((__ldg(mcol + static_cast<int64_t>(i) * mask_words) >> (j & 31)) & 1u);
    count += __popc(__ballot_sync(0xffffffffu, kept));
  }
  if (lane == 0) tcount[bh * nb + j] = count;
}

// toff[head][j] = sum of tcount[head][0 .. j-1] (one 1024-thread CTA per head).
__global__ void __launch_bounds__(1024) k_bwd_list_scan(int nb, const int32_t* __restrict__ tcount,
                                                        int32_t* __restrict__ toff) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int64_t bh = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int32_t* cnt = tcount + bh * nb;
  int32_t* off = toff + bh * (nb + 1);
  if (t == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < nb; base += 1024) {
    const int v = base + t < nb ? cnt[base + t] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;                       // inclusive scan of the warp totals
    }
    __syncthreads();
    const int excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
    if (base + t < nb) off[base + t] = excl;
    __syncthreads();
    if (t == 0) carry += warp_sums[31];
    __syncthreads();
  }
  if (t == 0) off[nb] = carry;
}

__global__ void k_bwd_list_fill(int nb, int k, int mask_words, int64_t BH,
                                const uint32_t* __restrict__ mask, const int32_t* __restrict__ toff,
                                int32_t* __restrict__ tlist, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  if (w >= BH * nb) return;
  const int64_t bh = w / nb;
  const int j = static_cast<int>(w - bh * nb);
  const uint32_t* mcol = mask + bh * nb * static_cast<int64_t>(mask_words) + (j >> 5);
  int32_t* out = tlist + bh * nb * static_cast<int64_t>(k) + toff[bh * (nb + 1) + j];
  int count = 0;
  for (int i0 = 0; i0 < nb; i0 += 32) {
    const int i = i0 + lane;
    const bool kept = i < nb && ((__ldg(mcol + static_cast<int64_t>(i) * mask_words) >> (j & 31)) & 1u);
    const uint32_t bits = __ballot_sync(0xffffffffu, kept);
    const int pos = count + __popc(bits & ((1u << lane) - 1u));
    if (kept && in_range(toff[bh * (nb + 1) + j] + pos, static_cast<long long>(nb) * k, status))
      out[pos] = i;
    count += __popc(bits);
  }
}

// amask [head][nb_m_pad][nb_k_pad] (1 where the key block is not kept) -> its transpose,
// [head][nb_m_pad][nb_m_pad] with zero rows past nb_k_pad (the row extent of the complement
// GEMM is a multiple of 128), by 32 x 32 tiles through shared memory.
__global__ void k_bwd_transpose_mask(int nb_m_pad, int nb_k_pad, const uint16_t* __restrict__ src,
                                     uint16_t* __restrict__ dst) {
  __shared__ uint16_t t[32][33];
  const int64_t bh = blockIdx.z;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;   // source row i, source column j
  const uint16_t* s = src + bh * nb_m_pad * static_cast<int64_t>(nb_k_pad);
  uint16_t* d = dst + bh * nb_m_pad * static_cast<int64_t>(nb_m_pad);
  for (int r = threadIdx.y; r < 32; r += blockDim.y)
    t[r][threadIdx.x] = j0 + threadIdx.x < nb_k_pad
                            ? s[static_cast<int64_t>(i0 + r) * nb_k_pad + j0 + threadIdx.x]
                            : static_cast<uint16_t>(0);
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y)
    d[static_cast<int64_t>(j0 + r) * nb_m_pad + i0 + threadIdx.x] = t[threadIdx.x][r];
}

// ------------------------------------------------------------------ sparse branch (tcgen05)

// Instruction descriptors: M=64 BF16 MMAs with fp32 accumulation.
constexpr uint32_t kIdescKK64 = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 0, 64, 64);   // S-like
constexpr uint32_t kIdescKM128 = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 1, 64, 128); // P.V-like

// K-major operand of 64 rows x 128 (bf16, two 8 KB chunks of 64 columns): K-step kk of 16.
__device__ __forceinline__ uint64_t desc_k128(uint32_t base, int kk) {
  return make_sdesc(base + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
}
// K-major 64 x 64 operand (P, dS; one 128-byte atom per row): K-step kk of 16.
__device__ __forceinline__ uint64_t desc_k64(uint32_t base, int kk) {
  return make_sdesc(base + kk * 32, 16, 1024, kLayoutSW128);
}
// MN-major operand: 64 rows of K x 128 columns of N (two 8 KB chunks of 64 N): K-step kk.
__device__ __forceinline__ uint64_t desc_mn128(uint32_t base, int kk) {
  return make_sdesc(base + kk * 2048, 8192, 1024, kLayoutSW128);
}

// A 64 x 128 tile of rows [row, row + 64) of a packed buffer, key-interleaved (two 8 KB
// loads, one per 64-column chunk) through the four-dimensional map of that buffer.
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                          int block_row) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(0), "r"(0), "r"(0),
      "r"(block_row)
      : "memory");
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst + 8192)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(64), "r"(0), "r"(0),
      "r"(block_row)
      : "memory");
}

struct BwdParams {
  const int32_t* kept;     // [BH][nb][k]
  const int32_t* tcount;   // [BH][nb]
  const int32_t* toff;     // [BH][nb + 1]
  const int32_t* tlist;    // [BH][nb * k], compressed per head
  const uint16_t* qn;      // packed bf16 rows [BH][n_pad][128]
  const uint16_t* dn;      // packed dO
  float* lse;              // [BH][n_pad], base-2 log-sum-exp of the scaled scores
  float* dd;               // [BH][n_pad], D = rowsum(dO * O_s)
  const float* lin_q;      // [BH][n_pad][128] linear-branch dq (null: none)
  const float* lin_k;
  const float* lin_v;
  void* dq; void* dk; void* dv;
  int64_t dq_sb, dq_sh, dq_sn, dk_sb, dk_sh, dk_sn, dv_sb, dv_sh, dv_sn;
  int32_t g_dtype;         // SAGESLA_F32 or SAGESLA_BF16 for dq, dk, dv
  int* status;
  int N, nb, n_pad, k, n_last, H;
};


// Online-softmax pass of one query block over its kept key blocks (bf16 MMAs): writes the
// base-2 log-sum-exp L of the scaled scores and D = rowsum(dO * O_s) of its 64 rows. D is
// taken as rowsum(P * dP) with dP = dO V^T (the same sum: O_s = P V), accumulated online like
// the normalizer, both rescaled by the per-row factor when the running maximum moves, so the
// pass needs neither a P operand tile nor an O accumulator.
// Warps 0-3 take the softmax (one row pair per lane pair, as everywhere here); warp 4 issues
// S = Q K^T and warp 5 dP = dO V^T of each block into double buffers (TMEM [0, 128) and
// [128, 256)), running ahead of the softmax by one block; warp 6 loads the K and V tiles into
// a two-stage ring, refilling a stage as soon as the MMAs of the block in it have completed.
// Everything is ordered by mbarriers (no block-wide barrier in the loop); every wait is
// bounded, and a timed-out wait ends every role's loop through abort_flag.
// Wait of the role-warp kernels: a completed phase passes at once; otherwise the CTA's abort
// flag is read (set: give up at once), then the bounded wait. Trying the barrier first keeps
// the shared-memory read of the flag off the path of waits that need not block.
__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, volatile int& abort_flag,
                                         int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  if (abort_flag) return false;
  return mbar_wait(bar, parity, status);
}

constexpr int kLseThreads = 224;

__global__ void __launch_bounds__(kLseThreads, 2)
k_bwd_lse(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          BwdParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* q_t = smem;                   // Q tile
  uint8_t* do_t = smem + kTile;          // dO tile
  uint8_t* k_t = smem + 2 * kTile;       // 2 K stages
  uint8_t* v_t = smem + 4 * kTile;       // 2 V stages
  __shared__ uint64_t q_full, k_full[2], v_full[2], s_done[2], s_free[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int U = prm.k;
  const int32_t* klist = prm.kept + (bh * prm.nb + i) * static_cast<int64_t>(prm.k);
  const int blk0 = static_cast<int>(bh * (prm.n_pad / 64));   // first 64-row block of the head
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1); mbar_init(&v_full[s], 1);
      mbar_init(&s_done[s], 2);          // the S and the dP commit of a block
      mbar_init(&s_free[s], 4);          // the four softmax warps have read a block
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;
  if (warp == 6) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q); prefetch_tmap(&tm_do); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&q_full, 2 * kTile);
      load_tile(q_t, &tm_q, &q_full, blk0 + i);
      load_tile(do_t, &tm_do, &q_full, blk0 + i);
      for (int m = 0; m < U; ++m) {
        const int b = m & 1;
        // stage b held block m - 2: its S and dP MMAs must have completed
        if (m >= 2 && !bwd_wait(&s_done[b], ((m - 2) >> 1) & 1, abort_flag, prm.status)) {
          ok = false;
          break;
        }
        const int jk = __ldg(klist + m);
        if (!in_range(jk, prm.nb, prm.status)) {   // checking build: the tile is not loaded
          ok = false;
          break;
        }
        const int jm = blk0 + jk;
        mbar_arrive_expect_tx(&k_full[b], kTile);
        load_tile(k_t + b * kTile, &tm_k, &k_full[b], jm);
        mbar_arrive_expect_tx(&v_full[b], kTile);
        load_tile(v_t + b * kTile, &tm_v, &v_full[b], jm);
      }
      if (!ok) abort_flag = 1;
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ MMA issuers: warp 4 S, warp 5 dP
    if (lane == 0) {
      const bool is_s = warp == 4;
      uint64_t* full = is_s ? k_full : v_full;
      const uint32_t a = smem_u32(is_s ? q_t : do_t);
      const uint32_t stage = smem_u32(is_s ? k_t : v_t);
      const uint32_t dcol = is_s ? 0u : 128u;
      ok = mbar_wait(&q_full, 0, prm.status);
      for (int n = 0; n < U && ok; ++n) {
        const int b = n & 1;
        // buffer b held block n - 2: the softmax warps must have read it
        if (n >= 2) ok = bwd_wait(&s_free[b], ((n - 2) >> 1) & 1, abort_flag, prm.status);
        ok = ok && bwd_wait(&full[b], (n >> 1) & 1, abort_flag, prm.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t bsm = stage + b * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + dcol + 64 * b, desc_k128(a, kk), desc_k128(bsm, kk), kIdescKK64,
                   kk > 0 ? 1u : 0u);
        mma_commit(&s_done[b]);
      }
      if (!ok) abort_flag = 1;
    }
  } else {
    // ------------------------------------------------ softmax warps
    const int row = frag_row(warp, lane);
    const int kh = (lane >> 1) & 1;
    const uint32_t lane_s = static_cast<uint32_t>(32 * warp) << 16;
    const float c2 = kScale * kLog2e;
    float m_run = -INFINITY, l_part = 0.f, d_part = 0.f;
    for (int n = 0; n < U; ++n) {
      const int st = n & 1;
      ok = bwd_wait(&s_done[st], (n >> 1) & 1, abort_flag, prm.status);
      ok = __all_sync(0xffffffffu, ok) != 0;      // the warp leaves together
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32], pr[32];
      tmem_ld16x64(tmem + lane_s + 64 * st, sr);
      tmem_ld16x64(tmem + lane_s + 128 + 64 * st, pr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[st]);
      const int j = __ldg(klist + n);
      const int valid = (j == prm.nb - 1) ? prm.n_last - 32 * kh : 32;   // real keys of this thread
      float x[32], mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        x[e] = e < valid ? __uint_as_float(sr[e]) * c2 : -INFINITY;
        mx = fmaxf(mx, x[e]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const float alpha = ex2_approx(m_run - m_new);
      float rs = 0.f, pd = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p = ex2_approx(x[e] - m_new);
        rs += p;
        pd = fmaf(p, __uint_as_float(pr[e]), pd);
      }
      l_part = alpha * l_part + rs;
      d_part = alpha * d_part + pd;
      m_run = m_new;
    }
    if (!ok) abort_flag = 1;
    const float l_row = l_part + __shfl_xor_sync(0xffffffffu, l_part, 2);
    const float d_row = d_part + __shfl_xor_sync(0xffffffffu, d_part, 2);
    const int tok = tile_token(row);
    const int64_t grow = bh * prm.n_pad + 64 * static_cast<int64_t>(i) + tok;
    if (ok && kh == 0) {
      prm.lse[grow] = m_run + log2f(l_row);
      prm.dd[grow] = d_row / l_row;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// Stores this thread's 32 values of chunk cb of a gradient row (columns 64cb + kh + 2e, in
// g[e]) to the output row: an exchange with lane ^ 2 gives each thread the 32 contiguous
// columns 64cb + 32kh .. +31, written 16 (f32) or 8 (bf16) bytes at a time.
__device__ __forceinline__ void store_grad_chunk(const float (&g)[32], int cb, int kh, void* base,
                                                 int32_t dtype) {
  const int col0 = 64 * cb + 32 * kh;
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    float w4[4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      // kh = 0 keeps columns 2(e+u), 2(e+u)+1 of the chunk's first half; kh = 1 the second
      const float mine0 = g[e + u], mine1 = g[16 + e + u];
      const float recv = __shfl_xor_sync(0xffffffffu, kh ? mine0 : mine1, 2);
      w4[2 * u] = kh ? recv : mine0;
      w4[2 * u + 1] = kh ? mine1 : recv;
    }
    if (base == nullptr) continue;
    if (dtype == SAGESLA_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(base) + col0 + 2 * e) =
          make_float4(w4[0], w4[1], w4[2], w4[3]);
    } else {
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(base) + col0 + 2 * e) =
          make_uint2(pack_bf16x2(w4[0], w4[1]), pack_bf16x2(w4[2], w4[3]));
    }
  }
}

__device__ __forceinline__ void* grad_row(void* base, int32_t dtype, int64_t sb, int64_t sh,
                                          int64_t sn, int64_t bh, int H, int tok) {
  const int64_t b = bh / H, h = bh % H;
  const int64_t off = b * sb + h * sh + static_cast<int64_t>(tok) * sn;
  return static_cast<char*>(base) + off * (dtype == SAGESLA_F32 ? 4 : 2);
}

// dQ of one query block over its kept key blocks: S = Q K^T and dP = dO V^T (M=64 N=64 each;
// S in TMEM lanes 0-15 and dP in lanes 16-31 of each quadrant, double-buffered in columns
// [0, 64) and [64, 128)), dS = P (dP - D) with P = 2^(S c - L), dQ += dS K (columns
// [128, 256)). Role warps ordered by mbarriers: warps 0-3 the softmax (dS into two shared
// tiles, so that storing dS of block n waits only for the dQ of block n - 2), warp 4 issues S
// and warp 5 dP one block ahead, warp 6 dQ, warp 7 loads K and V of each block into a
// two-stage ring, refilling a stage once the dQ of its block (the last reader of K) has
// completed. The tiles take 112 KB (dynamic shared memory declared 1024-byte aligned and
// checked, as in k_bwd_dkv). The linear-branch dq is added before the store.
constexpr int kDqThreads = 256;

__global__ void __launch_bounds__(kDqThreads, 2)
k_bwd_dq(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
         BwdParams prm) {
  extern __shared__ __align__(1024) uint8_t smem_dq[];
  uint8_t* q_t = smem_dq;                // Q tile
  uint8_t* o_t = smem_dq + kTile;        // dO tile
  uint8_t* k_t = smem_dq + 2 * kTile;    // 2 K stages
  uint8_t* v_t = smem_dq + 4 * kTile;    // 2 V stages
  uint8_t* s_t = smem_dq + 6 * kTile;    // 2 dS tiles
  __shared__ uint64_t q_full, kv_full[2], s_done[2], s_free[2], ds_full[2], dq_done[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  if (smem_u32(smem_dq) & 1023u) {           // same for every thread of the CTA
    if (threadIdx.x == 0) record_error(prm.status, SAGESLA_ERR_DEVICE_CHECK);
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int U = prm.k;
  const int32_t* klist = prm.kept + (bh * prm.nb + i) * static_cast<int64_t>(prm.k);
  const int blk0 = static_cast<int>(bh * (prm.n_pad / 64));
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&s_done[s], 2);          // the S and the dP commit of a block
      mbar_init(&s_free[s], 4);          // the four softmax warps have read S and dP
      mbar_init(&dq_done[s], 1);
      mbar_init(&ds_full[s], 4);         // the four softmax warps have stored dS
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;
  if (warp == 7) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(&q_full, 2 * kTile);
      load_tile(q_t, &tm_q, &q_full, blk0 + i);
      load_tile(o_t, &tm_do, &q_full, blk0 + i);
      for (int m = 0; m < U; ++m) {
        const int b = m & 1;
        // stage b held block m - 2: its dQ (after its S and dP) must have completed
        if (m >= 2 && !bwd_wait(&dq_done[b], ((m - 2) >> 1) & 1, abort_flag, prm.status)) {
          ok = false;
          break;
        }
        const int jk = __ldg(klist + m);
        if (!in_range(jk, prm.nb, prm.status)) {   // checking build: the tile is not loaded
          ok = false;
          break;
        }
        const int jm = blk0 + jk;
        mbar_arrive_expect_tx(&kv_full[b], 2 * kTile);
        load_tile(k_t + b * kTile, &tm_k, &kv_full[b], jm);
        load_tile(v_t + b * kTile, &tm_v, &kv_full[b], jm);
      }
      if (!ok) abort_flag = 1;
    }
  } else if (warp == 6) {
    // ------------------------------------------------ dQ issuer
    if (lane == 0) {
      for (int n = 0; n < U; ++n) {
        ok = bwd_wait(&ds_full[n & 1], (n >> 1) & 1, abort_flag, prm.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(s_t + (n & 1) * kPTile);
        const uint32_t kb = smem_u32(k_t + (n & 1) * kTile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 128, desc_k64(sa, kk), desc_mn128(kb, kk), kIdescKM128,
                   (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&dq_done[n & 1]);
      }
      if (!ok) abort_flag = 1;
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ S (warp 4) and dP (warp 5) issuers
    if (lane == 0) {
      const bool is_s = warp == 4;
      const uint32_t a = smem_u32(is_s ? q_t : o_t);
      const uint32_t stage = smem_u32(is_s ? k_t : v_t);
      const uint32_t dbase = is_s ? tmem : tmem + (16u << 16);
      ok = mbar_wait(&q_full, 0, prm.status);
      for (int n = 0; n < U && ok; ++n) {
        const int b = n & 1;
        // buffer b held block n - 2: the softmax warps must have read it
        if (n >= 2) ok = bwd_wait(&s_free[b], ((n - 2) >> 1) & 1, abort_flag, prm.status);
        ok = ok && bwd_wait(&kv_full[b], (n >> 1) & 1, abort_flag, prm.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t bsm = stage + b * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(dbase + 64 * b, desc_k128(a, kk), desc_k128(bsm, kk), kIdescKK64,
                   kk > 0 ? 1u : 0u);
        mma_commit(&s_done[b]);
      }
      if (!ok) abort_flag = 1;
    }
  } else {
    // ------------------------------------------------ softmax warps
    const int row = frag_row(warp, lane);
    const int kh = (lane >> 1) & 1;
    const int tok = tile_token(row);
    const int64_t grow = bh * prm.n_pad + 64 * static_cast<int64_t>(i) + tok;
    const float l2 = prm.lse[grow], dterm = prm.dd[grow];
    const uint32_t lane_s = static_cast<uint32_t>(32 * warp) << 16;
    const uint32_t lane_p = static_cast<uint32_t>(32 * warp + 16) << 16;
    const float c2 = kScale * kLog2e;
    for (int n = 0; n < U; ++n) {
      const int b = n & 1;
      ok = bwd_wait(&s_done[b], (n >> 1) & 1, abort_flag, prm.status);
      ok = __all_sync(0xffffffffu, ok) != 0;      // the warp leaves together
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32], pr[32];
      tmem_ld16x64(tmem + lane_s + 64 * b, sr);
      tmem_ld16x64(tmem + lane_p + 64 * b, pr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      float ds[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p = ex2_approx(__uint_as_float(sr[e]) * c2 - l2);
        ds[e] = p * (__uint_as_float(pr[e]) - dterm);
      }
      // dQ of block n - 2 has read dS tile b
      if (n >= 2) {
        ok = bwd_wait(&dq_done[b], ((n - 2) >> 1) & 1, abort_flag, prm.status);
        ok = __all_sync(0xffffffffu, ok) != 0;
        if (!ok) break;
      }
      store_row_operand(s_t + b * kPTile, row, kh, ds);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[b]);
    }
    if (ok) ok = mbar_wait(&dq_done[(U - 1) & 1], ((U - 1) >> 1) & 1, prm.status);
    ok = __all_sync(0xffffffffu, ok) != 0;
    if (!ok) abort_flag = 1;
    tc_fence_after();
    if (ok) {
      const float* lin = prm.lin_q ? prm.lin_q + grow * 128 : nullptr;
      const int t = 64 * i + tok;
      void* dst = t < prm.N ? grad_row(prm.dq, prm.g_dtype, prm.dq_sb, prm.dq_sh, prm.dq_sn, bh,
                                       prm.H, t)
                            : nullptr;
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {
        uint32_t o[32];
        tmem_ld16x64(tmem + lane_s + 128 + 64 * cb, o);
        tmem_ld_wait();
        float g[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          g[e] = __uint_as_float(o[e]) * kScale + (lin ? lin[64 * cb + kh + 2 * e] : 0.f);
        store_grad_chunk(g, cb, kh, dst, prm.g_dtype);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// dK, dV of one key block over the query blocks that keep it: S^T = K Q^T and dP^T = V dO^T
// (TMEM lanes 0-15 / 16-31, double-buffered in columns [0, 64) and [64, 128)),
// P^T = 2^(S^T c - L), dS^T = P^T (dP^T - D), dV += P^T dO (lanes 0-15) and dK += dS^T Q
// (lanes 16-31), columns [128, 256). Role warps ordered by mbarriers: warps 0-3 the softmax
// (P^T and dS^T into shared tiles), warp 4 issues S^T and warp 5 dP^T one query block ahead,
// warp 6 dV and dK, warp 7 loads K and V once and the Q / dO tiles of each query block into a
// two-stage ring, refilling a stage once the dV / dK MMAs of its block have completed. The
// softmax warpgroup takes 168 registers and the role warpgroup 56 (setmaxnreg; 4 x 32 x 168 +
// 4 x 32 x 56 = 28672 of the 256 x 128 a CTA is launched with). The seven tiles fill 112 KB
// exactly, so that two CTAs share an SM: the dynamic shared memory is declared 1024-byte
// aligned instead of being aligned by hand, and the kernel checks it. The linear-branch dk,
// dv are added before the stores.
constexpr int kDkvThreads = 256;
constexpr int kDkvSmem = 6 * kTile + 2 * kPTile;   // K, V, Q x 2, dO x 2, P^T, dS^T
constexpr int kDkvSoftmaxRegs = 168, kDkvRoleRegs = 56;
static_assert(4 * 32 * kDkvSoftmaxRegs + 4 * 32 * kDkvRoleRegs <= kDkvThreads * 128,
              "register split exceeds the launch's registers");

__global__ void __launch_bounds__(kDkvThreads, 2)
k_bwd_dkv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
          BwdParams prm) {
  extern __shared__ __align__(1024) uint8_t smem_dkv[];
  uint8_t* k_t = smem_dkv;                     // K tile
  uint8_t* v_t = smem_dkv + kTile;             // V tile
  uint8_t* q_t = smem_dkv + 2 * kTile;         // 2 Q stages
  uint8_t* o_t = smem_dkv + 4 * kTile;         // 2 dO stages
  uint8_t* p_t = smem_dkv + 6 * kTile;         // P^T tile
  uint8_t* s_t = smem_dkv + 6 * kTile + kPTile;   // dS^T tile
  __shared__ uint64_t kv_full, qo_full[2], s_done[2], s_free[2], p_full, acc_done[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  if (smem_u32(smem_dkv) & 1023u) {          // same for every thread of the CTA
    if (threadIdx.x == 0) record_error(prm.status, SAGESLA_ERR_DEVICE_CHECK);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int T = prm.tcount[bh * prm.nb + j];
  const int32_t* ilist = prm.tlist + bh * prm.nb * static_cast<int64_t>(prm.k) +
                         prm.toff[bh * (prm.nb + 1) + j];
  const int blk0 = static_cast<int>(bh * (prm.n_pad / 64));
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(&kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qo_full[s], 1);
      mbar_init(&s_done[s], 2);          // the S^T and the dP^T commit of a query block
      mbar_init(&s_free[s], 4);          // the four softmax warps have read S^T and dP^T
      mbar_init(&acc_done[s], 1);
    }
    mbar_init(&p_full, 4);               // the four softmax warps have stored P^T and dS^T
    abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;
  if (warp >= 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDkvRoleRegs));
    if (warp == 7) {
      // ---------------------------------------------- TMA producer
      if (lane == 0 && T > 0) {
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_do);
        mbar_arrive_expect_tx(&kv_full, 2 * kTile);
        load_tile(k_t, &tm_k, &kv_full, blk0 + j);
        load_tile(v_t, &tm_v, &kv_full, blk0 + j);
        for (int m = 0; m < T; ++m) {
          const int b = m & 1;
          // stage b held query block m - 2: its dV / dK MMAs must have completed
          if (m >= 2 && !bwd_wait(&acc_done[b], ((m - 2) >> 1) & 1, abort_flag, prm.status)) {
            ok = false;
            break;
          }
          const int ik = __ldg(ilist + m);
          if (!in_range(ik, prm.nb, prm.status)) {   // checking build: the tile is not loaded
            ok = false;
            break;
          }
          const int im = blk0 + ik;
          mbar_arrive_expect_tx(&qo_full[b], 2 * kTile);
          load_tile(q_t + b * kTile, &tm_q, &qo_full[b], im);
          load_tile(o_t + b * kTile, &tm_do, &qo_full[b], im);
        }
        if (!ok) abort_flag = 1;
      }
    } else if (warp == 6) {
      // ---------------------------------------------- dV and dK issuer
      if (lane == 0) {
        const uint32_t pa = smem_u32(p_t), sa = smem_u32(s_t);
        for (int n = 0; n < T; ++n) {
          ok = bwd_wait(&p_full, n & 1, abort_flag, prm.status);
          if (!ok) break;
          tc_fence_after();
          const int b = n & 1;
          const uint32_t ob = smem_u32(o_t + b * kTile), qb = smem_u32(q_t + b * kTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + 128, desc_k64(pa, kk), desc_mn128(ob, kk), kIdescKM128,
                     (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + (16u << 16) + 128, desc_k64(sa, kk), desc_mn128(qb, kk), kIdescKM128,
                     (n > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&acc_done[b]);
        }
        if (!ok) abort_flag = 1;
      }
    } else {
      // ---------------------------------------------- S^T (warp 4) and dP^T (warp 5) issuers
      if (lane == 0 && T > 0) {
        const bool is_s = warp == 4;
        const uint32_t a = smem_u32(is_s ? k_t : v_t);
        const uint32_t stage = smem_u32(is_s ? q_t : o_t);
        const uint32_t dbase = is_s ? tmem : tmem + (16u << 16);
        ok = mbar_wait(&kv_full, 0, prm.status);
        for (int n = 0; n < T && ok; ++n) {
          const int b = n & 1;
          // buffer b held query block n - 2: the softmax warps must have read it
          if (n >= 2) ok = bwd_wait(&s_free[b], ((n - 2) >> 1) & 1, abort_flag, prm.status);
          ok = ok && bwd_wait(&qo_full[b], (n >> 1) & 1, abort_flag, prm.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bsm = stage + b * kTile;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(dbase + 64 * b, desc_k128(a, kk), desc_k128(bsm, kk), kIdescKK64,
                     kk > 0 ? 1u : 0u);
          mma_commit(&s_done[b]);
        }
        if (!ok) abort_flag = 1;
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDkvSoftmaxRegs));
    // ------------------------------------------------ softmax warps
    const int row = frag_row(warp, lane);
    const int kh = (lane >> 1) & 1;
    const uint32_t lane_s = static_cast<uint32_t>(32 * warp) << 16;
    const uint32_t lane_p = static_cast<uint32_t>(32 * warp + 16) << 16;
    const float c2 = kScale * kLog2e;
    for (int n = 0; n < T; ++n) {
      const int b = n & 1;
      const int i = __ldg(ilist + n);
      // L and D of the query tokens 32kh + e of block i (this thread's columns)
      const int64_t qrow = bh * prm.n_pad + 64 * static_cast<int64_t>(i) + 32 * kh;
      float lq[32], dq_[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(prm.lse + qrow) + u);
        const float4 c = __ldg(reinterpret_cast<const float4*>(prm.dd + qrow) + u);
        lq[4 * u] = a.x; lq[4 * u + 1] = a.y; lq[4 * u + 2] = a.z; lq[4 * u + 3] = a.w;
        dq_[4 * u] = c.x; dq_[4 * u + 1] = c.y; dq_[4 * u + 2] = c.z; dq_[4 * u + 3] = c.w;
      }
      ok = bwd_wait(&s_done[b], (n >> 1) & 1, abort_flag, prm.status);
      ok = __all_sync(0xffffffffu, ok) != 0;      // the warp leaves together
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32], pr[32];
      tmem_ld16x64(tmem + lane_s + 64 * b, sr);
      tmem_ld16x64(tmem + lane_p + 64 * b, pr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      float pt[32], ds[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        pt[e] = ex2_approx(__uint_as_float(sr[e]) * c2 - lq[e]);
        ds[e] = pt[e] * (__uint_as_float(pr[e]) - dq_[e]);
      }
      // dV / dK of query block n - 1 have read the P^T and dS^T tiles
      if (n >= 1) {
        ok = bwd_wait(&acc_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, prm.status);
        ok = __all_sync(0xffffffffu, ok) != 0;
        if (!ok) break;
      }
      store_row_operand(p_t, row, kh, pt);
      store_row_operand(s_t, row, kh, ds);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full);
    }
    if (ok && T > 0) ok = mbar_wait(&acc_done[(T - 1) & 1], ((T - 1) >> 1) & 1, prm.status);
    ok = __all_sync(0xffffffffu, ok) != 0;
    if (!ok) abort_flag = 1;
    tc_fence_after();
    if (ok) {
      const int tok = tile_token(row);
      const int t_key = 64 * j + tok;
      const int64_t grow = bh * prm.n_pad + t_key;
      const bool real = t_key < prm.N;
      void* dst_k = real ? grad_row(prm.dk, prm.g_dtype, prm.dk_sb, prm.dk_sh, prm.dk_sn, bh,
                                    prm.H, t_key)
                         : nullptr;
      void* dst_v = real ? grad_row(prm.dv, prm.g_dtype, prm.dv_sb, prm.dv_sh, prm.dv_sn, bh,
                                    prm.H, t_key)
                         : nullptr;
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {
        uint32_t ov[32], okk[32];
        if (T > 0) {
          tmem_ld16x64(tmem + lane_s + 128 + 64 * cb, ov);
          tmem_ld16x64(tmem + lane_p + 128 + 64 * cb, okk);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) { ov[e] = 0u; okk[e] = 0u; }
        }
        float gk[32], gv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = 64 * cb + kh + 2 * e;
          gv[e] = __uint_as_float(ov[e]) + (prm.lin_v ? prm.lin_v[grow * 128 + c] : 0.f);
          gk[e] = __uint_as_float(okk[e]) * kScale + (prm.lin_k ? prm.lin_k[grow * 128 + c] : 0.f);
        }
        store_grad_chunk(gk, cb, kh, dst_k, prm.g_dtype);
        store_grad_chunk(gv, cb, kh, dst_v, prm.g_dtype);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------ linear branch (tcgen05)

// A [129][128] state block (G_i or dH_j, bf16 [n][c]) lives in shared memory as rows n < 128
// only, two 16 KB chunks of 64 channels (128-byte swizzled), loaded by TMA; row 128 is read
// from global memory. As a B operand it is K-major with K = c (N = n) or MN-major with K = n
// (N = c).
__device__ __forceinline__ uint64_t desc_state_kmajor(uint32_t base, int kk) {   // K = c
  return make_sdesc(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
}
__device__ __forceinline__ uint64_t desc_state_mnmajor(uint32_t base, int kk) {  // K = n
  return make_sdesc(base + kk * 2048, 16384, 1024, kLayoutSW128);
}
constexpr uint32_t kStateTile = 2 * 16384;
constexpr uint32_t kIdescMM128 = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 1, 1, 128, 128);
constexpr uint32_t kIdescKK128 = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 0, 64, 128);

// This thread's half of phi over a packed bf16 row (channels 64 kh .. 64 kh + 63; the row's
// other half is lane ^ 2) into the K-major A tile (chunk kh of row r) and the f32 copy a32.
__device__ __forceinline__ void phi_half_row(const uint16_t* row, int r, int kh, uint8_t* tile,
                                             float* a32) {
  const uint4* r4 = reinterpret_cast<const uint4*>(row) + 8 * kh;
  float x[64];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint4 w = __ldg(r4 + u);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int z = 0; z < 4; ++z) {
      x[8 * u + 2 * z] = bf16_bits_to_f32(ww[z] & 0xFFFFu);
      x[8 * u + 2 * z + 1] = bf16_bits_to_f32(ww[z] >> 16);
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < 64; ++e) mx = fmaxf(mx, x[e]);
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < 64; ++e) { x[e] = __expf(x[e] - mx); sum += x[e]; }
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  const float inv = 1.f / sum;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int z = 0; z < 4; ++z) {
      const float lo = x[8 * u + 2 * z] * inv, hi = x[8 * u + 2 * z + 1] * inv;
      a32[r * 132 + 64 * kh + 8 * u + 2 * z] = lo;
      a32[r * 132 + 64 * kh + 8 * u + 2 * z + 1] = hi;
      w[z] = pack_bf16x2(lo, hi);
    }
    *reinterpret_cast<uint4*>(tile + kh * 8192 + sw128_offset(r, u)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// This thread's 64 values of row r of a 64 x 128 K-major bf16 operand (columns 64cb + kh + 2e
// in x[cb][e]) written after an exchange with lane ^ 2, 32 contiguous columns per chunk.
__device__ __forceinline__ void store_row128(uint8_t* tile, int r, int kh, const float (&x)[2][32]) {
#pragma unroll
  for (int cb = 0; cb < 2; ++cb) {
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      float w4[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float mine0 = x[cb][e + u], mine1 = x[cb][16 + e + u];
        const float recv = __shfl_xor_sync(0xffffffffu, kh ? mine0 : mine1, 2);
        w4[2 * u] = kh ? recv : mine0;
        w4[2 * u + 1] = kh ? mine1 : recv;
      }
      w[e] = pack_bf16x2(w4[0], w4[1]);
      w[e + 1] = pack_bf16x2(w4[2], w4[3]);
    }
    // columns 64cb + 32kh .. +31 = 16-byte chunks 4kh .. 4kh + 3 of chunk cb's row
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(tile + cb * 8192 + sw128_offset(r, 4 * kh + c)) =
          make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
  }
}

constexpr int kLinThreads = 128;
constexpr int kLinSmem = 1024 + 2 * kTile + kStateTile + 64 * 132 * 4 + 129 * 4 + 64 * 4;

// Query side of the linear branch for one query block (M=64 rows = tokens in order):
//   num = phi(Q) G[:, :128]          (tcgen05, TMEM lanes 0-15, columns [0, 128))
//   den = phi(q) . G[:, 128], dnum = dO / den, dden = -(dO . num) / den^2
//   da = dnum G[:, :128]^T           (lanes 16-31, columns [0, 128)) + dden G[:, 128]
//   dq_l = phi(q) * da;   dG = phi(Q)^T [dnum | dden]   (M=128 over channels, columns [128, 256))
__global__ void __launch_bounds__(kLinThreads, 2)
k_bwd_lin_query(const __grid_constant__ CUtensorMap tm_g, const uint16_t* __restrict__ qn,
                const uint16_t* __restrict__ dn, const uint16_t* __restrict__ gsum, int nb,
                int nb_m_pad, int n_pad, float* __restrict__ lin_q, uint16_t* __restrict__ dgsum,
                int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* a_t = smem;                               // phi(Q) bf16 [t][c]
  uint8_t* n_t = smem + kTile;                       // dnum bf16 [t][n]
  uint8_t* g_t = smem + 2 * kTile;                   // G rows n < 128
  float* a32 = reinterpret_cast<float*>(smem + 2 * kTile + kStateTile);   // [64][132]
  float* g128 = a32 + 64 * 132;                      // G[128][c]
  float* dden_s = g128 + 129;                        // [64]
  __shared__ uint64_t g_full, mma1, mma2;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int64_t grow0 = (bh * nb_m_pad + i) * 129;   // first state row of block i
  uint16_t* dg = dgsum + grow0 * 128;
  if (i >= nb) {   // padding rows of the transposed complement GEMM operand
    for (int e = threadIdx.x; e < kHFlat; e += kLinThreads) dg[e] = 0;
    return;
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(&g_full, 1); mbar_init(&mma1, 1); mbar_init(&mma2, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&g_full, kStateTile);
    tma_load_2d(g_t, &tm_g, &g_full, 0, static_cast<int>(grow0));
    tma_load_2d(g_t + 16384, &tm_g, &g_full, 64, static_cast<int>(grow0));
  }
  g128[threadIdx.x] = bf16_bits_to_f32(gsum[(grow0 + 128) * 128 + threadIdx.x]);
  const int r = frag_row(warp, lane);
  const int kh = (lane >> 1) & 1;
  const int64_t trow = bh * n_pad + 64 * static_cast<int64_t>(i) + r;
  phi_half_row(qn + trow * 128, r, kh, a_t, a32);
  __syncthreads();                                   // g128 and a32 complete
  float den = 0.f;
#pragma unroll 8
  for (int c = 64 * kh; c < 64 * kh + 64; ++c) den = fmaf(a32[r * 132 + c], g128[c], den);
  den += __shfl_xor_sync(0xffffffffu, den, 2);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (threadIdx.x == 0) {
    ok = mbar_wait(&g_full, 0, status);
    if (ok) {
      tc_fence_after();
      const uint32_t aa = smem_u32(a_t), gb = smem_u32(g_t);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem, desc_k128(aa, kk), desc_state_kmajor(gb, kk), kIdescKK128, kk > 0 ? 1u : 0u);
      mma_commit(&mma1);
    }
  }
  ok = mbar_wait(&mma1, 0, status);
  tc_fence_after();
  const uint32_t lane_a = static_cast<uint32_t>(32 * warp) << 16;
  const uint32_t lane_b = static_cast<uint32_t>(32 * warp + 16) << 16;
  float dnum[2][32];
  float dpart = 0.f;
  {
    const uint4* d4 = reinterpret_cast<const uint4*>(dn + trow * 128);
    const float inv_den = 1.f / den;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t o[32];
      tmem_ld16x64(tmem + lane_a + 64 * cb, o);
      tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint4 w = __ldg(d4 + 8 * cb + u);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const int e = 4 * u + z;
          const float dov = bf16_bits_to_f32(kh ? (ww[z] >> 16) : (ww[z] & 0xFFFFu));
          dpart = fmaf(dov, __uint_as_float(o[e]), dpart);
          dnum[cb][e] = dov * inv_den;
        }
      }
    }
  }
  dpart += __shfl_xor_sync(0xffffffffu, dpart, 2);
  const float dden = -dpart / (den * den);
  if (kh == 0) dden_s[r] = dden;
  store_row128(n_t, r, kh, dnum);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    const uint32_t nb_ = smem_u32(n_t), gb = smem_u32(g_t), aa = smem_u32(a_t);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)   // da = dnum G^T: K = n (128)
      mma_bf16(tmem + (16u << 16), desc_k128(nb_, kk), desc_state_mnmajor(gb, kk), kIdescKM128,
               kk > 0 ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)   // dG = phi(Q)^T dnum: M = c, N = n, K = t (64)
      mma_bf16(tmem + 128, desc_mn128(aa, kk), desc_mn128(nb_, kk), kIdescMM128,
               kk > 0 ? 1u : 0u);
    mma_commit(&mma2);
  }
  ok = ok && mbar_wait(&mma2, 0, status);
  tc_fence_after();
  if (ok) {
    // dq_l = phi(q) * (da + dden G[:, 128])
#pragma unroll 1
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t o[32];
      tmem_ld16x64(tmem + lane_b + 64 * cb, o);
      tmem_ld_wait();
      float g[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int c = 64 * cb + kh + 2 * e;
        g[e] = a32[r * 132 + c] * (__uint_as_float(o[e]) + dden * g128[c]);
      }
      store_grad_chunk(g, cb, kh, lin_q + trow * 128, SAGESLA_F32);
    }
    // dG rows n < 128: TMEM lane c = 32 warp + lane, columns 128 + n; row 128 = sum_t a dden
    const int c = 32 * warp + lane;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t o[32];
      tmem_ld32(tmem_addr(tmem, 32 * warp, 128 + 32 * cc), o);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e)
        dg[(32 * cc + e) * 128 + c] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(o[e])));
    }
    float s128 = 0.f;
#pragma unroll 8
    for (int t = 0; t < 64; ++t) s128 = fmaf(a32[t * 132 + c], dden_s[t], s128);
    dg[128 * 128 + c] = __bfloat16_as_ushort(__float2bfloat16_rn(s128));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// Key side of the linear branch for one key block (rows = tokens in order), b = phi(k):
//   db = V dH[:, :128]^T (lanes 0-15) + dH[:, 128];  dv_l = b dH[:, :128] (lanes 16-31);
//   dk_l = b * (db - b . db).
__global__ void __launch_bounds__(kLinThreads, 2)
k_bwd_lin_key(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_vn,
              const uint16_t* __restrict__ kn, const uint16_t* __restrict__ dhsum, int nb_m_pad,
              int n_pad, float* __restrict__ lin_k, float* __restrict__ lin_v, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* b_t = smem;                               // phi(K) bf16 [t][c]
  uint8_t* v_t = smem + kTile;                       // V bf16 [t][n]
  uint8_t* h_t = smem + 2 * kTile;                   // dH rows n < 128
  float* b32 = reinterpret_cast<float*>(smem + 2 * kTile + kStateTile);   // [64][132]
  float* h128 = b32 + 64 * 132;                      // dH[128][c]
  __shared__ uint64_t ld_full, mma1;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int64_t hrow0 = (bh * nb_m_pad + j) * 129;
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 128);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(&ld_full, 1); mbar_init(&mma1, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int64_t trow0 = bh * n_pad + 64 * static_cast<int64_t>(j);
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&ld_full, kStateTile + kTile);
    tma_load_2d(h_t, &tm_h, &ld_full, 0, static_cast<int>(hrow0));
    tma_load_2d(h_t + 16384, &tm_h, &ld_full, 64, static_cast<int>(hrow0));
    tma_load_2d(v_t, &tm_vn, &ld_full, 0, static_cast<int>(trow0));
    tma_load_2d(v_t + 8192, &tm_vn, &ld_full, 64, static_cast<int>(trow0));
  }
  h128[threadIdx.x] = bf16_bits_to_f32(dhsum[(hrow0 + 128) * 128 + threadIdx.x]);
  const int r = frag_row(warp, lane);
  const int kh = (lane >> 1) & 1;
  const int64_t trow = trow0 + r;
  phi_half_row(kn + trow * 128, r, kh, b_t, b32);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (threadIdx.x == 0) {
    ok = mbar_wait(&ld_full, 0, status);
    if (ok) {
      tc_fence_after();
      const uint32_t va = smem_u32(v_t), ba = smem_u32(b_t), hb = smem_u32(h_t);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)   // db = V dH^T: K = n
        mma_bf16(tmem, desc_k128(va, kk), desc_state_mnmajor(hb, kk), kIdescKM128, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)   // dv = b dH: K = c
        mma_bf16(tmem + (16u << 16), desc_k128(ba, kk), desc_state_kmajor(hb, kk), kIdescKK128,
                 kk > 0 ? 1u : 0u);
      mma_commit(&mma1);
    }
  }
  ok = mbar_wait(&mma1, 0, status);
  tc_fence_after();
  if (ok) {
    const uint32_t lane_a = static_cast<uint32_t>(32 * warp) << 16;
    const uint32_t lane_b = static_cast<uint32_t>(32 * warp + 16) << 16;
    float db[2][32];
    float proj = 0.f;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t o[32];
      tmem_ld16x64(tmem + lane_a + 64 * cb, o);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int c = 64 * cb + kh + 2 * e;
        db[cb][e] = __uint_as_float(o[e]) + h128[c];
        proj = fmaf(b32[r * 132 + c], db[cb][e], proj);
      }
    }
    proj += __shfl_xor_sync(0xffffffffu, proj, 2);
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      float g[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int c = 64 * cb + kh + 2 * e;
        g[e] = b32[r * 132 + c] * (db[cb][e] - proj);
      }
      store_grad_chunk(g, cb, kh, lin_k + trow * 128, SAGESLA_F32);
    }
#pragma unroll 1
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t o[32];
      tmem_ld16x64(tmem + lane_b + 64 * cb, o);
      tmem_ld_wait();
      float g[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) g[e] = __uint_as_float(o[e]);
      store_grad_chunk(g, cb, kh, lin_v + trow * 128, SAGESLA_F32);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace

bool make_backward_layout(const ForwardPlan& p, BackwardLayout* bl) {
  size_t off = p.lay.total_bytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) & ~static_cast<size_t>(255);
    return at;
  };
  const size_t rows = static_cast<size_t>(p.BH * p.n_pad);
  bl->qn = take(rows * 256);
  bl->kn = take(rows * 256);
  bl->vn = take(rows * 256);
  bl->dn = take(rows * 256);
  bl->lse = take(rows * 4);
  bl->dd = take(rows * 4);
  bl->tcount = take(static_cast<size_t>(p.BH * p.nb) * 4);
  bl->toff = take(static_cast<size_t>(p.BH * (p.nb + 1)) * 4);
  bl->tlist = take(static_cast<size_t>(p.BH * p.nb * p.k) * 4);
  if (!p.linear_empty) {
    bl->lin_q = take(rows * 512);
    bl->lin_k = take(rows * 512);
    bl->lin_v = take(rows * 512);
    bl->amask_t = take(static_cast<size_t>(p.BH * p.nb_m_pad * p.nb_m_pad) * 2);
    bl->dg = take(static_cast<size_t>(p.BH * p.nb_m_pad) * kHFlat * 2);
    bl->dh = take(static_cast<size_t>(p.BH * p.nb_m_pad) * kHFlat * 2);
  } else {
    bl->lin_q = bl->lin_k = bl->lin_v = bl->amask_t = bl->dg = bl->dh = 0;
  }
  bl->total = off;
  return true;
}

namespace {

// Four-dimensional map of a packed [rows][128] bf16 buffer whose box is one key-interleaved
// 64 x 64 tile: dims (column, half, row in half, 64-row block), strides 32 rows, 1 row and 64
// rows, box (64, 2, 32, 1); the box lands in shared memory as rows 2i + h <- token 32h + i.
bool encode_interleaved(CUtensorMap* map, const void* base, int64_t rows) {
  const uint64_t dims[4] = {128, 2, 32, static_cast<uint64_t>(rows / 64)};
  const uint64_t strides[3] = {32 * 256, 256, 64 * 256};
  const uint32_t box[4] = {64, 2, 32, 1};
  return encode_tmap_nd(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_sla_backward(const ForwardPlan& p, const BackwardLayout& bl, TensorArg q,
                                TensorArg k, TensorArg v, TensorArg d_out, const GradOut& g,
                                char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  const int64_t rows = p.BH * p.n_pad;
  cudaError_t e;
  // packed copies, transposed kept lists
  {
    const int64_t total = rows * 16;
    k_bwd_pack<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
        q, k, v, d_out, static_cast<int>(p.N), static_cast<int>(p.n_pad), total,
        reinterpret_cast<uint4*>(ws + bl.qn), reinterpret_cast<uint4*>(ws + bl.kn),
        reinterpret_cast<uint4*>(ws + bl.vn), reinterpret_cast<uint4*>(ws + bl.dn));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t warps = p.BH * p.nb;
    const unsigned lgrid = static_cast<unsigned>((warps * 32 + 255) / 256);
    const uint32_t* mask = reinterpret_cast<const uint32_t*>(ws + L.mask);
    k_bwd_list_count<<<lgrid, 256, 0, stream>>>(static_cast<int>(p.nb), static_cast<int>(p.mask_words),
                                                p.BH, mask, reinterpret_cast<int32_t*>(ws + bl.tcount));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_list_scan<<<static_cast<unsigned>(p.BH), 1024, 0, stream>>>(
        static_cast<int>(p.nb), reinterpret_cast<const int32_t*>(ws + bl.tcount),
        reinterpret_cast<int32_t*>(ws + bl.toff));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_list_fill<<<lgrid, 256, 0, stream>>>(static_cast<int>(p.nb), static_cast<int>(p.k),
                                               static_cast<int>(p.mask_words), p.BH, mask,
                                               reinterpret_cast<const int32_t*>(ws + bl.toff),
                                               reinterpret_cast<int32_t*>(ws + bl.tlist),
                                               reinterpret_cast<int*>(ws + p.lay.status));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  CUtensorMap tq, tk, tv, td;
  if (!encode_interleaved(&tq, ws + bl.qn, rows) || !encode_interleaved(&tk, ws + bl.kn, rows) ||
      !encode_interleaved(&tv, ws + bl.vn, rows) || !encode_interleaved(&td, ws + bl.dn, rows))
    return cudaErrorInvalidValue;
  BwdParams prm;
  prm.kept = reinterpret_cast<const int32_t*>(ws + L.kept);
  prm.tcount = reinterpret_cast<const int32_t*>(ws + bl.tcount);
  prm.toff = reinterpret_cast<const int32_t*>(ws + bl.toff);
  prm.tlist = reinterpret_cast<const int32_t*>(ws + bl.tlist);
  prm.qn = reinterpret_cast<const uint16_t*>(ws + bl.qn);
  prm.dn = reinterpret_cast<const uint16_t*>(ws + bl.dn);
  prm.lse = reinterpret_cast<float*>(ws + bl.lse);
  prm.dd = reinterpret_cast<float*>(ws + bl.dd);
  prm.lin_q = p.linear_empty ? nullptr : reinterpret_cast<const float*>(ws + bl.lin_q);
  prm.lin_k = p.linear_empty ? nullptr : reinterpret_cast<const float*>(ws + bl.lin_k);
  prm.lin_v = p.linear_empty ? nullptr : reinterpret_cast<const float*>(ws + bl.lin_v);
  prm.dq = g.dq; prm.dk = g.dk; prm.dv = g.dv;
  prm.dq_sb = g.dq_s[0]; prm.dq_sh = g.dq_s[1]; prm.dq_sn = g.dq_s[2];
  prm.dk_sb = g.dk_s[0]; prm.dk_sh = g.dk_s[1]; prm.dk_sn = g.dk_s[2];
  prm.dv_sb = g.dv_s[0]; prm.dv_sh = g.dv_s[1]; prm.dv_sn = g.dv_s[2];
  prm.g_dtype = g.dtype;
  prm.status = reinterpret_cast<int*>(ws + L.status);
  prm.N = static_cast<int>(p.N);
  prm.nb = static_cast<int>(p.nb);
  prm.n_pad = static_cast<int>(p.n_pad);
  prm.k = static_cast<int>(p.k);
  prm.n_last = p.n_last;
  prm.H = static_cast<int>(p.H);
  const dim3 grid(static_cast<unsigned>(p.nb), static_cast<unsigned>(p.BH));
  const int smem_lse = 1024 + 6 * kTile;
  const int smem_dq = 6 * kTile + 2 * kPTile;
  const int smem_dkv = kDkvSmem;
  // set on every call: the attribute belongs to the current device
  if ((e = cudaFuncSetAttribute(k_bwd_lse, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_lse)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(k_bwd_dq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(k_bwd_dkv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dkv)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(k_bwd_lin_query, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinSmem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(k_bwd_lin_key, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinSmem)) != cudaSuccess)
    return e;
  k_bwd_lse<<<grid, kLseThreads, smem_lse, stream>>>(tq, td, tk, tv, prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (!p.linear_empty) {
    CUtensorMap tg, th, tvn;
    if (!encode_tmap_2d(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128,
                        static_cast<uint64_t>(p.BH * p.nb_m_pad * 129), 256, ws + L.gsum, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128,
                        static_cast<uint64_t>(p.BH * p.nb_m_pad * 129), 256, ws + bl.dh, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(&tvn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, static_cast<uint64_t>(rows),
                        256, ws + bl.vn, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const dim3 gq(static_cast<unsigned>(p.nb_m_pad), static_cast<unsigned>(p.BH));
    k_bwd_lin_query<<<gq, kLinThreads, kLinSmem, stream>>>(
        tg, prm.qn, prm.dn, reinterpret_cast<const uint16_t*>(ws + L.gsum), static_cast<int>(p.nb),
        static_cast<int>(p.nb_m_pad), static_cast<int>(p.n_pad),
        reinterpret_cast<float*>(ws + bl.lin_q), reinterpret_cast<uint16_t*>(ws + bl.dg),
        prm.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 gt(static_cast<unsigned>(p.nb_m_pad / 32), static_cast<unsigned>(p.nb_m_pad / 32),
                  static_cast<unsigned>(p.BH));
    k_bwd_transpose_mask<<<gt, dim3(32, 8), 0, stream>>>(
        static_cast<int>(p.nb_m_pad), static_cast<int>(p.nb_k_pad),
        reinterpret_cast<const uint16_t*>(ws + L.amask), reinterpret_cast<uint16_t*>(ws + bl.amask_t));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dH = (1 - M)^T dG: the complement GEMM with the transposed mask, rows and depth nb_m_pad
    if ((e = launch_mask_gemm(ws + bl.amask_t, ws + bl.dg, ws + bl.dh, p.BH, p.nb_m_pad,
                              p.nb_m_pad, prm.status, stream)) != cudaSuccess)
      return e;
    const dim3 gk(static_cast<unsigned>(p.nb), static_cast<unsigned>(p.BH));
    k_bwd_lin_key<<<gk, kLinThreads, kLinSmem, stream>>>(
        th, tvn, reinterpret_cast<const uint16_t*>(ws + bl.kn),
        reinterpret_cast<const uint16_t*>(ws + bl.dh), static_cast<int>(p.nb_m_pad),
        static_cast<int>(p.n_pad), reinterpret_cast<float*>(ws + bl.lin_k),
        reinterpret_cast<float*>(ws + bl.lin_v), prm.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  k_bwd_dq<<<grid, kDqThreads, smem_dq, stream>>>(tq, tk, tv, td, prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_bwd_dkv<<<grid, kDkvThreads, smem_dkv, stream>>>(tq, tk, tv, td, prm);
  return cudaGetLastError();
}

}  // namespace sagesla
