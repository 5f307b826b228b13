// Sparse branch of the SageSLA forward (INT8 Q.K^T, FP8 P.V on tcgen05) with the linear
// branch's query-side contraction fused into the epilogue.
//
// Method: news.qq.com TurboDiffusion article, section 第一把钥匙 — exact attention only on the
// kept block pairs (Top-K ratio 0.1), with SageAttention's 8-bit operands on the tensor cores;
// the remaining blocks go through linear attention ("Sparse-Linear Attention", dgmzs.com.cn
// README translation, section 方法论). For a query row t of block i and kept blocks j in
// ascending order:
//     S = (Q8 K8^T) sq_i sk_j / sqrt(128);  m' = max(m, rowmax S);  p = exp(S - m');
//     l = e^(m-m') l + sum p;   o = e^(m-m') o + e4m3(448 p) . V8;   m = m'
//     out = o s_v / (448 l) + phi(q) G_i[:, :128] / phi(q) G_i[:, 128]
//
// B200 mapping. One CTA per PAIR of adjacent query blocks (128 rows = the tcgen05 M=128 tile)
// walking the union of the two blocks' kept lists; rows of a block that does not keep the
// current key block get P = 0 and skip their softmax work. Warp roles:
//   warps 0-7  softmax / correction / epilogue: two threads per query row (TMEM lane = row),
//              warp w exponentiates S columns 32*(w/4) .. +31 (both threads of a row read
//              all 64 for the block maximum) and owns O columns 64*(w/4) .. +63
//   warp 8     TMA producer: Q tile once, then K8/V8 tiles through a 4-stage ring
//   warp 9     MMA issuer: S(n) = Q K_j^T (kind::i8, M128 N64 K128) into one of two S
//              buffers, then O += P(n-1) V (kind::f8f6f4, M128 N128 K64) — S(n+1) overlaps
//              the softmax of n.
// TMEM (256 columns): O fp32 [0,128), S int32 [128,192) and [192,256); after the loop the S
// columns hold phi(Q) . G for the linear branch. Two CTAs fit on an SM.
//
// Softmax arithmetic per score: the int32 score becomes a float exactly through the 1.5*2^23
// bias (integer add, float subtract: no conversion-pipe instruction); one FFMA forms the
// base-2 exponent with the factor 448 of the P quantization folded in; 2^x comes from the
// MUFU ex2 unit for most columns and, for the rest, from Cody-Waite range reduction (round
// to nearest integer) plus a degree-5 polynomial fitted here by the Remez exchange algorithm
// for minimax relative error on [-1/2, 1/2] (max relative error 2.3e-7 in fp32), so that the
// FMA pipe takes part of the exponential load of the MUFU unit.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kNS = 4;                       // K/V ring stages
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr uint32_t kQBytes = 128 * 128;      // int8 Q tile
constexpr uint32_t kKVBytes = 64 * 128;      // one K8 or V8 tile
constexpr uint32_t kStageBytes = 2 * kKVBytes;
// e4m3 P tile, K-major without swizzle: core matrices of 8 rows x 16 keys (128 B); K-chunks
// 160 B apart and 8-row groups 672 B apart. The padding makes the 16-byte stores of the
// softmax threads (lanes of one store phase hold rows r, r+8, r+1, r+9 and key halves 0, 1)
// fall on eight distinct bank groups.
constexpr uint32_t kPChunk = 160, kPGroup = 672;
constexpr uint32_t kPBytes = 16 * kPGroup;
constexpr uint32_t kOffStages = kQBytes;
constexpr uint32_t kOffP = kOffStages + kNS * kStageBytes;
constexpr uint32_t kOffCtl = kOffP + 2 * kPBytes;
static_assert(kOffCtl >= 96 * 1024, "the linear epilogue reuses [0, 96 KB) for its operands");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemS = 128;              // first S buffer column
// Columns of each thread's 32 whose exponential uses the polynomial instead of MUFU ex2.
constexpr int kPolyFrom = 28;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kInvSqrtD = 0.08838834764831845f;
constexpr float kLog2_448 = 8.807354922057604f;

struct Ctl {
  uint64_t full[kNS], empty[kNS];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t q_full, g_full, a_full, la_done, la_free, lb_done, mma_done;
  uint32_t tmem_base;
  int list_len;
  volatile int abort;
  float s_v[128];
  float xf[2][128];          // [column half][row]: epilogue exchanges
  float xd[2][128];
};

struct AttnParams {
  const float* sq;            // [BH][nbq]
  const float* sk;            // [BH][nbq]
  const float* s_v;           // [BH][128]
  const uint32_t* mask;       // [BH][nb][mask_words]
  const __nv_bfloat16* gsum;  // [BH][nb_m_pad][129][128]
  TensorArg q;                // raw bf16 Q (for phi(q))
  void* out;
  int64_t out_sb, out_sh, out_sn;
  int32_t out_dtype;
  float* sparse_out;          // optional [BH][N][128]
  int* status;
  int N, nb, nbq, n_pad, mask_words, nb_m_pad, n_last, list_cap;
  int linear;                 // 0 when every key block is kept
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Ctl* ctl,
                                              int* status) {
  if (ctl->abort) return false;
  if (!mbar_wait(bar, parity, status)) {
    ctl->abort = 1;
    return false;
  }
  return true;
}

// Named barrier for the two warps (64 threads) that share a group of 32 rows. Used only in
// the epilogue, where both threads of a row execute it the same number of times on every
// path (a named barrier cannot time out).
__device__ __forceinline__ void pair_sync(int id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

// int32 -> float, exact for |s| < 2^22 (the INT8 product of a 128-channel row is < 2^21).
__device__ __forceinline__ float s32_to_f32(uint32_t s) {
  return __int_as_float(static_cast<int>(s + 0x4B400000u)) - 12582912.0f;
}

__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe: x = n + f with n = rint(x), f in [-1/2, 1/2]; 2^f by a degree-5
// minimax polynomial (coefficients from a Remez fit of relative error); 2^n added to the
// exponent field. x is clamped below at -125 so that the result stays a normal float.
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;              // rint(x) in the low mantissa bits
  const float f = x - (t - 12582912.0f);
  float p = fmaf(0.0013276472454890609f, f, 0.009675540961325169f);
  p = fmaf(p, f, 0.05550713092088699f);
  p = fmaf(p, f, 0.24022120237350464f);
  p = fmaf(p, f, 0.6931469440460205f);
  p = fmaf(p, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Maximum of this thread's valid scores (eight independent chains).
template <bool kFull>
__device__ __forceinline__ int row_block_max(const uint32_t (&a)[32], int valid) {
  int m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = INT_MIN;
#pragma unroll
  for (int q = 0; q < 32; ++q)
    if (kFull || q < valid) m[q & 7] = max(m[q & 7], static_cast<int>(a[q]));
  return max(max(max(m[0], m[1]), max(m[2], m[3])), max(max(m[4], m[5]), max(m[6], m[7])));
}

// 448 p = 2^(S c + neg), neg = log2(448) - m, for this thread's 32 scores -> packed e4m3
// codes and their sum.
template <bool kFull>
__device__ __forceinline__ float row_exp_pack(const uint32_t (&sr)[32], int valid, float c,
                                              float neg, uint32_t (&pk)[8]) {
  float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
  for (int q = 0; q < 32; q += 4) {
    float y[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float x = fmaf(s32_to_f32(sr[q + t]), c, neg);
      float v = (q + t < kPolyFrom) ? ex2_mufu(x) : ex2_poly(x);
      if (!kFull && q + t >= valid) v = 0.f;
      y[t] = v;
    }
    r0 += y[0];
    r1 += y[1];
    r2 += y[2];
    r3 += y[3];
    pk[q >> 2] = static_cast<uint32_t>(f32x2_to_e4m3x2(y[0], y[1])) |
                 (static_cast<uint32_t>(f32x2_to_e4m3x2(y[2], y[3])) << 16);
  }
  return (r0 + r1) + (r2 + r3);
}

__global__ void __launch_bounds__(kThreads, 2)
k_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
            AttnParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + kOffCtl);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + kOffCtl + sizeof(Ctl));
  float* list_sk = reinterpret_cast<float*>(list + prm.list_cap);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int ia = 2 * pair, ib = 2 * pair + 1;     // the two query blocks
  int* status = prm.status;

  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
    // union of the two kept lists, ascending; flags bit0 = kept by ia, bit1 = kept by ib
    const uint32_t* ma = prm.mask + (bh * prm.nb + ia) * prm.mask_words;
    const uint32_t* mb = ib < prm.nb ? prm.mask + (bh * prm.nb + ib) * prm.mask_words : nullptr;
    int base = 0;
    for (int w0 = 0; w0 < prm.mask_words; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t a = w < prm.mask_words ? ma[w] : 0u;
      const uint32_t b = (w < prm.mask_words && mb) ? mb[w] : 0u;
      uint32_t u = a | b;
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nv = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nv;
      }
      int pos = base + incl - cnt;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        const int j = 32 * w + bit;
        const uint32_t fl = ((a >> bit) & 1u) | (((b >> bit) & 1u) << 1);
        if (pos < prm.list_cap) {
          list[pos] = static_cast<uint32_t>(j) | (fl << 24);
          list_sk[pos] = prm.sk[bh * prm.nbq + j];
        }
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) ctl->list_len = min(base, prm.list_cap);
  } else if (warp == 1) {
    for (int c = lane; c < 128; c += 32) ctl->s_v[c] = prm.s_v[bh * 128 + c];
  } else if (threadIdx.x == 64) {
    for (int s = 0; s < kNS; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_free[s], kSoftmaxWarps);
      mbar_init(&ctl->p_full[s], kSoftmaxWarps);
      mbar_init(&ctl->pv_done[s], 1);
    }
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->g_full, 1);
    mbar_init(&ctl->a_full, kSoftmaxThreads);
    mbar_init(&ctl->la_done, 1);
    mbar_init(&ctl->la_free, kSoftmaxThreads / 2);
    mbar_init(&ctl->lb_done, 1);
    mbar_init(&ctl->mma_done, 1);
    ctl->abort = 0;
    fence_mbar_init();
  } else if (threadIdx.x == 96) {
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_g);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int U = ctl->list_len;
  const bool has_b = ib < prm.nb;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int row_base = static_cast<int>(bh * prm.n_pad);
      mbar_arrive_expect_tx(&ctl->q_full, kQBytes);
      tma_load_2d(smem, &tm_q, &ctl->q_full, 0, row_base + 128 * pair);
      for (int n = 0; n < U; ++n) {
        const int s = n % kNS;
        if (n >= kNS && !wait_or_abort(&ctl->empty[s], ((n / kNS) - 1) & 1, ctl, status)) break;
        const int j = static_cast<int>(list[n] & 0xFFFFFFu);
        uint8_t* st = smem + kOffStages + s * kStageBytes;
        mbar_arrive_expect_tx(&ctl->full[s], kStageBytes);
        tma_load_2d(st, &tm_k, &ctl->full[s], 0, row_base + 64 * j);
        tma_load_2d(st + kKVBytes, &tm_v, &ctl->full[s], 0, row_base + 64 * j);
      }
      // A parity wait only tells the last two phases apart, and this thread has not observed
      // the earlier P.V phases, so it waits on the single-phase "all MMAs of the loop done".
      if (prm.linear && wait_or_abort(&ctl->mma_done, 0, ctl, status)) {
        // The whole operand area is free now: G_ia -> [32K, 64K), G_ib -> [64K, 96K).
        const int gy = static_cast<int>((bh * prm.nb_m_pad + ia) * 129);
        mbar_arrive_expect_tx(&ctl->g_full, has_b ? 65536u : 32768u);
        tma_load_2d(smem + 32768, &tm_g, &ctl->g_full, 0, gy);
        tma_load_2d(smem + 32768 + 16384, &tm_g, &ctl->g_full, 64, gy);
        if (has_b) {
          tma_load_2d(smem + 65536, &tm_g, &ctl->g_full, 0, gy + 129);
          tma_load_2d(smem + 65536 + 16384, &tm_g, &ctl->g_full, 64, gy + 129);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc(kFmtS32, kFmtS8, kFmtS8, 0, 0, 128, 64);
      constexpr uint32_t idesc_pv = make_idesc(kFmtF32, kFmtE4M3, kFmtE4M3, 0, 1, 128, 128);
      const uint32_t q_addr = smem_u32(smem);
      auto issue_pv = [&](int m) -> bool {
        const int b = m & 1;
        if (!wait_or_abort(&ctl->p_full[b], (m >> 1) & 1, ctl, status)) return false;
        tc_fence_after();
        const uint32_t p_addr = smem_u32(smem + kOffP + b * kPBytes);
        const uint32_t v_addr = smem_u32(smem + kOffStages + (m % kNS) * kStageBytes + kKVBytes);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {   // 2 x K=32 keys
          // P: K-major, no swizzle (layout above). V: MN-major (d contiguous), 128-byte
          // swizzle, 8-key groups 1024 B apart.
          const uint64_t ad = make_sdesc(p_addr + kk * 2 * kPChunk, kPChunk, kPGroup, kLayoutNone);
          const uint64_t bd = make_sdesc(v_addr + kk * 4096, 8192, 1024, kLayoutSW128);
          mma_f8(tmem, ad, bd, idesc_pv, (m > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&ctl->pv_done[b]);
        mma_commit(&ctl->empty[m % kNS]);
        return true;
      };
      bool ok = wait_or_abort(&ctl->q_full, 0, ctl, status);
      for (int n = 0; n < U && ok; ++n) {
        const int s = n % kNS, b = n & 1;
        if (!wait_or_abort(&ctl->full[s], (n / kNS) & 1, ctl, status)) { ok = false; break; }
        if (n >= 2 && !wait_or_abort(&ctl->s_free[b], ((n >> 1) - 1) & 1, ctl, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + kOffStages + s * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {   // 4 x K=32 channels
          const uint64_t ad = make_sdesc(q_addr + kk * 32, 16, 1024, kLayoutSW128);
          const uint64_t bd = make_sdesc(k_addr + kk * 32, 16, 1024, kLayoutSW128);
          mma_i8(tmem + kTmemS + 64 * b, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ctl->s_full[b]);
        if (n >= 1 && !issue_pv(n - 1)) { ok = false; break; }
      }
      if (ok && U >= 1) ok = issue_pv(U - 1);
      mma_commit(&ctl->mma_done);
      if (ok && prm.linear) {
        // phi(Q) . G_ia into the S columns, then (after rows 0-63 read it) phi(Q) . G_ib.
        constexpr uint32_t idesc_l = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 0, 128, 128);
        ok = wait_or_abort(&ctl->a_full, 0, ctl, status) &&
             wait_or_abort(&ctl->g_full, 0, ctl, status);
        if (ok) {
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem);
          for (int half = 0; half < (has_b ? 2 : 1) && ok; ++half) {
            if (half == 1) {
              ok = wait_or_abort(&ctl->la_free, 0, ctl, status);
              if (!ok) break;
              tc_fence_after();
            }
            const uint32_t g_addr = smem_u32(smem + 32768 + half * 32768);
#pragma unroll
            for (int kc = 0; kc < 2; ++kc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = make_sdesc(a_addr + kc * 16384 + kk * 32, 16, 1024, kLayoutSW128);
                const uint64_t bd = make_sdesc(g_addr + kc * 16384 + kk * 32, 16, 1024, kLayoutSW128);
                mma_bf16(tmem + kTmemS, ad, bd, idesc_l, (kc | kk) ? 1u : 0u);
              }
            mma_commit(half == 0 ? &ctl->la_done : &ctl->lb_done);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Loop mapping (16x64b TMEM fragment): warp w reads lanes 32*(w&3) + 16*(w>>2) + 0..15;
    // lane t holds row lrow = t/4 + 8*(t&1) and key half p = (t>>1)&1, i.e. keys 32p..32p+31
    // of the block (the K8 rows are stored key-interleaved). Lanes t and t^2 share a row.
    const int quad = warp & 3;
    const int sub = warp >> 2;
    const int row = 32 * quad + 16 * sub + (lane >> 2) + 8 * (lane & 1);   // 0..127
    const int kh = (lane >> 1) & 1;              // key half
    const int half = row >> 6;                   // 0: block ia, 1: block ib (warp-uniform)
    const uint32_t my_bit = 1u << half;
    const int qblock = ia + half;
    const int bar_id = 1 + quad;                 // named barrier of warps quad, quad + 4
    const float cs = prm.sq[bh * prm.nbq + qblock] * (kLog2e * kInvSqrtD);
    const uint32_t lane16 = static_cast<uint32_t>(32 * quad + 16 * sub) << 16;
    const int valid = prm.n_last - 32 * kh;      // valid keys of this thread in the last block
    float m_run = -INFINITY, l_part = 0.f;
    bool ok = true;
    for (int n = 0; n < U; ++n) {
      const int b = n & 1;
      const uint32_t e = list[n];
      const int j = static_cast<int>(e & 0xFFFFFFu);
      const bool mine = ((e >> 24) & my_bit) != 0;     // warp-uniform
      if (!wait_or_abort(&ctl->s_full[b], (n >> 1) & 1, ctl, status)) { ok = false; break; }
      tc_fence_after();
      uint32_t pk[8];
      float alpha = 1.f;
      if (mine) {
        uint32_t sr[32];
        tmem_ld16x64(tmem + lane16 + kTmemS + 64 * b, sr);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->s_free[b]);
        const bool full = j != prm.nb - 1 || prm.n_last == 64;   // no padded keys
        int mxi = full ? row_block_max<true>(sr, 32) : row_block_max<false>(sr, valid);
        mxi = max(mxi, __shfl_xor_sync(0xffffffffu, mxi, 2));
        const float c = cs * list_sk[n];
        const float m_new = fmaxf(m_run, s32_to_f32(static_cast<uint32_t>(mxi)) * c);
        alpha = ex2_mufu(m_run - m_new);
        const float neg = kLog2_448 - m_new;      // 2^(S c + neg) = 448 p
        const float rs = full ? row_exp_pack<true>(sr, 32, c, neg, pk)
                              : row_exp_pack<false>(sr, valid, c, neg, pk);
        l_part = alpha * l_part + rs;
        m_run = m_new;
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->s_free[b]);
#pragma unroll
        for (int q = 0; q < 8; ++q) pk[q] = 0u;
      }
      // P(n) into buffer b once P.V(n-2) has read it
      if (n >= 2 && !wait_or_abort(&ctl->pv_done[b], ((n >> 1) - 1) & 1, ctl, status)) { ok = false; break; }
      uint8_t* pb = smem + kOffP + b * kPBytes + (row >> 3) * kPGroup + (row & 7) * 16 + 2 * kh * kPChunk;
      *reinterpret_cast<uint4*>(pb) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(pb + kPChunk) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      fence_proxy_async_smem();
      // rescale this row's O once P.V(n-1) has landed (skipped when no row of the warp moved
      // its max); the two threads of a row each take 64 of the 128 columns
      if (n >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_or_abort(&ctl->pv_done[b ^ 1], ((n - 1) >> 1) & 1, ctl, status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          tmem_ld16x64(tmem + lane16 + 64 * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st16x64(tmem + lane16 + 64 * cc, o);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[b]);
    }
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);      // the row's total of 448 p
    if (kh == 0) ctl->xf[0][row] = l_part;

    // ------------------------------------------------------------ epilogue
    // Epilogue mapping (32x32b fragment): warp w holds row 32*(w&3) + lane and owns O columns
    // 64*(w>>2) .. +63.
    if (ok) ok = wait_or_abort(&ctl->pv_done[(U - 1) & 1], ((U - 1) >> 1) & 1, ctl, status);
    tc_fence_after();
    pair_sync(bar_id);
    const int erow = 32 * quad + lane;
    const int ch = sub;
    const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;
    const float l448 = ctl->xf[0][erow];
    const int tok = 128 * pair + erow;           // token index within the head
    const bool store = ok && tok < prm.N;
    const int64_t b_ = bh / prm.q.H, h_ = bh % prm.q.H;
    float den = 0.f;
    if (prm.linear && ok) {
      // phi(q) for this row; this thread writes channels 64ch .. 64ch+63 of the A operand
      // (bf16, K-major, 128-byte swizzle) and sums its part of the normalizer.
      const uint16_t* qrow = static_cast<const uint16_t*>(prm.q.data) + b_ * prm.q.stride_b +
                             h_ * prm.q.stride_h + static_cast<int64_t>(min(tok, prm.N - 1)) * prm.q.stride_n;
      const uint4* q4 = reinterpret_cast<const uint4*>(qrow);
      float mx = -INFINITY;
#pragma unroll 4
      for (int u = 0; u < 16; ++u) {
        const uint4 r = __ldg(q4 + u);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int z = 0; z < 4; ++z)
          mx = fmaxf(mx, fmaxf(__uint_as_float(w[z] << 16), __uint_as_float(w[z] & 0xFFFF0000u)));
      }
      float sum = 0.f;
#pragma unroll 4
      for (int u = 0; u < 16; ++u) {
        const uint4 r = __ldg(q4 + u);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int z = 0; z < 4; ++z)
          sum += __expf(__uint_as_float(w[z] << 16) - mx) + __expf(__uint_as_float(w[z] & 0xFFFF0000u) - mx);
      }
      const float inv = 1.f / sum;
      const uint4* g128 = reinterpret_cast<const uint4*>(
          prm.gsum + ((bh * prm.nb_m_pad + qblock) * 129 + 128) * 128);
      float dsum = 0.f;
#pragma unroll 2
      for (int uu = 0; uu < 8; ++uu) {
        const int u = 8 * ch + uu;
        const uint4 r = __ldg(q4 + u);
        const uint4 gg = __ldg(g128 + u);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
        const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w};
        uint32_t packed[4];
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const float a0 = tok < prm.N ? __expf(__uint_as_float(w[z] << 16) - mx) * inv : 0.f;
          const float a1 = tok < prm.N ? __expf(__uint_as_float(w[z] & 0xFFFF0000u) - mx) * inv : 0.f;
          __nv_bfloat162 p2 = __floats2bfloat162_rn(a0, a1);
          packed[z] = *reinterpret_cast<uint32_t*>(&p2);
          dsum = fmaf(__low2float(p2), __uint_as_float(gw[z] << 16), dsum);
          dsum = fmaf(__high2float(p2), __uint_as_float(gw[z] & 0xFFFF0000u), dsum);
        }
        const uint32_t off = ch * 16384u + sw128_offset(erow, uu);
        *reinterpret_cast<uint4*>(smem + off) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ctl->a_full);
      den = dsum;
    }
    // normalizer of the linear branch from the two column halves (executed by every softmax
    // thread exactly once, whatever path it took)
    ctl->xd[ch][erow] = den;
    pair_sync(bar_id);
    den += ctl->xd[ch ^ 1][erow];
    if (prm.linear && ok) {
      // wait for this half's phi(Q) . G (rows of a missing second block store nothing)
      if (half == 0 || has_b) {
        ok = wait_or_abort(half == 0 ? &ctl->la_done : &ctl->lb_done, 0, ctl, status);
        tc_fence_after();
      } else {
        ok = false;
      }
    }
    const float inv_l = 1.f / l448;
    const float inv_den = 1.f / den;
    float* sp_row = (prm.sparse_out && store) ? prm.sparse_out + (bh * prm.N + tok) * 128 : nullptr;
    char* out_row = static_cast<char*>(prm.out) +
                    (b_ * prm.out_sb + h_ * prm.out_sh + static_cast<int64_t>(tok) * prm.out_sn) *
                        (prm.out_dtype == SAGESLA_F32 ? 4 : 2);
    if (ok) {
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int col0 = 64 * ch + 32 * cc;
        uint32_t o[32], lin[32];
        tmem_ld32(tmem + lane_base + col0, o);
        if (prm.linear) tmem_ld32(tmem + lane_base + kTmemS + col0, lin);
        tmem_ld_wait();
        float res[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float os = __uint_as_float(o[q]) * ctl->s_v[col0 + q] * inv_l;
          if (sp_row) sp_row[col0 + q] = os;
          res[q] = prm.linear ? os + __uint_as_float(lin[q]) * inv_den : os;
        }
        if (store) {
          if (prm.out_dtype == SAGESLA_F32) {
            float4* d = reinterpret_cast<float4*>(out_row) + col0 / 4;
#pragma unroll
            for (int q = 0; q < 8; ++q) d[q] = make_float4(res[4 * q], res[4 * q + 1], res[4 * q + 2], res[4 * q + 3]);
          } else {
            uint4* d = reinterpret_cast<uint4*>(out_row) + col0 / 8;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int z = 0; z < 4; ++z) {
                __nv_bfloat162 v2 = __floats2bfloat162_rn(res[8 * q + 2 * z], res[8 * q + 2 * z + 1]);
                w[z] = *reinterpret_cast<uint32_t*>(&v2);
              }
              d[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
    if (prm.linear && half == 0) {
      tc_fence_before();
      mbar_arrive(&ctl->la_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_attention(const ForwardPlan& p, TensorArg q, void* out, int32_t out_dtype,
                             int64_t out_sb, int64_t out_sh, int64_t out_sn, float* sparse_out,
                             char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  CUtensorMap tq, tk, tv, tg;
  const uint64_t rows = static_cast<uint64_t>(p.BH * p.n_pad);
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, ws + L.q8, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, ws + L.k8, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, ws + L.v8, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128,
                      static_cast<uint64_t>(p.BH * p.nb_m_pad * 129), 256, ws + L.gsum, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  AttnParams prm;
  prm.sq = reinterpret_cast<const float*>(ws + L.sq);
  prm.sk = reinterpret_cast<const float*>(ws + L.sk);
  prm.s_v = reinterpret_cast<const float*>(ws + L.s_v);
  prm.mask = reinterpret_cast<const uint32_t*>(ws + L.mask);
  prm.gsum = reinterpret_cast<const __nv_bfloat16*>(ws + L.gsum);
  prm.q = q;
  prm.out = out;
  prm.out_sb = out_sb;
  prm.out_sh = out_sh;
  prm.out_sn = out_sn;
  prm.out_dtype = out_dtype;
  prm.sparse_out = sparse_out;
  prm.status = reinterpret_cast<int*>(ws + L.status);
  prm.N = static_cast<int>(p.N);
  prm.nb = static_cast<int>(p.nb);
  prm.nbq = static_cast<int>(2 * p.n_pairs);
  prm.n_pad = static_cast<int>(p.n_pad);
  prm.mask_words = static_cast<int>(p.mask_words);
  prm.nb_m_pad = static_cast<int>(p.nb_m_pad);
  prm.n_last = p.n_last;
  prm.list_cap = static_cast<int>(p.nb < 2 * p.k ? p.nb : 2 * p.k);
  prm.linear = p.linear_empty ? 0 : 1;
  const size_t smem = 1024 + kOffCtl + sizeof(Ctl) + static_cast<size_t>(prm.list_cap) * 8;
  cudaError_t e = cudaFuncSetAttribute(k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.n_pairs), static_cast<unsigned>(p.BH));
  k_attention<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tg, prm);
  return cudaGetLastError();
}

}  // namespace sagesla
