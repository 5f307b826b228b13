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
// B200 mapping. One CTA holds two query blocks ("halves"). Each half runs its own pipeline
// over its own k kept blocks with M=64 tcgen05 MMAs: an M=64 result occupies TMEM lanes
// 0-15 of each 32-lane quadrant, and a lane offset of 16 in the D address puts the second
// half in lanes 16-31, so both halves share the TMEM columns (O fp32 [0,128); S int32 of a
// pair of kept blocks [128,256); the linear branch reuses the S columns at the end).
//   warps 0-3 / 4-7  softmax, correction and epilogue of half 0 / half 1 (16 rows per warp,
//                    two threads per row through the 16x64b TMEM fragment)
//   warp 8           TMA producer: Q rows, K8 tiles of pairs of kept blocks, V8 ring, G_i;
//                    the kept lists are staged in shared memory when the CTA starts, so no
//                    tile load waits for a global read of its block index
//   warp 9           S = Q K^T issuer for both halves: one M=64 N=128 MMA group (4 K-steps)
//                    per pair of kept blocks, whose K8 tiles sit side by side in shared memory
//   warps 10 / 11    P.V issuer of half 0 / half 1
// A tcgen05.mma blocks its issuing thread for about 100 cycles whatever its shape (measured
// on B200), while MMAs from different threads overlap: the N=128 pairs halve the S MMA count
// and the issue work is spread over three threads. The helper warpgroup (8-11) hands
// registers to the softmax warpgroups with setmaxnreg.
// Each half owns 48 KB of shared memory (its Q rows, the K8 pair, a 3-stage V8 ring), reused
// for the linear-branch operands once its main loop is done; its P tile sits after both halves.
//
// Softmax arithmetic per score: the block's row maximum is taken on the int32 scores (integer
// maxima), and each score becomes a float exactly (|S| < 2^21) by one conversion inside the
// exponential loop, where it overlaps the MUFU work (measured ~1% faster than converting all
// scores first and taking three-input float maxima, and ~2.5% faster than forming the floats
// through the 1.5*2^23 bias with an integer add and a packed f32x2 subtract);
// one packed FFMA forms the base-2 exponent with the factor 448 of the P quantization folded in; 2^x
// comes from the MUFU ex2 unit (measured faster here than moving part of the exponentials to
// a polynomial on the FMA pipe: the loop is bound by latency, not by MUFU throughput).
#include <cuda_bf16.h>
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kNV = 3;                       // V ring stages per half
constexpr int kProducerWarp = 8, kSWarp = 9, kPVWarp0 = 10;
constexpr int kThreads = 384;
// setmaxnreg split: 256 x 96 + 128 x 40 = 29696 registers, within the 384 x 80 a CTA is
// launched with (checked on the host before the launch). 96 / 40 measured 1.3% faster than
// 88 / 56 (the helper warps spill 12 bytes; the softmax warps none).
constexpr uint32_t kSoftmaxRegs = 96, kHelperRegs = 40;
constexpr uint32_t kChunk = 8192;            // 64 rows x 128 bytes: one SW128 tile chunk
constexpr uint32_t kHLinA = 0;               // epilogue: phi(Q) bf16, 2 x [64][128 B]
constexpr uint32_t kHLinG = 16384;           // epilogue: G_i bf16, 2 x [128][128 B]
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemS = 128;              // first S buffer column

// Shared-memory layout of one operand mode. kQK8: Q.K^T on INT8 codes (else bf16 Q and K);
// kPV8: P.V on e4m3 P and V codes (else bf16 P and raw bf16 V).
//   per half: Q rows (64 x 128 channels), K tiles of a pair of kept blocks, a kNV-stage V ring;
//   after both halves: one P tile per half; then the control block.
// A 16-bit tile of 128 channels is two 64-channel chunks (each 64 rows x 128 B, SW128); the
// K pair of bf16 keys is chunk 0 of both blocks (16 KB) then chunk 1 of both blocks, so that
// each chunk holds the 128 key rows an N=128 MMA reads.
template <bool kQK8, bool kPV8>
struct Lay {
  static constexpr uint32_t kQBytes = kQK8 ? kChunk : 2 * kChunk;
  static constexpr uint32_t kKBlock = kQK8 ? kChunk : 2 * kChunk;   // K tile of one key block
  static constexpr uint32_t kVBlock = kPV8 ? kChunk : 2 * kChunk;   // V tile of one key block
  static constexpr uint32_t kHQ = 0;
  static constexpr uint32_t kHK = kQBytes;
  static constexpr uint32_t kHV = kHK + 2 * kKBlock;
  static constexpr uint32_t kHalfBytes = kHV + kNV * kVBlock;
  // e4m3 P tile (64 rows), K-major without swizzle: core matrices of 8 rows x 16 keys
  // (128 B); K-chunks 160 B apart and 8-row groups 672 B apart. The padding makes the 16-byte
  // stores of the softmax threads (one store phase holds rows r, r+8, r+1, r+9 and key halves
  // 0, 1) fall on eight distinct bank groups. bf16 P tile: 64 rows x 128 B, SW128.
  static constexpr uint32_t kPChunk = 160, kPGroup = 672;
  static constexpr uint32_t kPBytes = kPV8 ? 8 * kPGroup : kChunk;
  static constexpr uint32_t kOffP = 2 * kHalfBytes;
  static constexpr uint32_t kOffCtl = kOffP + 2 * kPBytes;
  static_assert(kHLinG + 32768 <= kHalfBytes, "linear operands fit in the half region");
  static_assert(kHalfBytes % 1024 == 0 && kOffP % 1024 == 0 && kPBytes % 32 == 0,
                "swizzle atoms stay 1024-byte aligned");
  static_assert(kPV8 || kPBytes % 1024 == 0, "bf16 P tiles are SW128 atoms");
};
constexpr uint32_t kIdescPV8 = make_idesc(kFmtF32, kFmtE4M3, kFmtE4M3, 0, 1, 64, 128);
constexpr uint32_t kIdescPV16 = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 1, 64, 128);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kInvSqrtD = 0.08838834764831845f;
constexpr float kLog2_448 = 8.807354922057604f;

// Every barrier is waited on by parity, which is safe because none can complete a phase
// twice ahead of any of its waiters: each next phase needs an action that only follows the
// waiter's own wait (for p_full: the softmax warps wait for P.V(n-1) before writing P(n)).
struct HalfCtl {
  uint64_t k_full, s_full, s_free;          // one phase per pair of kept blocks
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t p_full, pv_done[2];              // one phase per kept block
  uint64_t q_full, g_full, a_full, l_done, mma_done;
};

// Entries of each half's kept list staged in shared memory (block indices < 2^15 fit 16 bits);
// entries past this come from global memory.
constexpr int kListCap = 768;

struct Ctl {
  HalfCtl hc[2];
  uint32_t tmem_base;
  volatile int abort;
  float s_v[128];
  uint16_t klist[2][kListCap];
};

// Dynamic shared memory of a mode: the layout, the control block and 1 KB of alignment slack.
template <bool kQK8, bool kPV8>
constexpr size_t attn_smem_bytes() { return 1024 + Lay<kQK8, kPV8>::kOffCtl + sizeof(Ctl); }
// The 8-bit mode runs two CTAs per SM: 228 KB of shared memory per SM, 1 KB reserved per CTA.
// The 16-bit modes run one (227 KB at most per CTA).
static_assert(2 * (attn_smem_bytes<true, true>() + 1024) <= 228 * 1024, "two CTAs fit on an SM");
static_assert(attn_smem_bytes<true, false>() <= 227 * 1024, "fits one CTA");
static_assert(attn_smem_bytes<false, false>() <= 227 * 1024, "fits one CTA");

// n-th kept key block of half h's query block: its kept list (shared-memory copy first), or
// block n itself when every block is kept (no list).
__device__ __forceinline__ int kept_at(const Ctl* ctl, int h, const int32_t* klist, int n) {
  if (!klist) return n;
  return n < kListCap ? static_cast<int>(ctl->klist[h][n]) : __ldg(klist + n);
}

// A block index as used for a load that runs ahead of its bounds check: unchanged in the
// normal build, clamped into [0, nb) in the checking build.
__device__ __forceinline__ int clamp_block(int j, int nb) {
  return kChecks ? min(max(j, 0), nb - 1) : j;
}

// n-th kept key block of a query block: its kept list, or block n itself when every block is
// kept (no list).
__device__ __forceinline__ int kept_block(const int32_t* klist, int n) {
  return klist ? __ldg(klist + n) : n;
}

struct AttnParams {
  const float* sq;            // [BH][nbq]
  const float* sk;            // [BH][nbq]
  const float* s_v;           // [BH][128]
  const int32_t* kept;        // [BH][nb][k], or null when every block is kept
  const __nv_bfloat16* gsum;  // [BH][nb_m_pad][129][128]
  TensorArg q;                // raw bf16 Q (for phi(q))
  void* out;
  int64_t out_sb, out_sh, out_sn;
  int32_t out_dtype;
  float* sparse_out;          // optional [BH][N][128]
  int* status;
  int N, nb, nbq, n_pad, k, nb_m_pad, n_last;
  int linear;                 // 0 when every key block is kept
  unsigned long long spin_ns; // limit of every wait (a shorter one only in failure-path tests)
  int skip_tile;              // failure-path test: CTA (0, 0) never loads its first K8 pair
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Ctl* ctl,
                                              int* status, unsigned long long limit_ns) {
  // A completed phase is safe to pass; the CTA's abort flag (a shared-memory load) is read only
  // when the wait would block (measured: 6% of the sparse kernel's time at 14B-720P).
  if (mbar_try_wait(bar, parity)) return true;
  if (ctl->abort) return false;
  if (!mbar_wait(bar, parity, status, limit_ns)) {
    ctl->abort = 1;
    return false;
  }
  return true;
}

// Largest of the first `valid` scores as a float: for int32 scores integer maxima in four
// chains (the conversion to float happens in the exponential loop), for float scores
// three-input float maxima.
template <bool kFull, bool kInt>
__device__ __forceinline__ float row_block_fmax(uint32_t (&a)[32], int valid) {
  if constexpr (kInt) {
    int m[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      int x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int q = 8 * c + u;
        x[u] = (kFull || q < valid) ? static_cast<int>(a[q]) : INT_MIN;
      }
      m[c] = max(max(max(x[0], x[1]), max(x[2], x[3])), max(max(x[4], x[5]), max(x[6], x[7])));
    }
    return __int2float_rn(max(max(m[0], m[1]), max(m[2], m[3])));
  }
  float m[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int q = 8 * c + u;
      x[u] = (kFull || q < valid) ? __uint_as_float(a[q]) : -INFINITY;
    }
    m[c] = fmaxf(fmax3(fmax3(x[0], x[1], x[2]), x[3], x[4]), fmax3(x[5], x[6], x[7]));
  }
  return fmaxf(fmax3(m[0], m[1], m[2]), m[3]);
}
// 448 p = 2^(S c + neg) for the thread's 32 scores: returns their sum and packs them into
// the P operand, as e4m3 codes (kP8: pk[0..7]) or as bf16 values (pk[0..15]).
template <bool kFull, bool kP8, bool kInt>
__device__ __forceinline__ float row_exp_pack(const uint32_t (&sr)[32], int valid, float c,
                                              float neg, uint32_t (&pk)[16]) {
  const unsigned long long c2 = f2_pack(c, c), neg2 = f2_pack(neg, neg);
  unsigned long long acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 32; q += 4) {
    float y[4];
#pragma unroll
    for (int t = 0; t < 4; t += 2) {
      const unsigned long long f2 =
          kInt ? f2_pack(__int2float_rn(static_cast<int>(sr[q + t])), __int2float_rn(static_cast<int>(sr[q + t + 1])))
               : f2_pack(__uint_as_float(sr[q + t]), __uint_as_float(sr[q + t + 1]));
      float x0, x1;
      f2_unpack(f2_fma(f2, c2, neg2), x0, x1);
      y[t] = ex2_mufu(x0);
      y[t + 1] = ex2_mufu(x1);
      if (!kFull) {
        if (q + t >= valid) y[t] = 0.f;
        if (q + t + 1 >= valid) y[t + 1] = 0.f;
      }
    }
    acc0 = f2_add(acc0, f2_pack(y[0], y[1]));
    acc1 = f2_add(acc1, f2_pack(y[2], y[3]));
    if (kP8) {
      pk[q >> 2] = static_cast<uint32_t>(f32x2_to_e4m3x2(y[0], y[1])) |
                   (static_cast<uint32_t>(f32x2_to_e4m3x2(y[2], y[3])) << 16);
    } else {
      __nv_bfloat162 b0 = __floats2bfloat162_rn(y[0], y[1]);
      __nv_bfloat162 b1 = __floats2bfloat162_rn(y[2], y[3]);
      pk[q >> 1] = *reinterpret_cast<uint32_t*>(&b0);
      pk[(q >> 1) + 1] = *reinterpret_cast<uint32_t*>(&b1);
    }
  }
  float a, b;
  f2_unpack(f2_add(acc0, acc1), a, b);
  return a + b;
}

template <bool kQK8, bool kPV8>
__global__ void __launch_bounds__(kThreads, 2)
k_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
            AttnParams prm) {
  using L = Lay<kQK8, kPV8>;
  constexpr uint32_t kHalfBytes = L::kHalfBytes, kHQ = L::kHQ, kHK = L::kHK, kHV = L::kHV;
  constexpr uint32_t kOffP = L::kOffP, kPBytes = L::kPBytes;
  constexpr uint32_t kPChunk = L::kPChunk, kPGroup = L::kPGroup;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + L::kOffCtl);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int ia = 2 * pair;                        // first query block of the CTA
  int* status = prm.status;
  int U[2];
  U[0] = prm.k;
  U[1] = (ia + 1 < prm.nb) ? prm.k : 0;           // the last pair may hold a single block

  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  } else if (warp == 1) {
    for (int c = lane; c < 128; c += 32) ctl->s_v[c] = prm.s_v[bh * 128 + c];
  } else if (threadIdx.x == 64) {
    for (int h = 0; h < 2; ++h) {
      HalfCtl& c = ctl->hc[h];
      mbar_init(&c.k_full, 1);
      mbar_init(&c.s_full, 1);
      mbar_init(&c.s_free, 4);
      for (int s = 0; s < kNV; ++s) { mbar_init(&c.v_full[s], 1); mbar_init(&c.v_empty[s], 1); }
      mbar_init(&c.p_full, 4);
      mbar_init(&c.pv_done[0], 1);
      mbar_init(&c.pv_done[1], 1);
      mbar_init(&c.q_full, 1);
      mbar_init(&c.g_full, 1);
      mbar_init(&c.a_full, 4);
      mbar_init(&c.l_done, 1);
      mbar_init(&c.mma_done, 1);
    }
    ctl->abort = 0;
    fence_mbar_init();
  } else if (threadIdx.x == 96) {
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_g);
  } else if (warp >= 4 && warp < 8 && prm.kept) {
    // both halves' kept lists into shared memory
    for (int h = 0; h < 2; ++h) {
      if (U[h] == 0) continue;
      const int32_t* kl = prm.kept + (bh * prm.nb + ia + h) * static_cast<int64_t>(prm.k);
      const int n = min(U[h], kListCap);
      for (int e = threadIdx.x - 128; e < n; e += 128)
        ctl->klist[h][e] = static_cast<uint16_t>(__ldg(kl + e));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp >= kProducerWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelperRegs));
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int row_base = static_cast<int>(bh * prm.n_pad);
      // A 16-bit tile of 128 channels arrives as two boxes of 64 channels (x = 0, 64).
      for (int h = 0; h < 2; ++h) {
        if (U[h] == 0) continue;
        if (!in_range(128 * pair + 64 * h, prm.n_pad, status)) { ctl->abort = 1; break; }
        mbar_arrive_expect_tx(&ctl->hc[h].q_full, L::kQBytes);
        uint8_t* qst = smem + h * kHalfBytes + kHQ;
        tma_load_2d(qst, &tm_q, &ctl->hc[h].q_full, 0, row_base + 128 * pair + 64 * h);
        if (!kQK8) tma_load_2d(qst + kChunk, &tm_q, &ctl->hc[h].q_full, 64, row_base + 128 * pair + 64 * h);
      }
      bool ok = true;
      const int Umax = max(U[0], U[1]);
      for (int n0 = 0; n0 < Umax && ok; n0 += 2) {
        // K8 of the pair (n0, n0 + 1): the stage is free once S of the previous pair is done
        for (int h = 0; h < 2 && ok; ++h) {
          if (n0 >= U[h]) continue;
          HalfCtl& c = ctl->hc[h];
          if (n0 > 0 && !(ok = wait_or_abort(&c.s_full, ((n0 >> 1) - 1) & 1, ctl, status, prm.spin_ns))) break;
          const int32_t* klist = prm.kept ? prm.kept + (bh * prm.nb + ia + h) * static_cast<int64_t>(prm.k) : nullptr;
          const int two = n0 + 1 < U[h] ? 2 : 1;
          // Failure-path test: the first pair of CTA (0, 0) is never loaded, so the waits for
          // it run out (nothing is left in flight: neither its bytes nor its copies exist).
          if (prm.skip_tile && n0 == 0 && h == 0 && pair == 0 && bh == 0) continue;
          int jk[2] = {kept_at(ctl, h, klist, n0), two > 1 ? kept_at(ctl, h, klist, n0 + 1) : 0};
          if (kChecks && !(in_range(jk[0], prm.nb, status) && in_range(jk[1], prm.nb, status))) {
            ctl->abort = 1;     // checking build: the out-of-range tile is not loaded
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&c.k_full, two * L::kKBlock);
          uint8_t* kst = smem + h * kHalfBytes + kHK;
          for (int b = 0; b < two; ++b) {
            const int y = row_base + 64 * jk[b];
            tma_load_2d(kst + b * kChunk, &tm_k, &c.k_full, 0, y);
            if (!kQK8) tma_load_2d(kst + 2 * kChunk + b * kChunk, &tm_k, &c.k_full, 64, y);
          }
        }
        // V8 of blocks n0 and n0 + 1: stage n % kNV is free once P.V(n - kNV) is done
        for (int n = n0; n < n0 + 2 && ok; ++n)
          for (int h = 0; h < 2 && ok; ++h) {
            if (n >= U[h]) continue;
            HalfCtl& c = ctl->hc[h];
            const int s = n % kNV;
            if (n >= kNV && !(ok = wait_or_abort(&c.v_empty[s], ((n / kNV) - 1) & 1, ctl, status, prm.spin_ns))) break;
            const int32_t* klist = prm.kept ? prm.kept + (bh * prm.nb + ia + h) * static_cast<int64_t>(prm.k) : nullptr;
            const int jv = kept_at(ctl, h, klist, n);
            if (!in_range(jv, prm.nb, status)) { ctl->abort = 1; ok = false; break; }
            mbar_arrive_expect_tx(&c.v_full[s], L::kVBlock);
            uint8_t* vst = smem + h * kHalfBytes + kHV + s * L::kVBlock;
            const int y = row_base + 64 * jv;
            tma_load_2d(vst, &tm_v, &c.v_full[s], 0, y);
            if (!kPV8) tma_load_2d(vst + kChunk, &tm_v, &c.v_full[s], 64, y);
          }
      }
      // G_i once the half's loop MMAs are done (its tile overlaps the K and V stages)
      for (int h = 0; h < 2 && ok && prm.linear; ++h) {
        if (U[h] == 0) continue;
        HalfCtl& c = ctl->hc[h];
        if (!(ok = wait_or_abort(&c.mma_done, 0, ctl, status, prm.spin_ns))) break;
        if (!(ok = in_range(ia + h, prm.nb_m_pad, status))) { ctl->abort = 1; break; }
        const int gy = static_cast<int>((bh * prm.nb_m_pad + ia + h) * 129);
        uint8_t* hb = smem + h * kHalfBytes;
        mbar_arrive_expect_tx(&c.g_full, 32768u);
        tma_load_2d(hb + kHLinG, &tm_g, &c.g_full, 0, gy);
        tma_load_2d(hb + kHLinG + 16384, &tm_g, &c.g_full, 64, gy);
      }
    }
  } else if (warp == kSWarp) {
    // ------------------------------------------------------------ S = Q K^T issuer (both
    // halves, one M=64 N=128 group per pair of kept blocks) and the linear-branch MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc(kFmtS32, kFmtS8, kFmtS8, 0, 0, 64, 128);
      constexpr uint32_t idesc_s16 = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 0, 64, 128);
      constexpr uint32_t idesc_l = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 0, 64, 128);
      bool ok = true;
      for (int h = 0; h < 2 && ok; ++h)
        if (U[h] > 0) ok = wait_or_abort(&ctl->hc[h].q_full, 0, ctl, status, prm.spin_ns);
      // Q rows and K pair descriptors; the K-steps of 32 bytes add 2 to the address field.
      uint64_t dq[2], dk[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t hb = smem_u32(smem + h * kHalfBytes);
        dq[h] = make_sdesc(hb + kHQ, 16, 1024, kLayoutSW128);
        dk[h] = make_sdesc(hb + kHK, 16, 1024, kLayoutSW128);
      }
      const int Umax = max(U[0], U[1]);
      for (int n0 = 0; n0 < Umax && ok; n0 += 2) {
        for (int h = 0; h < 2 && ok; ++h) {
          if (n0 >= U[h]) continue;
          HalfCtl& c = ctl->hc[h];
          const int p = n0 >> 1;
          if (!(ok = wait_or_abort(&c.k_full, p & 1, ctl, status, prm.spin_ns))) break;
          if (p > 0 && !(ok = wait_or_abort(&c.s_free, (p - 1) & 1, ctl, status, prm.spin_ns))) break;
          tc_fence_after();
          const uint32_t d = tmem + (static_cast<uint32_t>(16 * h) << 16) + kTmemS;
          if (kQK8) {
            mma_i8(d, dq[h], dk[h], idesc_s, 0u);
            mma_i8(d, dq[h] + 2, dk[h] + 2, idesc_s, 1u);
            mma_i8(d, dq[h] + 4, dk[h] + 4, idesc_s, 1u);
            mma_i8(d, dq[h] + 6, dk[h] + 6, idesc_s, 1u);
          } else {
            // bf16: eight K-steps of 16 channels (32 bytes), four per 64-channel chunk; the
            // address field counts 16-byte units.
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16(d, dq[h] + (kk >> 2) * (kChunk >> 4) + (kk & 3) * 2,
                       dk[h] + (kk >> 2) * (2 * kChunk >> 4) + (kk & 3) * 2, idesc_s16,
                       kk ? 1u : 0u);
          }
          mma_commit(&c.s_full);
        }
      }
      for (int h = 0; h < 2 && ok && prm.linear; ++h) {
        // phi(Q_i) . G_i into this half's S columns, once the loop's P.V are done
        if (U[h] == 0) continue;
        HalfCtl& c = ctl->hc[h];
        if (!(ok = wait_or_abort(&c.mma_done, 0, ctl, status, prm.spin_ns) && wait_or_abort(&c.a_full, 0, ctl, status, prm.spin_ns) &&
                   wait_or_abort(&c.g_full, 0, ctl, status, prm.spin_ns))) break;
        tc_fence_after();
        const uint32_t dlane = static_cast<uint32_t>(16 * h) << 16;
        const uint32_t hb = smem_u32(smem + h * kHalfBytes);
#pragma unroll
        for (int kc = 0; kc < 2; ++kc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc(hb + kHLinA + kc * 8192 + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = make_sdesc(hb + kHLinG + kc * 16384 + kk * 32, 16, 1024, kLayoutSW128);
            mma_bf16(tmem + dlane + kTmemS, ad, bd, idesc_l, (kc | kk) ? 1u : 0u);
          }
        mma_commit(&c.l_done);
      }
    }
  } else if (warp >= kPVWarp0) {
    // ------------------------------------------------------------ P.V issuer of one half
    if (lane == 0) {
      const int h = warp - kPVWarp0;
      HalfCtl& c = ctl->hc[h];
      const uint32_t p_addr = smem_u32(smem) + kOffP + h * kPBytes;
      const uint64_t dp0 = make_sdesc(p_addr, kPChunk, kPGroup, kLayoutNone);
      const uint64_t dp1 = make_sdesc(p_addr + 2 * kPChunk, kPChunk, kPGroup, kLayoutNone);
      const uint64_t dp16 = make_sdesc(p_addr, 16, 1024, kLayoutSW128);   // bf16 P, SW128
      const uint32_t vb = smem_u32(smem + h * kHalfBytes) + kHV;
      const uint32_t d = tmem + (static_cast<uint32_t>(16 * h) << 16);
      for (int n = 0; n < U[h]; ++n) {
        const int s = n % kNV;
        if (!wait_or_abort(&c.p_full, n & 1, ctl, status, prm.spin_ns)) break;
        if (!wait_or_abort(&c.v_full[s], (n / kNV) & 1, ctl, status, prm.spin_ns)) break;
        tc_fence_after();
        // P: K-major (e4m3: no swizzle, layout above; bf16: SW128). V: MN-major (d
        // contiguous), 128-byte swizzle, 8-key groups 1024 B apart, bf16 channel chunks
        // 8 KB apart.
        const uint32_t v_addr = vb + s * L::kVBlock;
        if (kPV8) {
          mma_f8(d, dp0, make_sdesc(v_addr, 8192, 1024, kLayoutSW128), kIdescPV8, n > 0 ? 1u : 0u);
          mma_f8(d, dp1, make_sdesc(v_addr + 4096, 8192, 1024, kLayoutSW128), kIdescPV8, 1u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // K-steps of 16 keys: 32 B of P, 2 KB of V
            mma_bf16(d, dp16 + kk * 2, make_sdesc(v_addr + kk * 2048, 8192, 1024, kLayoutSW128),
                     kIdescPV16, (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&c.pv_done[n & 1]);
        mma_commit(&c.v_empty[s]);
        if (n == U[h] - 1) mma_commit(&c.mma_done);
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------------------------------------------------------ softmax / epilogue
    // Warp w serves half h = w/4 and reads TMEM lanes 32*(w&3) + 16h + 0..15 (16x64b
    // fragment): lane t holds row r = 16*(w&3) + t/4 + 8*(t&1) of the half's query block and
    // key half kh = (t>>1)&1, i.e. keys 32kh..32kh+31 of the block (the K8 rows are stored
    // key-interleaved). Lanes t and t^2 share a row.
    const int h = warp >> 2;
    const int quad = warp & 3;
    HalfCtl& c = ctl->hc[h];
    uint8_t* hbase = smem + h * kHalfBytes;
    const int r = 16 * quad + (lane >> 2) + 8 * (lane & 1);    // row within the block
    const int kh = (lane >> 1) & 1;
    const int qblock = ia + h;
    const int Uh = U[h];
    const uint32_t lane16 = static_cast<uint32_t>(32 * quad + 16 * h) << 16;
    const int valid = prm.n_last - 32 * kh;      // valid keys of this thread in the last block
    bool ok = Uh > 0;
    float m_run = -INFINITY, l_part = 0.f;
    if (ok) {
      // base-2 exponent per unit of S: sq sk log2(e) / sqrt(128) for INT8 scores, log2(e) /
      // sqrt(128) for bf16 scores
      const float cs = kQK8 ? prm.sq[bh * prm.nbq + qblock] * (kLog2e * kInvSqrtD)
                            : kLog2e * kInvSqrtD;
      const int32_t* klist = prm.kept ? prm.kept + (bh * prm.nb + qblock) * static_cast<int64_t>(prm.k) : nullptr;
      const float* skh = prm.sk + bh * prm.nbq;
      // kept indices are read two blocks ahead and scales one block ahead, so that no load
      // of the loop waits for another one
      int j_cur = kept_block(klist, 0);
      int j_ahead = Uh > 1 ? kept_block(klist, 1) : 0;
      // (the scale loads run ahead of the checks: the checking build clamps their index)
      float sk_next = kQK8 ? __ldg(skh + clamp_block(j_cur, prm.nb)) : 1.f;
      for (int n = 0; n < Uh; ++n) {
        const int b = n & 1;
        const int j = j_cur;
        const float skj = sk_next;
        // checking build: an out-of-range kept entry stops the CTA before it is used
        if (kChecks && !__all_sync(0xffffffffu, in_range(j, prm.nb, status))) {
          ctl->abort = 1;
          ok = false;
          break;
        }
        if (n + 1 < Uh) {
          if (kQK8) sk_next = __ldg(skh + clamp_block(j_ahead, prm.nb));
          j_cur = j_ahead;
          if (n + 2 < Uh) j_ahead = kept_block(klist, n + 2);
        }
        if (b == 0 && !wait_or_abort(&c.s_full, (n >> 1) & 1, ctl, status, prm.spin_ns)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld16x64(tmem + lane16 + kTmemS + 64 * b, sr);
        tmem_ld_wait();
        if (b == 1) {                            // both blocks of the pair are read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.s_free);
        }
        const bool full = j != prm.nb - 1 || prm.n_last == 64;   // no padded keys
        float mx = full ? row_block_fmax<true, kQK8>(sr, 32) : row_block_fmax<false, kQK8>(sr, valid);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float cst = kQK8 ? cs * skj : cs;
        const float m_new = fmaxf(m_run, mx * cst);
        const float alpha = ex2_mufu(m_run - m_new);
        const float neg = kLog2_448 - m_new;    // 2^(S c + neg) = 448 p
        uint32_t pk[16];
        const float rs = full ? row_exp_pack<true, kPV8, kQK8>(sr, 32, cst, neg, pk)
                              : row_exp_pack<false, kPV8, kQK8>(sr, valid, cst, neg, pk);
        l_part = alpha * l_part + rs;
        m_run = m_new;
        // P.V(n-1) must be done: it frees P buffer b (read by P.V(n-2) before it), makes O
        // stable for the rescale, and orders the P.V MMAs issued from different warps.
        if (n >= 1 && !wait_or_abort(&c.pv_done[b ^ 1], ((n - 1) >> 1) & 1, ctl, status, prm.spin_ns)) { ok = false; break; }
        tc_fence_after();
        if (kPV8) {
          uint8_t* pb = smem + kOffP + h * kPBytes + (r >> 3) * kPGroup + (r & 7) * 16 + 2 * kh * kPChunk;
          *reinterpret_cast<uint4*>(pb) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(pb + kPChunk) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          // bf16 P row r: this thread's 32 keys are the 16-byte chunks 4kh .. 4kh+3 (SW128)
          uint8_t* pt = smem + kOffP + h * kPBytes;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<uint4*>(pt + sw128_offset(r, 4 * kh + e)) =
                make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
        fence_proxy_async_smem();
        // rescale this row's O (skipped when no row of the warp moved its max); the two
        // threads of a row each take 64 of the 128 columns
        if (n >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
          const unsigned long long a2 = f2_pack(alpha, alpha);
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            tmem_ld16x64(tmem + lane16 + 64 * cc, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; q += 2) {
              float x0, x1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[q]), __uint_as_float(o[q + 1])), a2), x0, x1);
              o[q] = __float_as_uint(x0);
              o[q + 1] = __float_as_uint(x1);
            }
            tmem_st16x64(tmem + lane16 + 64 * cc, o);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.p_full);
      }
      if (ok) ok = wait_or_abort(&c.pv_done[(Uh - 1) & 1], ((Uh - 1) >> 1) & 1, ctl, status, prm.spin_ns);
      tc_fence_after();
    }

    // ------------------------------------------------------------ epilogue
    const float l448 = l_part + __shfl_xor_sync(0xffffffffu, l_part, 2);   // row total of 448 p
    const int tok = 64 * qblock + r;             // token index within the head
    const int64_t b_ = bh / prm.q.H, h_ = bh % prm.q.H;
    float den = 0.f;
    // the branch below exchanges values with lane ^ 2: take it warp-uniformly even when a
    // timed-out wait (read per lane from ctl->abort) left the lanes disagreeing
    ok = __all_sync(0xffffffffu, ok) != 0;
    if (prm.linear && ok) {
      // phi(q) of this row: the thread takes channels 64kh .. 64kh+63 (chunk kh of the A
      // operand: bf16, K-major, 128-byte swizzle), the other half is lane ^ 2; the pair reduces
      // the max and the normalizer, and each thread sums its part of the denominator.
      const uint16_t* qrow = static_cast<const uint16_t*>(prm.q.data) + b_ * prm.q.stride_b +
                             h_ * prm.q.stride_h + static_cast<int64_t>(min(tok, prm.N - 1)) * prm.q.stride_n;
      const uint4* q4 = reinterpret_cast<const uint4*>(qrow) + 8 * kh;
      float mx = -INFINITY;
#pragma unroll 4
      for (int u = 0; u < 8; ++u) {
        const uint4 rr = __ldg(q4 + u);
        const uint32_t w[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
        for (int z = 0; z < 4; ++z)
          mx = fmaxf(mx, fmaxf(__uint_as_float(w[z] << 16), __uint_as_float(w[z] & 0xFFFF0000u)));
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float sum = 0.f;
#pragma unroll 4
      for (int u = 0; u < 8; ++u) {
        const uint4 rr = __ldg(q4 + u);
        const uint32_t w[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
        for (int z = 0; z < 4; ++z)
          sum += __expf(__uint_as_float(w[z] << 16) - mx) + __expf(__uint_as_float(w[z] & 0xFFFF0000u) - mx);
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      const float inv = tok < prm.N ? 1.f / sum : 0.f;
      const uint4* g128 = reinterpret_cast<const uint4*>(
          prm.gsum + ((bh * prm.nb_m_pad + qblock) * 129 + 128) * 128) + 8 * kh;
      float dsum = 0.f;
#pragma unroll 2
      for (int uu = 0; uu < 8; ++uu) {
        const uint4 rr = __ldg(q4 + uu);
        const uint4 gg = __ldg(g128 + uu);
        const uint32_t w[4] = {rr.x, rr.y, rr.z, rr.w};
        const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w};
        uint32_t packed[4];
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const float a0 = __expf(__uint_as_float(w[z] << 16) - mx) * inv;
          const float a1 = __expf(__uint_as_float(w[z] & 0xFFFF0000u) - mx) * inv;
          __nv_bfloat162 p2 = __floats2bfloat162_rn(a0, a1);
          packed[z] = *reinterpret_cast<uint32_t*>(&p2);
          dsum = fmaf(__low2float(p2), __uint_as_float(gw[z] << 16), dsum);
          dsum = fmaf(__high2float(p2), __uint_as_float(gw[z] & 0xFFFF0000u), dsum);
        }
        const uint32_t off = kHLinA + kh * 8192u + sw128_offset(r, uu);
        *reinterpret_cast<uint4*>(hbase + off) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      den = dsum + __shfl_xor_sync(0xffffffffu, dsum, 2);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.a_full);
      ok = wait_or_abort(&c.l_done, 0, ctl, status, prm.spin_ns);
      tc_fence_after();
    }
    const float inv_l = 1.f / l448;
    const float inv_den = 1.f / den;
    const bool store = ok && tok < prm.N;
    float* sp_row = (prm.sparse_out && store) ? prm.sparse_out + (bh * prm.N + tok) * 128 : nullptr;
    char* out_row = static_cast<char*>(prm.out) +
                    (b_ * prm.out_sb + h_ * prm.out_sh + static_cast<int64_t>(tok) * prm.out_sn) *
                        (prm.out_dtype == SAGESLA_F32 ? 4 : 2);
    if (ok) {
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {
        // this thread holds columns 64cb + 2e + kh (e = 0..31) of its row
        uint32_t o[32], lin[32];
        tmem_ld16x64(tmem + lane16 + 64 * cb, o);
        if (prm.linear) tmem_ld16x64(tmem + lane16 + kTmemS + 64 * cb, lin);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float os = kPV8 ? __uint_as_float(o[e]) * ctl->s_v[64 * cb + 2 * e + kh] * inv_l
                                : __uint_as_float(o[e]) * inv_l;
          o[e] = __float_as_uint(os);
          lin[e] = __float_as_uint(prm.linear ? os + __uint_as_float(lin[e]) * inv_den : os);
        }
        // Pair exchange with lane ^ 2 so that each thread stores contiguous columns: kh = 0
        // stores 64cb + 0..31 and kh = 1 stores 64cb + 32..63, four at a time.
        const int col0 = 64 * cb + 32 * kh;
        auto exchange_store = [&](const uint32_t (&v)[32], float* dst_f32, uint16_t* dst_bf16) {
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float w4[4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float mine0 = __uint_as_float(v[e + u]), mine1 = __uint_as_float(v[16 + e + u]);
              const float recv = __shfl_xor_sync(0xffffffffu, kh ? mine0 : mine1, 2);
              w4[2 * u] = kh ? recv : mine0;
              w4[2 * u + 1] = kh ? mine1 : recv;
            }
            if (dst_f32) {
              *reinterpret_cast<float4*>(dst_f32 + 2 * e) = make_float4(w4[0], w4[1], w4[2], w4[3]);
            } else if (dst_bf16) {
              __nv_bfloat162 a2 = __floats2bfloat162_rn(w4[0], w4[1]);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(w4[2], w4[3]);
              *reinterpret_cast<uint2*>(dst_bf16 + 2 * e) =
                  make_uint2(*reinterpret_cast<uint32_t*>(&a2), *reinterpret_cast<uint32_t*>(&b2));
            }
          }
        };
        if (prm.sparse_out) exchange_store(o, sp_row ? sp_row + col0 : nullptr, nullptr);
        if (prm.out_dtype == SAGESLA_F32)
          exchange_store(lin, store ? reinterpret_cast<float*>(out_row) + col0 : nullptr, nullptr);
        else
          exchange_store(lin, nullptr, store ? reinterpret_cast<uint16_t*>(out_row) + col0 : nullptr);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

namespace {

// Tensor map of a per-head operand buffer [BH * n_pad rows][128 channels]: 8-bit codes in one
// 128-byte box per row, or bf16 values in boxes of 64 channels (128 B), 64 rows, SW128.
bool operand_map(CUtensorMap* m, bool eight_bit, const void* base, uint64_t rows) {
  return eight_bit ? encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, base, 128,
                                    64, CU_TENSOR_MAP_SWIZZLE_128B)
                   : encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, rows, 256, base, 64,
                                    64, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <bool kQK8, bool kPV8>
cudaError_t launch_mode(const ForwardPlan& p, const AttnParams& prm, const char* ws,
                        cudaStream_t stream) {
  const auto& L = p.lay;
  CUtensorMap tq, tk, tv, tg;
  const uint64_t rows = static_cast<uint64_t>(p.BH * p.n_pad);
  if (!operand_map(&tq, kQK8, ws + (kQK8 ? L.q8 : L.qb), rows) ||
      !operand_map(&tk, kQK8, ws + (kQK8 ? L.k8 : L.kb), rows) ||
      !operand_map(&tv, kPV8, ws + (kPV8 ? L.v8 : L.vb), rows) ||
      !encode_tmap_2d(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128,
                      static_cast<uint64_t>(p.BH * p.nb_m_pad * 129), 256, ws + L.gsum, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // The register split (setmaxnreg) must fit the registers the CTA is launched with, or the
  // softmax warps would wait for registers forever. The count is a property of the loaded
  // module; it is queried per call (cheap, and right for every device and thread).
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, k_attention<kQK8, kPV8>) != cudaSuccess)
    return cudaErrorInvalidDeviceFunction;
  if (static_cast<uint32_t>(fa.numRegs) * kThreads < 256 * kSoftmaxRegs + 128 * kHelperRegs)
    return cudaErrorInvalidConfiguration;
  const size_t smem = attn_smem_bytes<kQK8, kPV8>();
  cudaError_t e = cudaFuncSetAttribute(k_attention<kQK8, kPV8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.n_pairs), static_cast<unsigned>(p.BH));
  k_attention<kQK8, kPV8><<<grid, kThreads, smem, stream>>>(tq, tk, tv, tg, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const ForwardPlan& p, TensorArg q, void* out, int32_t out_dtype,
                             int64_t out_sb, int64_t out_sh, int64_t out_sn, float* sparse_out,
                             char* ws, const AttnTestHooks& hooks, cudaStream_t stream) {
  const auto& L = p.lay;
  AttnParams prm;
  prm.sq = reinterpret_cast<const float*>(ws + L.sq);
  prm.sk = reinterpret_cast<const float*>(ws + L.sk);
  prm.s_v = reinterpret_cast<const float*>(ws + L.s_v);
  prm.kept = p.linear_empty ? nullptr : reinterpret_cast<const int32_t*>(ws + L.kept);
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
  prm.k = static_cast<int>(p.k);
  prm.nb_m_pad = static_cast<int>(p.nb_m_pad);
  prm.n_last = p.n_last;
  prm.linear = p.linear_empty ? 0 : 1;
  prm.spin_ns = hooks.spin_limit_us ? 1000ull * hooks.spin_limit_us : kSpinLimitNs;
  prm.skip_tile = hooks.skip_tile;
  if (p.quant && p.pv_fp8) return launch_mode<true, true>(p, prm, ws, stream);
  if (p.quant) return launch_mode<true, false>(p, prm, ws, stream);
  if (!p.pv_fp8) return launch_mode<false, false>(p, prm, ws, stream);
  return cudaErrorInvalidValue;     // bf16 Q.K^T with e4m3 P.V is not a mode
}

}  // namespace sagesla
