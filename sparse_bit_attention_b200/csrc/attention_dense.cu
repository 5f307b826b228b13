// Dense mode of the SageSLA forward (every key block kept): the sparse branch's online softmax
// over all key blocks in ascending order, INT8 Q.K^T and FP8 P.V on tcgen05 at M=128.
//
// Method: news.qq.com TurboDiffusion article, section 第一把钥匙 — SageAttention's 8-bit
// attention alone, the Top-K ratio 1 end of the sparse-linear attention (the complement, and
// with it the linear branch, is empty). For a query row t and key blocks j = 0, 1, ...:
//     S = (Q8 K8^T) sq sk_j / sqrt(128);  m' = max(m, rowmax S);  p = exp(S - m');
//     l = e^(m-m') l + sum p;   o = e^(m-m') o + e4m3(448 p) . V8;   m = m'
//     out = o s_v / (448 l)
//
// B200 mapping. With every block kept, the two query blocks of a CTA read the same K8 / V8
// tiles, so one CTA takes 128 query rows and every MMA is M=128 (the full tensor-core rate;
// M=64 runs at half of it). One softmax thread per row: the 32x32b TMEM fragment gives thread
// t of warp w row 32w + t with all 64 scores of a key block, so the row maximum and the row
// sum need no shuffles and each thread has 64 independent exponentials per block.
//   warps 0-3  softmax, O rescale and epilogue (one row per thread)
//   warp 4     TMA producer: the 128 Q8 rows once, K8 and V8 tiles through kStages-deep rings
//   warp 5     S = Q8 K8^T issuer: M=128 N=64 (4 K-steps of 32) per key block into one of two
//              TMEM buffers, one block ahead of the softmax
//   warp 6     P.V issuer: M=128 N=128 (2 K-steps of 32) per key block
// TMEM: O fp32 [0, 128), S int32 [128, 192) and [192, 256); two CTAs per SM.
// Shared memory: Q8 16 KB, the K8 and V8 rings (8 KB per stage), two e4m3 P tiles of 8 KB
// (K-major core matrices of 8 rows x 16 keys, 8-row groups 512 B apart: the quarter-warp of
// a 16-byte store holds 8 consecutive rows, which fall on 8 distinct bank groups).
// The row maximum is taken on the int32 scores (integer maxima) and each score is converted to
// float inside the exponential loop, where the conversions overlap the MUFU work (measured
// 4.6% faster at 14B-720P than converting first and taking float maxima).
// K8 rows are stored key-interleaved in each 64-key block (row 2(u mod 32) + u div 32 holds
// key u), so score column c is key (c >> 1) + 32 (c & 1); the P row is written in natural key
// order (a compile-time permutation of the registers), matching the V8 rows.
#include <cuda_bf16.h>
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kDThreads = 224;                  // 7 warps
constexpr int kDProducer = 4, kDSIssuer = 5, kDPVIssuer = 6;
constexpr int kStages = 4;                      // K8 and V8 ring depth
constexpr uint32_t kTile = 8192;                // one 64-row, 128-byte tile
constexpr uint32_t kOffQ = 0;                   // 128 Q8 rows, SW128
constexpr uint32_t kOffK = 2 * kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kOffP = kOffV + kStages * kTile;   // two P tiles
constexpr uint32_t kPLbo = 128, kPSbo = 512;          // P: K-chunk and 8-row group strides
constexpr uint32_t kOffCtlD = kOffP + 2 * kTile;
constexpr uint32_t kDTmemCols = 256;
constexpr uint32_t kDTmemS = 128;
constexpr float kLog2eD = 1.4426950408889634f;
constexpr float kInvSqrtDD = 0.08838834764831845f;
constexpr float kLog2_448D = 8.807354922057604f;

// Barriers are waited on by parity; none can complete a phase twice ahead of any waiter (each
// next phase needs an action that follows the waiter's own wait).
struct DenseCtl {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_free[2];     // S buffer b: one phase per key block n with n & 1 == b
  uint64_t p_full[2], pv_done[2];    // P tile b: likewise
  uint32_t tmem_base;
  volatile int abort;
  float s_v[128];
};
static_assert(2 * (1024 + kOffCtlD + sizeof(DenseCtl) + 1024) <= 228 * 1024,
              "two CTAs fit on an SM");

struct DenseParams {
  const float* sq;            // [BH][nbq]
  const float* sk;            // [BH][nbq]
  const float* s_v;           // [BH][128]
  void* out;
  int64_t out_sb, out_sh, out_sn;
  int32_t out_dtype;
  int32_t out_H;
  float* sparse_out;          // optional [BH][N][128] (equal to out here: no linear branch)
  int* status;
  int N, nb, nbq, n_pad, n_last;
  unsigned long long spin_ns;
  int skip_tile;              // failure-path test: CTA (0, 0) never loads its first K8 tile
};

__device__ __forceinline__ bool dwait(uint64_t* bar, uint32_t parity, DenseCtl* ctl, int* status,
                                      unsigned long long limit_ns) {
  // A completed phase is safe to pass; the CTA's abort flag (a shared-memory load) is read only
  // when the wait would block (measured: 3.6% of the dense kernel's time at 14B-720P).
  if (mbar_try_wait(bar, parity)) return true;
  if (ctl->abort) return false;
  if (!mbar_wait(bar, parity, status, limit_ns)) {
    ctl->abort = 1;
    return false;
  }
  return true;
}

__device__ __forceinline__ void tmem_ld32x64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
        "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
        "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
        "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
        "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

// Score column holding natural key u of the block (the K8 rows are key-interleaved).
__host__ __device__ constexpr int key_column(int u) { return 2 * (u & 31) + (u >> 5); }

// Largest int32 score over the keys below `valid` (integer maxima in eight chains), as a float.
template <bool kFull>
__device__ __forceinline__ float dense_row_max(uint32_t (&a)[64], int valid) {
  int m[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    int x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = 8 * g + u;
      const int key = (c >> 1) + 32 * (c & 1);
      x[u] = (kFull || key < valid) ? static_cast<int>(a[c]) : INT_MIN;
    }
    m[g] = max(max(max(x[0], x[1]), max(x[2], x[3])), max(max(x[4], x[5]), max(x[6], x[7])));
  }
  return __int2float_rn(max(max(max(m[0], m[1]), max(m[2], m[3])), max(max(m[4], m[5]), max(m[6], m[7]))));
}

// 448 p = 2^(S c + neg) for the row's 64 keys in natural order: returns their sum and packs
// the e4m3 codes, four keys per word (pk[u / 4] holds keys u .. u + 3).
template <bool kFull>
__device__ __forceinline__ float dense_row_exp(const uint32_t (&s)[64], int valid, float c,
                                               float neg, uint32_t (&pk)[16], uint8_t* prow) {
  const unsigned long long c2 = f2_pack(c, c), neg2 = f2_pack(neg, neg);
  unsigned long long acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int u = 0; u < 64; u += 4) {
    float y[4];
#pragma unroll
    for (int t = 0; t < 4; t += 2) {
      const unsigned long long f2 = f2_pack(__int2float_rn(static_cast<int>(s[key_column(u + t)])),
                                         __int2float_rn(static_cast<int>(s[key_column(u + t + 1)])));
      float x0, x1;
      f2_unpack(f2_fma(f2, c2, neg2), x0, x1);
      y[t] = ex2_mufu(x0);
      y[t + 1] = ex2_mufu(x1);
      if (!kFull) {
        if (u + t >= valid) y[t] = 0.f;
        if (u + t + 1 >= valid) y[t + 1] = 0.f;
      }
    }
    acc0 = f2_add(acc0, f2_pack(y[0], y[1]));
    acc1 = f2_add(acc1, f2_pack(y[2], y[3]));
    pk[u >> 2] = static_cast<uint32_t>(f32x2_to_e4m3x2(y[0], y[1])) |
                 (static_cast<uint32_t>(f32x2_to_e4m3x2(y[2], y[3])) << 16);
    if ((u & 15) == 12) {   // keys u - 12 .. u + 3: one 16-key K-chunk of the P row
      const int cc = u >> 4;
      *reinterpret_cast<uint4*>(prow + cc * kPLbo) =
          make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
    }
  }
  float a, b;
  f2_unpack(f2_add(acc0, acc1), a, b);
  return a + b;
}

__global__ void __launch_bounds__(kDThreads, 2)
k_attention_dense(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, DenseParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DenseCtl* ctl = reinterpret_cast<DenseCtl*>(smem + kOffCtlD);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int nb = prm.nb;
  int* status = prm.status;

  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, kDTmemCols);
    tmem_relinquish();
  } else if (warp == 1) {
    for (int c = lane; c < 128; c += 32) ctl->s_v[c] = prm.s_v[bh * 128 + c];
  } else if (threadIdx.x == 64) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->s_full[b], 1);
      mbar_init(&ctl->s_free[b], 4);
      mbar_init(&ctl->p_full[b], 4);
      mbar_init(&ctl->pv_done[b], 1);
    }
    ctl->abort = 0;
    fence_mbar_init();
  } else if (threadIdx.x == 96) {
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int row_base = static_cast<int>(bh * prm.n_pad);

  if (warp == kDProducer) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !in_range(128 * pair + 64, prm.n_pad, status)) ctl->abort = 1;
    else if (lane == 0) {
      mbar_arrive_expect_tx(&ctl->q_full, 2 * kTile);
      tma_load_2d(smem + kOffQ, &tm_q, &ctl->q_full, 0, row_base + 128 * pair);
      tma_load_2d(smem + kOffQ + kTile, &tm_q, &ctl->q_full, 0, row_base + 128 * pair + 64);
      for (int n = 0; n < nb; ++n) {
        const int s = n % kStages;
        const uint32_t par = ((n / kStages) - 1) & 1;
        if (n >= kStages && !dwait(&ctl->k_empty[s], par, ctl, status, prm.spin_ns)) break;
        if (!in_range(64 * n, prm.n_pad, status)) { ctl->abort = 1; break; }
        // failure-path test: the first K tile of CTA (0, 0) is never loaded
        if (!(prm.skip_tile && n == 0 && pair == 0 && bh == 0)) {
          mbar_arrive_expect_tx(&ctl->k_full[s], kTile);
          tma_load_2d(smem + kOffK + s * kTile, &tm_k, &ctl->k_full[s], 0, row_base + 64 * n);
        }
        if (n >= kStages && !dwait(&ctl->v_empty[s], par, ctl, status, prm.spin_ns)) break;
        mbar_arrive_expect_tx(&ctl->v_full[s], kTile);
        tma_load_2d(smem + kOffV + s * kTile, &tm_v, &ctl->v_full[s], 0, row_base + 64 * n);
      }
    }
  } else if (warp == kDSIssuer) {
    // ------------------------------------------------------------ S = Q8 K8^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(kFmtS32, kFmtS8, kFmtS8, 0, 0, 128, 64);
      bool ok = dwait(&ctl->q_full, 0, ctl, status, prm.spin_ns);
      const uint64_t dq = make_sdesc(smem_u32(smem + kOffQ), 16, 1024, kLayoutSW128);
      for (int n = 0; n < nb && ok; ++n) {
        const int s = n % kStages, b = n & 1;
        if (!(ok = dwait(&ctl->k_full[s], (n / kStages) & 1, ctl, status, prm.spin_ns))) break;
        if (n >= 2 && !(ok = dwait(&ctl->s_free[b], ((n - 2) >> 1) & 1, ctl, status, prm.spin_ns))) break;
        tc_fence_after();
        const uint64_t dk = make_sdesc(smem_u32(smem + kOffK + s * kTile), 16, 1024, kLayoutSW128);
        const uint32_t d = tmem + kDTmemS + 64 * b;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_i8(d, dq + 2 * kk, dk + 2 * kk, idesc, kk ? 1u : 0u);
        mma_commit(&ctl->s_full[b]);
        mma_commit(&ctl->k_empty[s]);
      }
    }
  } else if (warp == kDPVIssuer) {
    // ------------------------------------------------------------ P.V issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(kFmtF32, kFmtE4M3, kFmtE4M3, 0, 1, 128, 128);
      for (int n = 0; n < nb; ++n) {
        const int s = n % kStages, b = n & 1;
        if (!dwait(&ctl->p_full[b], (n >> 1) & 1, ctl, status, prm.spin_ns)) break;
        if (!dwait(&ctl->v_full[s], (n / kStages) & 1, ctl, status, prm.spin_ns)) break;
        tc_fence_after();
        const uint32_t p_addr = smem_u32(smem + kOffP + b * kTile);
        const uint32_t v_addr = smem_u32(smem + kOffV + s * kTile);
        // P: K-major core matrices (32 keys = 2 K-chunks per step). V: MN-major, SW128.
        mma_f8(tmem, make_sdesc(p_addr, kPLbo, kPSbo, kLayoutNone),
               make_sdesc(v_addr, 8192, 1024, kLayoutSW128), idesc, n > 0 ? 1u : 0u);
        mma_f8(tmem, make_sdesc(p_addr + 2 * kPLbo, kPLbo, kPSbo, kLayoutNone),
               make_sdesc(v_addr + 4096, 8192, 1024, kLayoutSW128), idesc, 1u);
        mma_commit(&ctl->pv_done[b]);
        mma_commit(&ctl->v_empty[s]);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax / epilogue
    const int r = 32 * warp + lane;               // this thread's row of 128 (TMEM lane r)
    const int qblock = 2 * pair + (r >> 6);
    const int tok = 64 * qblock + (r & 63);       // token index within the head
    const uint32_t lane_addr = static_cast<uint32_t>(32 * warp) << 16;
    // base-2 exponent per unit of S with the row's block scale: sq log2(e) / sqrt(128)
    const float cs = prm.sq[bh * prm.nbq + qblock] * (kLog2eD * kInvSqrtDD);
    const float* skh = prm.sk + bh * prm.nbq;
    float m_run = -INFINITY, l448 = 0.f;
    bool ok = true;
    float sk_next = __ldg(skh);
    // Every wait result is made warp-uniform, since the warp's TMEM accesses are collective.
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, dwait(bar, parity, ctl, status, prm.spin_ns)) != 0;
    };
    for (int n = 0; n < nb; ++n) {
      const int b = n & 1;
      const float skj = sk_next;
      if (n + 1 < nb) sk_next = __ldg(skh + n + 1);
      if (!wwait(&ctl->s_full[b], (n >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32x64(tmem + lane_addr + kDTmemS + 64 * b, sr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_free[b]);
      const bool full = n != nb - 1 || prm.n_last == 64;     // no padded keys
      const float mx = full ? dense_row_max<true>(sr, 64) : dense_row_max<false>(sr, prm.n_last);
      const float cst = cs * skj;
      const float m_new = fmaxf(m_run, mx * cst);
      const float alpha = ex2_mufu(m_run - m_new);               // 0 on the first block
      const float neg = kLog2_448D - m_new;                  // 2^(S c + neg) = 448 p
      // P tile b is free once P.V(n - 2) has read it (long done by now, as a rule); the P row
      // is stored chunk by chunk inside the exponential loop
      if (n >= 2 && !wwait(&ctl->pv_done[b], ((n - 2) >> 1) & 1)) { ok = false; break; }
      uint8_t* prow = smem + kOffP + b * kTile + (r >> 3) * kPSbo + (r & 7) * 16;
      uint32_t pk[16];
      const float rs = full ? dense_row_exp<true>(sr, 64, cst, neg, pk, prow)
                            : dense_row_exp<false>(sr, prm.n_last, cst, neg, pk, prow);
      l448 = alpha * l448 + rs;
      m_run = m_new;
      fence_proxy_async_smem();
      // Rescale the row of O when some row of the warp moved its maximum (exact: alpha = 1
      // otherwise); O is stable once P.V(n - 1) is done.
      if (n >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wwait(&ctl->pv_done[b ^ 1], ((n - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const unsigned long long a2 = f2_pack(alpha, alpha);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_addr + 32 * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float x0, x1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), x0, x1);
            o[e] = __float_as_uint(x0);
            o[e + 1] = __float_as_uint(x1);
          }
          tmem_st32(tmem + lane_addr + 32 * cc, o);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[b]);
    }
    if (ok) ok = wwait(&ctl->pv_done[(nb - 1) & 1], ((nb - 1) >> 1) & 1);
    tc_fence_after();
    if (ok) {
      const float inv_l = 1.f / l448;
      const bool store = tok < prm.N;
      const int64_t b_ = bh / prm.out_H, h_ = bh % prm.out_H;
      char* out_row = static_cast<char*>(prm.out) +
                      (b_ * prm.out_sb + h_ * prm.out_sh + static_cast<int64_t>(tok) * prm.out_sn) *
                          (prm.out_dtype == SAGESLA_F32 ? 4 : 2);
      float* sp_row = prm.sparse_out ? prm.sparse_out + (bh * prm.N + tok) * 128 : nullptr;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + 32 * cc, o);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * ctl->s_v[32 * cc + e] * inv_l;
        if (!store) continue;
        if (prm.out_dtype == SAGESLA_F32) {
          float4* dst = reinterpret_cast<float4*>(out_row) + 8 * cc;
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(out_row) + 4 * cc;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
              __nv_bfloat162 t2 = __floats2bfloat162_rn(v[8 * e + 2 * z], v[8 * e + 2 * z + 1]);
              w[z] = *reinterpret_cast<uint32_t*>(&t2);
            }
            dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        if (sp_row) {
          float4* dst = reinterpret_cast<float4*>(sp_row) + 8 * cc;
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kDTmemCols);
}

}  // namespace

cudaError_t launch_attention_dense(const ForwardPlan& p, TensorArg q, void* out, int32_t out_dtype,
                                   int64_t out_sb, int64_t out_sh, int64_t out_sn,
                                   float* sparse_out, char* ws, const AttnTestHooks& hooks,
                                   cudaStream_t stream) {
  const auto& L = p.lay;
  CUtensorMap tq, tk, tv;
  const uint64_t rows = static_cast<uint64_t>(p.BH * p.n_pad);
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, ws + L.q8, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, ws + L.k8, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, ws + L.v8, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  DenseParams prm;
  prm.sq = reinterpret_cast<const float*>(ws + L.sq);
  prm.sk = reinterpret_cast<const float*>(ws + L.sk);
  prm.s_v = reinterpret_cast<const float*>(ws + L.s_v);
  prm.out = out;
  prm.out_sb = out_sb;
  prm.out_sh = out_sh;
  prm.out_sn = out_sn;
  prm.out_dtype = out_dtype;
  prm.out_H = q.H;
  prm.sparse_out = sparse_out;
  prm.status = reinterpret_cast<int*>(ws + L.status);
  prm.N = static_cast<int>(p.N);
  prm.nb = static_cast<int>(p.nb);
  prm.nbq = static_cast<int>(2 * p.n_pairs);
  prm.n_pad = static_cast<int>(p.n_pad);
  prm.n_last = p.n_last;
  prm.spin_ns = hooks.spin_limit_us ? 1000ull * hooks.spin_limit_us : kSpinLimitNs;
  prm.skip_tile = hooks.skip_tile;
  const size_t smem = 1024 + kOffCtlD + sizeof(DenseCtl);
  cudaError_t e = cudaFuncSetAttribute(k_attention_dense, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.n_pairs), static_cast<unsigned>(p.BH));
  k_attention_dense<<<grid, kDThreads, smem, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace sagesla
