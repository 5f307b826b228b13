// Prologue of the SageSLA forward: per-head K/V statistics, key-block states for the linear
// branch, and the INT8 / FP8 quantization of Q, K, V.
//
//  k_stats    one CTA per (key block j, head): per-channel K sums (float64, exact for bf16
//             data of ordinary range), per-channel |V| maxima, the pooled K mean of the
//             block, and H_j = phi(K_j)^T [V_j | 1] with phi = softmax over the 128
//             channels. The 128x128 part of H_j is one tcgen05 BF16 MMA (M = channel,
//             N = value column, K = 64 tokens, both operands MN-major in 128-byte-swizzled
//             shared memory); column 128 is the per-channel sum of the same bf16 phi values.
//  k_finalize one CTA per head: K channel mean rounded to bf16 (the smoothing vector) and the
//             V channel scales.
//  k_quant    one CTA per (block i, head): pooled Q mean, INT8 codes of Q and of the smoothed
//             K with one scale per 64-token block, e4m3 codes of V with one scale per channel.
//
// Quantization follows the news.qq.com TurboDiffusion article, sections 第一把钥匙 (8-bit
// attention operands) and 第三把钥匙 (one scale per block; outliers smoothed before
// quantization); the linear-branch state follows the "Sparse-Linear Attention" method named
// in the dgmzs.com.cn README translation, section 方法论.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& raw, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ld_row_chunk(const uint16_t* base, int64_t off) {
  return __ldg(reinterpret_cast<const uint4*>(base + off));
}

// Round a double to the nearest bfloat16 value (ties to even), returned as a float.
// Exact for results of magnitude in [2^-126, 2^128); smaller magnitudes go through the
// float conversion (bf16 subnormal channel means are not expected).
__device__ __forceinline__ float double_to_bf16_rne(double x) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  if ((b & 0x7FFFFFFFFFFFFFFFull) == 0 || ((b >> 52) & 0x7FF) == 0x7FF) return static_cast<float>(x);
  const unsigned long long lsb = (b >> 45) & 1ull;   // lowest kept mantissa bit (7 kept)
  b += 0x00000FFFFFFFFFFFull + lsb;                  // 2^44 - 1 + lsb
  b &= ~((1ull << 45) - 1ull);
  return static_cast<float>(__longlong_as_double(static_cast<long long>(b)));
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}

constexpr int kStatsThreads = 128;
// Two 16 KB operand tiles + alignment slack. Four CTAs per SM, each holding 128 TMEM columns
// from its start (measured on B200: allocating TMEM only around the MMA, to let six CTAs
// share an SM, made the kernel almost twice as slow).
constexpr int kStatsSmem = 33 * 1024;

// kLinear = false (every key block kept, no linear branch): only the K sums, V amax and
// pooled K are needed, so phi, H_j and its MMA are skipped.
//
// Thread t serves the 8-channel chunk ch = t & 15 of rows g, g+8, ..., g+56 (g = t >> 4); the
// 16 chunks of a row sit in 16 lanes of one warp. K and V arrive by cp.async directly in the
// layout the MMA reads (128-byte-swizzled, MN-major: row r, chunk ch at
// (ch / 8) * 8 KB + sw128(r, ch % 8)), so each thread turns its own K chunks into phi in place.
template <bool kLinear>
__global__ void __launch_bounds__(kStatsThreads, 4)
k_stats(TensorArg K, TensorArg V, int N, int nb, int nb_k_pad, double* __restrict__ ksum_part,
        float* __restrict__ vmax_part, float* __restrict__ kbar, __nv_bfloat16* __restrict__ hflat,
        int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* a_tile = smem;               // K_j, then phi(K_j) as [token][channel], 2 x 8 KB
  uint8_t* b_tile = smem + 16384;       // V_j as [token][column], 2 x 8 KB
  // per-row-group partial sums, in the operand tiles once the MMA has read them
  double* red_k = reinterpret_cast<double*>(smem);                // [8][128]
  float* red_v = reinterpret_cast<float*>(smem + 8192);           // [8][128]
  float* red_p = red_v + 8 * 128;                                 // [8][128]

  const int j = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  __nv_bfloat16* hrow = hflat + (bh * nb_k_pad + j) * static_cast<int64_t>(kHFlat);

  if (j >= nb) {  // zero padding rows of the complement-sum GEMM operand
    if (kLinear)
      for (int e = t; e < kHFlat; e += kStatsThreads) hrow[e] = __float2bfloat16_rn(0.f);
    return;
  }

  const int64_t b = bh / K.H, h = bh % K.H;
  const uint16_t* kb = static_cast<const uint16_t*>(K.data) + b * K.stride_b + h * K.stride_h;
  const uint16_t* vb = static_cast<const uint16_t*>(V.data) + b * V.stride_b + h * V.stride_h;
  const int n0 = j * kBlock;
  const int nj = min(kBlock, N - n0);
  const int ch = t & 15;   // 8-channel chunk
  const int g = t >> 4;    // row group: rows g, g+8, ..., g+56

  if (kLinear && warp == 0) {
    tmem_alloc(&tmem_slot, 128);
    tmem_relinquish();
    tc_fence_before();
  }
  // all of this thread's K and V chunks in flight at once (rows past the end read as zeros)
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int r = g + 8 * s;
    const bool in = r < nj;
    const int64_t row = n0 + (in ? r : 0);
    const uint32_t off = (ch >> 3) * 8192u + sw128_offset(r, ch & 7);
    cp_async16(a_tile + off, kb + row * K.stride_n + 8 * ch, in ? 16u : 0u);
    cp_async16(b_tile + off, vb + row * V.stride_n + 8 * ch, in ? 16u : 0u);
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  if (kLinear && t == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();

  double ksum[8];
  float vmax[8], psum[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { ksum[e] = 0.0; vmax[e] = 0.f; psum[e] = 0.f; }

#pragma unroll 2
  for (int s = 0; s < 8; ++s) {
    const int r = g + 8 * s;
    const bool valid = r < nj;
    const uint32_t off = (ch >> 3) * 8192u + sw128_offset(r, ch & 7);
    float kf[8], vf[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(a_tile + off), kf);
    unpack_bf16x8(*reinterpret_cast<const uint4*>(b_tile + off), vf);
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ksum[e] += static_cast<double>(kf[e]);
      vmax[e] = fmaxf(vmax[e], fabsf(vf[e]));
      mx = fmaxf(mx, kf[e]);
    }
    if constexpr (kLinear) {
      // phi = softmax over the 128 channels of this token; the row lives in 16 lanes.
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float ex[8], sum = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) { ex[e] = __expf(kf[e] - mx); sum += ex[e]; }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = 1.0f / sum;
      uint32_t packed[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        __nv_bfloat162 p2 = __floats2bfloat162_rn(valid ? ex[e] * inv : 0.f,
                                                  valid ? ex[e + 1] * inv : 0.f);
        packed[e / 2] = *reinterpret_cast<uint32_t*>(&p2);
        psum[e] += __low2float(p2);
        psum[e + 1] += __high2float(p2);
      }
      *reinterpret_cast<uint4*>(a_tile + off) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }

  uint32_t tmem = 0;
  bool ok = true;
  if (kLinear) {
    fence_proxy_async_smem();
    __syncthreads();                     // phi and V complete; the barrier is initialized
    if (warp == 0) {
      tc_fence_after();
      if (lane == 0) {
        constexpr uint32_t idesc = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 1, 1, 128, 128);
        const uint32_t d = tmem_slot;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {   // 4 x K=16 tokens
          const uint64_t ad = make_sdesc(smem_u32(a_tile) + kk * 2048, 8192, 1024, kLayoutSW128);
          const uint64_t bd = make_sdesc(smem_u32(b_tile) + kk * 2048, 8192, 1024, kLayoutSW128);
          mma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar);
      }
    }
    // the operand tiles are free for the reductions once the MMA has read them
    ok = mbar_wait(&bar, 0, status);
  } else {
    __syncthreads();                     // every thread is done with the tiles
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    red_k[g * 128 + 8 * ch + e] = ksum[e];
    red_v[g * 128 + 8 * ch + e] = vmax[e];
    red_p[g * 128 + 8 * ch + e] = psum[e];
  }
  __syncthreads();
  if (kLinear) {                         // the TMEM address written by warp 0's allocation
    tc_fence_after();
    tmem = tmem_slot;
  }
  {  // per-channel reductions (thread t = channel t), fixed order over row groups
    const int c = t;
    double ks = 0.0;
    float vm = 0.f, ps = 0.f;
    for (int gg = 0; gg < 8; ++gg) {
      ks += red_k[gg * 128 + c];
      vm = fmaxf(vm, red_v[gg * 128 + c]);
      ps += red_p[gg * 128 + c];
    }
    const int64_t o = (bh * nb + j) * 128 + c;
    ksum_part[o] = ks;
    vmax_part[o] = vm;
    kbar[o] = static_cast<float>(ks / static_cast<double>(nj));
    if (kLinear) hrow[128 * 128 + c] = __float2bfloat16_rn(ps);
  }
  if (!kLinear) return;

  // H_j[c][n] (TMEM lane c, column n) -> hrow[n][c]: each warp stores 32 consecutive channels
  // (64 contiguous bytes) of one value column per store.
  if (ok) {
    const int c = 32 * warp + lane;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
      tmem_ld32(tmem_addr(tmem, 32 * warp, 32 * cc), r);
      tmem_ld_wait();
      uint16_t* dst = reinterpret_cast<uint16_t*>(hrow) + (32 * cc) * 128 + c;
#pragma unroll
      for (int e = 0; e < 32; ++e)
        dst[e * 128] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[e])));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

constexpr int kFinalizeThreads = 1024;   // 8 partitions x 128 channels

__global__ void __launch_bounds__(kFinalizeThreads)
k_finalize(int N, int nb, const double* __restrict__ ksum_part, const float* __restrict__ vmax_part,
           float* __restrict__ mu, float* __restrict__ s_v, float* __restrict__ inv_v) {
  __shared__ double sk[8][128];
  __shared__ float sv[8][128];
  const int64_t bh = blockIdx.x;
  const int c = threadIdx.x & 127, part = threadIdx.x >> 7;
  double s = 0.0;
  float m = 0.f;
  for (int j = part; j < nb; j += 8) {
    s += ksum_part[(bh * nb + j) * 128 + c];
    m = fmaxf(m, vmax_part[(bh * nb + j) * 128 + c]);
  }
  sk[part][c] = s;
  sv[part][c] = m;
  __syncthreads();
  if (part == 0) {
    double tot = 0.0;
    float amax = 0.f;
    for (int q = 0; q < 8; ++q) { tot += sk[q][c]; amax = fmaxf(amax, sv[q][c]); }
    mu[bh * 128 + c] = double_to_bf16_rne(tot / static_cast<double>(N));
    s_v[bh * 128 + c] = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    inv_v[bh * 128 + c] = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.0f;
  }
}

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
  return m;
}

__device__ __forceinline__ uint2 int8_codes(const float (&x)[8], float inv) {
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int c = __float2int_rn(__fmul_rn(x[e], inv));
    c = max(-127, min(127, c));
    w[e >> 2] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (e & 3));
  }
  return make_uint2(w[0], w[1]);
}

__global__ void __launch_bounds__(kQuantThreads)
k_quant(TensorArg Q, TensorArg K, TensorArg V, int N, int nb, int n_pad, int nbq,
        const float* __restrict__ mu, const float* __restrict__ inv_v, int8_t* __restrict__ q8,
        int8_t* __restrict__ k8, uint8_t* __restrict__ v8, float* __restrict__ sq,
        float* __restrict__ sk, float* __restrict__ qbar) {
  __shared__ float red[8];
  __shared__ float colsum[16][129];
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int t = threadIdx.x;
  const int ch = t & 15, g = t >> 4;    // rows g, g+16, g+32, g+48
  const int n0 = i * kBlock;
  const int ni = i < nb ? min(kBlock, N - n0) : 0;
  const int64_t b = bh / Q.H, h = bh % Q.H;
  const int64_t row0 = bh * n_pad + n0;

  // ---- Q: pooled mean and INT8 codes
  float x[4][8];
  {
    const uint16_t* base = static_cast<const uint16_t*>(Q.data) + b * Q.stride_b + h * Q.stride_h;
    float amax = 0.f;
    float cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int r = g + 16 * s;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (r < ni) raw = ld_row_chunk(base, (n0 + r) * Q.stride_n + 8 * ch);
      unpack_bf16x8(raw, x[s]);
#pragma unroll
      for (int e = 0; e < 8; ++e) { amax = fmaxf(amax, fabsf(x[s][e])); cs[e] += x[s][e]; }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) colsum[g][8 * ch + e] = cs[e];
    amax = block_max_256(amax, red);   // contains __syncthreads: colsum is complete
    if (i < nb && t < 128) {
      float s = 0.f;
      for (int gg = 0; gg < 16; ++gg) s += colsum[gg][t];
      qbar[(bh * nb + i) * 128 + t] = __fdiv_rn(s, static_cast<float>(ni));
    }
    const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int r = g + 16 * s;
      *reinterpret_cast<uint2*>(q8 + (row0 + r) * 128 + 8 * ch) = int8_codes(x[s], inv);
    }
    if (t == 0) sq[bh * nbq + i] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 1.0f;
  }
  // ---- K: smoothed by the channel mean, INT8 codes
  {
    const uint16_t* base = static_cast<const uint16_t*>(K.data) + b * K.stride_b + h * K.stride_h;
    float m8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m8[e] = mu[bh * 128 + 8 * ch + e];
    float amax = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int r = g + 16 * s;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (r < ni) raw = ld_row_chunk(base, (n0 + r) * K.stride_n + 8 * ch);
      unpack_bf16x8(raw, x[s]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[s][e] = r < ni ? __fsub_rn(x[s][e], m8[e]) : 0.f;
        amax = fmaxf(amax, fabsf(x[s][e]));
      }
    }
    amax = block_max_256(amax, red);
    const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int r = g + 16 * s;
      *reinterpret_cast<uint2*>(k8 + (row0 + k8_row_position(r)) * 128 + 8 * ch) =
          int8_codes(x[s], inv);
    }
    if (t == 0) sk[bh * nbq + i] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 1.0f;
  }
  // ---- V: e4m3 codes with the per-channel scale
  {
    const uint16_t* base = static_cast<const uint16_t*>(V.data) + b * V.stride_b + h * V.stride_h;
    float iv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) iv[e] = inv_v[bh * 128 + 8 * ch + e];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int r = g + 16 * s;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (r < ni) raw = ld_row_chunk(base, (n0 + r) * V.stride_n + 8 * ch);
      float vf[8];
      unpack_bf16x8(raw, vf);
      uint32_t w[2];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const uint16_t pair = f32x2_to_e4m3x2(__fmul_rn(vf[e], iv[e]), __fmul_rn(vf[e + 1], iv[e + 1]));
        if ((e & 2) == 0) w[e >> 2] = pair; else w[e >> 2] |= static_cast<uint32_t>(pair) << 16;
      }
      *reinterpret_cast<uint2*>(v8 + (row0 + r) * 128 + 8 * ch) = make_uint2(w[0], w[1]);
    }
  }
}

}  // namespace

cudaError_t launch_stats(const ForwardPlan& p, TensorArg k, TensorArg v, char* ws,
                         cudaStream_t stream) {
  // set on every call: the attribute belongs to the current device
  for (const void* f : {reinterpret_cast<const void*>(k_stats<true>),
                        reinterpret_cast<const void*>(k_stats<false>)}) {
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kStatsSmem);
    if (e != cudaSuccess) return e;
  }
  const auto& L = p.lay;
  dim3 grid(static_cast<unsigned>(p.nb_k_pad), static_cast<unsigned>(p.BH));
  auto kern = p.linear_empty ? k_stats<false> : k_stats<true>;
  kern<<<grid, kStatsThreads, kStatsSmem, stream>>>(
      k, v, static_cast<int>(p.N), static_cast<int>(p.nb), static_cast<int>(p.nb_k_pad),
      reinterpret_cast<double*>(ws + L.ksum_part), reinterpret_cast<float*>(ws + L.vmax_part),
      reinterpret_cast<float*>(ws + L.kbar), reinterpret_cast<__nv_bfloat16*>(ws + L.hflat),
      reinterpret_cast<int*>(ws + L.status));
  return cudaGetLastError();
}

cudaError_t launch_finalize(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  k_finalize<<<static_cast<unsigned>(p.BH), kFinalizeThreads, 0, stream>>>(
      static_cast<int>(p.N), static_cast<int>(p.nb),
      reinterpret_cast<const double*>(ws + L.ksum_part),
      reinterpret_cast<const float*>(ws + L.vmax_part), reinterpret_cast<float*>(ws + L.mu),
      reinterpret_cast<float*>(ws + L.s_v), reinterpret_cast<float*>(ws + L.inv_v));
  return cudaGetLastError();
}

// bf16 operand copies for the 16-bit modes of the attention: rows [head][n_pad][128] with
// zero rows past N, 16 bytes per thread. Q and V keep the token order; K rows are stored
// key-interleaved inside each 64-key block like the INT8 codes (row 2(r mod 32) + r div 32
// holds key r), so that every softmax thread's TMEM fragment holds 32 consecutive keys.
__global__ void k_pack_bf16(TensorArg src, int N, int n_pad, int64_t total, int interleave,
                            uint4* __restrict__ dst) {
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= total) return;
  const int chunk = static_cast<int>(idx & 15);
  const int64_t row = idx >> 4;
  const int64_t bh = row / n_pad;
  const int pos = static_cast<int>(row - bh * n_pad);
  // token held by stored row `pos`: the inverse of the interleaving within its block
  const int in_block = pos & 63;
  const int n = interleave ? (pos - in_block) + (in_block >> 1) + 32 * (in_block & 1) : pos;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (n < N) {
    const int64_t b = bh / src.H, h = bh % src.H;
    const uint16_t* base = static_cast<const uint16_t*>(src.data) + b * src.stride_b +
                           h * src.stride_h + static_cast<int64_t>(n) * src.stride_n;
    v = __ldg(reinterpret_cast<const uint4*>(base) + chunk);
  }
  dst[idx] = v;
}

cudaError_t launch_pack_bf16(const ForwardPlan& p, TensorArg q, TensorArg k, TensorArg v,
                             char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  const int64_t total = p.BH * p.n_pad * 16;
  const unsigned grid = static_cast<unsigned>((total + 255) / 256);
  const int N = static_cast<int>(p.N), n_pad = static_cast<int>(p.n_pad);
  if (!p.quant) {
    k_pack_bf16<<<grid, 256, 0, stream>>>(q, N, n_pad, total, 0, reinterpret_cast<uint4*>(ws + L.qb));
    k_pack_bf16<<<grid, 256, 0, stream>>>(k, N, n_pad, total, 1, reinterpret_cast<uint4*>(ws + L.kb));
  }
  if (!p.pv_fp8)
    k_pack_bf16<<<grid, 256, 0, stream>>>(v, N, n_pad, total, 0, reinterpret_cast<uint4*>(ws + L.vb));
  return cudaGetLastError();
}

cudaError_t launch_quant(const ForwardPlan& p, TensorArg q, TensorArg k, TensorArg v, char* ws,
                         cudaStream_t stream) {
  const auto& L = p.lay;
  const int nbq = static_cast<int>(2 * p.n_pairs);
  dim3 grid(static_cast<unsigned>(nbq), static_cast<unsigned>(p.BH));
  k_quant<<<grid, kQuantThreads, 0, stream>>>(
      q, k, v, static_cast<int>(p.N), static_cast<int>(p.nb), static_cast<int>(p.n_pad), nbq,
      reinterpret_cast<const float*>(ws + L.mu), reinterpret_cast<const float*>(ws + L.inv_v),
      reinterpret_cast<int8_t*>(ws + L.q8), reinterpret_cast<int8_t*>(ws + L.k8),
      reinterpret_cast<uint8_t*>(ws + L.v8), reinterpret_cast<float*>(ws + L.sq),
      reinterpret_cast<float*>(ws + L.sk), reinterpret_cast<float*>(ws + L.qbar));
  return cudaGetLastError();
}

}  // namespace sagesla
