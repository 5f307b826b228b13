// Fused LayerNorm / RMSNorm + AdaLN modulation + per-token INT8 quantization.
//
// News.qq.com TurboDiffusion article, section 第四把钥匙: LayerNorm and RMSNorm are rewritten
// and fused with their neighbouring operations so that the data crosses memory fewer times;
// section 第三把钥匙: the activations of the 8-bit linear layers are quantized to INT8 on the
// fly. Here one pass over a token row reads the bf16 row once and writes the normalized,
// modulated row (bf16) and/or its INT8 codes with one scale per row.
//
// B200 mapping (K <= 8192): one warp per row, four rows per CTA. The warp copies its row into
// shared memory with cp.async (lane l copies, reads and overwrites only the 16-byte chunks
// l + 32 i, so no barrier is needed), and every reduction (mean, variance or mean square, the
// row's absolute maximum) is a warp shuffle: a row never waits for the rest of its CTA. The
// arithmetic runs on packed f32x2 pairs (each lane rounds like the scalar operation), and
// each INT8 code is one round-to-nearest-even conversion of the fp32 product. Rows of more
// than 8192 channels use one 128-thread CTA per row with the row in registers. The kernels
// are bound by HBM bandwidth: per row 2K bytes in, 2K bytes of bf16 and K bytes of codes out.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kNormThreads = 128;
constexpr int kMaxChunks = 16;              // 16 x 8 x 128 = 16384 channels

struct NormParams {
  const uint16_t* x;
  int64_t x_stride;
  int64_t M;
  int K, kind;
  float eps;
  const uint16_t *gamma, *beta, *scale, *shift;
  int64_t rows_per_sample;
  uint16_t* y;
  int64_t y_stride;
  int8_t* codes;
  int64_t codes_stride;
  float* code_scale;
};

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Sum over the CTA of one float per thread (every thread gets the total).
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

// Rows of more than kWarpRowMaxK channels: one 128-thread CTA per row.
// kCh = chunks of 8 channels per thread (K <= 8 * 128 * kCh): the row stays in registers.
template <int kCh>
__global__ void __launch_bounds__(kNormThreads)
k_norm_quant(NormParams p) {
  __shared__ float red[4];
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const int nch = p.K >> 3;                   // 8-channel chunks; thread t takes t + 128 i
  const uint4* xr = reinterpret_cast<const uint4*>(p.x + row * p.x_stride);

  uint4 raw[kCh];
#pragma unroll
  for (int i = 0; i < kCh; ++i)
    raw[i] = (t + kNormThreads * i < nch) ? __ldg(xr + t + kNormThreads * i) : make_uint4(0, 0, 0, 0);

  // statistics (fp32 sums; padded chunks hold zeros and are left out of the LayerNorm
  // deviations)
  const float inv_k = 1.0f / static_cast<float>(p.K);
  float mu = 0.f, rstd;
  if (p.kind == SAGESLA_NO_NORM) {
    rstd = 1.0f;
  } else if (p.kind == SAGESLA_LAYER_NORM) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kCh; ++i) {
      float f[8];
      unpack8(raw[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) s += f[e];
    }
    mu = block_sum(s, red) * inv_k;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < kCh; ++i) {
      if (t + kNormThreads * i >= nch) continue;
      float f[8];
      unpack8(raw[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = f[e] - mu;
        q = fmaf(d, d, q);
      }
    }
    rstd = 1.0f / sqrtf(block_sum(q, red) * inv_k + p.eps);
  } else {
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < kCh; ++i) {
      float f[8];
      unpack8(raw[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) q = fmaf(f[e], f[e], q);
    }
    rstd = 1.0f / sqrtf(block_sum(q, red) * inv_k + p.eps);
  }

  // normalize, affine, modulate, round to bf16 (kept in raw[] for the quantization)
  const int64_t b = p.rows_per_sample > 0 ? row / p.rows_per_sample : 0;
  const uint4* g4 = reinterpret_cast<const uint4*>(p.gamma);
  const uint4* be4 = reinterpret_cast<const uint4*>(p.beta);
  const uint4* sc4 = p.scale ? reinterpret_cast<const uint4*>(p.scale + b * p.K) : nullptr;
  const uint4* sh4 = p.shift ? reinterpret_cast<const uint4*>(p.shift + b * p.K) : nullptr;
  uint4* yr = p.y ? reinterpret_cast<uint4*>(p.y + row * p.y_stride) : nullptr;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kCh; ++i) {
    const int c = t + kNormThreads * i;
    if (c >= nch) continue;
    float f[8], g[8], be[8], sc[8], sh[8];
    unpack8(raw[i], f);
    if (g4) unpack8(__ldg(g4 + c), g);
    if (be4) unpack8(__ldg(be4 + c), be);
    if (sc4) unpack8(__ldg(sc4 + c), sc);
    if (sh4) unpack8(__ldg(sh4 + c), sh);
    uint32_t packed[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float y = (f[e + u] - mu) * rstd;
        if (g4) y *= g[e + u];
        if (be4) y += be[e + u];
        if (sc4) y *= 1.0f + sc[e + u];
        if (sh4) y += sh[e + u];
        v[u] = y;
      }
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[0], v[1]);
      packed[e >> 1] = *reinterpret_cast<uint32_t*>(&h2);
      amax = fmaxf(amax, fmaxf(fabsf(__low2float(h2)), fabsf(__high2float(h2))));
    }
    raw[i] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    if (yr) yr[c] = raw[i];
  }
  if (!p.codes) return;

  // per-row INT8 codes of the bf16 row: inv = fl32(127 / a), code = rne(fl32(y * inv))
  const float a = block_max(amax, red);
  const float inv = a > 0.f ? 127.0f / a : 0.f;
  uint2* cr = reinterpret_cast<uint2*>(p.codes + row * p.codes_stride);
#pragma unroll
  for (int i = 0; i < kCh; ++i) {
    const int c = t + kNormThreads * i;
    if (c >= nch) continue;
    float f[8];
    unpack8(raw[i], f);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float q = fminf(fmaxf(rintf(f[e] * inv), -127.f), 127.f);
      w[e >> 2] |= (static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu) << (8 * (e & 3));
    }
    cr[c] = make_uint2(w[0], w[1]);
  }
  if (t == 0) p.code_scale[row] = a > 0.f ? a / 127.0f : 1.0f;
}

// One warp per row (K <= 8192), the row staged in shared memory.
constexpr int kRowsPerCta = 4;
constexpr int64_t kWarpRowMaxK = 8192;
__device__ __forceinline__ void cp_async16w(void* smem_dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// The two bf16 values of a word as a packed pair (exact).
__device__ __forceinline__ unsigned long long bf2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__global__ void __launch_bounds__(32 * kRowsPerCta)
k_norm_quant_warp(NormParams p) {
  extern __shared__ uint4 rows_s[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + w;
  if (row >= p.M) return;
  const int nch = p.K >> 3;
  uint4* rs = rows_s + static_cast<int64_t>(w) * nch;
  const uint4* xr = reinterpret_cast<const uint4*>(p.x + row * p.x_stride);
  for (int c = lane; c < nch; c += 32) cp_async16w(rs + c, xr + c);
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  const float inv_k = 1.0f / static_cast<float>(p.K);
  float mu = 0.f, rstd;
  if (p.kind == SAGESLA_NO_NORM) {
    rstd = 1.0f;
  } else if (p.kind == SAGESLA_LAYER_NORM) {
    unsigned long long s2 = 0ull;
    for (int c = lane; c < nch; c += 32) {
      const uint4 v = rs[c];
      s2 = f2_add(f2_add(s2, bf2(v.x)), f2_add(bf2(v.y), f2_add(bf2(v.z), bf2(v.w))));
    }
    float sa, sb;
    f2_unpack(s2, sa, sb);
    mu = warp_sum(sa + sb) * inv_k;
    const unsigned long long nmu2 = f2_pack(-mu, -mu);
    unsigned long long q2 = 0ull;
    for (int c = lane; c < nch; c += 32) {
      const uint4 v = rs[c];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const unsigned long long d2 = f2_add(bf2(wv[e]), nmu2);
        q2 = f2_fma(d2, d2, q2);
      }
    }
    float qa, qb;
    f2_unpack(q2, qa, qb);
    rstd = 1.0f / sqrtf(warp_sum(qa + qb) * inv_k + p.eps);
  } else {
    unsigned long long q2 = 0ull;
    for (int c = lane; c < nch; c += 32) {
      const uint4 v = rs[c];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const unsigned long long x2 = bf2(wv[e]);
        q2 = f2_fma(x2, x2, q2);
      }
    }
    float qa, qb;
    f2_unpack(q2, qa, qb);
    rstd = 1.0f / sqrtf(warp_sum(qa + qb) * inv_k + p.eps);
  }
  const int64_t b = p.rows_per_sample > 0 ? row / p.rows_per_sample : 0;
  const uint4* g4 = reinterpret_cast<const uint4*>(p.gamma);
  const uint4* be4 = reinterpret_cast<const uint4*>(p.beta);
  const uint4* sc4 = p.scale ? reinterpret_cast<const uint4*>(p.scale + b * p.K) : nullptr;
  const uint4* sh4 = p.shift ? reinterpret_cast<const uint4*>(p.shift + b * p.K) : nullptr;
  uint4* yr = p.y ? reinterpret_cast<uint4*>(p.y + row * p.y_stride) : nullptr;
  float amax = 0.f;
  for (int c = lane; c < nch; c += 32) {
    const uint4 xv = rs[c];
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    const uint4 gv = g4 ? __ldg(g4 + c) : zero4, bv = be4 ? __ldg(be4 + c) : zero4;
    const uint4 sv = sc4 ? __ldg(sc4 + c) : zero4, hv = sh4 ? __ldg(sh4 + c) : zero4;
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w}, sw[4] = {sv.x, sv.y, sv.z, sv.w};
    const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
    uint32_t packed[4];
    const unsigned long long nmu2 = f2_pack(-mu, -mu), rstd2 = f2_pack(rstd, rstd), one2 = f2_pack(1.f, 1.f);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      unsigned long long y2 = f2_mul(f2_add(bf2(xw[e]), nmu2), rstd2);
      if (g4) y2 = f2_mul(y2, bf2(gw[e]));
      if (be4) y2 = f2_add(y2, bf2(bw[e]));
      if (sc4) y2 = f2_mul(y2, f2_add(one2, bf2(sw[e])));
      if (sh4) y2 = f2_add(y2, bf2(hw[e]));
      float v[2];
      f2_unpack(y2, v[0], v[1]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[0], v[1]);
      packed[e] = *reinterpret_cast<uint32_t*>(&h2);
      amax = fmaxf(amax, fmaxf(fabsf(__low2float(h2)), fabsf(__high2float(h2))));
    }
    rs[c] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    if (yr) yr[c] = rs[c];
  }
  if (!p.codes) return;
  const float a = warp_max(amax);
  const float inv = a > 0.f ? 127.0f / a : 0.f;
  uint2* cr = reinterpret_cast<uint2*>(p.codes + row * p.codes_stride);
  if (a < INFINITY) {
    // rne(fl32(y * inv)) by one rounding conversion of the fp32 product; |y * inv| <= 127.5,
    // so the code needs no clamp
    const unsigned long long inv2 = f2_pack(inv, inv);
    for (int c = lane; c < nch; c += 32) {
      const uint4 v = rs[c];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      uint32_t b[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float t0, t1;
        f2_unpack(f2_mul(bf2(wv[e]), inv2), t0, t1);
        b[2 * e] = static_cast<uint32_t>(__float2int_rn(t0));
        b[2 * e + 1] = static_cast<uint32_t>(__float2int_rn(t1));
      }
      cr[c] = make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410),
                         __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410));
    }
  } else {
    for (int c = lane; c < nch; c += 32) {
      float f[8];
      unpack8(rs[c], f);
      uint32_t wd[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float q = fminf(fmaxf(rintf(f[e] * inv), -127.f), 127.f);
        wd[e >> 2] |= (static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu) << (8 * (e & 3));
      }
      cr[c] = make_uint2(wd[0], wd[1]);
    }
  }
  if (lane == 0) p.code_scale[row] = a > 0.f ? a / 127.0f : 1.0f;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlaps(const void* a0, size_t na, const void* b0, size_t nb) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(a0), b = reinterpret_cast<uintptr_t>(b0);
  return a < b + nb && b < a + na;
}

}  // namespace
}  // namespace sagesla

extern "C" sagesla_status sagesla_norm_quant(const sagesla_norm_args* a, void* stream) {
  using namespace sagesla;
  if (!a || !a->x) return SAGESLA_ERR_INVALID_ARG;
  if (a->M < 1 || a->K < 1) return SAGESLA_ERR_INVALID_ARG;
  if (a->K < 8 || a->K > 8 * kNormThreads * kMaxChunks || a->K % 8 != 0) return SAGESLA_ERR_UNSUPPORTED;
  if (a->M > 0x7FFFFFFF) return SAGESLA_ERR_UNSUPPORTED;
  if (a->kind != SAGESLA_LAYER_NORM && a->kind != SAGESLA_RMS_NORM && a->kind != SAGESLA_NO_NORM)
    return SAGESLA_ERR_INVALID_ARG;
  if (a->kind == SAGESLA_NO_NORM && a->gamma) return SAGESLA_ERR_INVALID_ARG;
  if (!(a->eps >= 0.f) || !std::isfinite(a->eps)) return SAGESLA_ERR_INVALID_ARG;
  if (a->beta && a->kind != SAGESLA_LAYER_NORM) return SAGESLA_ERR_INVALID_ARG;
  if (!a->y && !a->codes) return SAGESLA_ERR_INVALID_ARG;
  if ((a->codes == nullptr) != (a->code_scale == nullptr)) return SAGESLA_ERR_INVALID_ARG;
  if ((a->scale || a->shift) && a->rows_per_sample < 1) return SAGESLA_ERR_INVALID_ARG;
  if (a->x_stride < a->K || a->x_stride % 8 != 0 || !aligned(a->x, 16)) return SAGESLA_ERR_INVALID_ARG;
  for (const void* v : {static_cast<const void*>(a->gamma), static_cast<const void*>(a->beta),
                        static_cast<const void*>(a->scale), static_cast<const void*>(a->shift)})
    if (v && !aligned(v, 16)) return SAGESLA_ERR_INVALID_ARG;
  const size_t x_bytes = static_cast<size_t>((a->M - 1) * a->x_stride + a->K) * 2;
  if (a->y) {
    if (a->y_stride < a->K || a->y_stride % 8 != 0 || !aligned(a->y, 16)) return SAGESLA_ERR_INVALID_ARG;
    if (overlaps(a->y, static_cast<size_t>((a->M - 1) * a->y_stride + a->K) * 2, a->x, x_bytes))
      return SAGESLA_ERR_INVALID_ARG;
  }
  if (a->codes) {
    if (a->codes_stride < a->K || a->codes_stride % 8 != 0 || !aligned(a->codes, 8) ||
        !aligned(a->code_scale, 4))
      return SAGESLA_ERR_INVALID_ARG;
    if (overlaps(a->codes, static_cast<size_t>((a->M - 1) * a->codes_stride + a->K), a->x, x_bytes) ||
        overlaps(a->code_scale, static_cast<size_t>(a->M) * 4, a->x, x_bytes))
      return SAGESLA_ERR_INVALID_ARG;
  }
  sagesla_status st = require_b200();
  if (st != SAGESLA_OK) return st;
  NormParams p;
  p.x = a->x;
  p.x_stride = a->x_stride;
  p.K = static_cast<int>(a->K);
  p.kind = a->kind;
  p.eps = a->eps;
  p.gamma = a->gamma;
  p.beta = a->beta;
  p.scale = a->scale;
  p.shift = a->shift;
  p.rows_per_sample = (a->scale || a->shift) ? a->rows_per_sample : 0;
  p.y = a->y;
  p.y_stride = a->y_stride;
  p.codes = a->codes;
  p.codes_stride = a->codes_stride;
  p.code_scale = a->code_scale;
  p.M = a->M;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->K <= kWarpRowMaxK) {   // one warp per row, rows staged in shared memory
    const int smem = kRowsPerCta * static_cast<int>(a->K) * 2;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_norm_quant_warp, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return SAGESLA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>((a->M + kRowsPerCta - 1) / kRowsPerCta);
    k_norm_quant_warp<<<grid, 32 * kRowsPerCta, smem, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
  }
  const int ch = static_cast<int>((a->K / 8 + kNormThreads - 1) / kNormThreads);
  const dim3 grid(static_cast<unsigned>(a->M));
  if (ch <= 12) k_norm_quant<12><<<grid, kNormThreads, 0, s>>>(p);   // K in (8192, 12288]
  else k_norm_quant<kMaxChunks><<<grid, kNormThreads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}
