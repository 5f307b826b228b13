// W8A8 linear layer: INT8 weights in 128x128 blocks (one scale per block), INT8 activations
// with one scale per token row, the GEMM on the tcgen05 INT8 tensor cores.
//
// News.qq.com TurboDiffusion article, section 第三把钥匙: weights and activations both in
// 8-bit integers so that the whole linear layer runs in the integer domain on the INT8 tensor
// cores, with block-wise weight quantization (128x128 blocks, one scale per block) and
// activations quantized on the fly.
//
//  k_w8a8_quant_weight  one CTA per 128x128 weight block: block max, IEEE 127/a, codes
//                       rounded to nearest even (bit-exact with the block quantizer of the
//                       attention's INT8 step).
//  k_w8a8_gemm          Y tile 128 x 256 per CTA (one CTA per SM). Each 128-deep K block is
//                       one weight block: its exact int32 product comes out of 4 M=128 N=256
//                       K=32 kind::i8 MMAs into one of two TMEM buffers (2 x 256 columns),
//                       and eight "promotion" warps move it into fp32 register accumulators
//                       scaled by the block's weight scale (one exact int -> float conversion
//                       per element, |s| < 2^22, then one packed FMA), while the tensor core already
//                       works on the next K block in the other buffer. The epilogue multiplies
//                       by the token scale, adds the bias, rounds and leaves through shared
//                       memory with bulk tensor stores.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kWB = 128;                         // weight block (rows and columns)

// ------------------------------------------------------------------ weight quantization
__global__ void __launch_bounds__(256)
k_w8a8_quant_weight(const uint16_t* __restrict__ w, int N, int K, int64_t w_stride,
                    int8_t* __restrict__ w8, float* __restrict__ w_scale) {
  __shared__ float red[8];
  const int bk = blockIdx.x, bn = blockIdx.y;
  const int t = threadIdx.x;
  const int rows = min(kWB, N - kWB * bn);
  // 128 rows x 16 chunks of 8 columns; thread t takes chunk (t & 15) of rows t/16 + 16 i
  const int ch = t & 15, r0 = t >> 4;
  uint4 raw[8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + 16 * i;
    raw[i] = make_uint4(0, 0, 0, 0);
    if (r < rows)
      raw[i] = __ldg(reinterpret_cast<const uint4*>(
          w + (static_cast<int64_t>(kWB) * bn + r) * w_stride + kWB * bk + 8 * ch));
    const uint32_t v[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(v[e] << 16)),
                               fabsf(__uint_as_float(v[e] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  float a = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
  const float inv = a > 0.f ? 127.0f / a : 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + 16 * i;
    if (r >= rows) continue;
    const uint32_t v[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = __uint_as_float(e & 1 ? (v[e >> 1] & 0xFFFF0000u) : (v[e >> 1] << 16));
      const float q = fminf(fmaxf(rintf(x * inv), -127.f), 127.f);
      packed[e >> 2] |= (static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu) << (8 * (e & 3));
    }
    *reinterpret_cast<uint2*>(w8 + (static_cast<int64_t>(kWB) * bn + r) * K + kWB * bk + 8 * ch) =
        make_uint2(packed[0], packed[1]);
  }
  if (t == 0) w_scale[static_cast<int64_t>(bn) * (K / kWB) + bk] = a > 0.f ? a / 127.0f : 1.0f;
}

// ------------------------------------------------------------------ GEMM
constexpr int kGM = 128, kGN = 256;              // output tile
constexpr int kGStages = 4;
constexpr uint32_t kGABytes = kGM * kWB;         // 16 KB of x8
constexpr uint32_t kGBBytes = kGN * kWB;         // 32 KB of w8
constexpr uint32_t kGStageBytes = kGABytes + kGBBytes;
constexpr int kGThreads = 320;                   // warps 0-7 promotion, 8 producer, 9 MMA
constexpr int kGSmem = kGStages * kGStageBytes + 1024 + 256;

struct GemmParams {
  const float* x_scale;
  const float* w_scale;
  const uint16_t* bias;
  int M, N, nkb;
  int y_f32;
  int* status;
};

__device__ __forceinline__ void tma_store_2d_g(const CUtensorMap* map, const void* smem_src,
                                               int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y)
      : "memory");
}

__global__ void __launch_bounds__(kGThreads, 1)
k_w8a8_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
            const __grid_constant__ CUtensorMap tm_y, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* acc_full = empty + kGStages;           // [2] MMA done into TMEM buffer b
  uint64_t* acc_empty = acc_full + 2;              // [2] promotion warps done reading b
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kGN, m0 = blockIdx.y * kGM;
  const int nkb = p.nkb;

  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kGStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 8); }
    fence_mbar_init();
  }
  if (threadIdx.x == 64) { prefetch_tmap(&tm_x); prefetch_tmap(&tm_w); prefetch_tmap(&tm_y); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {   // TMA producer: x8 tile 128 x 128, w8 tile 256 x 128 per K block
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kGStages;
        if (kb >= kGStages && !mbar_wait(&empty[s], ((kb / kGStages) - 1) & 1, p.status)) break;
        uint8_t* a = smem + s * kGStageBytes;
        mbar_arrive_expect_tx(&full[s], kGStageBytes);
        tma_load_2d(a, &tm_x, &full[s], kWB * kb, m0);
        tma_load_2d(a + kGABytes, &tm_w, &full[s], kWB * kb, n0);
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {   // MMA issuer: 4 x (M=128 N=256 K=32) per K block into TMEM buffer kb & 1
      constexpr uint32_t idesc = make_idesc(kFmtS32, kFmtS8, kFmtS8, 0, 0, kGM, kGN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kGStages, b = kb & 1;
        if (!mbar_wait(&full[s], (kb / kGStages) & 1, p.status)) break;
        if (kb >= 2 && !mbar_wait(&acc_empty[b], ((kb >> 1) - 1) & 1, p.status)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * kGStageBytes);
        const uint64_t da = make_sdesc(a, 16, 1024, kLayoutSW128);
        const uint64_t dw = make_sdesc(a + kGABytes, 16, 1024, kLayoutSW128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // 32-byte K steps add 2 to the address field
          mma_i8(tmem + 256 * b, da + 2 * kk, dw + 2 * kk, idesc, kk > 0 ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&acc_full[b]);
      }
    }
  } else {
    // Promotion and epilogue. Warp w reads TMEM lanes 32 (w & 3) .. +31 (its rows) and the
    // columns 128 (w >> 2) .. +127 of each buffer; each thread keeps 128 fp32 accumulators
    // of its row as 64 packed pairs.
    const int q = warp & 3, hf = warp >> 2;
    const int nb = (n0 >> 7) + hf;                 // weight block row of these columns
    const float* wsc = p.w_scale + static_cast<int64_t>(nb) * nkb;
    unsigned long long acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0ull;
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      const int b = kb & 1;
      const float c = __ldg(wsc + kb);
      const unsigned long long c2 = f2_pack(c, c);
      if (!mbar_wait(&acc_full[b], (kb >> 1) & 1, p.status)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem, 32 * q, 256 * b + 128 * hf + 32 * cc), r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const unsigned long long f2 = f2_pack(__int2float_rn(static_cast<int>(r[e])),
                                             __int2float_rn(static_cast<int>(r[e + 1])));
          acc[16 * cc + (e >> 1)] = f2_fma(c2, f2, acc[16 * cc + (e >> 1)]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
    // every MMA has completed once the last buffer is read; the stage memory is free
    __syncwarp();
    if (ok) {
      const int m = m0 + 32 * q + lane;
      const float sx = m < p.M ? __ldg(p.x_scale + m) : 0.f;
      const int ncol0 = n0 + 128 * hf;
      float bias[2] = {0.f, 0.f};
      uint8_t* slab = smem + warp * 16384;       // 32 rows x 128 columns (f32: 16 KB)
      if (p.y_f32) {
        // four 32-row x 32-column f32 boxes, 128-byte swizzle
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float v0, v1;
          f2_unpack(acc[i], v0, v1);
          const int col = 2 * i;
          if (p.bias) {
            const int n = ncol0 + col;
            bias[0] = n < p.N ? __bfloat162float(__ushort_as_bfloat16(p.bias[n])) : 0.f;
            bias[1] = n + 1 < p.N ? __bfloat162float(__ushort_as_bfloat16(p.bias[n + 1])) : 0.f;
          }
          v0 = fmaf(v0, sx, bias[0]);
          v1 = fmaf(v1, sx, bias[1]);
          const int box = col >> 5, chunk = (col & 31) >> 2;
          float* dst = reinterpret_cast<float*>(slab + box * 4096 + lane * 128 +
                                                ((chunk ^ (lane & 7)) << 4)) + (col & 3);
          dst[0] = v0;
          dst[1] = v1;
        }
      } else {
        // two 32-row x 64-column bf16 boxes, 128-byte swizzle
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float v0, v1;
          f2_unpack(acc[i], v0, v1);
          const int col = 2 * i;
          if (p.bias) {
            const int n = ncol0 + col;
            bias[0] = n < p.N ? __bfloat162float(__ushort_as_bfloat16(p.bias[n])) : 0.f;
            bias[1] = n + 1 < p.N ? __bfloat162float(__ushort_as_bfloat16(p.bias[n + 1])) : 0.f;
          }
          __nv_bfloat162 h2 = __floats2bfloat162_rn(fmaf(v0, sx, bias[0]), fmaf(v1, sx, bias[1]));
          const int box = col >> 6, chunk = (col & 63) >> 3;
          uint32_t* dst = reinterpret_cast<uint32_t*>(slab + box * 4096 + lane * 128 +
                                                      ((chunk ^ (lane & 7)) << 4)) + ((col & 7) >> 1);
          *dst = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int boxes = p.y_f32 ? 4 : 2, bw = p.y_f32 ? 32 : 64;
        for (int bx = 0; bx < boxes; ++bx) {
          const int x = ncol0 + bw * bx;
          if (x < p.N && m0 + 32 * q < p.M) tma_store_2d_g(&tm_y, slab + bx * 4096, x, m0 + 32 * q);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool overlaps(uintptr_t a, size_t na, uintptr_t b, size_t nb) { return a < b + nb && b < a + na; }

}  // namespace
}  // namespace sagesla

extern "C" sagesla_status sagesla_w8a8_quantize_weight(const uint16_t* w, int64_t N, int64_t K,
                                                       int64_t w_stride, int8_t* w8,
                                                       float* w_scale, void* stream) {
  using namespace sagesla;
  if (!w || !w8 || !w_scale || N < 1 || K < 1) return SAGESLA_ERR_INVALID_ARG;
  if (K % kWB != 0 || K > (1 << 20) || N > 0x7FFFFFFF) return SAGESLA_ERR_UNSUPPORTED;
  if (w_stride < K || w_stride % 8 != 0 || !aligned16(w) || !aligned16(w8) ||
      (reinterpret_cast<uintptr_t>(w_scale) & 3) != 0)
    return SAGESLA_ERR_INVALID_ARG;
  const sagesla_status st = require_b200();
  if (st != SAGESLA_OK) return st;
  const dim3 grid(static_cast<unsigned>(K / kWB), static_cast<unsigned>((N + kWB - 1) / kWB));
  k_w8a8_quant_weight<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      w, static_cast<int>(N), static_cast<int>(K), w_stride, w8, w_scale);
  return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}

extern "C" sagesla_status sagesla_w8a8_gemm(const int8_t* x8, const float* x_scale, int64_t M,
                                            int64_t K, const int8_t* w8, const float* w_scale,
                                            int64_t N, const uint16_t* bias, void* y,
                                            int32_t y_dtype, int64_t y_stride, int32_t* status,
                                            void* stream) {
  using namespace sagesla;
  if (!x8 || !x_scale || !w8 || !w_scale || !y || M < 1 || N < 1 || K < 1)
    return SAGESLA_ERR_INVALID_ARG;
  if (y_dtype != SAGESLA_BF16 && y_dtype != SAGESLA_F32) return SAGESLA_ERR_INVALID_ARG;
  if (K % kWB != 0 || K > (1 << 20) || M > 0x7FFFFFFF || N > 0x7FFFFFFF || N % 8 != 0)
    return SAGESLA_ERR_UNSUPPORTED;
  const int64_t esz = y_dtype == SAGESLA_F32 ? 4 : 2;
  if (y_stride < N || (y_stride * esz) % 16 != 0) return SAGESLA_ERR_INVALID_ARG;
  for (const void* q : {static_cast<const void*>(x8), static_cast<const void*>(w8),
                        static_cast<const void*>(y), static_cast<const void*>(x_scale),
                        static_cast<const void*>(w_scale)})
    if (!aligned16(q)) return SAGESLA_ERR_INVALID_ARG;
  if (bias && !aligned16(bias)) return SAGESLA_ERR_INVALID_ARG;
  if (status && (reinterpret_cast<uintptr_t>(status) & 3) != 0) return SAGESLA_ERR_INVALID_ARG;
  const uintptr_t y0 = reinterpret_cast<uintptr_t>(y);
  const size_t ybytes = static_cast<size_t>((M - 1) * y_stride + N) * esz;
  if (overlaps(y0, ybytes, reinterpret_cast<uintptr_t>(x8), static_cast<size_t>(M * K)) ||
      overlaps(y0, ybytes, reinterpret_cast<uintptr_t>(w8), static_cast<size_t>(N * K)) ||
      overlaps(y0, ybytes, reinterpret_cast<uintptr_t>(x_scale), static_cast<size_t>(M) * 4) ||
      overlaps(y0, ybytes, reinterpret_cast<uintptr_t>(w_scale),
               static_cast<size_t>((N + kWB - 1) / kWB * (K / kWB)) * 4))
    return SAGESLA_ERR_INVALID_ARG;
  sagesla_status st = require_b200();
  if (st != SAGESLA_OK) return st;
  CUtensorMap tx, tw, ty;
  if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, x8, kWB, kGM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, w8, kWB, kGN,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&ty, y_dtype == SAGESLA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                  : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                      N, M, y_stride * esz, y, y_dtype == SAGESLA_F32 ? 32 : 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return SAGESLA_ERR_CUDA;
  // set on every call: the attribute belongs to the current device
  if (cudaFuncSetAttribute(k_w8a8_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem) !=
      cudaSuccess)
    return SAGESLA_ERR_CUDA;
  GemmParams p;
  p.x_scale = x_scale;
  p.w_scale = w_scale;
  p.bias = bias;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.nkb = static_cast<int>(K / kWB);
  p.y_f32 = y_dtype == SAGESLA_F32 ? 1 : 0;
  p.status = status;
  const dim3 grid(static_cast<unsigned>((N + kGN - 1) / kGN), static_cast<unsigned>((M + kGM - 1) / kGM));
  k_w8a8_gemm<<<grid, kGThreads, kGSmem, static_cast<cudaStream_t>(stream)>>>(tx, tw, ty, p);
  return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}
