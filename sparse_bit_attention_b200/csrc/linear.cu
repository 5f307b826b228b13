// Linear branch, step 1: the complement sums G_i = sum over key blocks j NOT kept by query
// block i of H_j (H_j = phi(K_j)^T [V_j | 1], built by k_stats).
//
// "Sparse-Linear Attention" (dgmzs.com.cn README translation, section 方法论; bonega.ai
// article, section "SLA: Sparse-Linear Attention"): the blocks the sparse branch skips are
// covered by linear attention. Per head this is one dense GEMM
//     G[nb x 16512] = (1 - M)[nb x nb] . Hflat[nb x 16512]
// with the binary complement mask as the A operand (exact in bf16). It runs on tcgen05:
// 256 x 256 output tiles as two M=128 accumulators that share each B tile (the whole 512-column
// TMEM of the SM), 64-deep K steps, a 3-stage TMA pipeline (A K-major, B MN-major, both
// 128-byte swizzled), one MMA-issuing thread, fp32 accumulation and a bf16 epilogue by eight
// warps. Sharing B between two accumulators cuts the L2 -> SM operand traffic per FLOP by a
// third against 128 x 256 tiles; that traffic, not the tensor pipe, bounds this GEMM.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

// Bulk tensor store of a shared-memory box to global memory (bulk async group of this thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int x,
                                             int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_store_commit_and_wait() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

constexpr int kStages = 3;
constexpr int kTileM = 256, kTileN = 256, kTileK = 64;   // kTileM = 2 accumulators x 128
constexpr uint32_t kABytes = kTileM * kTileK * 2;   // 32 KB
constexpr uint32_t kBBytes = kTileK * kTileN * 2;   // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kGemmSmem = kStages * kStageBytes + 1024 + 256;
constexpr int kGemmThreads = 320;   // warps 0-7 epilogue, 8 TMA producer, 9 MMA issuer

__global__ void __launch_bounds__(kGemmThreads, 1)
k_complement_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_g, int nb_m_pad, int nb_k_pad,
                  int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f0 = blockIdx.x * kTileN;
  const int m0 = blockIdx.y * kTileM;
  const int64_t bh = blockIdx.z;
  const int nkt = nb_k_pad / kTileK;
  const bool two = m0 + 128 < nb_m_pad;   // second accumulator has rows of this head

  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 64) { prefetch_tmap(&tm_a); prefetch_tmap(&tm_b); prefetch_tmap(&tm_g); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8 && lane == 0) {   // TMA producer
    const uint32_t bytes = (two ? kABytes : kABytes / 2) + kBBytes;
    for (int kt = 0; kt < nkt; ++kt) {
      const int s = kt % kStages;
      if (kt >= kStages && !mbar_wait(&empty[s], ((kt / kStages) - 1) & 1, status)) break;
      uint8_t* a = smem + s * kStageBytes;
      uint8_t* b = a + kABytes;
      mbar_arrive_expect_tx(&full[s], bytes);
      tma_load_2d(a, &tm_a, &full[s], kt * kTileK, static_cast<int>(bh * nb_m_pad + m0));
      if (two)
        tma_load_2d(a + kABytes / 2, &tm_a, &full[s], kt * kTileK,
                    static_cast<int>(bh * nb_m_pad + m0 + 128));
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tma_load_2d(b + q * 8192, &tm_b, &full[s], f0 + 64 * q,
                    static_cast<int>(bh * nb_k_pad + kt * kTileK));
    }
  } else if (warp == 9 && lane == 0) {   // MMA issuer
    constexpr uint32_t idesc = make_idesc(kFmtF32, kFmtBF16, kFmtBF16, 0, 1, 128, kTileN);
    bool ok = true;
    for (int kt = 0; kt < nkt && ok; ++kt) {
      const int s = kt % kStages;
      ok = mbar_wait(&full[s], (kt / kStages) & 1, status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * kStageBytes);
      const uint32_t b = a + kABytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {   // 4 x K=16
        const uint64_t bd = make_sdesc(b + kk * 2048, 8192, 1024, kLayoutSW128);
        mma_bf16(tmem, make_sdesc(a + kk * 32, 16, 1024, kLayoutSW128), bd, idesc,
                 (kt | kk) ? 1u : 0u);
        if (two)
          mma_bf16(tmem + 256, make_sdesc(a + kABytes / 2 + kk * 32, 16, 1024, kLayoutSW128), bd,
                   idesc, (kt | kk) ? 1u : 0u);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  } else if (warp < 8) {
    // Epilogue, warp w: accumulator w / 4, rows 32 (w % 4) + lane. The 32 x 256 bf16 slab goes
    // through the freed pipeline buffers as four 32 x 64 boxes in the 128-byte-swizzled layout
    // and leaves with bulk tensor stores (columns past the end of G are clipped by the store).
    const int acc = warp >> 2, quad = warp & 3;
    const bool ok = mbar_wait(done, 0, status);
    tc_fence_after();
    if (ok && (acc == 0 || two)) {
      uint8_t* slab = smem + warp * (32 * 512);   // 16 KB per warp
#pragma unroll 1
      for (int cc = 0; cc < kTileN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem, 32 * quad, 256 * acc + 32 * cc), r);
        tmem_ld_wait();
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]),
                                                    __uint_as_float(r[2 * e + 1]));
          packed[e] = *reinterpret_cast<uint32_t*>(&v2);
        }
        // columns 32cc .. 32cc+31 = chunks 4(cc&1) .. +3 of box cc/2
        uint8_t* box = slab + (cc >> 1) * 4096 + lane * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = 4 * (cc & 1) + q;
          *reinterpret_cast<uint4*>(box + ((chunk ^ (lane & 7)) << 4)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int row = static_cast<int>(bh * nb_m_pad + m0 + 128 * acc + 32 * quad);
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (f0 + 64 * b < kHFlat) tma_store_2d(&tm_g, slab + b * 4096, f0 + 64 * b, row);
        tma_store_commit_and_wait();
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_mask_gemm(const void* a, const void* b, void* c, int64_t BH, int64_t M,
                             int64_t K, int* status, cudaStream_t stream) {
  CUtensorMap ta, tb, tg;
  if (!encode_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, BH * M, K * 2, a, kTileK, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHFlat, BH * K,
                      static_cast<uint64_t>(kHFlat) * 2, b, 64, kTileK, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHFlat, BH * M,
                      static_cast<uint64_t>(kHFlat) * 2, c, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // set on every call: the attribute belongs to the current device
  cudaError_t e = cudaFuncSetAttribute(k_complement_gemm,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((kHFlat + kTileN - 1) / kTileN, static_cast<unsigned>((M + kTileM - 1) / kTileM),
            static_cast<unsigned>(BH));
  k_complement_gemm<<<grid, kGemmThreads, kGemmSmem, stream>>>(
      ta, tb, tg, static_cast<int>(M), static_cast<int>(K), status);
  return cudaGetLastError();
}

cudaError_t launch_complement_gemm(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  const auto& L = p.lay;
  return launch_mask_gemm(ws + L.amask, ws + L.hflat, ws + L.gsum, p.BH, p.nb_m_pad, p.nb_k_pad,
                          reinterpret_cast<int*>(ws + L.status), stream);
}

}  // namespace sagesla
