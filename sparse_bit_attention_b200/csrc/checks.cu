// Workspace canaries of the debug_checks option: 16 bytes after the end of every workspace
// region (the plan reserves the gap) are set to a known pattern before a forward's first
// kernel and compared after its last one. A kernel that wrote past the end of a region
// damages the pattern, and the comparison records SAGESLA_ERR_CANARY in the status word,
// which the host reads after synchronizing (sagesla_stream_status).
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

struct CanaryList {
  uint64_t off[kMaxCanaries];
  int n;
  uint64_t status;
};

// Pattern word w (0..3) of canary c: distinct per region and per word, never zero.
__host__ __device__ constexpr uint32_t canary_word(int c, int w) {
  return 0xC0DE5A17u ^ (static_cast<uint32_t>(c) << 8) ^ (static_cast<uint32_t>(w) << 4);
}

__global__ void k_canary_fill(char* ws, CanaryList l) {
  const int c = threadIdx.x;
  if (c >= l.n) return;
  *reinterpret_cast<uint4*>(ws + l.off[c]) =
      make_uint4(canary_word(c, 0), canary_word(c, 1), canary_word(c, 2), canary_word(c, 3));
}

__global__ void k_canary_verify(char* ws, CanaryList l) {
  const int c = threadIdx.x;
  if (c >= l.n) return;
  const uint4 v = *reinterpret_cast<const uint4*>(ws + l.off[c]);
  if (v.x != canary_word(c, 0) || v.y != canary_word(c, 1) || v.z != canary_word(c, 2) ||
      v.w != canary_word(c, 3))
    record_error(reinterpret_cast<int*>(ws + l.status), SAGESLA_ERR_CANARY);
}

CanaryList canary_list(const ForwardPlan& p) {
  CanaryList l;
  l.n = p.n_canary;
  for (int c = 0; c < kMaxCanaries; ++c) l.off[c] = c < p.n_canary ? p.canary[c] : 0;
  l.status = p.lay.status;
  return l;
}

}  // namespace

cudaError_t launch_canary_fill(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  k_canary_fill<<<1, kMaxCanaries, 0, stream>>>(ws, canary_list(p));
  return cudaGetLastError();
}

cudaError_t launch_canary_verify(const ForwardPlan& p, char* ws, cudaStream_t stream) {
  k_canary_verify<<<1, kMaxCanaries, 0, stream>>>(ws, canary_list(p));
  return cudaGetLastError();
}

}  // namespace sagesla
