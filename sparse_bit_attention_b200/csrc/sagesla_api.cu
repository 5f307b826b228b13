// Host side of the C ABI: argument validation, the workspace plan, tensor-map encoding and
// the launch sequence of one SageSLA forward. No allocation, no synchronization (except in
// sagesla_forward_host and sagesla_stream_status, which say so).
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool valid_ratio(double r) { return std::isfinite(r) && r > 0.0 && r <= 1.0; }

int64_t topk_count(int64_t nb, double r) {
  int64_t k = static_cast<int64_t>(std::ceil(r * static_cast<double>(nb) - 1e-9));
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return k;
}

// Problem-size limits of this implementation.
constexpr int64_t kMaxBH = 65535;              // grid.y
constexpr int64_t kMaxBlocks = 1 << 15;        // score row must fit in shared memory
constexpr size_t kMaxListSmem = 120 * 1024;    // kept-list union in the attention kernel

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

}  // namespace

bool make_plan(int64_t B, int64_t H, int64_t N, double topk_ratio, ForwardPlan* p, bool quant,
               bool pv_fp8) {
  if (B < 1 || H < 1 || N < 1 || !valid_ratio(topk_ratio)) return false;
  if (!quant && pv_fp8) return false;          // bf16 Q.K^T with e4m3 P.V is not a mode
  std::memset(p, 0, sizeof(*p));
  p->quant = quant;
  p->pv_fp8 = pv_fp8;
  p->B = B;
  p->H = H;
  p->N = N;
  p->BH = B * H;
  p->nb = ceil_div(N, kBlock);
  p->k = topk_count(p->nb, topk_ratio);
  p->n_pairs = ceil_div(p->nb, 2);
  p->n_pad = 128 * p->n_pairs;
  p->mask_words = ceil_div(p->nb, 32);
  p->scores_ld = ceil_div(p->nb, 4) * 4;
  p->nb_k_pad = ceil_div(p->nb, 64) * 64;
  p->nb_m_pad = ceil_div(p->nb, 128) * 128;
  p->n_last = static_cast<int32_t>(N - kBlock * (p->nb - 1));
  p->linear_empty = p->k == p->nb;
  if (p->BH > kMaxBH || p->nb > kMaxBlocks) return false;
  if (static_cast<size_t>(p->nb < 2 * p->k ? p->nb : 2 * p->k) * 8 > kMaxListSmem) return false;
  if (p->BH * p->nb_m_pad * 129 >= (int64_t(1) << 31) || p->BH * p->n_pad >= (int64_t(1) << 31))
    return false;

  sagesla_workspace_layout& L = p->lay;
  const int64_t BH = p->BH, nb = p->nb, nbq = 2 * p->n_pairs;
  size_t off = 0;
  // Each region starts on a kAlign boundary and is followed by its 16-byte canary (used by
  // debug_checks) at its end rounded up to 16.
  auto take = [&](size_t bytes) {
    const size_t at = off;
    const size_t canary = align_up(at + bytes, 16);
    if (p->n_canary < kMaxCanaries) p->canary[p->n_canary++] = canary;
    off = align_up(canary + 16, kAlign);
    return at;
  };
  L.nb = nb;
  L.k = p->k;
  L.n_pad = p->n_pad;
  L.mask_words = p->mask_words;
  L.nb_k_pad = p->nb_k_pad;
  L.nb_m_pad = p->nb_m_pad;
  L.status = take(sizeof(int32_t));
  L.q8 = take(static_cast<size_t>(BH * p->n_pad * 128));
  L.k8 = take(static_cast<size_t>(BH * p->n_pad * 128));
  L.v8 = take(static_cast<size_t>(BH * p->n_pad * 128));
  L.sq = take(static_cast<size_t>(BH * nbq) * 4);
  L.sk = take(static_cast<size_t>(BH * nbq) * 4);
  L.s_v = take(static_cast<size_t>(BH * 128) * 4);
  L.inv_v = take(static_cast<size_t>(BH * 128) * 4);
  L.mu = take(static_cast<size_t>(BH * 128) * 4);
  L.qbar = take(static_cast<size_t>(BH * nb * 128) * 4);
  L.kbar = take(static_cast<size_t>(BH * nb * 128) * 4);
  L.ksum_part = take(static_cast<size_t>(BH * nb * 128) * 8);
  L.vmax_part = take(static_cast<size_t>(BH * nb * 128) * 4);
  L.scores = take(static_cast<size_t>(BH * nb * p->scores_ld) * 4);
  L.kept = take(static_cast<size_t>(BH * nb * p->k) * 4);
  L.mask = take(static_cast<size_t>(BH * nb * p->mask_words) * 4);
  L.amask = take(static_cast<size_t>(BH * p->nb_m_pad * p->nb_k_pad) * 2);
  L.hflat = take(static_cast<size_t>(BH * p->nb_k_pad) * kHFlat * 2);
  L.gsum = take(static_cast<size_t>(BH * p->nb_m_pad) * kHFlat * 2);
  // bf16 operand copies of the 16-bit modes (offset 0 = absent: the status word is there)
  if (!quant) {
    L.qb = take(static_cast<size_t>(BH * p->n_pad) * 256);
    L.kb = take(static_cast<size_t>(BH * p->n_pad) * 256);
  }
  if (!pv_fp8) L.vb = take(static_cast<size_t>(BH * p->n_pad) * 256);
  L.total_bytes = off;
  return true;
}

namespace {
// cuTensorMapEncodeTiled through the runtime's driver entry point, resolved once.
bool have_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}
}  // namespace

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, const void* base, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle) {
  if (!have_encode()) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_nd(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                    const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                    CUtensorMapSwizzle swizzle) {
  if (!have_encode() || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (uint32_t r = 0; r < rank; ++r) { d[r] = dims[r]; b[r] = box[r]; es[r] = 1; }
  for (uint32_t r = 0; r + 1 < rank; ++r) st[r] = strides[r];
  const CUresult res = g_encode(map, dtype, rank, const_cast<void*>(base), d, st, b, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

namespace {

size_t elem_bytes(int32_t dtype) { return dtype == SAGESLA_F32 ? 4 : 2; }

// Byte range [lo, hi) touched by a tensor view.
void extent(const sagesla_tensor* t, uintptr_t* lo, uintptr_t* hi) {
  const size_t eb = elem_bytes(t->dtype);
  const int64_t last = (t->B - 1) * t->stride_b + (t->H - 1) * t->stride_h +
                       (t->N - 1) * t->stride_n + t->D;
  *lo = reinterpret_cast<uintptr_t>(t->data);
  *hi = *lo + static_cast<uintptr_t>(last) * eb;
}

bool overlaps(uintptr_t a0, uintptr_t a1, uintptr_t b0, uintptr_t b1) {
  return a0 < b1 && b0 < a1;
}

sagesla_status check_view(const sagesla_tensor* t, const sagesla_tensor* ref, bool is_out) {
  if (!t || !t->data) return SAGESLA_ERR_INVALID_ARG;
  if (t->D != kHeadDim) return SAGESLA_ERR_UNSUPPORTED;
  if (is_out ? (t->dtype != SAGESLA_BF16 && t->dtype != SAGESLA_F32) : t->dtype != SAGESLA_BF16)
    return SAGESLA_ERR_UNSUPPORTED;
  if (t->B < 1 || t->H < 1 || t->N < 1) return SAGESLA_ERR_INVALID_ARG;
  if (ref && (t->B != ref->B || t->H != ref->H || t->N != ref->N)) return SAGESLA_ERR_INVALID_ARG;
  const int64_t eb = static_cast<int64_t>(elem_bytes(t->dtype));
  if (t->stride_n < t->D || t->stride_h < 0 || t->stride_b < 0) return SAGESLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(t->data) & 15) != 0 || (t->stride_n * eb) % 16 != 0 ||
      (t->stride_h * eb) % 16 != 0 || (t->stride_b * eb) % 16 != 0)
    return SAGESLA_ERR_INVALID_ARG;
  return SAGESLA_OK;
}

TensorArg to_arg(const sagesla_tensor* t) {
  TensorArg a;
  a.data = t->data;
  a.stride_b = t->stride_b;
  a.stride_h = t->stride_h;
  a.stride_n = t->stride_n;
  a.H = static_cast<int32_t>(t->H);
  return a;
}

sagesla_status check_device() { return require_b200(); }

#define SAGESLA_LAUNCH(call)                            \
  do {                                                  \
    if ((call) != cudaSuccess) return SAGESLA_ERR_CUDA; \
  } while (0)

// NVTX range around the launches of one stage (named "sagesla.<stage>"), so that a timeline
// or an ncu --nvtx filter can find each kernel of a call; a no-op without a tool attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace

// The current device must be a compute-capability-10.0 part (B200).
sagesla_status require_b200() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGESLA_ERR_NO_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGESLA_ERR_NO_DEVICE;
  if (major != 10 || minor != 0) return SAGESLA_ERR_NO_DEVICE;
  return SAGESLA_OK;
}

}  // namespace sagesla

using namespace sagesla;

extern "C" {

const char* sagesla_status_string(sagesla_status s) {
  switch (s) {
    case SAGESLA_OK: return "ok";
    case SAGESLA_ERR_INVALID_ARG: return "invalid argument";
    case SAGESLA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SAGESLA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case SAGESLA_ERR_CUDA: return "CUDA error";
    case SAGESLA_ERR_TIMEOUT: return "device-side wait timed out";
    case SAGESLA_ERR_DEVICE_CHECK: return "device-side check failed";
    case SAGESLA_ERR_NO_DEVICE: return "no sm_100 device current";
    case SAGESLA_ERR_BOUNDS: return "index or coordinate out of range (access skipped)";
    case SAGESLA_ERR_CANARY: return "workspace canary overwritten";
  }
  return "unknown status";
}

int64_t sagesla_topk_count(int64_t N, double topk_ratio, int block) {
  if (N < 1 || block != kBlock || !valid_ratio(topk_ratio)) return -1;
  return topk_count(ceil_div(N, kBlock), topk_ratio);
}

int sagesla_build_checks(void) { return kChecks ? 1 : 0; }

void sagesla_options_init(sagesla_options* opt) {
  if (!opt) return;
  std::memset(opt, 0, sizeof(*opt));
  opt->quant = 1;
  opt->pv_fp8 = 1;
}

}  // extern "C"

namespace {
// Operand mode of a call: the options' quant / pv_fp8 (defaults without options).
sagesla_status read_mode(const sagesla_options* opt, bool* quant, bool* pv_fp8) {
  *quant = true;
  *pv_fp8 = true;
  if (!opt) return SAGESLA_OK;
  if ((opt->quant != 0 && opt->quant != 1) || (opt->pv_fp8 != 0 && opt->pv_fp8 != 1))
    return SAGESLA_ERR_INVALID_ARG;
  if (opt->quant == 0 && opt->pv_fp8 == 1) return SAGESLA_ERR_UNSUPPORTED;
  *quant = opt->quant != 0;
  *pv_fp8 = opt->pv_fp8 != 0;
  if (opt->debug_checks != 0 && opt->debug_checks != 1) return SAGESLA_ERR_INVALID_ARG;
  if (opt->debug_plant < 0 || opt->debug_plant > 2) return SAGESLA_ERR_INVALID_ARG;
  if (opt->debug_plant == 1 && !opt->debug_checks) return SAGESLA_ERR_INVALID_ARG;
  // an out-of-range kept index is only safe where the kernels check it
  if (opt->debug_plant == 2 && !kChecks) return SAGESLA_ERR_UNSUPPORTED;
  return SAGESLA_OK;
}
}  // namespace

extern "C" {

sagesla_status sagesla_get_workspace_layout_ex(int64_t B, int64_t H, int64_t N, int64_t D,
                                               double topk_ratio, int block,
                                               const sagesla_options* opt,
                                               sagesla_workspace_layout* layout) {
  if (!layout) return SAGESLA_ERR_INVALID_ARG;
  if (D != kHeadDim || block != kBlock) return SAGESLA_ERR_UNSUPPORTED;
  bool quant, pv_fp8;
  const sagesla_status st = read_mode(opt, &quant, &pv_fp8);
  if (st != SAGESLA_OK) return st;
  ForwardPlan p;
  if (!make_plan(B, H, N, topk_ratio, &p, quant, pv_fp8)) return SAGESLA_ERR_INVALID_ARG;
  *layout = p.lay;
  return SAGESLA_OK;
}

sagesla_status sagesla_get_workspace_layout(int64_t B, int64_t H, int64_t N, int64_t D,
                                            double topk_ratio, int block,
                                            sagesla_workspace_layout* layout) {
  return sagesla_get_workspace_layout_ex(B, H, N, D, topk_ratio, block, nullptr, layout);
}

size_t sagesla_workspace_size_ex(int64_t B, int64_t H, int64_t N, int64_t D, double topk_ratio,
                                 int block, const sagesla_options* opt) {
  sagesla_workspace_layout L;
  if (sagesla_get_workspace_layout_ex(B, H, N, D, topk_ratio, block, opt, &L) != SAGESLA_OK)
    return 0;
  return L.total_bytes;
}

size_t sagesla_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, double topk_ratio,
                              int block) {
  return sagesla_workspace_size_ex(B, H, N, D, topk_ratio, block, nullptr);
}

sagesla_status sagesla_forward_ex(const sagesla_tensor* q, const sagesla_tensor* k,
                                  const sagesla_tensor* v, double topk_ratio, int block,
                                  sagesla_tensor* out, void* workspace, size_t workspace_bytes,
                                  void* stream_ptr, const sagesla_options* opt) {
  sagesla_status st;
  if ((st = check_view(q, nullptr, false)) != SAGESLA_OK) return st;
  if ((st = check_view(k, q, false)) != SAGESLA_OK) return st;
  if ((st = check_view(v, q, false)) != SAGESLA_OK) return st;
  if ((st = check_view(out, q, true)) != SAGESLA_OK) return st;
  if (block != kBlock) return SAGESLA_ERR_UNSUPPORTED;
  if (!valid_ratio(topk_ratio)) return SAGESLA_ERR_INVALID_ARG;
  bool quant, pv_fp8;
  if ((st = read_mode(opt, &quant, &pv_fp8)) != SAGESLA_OK) return st;
  ForwardPlan p;
  if (!make_plan(q->B, q->H, q->N, topk_ratio, &p, quant, pv_fp8)) return SAGESLA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      workspace_bytes < p.lay.total_bytes)
    return SAGESLA_ERR_WORKSPACE;
  uintptr_t o0, o1, a0, a1;
  extent(out, &o0, &o1);
  for (const sagesla_tensor* t : {q, k, v}) {
    extent(t, &a0, &a1);
    if (overlaps(o0, o1, a0, a1)) return SAGESLA_ERR_INVALID_ARG;
  }
  const uintptr_t w0 = reinterpret_cast<uintptr_t>(workspace);
  if (overlaps(o0, o1, w0, w0 + p.lay.total_bytes)) return SAGESLA_ERR_INVALID_ARG;
  if ((st = check_device()) != SAGESLA_OK) return st;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  char* ws = static_cast<char*>(workspace);
  const TensorArg qa = to_arg(q), ka = to_arg(k), va = to_arg(v);
  void** ev = opt ? opt->stage_events : nullptr;
  auto mark = [&](int i) -> cudaError_t {
    return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), stream) : cudaSuccess;
  };
  const bool checks = opt && opt->debug_checks;
  const int plant = opt ? opt->debug_plant : 0;
  SAGESLA_LAUNCH(cudaMemsetAsync(ws + p.lay.status, 0, sizeof(int32_t), stream));
  if (checks) SAGESLA_LAUNCH(launch_canary_fill(p, ws, stream));
  // failure-path test: damage the canary after the scores region (host-side injection)
  if (plant == 1) SAGESLA_LAUNCH(cudaMemsetAsync(ws + p.canary[13], 0, 4, stream));
  NvtxRange call_range("sagesla.forward");
  SAGESLA_LAUNCH(mark(0));
  {
    NvtxRange r("sagesla.stats");
    SAGESLA_LAUNCH(launch_stats(p, ka, va, ws, stream));
  }
  SAGESLA_LAUNCH(mark(1));
  {
    NvtxRange r("sagesla.finalize");
    SAGESLA_LAUNCH(launch_finalize(p, ws, stream));
  }
  SAGESLA_LAUNCH(mark(2));
  {
    NvtxRange r("sagesla.quant");
    SAGESLA_LAUNCH(launch_quant(p, qa, ka, va, ws, stream));
    if (!p.quant || !p.pv_fp8) SAGESLA_LAUNCH(launch_pack_bf16(p, qa, ka, va, ws, stream));
  }
  SAGESLA_LAUNCH(mark(3));
  // With every key block kept (k == nb) the selection is the identity: the scores are only
  // computed when asked for, and the kept lists and masks only written when asked for.
  const bool want_lists = opt && (opt->kept_idx_out || opt->mask_out);
  if (!p.linear_empty || (opt && opt->scores_out)) {
    NvtxRange r("sagesla.scores");
    SAGESLA_LAUNCH(launch_scores(p, ws, stream));
  }
  SAGESLA_LAUNCH(mark(4));
  {
    NvtxRange r("sagesla.topk");
    if (!p.linear_empty) SAGESLA_LAUNCH(launch_topk(p, ws, stream));
    else if (want_lists) SAGESLA_LAUNCH(launch_fill_all_kept(p, ws, stream));
  }
  // failure-path test of the checking build: an out-of-range first kept index (-1)
  if (plant == 2) SAGESLA_LAUNCH(cudaMemsetAsync(ws + p.lay.kept, 0xFF, 4, stream));
  SAGESLA_LAUNCH(mark(5));
  if (!p.linear_empty) {
    NvtxRange r("sagesla.complement_gemm");
    SAGESLA_LAUNCH(launch_complement_gemm(p, ws, stream));
  }
  SAGESLA_LAUNCH(mark(6));
  AttnTestHooks hooks{};
  if (opt) {
    hooks.spin_limit_us = opt->debug_spin_limit_us;
    hooks.skip_tile = opt->debug_skip_tile != 0;
  }
  {
    NvtxRange r("sagesla.attention");
    if (p.linear_empty && p.quant && p.pv_fp8)
      SAGESLA_LAUNCH(launch_attention_dense(p, qa, out->data, out->dtype, out->stride_b,
                                            out->stride_h, out->stride_n,
                                            opt ? opt->sparse_out : nullptr, ws, hooks, stream));
    else
      SAGESLA_LAUNCH(launch_attention(p, qa, out->data, out->dtype, out->stride_b,
                                      out->stride_h, out->stride_n,
                                      opt ? opt->sparse_out : nullptr, ws, hooks, stream));
  }
  SAGESLA_LAUNCH(mark(SAGESLA_N_STAGES));
  if (checks) SAGESLA_LAUNCH(launch_canary_verify(p, ws, stream));
  if (opt) {
    if (opt->kept_idx_out)
      SAGESLA_LAUNCH(cudaMemcpyAsync(opt->kept_idx_out, ws + p.lay.kept,
                                     static_cast<size_t>(p.BH * p.nb * p.k) * 4,
                                     cudaMemcpyDeviceToDevice, stream));
    if (opt->mask_out)
      SAGESLA_LAUNCH(cudaMemcpyAsync(opt->mask_out, ws + p.lay.mask,
                                     static_cast<size_t>(p.BH * p.nb * p.mask_words) * 4,
                                     cudaMemcpyDeviceToDevice, stream));
    if (opt->scores_out) SAGESLA_LAUNCH(launch_scale_scores(p, ws, opt->scores_out, stream));
  }
  return SAGESLA_OK;
}

sagesla_status sagesla_forward(const sagesla_tensor* q, const sagesla_tensor* k,
                               const sagesla_tensor* v, double topk_ratio, int block,
                               sagesla_tensor* out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return sagesla_forward_ex(q, k, v, topk_ratio, block, out, workspace, workspace_bytes, stream,
                            nullptr);
}

size_t sagesla_sla_backward_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                           double topk_ratio, int block) {
  if (D != kHeadDim || block != kBlock) return 0;
  ForwardPlan p;
  if (!make_plan(B, H, N, topk_ratio, &p)) return 0;
  BackwardLayout bl;
  if (!make_backward_layout(p, &bl)) return 0;
  return bl.total;
}

sagesla_status sagesla_sla_backward(const sagesla_tensor* q, const sagesla_tensor* k,
                                    const sagesla_tensor* v, const sagesla_tensor* d_out,
                                    double topk_ratio, int block, sagesla_tensor* dq,
                                    sagesla_tensor* dk, sagesla_tensor* dv, void* workspace,
                                    size_t workspace_bytes, void* stream_ptr) {
  sagesla_status st;
  if ((st = check_view(q, nullptr, false)) != SAGESLA_OK) return st;
  for (const sagesla_tensor* t : {k, v, d_out})
    if ((st = check_view(t, q, false)) != SAGESLA_OK) return st;
  for (const sagesla_tensor* t : {dq, dk, dv})
    if ((st = check_view(t, q, true)) != SAGESLA_OK) return st;
  if (dk->dtype != dq->dtype || dv->dtype != dq->dtype) return SAGESLA_ERR_UNSUPPORTED;
  if (block != kBlock) return SAGESLA_ERR_UNSUPPORTED;
  if (!valid_ratio(topk_ratio)) return SAGESLA_ERR_INVALID_ARG;
  ForwardPlan p;
  if (!make_plan(q->B, q->H, q->N, topk_ratio, &p)) return SAGESLA_ERR_INVALID_ARG;
  BackwardLayout bl;
  if (!make_backward_layout(p, &bl)) return SAGESLA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      workspace_bytes < bl.total)
    return SAGESLA_ERR_WORKSPACE;
  // outputs must not overlap the inputs, each other or the workspace
  const uintptr_t w0 = reinterpret_cast<uintptr_t>(workspace);
  const sagesla_tensor* outs[3] = {dq, dk, dv};
  for (int a = 0; a < 3; ++a) {
    uintptr_t o0, o1, x0, x1;
    extent(outs[a], &o0, &o1);
    if (overlaps(o0, o1, w0, w0 + bl.total)) return SAGESLA_ERR_INVALID_ARG;
    for (const sagesla_tensor* t : {q, k, v, d_out}) {
      extent(t, &x0, &x1);
      if (overlaps(o0, o1, x0, x1)) return SAGESLA_ERR_INVALID_ARG;
    }
    for (int b = a + 1; b < 3; ++b) {
      extent(outs[b], &x0, &x1);
      if (overlaps(o0, o1, x0, x1)) return SAGESLA_ERR_INVALID_ARG;
    }
  }
  if ((st = check_device()) != SAGESLA_OK) return st;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  char* ws = static_cast<char*>(workspace);
  const TensorArg qa = to_arg(q), ka = to_arg(k), va = to_arg(v), da = to_arg(d_out);
  NvtxRange call_range("sagesla.sla_backward");
  SAGESLA_LAUNCH(cudaMemsetAsync(ws + p.lay.status, 0, sizeof(int32_t), stream));
  // the forward's selection and complement sums (same kernels, so the same block mask)
  {
    NvtxRange r("sagesla.backward_prologue");
    SAGESLA_LAUNCH(launch_stats(p, ka, va, ws, stream));
    SAGESLA_LAUNCH(launch_finalize(p, ws, stream));
    SAGESLA_LAUNCH(launch_quant(p, qa, ka, va, ws, stream));
    if (!p.quant || !p.pv_fp8) SAGESLA_LAUNCH(launch_pack_bf16(p, qa, ka, va, ws, stream));
    if (!p.linear_empty) {
      SAGESLA_LAUNCH(launch_scores(p, ws, stream));
      SAGESLA_LAUNCH(launch_topk(p, ws, stream));
      SAGESLA_LAUNCH(launch_complement_gemm(p, ws, stream));
    } else {
      SAGESLA_LAUNCH(launch_fill_all_kept(p, ws, stream));
    }
  }
  GradOut g;
  g.dq = dq->data; g.dk = dk->data; g.dv = dv->data;
  const sagesla_tensor* gs[3] = {dq, dk, dv};
  int64_t* dst[3] = {g.dq_s, g.dk_s, g.dv_s};
  for (int a = 0; a < 3; ++a) {
    dst[a][0] = gs[a]->stride_b;
    dst[a][1] = gs[a]->stride_h;
    dst[a][2] = gs[a]->stride_n;
  }
  g.dtype = dq->dtype;
  NvtxRange r("sagesla.backward_gradients");
  SAGESLA_LAUNCH(launch_sla_backward(p, bl, qa, ka, va, da, g, ws, stream));
  return SAGESLA_OK;
}

}  // extern "C"

namespace sagesla {
namespace {
// The host entry point works through the heads in chunks so that the host->device copy of
// one chunk, the forward of the previous one and the device->host copy of the one before
// overlap (three streams). Device memory: one forward workspace for a chunk of heads, two
// slots of chunk inputs and outputs, and one status word per chunk.
constexpr int64_t kHostChunks = 16;

int64_t host_chunk_heads(int64_t BH) { return ceil_div(BH, BH < kHostChunks ? BH : kHostChunks); }

struct HostPlan {
  int64_t hc, nchunks;
  size_t fw, in_bytes, out_bytes, slot_bytes, status_off, total;
};

bool host_plan(int64_t B, int64_t H, int64_t N, int64_t D, double topk_ratio, int block,
               int32_t out_dtype, HostPlan* hp) {
  if (out_dtype != SAGESLA_BF16 && out_dtype != SAGESLA_F32) return false;
  if (B < 1 || H < 1 || sagesla_workspace_size(B, H, N, D, topk_ratio, block) == 0) return false;
  const int64_t BH = B * H;
  hp->hc = host_chunk_heads(BH);
  hp->nchunks = ceil_div(BH, hp->hc);
  hp->fw = sagesla_workspace_size(1, hp->hc, N, D, topk_ratio, block);
  if (hp->fw == 0) return false;
  const size_t elems = static_cast<size_t>(hp->hc * N * D);
  hp->in_bytes = align_up(elems * 2, kAlign);
  hp->out_bytes = align_up(elems * elem_bytes(out_dtype), kAlign);
  hp->slot_bytes = 3 * hp->in_bytes + hp->out_bytes;
  hp->status_off = hp->fw + 2 * hp->slot_bytes;
  hp->total = hp->status_off + align_up(static_cast<size_t>(hp->nchunks) * 4, kAlign);
  return true;
}
}  // namespace
}  // namespace sagesla

extern "C" {

size_t sagesla_host_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                   double topk_ratio, int block, int32_t out_dtype) {
  HostPlan hp;
  return host_plan(B, H, N, D, topk_ratio, block, out_dtype, &hp) ? hp.total : 0;
}

sagesla_status sagesla_stream_status(void* stream_ptr, void* workspace) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SAGESLA_ERR_CUDA;
  if (!workspace) return SAGESLA_OK;
  int32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  if (word != 0) {
    const int32_t zero = 0;
    if (cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return SAGESLA_ERR_CUDA;
  }
  return static_cast<sagesla_status>(word);
}

sagesla_status sagesla_forward_host(const uint16_t* q_host, const uint16_t* k_host,
                                    const uint16_t* v_host, int64_t B, int64_t H, int64_t N,
                                    int64_t D, double topk_ratio, int block, void* out_host,
                                    int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                    void* stream_ptr) {
  if (!q_host || !k_host || !v_host || !out_host) return SAGESLA_ERR_INVALID_ARG;
  HostPlan hp;
  if (!host_plan(B, H, N, D, topk_ratio, block, out_dtype, &hp)) {
    if (D != kHeadDim || block != kBlock) return SAGESLA_ERR_UNSUPPORTED;
    return SAGESLA_ERR_INVALID_ARG;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      workspace_bytes < hp.total)
    return SAGESLA_ERR_WORKSPACE;
  sagesla_status st = check_device();
  if (st != SAGESLA_OK) return st;
  char* base = static_cast<char*>(workspace);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int64_t BH = B * H;
  const size_t head_elems = static_cast<size_t>(N * D);
  const size_t out_esz = elem_bytes(out_dtype);

  // Copy streams and the events that order the three stages (per call, so that concurrent
  // calls with their own workspaces stay independent).
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t in_ready[2] = {}, computed[2] = {}, out_free[2] = {};
  auto cleanup = [&]() {
    for (int s = 0; s < 2; ++s) {
      if (in_ready[s]) cudaEventDestroy(in_ready[s]);
      if (computed[s]) cudaEventDestroy(computed[s]);
      if (out_free[s]) cudaEventDestroy(out_free[s]);
    }
    if (h2d) cudaStreamDestroy(h2d);
    if (d2h) cudaStreamDestroy(d2h);
  };
  bool ok = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) == cudaSuccess;
  for (int s = 0; s < 2 && ok; ++s)
    ok = cudaEventCreateWithFlags(&in_ready[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&computed[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&out_free[s], cudaEventDisableTiming) == cudaSuccess;
  // the copies start after whatever the caller queued on `stream` before this call
  cudaEvent_t start = nullptr;
  if (ok) ok = cudaEventCreateWithFlags(&start, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventRecord(start, stream) == cudaSuccess &&
               cudaStreamWaitEvent(h2d, start, 0) == cudaSuccess;
  if (start) cudaEventDestroy(start);
  if (!ok) { cleanup(); return SAGESLA_ERR_CUDA; }

  for (int64_t c = 0; c < hp.nchunks && ok; ++c) {
    const int s = static_cast<int>(c & 1);
    const int64_t h0 = c * hp.hc, hn = (h0 + hp.hc <= BH) ? hp.hc : BH - h0;
    char* slot = base + hp.fw + s * hp.slot_bytes;
    char* dq = slot;
    char* dk = dq + hp.in_bytes;
    char* dv = dk + hp.in_bytes;
    char* dout = dv + hp.in_bytes;
    const size_t in_b = static_cast<size_t>(hn) * head_elems * 2;
    const size_t off = static_cast<size_t>(h0) * head_elems;
    // inputs of chunk c into slot s once the forward of chunk c - 2 has read that slot
    if (c >= 2) ok = cudaStreamWaitEvent(h2d, computed[s], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dq, q_host + off, in_b, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaMemcpyAsync(dk, k_host + off, in_b, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaMemcpyAsync(dv, v_host + off, in_b, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaEventRecord(in_ready[s], h2d) == cudaSuccess;
    // the forward of chunk c once its inputs are in and the output slot has been copied out
    ok = ok && cudaStreamWaitEvent(stream, in_ready[s], 0) == cudaSuccess;
    if (ok && c >= 2) ok = cudaStreamWaitEvent(stream, out_free[s], 0) == cudaSuccess;
    if (!ok) break;
    sagesla_tensor tq, tk, tv, to;
    for (sagesla_tensor* t : {&tq, &tk, &tv, &to}) {
      t->B = 1; t->H = hn; t->N = N; t->D = D;
      t->stride_n = D; t->stride_h = N * D; t->stride_b = hn * N * D;
    }
    tq.data = dq; tk.data = dk; tv.data = dv; to.data = dout;
    tq.dtype = tk.dtype = tv.dtype = SAGESLA_BF16;
    to.dtype = out_dtype;
    st = sagesla_forward(&tq, &tk, &tv, topk_ratio, block, &to, base, hp.fw, stream_ptr);
    if (st != SAGESLA_OK) { cleanup(); return st; }
    // keep this chunk's device status word (the next forward clears the workspace's)
    ok = cudaMemcpyAsync(base + hp.status_off + 4 * c, base, 4, cudaMemcpyDeviceToDevice, stream) ==
             cudaSuccess &&
         cudaEventRecord(computed[s], stream) == cudaSuccess &&
         cudaStreamWaitEvent(d2h, computed[s], 0) == cudaSuccess &&
         cudaMemcpyAsync(static_cast<char*>(out_host) + off * out_esz, dout,
                         static_cast<size_t>(hn) * head_elems * out_esz, cudaMemcpyDeviceToHost,
                         d2h) == cudaSuccess &&
         cudaEventRecord(out_free[s], d2h) == cudaSuccess;
  }
  // `stream` ends after the last output copy, as a single-stream call would
  for (int s = 0; s < 2 && ok; ++s) ok = cudaStreamWaitEvent(stream, out_free[s], 0) == cudaSuccess;
  const bool synced = cudaStreamSynchronize(stream) == cudaSuccess;
  cleanup();
  if (!ok || !synced) return SAGESLA_ERR_CUDA;
  // the first device-side error of any chunk
  int32_t words[kHostChunks] = {};
  if (cudaMemcpy(words, base + hp.status_off, static_cast<size_t>(hp.nchunks) * 4,
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  for (int64_t c = 0; c < hp.nchunks; ++c)
    if (words[c] != 0) return static_cast<sagesla_status>(words[c]);
  return SAGESLA_OK;
}

}  // extern "C"
