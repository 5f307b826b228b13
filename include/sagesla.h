/*
 * sagesla.h — C ABI of the B200 (sm_100a) SageSLA attention forward.
 *
 * SageSLA is the attention of the TurboDiffusion video diffusion transformer: sparse-linear
 * attention (SLA) combined with SageAttention-style low-bit quantization
 * (news.qq.com TurboDiffusion article, section 第一把钥匙; dgmzs.com.cn README translation,
 * section 方法论). Per (batch, head), with 64-token blocks:
 *   1. block scores s_ij = mean(Q_i) . mean(K_j) / sqrt(128); each query block keeps the
 *      k = clamp(ceil(r*nb - 1e-9), 1, nb) highest-scoring key blocks, ties to the lower j
 *      (same article, 第一把钥匙: Top-K ratio 0.1; 从训练到部署: 0.1-0.15);
 *   2. K is smoothed by its bf16-rounded channel mean; Q and smoothed K are quantized to
 *      INT8 with one scale per 64-token block, V to FP8 e4m3 with one scale per channel
 *      (same article, 第一把钥匙 and 第三把钥匙);
 *   3. sparse branch: online softmax over the kept blocks in ascending order, INT8 Q.K^T,
 *      P in e4m3 with scale 1/448, FP8 P.V;
 *   4. linear branch over the key blocks not kept: phi(q)(sum phi(k)^T [v|1]) normalized,
 *      phi = softmax over the 128 channels;
 *   5. out = sparse branch + linear branch.
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device addresses of the current device. The caller owns all
 *     buffers (inputs, output, workspace) and the stream; the library never allocates,
 *     frees or synchronizes except where stated.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream) unless stated; a return of SAGESLA_OK means the work was enqueued.
 *   - No exception crosses the ABI. Arguments are validated before anything is launched.
 *   - Errors detected on the device (a wait that timed out) are recorded in a status word in
 *     the workspace and read back by sagesla_stream_status().
 *   - Re-entrant across streams provided each concurrent call has its own workspace.
 */
#ifndef SAGESLA_H_
#define SAGESLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGESLA_OK = 0,
  SAGESLA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape/stride/ratio, aliasing output */
  SAGESLA_ERR_UNSUPPORTED = 2,  /* D != 128, block != 64, dtype not supported */
  SAGESLA_ERR_WORKSPACE = 3,    /* workspace missing, too small or misaligned */
  SAGESLA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  SAGESLA_ERR_TIMEOUT = 5,      /* a device-side wait exceeded its limit (see stream_status) */
  SAGESLA_ERR_DEVICE_CHECK = 6, /* a device-side consistency check failed */
  SAGESLA_ERR_NO_DEVICE = 7,    /* no sm_100 device is current */
  SAGESLA_ERR_BOUNDS = 8,       /* bounds-checking build: an index or TMA coordinate was out of
                                 * range; the access was skipped (see sagesla_build_checks) */
  SAGESLA_ERR_CANARY = 9        /* debug_checks: a workspace canary was overwritten */
} sagesla_status;

typedef enum { SAGESLA_BF16 = 0, SAGESLA_F32 = 1 } sagesla_dtype;

/* A [B, H, N, D] tensor view. Strides are in elements; the D axis is contiguous (stride 1).
 * Every row (b, h, n) must start on a 16-byte boundary. */
typedef struct {
  void* data;
  int32_t dtype; /* sagesla_dtype */
  int64_t B, H, N, D;
  int64_t stride_b, stride_h, stride_n;
} sagesla_tensor;

/* Optional extra outputs of sagesla_forward_ex (device pointers, may be NULL):
 *   kept_idx_out [B*H][nb][k] int32: kept key blocks of each query block, ascending;
 *   mask_out     [B*H][nb][ceil(nb/32)] uint32: bit j%32 of word j/32 set if j is kept;
 *   scores_out   [B*H][nb][nb] float: the block scores s_ij;
 *   sparse_out   [B*H][N][128] float: the sparse branch o*s_v/(448 l) before the linear
 *                branch is added. */
typedef struct {
  int32_t* kept_idx_out;
  uint32_t* mask_out;
  float* scores_out;
  float* sparse_out;   /* [B*H][N][128] float: the sparse-branch output alone */
  /* NULL, or SAGESLA_N_STAGES + 1 cudaEvent_t handles (created by the caller): event i is
   * recorded on the stream before stage i and the last one after the final stage, so that
   * the caller can time each kernel on the launching stream. Stages, in order: K/V statistics
   * and key-block states, statistics finalize, quantization, block scores, Top-K selection,
   * complement sums (skipped when every block is kept), sparse attention + linear branch. */
  void** stage_events;
  /* Test hooks of the failure path; leave both 0 in normal use.
   *   debug_spin_limit_us > 0 replaces the 2 s limit of every wait of the attention kernel by
   *   that many microseconds for this call.
   *   debug_skip_tile = 1 makes the attention kernel's first CTA skip one tile load (and the
   *   byte count announced for it), so that the waits for that tile run out: the call then
   *   ends normally with SAGESLA_ERR_TIMEOUT in the workspace's status word and that CTA's
   *   output rows unwritten. Nothing is left in flight, and the next call on the same
   *   workspace starts clean. */
  uint32_t debug_spin_limit_us;
  int32_t debug_skip_tile;
  /* Operand precision of the sparse branch (news.qq.com TurboDiffusion article, section
   * 从训练到部署: SLA without the low-bit quantization is the attention that is fine-tuned;
   * SageSLA, SLA plus SageAttention's 8-bit operands, replaces it at inference).
   *   quant = 1, pv_fp8 = 1: INT8 Q.K^T (smoothed K, per-block scales), e4m3 P and V (the
   *                          SageSLA forward);
   *   quant = 1, pv_fp8 = 0: INT8 Q.K^T, P rounded to bf16 times the raw bf16 V;
   *   quant = 0, pv_fp8 = 0: bf16 Q.K^T and bf16 P.V (the unquantized SLA forward, the one
   *                          sagesla_sla_backward differentiates).
   * quant = 0 with pv_fp8 = 1 is rejected (SAGESLA_ERR_UNSUPPORTED), other values
   * (SAGESLA_ERR_INVALID_ARG). sagesla_options_init sets both to 1; a zero-filled struct
   * selects the unquantized forward. The 16-bit modes need a larger workspace
   * (sagesla_workspace_size_ex with the same options) and run one CTA per SM. */
  int32_t quant;
  int32_t pv_fp8;
  /* debug_checks = 1: the call writes a 16-byte canary after every workspace region before
   * its first kernel and verifies them all after its last one, on the stream; a damaged
   * canary leaves SAGESLA_ERR_CANARY in the status word (read it with sagesla_stream_status).
   * Two extra kernels, nothing else changes.
   * debug_plant (failure-path tests, host-side fault injection; 0 in normal use):
   *   1 = after the canaries are written, overwrite one of them (needs debug_checks = 1): the
   *       call ends with SAGESLA_ERR_CANARY;
   *   2 = after the Top-K selection, overwrite the first kept-list entry with -1: the
   *       bounds-checking build (sagesla_build_checks() == 1) skips the access and ends with
   *       SAGESLA_ERR_BOUNDS; the normal build rejects this value (SAGESLA_ERR_UNSUPPORTED).
   * Other values: SAGESLA_ERR_INVALID_ARG. */
  int32_t debug_checks;
  int32_t debug_plant;
} sagesla_options;

/* Fills *opt with the defaults: every pointer NULL, test hooks 0, quant = pv_fp8 = 1. */
void sagesla_options_init(sagesla_options* opt);

/* 1 for the bounds-checking build of this library (compiled with SAGESLA_CHECKS=1:
 * libsagesla_checks.so), 0 for the normal build. In the checking build every kept-list entry
 * a kernel reads, every Top-K output position and every TMA row coordinate of the attention
 * kernels is checked before use; a failed check records SAGESLA_ERR_BOUNDS in the status
 * word, the access is skipped, and the CTA stops (no trap, no assert: the context stays
 * usable). */
int sagesla_build_checks(void);

#define SAGESLA_N_STAGES 7

/* Offsets (bytes, from the workspace start) of the intermediates a forward call leaves in
 * its workspace, for inspection after the stream has completed. Per-head arrays are
 * contiguous over B*H; n_pad = 128*ceil(nb/2) token rows per head. Regions start on 256-byte
 * boundaries, and at least 16 bytes separate the end of each region from the next one: the
 * 16 bytes at the end rounded up to 16 hold the region's canary when debug_checks is set. */
typedef struct {
  size_t total_bytes;
  int64_t nb, k, n_pad, mask_words, nb_k_pad, nb_m_pad;
  size_t status;      /* int32 status word */
  size_t q8, k8;      /* int8  [B*H][n_pad][128] codes (zero rows past N) */
  size_t v8;          /* uint8 [B*H][n_pad][128] e4m3 codes */
  size_t sq, sk;      /* float [B*H][2*ceil(nb/2)] per-block scales */
  size_t s_v;         /* float [B*H][128] per-channel V scale */
  size_t inv_v;       /* float [B*H][128] 448 / channel amax */
  size_t mu;          /* float [B*H][128] bf16 channel mean of K, stored as float */
  size_t qbar, kbar;  /* float [B*H][nb][128] block means */
  size_t ksum_part;   /* double [B*H][nb][128] per-block K channel sums */
  size_t vmax_part;   /* float [B*H][nb][128] per-block V channel amax */
  size_t scores;      /* float [B*H][nb][ld] raw block dot products, ld = nb rounded up to 4 */
  size_t kept;        /* int32 [B*H][nb][k] */
  size_t mask;        /* uint32 [B*H][nb][mask_words] */
  size_t amask;       /* bf16 [B*H][nb_m_pad][nb_k_pad] complement mask (1 = not kept) */
  size_t hflat;       /* bf16 [B*H][nb_k_pad][129*128] key-block states H_j as [n][c] */
  size_t gsum;        /* bf16 [B*H][nb_m_pad][129*128] complement sums G_i as [n][c] */
  size_t qb, kb;      /* bf16 [B*H][n_pad][128] copies of Q and K (K rows key-interleaved
                       * within each 64-key block) for quant = 0; 0 when absent */
  size_t vb;          /* bf16 [B*H][n_pad][128] copy of V for pv_fp8 = 0; 0 when absent */
} sagesla_workspace_layout;

/* Human-readable name of a status code (static string). */
const char* sagesla_status_string(sagesla_status status);

/* k, the number of key blocks each query block keeps, for N tokens and ratio r (block 64):
 * clamp(ceil(r*ceil(N/64) - 1e-9), 1, ceil(N/64)); -1 for invalid arguments. */
int64_t sagesla_topk_count(int64_t N, double topk_ratio, int block);

/* Bytes of device workspace sagesla_forward needs; 0 for invalid arguments. */
size_t sagesla_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, double topk_ratio,
                              int block);

/* Fills *layout for the given problem. Returns SAGESLA_ERR_INVALID_ARG / SAGESLA_ERR_UNSUPPORTED on bad
 * arguments. Host only, no CUDA call. */
sagesla_status sagesla_get_workspace_layout(int64_t B, int64_t H, int64_t N, int64_t D,
                                            double topk_ratio, int block,
                                            sagesla_workspace_layout* layout);

/* As sagesla_workspace_size / sagesla_get_workspace_layout for the operand mode of *opt
 * (quant, pv_fp8; opt NULL = the defaults): the 16-bit modes add bf16 copies of their
 * operands. Errors as sagesla_forward_ex's mode checks; 0 bytes for invalid arguments. */
size_t sagesla_workspace_size_ex(int64_t B, int64_t H, int64_t N, int64_t D, double topk_ratio,
                                 int block, const sagesla_options* opt);
sagesla_status sagesla_get_workspace_layout_ex(int64_t B, int64_t H, int64_t N, int64_t D,
                                               double topk_ratio, int block,
                                               const sagesla_options* opt,
                                               sagesla_workspace_layout* layout);

/* The SageSLA forward: out = sparse(Q,K,V) + linear(Q,K,V) as defined above.
 *   q, k, v   : bf16 [B,H,N,128] device tensors (read only)
 *   topk_ratio: r in (0, 1]
 *   block     : must be 64
 *   out       : bf16 or f32 [B,H,N,128] device tensor, must not overlap q, k, v or workspace
 *   workspace : device buffer of at least sagesla_workspace_size() bytes, 256-byte aligned;
 *               its contents on entry are ignored; it holds the intermediates on exit
 *   stream    : cudaStream_t as void*
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA, NO_DEVICE (nothing launched). */
sagesla_status sagesla_forward(const sagesla_tensor* q, const sagesla_tensor* k,
                               const sagesla_tensor* v, double topk_ratio, int block,
                               sagesla_tensor* out, void* workspace, size_t workspace_bytes,
                               void* stream);

/* As sagesla_forward, plus the optional outputs and the operand mode of *opt (opt may be
 * NULL: no extra outputs, quant = pv_fp8 = 1). The workspace must hold
 * sagesla_workspace_size_ex(..., opt) bytes. */
sagesla_status sagesla_forward_ex(const sagesla_tensor* q, const sagesla_tensor* k,
                                  const sagesla_tensor* v, double topk_ratio, int block,
                                  sagesla_tensor* out, void* workspace, size_t workspace_bytes,
                                  void* stream, const sagesla_options* opt);

/* Bytes of device workspace sagesla_forward_host needs: the forward workspace for a chunk
 * of ceil(B*H / min(B*H, 16)) heads, two slots of that chunk's Q, K, V and output, and one
 * status word per chunk; 0 for invalid arguments. */
size_t sagesla_host_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                   double topk_ratio, int block, int32_t out_dtype);

/* Forward on HOST buffers: contiguous [B,H,N,128] bf16 inputs (uint16 bit patterns) and a
 * contiguous bf16/f32 output in host memory (page-locked memory gives asynchronous copies).
 * Works through the heads in up to 16 chunks: the host->device copy of one chunk (its own
 * stream), the forward of the previous chunk (on `stream`) and the device->host copy of the
 * one before (its own stream) overlap. The copies start after the work already queued on
 * `stream`; the call synchronizes `stream` before returning and also returns device-side
 * errors (TIMEOUT) of any chunk. */
sagesla_status sagesla_forward_host(const uint16_t* q_host, const uint16_t* k_host,
                                    const uint16_t* v_host, int64_t B, int64_t H, int64_t N,
                                    int64_t D, double topk_ratio, int block, void* out_host,
                                    int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Size of the fixed scratch area used by sagesla_forward_no_alloc (64 MiB). */
#define SAGESLA_NO_ALLOC_SCRATCH_BYTES (64ull << 20)

/* Forward for callers that cannot allocate device memory (for example a host integration
 * that only hands over input and output buffers, code inside a memory pool that may not
 * grow, or a process that must not call cudaMalloc once loaded). The paper has no counterpart
 * of this call: it exists for such integrations.
 *   - Same arguments and result as sagesla_forward, without the workspace: the forward's
 *     scratch lives in a device array of SAGESLA_NO_ALLOC_SCRATCH_BYTES that is part of this
 *     library; every GPU that loads the library holds it until the process exits.
 *   - Problems whose sagesla_workspace_size() exceeds SAGESLA_NO_ALLOC_SCRATCH_BYTES are
 *     rejected with SAGESLA_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture. The address
 *     is kept until the process exits: after a cudaDeviceReset of that device it is stale, so
 *     do not use this call on a device after resetting it.
 *   - Every call shares the one array, which keeps the last call's contents; calls whose GPU
 *     work overlaps (different streams, or threads without ordering) race on it.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - Asynchronous on `stream`; device-side timeouts are not reported back (there is no
 *     workspace to pass to sagesla_stream_status). */
sagesla_status sagesla_forward_no_alloc(const sagesla_tensor* q, const sagesla_tensor* k,
                                        const sagesla_tensor* v, double topk_ratio, int block,
                                        sagesla_tensor* out, void* stream);

/* ---------------------------------------------------------------------------------------
 * Fused normalization, modulation and INT8 activation quantization: the LayerNorm / RMSNorm
 * of a DiT block feeding an 8-bit linear layer. News.qq.com TurboDiffusion article, section
 * 第四把钥匙 (LayerNorm and RMSNorm rewritten and fused with neighbouring operations so that
 * data crosses memory fewer times) and section 第三把钥匙 (activations quantized to INT8 on
 * the fly). Per token row x (bf16, K channels):
 *   LayerNorm: y = (x - mean) / sqrt(var + eps), then y * gamma + beta   (biased variance)
 *   RMSNorm:   y = x / sqrt(mean(x^2) + eps), then y * gamma
 *   none:      y = x (the per-token INT8 quantizer of any activation row)
 *   modulation, if given: y = y * (1 + scale[b]) + shift[b], b = row / rows_per_sample
 *   y_out = bf16(y) (round to nearest even)
 *   INT8, if asked: a = max |y_out| over the row; code = clamp(rne(y_out * fl32(127 / a)),
 *   -127, 127) and code_scale = fl32(a / 127); a = 0 gives scale 1 and zero codes.
 * The arithmetic is fp32 (fp32 sums over the row), so y_out can differ by one bf16 ulp from
 * the real-number y rounded to bf16; the codes are exact functions of y_out. */
typedef enum { SAGESLA_LAYER_NORM = 0, SAGESLA_RMS_NORM = 1, SAGESLA_NO_NORM = 2 } sagesla_norm_kind;

typedef struct {
  const uint16_t* x;       /* bf16 [M][K] device (read only), row stride x_stride elements */
  int64_t M, K, x_stride;
  int32_t kind;            /* sagesla_norm_kind */
  float eps;               /* >= 0, finite */
  const uint16_t* gamma;   /* bf16 [K] or NULL (1); not with SAGESLA_NO_NORM */
  const uint16_t* beta;    /* bf16 [K] or NULL (0); LayerNorm only */
  const uint16_t* scale;   /* bf16 [ceil(M / rows_per_sample)][K] or NULL (0) */
  const uint16_t* shift;   /* same shape as scale, or NULL (0) */
  int64_t rows_per_sample; /* >= 1 when scale or shift is given */
  uint16_t* y;             /* bf16 [M][K] out, row stride y_stride elements, or NULL */
  int64_t y_stride;
  int8_t* codes;           /* int8 [M][K] out, row stride codes_stride bytes, or NULL */
  int64_t codes_stride;
  float* code_scale;       /* float [M] out, given exactly when codes is given */
} sagesla_norm_args;

/* Runs the fused normalization asynchronously on `stream` (cudaStream_t as void*); all
 * pointers are device pointers owned by the caller. Requirements: M >= 1; 8 <= K <= 16384
 * and K a multiple of 8; x and y rows 16-byte aligned (strides multiples of 8 elements, at
 * least K), codes rows 8-byte aligned (stride a multiple of 8, at least K); gamma, beta,
 * scale, shift 16-byte aligned; at least one of y and codes; the outputs must not overlap x.
 * Errors: INVALID_ARG (bad pointers, strides, kind, eps), UNSUPPORTED (K out of range),
 * CUDA, NO_DEVICE (nothing launched in every case). */
sagesla_status sagesla_norm_quant(const sagesla_norm_args* args, void* stream);

/* ---------------------------------------------------------------------------------------
 * W8A8 linear layer: INT8 weights in 128x128 blocks with one scale per block, INT8
 * activations with one scale per token row, the GEMM on the INT8 tensor cores.
 * News.qq.com TurboDiffusion article, section 第三把钥匙 (weights and activations both in
 * 8-bit integers so that the whole linear layer runs in the integer domain; block-wise weight
 * quantization with 128x128 blocks; activations quantized on the fly). The activation codes
 * come from sagesla_norm_quant (any kind, including SAGESLA_NO_NORM). */

/* Offline weight quantization. w: bf16 [N][K] device, row stride w_stride elements (a
 * multiple of 8, at least K, 16-byte aligned base); K a multiple of 128 (<= 2^20), N >= 1.
 * For each block of rows 128*bn.. (the last block may hold fewer rows) and columns
 * 128*bk..128*bk+127: a = max |w|; a = 0 gives scale 1 and zero codes, else code =
 * clamp(rne(w * fl32(127 / a)), -127, 127), w_scale[bn][bk] = fl32(a / 127).
 * Outputs: w8 int8 [N][K] (contiguous, 16-byte aligned), w_scale float [ceil(N/128)][K/128].
 * Asynchronous on `stream`. Errors: INVALID_ARG, UNSUPPORTED (K not a multiple of 128),
 * CUDA, NO_DEVICE (nothing launched). */
sagesla_status sagesla_w8a8_quantize_weight(const uint16_t* w, int64_t N, int64_t K,
                                            int64_t w_stride, int8_t* w8, float* w_scale,
                                            void* stream);

/* y[m][n] = x_scale[m] * sum_bk w_scale[n/128][bk] * sum_{k in block bk} x8[m][k] w8[n][k]
 *           (+ bias[n]), summed over the K blocks in fp32 from exact int32 block products.
 *   x8      int8 [M][K] contiguous, x_scale float [M] (per token row)
 *   w8      int8 [N][K] contiguous, w_scale float [ceil(N/128)][K/128]
 *   bias    bf16 [N] or NULL
 *   y       bf16 (y_dtype SAGESLA_BF16, round to nearest even) or float (SAGESLA_F32)
 *           [M][N], row stride y_stride elements (16-byte aligned rows)
 *   status  device int32 or NULL: a device-side timeout of the kernel's bounded waits writes
 *           SAGESLA_ERR_TIMEOUT there (the caller zeroes it)
 * Requirements: M, N >= 1 (< 2^31); K a multiple of 128; N a multiple of 8; all buffers
 * 16-byte aligned; y must not overlap the inputs. Asynchronous on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA, NO_DEVICE (nothing launched). */
sagesla_status sagesla_w8a8_gemm(const int8_t* x8, const float* x_scale, int64_t M, int64_t K,
                                 const int8_t* w8, const float* w_scale, int64_t N,
                                 const uint16_t* bias, void* y, int32_t y_dtype,
                                 int64_t y_stride, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * SLA backward: gradients of the unquantized sparse-linear attention for fine-tuning.
 * News.qq.com TurboDiffusion article, section 从训练到部署 (full attention is replaced by SLA
 * and fine-tuned; SageSLA, SLA plus low-bit quantization, replaces it only at inference).
 * Forward differentiated: O = O_s + O_l with O_s the exact softmax attention of each query
 * block over the tokens of its kept key blocks (scale 1/sqrt(128), padded keys excluded) and
 * O_l the normalized linear attention phi(q) G_i[:, :128] / phi(q) G_i[:, 128] over the key
 * blocks it does not keep (G_i = sum of H_j = phi(K_j)^T [V_j | 1], phi = softmax over the
 * 128 channels). The block selection is the forward's (same pooled scores and Top-K ratio)
 * and is held fixed: the gradients are those of O with the mask constant. */

/* Bytes of device workspace sagesla_sla_backward needs (the forward's layout of
 * sagesla_get_workspace_layout, followed by the backward's own regions); 0 for invalid
 * arguments. */
size_t sagesla_sla_backward_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                           double topk_ratio, int block);

/* dq, dk, dv = gradients of sum(O * d_out) with respect to q, k, v.
 *   q, k, v, d_out  bf16 views [B, H, N, 128] (the requirements of sagesla_forward)
 *   dq, dk, dv      bf16 or f32 views of the same shape, one dtype for all three; written
 *                   in full (f32 results of fp32 accumulation, rounded to nearest even for
 *                   bf16); they must not overlap the inputs, each other or the workspace
 *   workspace       device, 256-byte aligned, sagesla_sla_backward_workspace_size bytes; it
 *                   holds the forward's selection (kept lists, mask) at the forward layout's
 *                   offsets afterwards
 * Asynchronous on `stream`; device-side timeouts land in the workspace's status word
 * (sagesla_stream_status). Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA, NO_DEVICE
 * (nothing launched on any error found before the launches). */
sagesla_status sagesla_sla_backward(const sagesla_tensor* q, const sagesla_tensor* k,
                                    const sagesla_tensor* v, const sagesla_tensor* d_out,
                                    double topk_ratio, int block, sagesla_tensor* dq,
                                    sagesla_tensor* dk, sagesla_tensor* dv, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Synchronizes `stream`, then reads and clears the device status word of `workspace`
 * (the one used by the last forward on that workspace). Returns SAGESLA_OK, TIMEOUT,
 * DEVICE_CHECK, or CUDA if the stream reported an error. */
sagesla_status sagesla_stream_status(void* stream, void* workspace);

#ifdef __cplusplus
}
#endif

#endif /* SAGESLA_H_ */
