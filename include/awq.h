/*
 * awq.h - C ABI of the B200 (sm_100a) AWQ activation-aware scale search and INT4 group quantizer.
 *
 * What the library computes (sources are five web pages about AWQ, cited by title and section):
 *
 *   (1) act_mean[k] = mean_i |X[i,k]|            "显著权重的识别" on the bjdmk.com.cn AWQ article
 *                                                 (S_X(i) = 1/N sum_j |X_ji|); 原理 on the msModelSlim page
 *                                                 "AWQ：激活感知权重量化算法说明" (act_mean = mean(abs(act))).
 *   (2) for ratio_j = j / n_grid, j = 0..n_grid-1 (the grid [0, 1) with step 1/n_grid, 原理 on the
 *       msModelSlim page): s = clamp(act_mean^ratio, min 1e-4); s = s / sqrt(max(s) * min(s)).
 *   (3) W' = W diag(s); asymmetric 4-bit quantization of W' in groups of 128 consecutive in-features:
 *       step = clamp((max - min) / 15, min 1e-5), z = round(-min / step),
 *       q = clamp(round(w' / step) + z, 0, 15), deq = (q - z) * step, w_hat = deq / s
 *       (section 二 of "AWQ 离群激活平滑实操逐通道等价缩放与 4-bit 精度无损转换", gsyq.cn; that page clamps the
 *       step at 1e-8, this library at 1e-5).
 *   (4) loss_j = mean over the N*O outputs of (X W^T - X W_hat_j^T)^2 (the loss L(s) in
 *       "数学等价变换与通道自适应缩放" on the bjdmk.com.cn article; the MSE step of 缩放因子搜索流程 on the
 *       msModelSlim page); the best ratio is the first j reaching the minimum (strict '<' update in the
 *       search loops of both pages).
 *   (5) the INT4 codes of W at the best scales, 8 codes per uint32, plus per-group steps and zeros
 *       (two codes per byte in "GPU 硬件级反量化算子内联融合" on the bjdmk.com.cn article; this library
 *       packs code of in-feature k into word k/8, bits 4*(k%8) .. 4*(k%8)+3).
 *
 * Several linears that read the same input (q/k/v after one norm; NormLinearSubgraph on the msModelSlim
 * page) share one scale vector: pass their weights stacked row-wise as one [O_total, K] matrix.
 *
 * Conventions for every entry point
 *   - Matrices are row-major bfloat16 bit patterns: X is [N, K] (tokens x in-features) with row stride
 *     ldx elements, W is [O, K] (out-features x in-features, torch nn.Linear layout) with row stride ldw.
 *   - Every pointer except those documented as host pointers is a DEVICE pointer of the current CUDA
 *     device. The caller owns all memory; the library never allocates device or host memory.
 *   - Every call is asynchronous on `stream` (NULL selects the legacy default stream) and returns after
 *     validation and enqueueing. A non-OK status means nothing was enqueued, except AWQ_ERR_CUDA from a
 *     failed launch. awq_last_error() then returns a message (thread-local, valid until the next call).
 *   - Pointers must be 16-byte aligned and ldx, ldw multiples of 8 (rows start on 16-byte boundaries).
 *   - group must be 128 (AWQ_ERR_UNSUPPORTED otherwise); K must be a multiple of 128.
 *   - Inputs must be finite; NaN or Inf give unspecified (but memory-safe) results.
 *   - Calls that share a workspace must not overlap on the GPU (serialise them on one stream).
 *   - Device waits inside the kernels are bounded (default 2 s, see awq_set_wait_limit_ns); a wait that
 *     gives up records AWQ_ERR_TIMEOUT in the workspace, makes the remaining kernels of the call skip
 *     their work, and sets *best_j = -1; awq_search_status() reports it.
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

typedef struct CUstream_st *awq_stream_t; /* identical to cudaStream_t */

typedef enum awq_status {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment, n_grid out of range */
  AWQ_ERR_UNSUPPORTED = 2, /* group not 128 (0 with AWQ_FLAG_QUANT_INT8), or a device other than sm_100 */
  AWQ_ERR_WORKSPACE = 3,   /* workspace null or smaller than the *_workspace_size() query */
  AWQ_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed; message from the runtime */
  AWQ_ERR_TIMEOUT = 5      /* a bounded device wait gave up (reported by awq_search_status) */
} awq_status;

/* Flags for the *_ex entry points (0 = the production behaviour of the plain entry points). */
#define AWQ_FLAG_EXACT_DIVISION 0x1u /* every w'/step quotient by IEEE division, no reciprocal fast path;
                                        in the search also the unscale w_hat = RN32(deq / s) */
#define AWQ_FLAG_EXACT_POW 0x2u      /* every act_mean^ratio by the double-double path, no fp64 pow */
#define AWQ_FLAG_INJECT_STALL 0x100u /* test hook: the loss GEMM waits on a barrier nobody signals */
/* Candidate-scale rule of the search (default: 原理 on the msModelSlim page, see (2) below). */
#define AWQ_FLAG_SCALES_WEIGHT_AWARE 0x10u /* AWQChannelScaler on the bjdmk.com.cn article: see (2) */
#define AWQ_FLAG_SCALES_RMS 0x20u          /* search_smooth_scaling_factors, gsyq.cn section 二: see (2) */
/* Weight quantizer of the search (default: asymmetric INT4 in groups of 128, see (3)). */
#define AWQ_FLAG_QUANT_INT8 0x40u /* symmetric INT8, one step per output channel: see (5b); group must be 0 */

#define AWQ_MAX_N_GRID 64

/* Message of the last failing call on this thread ("" if none). */
AWQ_API const char *awq_last_error(void);

/* Library ABI version (major * 100 + minor). */
AWQ_API int awq_version(void);

/* Upper bound, in nanoseconds, of every device-side wait (mbarrier waits of the loss GEMM). Default
 * 2e9. Applies to calls enqueued after it. Values below 1e6 are raised to 1e6. */
AWQ_API void awq_set_wait_limit_ns(uint64_t ns);

/* ---------------------------------------------------------------------------------------------------
 * (1) Activation statistic.  act_mean[k] = RN32(RN64(S_k / N)) with S_k = sum_i |X[i,k]| accumulated
 * in fp64 in a fixed order: rows in consecutive chunks of 256, inside a chunk one row at a time in
 * increasing order, then the chunk totals in chunk order. Deterministic and bit-reproducible.
 *   X         device, bf16 [N, K], row stride ldx (elements)
 *   workspace device, >= awq_act_stats_workspace_size(N, K) bytes, contents need not be initialised
 *   act_mean  device, float [K] (output)
 * Requires N >= 1, K >= 1, K % 2 == 0 and ceil(N / 256) <= 65535 (N <= 16,776,960), else
 * AWQ_ERR_INVALID_ARG before any launch.
 * ------------------------------------------------------------------------------------------------- */
AWQ_API size_t awq_act_stats_workspace_size(int64_t N, int64_t K);
AWQ_API awq_status awq_act_stats(const void *X, int64_t N, int64_t K, int64_t ldx, void *workspace,
                         size_t ws_bytes, float *act_mean, awq_stream_t stream);

/* ---------------------------------------------------------------------------------------------------
 * Activation statistic that allocates nothing. The pages have no counterpart: this is a deployment
 * convenience. Some callers cannot call cudaMalloc when they invoke the statistic: a plugin running
 * inside an inference engine that owns all device memory and forbids allocation on its execution path,
 * or a process that reserved nearly all HBM up front (KV caches, weight pools) where cudaMalloc would
 * fail or implicitly synchronise the device. For them this variant takes no workspace: its fp64 chunk
 * sums live in a fixed 16 MiB device array inside the library (AWQ_NOALLOC_SCRATCH_DOUBLES doubles),
 * which every GPU that loads the library holds until the process exits.
 *   Same inputs, output and result as awq_act_stats (bit-identical act_mean).
 *   Limit: ceil(N / 256) * K <= AWQ_NOALLOC_SCRATCH_DOUBLES, else AWQ_ERR_INVALID_ARG and no launch
 *   (e.g. N = 16384 with K <= 32768, or N = 4096 with K <= 131072).
 *   The first call on each device looks up the array's device address (cudaGetSymbolAddress, which may
 *   load the library's device code on that device); make that first call before any stream capture.
 *   The address is kept per device and CUDA context: after cudaDeviceReset (a new primary context, in
 *   which the library's device code and the array are loaded afresh) the next call looks it up again,
 *   so that call too belongs before any capture.
 *   All calls share the one array, which keeps the last call's contents (every value a call reads is
 *   first written by that call, so nothing needs clearing): calls that overlap on the GPU, e.g. on two
 *   streams, race and give wrong results. Serialise them.
 * ------------------------------------------------------------------------------------------------- */
#define AWQ_NOALLOC_SCRATCH_DOUBLES (1ull << 21)
AWQ_API awq_status awq_act_stats_noalloc(const void *X, int64_t N, int64_t K, int64_t ldx, float *act_mean,
                                         awq_stream_t stream);

/* ---------------------------------------------------------------------------------------------------
 * (2) Scale table alone (the first stage of awq_search, exposed for testing and for callers that want
 * the candidates). Row j of table (device, float [n_grid, K]) receives, with r = RN32(j / n_grid):
 *   t = correctly rounded fp32 of act_mean[k]^r (0^0 = 1), t = max(t, RN32(1e-4)),
 *   d = RN32(sqrt(RN32(max_k t * min_k t))), s = RN32(t / d).
 * flags: 0 or AWQ_FLAG_EXACT_POW, optionally with one of the alternative rules (also accepted by
 * awq_search_ex), all bit-exact, P_j = RN32(j / (n_grid - 1)) (linspace(0, 1, n_grid), 1.0 included):
 *   AWQ_FLAG_SCALES_WEIGHT_AWARE: t = max(RN32(CR32(a^P) / RN32(CR32(wm^RN32(1 - P)) + RN32(1e-6))), 1e-4),
 *     then the same geometric normalisation; wm[k] = mean_o |W[o,k]| (fixed order as in (1)); only through
 *     awq_scale_table_ex (which takes wm) or awq_search_ex.
 *   AWQ_FLAG_SCALES_RMS: t = CR32(max(a, RN32(1e-5))^P); m = RN32(RN64(S / K)), S = fp64 sum of RN32(t^2)
 *     in 256-column chunks (in order, chunk totals in order); s = max(RN32(t / RN32(sqrt(m))), 1e-4)
 *     (n_grid = 11 gives the page's 0, 0.1, ..., 1.0).
 * 1 <= n_grid <= AWQ_MAX_N_GRID.
 * ------------------------------------------------------------------------------------------------- */
AWQ_API size_t awq_scale_table_workspace_size(int64_t K, int n_grid);
AWQ_API awq_status awq_scale_table(const float *act_mean, int64_t K, int n_grid, unsigned flags, void *workspace,
                           size_t ws_bytes, float *table, awq_stream_t stream);
AWQ_API awq_status awq_scale_table_ex(const float *act_mean, const float *weight_mean, int64_t K, int n_grid,
                                      unsigned flags, void *workspace, size_t ws_bytes, float *table,
                                      awq_stream_t stream);

/* ---------------------------------------------------------------------------------------------------
 * (2)-(4) The search. For every candidate j it forms the weight error dW_j = W - W_hat_j (fp32, rounded
 * to bf16) and evaluates loss_j = sum((X dW_j^T)^2) / (N * O) with tensor cores (bf16 x bf16, fp32
 * accumulation in tensor memory, squares reduced in fp32 per row and fp64 across rows and tiles in a
 * fixed order); the [N, O] product is never written to memory.
 *   X, W       device bf16 as above; W holds the stacked rows of every linear that reads X
 *   act_mean   device float [K] (from awq_act_stats or the caller)
 *   workspace  device, >= awq_search_workspace_size(N, K, O, group, n_grid) bytes, 1024-byte aligned
 *   losses     device double [n_grid] (output)
 *   best_j     device int (output): first index of the minimum loss; -1 after a device timeout
 *   scales     device float [K] (output): row best_j of the scale table
 * The scales, and the codes/steps/zeros that awq_quantize_pack derives from them, are bit-exact
 * functions of (act_mean, W); the losses carry bf16 rounding of dW and fp32 tensor-core accumulation.
 * Requires N >= 1, O >= 1, K >= 128, K % 128 == 0, N, O, K < 2^31, 1 <= n_grid <= AWQ_MAX_N_GRID.
 * group: 128 (INT4 groups of 128 in-features), or 0 (per output channel) together with
 * AWQ_FLAG_QUANT_INT8; the workspace size is the same for both.
 * ------------------------------------------------------------------------------------------------- */
AWQ_API size_t awq_search_workspace_size(int64_t N, int64_t K, int64_t O, int group, int n_grid);
AWQ_API awq_status awq_search(const void *X, int64_t N, int64_t K, int64_t ldx, const void *W, int64_t O,
                      int64_t ldw, const float *act_mean, int group, int n_grid, void *workspace,
                      size_t ws_bytes, double *losses, int *best_j, float *scales, awq_stream_t stream);
/* Same, with flags (AWQ_FLAG_EXACT_DIVISION, AWQ_FLAG_EXACT_POW, AWQ_FLAG_INJECT_STALL, one of
 * AWQ_FLAG_SCALES_WEIGHT_AWARE / AWQ_FLAG_SCALES_RMS to search the alternative candidate scales, and
 * AWQ_FLAG_QUANT_INT8 with group 0 to search with the INT8 per-channel quantizer of (5b)). */
AWQ_API awq_status awq_search_ex(const void *X, int64_t N, int64_t K, int64_t ldx, const void *W, int64_t O,
                         int64_t ldw, const float *act_mean, int group, int n_grid, unsigned flags,
                         void *workspace, size_t ws_bytes, double *losses, int *best_j, float *scales,
                         awq_stream_t stream);

/* Synchronises `stream`, then reads the device status word of a workspace last used by awq_search:
 * AWQ_OK or AWQ_ERR_TIMEOUT (message names the wait that gave up). */
AWQ_API awq_status awq_search_status(const void *workspace, size_t ws_bytes, awq_stream_t stream);

/* Where awq_search leaves its per-tile partial sums inside the workspace (valid after the call):
 * double partial[n_grid][tiles_o][tiles_n][partials_per_tile] at byte offset partials_offset;
 * partial[j][a][b][e] is the sum of squares of the outputs of token rows
 * [b*tile_n + e*r, b*tile_n + (e+1)*r), r = tile_n / partials_per_tile, and output rows
 * [a*tile_o, (a+1)*tile_o) for candidate j (rows past N or O contribute zero). */
typedef struct awq_search_layout {
  int64_t tile_n, tile_o;   /* tile extent along tokens and along output rows */
  int64_t tiles_n, tiles_o; /* tiles per candidate along tokens and along output rows */
  int64_t partials_per_tile;
  size_t partials_offset;   /* bytes from the workspace start */
  size_t workspace_bytes;   /* same as awq_search_workspace_size() */
} awq_search_layout;
AWQ_API awq_status awq_search_get_layout(int64_t N, int64_t K, int64_t O, int group, int n_grid,
                                 awq_search_layout *out /* host */);

/* Measurement hook: when set (non-NULL), every later awq_search* call on this thread records the CUDA
 * event `before` on its stream right before the loss-GEMM launch and `after` right after it, so a caller
 * can time that kernel alone. Both are cudaEvent_t handles created by the caller; pass NULL, NULL to
 * stop. */
AWQ_API void awq_set_profile_events(void *before_loss_gemm, void *after_loss_gemm);

/* ---------------------------------------------------------------------------------------------------
 * (5) Codes of W at given scales (normally the `scales` output of awq_search):
 *   codes  device uint32 [O, K/8]: code of in-feature k at bits 4*(k%8) of word k/8
 *   steps  device float [O, K/group]: per-group step
 *   zeros  device float [O, K/group]: per-group zero point (integer-valued, not clamped, never -0)
 * Bit-exact: every operation is one IEEE fp32 operation in the order given in (3).
 * ------------------------------------------------------------------------------------------------- */
AWQ_API awq_status awq_quantize_pack(const void *W, int64_t O, int64_t K, int64_t ldw, const float *scales,
                             int group, uint32_t *codes, float *steps, float *zeros, awq_stream_t stream);
/* Same, with flags (AWQ_FLAG_EXACT_DIVISION). */
AWQ_API awq_status awq_quantize_pack_ex(const void *W, int64_t O, int64_t K, int64_t ldw, const float *scales,
                                int group, unsigned flags, uint32_t *codes, float *steps, float *zeros,
                                awq_stream_t stream);

/* ---------------------------------------------------------------------------------------------------
 * (5b) Symmetric INT8 codes of W at given scales, one step per output channel (formula of section 2.1
 * of the hncyxsy.com large-model outlier article, with the per-channel weight setting of the
 * quantization YAML on the msModelSlim page). With w' = RN32(w * s_k) over the row's K in-features:
 *   step_o = max(RN32(max_k |w'| / 127), RN32(1e-5))    q = min(max(rint(RN32(w' / step_o)), -127), 127)
 * and the dequantized value is RN32(q * step_o). The search with AWQ_FLAG_QUANT_INT8 scores exactly this
 * quantizer (w_hat = RN32(q * step_o) * RN32(1 / s_k), as for INT4).
 *   W      device bf16 [O, ldw] as in awq_search
 *   scales device float [K], 16-byte aligned
 *   codes  device int8 [O, K] row-major (row stride K), 8-byte aligned (output)
 *   steps  device float [O] (output)
 *   flags  0 or AWQ_FLAG_EXACT_DIVISION
 * Bit-exact: every operation is one IEEE fp32 operation in the order above. Requires K % 8 == 0.
 * ------------------------------------------------------------------------------------------------- */
AWQ_API awq_status awq_quantize_pack_int8(const void *W, int64_t O, int64_t K, int64_t ldw, const float *scales,
                                          unsigned flags, int8_t *codes, float *steps, awq_stream_t stream);

/* ---------------------------------------------------------------------------------------------------
 * Applying the chosen scales (SubgraphFusionFactory step of 缩放因子搜索流程 on the msModelSlim page):
 * the target linears get forward scaling of their input columns, W' = W diag(s); the producer of their
 * input gets the inverse: the norm weight gamma' = gamma / s (NormLinearSubgraph), or the output rows
 * (and bias) of the source linear divided by s (LinearLinearSubgraph linear1, OVSubgraph v_proj for
 * multi-head attention, UpDownSubgraph up_proj), so that section 一's identity
 * X W^T = (X diag(s)^-1)(diag(s) W)^T keeps the subgraph's output.
 *   awq_scale_columns: out[r, c] = bf16(RN32(A[r, c] op s[c]))
 *   awq_scale_rows:    out[r, c] = bf16(RN32(A[r, c] op s[r]))
 * op = AWQ_SCALE_MULTIPLY or AWQ_SCALE_DIVIDE (IEEE fp32 division); A, out bf16 row-major with row
 * strides lda, ldo (multiples of 8); C % 8 == 0; out may equal A (in place). A norm weight or a bias is
 * a 1 x C matrix. Bit-exact.
 * ------------------------------------------------------------------------------------------------- */
#define AWQ_SCALE_MULTIPLY 0
#define AWQ_SCALE_DIVIDE 1
AWQ_API awq_status awq_scale_columns(const void *A, int64_t R, int64_t C, int64_t lda, const float *s, int op,
                                     void *out, int64_t ldo, awq_stream_t stream);
AWQ_API awq_status awq_scale_rows(const void *A, int64_t R, int64_t C, int64_t lda, const float *s, int op,
                                  void *out, int64_t ldo, awq_stream_t stream);

/* ---------------------------------------------------------------------------------------------------
 * Deployment GEMM of a quantized linear (W4A16): Y = X' deq(W)^T, the weights read as the packed codes,
 * steps and zeros of awq_quantize_pack and dequantized on the fly ("GPU 硬件级反量化算子内联融合" on the
 * bjdmk.com.cn AWQ article), deq(W)[o, k] = (q[o,k] - z[o,g]) * step[o,g], g = k / 128.
 * X' is the layer input with the AWQ scales already folded out (X diag(s)^-1, e.g. by awq_scale_columns
 * on the previous norm weight). fp32 accumulation on the tensor cores, bf16 output. The weight enters as:
 *   M > 64 tokens:  bf16(RN32(RN32(q - z) * step)), dequantized into the tensor-core operand tiles;
 *   M <= 64 tokens: its exact value: the tensor cores sum (128 + q) * x' per group of 128 in-features
 *                   (exact bf16 operands) and the step and zero point are applied per group and output,
 *                   Y = sum_g step_g * (S_g - (128 + z_g) * sum_{k in g} x'_k), in fp32.
 *   X       device bf16 [M, K], row stride ldx (multiple of 8)
 *   codes   device uint32 [O, K/8], steps / zeros device float [O, K/128] (contiguous, as packed)
 *   Y       device bf16 [M, O], row stride ldy (multiple of 8)
 *   workspace  device, >= awq_w4a16_workspace_size(K, O) bytes, ZERO-FILLED BEFORE ITS FIRST USE
 *              (e.g. cudaMemsetAsync once after allocating it). It holds the status word and a tile
 *              counter, a fixed 256 KB region of per-block counters (M <= 64 tokens; every call leaves
 *              them at zero, and nothing else writes there, so one zero fill serves all later calls
 *              whatever their shapes), a group-major copy of steps and zeros (many tokens), and for
 *              M <= 64 a permuted copy of X (64 rows), its per-group sums and split-K partial sums.
 *              After a device timeout the counters may be left set: zero-fill the workspace again
 *              before reusing it. M <= 64 is two launches on `stream`: a small kernel that writes the
 *              X copy and group sums, and the GEMM as its programmatic dependent (it starts early and
 *              waits for them).
 * Requires K % 128 == 0, O % 8 == 0, M >= 1. M <= 64 runs a few-token kernel (weight rows on the MMA's M
 * side, groups split across CTAs, partial sums added in a fixed order). Both are deterministic. A device
 * timeout is reported by awq_search_status() on the same workspace.
 * ------------------------------------------------------------------------------------------------- */
AWQ_API size_t awq_w4a16_workspace_size(int64_t K, int64_t O);
AWQ_API awq_status awq_w4a16_gemm(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *codes,
                                  const float *steps, const float *zeros, int64_t O, void *Y, int64_t ldy,
                                  void *workspace, size_t ws_bytes, awq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
