/*
 * moe.h -- C ABI of libmoe.so: the single-GPU forward pass of a routed-expert
 * mixture-of-experts MLP, as hand-written CUDA kernels for sm_100a (B200).
 *
 * Pipeline (one CUDA stream, no host synchronisation, no allocation):
 *
 *   logits --moe_route--> ids, w --moe_permute--> counts, offsets, row2assign, assign2row
 *   x (--moe_quantize_x--> xq, sx)            [block-scaled path only]
 *   x rows gathered by row2assign --moe_grouped_gemm1_swiglu--> act (expert-sorted rows)
 *   act --moe_grouped_gemm2--> y (expert-sorted rows)
 *   y, w, assign2row --moe_combine--> out (token order)
 *   moe_forward runs all of the above on one stream with the caller's workspace.
 *
 * Sources of the operations (web pages on routed MoE kernels; none gives an API):
 *   - TileScale PR #70 (distributed FP8 MegaMoE example), "Design": routing, GEMM1 with
 *     fused SwiGLU and FP8 requantisation (kernel 1), GEMM2 and the top-k slot reduction
 *     (kernel 2); the flat m-task queue that replaced a per-tile expert rescan (first
 *     change listed in the PR description); fp32 per-128-element activation scales.
 *   - FlashInfer PR #5129 (cuTile BF16 fused MoE), "sorted I/O": GEMM1 writes a padded
 *     expert-sorted row space that GEMM2 reads contiguously; combine unchanged.
 *   - FlashInfer PR #6465 (Hopper MXFP4 x FP8 MegaMoE tuning), benchmark setup: MXFP4
 *     weights with K32 scaling, FP8 activations, BF16 input/output, H=2560, E=512,
 *     top-k 10, I=640.
 *   - Liger-Kernel PR #1463 (SM90 MoE), benchmark definition: BF16 routed-expert MoE
 *     MLP forward, TFLOP/s counted over routed experts only.
 *
 * Conventions shared by every entry point
 *   - Notation: T tokens, H hidden size, I expert intermediate size (GEMM1 width 2I),
 *     E experts, k experts per token, R = T*k routed rows.
 *   - Every pointer argument is a DEVICE pointer on the current device unless marked
 *     "host".  The caller owns every buffer; the library never allocates, frees or
 *     synchronises on these paths.  All work is enqueued on `stream` (0 = legacy default).
 *   - Layouts are row-major.  Weights are K-major: W13 is [E][2I][H] with rows [0,I) the
 *     gate projection and rows [I,2I) the up projection; W2 is [E][H][I].
 *   - Argument checks run on the host before any launch and return an error without
 *     enqueuing work.  A failed launch returns MOE_ERR_CUDA.  A device-side bounded wait
 *     that expires, or a routing id out of range, sets a status word in the workspace;
 *     moe_get_device_status() reads it.
 *   - Device pointers must be 16-byte aligned.  BF16 path: H % 64 == 0 and I % 64 == 0.
 *     Block-scaled path: H % 128 == 0 and I % 128 == 0.  1 <= k <= min(E, 32),
 *     E <= 1024, 0 <= T and T*k < 2^31.  T == 0 is a valid no-op.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,          /* null pointer, bad enum, k > E, negative T ...      */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,    /* shape outside the preconditions above             */
  MOE_ERR_MISALIGNED = 3,           /* a pointer is not 16-byte aligned                  */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes < moe_workspace_size(shape)              */
  MOE_ERR_CUDA = 5,                 /* a CUDA runtime/driver call or launch failed       */
  MOE_ERR_DEVICE_TIMEOUT = 6,       /* device status: a bounded wait expired             */
  MOE_ERR_DEVICE_BAD_INDEX = 7      /* device status: an expert id outside [0, E)        */
} moe_status_t;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_t;
typedef enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_FP8_MXFP4 = 1 } moe_dtype_t;
/* GEMM1's activation.  SWIGLU: W13 [E][2I][H] (gate rows then up rows), act =
 * silu(gate) * up.  RELU2 (BF16 only; FlashInfer PR #5129 measures the Nemotron-3.5-
 * Lightning shape with it, read as the non-gated squared ReLU): W13 is W1 [E][I][H] and
 * act = max(x.W1^T, 0)^2. */
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_RELU2 = 1 } moe_act_t;

/* Problem description.  score: moe_score_t; renormalize: 1 = divide the k selected
 * weights by their sum; dtype: moe_dtype_t; activation: moe_act_t.
 * n_shared: shared experts (0 = none), run on every token with weight 1 (GC-MoE folds
 * shared experts into the compute role; DeepGEMM's SM100 path fuses them).  They are
 * experts E .. E+n_shared-1 of the weight tensors (which then hold E + n_shared experts;
 * logits stay [T][E]) and each token gets them as slots k .. k+n_shared-1 after its k
 * routed ones: every "k" and "E" below, past routing's own top-k selection, means
 * k + n_shared and E + n_shared (ids and w are [T][k + n_shared], R = T*(k + n_shared),
 * counts [E + n_shared]).  k + n_shared <= 32 and E + n_shared <= 1024. */
typedef struct {
  int64_t T;
  int32_t H, I, E, k;
  int32_t score;
  int32_t renormalize;
  int32_t dtype;
  int32_t activation;
  int32_t n_shared;
} moe_shape_t;

/* Bytes of device workspace moe_forward needs for `shape` (the stage entry points need
 * at most the same).  The first 256 bytes hold the device status word; the rest holds
 * routing metadata, the expert-sorted activations and expert outputs.  Returns 0 for an
 * invalid shape.  Sizes grow linearly in T*k*(H+I). */
MOE_API size_t moe_workspace_size(const moe_shape_t *shape);

/* Regions of the workspace in which moe_forward leaves the routing metadata of its last
 * call: the top-k ids (only when moe_forward's ids_out is NULL) and weights [T][k], the
 * per-expert counts [E] and offsets [E+1], and the expert-sorted permutation row2assign
 * and assign2row [R] (int32, except MOE_WS_W which is fp32).  They let a caller inspect
 * what the forward pass routed without running the stage entry points a second time; the
 * layout is the forward pass's (FlashInfer PR #5129 "sorted I/O": the permutation of the
 * expert-sorted row space).  On success *offset receives the region's byte offset from
 * the workspace base (a multiple of 256) and *bytes its size (host pointers).  Returns
 * MOE_ERR_INVALID_ARG for a bad shape, region or null pointer.  No device work. */
typedef enum {
  MOE_WS_IDS = 0,
  MOE_WS_W = 1,
  MOE_WS_COUNTS = 2,
  MOE_WS_OFFSETS = 3,
  MOE_WS_ROW2ASSIGN = 4,
  MOE_WS_ASSIGN2ROW = 5
} moe_ws_region_t;
MOE_API moe_status_t moe_workspace_region(const moe_shape_t *shape, int32_t region,
                                          size_t *offset, size_t *bytes);

/* Zero the status block of a workspace (call once after allocating it). */
MOE_API moe_status_t moe_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream);

/* Routing (TileScale PR #70 "Design"; FlashInfer PR #6465 top-k 10 workload).
 * logits: fp32 [T][E] router logits.  ids: int32 [T][k] out, slot j = j-th largest logit,
 * ties to the lower expert index.  w: fp32 [T][k] out: softmax over the selected logits
 * when renormalize (else over all E), or sigmoid of the selected logit (renormalised to
 * sum 1 when renormalize).  No workspace. */
MOE_API moe_status_t moe_route(const moe_shape_t *shape, const float *logits, int32_t *ids, float *w,
                       cudaStream_t stream);

/* Histogram + exclusive prefix sum + stable scatter into the expert-sorted row space
 * (FlashInfer PR #5129 "sorted I/O").  ids: int32 [T*k] in.  counts: int32 [E] out.
 * offsets: int32 [E+1] out, offsets[e] = first sorted row of expert e.  row2assign: int32
 * [R] out, the assignment a = t*k + j held by sorted row r; rows of one expert are in
 * ascending a.  assign2row: int32 [R] out, its inverse.  ws: workspace (scratch for
 * per-chunk histograms + status word).  Ids outside [0,E) set MOE_ERR_DEVICE_BAD_INDEX in
 * the status word and are skipped. */
MOE_API moe_status_t moe_permute(const moe_shape_t *shape, const int32_t *ids, int32_t *counts,
                         int32_t *offsets, int32_t *row2assign, int32_t *assign2row, void *ws,
                         size_t ws_bytes, cudaStream_t stream);

/* Allocation-free variant of moe_permute, for callers that cannot hand the library a
 * workspace: host code that runs where device allocation is not allowed or not
 * possible -- for example an integration layer whose memory is a fixed pool reserved at
 * start-up and which has no scratch buffer to pass down.  (This entry point has no
 * counterpart on the pages; it is a packaging variant of the permutation above.)
 * Same inputs, outputs and results as moe_permute, bit for bit.  The per-chunk
 * histograms and their scans live in a 512 KB file-scope device array instead of the
 * workspace; it needs (2 * nch + 1) * E <= 131072 ints, where nch = ceil(T / 64) up to
 * T = 8192 and 128 beyond (the chunks grow), so every T works for E <= 510, where E
 * counts the shared experts (E + n_shared).  Larger problems return
 * MOE_ERR_UNSUPPORTED_SHAPE without launching anything.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress, with that device current)
 * and caches it with the id of the current context; the first call in a new context
 * (for example after cudaDeviceReset) looks it up again.  Make that first call before
 * any stream capture.  Every call shares the array: calls
 * whose kernels overlap on the GPU (other streams, other host threads) race on it;
 * calls ordered on one stream are safe, and no state carries over between them.  Ids
 * outside [0, E) are skipped, as in moe_permute, but there is no status word to record
 * them in.  Calls no cudaMalloc, cudaFree or allocating library routine. */
MOE_API moe_status_t moe_permute_noalloc(const moe_shape_t *shape, const int32_t *ids,
                                         int32_t *counts, int32_t *offsets, int32_t *row2assign,
                                         int32_t *assign2row, cudaStream_t stream);

/* Block-scaled path: per token and per 128 consecutive columns, the smallest power of two
 * s = 2^e (e clamped to [-127,127]) with max|x| <= 448*s, and e4m3 codes of x/s (round to
 * nearest even, saturating).  TileScale PR #70 "Design" (FP8 E4M3, fp32 per-128 scales).
 * x: bf16 [T][H].  xq: uint8 e4m3 [T][H] out.  sx: fp32 [T][H/128] out. */
MOE_API moe_status_t moe_quantize_x(const moe_shape_t *shape, const uint16_t *x, uint8_t *xq, float *sx,
                            cudaStream_t stream);

/* One-off weight preparation for the block-scaled path (not on the forward path): MXFP4
 * per the OCP MX rule, one UE8M0 scale per 32 consecutive K elements: byte =
 * clamp(floor(log2 amax) - 2 + 127, 0, 254) (0 when amax == 0), codes = e2m1 of
 * w / 2^(byte-127), round to nearest even, saturating.  FlashInfer PR #6465 (MXFP4 K32).
 * w: bf16 [rows][K] (K % 32 == 0).  packed: uint8 [rows][K/2] out, element 2i in the low
 * nibble of byte i.  sf: uint8 [rows][K/32] out. */
MOE_API moe_status_t moe_quantize_weights_mxfp4(int64_t rows, int32_t K, const uint16_t *w,
                                        uint8_t *packed, uint8_t *sf, cudaStream_t stream);

/* Grouped GEMM1 with fused SwiGLU over the expert-sorted rows (TileScale PR #70 kernel 1;
 * FlashInfer PR #5129 gathered-A GEMM1).  For sorted row r of expert e with token
 * t = row2assign[r] / k:  act[r][i] = silu(x[t].W13[e][i]) * (x[t].W13[e][I+i]), fp32
 * accumulation, silu(g) = g / (1 + exp(-g)); with activation RELU2,
 * act[r][i] = max(x[t].W1[e][i], 0)^2.
 *   BF16:  a = x bf16 [T][H]; sa, w13_sf, act_sf unused (may be NULL); w13 bf16 [E][2I][H]
 *          (RELU2: W1 bf16 [E][I][H]); act bf16 [R][I] out.
 *   FP8:   a = xq e4m3 [T][H]; sa = sx fp32 [T][H/128]; w13 = MXFP4 [E][2I][H/2];
 *          w13_sf = UE8M0 [E][2I][H/32]; act = e4m3 [R][I] out, requantised per 1x128
 *          with the moe_quantize_x rule; act_sf fp32 [R][I/128] out.
 * offsets: int32 [E+1] from moe_permute.  ws: workspace (status word). */
MOE_API moe_status_t moe_grouped_gemm1_swiglu(const moe_shape_t *shape, const void *a, const float *sa,
                                      const int32_t *row2assign, const int32_t *offsets,
                                      const void *w13, const uint8_t *w13_sf, void *act,
                                      float *act_sf, void *ws, size_t ws_bytes,
                                      cudaStream_t stream);

/* Grouped GEMM2 (down projection) over the expert-sorted rows (TileScale PR #70 kernel 2;
 * FlashInfer PR #5129 sorted-I/O GEMM2).  y[r][o] = act[r].W2[e][o], fp32 accumulation,
 * bf16 out.
 *   BF16:  act bf16 [R][I]; w2 bf16 [E][H][I]; act_sf, w2_sf unused.
 *   FP8:   act e4m3 [R][I] + act_sf fp32 [R][I/128]; w2 MXFP4 [E][H][I/2] + w2_sf UE8M0
 *          [E][H][I/32].
 * y: bf16 [R][H] out.  offsets: int32 [E+1].  ws: workspace (status word). */
MOE_API moe_status_t moe_grouped_gemm2(const moe_shape_t *shape, const void *act, const float *act_sf,
                               const int32_t *offsets, const void *w2, const uint8_t *w2_sf,
                               uint16_t *y, void *ws, size_t ws_bytes, cudaStream_t stream);

/* Top-k weighted combine back to token order (TileScale PR #70, the slot reduction of
 * kernel 2).  out[t][h] = bf16_rne( sum_{j<k, ascending} w[t][j] * y[assign2row[t*k+j]][h] ),
 * fp32 sum.  y bf16 [R][H]; w fp32 [T][k]; assign2row int32 [R]; out bf16 [T][H]. */
MOE_API moe_status_t moe_combine(const moe_shape_t *shape, const uint16_t *y, const float *w,
                         const int32_t *assign2row, uint16_t *out, cudaStream_t stream);

/* The whole forward pass on one stream.  x bf16 [T][H]; logits fp32 [T][E]; weights as in
 * the GEMM entry points for shape->dtype; out bf16 [T][H].  ids_out: optional int32 [T][k]
 * copy of the routing ids (NULL to skip).  ws: >= moe_workspace_size(shape) bytes,
 * 256-byte aligned, initialised once with moe_workspace_init. */
MOE_API moe_status_t moe_forward(const moe_shape_t *shape, const uint16_t *x, const float *logits,
                         const void *w13, const uint8_t *w13_sf, const void *w2,
                         const uint8_t *w2_sf, uint16_t *out, int32_t *ids_out, void *ws,
                         size_t ws_bytes, cudaStream_t stream);

/* Synchronise `stream`, read the workspace status word, clear it, and return it
 * (MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_BAD_INDEX).  A non-OK status also
 * resets the rest of the 256-byte status block (the front end's grid-barrier words), so
 * the workspace is usable again without moe_workspace_init. */
MOE_API moe_status_t moe_get_device_status(void *ws, cudaStream_t stream);

/* Static string for a status code (host). */
MOE_API const char *moe_status_string(moe_status_t status);

/* Test hooks for failure detection (host).  moe_debug_set_wait_limit_ns sets the bound on
 * every device-side wait (default 4 s; 0 restores the default).  moe_debug_inject_stall(1)
 * makes CTA 0 of every following grouped-GEMM launch leave its first pipeline stage
 * unfilled, so that its consumer's bounded wait expires, the kernel unwinds and the status
 * word reads MOE_ERR_DEVICE_TIMEOUT; outputs of such calls are undefined.  It also makes
 * the grid-wide barrier of moe_forward's large-batch front end (routing and permutation in
 * one launch) wait for one arrival more than there are CTAs, with the same outcome.
 * (0 = off.) */
MOE_API void moe_debug_set_wait_limit_ns(uint64_t ns);
MOE_API void moe_debug_inject_stall(int on);

/* Per-stage timing of moe_forward (host), for the per-kernel breakdown of a benchmark.
 * After moe_debug_time_stages(1), every moe_forward call on this host thread records a
 * CUDA event (owned by the library) on its stream before its first launch and after each
 * stage: "route_permute" (routing and permutation, one launch at every batch size),
 * "quantize_x" (FP8 x MXFP4), "gemm1_swiglu" (with the decode-sized K-split finish),
 * "gemm2" and "combine".  The events take away the overlap that programmatic
 * dependent launch gives consecutive kernels, so time whole steps with it off, and do not
 * turn it on while capturing a CUDA graph.  moe_debug_stage_times waits for the last
 * forward's final event, writes up to `max` stage names (static strings) and times in
 * milliseconds, and returns the number of stages that forward recorded (0 if none, -1 on
 * a CUDA error).  moe_debug_time_stages(0) turns recording off. */
MOE_API void moe_debug_time_stages(int on);
MOE_API int moe_debug_stage_times(const char **names, float *ms, int max);

/* Number of kernel launches the last successful call of each entry point enqueued on
 * this host thread (host). */
MOE_API int moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
