/*
 * llmint8.h — C ABI of the B200 (sm_100a) LLM.int8() linear-layer library.
 *
 * The library computes C = X.W for a transformer linear layer the way the
 * LLM.int8() method does it:
 *
 *   Step 1  outlier detection: O = { j : some row i has |X[i][j]| >= alpha }
 *   Step 2  decomposition: X^O = X[:, O] and W^O = W[O, :] (fp16);
 *           the rest of X and W goes to the int8 path
 *   Step 3  fp16 outlier product X^O . W^O (fp32 accumulation)
 *   Step 4  vector-wise absmax quantisation: one scale per row of X (over the
 *           non-outlier columns), one per column of W; int8 x int8 product
 *           accumulated in int32; dequantised by the outer product of the
 *           scales (divided by 127*127)
 *   Step 5  sum of the two parts, stored once as fp16.
 *
 * Sources: "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale"
 * (paper-graph-ui summary), section "The Full LLM.int8() Algorithm", Steps 1-5,
 * and sections "Vector-wise Quantization" and "Mixed-Precision Decomposition";
 * "tm_llm_int8" (aicassindra.com), sections "Absmax INT8 quantization from
 * first principles" and "The mixed-precision decomposition";
 * "LLM.int8() 完全拆解" (pinghaoyang.com.cn), sections "第一件武器：向量级量化"
 * and "第二件武器：混合精度分解".
 *
 * Conventions for every entry point:
 *  - Half-precision tensors are IEEE binary16, passed as uint16_t bit
 *    patterns. All tensors are dense and row-major unless stated.
 *  - Pointers named *_dev are device pointers of the current CUDA device,
 *    owned by the caller; the library never allocates or frees device memory
 *    (scratch space comes from the caller's workspace).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Calls are asynchronous: LLMINT8_OK means "validated and
 *    enqueued", except where a function says it synchronises.
 *  - Arguments are validated on the host before anything is enqueued; on an
 *    error return nothing has been enqueued and no output was touched.
 *  - Shape rules: 16 <= h <= 133144 and h % 16 == 0 (16-byte TMA row
 *    strides for int8; 127*127*h must fit int32); o >= 16 and o % 16 == 0;
 *    s >= 0 (s == 0 is a no-op that returns LLMINT8_OK). Device pointers to
 *    fp16/int8 tensors must be 16-byte aligned; the workspace 256-byte aligned.
 *  - alpha must be >= 0 (and not NaN); alpha = +inf switches the
 *    decomposition off (pure vector-wise int8). The comparison is |x| >= alpha.
 *  - Rounding of int8 codes: q = round-half-away-from-zero(fp32(127*x) / a)
 *    with one IEEE fp32 division; a == 0 gives q == 0.
 *  - The kernels contain only bounded waits. If one runs out (it should not),
 *    the kernel records a bit in the workspace's status word and returns;
 *    llmint8_read_device_status() reports and clears it. A caller that gives
 *    llmint8_matmul_ex a mapped host status word (opts.status_host) has the
 *    bits of each call copied there by the call's last kernel, and its next
 *    call on that word returns LLMINT8_ERR_DEVICE_STATUS without enqueuing
 *    anything, with no synchronisation.
 *  - Only sm_100 devices are supported; other devices give
 *    LLMINT8_ERR_UNSUPPORTED. There is no CPU fallback.
 */
#ifndef LLMINT8_H_
#define LLMINT8_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLMINT8_API __attribute__((visibility("default")))
#else
#define LLMINT8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LLMINT8_OK = 0,
    LLMINT8_ERR_NULL = -1,          /* a required pointer is NULL */
    LLMINT8_ERR_SHAPE = -2,         /* a size breaks the shape rules */
    LLMINT8_ERR_ALIGN = -3,         /* a pointer breaks the alignment rules */
    LLMINT8_ERR_WORKSPACE = -4,     /* workspace smaller than required */
    LLMINT8_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed */
    LLMINT8_ERR_DEVICE_STATUS = -6, /* a kernel flagged an anomaly (see status_host) */
    LLMINT8_ERR_ARG = -7,           /* a scalar argument is invalid */
    LLMINT8_ERR_UNSUPPORTED = -8,   /* current device is not sm_100 */
    LLMINT8_ERR_TOO_LARGE = -9      /* problem exceeds the no-alloc scratch */
} llmint8_status;

/* Bits of the device status word (llmint8_read_device_status). */
#define LLMINT8_DEV_TIMEOUT_PRODUCER 0x1  /* TMA producer gave up waiting */
#define LLMINT8_DEV_TIMEOUT_MMA 0x2       /* MMA issuer gave up waiting */
#define LLMINT8_DEV_TIMEOUT_EPILOGUE 0x4  /* epilogue gave up waiting */
#define LLMINT8_DEV_TIMEOUT_DRAIN 0x8     /* drain after an abort timed out */
#define LLMINT8_DEV_TIMEOUT_ROWS 0x10     /* activation row stream gave up waiting */
#define LLMINT8_DEV_TIMEOUT_SELFTEST 0x20 /* llmint8_wait_selftest's waits ran out */
#define LLMINT8_DEV_OUTLIER_CAP 0x40      /* |O| above the workspace's outlier
                                             capacity: the call's output has no
                                             fp16 outlier product */

/* A prepared (offline-quantised) weight. Buffers are caller-owned device
 * memory: wq_dev is int8 [o][h] (the reduction index k contiguous, i.e. the
 * transpose of W), aw_dev is fp32 [o] holding each column's absmax (an exact
 * binary16 value). */
typedef struct {
    int64_t h;
    int64_t o;
    int8_t *wq_dev;
    float *aw_dev;
    /* Optional (NULL: off): the caller's fp16 weight W [h][o] (16-byte
     * aligned), kept alive by the caller while the weight is in use. When
     * set, the fp16 outlier rows of W are W's own values, WO[t][j] =
     * W[O_t][j] ("Mixed-Precision Decomposition": the outlier part of W stays
     * in fp16), instead of being recovered from wq. prepare_weight ignores
     * it. */
    const uint16_t *w16_dev;
} llmint8_weight;

/* llmint8_matmul_opts.path */
#define LLMINT8_PATH_AUTO 0
#define LLMINT8_PATH_PREFILL 1
#define LLMINT8_PATH_DECODE 2
#define LLMINT8_PATH_PREFILL_SINGLE 3
#define LLMINT8_PATH_PREFILL_PAIR 4

/* The kernel llmint8_matmul runs, on the current device, for an [s, h] x
 * [h, o] call with the automatic path: LLMINT8_PATH_DECODE (s <= 16) or
 * LLMINT8_PATH_PREFILL_SINGLE (the CTA-pair kernel runs only when asked for
 * with LLMINT8_PATH_PREFILL_PAIR).
 * A negative llmint8_status on error (LLMINT8_ERR_SHAPE for s < 0, h <= 0
 * or o <= 0; no usable device). Enqueues nothing. */
LLMINT8_API int32_t llmint8_prefill_kernel(int64_t s, int64_t h, int64_t o);

/* Optional extras for llmint8_matmul_ex (all fields may be zero/NULL).
 *  gemm_event_start/stop: cudaEvent_t (as void*) recorded on `stream`
 *      immediately before and after the int8 GEMM kernel launch, for timing
 *      the dominant kernel from the caller.
 *  ci_dev: if non-NULL, int32 [s][o] receives the exact int32 accumulators
 *      of Step 4 (testing; costs an extra 4*s*o bytes of stores).
 *  path: LLMINT8_PATH_AUTO (0) = automatic; LLMINT8_PATH_PREFILL (1) = the
 *      prefill GEMM, its kernel chosen automatically; LLMINT8_PATH_DECODE
 *      (2) = the decode (s <= 16) kernel, LLMINT8_ERR_ARG with s > 16;
 *      LLMINT8_PATH_PREFILL_SINGLE (3) = the prefill GEMM with one CTA per
 *      128 x 256 tile; LLMINT8_PATH_PREFILL_PAIR (4) = the prefill GEMM with
 *      a pair of CTAs (a cluster of two) per 256 x 256 tile,
 *      LLMINT8_ERR_UNSUPPORTED where no such cluster fits the device. Every
 *      kernel gives the same results bit for bit.
 *  launches (out): number of kernels this call enqueued.
 *  x_scale: LLMINT8_SCALE_VECTORWISE (0, the method: one absmax per row of
 *      X) or LLMINT8_SCALE_TENSORWISE (one absmax for all of X, the largest
 *      row scale, so every ax[i] is that constant); anything else is
 *      LLMINT8_ERR_ARG. Outlier columns are split off in both modes.
 *  max_outliers: outlier columns the workspace holds (0: h, the default and
 *      the worst case). The workspace must then hold
 *      llmint8_workspace_size_ex(s, h, o, max_outliers) bytes. A call whose
 *      |O| exceeds it writes no outlier tile, skips the fp16 outlier product
 *      (the output is the int8 part alone; the outlier columns are still
 *      removed from it) and sets LLMINT8_DEV_OUTLIER_CAP. Negative or above
 *      h: LLMINT8_ERR_ARG.
 *  status_host: NULL, or a 4-byte word of pinned host memory that the device
 *      can address (cudaHostAlloc / cudaMallocHost memory under unified
 *      addressing; anything else is LLMINT8_ERR_ARG). When the word is
 *      nonzero on entry the call returns LLMINT8_ERR_DEVICE_STATUS at once;
 *      otherwise the call's last kernel ORs the workspace's status bits into
 *      it as it finishes. The caller clears the word, and re-initialises the
 *      workspace (llmint8_workspace_init), before going on.
 *  wo_build: where the prefill path builds the fp16 outlier rows of W
 *      (Step 2, W side); results are the same bit for bit in every form.
 *      LLMINT8_WO_SHARED (0, default): the GEMM's CTAs, each a share, while
 *      their first mainloops run; each then waits a short, bounded time for
 *      the other shares, and a CTA that does not see them all in time (its
 *      peers not resident, e.g. under SM partitioning) builds every row
 *      itself, so the result never depends on how many CTAs run at once.
 *      LLMINT8_WO_BEFORE_GEMM (1): the activation kernels, before the GEMM;
 *      no CTA of the GEMM waits for another. LLMINT8_WO_EACH_CTA (2): every
 *      GEMM CTA builds all rows itself at once (the fallback above, on
 *      purpose; for testing). Anything else is LLMINT8_ERR_ARG. */
typedef struct {
    void *gemm_event_start;
    void *gemm_event_stop;
    int32_t *ci_dev;
    int32_t path;
    int32_t launches;
    int32_t x_scale;
    int32_t max_outliers;
    int32_t *status_host;
    int32_t wo_build;
} llmint8_matmul_opts;

#define LLMINT8_WO_SHARED 0
#define LLMINT8_WO_BEFORE_GEMM 1
#define LLMINT8_WO_EACH_CTA 2

/* Scale granularity ("Quantization Primitives": absmax over a whole tensor;
 * "Vector-wise Quantization": one constant per row of X and per column of
 * W). The tensor-wise modes are the Table 1 baselines ("Int8 absmax"), kept
 * for comparison; vector-wise is the method. */
#define LLMINT8_SCALE_VECTORWISE 0
#define LLMINT8_SCALE_TENSORWISE 1

/* Human-readable name of a status code (static storage). */
LLMINT8_API const char *llmint8_status_string(llmint8_status st);

/* Bytes of device workspace llmint8_matmul needs for an [s,h] x [h,o]
 * problem. Sized for the worst case |O| = h, so any alpha fits:
 * about s*h (int8 codes) + 2*s*h (fp16 outlier columns of X) + 2*h*o (fp16
 * outlier rows of W) + 4*16*o (decode accumulators) + O(h + s). */
LLMINT8_API size_t llmint8_workspace_size(int64_t s, int64_t h, int64_t o);

/* Workspace for calls whose opts.max_outliers is max_outliers (0: h): the
 * outlier tiles shrink to 2*s*max_outliers + 2*max_outliers*o bytes. For the
 * OPT-175B shapes (h = 12288, o = 49152) and 64 outlier columns that is tens
 * of MB instead of the 1.2 GB of the worst case. 0 if max_outliers is
 * negative or above h. */
LLMINT8_API size_t llmint8_workspace_size_ex(int64_t s, int64_t h, int64_t o,
                                             int64_t max_outliers);

/* Bytes at the front of a workspace that hold state kept between calls: the
 * status words (first 256 bytes), then the outlier bitmask that the one-read
 * activation pass accumulates into and leaves zero when it finishes. */
#define LLMINT8_WORKSPACE_STATE_BYTES 17152

/* Clears the workspace's state block (its first LLMINT8_WORKSPACE_STATE_BYTES
 * bytes; ws_bytes must cover them). Call once on a new workspace before its
 * first llmint8_matmul, and again before reusing a workspace after a call
 * returned LLMINT8_ERR_DEVICE_STATUS (an aborted kernel may leave the state
 * dirty). Asynchronous on `stream`. */
LLMINT8_API llmint8_status llmint8_workspace_init(void *ws_dev, size_t ws_bytes, void *stream);

/* Workspace for llmint8_matmul_host: llmint8_workspace_size plus staging
 * for the device copies of X (2*s*h bytes) and of C (2*s*o bytes). */
LLMINT8_API size_t llmint8_workspace_size_host(int64_t s, int64_t h, int64_t o);
LLMINT8_API size_t llmint8_workspace_size_host_ex(int64_t s, int64_t h, int64_t o,
                                                  int64_t max_outliers);

/* Offline weight preparation ("The Full LLM.int8() Algorithm", Step 1 remark
 * that W's part is fixed at model-load time, and section "Why vector-wise
 * rather than row-wise": column constants precomputed once):
 *   aw[j]    = max_k |W[k][j]|            over all h rows
 *   wq[j][k] = q(W[k][j], aw[j])           (see rounding rule above)
 * W_dev is fp16 [h][o]. out->h, out->o must equal h, o and out->wq_dev /
 * out->aw_dev must point at caller buffers of o*h and o elements. */
LLMINT8_API llmint8_status llmint8_prepare_weight(const uint16_t *W_dev, int64_t h,
                                      int64_t o, llmint8_weight *out,
                                      void *stream);

/* llmint8_prepare_weight with a scale granularity: w_scale =
 * LLMINT8_SCALE_VECTORWISE is llmint8_prepare_weight; TENSORWISE sets every
 * aw[j] to max_{k,j} |W[k][j]| and quantises all of W against it. Any other
 * w_scale is LLMINT8_ERR_ARG. */
LLMINT8_API llmint8_status llmint8_prepare_weight_ex(const uint16_t *W_dev, int64_t h,
                                         int64_t o, int32_t w_scale,
                                         llmint8_weight *out, void *stream);

/* Column-parallel preparation ("LLM.int8(): 8-bit Matrix Multiplication for
 * Transformers at Scale", Appendix D: a 175B-size layer spread over several
 * GPUs): prepares columns [col0, col0 + o) of a weight W_dev [h][ldw] (row
 * stride ldw elements) exactly as llmint8_prepare_weight prepares a weight
 * made of those columns alone. Every column's scale and codes depend on
 * that column only, so the shards of a layer, each on its own GPU, together
 * hold the whole prepared weight, and each shard's llmint8_matmul output is
 * that block of the layer's output columns, bit for bit. Rules: o as for
 * llmint8_prepare_weight; ldw >= col0 + o; ldw and col0 multiples of 8 (so
 * that W_dev + col0 is 16-byte aligned); out->o == o, out->h == h; w_scale
 * as in llmint8_prepare_weight_ex. */
LLMINT8_API llmint8_status llmint8_prepare_weight_cols(const uint16_t *W_dev, int64_t h,
                                           int64_t ldw, int64_t col0, int64_t o,
                                           int32_t w_scale, llmint8_weight *out,
                                           void *stream);

/* Steps 1 and 4 (activation side) on their own, for testing:
 *   flags_dev[j]  = 1 if column j is an outlier column, else 0   (u8 [h])
 *   idx_dev[0..n) = outlier columns in ascending order           (i32 [h])
 *   *n_outliers_dev = n                                          (i32 scalar)
 *   ax_dev[i]     = max over non-outlier j of |X[i][j]| (0 if none) (f32 [s])
 *   Xq_dev[i][j]  = q(X[i][j], ax[i]) for non-outlier j, else 0  (i8 [s][h])
 * X_dev is fp16 [s][h]. scratch_dev must hold
 * llmint8_quantize_rows_scratch_size(h) bytes (256-byte aligned); its
 * contents need no initialisation (word 1 receives device status bits). */
LLMINT8_API size_t llmint8_quantize_rows_scratch_size(int64_t h);
LLMINT8_API llmint8_status llmint8_quantize_rows(const uint16_t *X_dev, int64_t s,
                                     int64_t h, float alpha, int8_t *Xq_dev,
                                     float *ax_dev, uint8_t *flags_dev,
                                     int32_t *idx_dev, int32_t *n_outliers_dev,
                                     void *scratch_dev, size_t scratch_bytes,
                                     void *stream);

/* llmint8_quantize_rows with a scale granularity: x_scale =
 * LLMINT8_SCALE_TENSORWISE makes every ax[i] the largest of the row scales
 * above and quantises all rows against it (outlier columns still 0);
 * VECTORWISE is llmint8_quantize_rows; anything else is LLMINT8_ERR_ARG. */
LLMINT8_API llmint8_status llmint8_quantize_rows_ex(const uint16_t *X_dev, int64_t s,
                                        int64_t h, float alpha, int32_t x_scale,
                                        int8_t *Xq_dev, float *ax_dev,
                                        uint8_t *flags_dev, int32_t *idx_dev,
                                        int32_t *n_outliers_dev, void *scratch_dev,
                                        size_t scratch_bytes, void *stream);

/* The whole layer, Steps 1-5: out_dev (fp16 [s][o]) = LLM.int8()(X_dev, w).
 *   out[i][j] = fp16( Ci[i][j] * ax[i] * aw[j] / (127*127)
 *                     + sum_{t in O} X[i][t] * WO[t][j] )
 * where WO[t][j] = fp16( fp32(fp32(wq[j][t]) * aw[j]) / 127 ) is the fp16
 * outlier row of W recovered from the int8 weight (the prepared weight is
 * the only copy of W the library holds). Ci is exact; the fp16 outlier
 * product and the dequantisation use fp32 arithmetic. ws_dev must hold
 * llmint8_workspace_size(s, h, o) bytes and have been cleared once with
 * llmint8_workspace_init; it may be reused across calls on the same stream
 * (with any s, h, o it is large enough for), not shared by calls that can
 * overlap. |O| stays on the device: the call never synchronises. */
LLMINT8_API llmint8_status llmint8_matmul(const uint16_t *X_dev, int64_t s,
                              const llmint8_weight *w, float alpha,
                              uint16_t *out_dev, void *ws_dev, size_t ws_bytes,
                              void *stream);

/* llmint8_matmul with the extras of llmint8_matmul_opts (opts may be NULL). */
LLMINT8_API llmint8_status llmint8_matmul_ex(const uint16_t *X_dev, int64_t s,
                                 const llmint8_weight *w, float alpha,
                                 uint16_t *out_dev, void *ws_dev,
                                 size_t ws_bytes, llmint8_matmul_opts *opts,
                                 void *stream);

/* End-to-end form with HOST buffers: copies X_host (fp16 [s][h], ideally
 * pinned) into the workspace, runs llmint8_matmul, copies C back into
 * out_host (fp16 [s][o]) and synchronises `stream` before returning.
 * ws_dev must hold llmint8_workspace_size_host(s, h, o) bytes. */
LLMINT8_API llmint8_status llmint8_matmul_host(const uint16_t *X_host, int64_t s,
                                   const llmint8_weight *w, float alpha,
                                   uint16_t *out_host, void *ws_dev,
                                   size_t ws_bytes, void *stream);

/* llmint8_matmul_host with the extras of llmint8_matmul_opts (opts may be
 * NULL; the same fields and errors as llmint8_matmul_ex). */
LLMINT8_API llmint8_status llmint8_matmul_host_ex(const uint16_t *X_host, int64_t s,
                                      const llmint8_weight *w, float alpha,
                                      uint16_t *out_host, void *ws_dev,
                                      size_t ws_bytes, llmint8_matmul_opts *opts,
                                      void *stream);

/* The fp16 outlier tiles of the last llmint8_matmul on this workspace:
 * copies n_outliers (to *n_out_host), XO (fp16 [s][n], to XO_host if
 * non-NULL) and WO (fp16 [n][o], to WO_host if non-NULL) from the workspace
 * to host memory sized for n = h. s, h, o must be those of that call (the
 * workspace layout depends on them). Synchronises `stream`. Testing aid. */
LLMINT8_API llmint8_status llmint8_read_outlier_tiles(const void *ws_dev, size_t ws_bytes,
                                          int64_t s, int64_t h, int64_t o,
                                          int32_t *n_out_host,
                                          uint16_t *XO_host, uint16_t *WO_host,
                                          void *stream);

/* llmint8_read_outlier_tiles for a call made with opts.max_outliers =
 * max_outliers (the layout depends on it). When the call's |O| exceeded
 * that capacity, *n_out_host is still |O| and nothing else is copied. */
LLMINT8_API llmint8_status llmint8_read_outlier_tiles_ex(const void *ws_dev, size_t ws_bytes,
                                             int64_t s, int64_t h, int64_t o,
                                             int64_t max_outliers, int32_t *n_out_host,
                                             uint16_t *XO_host, uint16_t *WO_host,
                                             void *stream);

/* Reads and clears the device status word kept in a matmul workspace;
 * synchronises `stream`. Returns LLMINT8_ERR_DEVICE_STATUS if any bit was
 * set (bits also stored in *bits_out when non-NULL), else LLMINT8_OK. */
LLMINT8_API llmint8_status llmint8_read_device_status(void *ws_dev, size_t ws_bytes,
                                          int32_t *bits_out, void *stream);

/* Testing aid for the bounded waits every kernel of this library uses:
 * enqueues one small kernel whose two waits can never be satisfied — an
 * mbarrier phase that nothing completes, and a word of the workspace's
 * state block that nothing sets (zeroed here first) — each limited to
 * limit_ns nanoseconds (1e3 <= limit_ns <= 1e10, else LLMINT8_ERR_ARG).
 * Both give up, the kernel sets LLMINT8_DEV_TIMEOUT_SELFTEST in the status
 * word and returns, and the CUDA context stays usable. ws_dev is a matmul
 * workspace (at least LLMINT8_WORKSPACE_STATE_BYTES). Asynchronous on
 * `stream`; read the result with llmint8_read_device_status. */
LLMINT8_API llmint8_status llmint8_wait_selftest(void *ws_dev, size_t ws_bytes,
                                     uint64_t limit_ns, void *stream);

/* Allocation-free form of llmint8_matmul (the pages have no counterpart: it
 * is a deployment convenience, not part of the method).
 *
 * Some callers cannot give the library a device workspace: they run where
 * device allocation is not allowed or not possible at call time, e.g. an
 * operator invoked from inside another runtime's execution callback whose
 * memory plan is fixed, or a host program with no allocator of its own for
 * scratch buffers. For them this entry point takes only the inputs and the
 * output and uses instead a scratch buffer that lives inside the library: a
 * static device array of LLMINT8_NOALLOC_MAX_SCRATCH_BYTES bytes, which every
 * GPU that loads the library keeps reserved until the process exits.
 *
 * - It accepts the problems whose workspace, llmint8_workspace_size(s, h, o),
 *   fits that maximum and returns LLMINT8_ERR_TOO_LARGE for the others.
 * - It never calls cudaMalloc/cudaFree or any allocating routine.
 * - The first call on a device looks up the array's device address with that
 *   device current and clears the array's status block; make that first call
 *   before any stream capture on that device.
 * - Every call on a device shares the one array and leaves its contents
 *   behind for the next call (each call resets what it needs). Calls whose
 *   execution can overlap on the GPU (other streams, other host threads)
 *   race on it and must be serialised by the caller.
 * Results equal llmint8_matmul's for the same inputs. */
#define LLMINT8_NOALLOC_MAX_SCRATCH_BYTES (64ull << 20)
LLMINT8_API llmint8_status llmint8_matmul_noalloc(const uint16_t *X_dev, int64_t s,
                                                  const llmint8_weight *w, float alpha,
                                                  uint16_t *out_dev, void *stream);

/* Status of the allocation-free entry point on the current device (no
 * counterpart on the pages either). Its kernels record anomalies (a bounded
 * wait that ran out) in a status word inside the library's scratch array,
 * where no caller buffer can see them; this reads that word into *bits_out
 * (when non-NULL), clears it and clears the rest of the array's state block.
 * Synchronises `stream`. Returns LLMINT8_ERR_DEVICE_STATUS if any bit was
 * set, else LLMINT8_OK. Each llmint8_matmul_noalloc call starts from a clean
 * activation state of its own, so a failed call does not spoil later ones,
 * but its output is wrong and only this function reports it. Before the
 * first no-alloc call on a device it returns LLMINT8_OK with no bits. */
LLMINT8_API llmint8_status llmint8_noalloc_read_device_status(int32_t *bits_out, void *stream);

/* Largest s the decode kernel accepts. */
LLMINT8_API int64_t llmint8_decode_max_rows(void);

#ifdef __cplusplus
}
#endif

#endif /* LLMINT8_H_ */
