/*
 * w8a8.h -- C ABI of libw8a8.so: the W8A8 int8-dynamic linear layer on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (scheme from "Issue 5 probe: int8 quantized DiT serve paths on the
 * RTX 3090 (24 GB)", section "Round two ... W8A8 int8-dynamic": int8 weights
 * with fp32 per-output-channel scales, dynamic per-token symmetric int8
 * activations; "Int8 Quantization" user guide, "Overview" and "Parameters":
 * activation scales are computed online, static scaling is not supported):
 *
 *   s_a[m] = max_k |x[m,k]| / 127                       (fp32, IEEE, RNE)
 *   q[m,k] = clamp(rint(x[m,k] / s_a[m]), -127, 127)     (ties to even; a row
 *                                                          with max 0 has s_a = 0, q = 0)
 *   acc[m,n] = sum_k q[m,k] * Wq[n,k]                   (exact int32)
 *   y[m,n] = bf16_rne( ((float)acc * s_a[m]) * s_w[n] + (float)bias[n] )
 *
 * with Wq, s_w obtained by the same per-row rule from the bf16 weight W[N,K]
 * (per-output-channel weight quantization: same "Round two" section; "Qwen-Image-2.1:
 * TE AutoRound-AWQ on GPU + all-resident single-3090 stack", section
 * "Whole-pipeline follow-up", on per-token activation and per-channel weight
 * quantization).  The small-M path (M <= 16) serves the AdaLN modulation and
 * conditioning-embedder layers that run at M = batch (unsloth commit history of
 * test_diffusion_transformer_quant.py, the commit on torch._int_mm requiring
 * more than 16 rows).
 *
 * Conventions for every call
 * --------------------------
 *  - Layouts are row-major.  x bf16 [M,K] (row stride ldx elements), W bf16
 *    [N,K] (row stride ldw), Wq int8 [N,K] dense (row stride K), q int8 [M,K]
 *    dense, s_a fp32 [M], s_w fp32 [N], bias bf16 [N] or NULL, y bf16 [M,N]
 *    (row stride ldy elements).  bf16 values are passed as `const void *` to
 *    keep this header free of CUDA headers.
 *  - All tensor pointers are DEVICE pointers owned by the caller, except where
 *    a call says "host".  The library never allocates memory; scratch memory
 *    is the caller's `workspace`.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and returns a w8a8_status.  On any error nothing has been
 *    launched.  Calls never abort the process.
 *  - Preconditions checked on the host: sizes >= 1; K % 16 == 0 (16-byte int8
 *    rows for the tensor-memory-accelerator loads); N % 8 == 0 (16-byte bf16
 *    output rows); K <= 133144 (127*127*K must fit int32); ldx, ldw >= K and
 *    multiples of 8; ldy >= N and a multiple of 8; every pointer 16-byte
 *    aligned (s_a 4-byte); the current device is sm_100.
 *  - Inputs must be finite: NaN or Inf in x or W is outside the contract.
 *  - Calls on different streams are independent and thread-safe; calls that
 *    share a workspace must be ordered by the caller.
 *  - State the library keeps: the device properties read at first use; a
 *    per-thread cache of encoded tensor maps (host memory, keyed by every
 *    value encoded into a map, so a hit equals a fresh encoding); two
 *    streams and their events per device for w8a8_linear_fused_host, made at
 *    its first call and used under a mutex; the static scratch of
 *    w8a8_linear_fused_noalloc.
 */
#ifndef W8A8_H
#define W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define W8A8_API __attribute__((visibility("default")))
#else
#define W8A8_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *w8a8_stream_t;

typedef enum {
    W8A8_OK = 0,
    W8A8_ERR_INVALID_ARG = 1,        /* NULL pointer, size < 1, ld too small */
    W8A8_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 16, N % 8, K > 133144, ld % 8 */
    W8A8_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
    W8A8_ERR_WORKSPACE = 4,          /* workspace NULL or smaller than needed */
    W8A8_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    W8A8_ERR_DEVICE_TIMEOUT = 6,     /* a bounded device-side wait gave up */
    W8A8_ERR_UNSUPPORTED_DEVICE = 7  /* current device is not sm_100 */
} w8a8_status;

/* Kernel variants, for w8a8_linear_ex / w8a8_select.  AUTO lets the selector
 * choose from (M, N, K). */
typedef enum {
    W8A8_VARIANT_AUTO = 0,
    W8A8_VARIANT_GEMV = 1,          /* M <= 16: CUDA-core int8 dot products */
    W8A8_VARIANT_GEMM_BN128 = 2,    /* tcgen05 kind::i8, 128x128 tiles */
    W8A8_VARIANT_GEMM_BN256 = 3,    /* tcgen05 kind::i8, 128x256 tiles */
    W8A8_VARIANT_GEMM_PAIR = 4,     /* tcgen05 kind::i8 on CTA pairs, 256x256 tiles */
    W8A8_VARIANT_GEMM_BN64 = 5,     /* tcgen05 kind::i8, 128x64 tiles (small M: more
                                       CTAs streaming the weights) */
    W8A8_VARIANT_GEMV_TC = 6        /* M <= 128: tcgen05 kind::i8 with the weights as
                                       the MMA's 128-row side and the activation rows
                                       (padded to 16/32/64/128) as its N side; K split
                                       among the CTAs of a cluster when tiles are few */
} w8a8_variant;

/* The selector's decision for one (M, N, K); see w8a8_select. */
typedef struct {
    int32_t variant;       /* a w8a8_variant other than AUTO */
    int32_t tile_m;        /* rows of y per tile (GEMM) or 0 */
    int32_t tile_n;        /* columns of y per tile (GEMM) or 0 */
    int32_t num_tiles;     /* GEMM tiles, or GEMV output rows of W */
    int32_t grid;          /* CTAs launched */
    int32_t waves_x100;    /* tile rounds per CTA (pair) x 100, counting the
                              K-split tail as its share of a round (GEMM), else 0 */
    int32_t split_tiles;   /* GEMM_PAIR: the last split_tiles tiles (one to two
                              waves) are shared out along K among all pairs;
                              0 = none */
    int32_t split_kblocks_per_pair; /* GEMM_PAIR with split_tiles > 0: 128-deep
                              k-blocks of that region per pair, else 0 */
    int32_t tail_tiles_nsplit; /* GEMM_PAIR: 2 when the tiles of the last,
                              partial round are cut along N into two
                              128-column tiles (one per pair); else 0 */
    int32_t quant_in_gemm_launch; /* GEMM_PAIR: 1 when w8a8_linear_fused_ex
                              with W8A8_FUSED_ONE_LAUNCH can run the per-token
                              quantization inside the GEMM launch (K <= 12288,
                              given the full workspace); GEMV: 1 when
                              w8a8_linear_fused quantizes the rows inside the
                              GEMV launch (M = 1, or M = 2 with K <= 8192;
                              no workspace needed); else 0 */
    int32_t k_split;       /* GEMV_TC: CTAs (one cluster) sharing each 128-row
                              weight tile along K, 1..8; else 0 */
} w8a8_plan;

/* Human-readable name of a status code (static string, never NULL). */
W8A8_API const char *w8a8_status_string(int status);

/*
 * Weight quantization, run once per layer at load time.
 * W bf16 [N,K] (row stride ldw) -> Wq int8 [N,K] dense, s_w fp32 [N]:
 * s_w[n] = max_k |W[n,k]| / 127, Wq = clamp(rint(W / s_w), -127, 127).
 * Wq is K-major, exactly the layout the GEMM reads (no repacking step).
 */
W8A8_API int w8a8_quantize_weights(const void *W_bf16, int64_t N, int64_t K, int64_t ldw,
                          int8_t *Wq, float *s_w, w8a8_stream_t stream);

/*
 * Weight loading from packed int32 storage, run once per layer at load time
 * (the serialized checkpoint form: "Issue 5 probe: int8 quantized DiT serve
 * paths on the RTX 3090 (24 GB)", section "Artifact (outside Git, under the
 * helper state root)": the quantized transformer is packed with
 * compressed-tensors' pack_to_int32 -- each int8 code stored as an unsigned
 * byte biased by 128, four per int32 word).  packed int32 [N, K/4] dense: word g of row n
 * holds the codes of columns 4g .. 4g+3, column 4g in the least significant
 * byte -> Wq int8 [N,K] dense, Wq[n,k] = byte - 128.  The per-channel scales
 * s_w are stored beside the packed codes and are used as they are.
 * A code of -128 (byte 0) is passed through; with such codes the GEMM is
 * exact for K <= 132104 (127 * 128 * K < 2^31).
 * Preconditions as for w8a8_quantize_weights (K % 16 == 0, both pointers
 * 16-byte aligned).
 */
W8A8_API int w8a8_unpack_int32_weights(const int32_t *packed, int64_t N, int64_t K, int8_t *Wq,
                                       w8a8_stream_t stream);

/*
 * Per-token dynamic activation quantization.
 * x bf16 [M,K] (row stride ldx) -> q int8 [M,K] dense, s_a fp32 [M].
 */
W8A8_API int w8a8_quant_act(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                   int8_t *q, float *s_a, w8a8_stream_t stream);

/*
 * Scratch bytes for (M, N, K) on a 148-SM B200: w8a8_linear_fused's int8
 * activations and their scales, one 64-bit counter per 128 rows (used by
 * the one-launch option of w8a8_linear_fused_ex), plus, when the plan shares
 * its last tiles out along K (w8a8_plan.split_tiles > 0), the int32 partial
 * sums and arrival counters of that region.  The caller need not initialize
 * it: a call that uses counters clears them on its stream first (an
 * asynchronous memset of a few KB; nothing is allocated).  A workspace
 * holding only q and s_a still works: the layer then runs without the K
 * split.  0 when the plan is the GEMV quantizing its own rows (M = 1, or
 * M = 2 with K <= 8192).
 */
W8A8_API int w8a8_workspace_size(int64_t M, int64_t N, int64_t K, size_t *bytes);

/*
 * As w8a8_workspace_size, for the plan of a given variant (w8a8_variant;
 * AUTO gives w8a8_workspace_size's answer): a caller that forces the pair
 * kernel through w8a8_linear_ex sizes its workspace here, so that the K-split
 * region of that plan fits (the automatic plan may have none).  Returns
 * W8A8_ERR_UNSUPPORTED_SHAPE where the variant cannot run (M, N, K).
 */
W8A8_API int w8a8_workspace_size_ex(int64_t M, int64_t N, int64_t K, int variant,
                                    size_t *bytes);

/*
 * int8 GEMM + fused epilogue on already-quantized activations.
 * q int8 [M,K] dense, s_a fp32 [M], Wq int8 [N,K] dense, s_w fp32 [N],
 * bias bf16 [N] or NULL -> y bf16 [M,N] (row stride ldy).
 * acc_debug: NULL, or int32 [M,N] dense; when given, the raw int32
 * accumulators are written there INSTEAD of y (y may then be NULL).
 * workspace / ws_bytes: optional (NULL / 0 allowed).  With at least
 * w8a8_workspace_size(M,N,K) bytes (16-byte aligned) the pair kernel's K-split
 * tail is used.  Its contents need no initialization: the call clears the
 * region's arrival counters on `stream` before the launch, and the counters
 * also carry a per-launch tag drawn from a random per-process start, so
 * words another launch left behind count as zero.  The workspace must not
 * be in use by other work while the call runs.  After a launch that reported
 * W8A8_ERR_DEVICE_TIMEOUT, replaying a captured graph of it on the same
 * workspace is outside the contract.
 */
W8A8_API int w8a8_linear(const int8_t *q, const float *s_a, int64_t M, int64_t K,
                const int8_t *Wq, const float *s_w, const void *bias_bf16_or_null, int64_t N,
                void *y_bf16, int64_t ldy, int32_t *acc_debug_or_null,
                void *workspace, size_t ws_bytes, w8a8_stream_t stream);

/* w8a8_linear with an explicit kernel variant (AUTO = the selector's choice).
 * GEMV requires M <= 16.  workspace as in w8a8_linear (GEMM_PAIR uses it for
 * the K-split tail when it holds w8a8_workspace_size_ex(M, N, K,
 * W8A8_VARIANT_GEMM_PAIR) bytes; NULL runs the pair kernel unsplit). */
W8A8_API int w8a8_linear_ex(const int8_t *q, const float *s_a, int64_t M, int64_t K,
                   const int8_t *Wq, const float *s_w, const void *bias_bf16_or_null, int64_t N,
                   void *y_bf16, int64_t ldy, int32_t *acc_debug_or_null,
                   int variant, void *workspace, size_t ws_bytes, w8a8_stream_t stream);

/*
 * The whole layer from bf16 activations: quantize x per token, then the int8
 * GEMM with the fused epilogue.  x bf16 [M,K] (row stride ldx) -> y bf16 [M,N].
 * q_out / s_a_out: NULL, or int8 [M,K] dense / fp32 [M] to receive the
 * intermediates (then they are used instead of workspace).
 * workspace: w8a8_workspace_size(M,N,K) bytes, 16-byte aligned (256
 * recommended).  Required: the bytes for q and s_a, unless both q_out and
 * s_a_out are given; the rest (row-block counters, K-split region) is
 * optional, see w8a8_workspace_size.  Two launches: the quantization kernel,
 * then the GEMM (or the small-M variant the selector picks) as a programmatic
 * dependent launch; one launch when the plan is the GEMV quantizing its own
 * rows (w8a8_plan.quant_in_gemm_launch on a GEMV plan).
 */
W8A8_API int w8a8_linear_fused(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                      const int8_t *Wq, const float *s_w, const void *bias_bf16_or_null, int64_t N,
                      void *y_bf16, int64_t ldy, int8_t *q_out_or_null, float *s_a_out_or_null,
                      void *workspace, size_t ws_bytes, w8a8_stream_t stream);

/* Options of w8a8_linear_fused_ex. */
#define W8A8_FUSED_ONE_LAUNCH 1  /* quantize inside the GEMM launch when the plan
                                    allows it (w8a8_plan.quant_in_gemm_launch) */

/*
 * w8a8_linear_fused with options.  W8A8_FUSED_ONE_LAUNCH: on a CTA-pair plan
 * with quant_in_gemm_launch set (K <= 12288) and a workspace holding the
 * row-block counters (w8a8_workspace_size bytes), the pair kernel quantizes x
 * itself: the epilogue warps of all CTAs quantize the rows in row-block
 * order -- the rows the first round of tiles reads through the not yet used
 * operand ring (bulk copies), later rows through registers while the first
 * tiles' MMAs run, taking the epilogue of any finished tile between passes --
 * and each producer waits only for the 128-row block it loads.  The counters
 * are cleared on the stream before the launch, so the call may be captured in
 * a CUDA graph.  One launch instead of two, bit-identical results; on a B200
 * it measured slower than the two launches (QKV 96 vs 89 us: the quantization
 * traffic during the first rounds slows the GEMM more than the overlap
 * saves), so it is not the default.  Otherwise the call is exactly
 * w8a8_linear_fused.  Unknown option bits: W8A8_ERR_INVALID_ARG.
 */
W8A8_API int w8a8_linear_fused_ex(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                      const int8_t *Wq, const float *s_w, const void *bias_bf16_or_null, int64_t N,
                      void *y_bf16, int64_t ldy, int8_t *q_out_or_null, float *s_a_out_or_null,
                      void *workspace, size_t ws_bytes, int options, w8a8_stream_t stream);

/*
 * End-to-end form of w8a8_linear_fused for callers holding HOST buffers:
 * enqueues on `stream` the copy x_host -> x_dev, the layer, and the copy
 * y_dev -> y_host.  x_host: host bf16 [M,K] dense (pinned memory gives
 * asynchronous copies); y_host: host bf16 [M,N] dense.  x_dev [M,K] dense and
 * y_dev [M,N] dense are caller-owned device staging buffers; Wq, s_w, bias and
 * workspace are device pointers as in w8a8_linear_fused.  The call returns
 * after enqueueing; synchronize `stream` before reading y_host.
 * The rows go in up to 8 chunks (at least 256 rows each): chunk c is copied
 * in on `stream`, computed on an internal stream of the library and copied
 * out on a second internal one, so that the two copy directions and the
 * layer overlap; the internal streams fork from and join back into `stream`
 * through events (the call may be captured in a CUDA graph).  The result is
 * identical to one layer call over all rows.  Calls on one device take a
 * library mutex while they enqueue.
 */
W8A8_API int w8a8_linear_fused_host(const void *x_host, int64_t M, int64_t K,
                           const int8_t *Wq, const float *s_w, const void *bias_bf16_or_null,
                           int64_t N, void *y_host, void *x_dev, void *y_dev,
                           void *workspace, size_t ws_bytes, w8a8_stream_t stream);

/*
 * The weight-only variant (W8A16): int8 weights with per-output-channel fp32
 * scales, bf16 activations used as they are ("Issue 5 probe: int8 quantized
 * DiT serve paths on the RTX 3090 (24 GB)", section "Round one: int8
 * weight-only via compressed-tensors").  x bf16 [M,K] (row stride ldx),
 * Wq int8 [N,K] dense, s_w fp32 [N], bias bf16 [N] or NULL -> y bf16 [M,N]
 * (row stride ldy):  y = bf16( (sum_k x[m,k] * Wq[n,k]) * s_w[n] + bias[n] ),
 * the sum accumulated in fp32 by the tensor cores (order unspecified; each
 * product is exact), the scale and bias applied once as rounded fp32
 * operations.  The int8 weights are widened to bf16 inside the kernel; no
 * workspace.  Preconditions as for w8a8_linear_fused.
 */
W8A8_API int w8a16_linear(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                          const int8_t *Wq, const float *s_w, const void *bias_bf16_or_null,
                          int64_t N, void *y_bf16, int64_t ldy, w8a8_stream_t stream);

/*
 * Host-only: the selector's plan for (M, N, K) on a device with num_sms SMs
 * (148 on B200).  Pure function of its arguments; needs no GPU.
 */
W8A8_API int w8a8_select(int64_t M, int64_t N, int64_t K, int32_t num_sms, int variant,
                w8a8_plan *plan);

/*
 * Synchronizes `stream`, then reads and clears the library's device error
 * word.  Returns W8A8_ERR_DEVICE_TIMEOUT if a bounded device-side wait (an
 * mbarrier wait in a pipelined kernel) gave up since the last call, W8A8_OK
 * otherwise, or W8A8_ERR_CUDA if the synchronization itself failed.
 */
W8A8_API int w8a8_last_device_error(w8a8_stream_t stream);

/*
 * Self-test of the bounded device-side wait: launches one block that waits,
 * with a limit of limit_ns nanoseconds (1e3 .. 1e10), on an mbarrier that
 * nothing ever arrives on.  The wait gives up, records the timeout in the
 * device error word and the kernel returns; a following
 * w8a8_last_device_error() reports W8A8_ERR_DEVICE_TIMEOUT.
 */
W8A8_API int w8a8_selftest_bounded_wait(int64_t limit_ns, w8a8_stream_t stream);

/*
 * w8a8_linear_fused for callers that cannot allocate device memory and so
 * cannot supply a workspace: for example a plugin running inside a serving
 * runtime or framework that reserves all device memory at start-up and
 * forbids any later allocation, or code held to a fixed memory budget.  It
 * computes exactly what w8a8_linear_fused computes (same arguments minus
 * q_out / s_a_out / workspace), but keeps the int8 activations and their
 * scales in a scratch area compiled into the library: a static device array
 * of 16 MiB for q plus 64 KiB for the row scales and 4 KiB of counters.  Every GPU that loads this
 * library holds that array until the process exits.
 *
 * Limits: M * K <= 16 MiB (16777216) and M <= 16384; a larger call returns
 * W8A8_ERR_WORKSPACE and launches nothing.  It never calls cudaMalloc,
 * cudaFree or any allocating routine.
 *
 * Set-up: the first call on each device looks up the device address of the
 * scratch array (with that device current) and caches it; make that first
 * call before any stream capture begins.
 *
 * Sharing: all calls on a device use the same scratch array, which keeps
 * whatever the previous call left there.  Each call writes the scratch it
 * reads before reading it, so nothing needs to start at zero; but calls whose
 * execution overlaps on the GPU (different streams, or threads that do not
 * order their calls) race on the array -- the caller must serialize them.
 *
 * The source pages describe no counterpart to this entry point.
 */
W8A8_API int w8a8_linear_fused_noalloc(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                                       const int8_t *Wq, const float *s_w,
                                       const void *bias_bf16_or_null, int64_t N, void *y_bf16,
                                       int64_t ldy, w8a8_stream_t stream);

/*
 * Self-test of the division-free quantization step the kernels use: on the
 * GPU, for every positive finite bf16 row maximum a and every bf16 value x
 * with |x| <= a, compares the code the fast step produces -- in its scalar
 * form and in the packed fp32x2 form -- against clamp(rint(x / s), -127, 127)
 * computed with an IEEE division, s = a / 127.
 * counts_dev: device array of 2 unsigned 64-bit integers, zeroed by the call;
 * receives [0] the number of (x, a) pairs checked on the fast step and [1] the
 * number of pairs whose code differs (expected 0).  About 10^9 pairs; takes
 * on the order of a second.
 */
W8A8_API int w8a8_selftest_quant_exhaustive(unsigned long long *counts_dev, w8a8_stream_t stream);

/*
 * Measurement of the device's int8 tensor-core ceiling, the denominator of
 * the GEMM's roofline: `pairs` CTA pairs (1 .. SMs / 2) each issue
 * 4 * iterations tcgen05.mma.cta_group::2.kind::i8 instructions (M = 256,
 * N = 256, K = 32: the GEMM's own instruction) from operands held in shared
 * memory, with no global-memory traffic.  The launch performs
 * pairs * iterations * 16,777,216 int8 operations; the caller times it
 * (CUDA events on `stream`).  iterations: 1 .. 500000 (a fraction of a
 * second), else W8A8_ERR_INVALID_ARG.  Asynchronous; nothing is allocated.
 */
W8A8_API int w8a8_bench_mma_i8_peak(int64_t iterations, int32_t pairs, w8a8_stream_t stream);

/*
 * Test support: the launch tag that the next call using arrival counters
 * (a K-split tail, or the one-launch option of w8a8_linear_fused_ex) will
 * draw, in its low 56 bits (the one-launch option uses the low 48).  A test
 * can plant a counter word carrying this tag in a workspace and check that
 * the call still computes the right result.  Host-only; needs no GPU.
 */
W8A8_API int w8a8_debug_peek_tag(uint64_t *tag);

/* Library version string, e.g. "w8a8 1.0 sm_100a". */
W8A8_API const char *w8a8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H */
