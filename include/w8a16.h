/*
 * w8a16.h -- C ABI of libw8a16.so, a W8A16 (int8 weight, fp16 activation)
 * linear layer for NVIDIA B200 (sm_100a).
 *
 * The operation (TPU-MLIR ChatGLM2 W8A16 article, section 2 "quantization
 * scheme" and section 4 "backend performance", steps 1-5; LightSeq 2020
 * slides "quantization: clipping + symmetric"):
 *
 *   quantize   s_n = fp16_rne( fp32(max_k |W[k,n]|) / 127 )          (per n)
 *              q[k,n] = clamp( rne( W[k,n] / float(s_n) ), -127, 127 )
 *              (s_n == 0 for an all-zero column, and then q = 0)
 *   linear     Y[m,n] = fp16_rne( s_n * sum_k X[m,k] * q[k,n] + bias_n )
 *              with the sum accumulated in fp32.
 *
 * The page dequantizes the weight (cast int8 -> F16, multiply by the scale)
 * before the matmul; here the per-channel scale is applied once per output
 * element after the sum, which is the same value in exact arithmetic.
 *
 * Conventions for every entry point
 *  - Tensors are dense row-major.  W and q are [K, N] (K = input features,
 *    the reduction dimension; N = output features / channels, contiguous).
 *    X is [M, K], Y is [M, N], scales and bias are [N].
 *  - fp16 buffers are passed as uint16_t* holding IEEE binary16 bit patterns.
 *  - Every pointer except `bias` (nullable) and host-side outputs is a
 *    DEVICE pointer on the current CUDA device and must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work on that stream; they never allocate
 *    device memory and never synchronize (except the diagnostic
 *    w8_device_status).  The caller owns every buffer.
 *  - Invalid arguments are detected on the host before anything is launched
 *    and reported by a negative w8_status; nothing is written then.  A
 *    launch failure is W8_ERR_CUDA.  Errors raised while a kernel runs
 *    surface at the caller's next synchronization.
 *  - Every wait inside a kernel is bounded (about one second); a wait that
 *    runs out records a status word readable with w8_device_status() and the
 *    kernel returns early instead of hanging.
 *  - The library keeps no per-call state.  It is safe to call from several
 *    host threads on different streams, provided calls that share a
 *    workspace do not overlap on the device.
 */
#ifndef W8A16_H
#define W8A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W8_OK = 0,
    W8_ERR_NULL = -1,       /* a required pointer is NULL */
    W8_ERR_SHAPE = -2,      /* a size is out of range or not a multiple of 8 */
    W8_ERR_ALIGN = -3,      /* a pointer is not 16-byte aligned */
    W8_ERR_DTYPE = -4,      /* unknown w8_dtype */
    W8_ERR_WORKSPACE = -5,  /* workspace missing or smaller than required */
    W8_ERR_CUDA = -6,       /* a CUDA runtime call or launch failed */
    W8_ERR_TIMEOUT = -7,    /* a bounded device wait ran out (see w8_device_status) */
    W8_ERR_ALIAS = -8,      /* the output overlaps an input */
    W8_ERR_DEVICE = -9,     /* the current device is not sm_100 */
    W8_ERR_LIMIT = -10      /* a size exceeds the fixed scratch of
                               w8a16_linear_decode_static */
} w8_status;

typedef enum { W8_F32 = 0, W8_F16 = 1 } w8_dtype;

/* Tile geometry of the packed weight layout (see w8_prepack). */
#define W8_TILE_N 128
#define W8_TILE_K 64
#define W8_TILE_BYTES (W8_TILE_N * W8_TILE_K)

/*
 * w8_quantize_per_channel -- per-output-channel symmetric int8 quantization
 * (the weight quantizer of the TPU-MLIR article, section 3: a 2-D weight
 * R = 4096 x 27392 becomes int8 plus an F16 scale per channel).
 *
 *   W       [K, N] input weight, fp32 or fp16 as given by w_dtype (W8_F32 /
 *           W8_F16); fp16 is widened exactly to fp32 first.
 *   q       [K, N] int8 output codes in [-127, 127].
 *   scales  [N] fp16 output scales.
 *   K >= 1; N >= 0 with N % 8 == 0 (N == 0 is a no-op and the pointers
 *   may then be NULL).
 * The result is bit-exact: fp32 divisions are IEEE round-to-nearest, the
 * fp32 -> fp16 and fp32 -> int conversions round half to even, fp16
 * subnormal scales are kept.  Inputs must be finite.
 * Errors: W8_ERR_NULL, W8_ERR_SHAPE, W8_ERR_ALIGN, W8_ERR_DTYPE,
 *         W8_ERR_ALIAS (q overlaps W), W8_ERR_CUDA.
 */
int w8_quantize_per_channel(const void *W, int w_dtype, int64_t K, int64_t N,
                            int8_t *q, uint16_t *scales, void *stream);

/*
 * w8_quantize_per_channel_asym -- per-output-channel ASYMMETRIC (affine)
 * int8 quantization: the variant the LightSeq 2020 slides compare with the
 * symmetric one (slide "quantization: clipping + symmetric", where a value
 * is (i - z) S), with the range, scale and zero point of the
 * integer-arithmetic quantization paper those slides cite (arXiv
 * 1712.05877, section 2).  For each channel n:
 *   lo = min(0, min_k W[k,n]),  hi = max(0, max_k W[k,n])
 *   S_n = fp16_rne( fp32(hi - lo) / 255 )
 *   z_n = clamp( rne( -128 - lo / S_n ), -128, 127 )
 *   q[k,n] = clamp( rne( W[k,n] / S_n ) + z_n, -128, 127 )
 * (IEEE fp32 operations, S_n widened from fp16; S_n = 0 gives z_n = 0 and
 * q = 0).  A weight is dequantized as (q - z_n) S_n; 0 is exact.
 *   zeros   [N] int8 output zero points.
 * Other arguments, exactness and errors as w8_quantize_per_channel (zeros
 * must not overlap W, q or scales).
 */
/*
 * w8_quantize_per_channel_batched -- w8_quantize_per_channel for `count`
 * weights in as few launches as possible (up to 64 weights per launch: the
 * launch's clusters walk all their column panels), e.g. every weight of a
 * model at load time (BERT-base: 48).  The arrays are host arrays of
 * length count: W[i] [K[i], N[i]] (all of dtype w_dtype), q[i] [K[i], N[i]]
 * int8 and scales[i] [N[i]] fp16 device pointers.  The result equals
 * `count` separate w8_quantize_per_channel calls bit for bit.  No output
 * may overlap any weight or any other output.  count == 0 and entries with
 * N[i] == 0 are no-ops.  Errors as w8_quantize_per_channel.
 */
int w8_quantize_per_channel_batched(int count, const void *const *W, int w_dtype, const int64_t *K,
                                    const int64_t *N, int8_t *const *q, uint16_t *const *scales, void *stream);

int w8_quantize_per_channel_asym(const void *W, int w_dtype, int64_t K, int64_t N, int8_t *q,
                                 uint16_t *scales, int8_t *zeros, void *stream);

/*
 * w8_quantize_per_channel_clip -- symmetric int8 quantization with a
 * clipped bound: the "fixed range clip" and "percentage clip" calibrations
 * the LightSeq 2020 slides evaluate against max|W| (slide "quantization:
 * clipping + symmetric").  Per channel n the bound put on level 127 is
 *   W8_CLIP_FIXED:      bound_n = min( max_k |W[k,n]|, c ),  c = (float)clip_param >= 0
 *   W8_CLIP_PERCENTILE: bound_n = the r-th smallest |W[k,n]|,
 *                       r = clamp( ceil(p K), 1, K ) in IEEE double, p = clip_param in (0, 1]
 * and then s_n = fp16_rne( fp32(bound_n) / 127 ), q = clamp( rne(W / s_n),
 * -127, 127 ) as in w8_quantize_per_channel: weights beyond the bound land on
 * +-127.  The output is in the symmetric format (w8_prepack, w8a16_linear).
 * c = +inf and p = 1 give w8_quantize_per_channel's result bit for bit.
 * The percentile form finds the order statistic by radix selection on the
 * bit patterns of |w| (digits of 9, 8, 7 and 7 bits; a column's last
 * candidates, at most 768, are selected in shared memory) and streams W
 * three times for usual weights, at most five times (the passes after the
 * first mostly from L2).
 * Errors: as w8_quantize_per_channel; W8_ERR_SHAPE also for a clip_param
 * out of range, W8_ERR_DTYPE for an unknown clip_mode.
 */
typedef enum { W8_CLIP_FIXED = 0, W8_CLIP_PERCENTILE = 1 } w8_clip_mode;

int w8_quantize_per_channel_clip(const void *W, int w_dtype, int64_t K, int64_t N, int clip_mode,
                                 double clip_param, int8_t *q, uint16_t *scales, void *stream);

/*
 * Outlier split -- the observation of the GOBO page (a few large weights
 * inflate the scale; keep them apart, exactly) applied to W8A16.  Per channel
 * n, with bound_n = the r-th smallest |W[k,n]|, r = clamp(ceil(p K), 1, K) in
 * IEEE double (the percentage clip's bound):
 *   outliers: every k with |W[k,n]| > bound_n, kept as (k, fp16_rne(W[k,n]))
 *             in increasing k, with code 0;
 *   the rest: s_n = fp16_rne(fp32(bound_n)/127), q = clamp(rne(W/s_n), -127, 127).
 * At most cap = K - r weights of a channel are outliers.  The side list has
 * cap slots per channel: o_count [N] int32, o_rows [N][cap] int32, o_vals
 * [N][cap] fp16; unused slots are 0.  p = 1 gives cap = 0 and the plain
 * symmetric quantizer.
 *
 * w8_outlier_capacity -- cap for (K, p); 0 for arguments out of range.
 * w8_quantize_per_channel_outliers -- the split above.  0 < p <= 1; cap must
 *   not exceed 64 (W8_ERR_LIMIT), i.e. p >= 1 - 64/K roughly; o_rows and
 *   o_vals may be NULL when cap == 0.  Bit-exact; other arguments and errors
 *   as w8_quantize_per_channel.
 * w8a16_linear_outliers -- Y = X . dequant(q) + X . outliers (+ bias):
 *   Y[m,n] = s_n sum_k X[m,k] q[k,n] + sum_j X[m, rows_j] vals_j + bias_n,
 *   the outlier products added in fp32 before the single rounding to fp16.
 *   packed/scales from w8_prepack of the split's q; o_cap the cap it was made
 *   with.  The workspace must hold w8a16_linear_outliers_workspace_bytes(M,
 *   K, N) bytes (for M > 64 it also holds X transposed, written by the call).
 *   Accuracy, stream ordering and errors as w8a16_linear; W8_ERR_LIMIT for
 *   o_cap > 64.
 */
size_t w8_outlier_capacity(int64_t K, double p);
int w8_quantize_per_channel_outliers(const void *W, int w_dtype, int64_t K, int64_t N, double p, int8_t *q,
                                     uint16_t *scales, int32_t *o_count, int32_t *o_rows, uint16_t *o_vals,
                                     void *stream);
size_t w8a16_linear_outliers_workspace_bytes(int64_t M, int64_t K, int64_t N);
int w8a16_linear_outliers(const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                          const int32_t *o_count, const int32_t *o_rows, const uint16_t *o_vals, int64_t o_cap,
                          const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * w8_prepacked_bytes -- size of the packed weight for a [K, N] q:
 * ceil(N/128) * ceil(K/64) * 8192 bytes (== K*N when K % 64 == 0 and
 * N % 128 == 0).  Returns 0 for K < 1 or N < 1.
 */
size_t w8_prepacked_bytes(int64_t K, int64_t N);

/*
 * w8_prepack -- reorder q [K, N] into the tiled layout both linear kernels
 * stream (done once per weight, off the per-call path).
 *
 * Layout: tiles of 128 output channels x 64 input features, 8192 bytes
 * each.  Tile (b, kb) -- channels n in [128b, 128b+128), features k in
 * [64kb, 64kb+64) -- starts at byte (b * ceil(K/64) + kb) * 8192, so the
 * tiles of one channel block are contiguous along K.  Inside a tile, row r
 * (channel n = 128b + r) takes bytes [64r, 64r + 64); its 16-byte chunk c
 * (features 64kb + 16c ... +15, in natural order) is stored at chunk slot
 * c XOR ((r >> 1) & 3).  Each byte holds q + 128 (offset binary, i.e.
 * q XOR 0x80).  Positions with k >= K or n >= N hold 0x80 (q = 0).
 *   q       [K, N] int8 input; packed: w8_prepacked_bytes(K, N) output bytes.
 *   K >= 1, N >= 1, N % 8 == 0.
 * Errors: W8_ERR_NULL, W8_ERR_SHAPE, W8_ERR_ALIGN, W8_ERR_ALIAS, W8_ERR_CUDA.
 */
int w8_prepack(const int8_t *q, int64_t K, int64_t N, uint8_t *packed, void *stream);

/*
 * w8_unpack -- inverse of w8_prepack (packed -> q [K, N]); for tests and
 * inspection.  Same argument rules as w8_prepack.
 */
int w8_unpack(const uint8_t *packed, int64_t K, int64_t N, int8_t *q, void *stream);

/*
 * w8a16_workspace_bytes -- device scratch w8a16_linear needs for this shape
 * on the CURRENT device (it depends on the SM count); 0 only for an empty
 * shape or when no device is usable.  Both kernels split the reduction over
 * K across thread blocks where the output alone would not fill the GPU and
 * need room for fp32 partial sums (a fixed 256 KB per multiprocessor, the
 * same for every shape) plus int32 counters (the larger of one per 128
 * output channels and two per multiprocessor).
 */
size_t w8a16_workspace_bytes(int64_t M, int64_t K, int64_t N);

/*
 * w8a16_linear -- Y = X . dequant(packed, scales) (+ bias).
 *
 *   X          [M, K] fp16 activations.
 *   packed     w8_prepack output for the [K, N] weight.
 *   scales     [N] fp16 per-channel scales (w8_quantize_per_channel output).
 *   bias       [N] fp16 or NULL.
 *   Y          [M, N] fp16 output; must not overlap X, packed or scales.
 *   M >= 0 (0 is a no-op; X and Y may then be NULL); K >= 1 with
 *   K % 8 == 0; N >= 1 with N % 8 == 0.  For M <= 64 the number of 8 KB
 *   weight tiles times (multiprocessors + 1) must stay below 2^32 (weights
 *   up to about 230 GB on a B200), else W8_ERR_SHAPE.
 * Stream ordering: both kernels are launched with programmatic stream
 *   serialization, so their prologue (and, for M <= 64, an L2 prefetch of
 *   the first weight tiles) may overlap the previous kernel in the stream;
 *   they read X, the weights, scales and bias and write Y, the workspace and
 *   the counters only after that kernel has completed, as with an ordinary
 *   launch.
 *   workspace  device scratch of at least w8a16_workspace_bytes(M, K, N)
 *              bytes (may be NULL when that is 0).  It must be all zero
 *              before its first use; every call that completes leaves it
 *              ready for the next one, whatever the next call's shape.
 *              Calls sharing one workspace must not run concurrently on
 *              the device.  After a call whose device wait ran out (see
 *              w8_device_status) the workspace must be zeroed again.
 * Kernel choice (internal): M <= 64 streams the weight once with a
 * split-K kernel on the legacy tensor-core path (HBM-bound up to about 32
 * tokens): an even split of all tiles over the SMs, or, up to 16 tokens on
 * weights with few 128-channel blocks, one thread-block cluster per block
 * whose CTAs add their parts in distributed shared memory (this form does
 * not touch the workspace); larger M runs a tcgen05 tensor-core kernel on
 * pairs of SMs (clusters of two thread blocks) with the widened weight
 * tile held in tensor memory, whole 256 x 256 output tiles per pair where
 * they fill the GPU and a K split over all pairs for the tiles that do
 * not.  Every form adds a tile's partial sums in a fixed order: results are
 * the same on every call.
 * Accuracy: |Y - Y_exact| <= 2^-9 |Y_exact| + 1e-3 rms(Y_exact).
 * Errors: W8_ERR_NULL, W8_ERR_SHAPE, W8_ERR_ALIGN, W8_ERR_WORKSPACE,
 *         W8_ERR_ALIAS, W8_ERR_DEVICE, W8_ERR_CUDA.
 */
int w8a16_linear(const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                 const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * w8a16_linear_asym -- Y = X . ((q - z) o S) (+ bias) for codes from
 * w8_quantize_per_channel_asym: Y[m,n] = S_n sum_k X[m,k] (q[k,n] - z_n)
 * + bias_n, the expansion of the slides' (i - z) S product with the
 * activation kept in fp16.  The kernels widen each code to q - z_n, exact
 * in fp16 (|q - z| <= 255), so the arithmetic and the accuracy bound are
 * those of w8a16_linear.
 *   zeros   [N] int8 zero points (must not overlap Y).
 * Every other argument, the workspace and the errors as w8a16_linear.
 */
int w8a16_linear_asym(const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                      const int8_t *zeros, const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K,
                      int64_t N, void *workspace, size_t workspace_bytes, void *stream);

/*
 * w8a16_linear_decode_static -- the decode path of w8a16_linear (M <= 16)
 * without a caller-provided workspace.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory, such
 * as an operator plugged into a host framework whose fixed signature has no
 * workspace argument, or a serving loop whose device memory is planned up
 * front by another allocator and where a cudaMalloc would synchronize the
 * device.  Their inputs and outputs are still passed in.
 *
 * The split-K scratch (fp32 partial sums and per-block counters) lives in
 * one array of W8_STATIC_SCRATCH_BYTES bytes of static device memory inside
 * this library; every GPU that loads the library holds it until the
 * process exits.  Nothing is allocated or freed by the call.
 *
 *   The kernel, its split of the weight and the order in which partial
 *   sums are added are those w8a16_linear takes for the same shape, so the
 *   two return the same bits; where w8a16_linear's form needs no workspace,
 *   this one touches no scratch either.
 *   Arguments and results as for w8a16_linear, with these limits:
 *   1 <= M <= 16 (M == 0 is a no-op), N <= W8_STATIC_MAX_N, and the device
 *   has at most W8_STATIC_MAX_SMS multiprocessors.  Beyond them the call
 *   returns W8_ERR_LIMIT before anything is launched.
 *   Each call first clears the counters it uses (cudaMemsetAsync on
 *   `stream`), so leftovers of an earlier call, finished or not, do no harm.
 *   All calls share the one array: calls that can overlap on the GPU (on
 *   different streams, or from different host threads) race and must be
 *   ordered by the caller.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   outside any stream capture.
 * Errors: those of w8a16_linear except W8_ERR_WORKSPACE, plus W8_ERR_LIMIT.
 */
#define W8_STATIC_MAX_SMS 160
#define W8_STATIC_MAX_N (1 << 20)
#define W8_STATIC_SCRATCH_BYTES (2 * W8_STATIC_MAX_SMS * 8192 + (W8_STATIC_MAX_N / 128) * 4)
int w8a16_linear_decode_static(const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                               const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N,
                               void *stream);

/* w8_error_string -- static text for a w8_status value. */
const char *w8_error_string(int status);

/*
 * w8_device_status -- diagnostic: synchronizes `stream`, then reads and
 * clears the device status word of the current device into *out.  0 means
 * no kernel gave up a wait; otherwise bit 0 is set and bits 8..15 name the
 * wait site.  Returns W8_OK, W8_ERR_NULL or W8_ERR_CUDA.
 */
int w8_device_status(void *stream, uint32_t *out);

/*
 * w8_test_bounded_wait -- self-test of the bounded-wait machinery: launches
 * one thread that waits on a barrier nothing will complete, with the given
 * limit in nanoseconds (1e3 .. 5e9); the wait gives up, records site 0xEE in
 * the device status word and the kernel returns.  Used by the tests to
 * check that a wait that runs out ends the kernel cleanly.
 */
int w8_test_bounded_wait(uint64_t limit_ns, void *stream);

/*
 * w8_test_set_decode_helper_delay -- test hook for the decode kernel's
 * split-K bookkeeping on the current device: until set back to 0, each CTA
 * waits `delay_ns` (0 .. 1e6) before counting the partial sum it publishes
 * for its first channel block.  That forces the rarely taken paths -- the
 * previous CTA finishing the shared block through the general last-arriver
 * path, and a CTA finishing its first block after its own stream -- whose
 * results must equal the normal ones bit for bit.  Not for production use
 * (it slows every decode call).  Synchronous; returns W8_OK, W8_ERR_SHAPE
 * (delay out of range) or W8_ERR_CUDA.
 */
int w8_test_set_decode_helper_delay(uint64_t delay_ns);

/* w8_version -- ABI version of this header (major * 100 + minor). */
int w8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W8A16_H */
