/*
 * bitlinear.h -- C ABI of libbitlinear.so, the B200 (sm_100a) ternary BitLinear
 * mixed-precision matmul (BitNet b1.58, I2_S-style "int2 with scale").
 *
 * The path, per linear layer with latent weights W[M,K] (row-major, torch
 * nn.Linear [out_features, in_features]) and activations x[N,K]:
 *
 *   offline   alpha = mean|W| (fp32, exact sum, rounded once),
 *             c = clamp(round_half_even(W/alpha), -1, 1), packed 2 bits/weight
 *   per step  amax_n = max_k|x[n,k]|, q = clamp(round_half_even(x * (127/amax_n)))
 *             acc[n,m] = sum_k c[m,k] q[n,k]   (int32)
 *             y[n,m]   = (float)acc * (alpha * (amax_n / 127))
 *
 * Sources: "Bitnet.cpp: Efficient Edge Inference for Ternary LLMs" reading
 * notes -- section 1.1 (weights in {-1,0,1}), section 2.3 (I2_S: ternary
 * weights with a scale, int8 activations, 2.0 bits per weight, lossless),
 * section 4.1 (MAD-based int8 multiply-add; lossless-inference conditions);
 * FairyFuse article, "fused kernel design" (unpack and accumulate in one pass
 * over bit-packed codes, no intermediate writes).
 *
 * Packed weight layout ("I2_S-style", defined by this library):
 *   row m occupies WP(K) = 4*ceil(K/64) little-endian uint32 words, rows
 *   contiguous: K/16 words (K/4 bytes, exactly 2.0 bits per weight) when K is
 *   a multiple of 64, otherwise padded to the next 16-byte boundary;
 *   weight k lives in word k/16 of its row at bit 8*(k%4) + 2*((k%16)/4);
 *   the 2-bit field holds c+1 (0 -> -1, 1 -> 0, 2 -> +1); 3 is never written;
 *   padding fields past K hold 01 (code 0).
 *   So (word >> 2j) & 0x03030303 gives, one per byte, the fields of weights
 *   16*(k/16)+4j .. +3 in k order.
 *
 * Conventions for every entry point:
 *   - Ownership: the caller owns every buffer.  The library allocates no
 *     device or host memory and keeps no per-call state.
 *   - Pointers are DEVICE pointers unless stated otherwise.  Array pointers
 *     (W, packed, x, xq, y, acc, workspace) must be 16-byte aligned; the
 *     scalar-per-token pointers (alpha, amax, xsum) 4-byte aligned.
 *   - Shapes: K must be a positive multiple of 16 and at most 131072; any
 *     M >= 1; M*K <= 2^40.  N = 0 is a no-op.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream).  Argument errors are returned synchronously before anything is
 *     launched; a failed launch returns BITLINEAR_ERR_CUDA.
 *   - Activations q are int8 [N,K] row-major; outputs y are fp32 [N,M]
 *     row-major (token-major); the optional acc is int32 [N,M].
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BITLINEAR_API __attribute__((visibility("default")))
#else
#define BITLINEAR_API
#endif

/* ABI-identical to cudaStream_t. */
typedef struct CUstream_st* bitlinear_stream_t;

typedef enum {
    BITLINEAR_OK = 0,
    BITLINEAR_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size */
    BITLINEAR_ERR_UNSUPPORTED_SHAPE = 2, /* K % 16, N range, size limits */
    BITLINEAR_ERR_MISALIGNED = 3,        /* pointer not 16-byte aligned */
    BITLINEAR_ERR_WORKSPACE = 4,         /* workspace NULL or smaller than required */
    BITLINEAR_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    BITLINEAR_ERR_DEVICE_TIMEOUT = 6,    /* a kernel gave up a bounded wait */
    BITLINEAR_ERR_NONFINITE = 7          /* packed weights held inf or NaN */
} bitlinear_status;

/* Static, human-readable name of a status code.  Never NULL. */
BITLINEAR_API const char* bitlinear_status_string(int status);

/* Library ABI version (major*100 + minor). */
BITLINEAR_API int bitlinear_version(void);

/* ---------------------------------------------------------------- weights */

/* Bytes of device workspace bitlinear_pack_weights needs (exponent bins and a
 * flag word); the contents need not be initialised. */
BITLINEAR_API size_t bitlinear_pack_workspace_bytes(int64_t M, int64_t K);

/*
 * Absmean-ternarise and pack one weight tensor (reading notes section 1.1 and
 * 2.3; scale rule as in BitNet b1.58, alpha = mean|W|).
 *   W        fp32 [M,K] latent weights (device, read only)
 *   packed   uint32 [M, WP(K)] output in the layout above (M*K/4 bytes when
 *            K is a multiple of 64)
 *   alpha    fp32 [1] output: mean|W| rounded to nearest-even once, from an
 *            exact, order-independent sum; 0 when W is all zero (every code 0)
 *   workspace, workspace_bytes: scratch of bitlinear_pack_workspace_bytes()
 * If W holds inf or NaN, *alpha is written as NaN, every code is 0, and the
 * device error word records it: a later bitlinear_device_error() reports
 * BITLINEAR_ERR_NONFINITE (the call itself cannot know without waiting for
 * the device, and it returns before the kernels run).
 * Tie rule: |W/alpha| == 0.5 exactly gives code 0 (round half to even).
 */
BITLINEAR_API bitlinear_status bitlinear_pack_weights(const float* W, int64_t M, int64_t K,
                                        uint32_t* packed, float* alpha,
                                        void* workspace, size_t workspace_bytes,
                                        bitlinear_stream_t stream);

/* ------------------------------------------------------------ activations */

/*
 * Per-token absmax int8 quantisation (reading notes section 2.3: int8
 * activations; one scale per token row).
 *   x     fp32 [N,K] (device, read only)
 *   xq    int8 [N,K] output: clamp(round_half_even(x * (127/amax)), -128, 127)
 *   amax  fp32 [N] output: max_k |x[n,k]| (exact)
 *   xsum  int32 [N] output sum_k xq[n,k], or NULL to skip it
 * A token with amax == 0 gets xq = 0.  If 127/amax overflows to inf, +-inf
 * products clamp to 127/-128 and 0*inf is taken as 0.
 */
BITLINEAR_API bitlinear_status bitlinear_quant_act(const float* x, int64_t N, int64_t K,
                                     int8_t* xq, float* amax, int32_t* xsum,
                                     bitlinear_stream_t stream);

/*
 * Per-tensor variant of bitlinear_quant_act: one absmax over the whole x
 * [N,K], as in the reading notes' I2_S setting (section 2.3 "technical
 * details", section 4.1: per-tensor int8 activations).  Every amax[n] receives
 * that one maximum and every element uses s = 127/amax; the results feed
 * bitlinear_gemv / bitlinear_gemm unchanged.  At N = 1 it equals the
 * per-token call.
 *   workspace: device scratch of bitlinear_quant_act_per_tensor_workspace_bytes()
 *   bytes (16-byte aligned, contents need not be initialised; it is cleared on
 *   the stream).  Two launches.
 */
BITLINEAR_API size_t bitlinear_quant_act_per_tensor_workspace_bytes(void);
BITLINEAR_API bitlinear_status bitlinear_quant_act_per_tensor(const float* x, int64_t N, int64_t K,
                                                              int8_t* xq, float* amax,
                                                              int32_t* xsum, void* workspace,
                                                              size_t workspace_bytes,
                                                              bitlinear_stream_t stream);

/* One activation matrix of a grouped quantisation call (same conventions and
 * results as bitlinear_quant_act, per matrix). */
typedef struct {
    const float* x;           /* [N, K] fp32 */
    int64_t N;
    int64_t K;
    int8_t* xq;               /* [N, K] output */
    float* amax;              /* [N] output */
    int32_t* xsum;            /* [N] output, or NULL */
} bitlinear_act;

/*
 * Quantise several activation matrices (e.g. every layer input of a decode
 * step) in one launch per 64 matrices.  `acts` is a HOST array of `count`
 * entries, read during the call only.
 */
BITLINEAR_API bitlinear_status bitlinear_quant_act_grouped(const bitlinear_act* acts,
                                                           int64_t count,
                                                           bitlinear_stream_t stream);

/* ----------------------------------------------------------------- matmul */

/*
 * Decode GEMV, 1 <= N <= 16 tokens, on the CUDA cores: streams the packed
 * weights once, accumulates the ternary x int8 products in int32 and fuses
 * the rescale (reading notes section 4.1 "MAD-based"; FairyFuse "fused kernel
 * design").
 *   packed, alpha   from bitlinear_pack_weights (alpha is a device pointer)
 *   xq, amax, xsum  from bitlinear_quant_act (xsum is required here)
 *   y    fp32 [N,M] output: (float)acc * (alpha * (amax[n]/127))
 *   acc  int32 [N,M] output of the raw accumulators, or NULL
 * N > 16 returns BITLINEAR_ERR_UNSUPPORTED_SHAPE.
 * Two kernels give the same results.  A launch with at least as many 32-row
 * units as the GPU has resident warps streams them with one warp per run of
 * units.  A smaller launch, or one where whole runs of units per warp would
 * leave more than a quarter of the resident warps idle, takes one 4-warp CTA
 * per unit, whose warps split the unit's k-chunks and add their int32 sums at
 * the end.
 */
BITLINEAR_API bitlinear_status bitlinear_gemv(const uint32_t* packed, const float* alpha,
                                int64_t M, int64_t K,
                                const int8_t* xq, const float* amax, const int32_t* xsum,
                                int64_t N, float* y, int32_t* acc,
                                bitlinear_stream_t stream);

/*
 * Prefill GEMM, any N >= 1, on the int8 tensor cores (tcgen05.mma kind::i8,
 * accumulators in tensor memory): packed weight tiles are brought in by TMA,
 * expanded to int8 in shared memory and multiplied with TMA-loaded int8
 * activation tiles; the rescale is fused into the epilogue.  Same arguments
 * and results as bitlinear_gemv, any M.  Ragged tiles read zeros past M, K
 * and N through the tensor maps; when 4*M is not a multiple of 16 the
 * outputs are written with plain stores instead of tensor stores.
 * The reading notes (section 4.4) name prefill, where the work turns
 * compute-bound, as the stage their CPU kernels leave unoptimised.
 */
BITLINEAR_API bitlinear_status bitlinear_gemm(const uint32_t* packed, const float* alpha,
                                int64_t M, int64_t K,
                                const int8_t* xq, const float* amax, const int32_t* xsum,
                                int64_t N, float* y, int32_t* acc,
                                bitlinear_stream_t stream);

/*
 * One linear layer of a grouped call.  Every pointer follows the conventions
 * above; M and K are this layer's shape.  All layers of one call share the
 * token count N.
 */
typedef struct {
    const uint32_t* packed;   /* [M, WP(K)] words */
    const float* alpha;       /* [1] */
    int64_t M;
    int64_t K;
    const int8_t* xq;         /* [N, K] */
    const float* amax;        /* [N] */
    const int32_t* xsum;      /* [N] */
    float* y;                 /* [N, M] output */
    int32_t* acc;             /* [N, M] output, or NULL */
} bitlinear_problem;

/*
 * Decode GEMV over a list of independent layers in as few launches as
 * possible (one per 256 layers): the same arithmetic as bitlinear_gemv for
 * each entry.  Meant for layers whose activations are known at the same time
 * -- the q/k/v or gate/up projections of one decoder layer, or a stream of
 * layers whose inputs are all available.  `problems` is a HOST array of
 * `count` entries, read during the call only.  1 <= N <= 16.
 */
BITLINEAR_API bitlinear_status bitlinear_gemv_grouped(const bitlinear_problem* problems,
                                                      int64_t count, int64_t N,
                                                      bitlinear_stream_t stream);

/*
 * Tensor-core GEMM over a list of independent layers in one persistent
 * launch per 8 layers (tiles of all layers share the grid, the layers with the
 * largest K first): the same arithmetic as bitlinear_gemm for each entry.
 * `problems` is a HOST array read during the call only.  N >= 1.
 */
BITLINEAR_API bitlinear_status bitlinear_gemm_grouped(const bitlinear_problem* problems,
                                                      int64_t count, int64_t N,
                                                      bitlinear_stream_t stream);

/* -------------------------------------------- decode with fused quantiser */

/*
 * Decode GEMV that takes fp32 activations and quantises them itself, in the
 * same launch: per token amax = max|x|, q = clamp(rint(x * (127/amax)),
 * -128, 127) exactly as bitlinear_quant_act, then the product and rescale of
 * bitlinear_gemv.  The int8 activations never reach global memory.  This is
 * the fused form of the I2_S path (reading notes section 2.3 and section 4.1;
 * FairyFuse "fused kernel design": quantisation, unpacking and accumulation in
 * one kernel with no intermediate writes).
 *   x    fp32 [N,K] activations, 16-byte aligned, row stride K
 *   y    fp32 [N,M] output, bit-identical to quant_act followed by gemv
 *   acc  int32 [N,M] raw accumulators, or NULL
 * 1 <= N <= 16, and N * 512 * ceil(K/512) <= 65536 (the int8 copy each CTA
 * keeps in shared memory): N = 1 takes K up to 65536, N = 16 up to 4096.
 * Larger cases return BITLINEAR_ERR_UNSUPPORTED_SHAPE; quantise with
 * bitlinear_quant_act and call bitlinear_gemv for them.
 * One kernel: each CTA owns a contiguous range of 32-row units with about
 * the same number of (unit, 512-weight k-chunk) pairs as the others,
 * quantises the input once into shared memory with all its threads, and its
 * warps split the range's pairs, adding the int32 sums of units they share
 * at the end (integer sums: the result does not depend on the split).
 */
BITLINEAR_API bitlinear_status bitlinear_gemv_quant(const uint32_t* packed, const float* alpha,
                                                    int64_t M, int64_t K, const float* x,
                                                    int64_t N, float* y, int32_t* acc,
                                                    bitlinear_stream_t stream);

/* One layer of a fused grouped call: the layer and its fp32 input. */
typedef struct {
    const uint32_t* packed;   /* [M, WP(K)] words */
    const float* alpha;       /* [1] */
    int64_t M;
    int64_t K;
    const float* x;           /* [N, K] fp32 */
    float* y;                 /* [N, M] output */
    int32_t* acc;             /* [N, M] output, or NULL */
} bitlinear_fused_problem;

/*
 * bitlinear_gemv_quant over a list of layers, one launch per 256 layers.
 * Each CTA quantises an input once for the run of rows it owns, so layers
 * that read the same activations (q, k and v; gate and up) should carry the
 * same x pointer and sit next to each other in the list.  `problems` is a HOST
 * array read during the call only.  The shared-memory limit above applies to
 * the largest K of each launch.  All layers are checked before anything is
 * launched.
 */
BITLINEAR_API bitlinear_status bitlinear_gemv_quant_grouped(
    const bitlinear_fused_problem* problems, int64_t count, int64_t N,
    bitlinear_stream_t stream);

/* --------------------------------------- TL2-style storage, 5/3 bits/weight */

/*
 * A second storage of the same ternary codes at 5 bits per three weights:
 * each group of three is folded onto its mirror image and stored as a 1-bit
 * sign and a 4-bit index, and K is split into a part stored in groups of
 * three and a remainder (reading notes section 2.3 "technical details":
 * signed-unsigned weight splitting, block-fitting weight splitting; 1.67
 * bits per weight).  It moves 1/6 fewer weight bytes than the 2-bit layout.
 * Row layout (this library's own; rows contiguous, each 16-byte aligned):
 *   [0, 16*nb)            index plane, nb = floor(K/96) blocks of 96 weights:
 *                         group g of block b (weights 96b+3g .. 96b+3g+2) has
 *                         its index in byte 16b + g/2, low nibble for even g
 *   [16*nb, +16*ceil(nb/4))  sign plane: uint32 per block, bit g; zero padding
 *   then 16*ceil(K2/64)   the last K2 = K - 96*nb weights in the 2-bit layout
 *                         above (a K2-wide row, padded with code 0)
 * For codes (c0,c1,c2) let v = 9(c0+1) + 3(c1+1) + (c2+1) in [0, 26]: the
 * index is |v - 13| and the sign is (v < 13).
 */

/* Bytes of one TL2 row for K (a multiple of 16, at most 131072), else 0. */
BITLINEAR_API size_t bitlinear_tl2_row_bytes(int64_t K);

/*
 * Re-encode packed 2-bit weights [M, WP(K)] (from bitlinear_pack_weights) as
 * TL2 rows: tl2 receives M * bitlinear_tl2_row_bytes(K) bytes.  alpha is
 * unchanged and is used with either storage.
 */
BITLINEAR_API bitlinear_status bitlinear_tl2_from_packed(const uint32_t* packed, int64_t M,
                                                         int64_t K, uint8_t* tl2,
                                                         bitlinear_stream_t stream);

/*
 * Decode GEMV (1 <= N <= 16) over TL2 rows: the results of bitlinear_gemv
 * (y, and acc when non-NULL) for the same codes and activations.  xq and
 * amax come from a quantiser call; the activation sum is not needed.
 */
BITLINEAR_API bitlinear_status bitlinear_gemv_tl2(const uint8_t* tl2, const float* alpha,
                                                  int64_t M, int64_t K, const int8_t* xq,
                                                  const float* amax, int64_t N, float* y,
                                                  int32_t* acc, bitlinear_stream_t stream);

/* One layer of a grouped TL2 call. */
typedef struct {
    const uint8_t* tl2;       /* [M, bitlinear_tl2_row_bytes(K)] bytes */
    const float* alpha;       /* [1] */
    int64_t M;
    int64_t K;
    const int8_t* xq;         /* [N, K] */
    const float* amax;        /* [N] */
    float* y;                 /* [N, M] output */
    int32_t* acc;             /* [N, M] output, or NULL */
} bitlinear_tl2_problem;

/* bitlinear_gemv_tl2 over a list of layers, one launch per 256 layers;
 * `problems` is a HOST array read during the call only. */
BITLINEAR_API bitlinear_status bitlinear_gemv_tl2_grouped(const bitlinear_tl2_problem* problems,
                                                          int64_t count, int64_t N,
                                                          bitlinear_stream_t stream);

/* ------------------------------------------------- weights, no allocation */

/*
 * bitlinear_pack_weights for callers that cannot allocate device memory at
 * all -- not even the small workspace the entry point above asks for.  Typical
 * cases: a plugin inside a host process (an inference server, a game engine)
 * that owns the whole device memory budget through its own pool and forbids
 * its libraries from calling cudaMalloc; or a latency-critical path where
 * cudaMalloc/cudaFree are unacceptable because they can synchronise the
 * device.  The pages describe no such entry point; it exists only for these
 * callers.
 *
 * Same arguments, results and errors as bitlinear_pack_weights minus the
 * workspace: the exponent bins live in a fixed 2064-byte array that the
 * library keeps in device global memory (one copy per GPU that loads the
 * library, held until the process exits).  That array bounds nothing but the
 * element count: M*K must not exceed 2^40 (BITLINEAR_ERR_UNSUPPORTED_SHAPE
 * otherwise), the same limit as the workspace version.  The array is cleared
 * on the stream at the start of every call.
 *
 * The first call on each device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  The call
 * allocates nothing, host or device.  All calls on one device share the array:
 * calls whose work may overlap on the GPU (different streams without ordering
 * between them) race and give wrong results; order them on one stream, or use
 * bitlinear_pack_weights with separate workspaces.
 */
BITLINEAR_API bitlinear_status bitlinear_pack_weights_noalloc(const float* W, int64_t M,
                                                              int64_t K, uint32_t* packed,
                                                              float* alpha,
                                                              bitlinear_stream_t stream);

/* ------------------------------------------------------------ diagnostics */

/*
 * Read (and, if clear != 0, reset) the device-side error words: kernels set
 * them when a bounded wait gives up, and the pack step when the weights hold
 * inf or NaN.  Synchronises the device.  *status_out is BITLINEAR_OK,
 * BITLINEAR_ERR_DEVICE_TIMEOUT (if any wait gave up) or else
 * BITLINEAR_ERR_NONFINITE; the return value reports whether the read itself
 * worked.
 */
BITLINEAR_API bitlinear_status bitlinear_device_error(int* status_out, int clear);

/*
 * Wall-time limit, in nanoseconds, of every bounded wait in the kernels
 * launched after this call (process-wide; 0 restores the default of 2 s).
 * Returns the previous limit.  A wait that runs out makes its kernel wind
 * down: it stops issuing work, waits (with a fixed 2 s limit) for the copies
 * and tensor-core operations it has in flight, releases its tensor memory and
 * returns, leaving its outputs incomplete and BITLINEAR_ERR_DEVICE_TIMEOUT in
 * the device error word.  Normal waits last microseconds; a short limit is a
 * way to exercise that path (or to bound the cost of a stalled device) without
 * a fault.  Launches already enqueued keep the limit they were given.
 */
BITLINEAR_API unsigned long long bitlinear_set_wait_limit(unsigned long long limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
