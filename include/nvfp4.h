/*
 * libnvfp4 — NVFP4 two-level micro-scaling quantization and the block-scaled
 * GEMM that consumes it, for NVIDIA B200 (sm_100a).
 *
 * Format (defined by the pages this library follows):
 *   - elements: 4-bit E2M1 codes, values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}
 *     ("NVIDIA NVFP4 与 Micro-Scaling" section 二; "mxFP4/nvFP4 最小化知识",
 *     nvFP4的数据结构设计), packed two per byte, first element in the low
 *     nibble ("FP4" wiki, 技術原理: ONNX FLOAT4E2M1 packing);
 *   - one E4M3 block scale per 16 consecutive elements along K
 *     ("Introducing NVFP4 ...", 二级微块 scaling 策略);
 *   - one FP32 per-tensor scale.  The library stores the encode scale
 *     g = 2688 / amax = 1 / s_global, s_global = amax / (6 * 448)
 *     ("low-precision-floats", section FP4 / MXFP4 / NVFP4).
 *
 * Quantization rule, per 16-element block with block amax ab:
 *     s  = e4m3_rne_satfinite((ab * g) / 6)          (fp32 multiply, fp32 divide)
 *     q  = e2m1_rne_sat((x * g) / decode(s))           (fp32 multiply, IEEE fp32 divide)
 *   with q = 0 for every element of a block whose scale decodes to 0, and
 *   g = 1 for an all-zero tensor.
 *
 * GEMM: D = alpha * (s_a (.) A)(s_b (.) B)^T, alpha = 1 / (g_a * g_b) in fp32,
 *   FP32 accumulation in tensor memory ("NVIDIA NVFP4 与 Micro-Scaling"
 *   section 三 scaled GEMM and section 五 data layout).  A is [M, K], B is
 *   [N, K]; both K-major ("NT").
 *
 * Conventions for every entry point:
 *   - All buffers are device memory owned and allocated by the caller, except
 *     where a parameter says "host".  The library never allocates or frees
 *     memory and never synchronises, except nvfp4_check_device_status().
 *   - Work is enqueued on the caller's stream (a cudaStream_t; NULL is the
 *     legacy default stream).  Global scales stay on the device, so a chain of
 *     calls needs no host round trip.
 *   - Argument, shape, alignment and architecture errors are returned before
 *     anything is enqueued.  A failed launch returns NVFP4_ERR_CUDA.
 *   - Errors met on the device (a bounded wait that gave up, a tensor whose
 *     global scale is not finite) are recorded in a per-device status word,
 *     read and cleared by nvfp4_check_device_status().
 *   - Codes are dense: row r of a [rows, K] code matrix starts at byte
 *     r * K / 2.  bf16 inputs have a row pitch ld (in elements).
 *   - Input and code/scale pointers must be 16-byte aligned and the bf16
 *     input pitch must keep every row 16-byte aligned (ld % 8 == 0).  Output
 *     pointers need only element alignment.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same type as cudaStream_t */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of the required block, M too large, ... */
  NVFP4_ERR_MISALIGNED = 3,        /* pointer or leading dimension breaks 16-byte alignment */
  NVFP4_ERR_ARCH = 4,              /* current device is not sm_100 */
  NVFP4_ERR_CUDA = 5,              /* a CUDA call or kernel launch failed */
  NVFP4_ERR_TIMEOUT = 6,           /* a bounded device wait gave up (device status) */
  NVFP4_ERR_RANGE = 7,             /* 2688/amax not finite: non-finite input or amax < ~7.9e-36 (device status) */
  NVFP4_ERR_WORKSPACE = 8          /* workspace smaller than nvfp4_workspace_bytes() */
} nvfp4_status;

typedef enum {
  NVFP4_SF_ROWMAJOR = 0, /* [rows, K/16] bytes, row-major */
  NVFP4_SF_TCGEN05 = 1   /* tensor-core scale atoms, see nvfp4_sf_bytes() */
} nvfp4_sf_layout;

typedef enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_F32 = 1 } nvfp4_out_dtype;

typedef enum { NVFP4_OP_GEMV_BATCHED = 1, NVFP4_OP_GEMM_QUANT_A = 2 } nvfp4_op;

/* ABI version of this header (bumped on incompatible changes). */
NVFP4_API int nvfp4_abi_version(void);

/* Human-readable name of a status code (static string). */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

/*
 * Bytes of a block-scale array for a [rows, k] tensor.
 *   NVFP4_SF_ROWMAJOR: rows * k/16.
 *   NVFP4_SF_TCGEN05 : the layout the sm_100 block-scaled MMA reads through
 *     tensor memory.  Rows are padded to a multiple of 128 and the k/16 blocks
 *     to a multiple of 4.  The array is a sequence of 512-byte atoms, atom
 *     (i, j) covering rows 128i..128i+127 and blocks 4j..4j+3 at byte offset
 *     512 * (i * (padded blocks / 4) + j); inside an atom, (row r, block b)
 *     sits at (r % 32) * 16 + ((r % 128) / 32) * 4 + (b % 4).  Padding is 0.
 *     (The pages do not describe this layout; it is the tensor core's.)
 * Returns 0 for negative sizes or k not a multiple of 16.
 */
NVFP4_API size_t nvfp4_sf_bytes(int64_t rows, int64_t k, nvfp4_sf_layout layout);

/*
 * Tensor amax ("NVIDIA NVFP4 与 Micro-Scaling" section 三, step 1:
 * |X|_max): *amax_dev = max |x| over a bf16 [rows, k] tensor with row pitch
 * ldx.  The callee zeroes *amax_dev first (on the stream).  k % 8 == 0.
 * Non-finite inputs propagate to *amax_dev (a later quantize reports RANGE).
 */
NVFP4_API nvfp4_status nvfp4_amax(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, float* amax_dev,
                        nvfp4_stream_t stream);

/*
 * Two-level NVFP4 quantization of a bf16 [rows, k] tensor
 * ("low-precision-floats" section FP4 / MXFP4 / NVFP4, the s_global,
 * s_block and x_hat formulas; "Introducing NVFP4 ..." 二级微块 scaling).
 *   codes : out, [rows, k/2] bytes (two E2M1 codes per byte, low nibble first)
 *   sf    : out, block scales in `layout` (nvfp4_sf_bytes(rows, k, layout) bytes;
 *           padding of the TCGEN05 layout is written as 0)
 *   g_dev : out, one fp32, the encode scale 2688 / amax (1 for an all-zero tensor)
 *   amax_dev : one fp32.  amax_given == 0: workspace and out, the callee
 *           computes the tensor amax into it (two passes over x).
 *           amax_given == 1: in, the callee uses *amax_dev as the amax (one pass).
 * k % 16 == 0 for NVFP4_SF_ROWMAJOR, k % 64 == 0 for NVFP4_SF_TCGEN05.
 * An empty tensor (rows == 0 or k == 0) is valid: x, codes and sf may then be
 * null; the amax is 0 and *g_dev is 1.
 * If 2688/amax is not finite, codes and scales are written as 0, *g_dev as 0,
 * and the device status records NVFP4_ERR_RANGE.
 */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, void* codes, void* sf,
                            nvfp4_sf_layout layout, float* g_dev, float* amax_dev, int amax_given,
                            nvfp4_stream_t stream);

/*
 * NVFP4 quantization with stochastic rounding of the element codes ("FP4"
 * encyclopedia entry, 技術原理: NVFP4 quantization rounds stochastically
 * instead of truncating).  amax, the global scale and the E4M3 block scales
 * are those of nvfp4_quantize (round to nearest even).  Each element's
 * u = fp32(fp32(x * g) / sd) lies between adjacent E2M1 magnitudes lo <= |u| < hi;
 * it rounds to hi when R < f * 2^16, f = (|u| - lo) / (hi - lo), with R a 16-bit
 * random integer, so E[x_hat] = x to within 2^-16 of a grid step; |u| >= 6 gives
 * 6; the sign bit is kept.  R is drawn in the kernel by Philox4x32-10 (Salmon
 * et al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011): key =
 * (seed mod 2^32, seed div 2^32); block b (16 elements) of row r uses the
 * counters (2b + h, r, offset mod 2^32, offset div 2^32), h = 0, 1, and element
 * 8h + 2i + m of the block takes bits 16m..16m+15 of output word i.  Equal
 * (seed, offset) give equal codes; advance `offset` per call for fresh bits.
 * Arguments, constraints and errors otherwise as nvfp4_quantize.
 */
NVFP4_API nvfp4_status nvfp4_quantize_stochastic(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx,
                                       void* codes, void* sf, nvfp4_sf_layout layout, float* g_dev,
                                       float* amax_dev, int amax_given, uint64_t seed, uint64_t offset,
                                       nvfp4_stream_t stream);

/*
 * Hadamard-rotated NVFP4 quantization ("NVIDIA NVFP4 与 Micro-Scaling",
 * section 4.1 旋转/阿达玛变换: x is multiplied by an orthogonal Walsh-Hadamard
 * matrix before quantization, which spreads outlier channels over all
 * channels; giving the weights the same rotation along K leaves the product
 * A W^T unchanged, since (A H)(W H)^T = A W^T).
 *   y = x H, H = blockdiag(H_n, ..., H_n) / sqrt(n), H_n the Sylvester-ordered
 *   Walsh-Hadamard matrix of order n.  y is formed in fp32 by the fast
 *   transform (stages h = 1, 2, 4, ..., n/2, each pair (i, i + h) with bit h of
 *   i clear becoming (y_i + y_{i+h}, y_i - y_{i+h})), then y * fp32(1/sqrt(n)).
 *   y is then quantized exactly as nvfp4_quantize quantizes x, with the amax
 *   taken over y.
 *   hadamard_order : n, a power of two from 1 to 512 dividing k (1 leaves x
 *           unrotated and gives nvfp4_quantize's result).
 *   codes, sf, g_dev, layout, k constraints: as nvfp4_quantize.
 *   amax_dev : amax_given == 0: out, max |y| (two passes over x, the transform
 *           recomputed in the second).  amax_given == 1: in, used as max |y|.
 * Rotate both GEMM operands with the same n; nvfp4_gemm then gives
 * approximately A W^T.  Errors: INVALID_ARG for an order that is not a power
 * of two in [1, 512], UNSUPPORTED_SHAPE when it does not divide k; a non-finite
 * max |y| behaves as in nvfp4_quantize (zero outputs, device status RANGE).
 */
NVFP4_API nvfp4_status nvfp4_quantize_hadamard(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx,
                                     int hadamard_order, void* codes, void* sf, nvfp4_sf_layout layout,
                                     float* g_dev, float* amax_dev, int amax_given, nvfp4_stream_t stream);

/*
 * The rotated quantizer with stochastic rounding of the codes: y = x H as in
 * nvfp4_quantize_hadamard, then y quantized as nvfp4_quantize_stochastic
 * quantizes x (block scales round to nearest; each code rounds up with
 * probability ceil(f * 2^16) / 2^16 from Philox4x32-10 bits, the counters of
 * block b of row r being (2b + h, r, offset mod 2^32, offset div 2^32), key =
 * seed).  The "FP4" encyclopedia entry (技術原理) names the two techniques
 * together.  Arguments, constraints and errors as nvfp4_quantize_hadamard,
 * plus seed and offset as nvfp4_quantize_stochastic.
 */
NVFP4_API nvfp4_status nvfp4_quantize_hadamard_stochastic(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx,
                                                int hadamard_order, void* codes, void* sf,
                                                nvfp4_sf_layout layout, float* g_dev, float* amax_dev,
                                                int amax_given, uint64_t seed, uint64_t offset,
                                                nvfp4_stream_t stream);

/*
 * MXFP4, the format the pages set against NVFP4 ("mxFP4/nvFP4 最小化知识",
 * (一) mxFP4的技术局限; "low-precision-floats", FP4 / MXFP4 / NVFP4): one E8M0
 * (power-of-two) scale per 32 consecutive elements along K and no global
 * scale.  With A the block max |x|:
 *     k  = ceil(log2(A / 6))   (A / 6 an fp32 RN divide; rounded up, as the page
 *                               says TensorRT does; clamped to [-127, 127];
 *                               A == 0 gives -127)
 *     scale byte = k + 127     (torch.float8_e8m0fnu)
 *     q  = e2m1_rne_sat(x * 2^-k)   (|x * 2^-k| <= 6)
 * One pass over x.  codes: out, [rows, k/2] bytes (16-byte aligned); sf: out,
 * nvfp4_mxfp4_sf_bytes(rows, k, layout) bytes.  k % 32 == 0 for
 * NVFP4_SF_ROWMAJOR, k % 128 == 0 for NVFP4_SF_TCGEN05 (atoms of 128 rows x 4
 * scales, laid out as in nvfp4_sf_bytes, each scale covering 32 elements).
 * A block holding a non-finite value gets scale byte 0xFF and zero codes, and
 * the device status records NVFP4_ERR_RANGE.
 */
NVFP4_API size_t nvfp4_mxfp4_sf_bytes(int64_t rows, int64_t k, nvfp4_sf_layout layout);
NVFP4_API nvfp4_status nvfp4_mxfp4_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ldx, void* codes,
                                  void* sf, nvfp4_sf_layout layout, nvfp4_stream_t stream);

/*
 * MXFP4 block-scaled GEMM on tcgen05.mma kind::mxf4 (.scale_vec::2X, E8M0
 * scales): D[m, n] = sum_k (s_a a)[m,k] (s_b b)[n,k], no global scales.
 *   a_codes [M, K/2], a_sf_tc: TCGEN05 MXFP4 scales of A (nvfp4_mxfp4_quantize)
 *   b_codes [N, K/2], b_sf_tc: the same for B
 *   d: out, [M, N], pitch ldd >= N, bf16 or fp32 per out_dtype (as nvfp4_gemm).
 * K % 128 == 0 (whole scale atoms), M, N >= 1.
 */
NVFP4_API nvfp4_status nvfp4_mxfp4_gemm(const void* a_codes, const void* a_sf_tc, const void* b_codes,
                              const void* b_sf_tc, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                              nvfp4_out_dtype out_dtype, nvfp4_stream_t stream);

/*
 * Re-layout of row-major block scales [rows, k/16] into the TCGEN05 layout
 * (see nvfp4_sf_bytes), padding written as 0.  k % 64 == 0.  Pure byte
 * permutation; the pages are silent on the tensor core's scale layout.
 */
NVFP4_API nvfp4_status nvfp4_swizzle_sf(const void* sf_rowmajor, int64_t rows, int64_t k, void* sf_tcgen05,
                              nvfp4_stream_t stream);

/*
 * Block-scaled GEMM on tcgen05.mma kind::mxf4nvf4 ("NVIDIA NVFP4 与
 * Micro-Scaling" section 三: D = g_d((g_a s_a (.) A)(g_b s_b (.) W)); section 五:
 * the tensor core consumes (FP4 data, FP8 block scale) pairs and accumulates
 * in FP32).  Here D[m, n] = alpha * sum_k (s_a a)[m,k] (s_b b)[n,k] with
 * alpha = 1 / (g_a * g_b) computed in fp32 from *g_a_dev and *g_b_dev.
 *   a_codes [M, K/2], a_sf_tc TCGEN05 scales of A, g_a_dev one fp32 (encode scale of A)
 *   b_codes [N, K/2], b_sf_tc TCGEN05 scales of B, g_b_dev one fp32
 *   d: out, [M, N] with row pitch ldd >= N elements, bf16 (round to nearest
 *      even) or fp32 per out_dtype; element-aligned (16-byte aligned rows get
 *      vector stores, other pitches element stores).
 * K % 64 == 0, K > 0, M, N >= 1 (any value; tails are masked).
 */
NVFP4_API nvfp4_status nvfp4_gemm(const void* a_codes, const void* a_sf_tc, const float* g_a_dev, const void* b_codes,
                        const void* b_sf_tc, const float* g_b_dev, int64_t M, int64_t N, int64_t K, void* d,
                        int64_t ldd, nvfp4_out_dtype out_dtype, nvfp4_stream_t stream);

/*
 * The GEMM of nvfp4_gemm with its result landing under an output scale g_d
 * ("NVIDIA NVFP4 与 Micro-Scaling" section 三: D = g_d * (...), "output
 * dequantization by g_d, the output often landing as FP8"; its _scaled_mm
 * example passes scale_result=g_d with a float8_e4m3fn output).  With
 * v = fp32(alpha * acc), the value nvfp4_gemm's fp32 output holds:
 *
 * nvfp4_gemm_fp8_out: d_e4m3[m, n] = e4m3_rne_satfinite(fp32(v * g_d)), one
 *   byte per element (float8_e4m3fn), row pitch ldd bytes >= N; d_e4m3 16-byte
 *   aligned and ldd % 16 == 0.
 *
 * nvfp4_gemm_requant: D quantized to NVFP4 for the next layer, g_d being D's
 *   global encode scale (given; e.g. 2688 / amax of a previous step): per 16
 *   consecutive columns s = e4m3_rne_satfinite(fp32(fp32(ab * g_d) / 6)) with
 *   ab = max |v| over the block, codes e2m1_rne_sat(fp32(fp32(v * g_d) / sd))
 *   (zero codes when sd == 0), two per byte, first in the low nibble.
 *   d_codes [M, N/2] with row pitch ldd_bytes >= N/2 (16-byte aligned rows);
 *   d_sf: block scales in d_sf_layout (nvfp4_sf_bytes(M, N, layout) bytes; in
 *   the TCGEN05 layout the rows past M of the last 128-row group are not
 *   written).  N % 16 == 0, and N % 64 == 0 for the TCGEN05 layout.
 *
 * Both: g_d_dev one fp32 on the device; amax_d_dev (optional, may be null)
 * receives max |v| over D (zeroed by the call first), the input of the next
 * step's encode scale.  Other arguments, shapes and errors as nvfp4_gemm.
 */
NVFP4_API nvfp4_status nvfp4_gemm_fp8_out(const void* a_codes, const void* a_sf_tc, const float* g_a_dev,
                              const void* b_codes, const void* b_sf_tc, const float* g_b_dev, int64_t M,
                              int64_t N, int64_t K, const float* g_d_dev, void* d_e4m3, int64_t ldd,
                              float* amax_d_dev, nvfp4_stream_t stream);
NVFP4_API nvfp4_status nvfp4_gemm_requant(const void* a_codes, const void* a_sf_tc, const float* g_a_dev,
                              const void* b_codes, const void* b_sf_tc, const float* g_b_dev, int64_t M,
                              int64_t N, int64_t K, const float* g_d_dev, void* d_codes, int64_t ldd_bytes,
                              void* d_sf, nvfp4_sf_layout d_sf_layout, float* amax_d_dev,
                              nvfp4_stream_t stream);

/* Workspace bytes needed by an op for the given sizes (0 for bad sizes). */
NVFP4_API size_t nvfp4_workspace_bytes(nvfp4_op op, int64_t M, int64_t N, int64_t K);

/*
 * Decode batched GEMV: y[m, n] = alpha * sum_k (s_x x_q)[m,k] (s_w w)[n,k]
 * for M <= 32 activation rows x (bf16 [M, K], pitch ldx) quantized on the fly
 * with the same rule as nvfp4_quantize (its own amax and global scale), and
 * pre-quantized weights w (codes [N, K/2], TCGEN05 scales, *g_w_dev).  The
 * weight stream dominates (decode is memory-bound: "NVIDIA NVFP4 与
 * Micro-Scaling" section 六).  y: out, bf16 [M, N], pitch ldy.
 * workspace: device scratch of nvfp4_workspace_bytes(NVFP4_OP_GEMV_BATCHED, M, N, K)
 *   bytes (quantized x, its scales and g, fp32 partial sums, tile counters).
 *   It needs no clearing, before the first call or between calls:
 *     - M > 8: the call's first kernel rewrites the quantized x and zeroes
 *       the counters;
 *     - M <= 8: each counter holds a 48-bit tag drawn per launch beside its
 *       count, and a counter with another tag counts as zero, so stale bytes
 *       are taken for this launch's only by a 2^-48 chance; every launch that
 *       completes returns the counters it used to zero, so a CUDA graph that
 *       replays one launch (one tag) starts each replay from zeros;
 *     - partial sums are written before they are read.
 *   After a call that reported NVFP4_ERR_TIMEOUT, zero the workspace before
 *   reusing it.  Calls sharing a workspace must not overlap on the device.
 * K % 64 == 0, 1 <= M <= 32.
 */
NVFP4_API nvfp4_status nvfp4_gemv_batched(const void* x_bf16, int64_t M, int64_t ldx, const void* w_codes,
                                const void* w_sf_tc, const float* g_w_dev, int64_t N, int64_t K, void* y_bf16,
                                int64_t ldy, void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_gemv_batched without a workspace argument, for callers that cannot
 * allocate device memory: a plug-in whose host framework owns all device
 * memory and hands it only input and output buffers, or a real-time path
 * that may not call the allocator once it has started (an allocation can
 * block, synchronise the device or fail when memory is short).  The pages
 * have no counterpart of this entry point; it computes exactly what
 * nvfp4_gemv_batched computes.
 *   Scratch: a fixed 4 MiB array inside the library, present on every GPU
 *     that loads it until the process exits.  Shapes whose workspace
 *     (nvfp4_workspace_bytes(NVFP4_OP_GEMV_BATCHED, M, N, K)) exceeds 4 MiB
 *     are rejected with NVFP4_ERR_WORKSPACE, before anything is enqueued;
 *     M <= 16 with N <= 32768 and K <= 16384 always fits.
 *   Set-up: the first call on a device (made with that device current) looks
 *     up the scratch's device address; make that first call before any stream
 *     capture.  Nothing is allocated or freed, then or later.
 *   Sharing: every call on a device uses the same scratch and overwrites what
 *     the previous call left there; what must start at zero is cleared by the
 *     call (M > 8) or tagged per launch and returned to zero at its end
 *     (M <= 8), as for nvfp4_gemv_batched's workspace.  Calls that overlap on
 *     the device race: serialise them, e.g. on one stream.
 * Other arguments, constraints and errors as nvfp4_gemv_batched.
 */
NVFP4_API nvfp4_status nvfp4_gemv_batched_noalloc(const void* x_bf16, int64_t M, int64_t ldx, const void* w_codes,
                                const void* w_sf_tc, const float* g_w_dev, int64_t N, int64_t K,
                                void* y_bf16, int64_t ldy, nvfp4_stream_t stream);

/*
 * GEMM whose A operand arrives in bf16 (an activation): A [M, K] (pitch lda)
 * is quantized to NVFP4 with the nvfp4_quantize rule (tensor amax first),
 * then multiplied by pre-quantized B as in nvfp4_gemm ("NVIDIA NVFP4 与
 * Micro-Scaling" section 三: activations quantized with a per-tensor global
 * scale and per-block micro-scales, then the block-scaled product).
 *   When M > 128 and N > 128 (and K <= 262144), one kernel does both after
 *   the amax pass: extra warps quantize A in units (one row, 4096 elements
 *   of K) while the tensor cores multiply the parts already done.  Where B's
 *   codes (N * K / 2 bytes) are at most 64 MiB the tiles go row block by row
 *   block and A is quantized row by row (B stays in L2); for larger B (long
 *   K) the 256-row blocks form about four groups, taken in turn, with the
 *   tiles m-fastest inside a group and A quantized chunk by chunk along K, so
 *   B is read from DRAM about four times and the first tiles wait for one
 *   chunk of a quarter of A.
 *   Other shapes run the quantize pass and the GEMM as two kernels.  All
 *   give the same codes, scales, g_a and D bit for bit.
 * workspace: nvfp4_workspace_bytes(NVFP4_OP_GEMM_QUANT_A, M, N, K) bytes:
 *   A's codes [M, K/2] at byte 0, A's tensor-core scales from
 *   round_up(M * K / 2, 256), then at the next 256-byte boundary g_a (fp32),
 *   amax_a 16 bytes after it, a unit ticket at byte 64 and readiness
 *   counters (one int per 256-row block and 4096-wide K chunk) from byte 128
 *   there, which the call zeroes itself.  It needs no clearing; calls
 *   sharing a workspace must not overlap.
 * Concurrency: the one-kernel form's warps take units of A from a ticket
 *   counter, so whichever CTAs are resident quantize what the tiles wait
 *   for; it runs at speed with its whole grid resident.  Calls that share
 *   nothing may overlap.
 * K % 64 == 0.
 */
NVFP4_API nvfp4_status nvfp4_gemm_quant_a(const void* a_bf16, int64_t lda, const void* b_codes, const void* b_sf_tc,
                                const float* g_b_dev, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
                                nvfp4_out_dtype out_dtype, void* workspace, size_t ws_bytes,
                                nvfp4_stream_t stream);

/*
 * nvfp4_gemm_quant_a in two calls on one stream, the same A and workspace:
 * _prepare zeroes what the second call counts on and runs the amax pass of A
 * into the workspace (it reads no B and writes no D); _run quantizes A and
 * multiplies.  _prepare then _run computes exactly what nvfp4_gemm_quant_a
 * computes; work may be enqueued between them if it leaves A and the
 * workspace alone.  A _run without a _prepare since the last _run on that
 * workspace is an error the library cannot detect: D may then come from a
 * stale amax or from rows of A not yet quantized.
 */
NVFP4_API nvfp4_status nvfp4_gemm_quant_a_prepare(const void* a_bf16, int64_t lda, int64_t M, int64_t N, int64_t K,
                                void* workspace, size_t ws_bytes, nvfp4_stream_t stream);
NVFP4_API nvfp4_status nvfp4_gemm_quant_a_run(const void* a_bf16, int64_t lda, const void* b_codes,
                                const void* b_sf_tc, const float* g_b_dev, int64_t M, int64_t N, int64_t K,
                                void* d, int64_t ldd, nvfp4_out_dtype out_dtype, void* workspace,
                                size_t ws_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_quant_a with A's tensor amax already on the device: amax_dev
 * (one fp32, read-only) holds max |A|, e.g. from nvfp4_amax on the same A
 * earlier on the stream; the call skips its own amax pass.  Null amax_dev:
 * NVFP4_ERR_INVALID_ARG.  Everything else as nvfp4_gemm_quant_a.
 */
NVFP4_API nvfp4_status nvfp4_gemm_quant_a_amax(const void* a_bf16, int64_t lda, const float* amax_dev,
                                const void* b_codes, const void* b_sf_tc, const float* g_b_dev, int64_t M,
                                int64_t N, int64_t K, void* d, int64_t ldd, nvfp4_out_dtype out_dtype,
                                void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * Synchronises the stream, then returns and clears the device status word of
 * the current device: NVFP4_OK, NVFP4_ERR_TIMEOUT or NVFP4_ERR_RANGE (or
 * NVFP4_ERR_CUDA if the synchronisation itself failed).
 */
NVFP4_API nvfp4_status nvfp4_check_device_status(nvfp4_stream_t stream);

/*
 * Limit, in nanoseconds of device global time, for every bounded wait inside
 * the library's kernels (default 2e9).  A wait that runs out records
 * NVFP4_ERR_TIMEOUT and its kernel returns.  Applies to later launches.
 */
NVFP4_API void nvfp4_set_wait_limit_ns(uint64_t limit_ns);

/*
 * Self-test of the bounded-wait path: one thread waits on an mbarrier that
 * nothing arrives on, for at most limit_ns, then records NVFP4_ERR_TIMEOUT in
 * the device status.  Nothing else is in flight, so the context stays usable.
 */
NVFP4_API nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
