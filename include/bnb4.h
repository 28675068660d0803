/*
 * bnb4.h -- C ABI of the B200 (sm_100a) library for 4-bit blockwise weight
 * quantization (NF4 / FP4), double quantization of the per-block absmax,
 * dequantization, and the fused 4-bit-weight x bf16-activation GEMV (decode)
 * and GEMM (prefill).
 *
 * Sources, by page title and section:
 *  - CSDN article "bitsandbytes 是一个用于高效量化和加载大型语言模型（LLM）的开源库",
 *    section "数学原理对比": the NF4 codebook of 16 normal-quantile values in
 *    [-1, 1] with an exact 0, the per-block absmax scale, no zero-point; the
 *    closing remarks: fp4 as an E2M1-like format; section "实际性能差异":
 *    double quantization (weights to 4 bits, then the scales to 8 bits).
 *  - ossradar repository page for bitsandbytes, release notes 0.50.0 (fused
 *    4-bit dequantize + GEMM for inference; nested quantization fused in),
 *    0.50.2 (absmax store of a partial last block is masked), 0.49.2
 *    (blocksize 32 and 64 for 4-bit), and the gemv_4bit / quantize /
 *    dequantize op names.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned and allocated by the caller.
 *    The library never allocates, frees or synchronizes (except
 *    bnb4_device_status, which synchronizes the stream it is given).
 *  - Memory kinds (checked with cudaPointerGetAttributes before any launch):
 *    the linear entry points (bnb_gemv_4bit, bnb_gemm_4bit, bnb_linear_4bit)
 *    take device memory only, for x, y, bias and the weight's arrays (their
 *    larger tiers move tiles with TMA); quantize and dequantize take device
 *    or managed memory, and the quantize input x may also be page-locked host
 *    memory.  Any other pointer -- pageable host memory in particular, which
 *    a kernel cannot dereference -- returns BNB4_ERR_INVALID_ARG with nothing
 *    launched.
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Work is enqueued asynchronously on it.
 *  - Every call returns a status (BNB4_OK = 0, negative on error).  On an
 *    argument error nothing is launched and no memory is touched.  No C++
 *    exception crosses the ABI.
 *  - Tensors are dense and row-major.  A weight W[N, K] (out features N, in
 *    features K) is quantized as the flat array of N*K elements, so its
 *    blocks run along K.
 *  - Alignment: x / out / codes / X / Y pointers must be 16-byte aligned;
 *    fp32 arrays and absmax_q 4-byte aligned.  Misalignment returns
 *    BNB4_ERR_ALIGNMENT.
 *  - Results are deterministic for a given input and device: codes, absmax,
 *    double-quant fields and dequantized values are bit-identical to the
 *    reference definition below.  The GEMV / GEMM accumulate in fp32 and round
 *    once to bf16 at the end.
 *  - Every call is ordered after the stream's earlier work as a plain launch
 *    would be.  While the stream is being captured into a CUDA graph, the
 *    quantize, dequantize, decode and small-batch kernels that follow a
 *    kernel node are captured as programmatic dependents of it (they may
 *    start while it finishes and wait for it before reading or writing
 *    memory; only L2 prefetches of their inputs come earlier, and since L2
 *    is coherent across the GPU a prefetch never yields stale data);
 *    eagerly, and after any other node, they launch plainly.
 */
#ifndef BNB4_H_
#define BNB4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BNB4_ABI_VERSION 4

/* Every entry point is exported from the shared library (the library is
 * built with hidden visibility by default). */
#if defined(__GNUC__)
#define BNB4_API __attribute__((visibility("default")))
#else
#define BNB4_API
#endif

/* ----------------------------------------------------------- status codes */
#define BNB4_OK 0
#define BNB4_ERR_INVALID_ARG (-1)    /* null pointer, n <= 0, bad enum value */
#define BNB4_ERR_UNSUPPORTED (-2)    /* blocksize not 32/64/128/256, dtype */
#define BNB4_ERR_ALIGNMENT (-3)      /* a pointer misses its alignment */
#define BNB4_ERR_SHAPE (-4)          /* shape constraint (see each call) */
#define BNB4_ERR_WORKSPACE (-5)      /* workspace missing or too small */
#define BNB4_ERR_CUDA (-6)           /* a CUDA runtime call or launch failed */
#define BNB4_ERR_DEVICE_TIMEOUT (-7) /* a kernel's bounded wait expired */
#define BNB4_ERR_SCRATCH_LIMIT (-8)  /* input larger than the fixed scratch of
                                        bnb_quantize_4bit_noalloc */

/* -------------------------------------------------------------- enums */
#define BNB4_NF4 0  /* normal-quantile codebook */
#define BNB4_FP4 1  /* E2M1 magnitudes / 6, sign-magnitude codes */
#define BNB4_F32 0  /* fp32 element type */
#define BNB4_BF16 1 /* bf16 element type (raw 16-bit patterns) */
#define BNB4_F16 2  /* IEEE fp16 element type (raw 16-bit patterns) */

/*
 * Quantization state of n elements: the packed codes plus the block scales.
 * nb = ceil(n / blocksize) blocks of `blocksize` consecutive elements (the
 * last may be short); ng = ceil(nb / 256) double-quant groups.
 *
 *  codes     uint8[ceil(n/2)]: byte j = code[2j] << 4 | code[2j+1]; an odd n
 *            leaves the low nibble of the last byte 0.  16-byte aligned.
 *  absmax    float[nb]: exact per-block max |x|.  Written by quantize in both
 *            modes; read by the consumers only when double_quant == 0.
 *  absmax_q  uint8[nb]: u = q + 128, q = clamp(rint((absmax - offset) / s),
 *            -127, 127) with s the scale of the block's group (double quant).
 *            4-byte aligned.
 *  scale2    float[ng]: s = max |absmax - offset| over the group / 127.
 *  offset    float[1]: mean of absmax (fp64 sum, rounded to fp32).
 * The decoded scale of block b is fma(u_b - 128, scale2[b/256], offset) with
 * double quant, absmax[b] without.
 */
typedef struct bnb4_qstate {
  uint8_t* codes;
  float* absmax;
  uint8_t* absmax_q;
  float* scale2;
  float* offset;
  int64_t n;
  int32_t blocksize;
  int32_t qtype;
  int32_t double_quant;
  int32_t reserved; /* must be 0 */
} bnb4_qstate;

/* Byte sizes of every buffer of a quantization state of n elements. */
typedef struct bnb4_sizes {
  size_t codes;     /* ceil(n/2) */
  size_t absmax;    /* 4 * nb */
  size_t absmax_q;  /* nb (0 without double quant) */
  size_t scale2;    /* 4 * ng (0 without double quant) */
  size_t offset;    /* 4 (0 without double quant) */
  size_t workspace; /* scratch bnb_quantize_4bit needs (0 without dq) */
} bnb4_sizes;

/*
 * Fills *out with the buffer sizes for n elements.  Pure host function.
 * Errors: INVALID_ARG (n <= 0, out NULL), UNSUPPORTED (blocksize).
 */
BNB4_API int bnb4_query_sizes(int64_t n, int32_t blocksize, int32_t double_quant,
                     bnb4_sizes* out);

/*
 * Blockwise 4-bit quantization (NF4 article, section "数学原理对比": absmax
 * scale per block, nearest codebook entry, 16 codes packed two per byte;
 * section "实际性能差异": double quantization of the scales to 8 bits).
 *
 *  x           st->n elements of x_dtype (BNB4_F32, BNB4_BF16 or BNB4_F16;
 *              16-bit inputs are widened to fp32 exactly), 16-byte aligned,
 *              in device memory or in page-locked host memory (the kernel
 *              then reads the checkpoint over the bus and quantizes it on
 *              the way in, with no device copy of the unquantized tensor --
 *              the icman guide's quantize-when-moved-to-the-GPU step).
 *              Pageable host memory is rejected (INVALID_ARG).
 *  st          state whose buffers receive the result: codes and absmax
 *              always; absmax_q, scale2 and offset when st->double_quant.
 *  workspace   device scratch of at least bnb4_query_sizes(...).workspace
 *              bytes, 16-byte aligned (may be NULL when the size is 0).
 *              Any contents; every call overwrites what it reads.  Do not
 *              share one workspace between calls that may overlap on the
 *              GPU (different streams).
 * With double quantization two kernels run: the quantize kernel (codes,
 * absmax and one fp64 partial sum of the absmax per CTA), then, as a
 * programmatic dependent launch of it, the double quantization (the mean of
 * the partial sums in a fixed order, then the 8-bit codes of each group of
 * 256 absmax).
 * Per block: a = max|x|; r = RN(1/a) (0 for a = 0); v = RN(x*r); code =
 * number of fp32 codebook midpoints RN(RN(t[i]+t[i+1])*0.5) strictly below v
 * (FP4: of magnitude midpoints below |v|, sign bit set for v < 0 with a
 * non-zero magnitude).  Ties at a midpoint go to the lower index.
 * Bit-exact: codes, absmax, absmax_q, scale2 and offset equal the reference
 * definition for finite inputs; the offset equals it whenever the fp64 sum
 * of absmax is exact in every order (true for absmax values within ~29 -
 * log2(nb) binades of each other).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA.
 */
BNB4_API int bnb_quantize_4bit(const void* x, int32_t x_dtype, const bnb4_qstate* st,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Allocation-free variant of bnb_quantize_4bit with double quantization.
 * The pages describe no such call; it exists for callers that cannot
 * allocate device memory or pass a workspace -- for example a plugin whose
 * host framework owns every device allocation, or a latency-critical loader
 * that must not call cudaMalloc (which can synchronize the device or fail
 * under memory pressure).
 *
 * Same method and bit-identical results as bnb_quantize_4bit with
 * st->double_quant = 1, except that the exact fp32 absmax is not returned:
 * st->absmax is ignored (may be NULL) and the intermediate absmax and the
 * per-CTA fp64 partial sums of the grid-wide mean live in a fixed array in
 * the library's own device memory (32 KiB + 4 MiB per GPU that loads the
 * library, held until the process exits).  The caller passes x and the outputs codes, absmax_q,
 * scale2 and offset, with the alignment rules of bnb_quantize_4bit.
 *  - Limit: at most BNB4_NOALLOC_MAX_BLOCKS blocks (ceil(n / blocksize));
 *    larger inputs return BNB4_ERR_SCRATCH_LIMIT and launch nothing.
 *  - st->double_quant must be 1 (without double quantization
 *    bnb_quantize_4bit needs no workspace anyway): else INVALID_ARG.
 *  - x follows the rules of bnb_quantize_4bit (device, managed or
 *    page-locked host memory; pageable host memory returns INVALID_ARG);
 *    the outputs must be device or managed memory.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, once per device, with that device current).
 *    With lazy module loading (CUDA's default) that lookup also loads the
 *    array's module and maps its 4 MiB on the device, so the first call can
 *    return BNB4_ERR_CUDA when the device is out of memory: make it at
 *    start-up, before any stream capture on the device.
 *  - Every call shares the one array.  A call overwrites all of the scratch
 *    it reads, so no result carries over from the previous call; calls that
 *    overlap on the GPU (different streams) race on it and must be
 *    serialized by the caller.
 * Allocates nothing and calls no allocating routine.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, SCRATCH_LIMIT, CUDA.
 */
#define BNB4_NOALLOC_MAX_BLOCKS (1 << 20)
BNB4_API int bnb_quantize_4bit_noalloc(const void* x, int32_t x_dtype,
                                       const bnb4_qstate* st, void* stream);

/*
 * Quantization of a non-contiguous 2-D input (release notes 0.49.2:
 * quantize / dequantize handle non-contiguous tensors): x is a row-major
 * [rows, cols] view whose rows start ld elements apart.  Blocks run over the
 * logical row-major element order, so every output equals that of
 * bnb_quantize_4bit on the contiguous copy of the view, bit for bit.  x may
 * be device or page-locked host memory as for bnb_quantize_4bit.
 * Constraints: st->n == rows * cols < 2^32; ld >= cols; cols and ld
 * multiples of 8 elements (16-bit x_dtype) or 4 (fp32), so every row starts
 * on a 16-byte boundary.  ld == cols is the contiguous case.
 * Errors: as bnb_quantize_4bit, SHAPE for the view.
 */
BNB4_API int bnb_quantize_4bit_2d(const void* x, int32_t x_dtype, int64_t rows,
                                  int64_t cols, int64_t ld, const bnb4_qstate* st,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dequantization (NF4 article, section "实际性能差异": the 4-bit codes times
 * the decoded block scale).  w = RN(t[code] * a_hat) in fp32; with out_dtype
 * BNB4_BF16 or BNB4_F16 the output is the round-to-nearest-even of w in that
 * format (fp16: infinity past 65504, subnormals kept).  out: device, st->n
 * elements, 16-byte aligned.  Bit-exact to the reference definition.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA.
 */
BNB4_API int bnb_dequantize_4bit(const bnb4_qstate* st, void* out, int32_t out_dtype,
                        void* stream);

/*
 * Dequantization into a non-contiguous 2-D output (release notes 0.49.2):
 * out is a row-major [rows, cols] view, rows ld elements apart, device
 * memory; element (r, c) receives logical element r * cols + c, bit-equal to
 * bnb_dequantize_4bit.  Elements between the rows (ld > cols) are not
 * written.  Constraints: st->n == rows * cols < 2^32; ld >= cols; cols and
 * ld multiples of 8 (16-bit out_dtype) or 4 (fp32).
 * Errors: as bnb_dequantize_4bit, SHAPE for the view.
 */
BNB4_API int bnb_dequantize_4bit_2d(const bnb4_qstate* st, void* out, int32_t out_dtype,
                                    int64_t rows, int64_t cols, int64_t ld, void* stream);

/*
 * Decode GEMV (release notes 0.50.0 / gemv_4bit):
 *   y[b, n] = bf16( sum_k x[b, k] * What[n, k] ),  b < B, n < N,
 * What[n, k] = bf16(RN(t[code] * a_hat)) the dequantized weight, products
 * exact, fp32 accumulation (order unspecified), one final rounding to bf16.
 *  x  device bf16 [B, K], 16-byte aligned;   y  device bf16 [B, N].
 *  W  quantization state of the weight [N, K] (W->n == N*K).
 * Constraints: 1 <= B <= 256; K % 64 == 0; K % W->blocksize == 0; N, K <
 * 2^31.  B <= 8 runs the one-launch decode kernel (one CTA per 16 rows,
 * packed codes loaded straight into registers two K steps ahead; mma.sync,
 * one 8-column group; partial sums over K added in a fixed order, so
 * results are bit-reproducible) -- measured faster for a single weight than
 * the persistent TMA-staged kernel that bnb_gemv_4bit_grouped runs for long
 * lists; so does 9 <= B <= 16 when x and W->codes are 32-byte aligned (x
 * then the MMA's 16-row operand; measured faster than the small-batch
 * kernel); other batches run the small-batch tcgen05 kernel of
 * bnb_gemm_4bit.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, SHAPE, CUDA.
 */
BNB4_API int bnb_gemv_4bit(const void* x, int64_t B, int64_t K, const bnb4_qstate* W,
                  int64_t N, void* y, void* stream);

/*
 * Several decode GEMVs in one launch (release notes 0.50.0 / gemv_4bit, as
 * used by a decoder step: the linears that read the same activations, such
 * as q / k / v or gate / up, or any list of independent batch-B linears):
 * for every problem i,
 *   y_i[b, n] = h( sum_k x_i[b, k] * What_i[n, k] + bias_i[n] ),
 * the arithmetic of bnb_linear_4bit with M = B (exact products, fp32
 * accumulation, one rounding).  With B = 1 and 4 or more problems the list
 * runs one persistent grid (one CTA of 16 warps per SM, the packed weight
 * tiles staged in shared memory by 2-D TMA copies) that streams all the
 * weights, so the start-up of a launch is paid once for the whole list;
 * shorter lists and B > 1 run one launch of the bnb_gemv_4bit kernel over
 * the whole list (one CTA per 16 rows of any weight) -- each choice the
 * faster one measured on B200.  With the persistent grid the order of the
 * fp32 sums over K follows how the row groups of the whole list are split
 * over the SMs, so a problem's result can differ in the last bit from a
 * single call; the same list on the same device gives identical bits.
 *  problems  host array of `count` descriptors (read during the call only):
 *            x device [B, K] of dtype, 16-byte aligned; W the quantization
 *            state of the weight [N, K] (W.n == N * K); bias device [N] of
 *            dtype, 16-byte aligned, or NULL; y device [B, N] of dtype,
 *            2-byte aligned.  x may be shared between problems; the y must
 *            not overlap each other or any x.
 *  count     1 .. BNB4_GROUP_MAX.
 *  B         1 .. 8 rows of every x.
 *  dtype     BNB4_BF16 or BNB4_F16 (the compute type of every problem).
 * Constraints: every problem has the same K (K % 64 == 0, K % blocksize ==
 * 0, K < 2^31) and every W the same blocksize, qtype and double_quant (the
 * linears that share an input, such as q / k / v, satisfy both); N < 2^31.
 * Lists longer than 32 problems run as several launches of up to 32.
 * Errors: INVALID_ARG, UNSUPPORTED (dtype, or mixed weight formats),
 * ALIGNMENT, SHAPE (including different K), CUDA.
 */
#define BNB4_GROUP_MAX 256
typedef struct bnb4_gemv_problem {
  const void* x;
  bnb4_qstate W;
  int64_t K;
  int64_t N;
  const void* bias;
  void* y;
} bnb4_gemv_problem;
BNB4_API int bnb_gemv_4bit_grouped(const bnb4_gemv_problem* problems, int32_t count,
                                   int64_t B, int32_t dtype, void* stream);

/*
 * Test entry (no counterpart on the pages): bnb_gemv_4bit_grouped with the
 * persistent TMA-staged kernel for every list, whatever its length and B,
 * so that the parity tests cover that kernel on every shape.  Same arguments,
 * results (within the tolerance) and errors.
 */
BNB4_API int bnb4_debug_gemv_grouped_persistent(const bnb4_gemv_problem* problems,
                                                int32_t count, int64_t B, int32_t dtype,
                                                void* stream);

/*
 * Prefill GEMM with the dequantization fused in (release notes 0.50.0):
 *   Y[m, n] = bf16( sum_k X[m, k] * What[n, k] ),  fp32 accumulation in
 * tensor memory (tcgen05 bf16 MMA), What as in bnb_gemv_4bit.
 *  X  device bf16 [M, K], 16-byte aligned;   Y  device bf16 [M, N],
 *     16-byte aligned.
 *  W  quantization state of the weight [N, K] (W->n == N*K).
 * Constraints: M >= 1; N % 8 == 0; K % 64 == 0; K % W->blocksize == 0.
 * M <= 8 -- and 9 <= M <= 16 when X and W->codes are 32-byte aligned -- runs
 * the decode kernel of bnb_gemv_4bit, other M <= 256 the small-batch kernel
 * (the 128 weight rows of a CTA are the MMA's M side and the tokens its N;
 * K split over a cluster of up to 8 CTAs whose partial sums are added in
 * rank order), larger M the 2-CTA prefill kernel (512 x 256 output tiles).
 * All are deterministic.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, SHAPE, CUDA.
 */
BNB4_API int bnb_gemm_4bit(const void* X, int64_t M, int64_t K, const bnb4_qstate* W,
                  int64_t N, void* Y, void* stream);

/*
 * The fused 4-bit linear layer in either 16-bit compute type, with an
 * optional bias (release notes 0.50.0: fused 4-bit GEMM with the nested
 * quantization and the bias folded in, bf16 or fp16 activations; NF4
 * article, configuration section: the compute dtype is a setting):
 *   y[m, n] = h( sum_k x[m, k] * What[n, k] + bias[n] ),  m < M, n < N,
 * What[n, k] = h(RN(t[code] * a_hat)), h = round to nearest even in the
 * compute type `dtype` (BNB4_BF16 or BNB4_F16); products exact, fp32
 * accumulation, the bias added in fp32, one final rounding.
 *  x     device [M, K] of dtype, 16-byte aligned.
 *  bias  device [N] of dtype, 16-byte aligned, or NULL for none.
 *  y     device [M, N] of dtype; 2-byte aligned for M <= 256, 16-byte aligned
 *        above.
 *  W     quantization state of the weight [N, K] (W->n == N*K).
 * Constraints: M >= 1; K % 64 == 0; K % W->blocksize == 0; N % 8 == 0 when
 * M > 256.  The kernel follows M as in bnb_gemm_4bit (the decode kernel up to
 * 8 rows, or 16 with x and W->codes 32-byte aligned, the small-batch kernel
 * up to 256, the prefill kernel above); with
 * dtype BNB4_BF16 and no bias the result equals that of bnb_gemm_4bit /
 * bnb_gemv_4bit bit for bit.
 * Errors: INVALID_ARG, UNSUPPORTED (dtype), ALIGNMENT, SHAPE, CUDA.
 */
BNB4_API int bnb_linear_4bit(const void* x, int32_t dtype, int64_t M, int64_t K,
                             const bnb4_qstate* W, int64_t N, const void* bias, void* y,
                             void* stream);

/*
 * Synchronizes `stream`, then reads the library's device error word of the
 * current device: BNB4_OK, or BNB4_ERR_DEVICE_TIMEOUT when a kernel gave up a
 * bounded wait (its output is then incomplete).  clear != 0 resets the word.
 * Errors: CUDA.
 */
BNB4_API int bnb4_device_status(void* stream, int32_t clear);

/*
 * Failure-detection diagnostic (no counterpart on the pages).  Runs the
 * kernel of bnb_gemm_4bit (same arguments and checks) with its first X tile
 * never loaded and every mbarrier wait bounded by wait_limit_us (1 ..
 * 1,000,000): the kernel's waits run out, it sets the device error word,
 * drains what it started, releases its tensor memory and exits.  A following
 * bnb4_device_status reports BNB4_ERR_DEVICE_TIMEOUT and the context stays
 * usable.  Y receives no defined values.  Nothing traps or hangs.
 * Errors: as bnb_gemm_4bit, INVALID_ARG for the limit.
 */
BNB4_API int bnb4_debug_gemm_withhold(const void* X, int64_t M, int64_t K,
                                      const bnb4_qstate* W, int64_t N, void* Y,
                                      int32_t wait_limit_us, void* stream);

/*
 * Self-check of the quantize kernel's reciprocal (no counterpart on the
 * pages).  bnb_quantize_4bit computes r = RN(1/absmax) for an absmax in
 * [2^-126, 2^126) with an approximate reciprocal refined by Newton-Raphson
 * and Markstein's correction; this call compares that value, bit for bit,
 * with CUDA's round-to-nearest reciprocal for every fp32 input of the range
 * (2,113,929,216 values, a few milliseconds).
 *  result   device, 16 bytes, 8-byte aligned: receives {uint64 number of
 *           mismatching inputs, uint32 smallest mismatching bit pattern
 *           (0xffffffff when none), uint32 0}.  Overwritten, never read.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
BNB4_API int bnb4_debug_check_rcp(void* result, void* stream);

/* Static description of a status code; never NULL. */
BNB4_API const char* bnb4_strerror(int status);

/* BNB4_ABI_VERSION of the built library. */
BNB4_API int bnb4_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BNB4_H_ */
