/*
 * bnb4_oracle.c -- plain, slow, single-threaded CPU oracle for 4-bit blockwise
 * NF4 / FP4 weight quantization, double quantization of the absmax array,
 * dequantization, and the fp64 reference of the 4-bit-weight linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no source with
 * the CUDA library and includes none of its headers.
 *
 * Sources (web pages on bitsandbytes, each cited by title and section):
 *  [NF4]  CSDN article "bitsandbytes 是一个用于高效量化和加载大型语言模型（LLM）的
 *         开源库", section "数学原理对比" (table rows 数值表示 / 缩放机制 / 零点)
 *         and section "实际性能差异" (row 训练稳定性: double quantization),
 *         and the closing remarks (fp4 is a simpler, E2M1-like format).
 *  [REL]  ossradar repository page for bitsandbytes, release notes 0.50.2
 *         (the absmax store of a partial last block is masked) and 0.49.2
 *         (blocksize 32 / 64 for 4-bit quantization), and the README, which
 *         cites the QLoRA paper for the 4-bit method.
 *
 * Readings where the pages are silent or garbled (each is also listed in the
 * design notes of the repository):
 *  R1  A block is `blocksize` consecutive elements of the flattened input; the
 *      last block may be short.  (The NF4 article's example of a square
 *      sub-matrix block is read as a garble; the release notes treat blocksize
 *      as an element count.)
 *  R2  absmax = max |x| over the block, exact in fp32 (the scale formula in the
 *      NF4 article is truncated right after the absolute value bar).
 *  R3  NF4 codebook: 16 normal quantiles (QLoRA construction): 8 positive
 *      quantiles at evenly spaced probabilities in (1/2, 1-delta], 7 negative
 *      ones in (1/2, 1-delta] mirrored, plus an exact 0, divided by the largest,
 *      delta = (1/32 + 1/30)/2.  It matches the printed -0.697 and -0.525; the
 *      printed positive 0.697 is read as a garble (a 16-entry table with an
 *      exact 0 cannot be symmetric).
 *  R4  FP4: sign-magnitude codes, bit 3 = sign, the magnitude index m = bits
 *      0..2 selects the E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} divided by 6.
 *  R5  Normalisation multiplies by the round-to-nearest fp32 reciprocal
 *      r = RN(1/absmax) (r = 0 for an all-zero block): v = RN(x * r).
 *  R6  Nearest code: code = number of midpoints strictly below v (ties at an
 *      exact midpoint go to the lower index); midpoints are fp32
 *      RN(RN(t[i] + t[i+1]) * 0.5).  FP4 applies this to |v| and sets the sign
 *      bit only when the magnitude index is non-zero (so -0 is never emitted).
 *  R7  Packing: byte j = (code[2j] << 4) | code[2j+1]; an odd tail leaves the
 *      low nibble of the last byte 0.
 *  R8  Double quantization (the weights are quantized to NF4 first, then their
 *      per-block scales to 8-bit integers): offset = fp32(sum(absmax) / nb), sum in fp64;
 *      c = RN(absmax - offset); groups of 256 consecutive entries, the last
 *      may be short; s = RN(max|c| / 127); q = clamp(rint(RN(c / s)), -127,
 *      127) (q = 0 when s = 0), stored as u = q + 128.  Codes are computed
 *      from the exact absmax, before double quantization.
 *  R9  Decoded absmax: a_hat = fma(u - 128, s, offset) with one rounding;
 *      dequantized weight w = RN(t[code] * a_hat); bf16 output = round to
 *      nearest even of w.
 *  R10 Linear layer reference: y = x . What^T summed in fp64, What being the
 *      bf16 dequantized weight (the operand the tensor cores consume).
 *  R11 fp16 compute type (the CSDN article's configuration section sets a
 *      compute dtype beside the quant type and the double-quant flag; the
 *      ossradar release notes' fused 4-bit GEMM takes fp16 or bf16
 *      activations): an fp16 input is decoded exactly to fp32 before the
 *      absmax; an fp16 dequantized weight is the IEEE binary16
 *      round-to-nearest-even of w (overflow to infinity); the fp16 linear
 *      layer uses fp16 x and What in R10.
 *  R12 Bias (the release notes fuse the bias into the 4-bit GEMM): y = x .
 *      What^T + bias[n], the bias in the compute type, added to the fp64 sum.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL (-1)

/* R3: NF4 codebook, ascending, exact 0 at index 7, endpoints -1 and +1. */
static const float kNF4[16] = {
    -0x1p+0f,          -0x1.647362p-1f, -0x1.0cd65cp-1f, -0x1.94653cp-2f,
    -0x1.234496p-2f,   -0x1.7a6a7ap-3f, -0x1.74f0d2p-4f, 0x0p+0f,
    0x1.45f602p-4f,    0x1.4995bep-3f,  0x1.f809b4p-3f,  0x1.5a066cp-2f,
    0x1.c3496ap-2f,    0x1.200f52p-1f,  0x1.722760p-1f,  0x1p+0f};

/* R4: FP4 (E2M1-style) magnitudes k/6 for k in {0, .5, 1, 1.5, 2, 3, 4, 6}. */
static const float kFP4Mag[8] = {
    0.0f,        0.5f / 6.0f, 1.0f / 6.0f, 1.5f / 6.0f,
    2.0f / 6.0f, 3.0f / 6.0f, 4.0f / 6.0f, 1.0f};

/* The 16 dequantization values of a code, indexed by the 4-bit code. */
static void codebook(int qtype, float t[16]) {
  int c;
  for (c = 0; c < 16; ++c) {
    if (qtype == 0) {
      t[c] = kNF4[c];
    } else {
      float m = kFP4Mag[c & 7];
      t[c] = (c & 8) ? -m : m;
    }
  }
}

int orc_codebook(int qtype, float* out16) {
  if (qtype != 0 && qtype != 1) return ORC_EINVAL;
  codebook(qtype, out16);
  return ORC_OK;
}

static float bf16_bits_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* R11: exact value of an IEEE binary16 bit pattern (1 sign bit, 5 exponent
 * bits with bias 15, 10 fraction bits; exponent field 0 = zero or subnormal
 * m * 2^-24, 31 = infinity or NaN). */
static float f16_bits_to_float(uint16_t h) {
  uint32_t sign = (uint32_t)(h >> 15) << 31;
  uint32_t e = (h >> 10) & 31u, m = h & 1023u, u;
  float f;
  if (e == 0) {
    f = (float)m * 0x1p-24f; /* exact: m < 2^10 */
    return sign ? -f : f;
  }
  if (e == 31)
    u = sign | 0x7f800000u | (m << 13);
  else
    u = sign | ((e + 112u) << 23) | (m << 13); /* rebias 15 -> 127 */
  memcpy(&f, &u, 4);
  return f;
}

float orc_f16_to_float(uint16_t h) { return f16_bits_to_float(h); }

/* R11: IEEE round-to-nearest-even of an fp32 value to binary16.  Values of
 * magnitude 65520 or more (the midpoint past the largest finite 65504) become
 * infinity; below 2^-14 the result is the subnormal RNE(|f| * 2^24) * 2^-24
 * (the scaling by 2^24 is exact and rintf rounds half to even); NaN stays NaN
 * with the quiet bit set. */
uint16_t orc_f16_rne(float f) {
  uint32_t u, sign, a;
  memcpy(&u, &f, 4);
  sign = (u >> 16) & 0x8000u;
  a = u & 0x7fffffffu;
  if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u | ((a >> 13) & 0x3ffu));
  if (a >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u); /* >= 65520 or inf */
  if (a >= 0x38800000u) {                                   /* >= 2^-14: normal */
    uint32_t r = a - 0x38000000u;                           /* exponent - 112 */
    r += 0x0fffu + ((r >> 13) & 1u);                        /* to nearest, ties even */
    return (uint16_t)(sign | (r >> 13));
  } else {
    float mag;
    memcpy(&mag, &a, 4);
    return (uint16_t)(sign | (uint32_t)rintf(mag * 0x1p24f));
  }
}

/* the element of an fp32 (0), bf16 (1) or fp16 (2) array as fp32 (exact) */
static float elem_f32(const void* x, int dtype, int64_t i) {
  if (dtype == 0) return ((const float*)x)[i];
  if (dtype == 1) return bf16_bits_to_float(((const uint16_t*)x)[i]);
  return f16_bits_to_float(((const uint16_t*)x)[i]);
}

/* R9: IEEE round-to-nearest-even of an fp32 value to bf16, from the bit
 * pattern; NaN stays NaN (quiet bit set). */
uint16_t orc_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* R6: code of one normalised value v. */
static int nearest_code(int qtype, float v) {
  int i, k = 0;
  if (qtype == 0) {
    for (i = 0; i < 15; ++i) {
      float mid = (kNF4[i] + kNF4[i + 1]) * 0.5f;
      if (v > mid) ++k;
    }
    return k;
  }
  {
    float av = fabsf(v);
    for (i = 0; i < 7; ++i) {
      float mid = (kFP4Mag[i] + kFP4Mag[i + 1]) * 0.5f;
      if (av > mid) ++k;
    }
    if (v < 0.0f && k > 0) k |= 8;
    return k;
  }
}

int orc_nearest_code(int qtype, float v) {
  if (qtype != 0 && qtype != 1) return ORC_EINVAL;
  return nearest_code(qtype, v);
}

static int valid_blocksize(int bs) {
  return bs == 32 || bs == 64 || bs == 128 || bs == 256;
}

/*
 * Quantize n elements (fp32 when x_dtype = 0, bf16 bit patterns when 1).
 * Writes codes[ceil(n/2)], absmax[nb] (always the exact fp32 absmax), and when
 * double_quant: absmax_q[nb], scale2[ceil(nb/256)], offset[1].
 * *sum_exact (may be NULL) is set to 1 when every partial sum of the absmax
 * array, in any order, is exact in fp64, i.e. when the mean does not depend on
 * the summation order (checked, not assumed).
 */
int orc_quantize_4bit(const void* x, int x_dtype, int64_t n, int blocksize,
                      int qtype, int double_quant, uint8_t* codes,
                      float* absmax, uint8_t* absmax_q, float* scale2,
                      float* offset, int* sum_exact) {
  int64_t nb, b, i;
  if (n <= 0 || !x || !codes || !absmax) return ORC_EINVAL;
  if (x_dtype != 0 && x_dtype != 1 && x_dtype != 2) return ORC_EINVAL;
  if (qtype != 0 && qtype != 1) return ORC_EINVAL;
  if (!valid_blocksize(blocksize)) return ORC_EINVAL;
  if (double_quant && (!absmax_q || !scale2 || !offset)) return ORC_EINVAL;

  nb = (n + blocksize - 1) / blocksize;
  memset(codes, 0, (size_t)((n + 1) / 2));

  for (b = 0; b < nb; ++b) {
    int64_t lo = b * blocksize;
    int64_t hi = lo + blocksize < n ? lo + blocksize : n;
    float a = 0.0f, r;
    /* R2 */
    for (i = lo; i < hi; ++i) {
      float xi = elem_f32(x, x_dtype, i);
      if (fabsf(xi) > a) a = fabsf(xi);
    }
    absmax[b] = a;
    /* R5 */
    r = a == 0.0f ? 0.0f : 1.0f / a;
    for (i = lo; i < hi; ++i) {
      float xi = elem_f32(x, x_dtype, i);
      float v = xi * r;
      int c = nearest_code(qtype, v);
      /* R7 */
      if (i % 2 == 0)
        codes[i / 2] |= (uint8_t)(c << 4);
      else
        codes[i / 2] |= (uint8_t)c;
    }
  }

  if (!double_quant) {
    if (sum_exact) *sum_exact = 1;
    return ORC_OK;
  }

  /* R8 */
  {
    double S = 0.0;
    int seq_exact = 1, emin = 1000;
    float off;
    int64_t ng = (nb + 255) / 256, g;
    for (b = 0; b < nb; ++b) {
      double a = (double)absmax[b];
      double s = S + a;
      double bb = s - S;
      double err = (S - (s - bb)) + (a - bb);
      if (err != 0.0) seq_exact = 0;
      S = s;
      if (absmax[b] != 0.0f) {
        int e;
        frexpf(absmax[b], &e);
        if (e < emin) emin = e;
      }
    }
    if (sum_exact) {
      /* every absmax is a multiple of unit = 2^(emin-24) (2^-149 at least);
       * if the total stays below 2^53 units, every partial sum in any order
       * is an exact fp64 number. */
      int ue = emin - 24 < -149 ? -149 : emin - 24;
      *sum_exact = seq_exact && (emin == 1000 || ldexp(S, -ue) < ldexp(1.0, 53));
    }
    off = (float)(S / (double)nb);
    offset[0] = off;
    for (g = 0; g < ng; ++g) {
      int64_t lo = g * 256, hi = lo + 256 < nb ? lo + 256 : nb;
      float M = 0.0f, s;
      for (b = lo; b < hi; ++b) {
        float c = absmax[b] - off;
        if (fabsf(c) > M) M = fabsf(c);
      }
      s = M / 127.0f;
      scale2[g] = s;
      for (b = lo; b < hi; ++b) {
        float c = absmax[b] - off;
        float q = 0.0f;
        if (s != 0.0f) {
          q = rintf(c / s);
          if (q > 127.0f) q = 127.0f;
          if (q < -127.0f) q = -127.0f;
        }
        absmax_q[b] = (uint8_t)((int)q + 128);
      }
    }
  }
  return ORC_OK;
}

/* R9: the decoded absmax of block b. */
static float decoded_absmax(int64_t b, int double_quant, const float* absmax,
                            const uint8_t* absmax_q, const float* scale2,
                            const float* offset) {
  if (!double_quant) return absmax[b];
  return fmaf((float)((int)absmax_q[b] - 128), scale2[b / 256], offset[0]);
}

/*
 * Dequantize n elements.  out_dtype 0 writes fp32 w, 1 writes bf16 bit
 * patterns (uint16), 2 fp16 bit patterns (R11).  Uses absmax when !double_quant, else absmax_q, scale2
 * and offset.
 */
int orc_dequantize_4bit(const uint8_t* codes, int64_t n, int blocksize,
                        int qtype, int double_quant, const float* absmax,
                        const uint8_t* absmax_q, const float* scale2,
                        const float* offset, void* out, int out_dtype) {
  float t[16];
  int64_t i;
  if (n <= 0 || !codes || !out) return ORC_EINVAL;
  if (qtype != 0 && qtype != 1) return ORC_EINVAL;
  if (!valid_blocksize(blocksize)) return ORC_EINVAL;
  if (out_dtype != 0 && out_dtype != 1 && out_dtype != 2) return ORC_EINVAL;
  if (double_quant ? (!absmax_q || !scale2 || !offset) : !absmax)
    return ORC_EINVAL;
  codebook(qtype, t);
  for (i = 0; i < n; ++i) {
    int c = (i % 2 == 0) ? (codes[i / 2] >> 4) : (codes[i / 2] & 15);
    float ah = decoded_absmax(i / blocksize, double_quant, absmax, absmax_q,
                              scale2, offset);
    float w = t[c] * ah;
    if (out_dtype == 0)
      ((float*)out)[i] = w;
    else if (out_dtype == 1)
      ((uint16_t*)out)[i] = orc_bf16_rne(w);
    else
      ((uint16_t*)out)[i] = orc_f16_rne(w);
  }
  return ORC_OK;
}

/*
 * R10, R11, R12: y[i][c] = sum_k x[rows[i]][k] * W[cols[c]][k] in fp64 (+
 * bias[cols[c]] when bias is not NULL), for x [M, K], W [N, K] and bias [N]
 * given as bf16 (dtype 1) or fp16 (dtype 2) bit patterns, row-major.
 * rows / cols may be NULL to mean all rows (n_rows = M) / all columns
 * (n_cols = N).
 */
int orc_linear_ref(const uint16_t* x, int dtype, int64_t M, int64_t K,
                   const int64_t* rows, int64_t n_rows, const uint16_t* W,
                   int64_t N, const int64_t* cols, int64_t n_cols,
                   const uint16_t* bias, double* y) {
  int64_t i, c, k;
  if (!x || !W || !y || M <= 0 || K <= 0 || N <= 0) return ORC_EINVAL;
  if (dtype != 1 && dtype != 2) return ORC_EINVAL;
  if (!rows) n_rows = M;
  if (!cols) n_cols = N;
  for (i = 0; i < n_rows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= M) return ORC_EINVAL;
    for (c = 0; c < n_cols; ++c) {
      int64_t nn = cols ? cols[c] : c;
      double acc = 0.0;
      if (nn < 0 || nn >= N) return ORC_EINVAL;
      for (k = 0; k < K; ++k)
        acc += (double)elem_f32(x, dtype, r * K + k) *
               (double)elem_f32(W, dtype, nn * K + k);
      if (bias) acc += (double)elem_f32(bias, dtype, nn);
      y[i * n_cols + c] = acc;
    }
  }
  return ORC_OK;
}
