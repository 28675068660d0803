// lut.cuh -- exact 4-bit -> 16-bit dequantization by byte permutes, shared
// by the linear kernels (decode GEMV, small-batch and prefill GEMM) and the
// dequantize kernel.
//
// A block's 16 dequantized values h(RN(t[c] * a_hat)) (h = round to the
// 16-bit compute format) are bit-identical to dequantizing every element
// (the CSDN article, section "数学原理对比": codebook value times the block
// scale).  The table is held split by byte in 8 registers; `prmt` (an
// 8-way byte select per output byte) looks codes up in it.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace bnb4 {
namespace {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// Per-block table of the 16 dequantized values in the 16-bit compute format
// F (BNB4_BF16 or BNB4_F16), split by byte: L[q] holds the low bytes of
// entries 4q..4q+3, H[q] the high bytes.
struct Lut {
  uint32_t L[4], H[4];
};

template <int QT>
__device__ __forceinline__ float table_value(int c) {
  if constexpr (QT == kQtNF4)
    return nf4_value(c);
  else
    return (c & 8) ? -fp4_magnitude(c & 7) : fp4_magnitude(c & 7);
}

template <int QT, int F>
__device__ __forceinline__ Lut make_lut(float ah) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    P[j] = pack2<F>(__fmul_rn(table_value<QT>(2 * j), ah),
                    __fmul_rn(table_value<QT>(2 * j + 1), ah));
  Lut l;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    l.L[q] = prmt(P[2 * q], P[2 * q + 1], 0x6420);
    l.H[q] = prmt(P[2 * q], P[2 * q + 1], 0x7531);
  }
  return l;
}

// 8 codes of one packed 32-bit word (natural order k0..k7) -> 8 16-bit
// values in k order as 4 words (pairs {k0,k1}, {k2,k3}, ...).  The low 3
// bits of each code select from the two 8-entry halves of the table, bit 3
// picks the half; one mask / shift of the whole word serves both 4-code
// halves (prmt reads the low 16 selector bits only).
__device__ __forceinline__ uint4 dq8(const Lut& l, uint32_t w) {
  const uint32_t sel = w & 0x77777777u;
  const uint32_t mix = ((w >> 1) & 0x44444444u) | 0x32103210u;
  uint4 o;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? sel >> 16 : sel;
    const uint32_t m = h ? mix >> 16 : mix;
    const uint32_t lo = prmt(prmt(l.L[0], l.L[1], s), prmt(l.L[2], l.L[3], s), m);
    const uint32_t hi = prmt(prmt(l.H[0], l.H[1], s), prmt(l.H[2], l.H[3], s), m);
    if (h == 0) {
      o.x = prmt(lo, hi, 0x4051);
      o.y = prmt(lo, hi, 0x6273);
    } else {
      o.z = prmt(lo, hi, 0x4051);
      o.w = prmt(lo, hi, 0x6273);
    }
  }
  return o;
}

// dq8 with its shifts on the FMA pipe: the byte permutes already keep the
// integer ALU pipe (half the FMA pipe's rate) busy, so the selector
// arithmetic uses multiply-high instead of shifts where it can.  k16 =
// 2^16 and k31 = 2^31 must come from a value the compiler cannot see (a
// kernel parameter), or it turns the multiplies back into shifts.
__device__ __forceinline__ uint32_t mulhi(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t madhi(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint4 dq8_fma(const Lut& l, uint32_t w, uint32_t k16, uint32_t k31) {
  const uint32_t sel = w & 0x77777777u;
  const uint32_t mix = madhi(w & 0x88888888u, k31, 0x32103210u);  // (bit 3 >> 1) | p
  uint4 o;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? mulhi(sel, k16) : sel;
    const uint32_t m = h ? mulhi(mix, k16) : mix;
    const uint32_t lo = prmt(prmt(l.L[0], l.L[1], s), prmt(l.L[2], l.L[3], s), m);
    const uint32_t hi = prmt(prmt(l.H[0], l.H[1], s), prmt(l.H[2], l.H[3], s), m);
    if (h == 0) {
      o.x = prmt(lo, hi, 0x4051);
      o.y = prmt(lo, hi, 0x6273);
    } else {
      o.z = prmt(lo, hi, 0x4051);
      o.w = prmt(lo, hi, 0x6273);
    }
  }
  return o;
}

}  // namespace
}  // namespace bnb4
