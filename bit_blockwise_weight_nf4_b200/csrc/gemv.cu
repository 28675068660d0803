// gemv.cu -- decode GEMV with 4-bit weights on sm_100a:
//   y[b, n] = bf16( sum_k x[b, k] * What[n, k] ),  1 <= B <= 8,
//   What[n, k] = bf16(RN(t[code] * a_hat))   (dequantized weight, exact).
//
// Method: bitsandbytes' gemv_4bit op (ossradar page, release notes 0.50.0)
// over the blockwise NF4 / FP4 format of the CSDN article (section
// "数学原理对比"), nested (double) quantization decoded in-kernel.
//
// Design (HBM-bound on the packed bytes; integer-ALU heavy):
//  * A warp owns 8 weight rows and a share of K; its 4 lanes of one quad hold
//    one row, each lane a contiguous 64-element (32-byte) segment per
//    256-wide K step, loaded with two 128-bit loads.
//  * Per (row, quant block) each lane builds a 16-entry bf16 table of
//    bf16(RN(t[i] * a_hat)) -- bit-identical to dequantizing every element --
//    split into low-byte and high-byte tables held in 8 registers.
//  * 8 packed codes become 4 bf16x2 words with byte permutes (prmt): the low
//    3 bits of each code select from the two 8-entry halves, bit 3 picks the
//    half, a last permute interleaves low/high bytes.
//  * The products go through mma.sync m16n8k16 (bf16 -> fp32) with the weight
//    as the B operand (8 rows) and x as the A operand (batch rows, zero
//    padded).  K is permuted identically in both operands, which leaves the
//    dot products unchanged.
//  * The 8 warps of a CTA split K; partial sums are reduced in shared memory
//    in a fixed order and rounded once to bf16.
#include "common.cuh"
#include "kernels.h"

namespace bnb4 {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kKStep = 256;  // K covered by one warp step (4 lanes x 64)

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// bf16 table of one quant block, split by byte: L[q] holds the low bytes of
// entries 4q..4q+3, H[q] the high bytes.
struct Lut {
  uint32_t L[4], H[4];
};

template <int QT>
__device__ __forceinline__ Lut make_lut(float ah) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float t0 = QT == kQtNF4 ? nf4_value(2 * j)
                                  : ((2 * j) & 8 ? -fp4_magnitude((2 * j) & 7)
                                                 : fp4_magnitude((2 * j) & 7));
    const float t1 = QT == kQtNF4 ? nf4_value(2 * j + 1)
                                  : ((2 * j + 1) & 8 ? -fp4_magnitude((2 * j + 1) & 7)
                                                     : fp4_magnitude((2 * j + 1) & 7));
    P[j] = pack_bf16x2(__fmul_rn(t0, ah), __fmul_rn(t1, ah));
  }
  Lut l;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    l.L[q] = prmt(P[2 * q], P[2 * q + 1], 0x6420);
    l.H[q] = prmt(P[2 * q], P[2 * q + 1], 0x7531);
  }
  return l;
}

// Four codes in the low 16 bits of w (nibble order k1 k0 k3 k2) -> two bf16x2
// words {k0, k1}, {k2, k3}.
__device__ __forceinline__ void dq4(const Lut& l, uint32_t w, uint32_t& o01,
                                    uint32_t& o23) {
  const uint32_t sel = w & 0x7777u;
  const uint32_t mix = ((w >> 1) & 0x4444u) | 0x3210u;
  const uint32_t lo = prmt(prmt(l.L[0], l.L[1], sel), prmt(l.L[2], l.L[3], sel), mix);
  const uint32_t hi = prmt(prmt(l.H[0], l.H[1], sel), prmt(l.H[2], l.H[3], sel), mix);
  o01 = prmt(lo, hi, 0x4051);
  o23 = prmt(lo, hi, 0x6273);
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a2,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

template <int BS, int QT, bool DQ>
__global__ void __launch_bounds__(kThreads)
    gemv4_kernel(const uint16_t* __restrict__ x, int B, int64_t K,
                 const uint8_t* __restrict__ codes,
                 const float* __restrict__ absmax,
                 const uint8_t* __restrict__ absmax_q,
                 const float* __restrict__ scale2,
                 const float* __restrict__ offset, int64_t N,
                 uint16_t* __restrict__ y) {
  __shared__ float red[kWarps][32][2];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;  // weight row within the group / batch row of x
  const int t = lane & 3;   // K segment of the step
  const int64_t n = static_cast<int64_t>(blockIdx.x) * 8 + g;
  const bool row_ok = n < N;
  const bool x_ok = g < B;
  const float off = DQ ? __ldg(offset) : 0.0f;
  const int64_t steps = (K + kKStep - 1) / kKStep;
  const uint8_t* wrow = codes + n * (K / 2);
  const uint16_t* xrow = x + static_cast<int64_t>(g) * K;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};

  for (int64_t s = warp; s < steps; s += kWarps) {
    // this lane's segment; past a ragged K edge (K % 256 != 0) the lane
    // feeds zeros, since mma.sync needs every lane of the warp
    const int64_t k0 = s * kKStep + 64 * t;
    const bool seg_ok = k0 < K;
    uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
    Lut lut0, lut1;
    if (row_ok && seg_ok) {
      c0 = ldg_stream_v4(wrow + k0 / 2);
      c1 = ldg_stream_v4(wrow + k0 / 2 + 16);
      const int64_t b = (n * K + k0) / BS;
      lut0 = make_lut<QT>(decoded_absmax<DQ>(b, absmax, absmax_q, scale2, off));
      if constexpr (BS == 32)
        lut1 = make_lut<QT>(decoded_absmax<DQ>(b + 1, absmax, absmax_q, scale2, off));
      else
        lut1 = lut0;
    } else {
      lut0 = make_lut<QT>(0.0f);
      lut1 = lut0;
    }
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int p = 0; p < 8; ++p) {  // 8 codes = k0 + 8p .. +7: two MMAs
      uint4 xa = make_uint4(0, 0, 0, 0);
      if (x_ok && seg_ok)
        xa = __ldg(reinterpret_cast<const uint4*>(xrow + k0 + 8 * p));
      const Lut& l = (BS == 32 && p >= 4) ? lut1 : lut0;
      uint32_t b0, b1, b2, b3;
      dq4(l, cw[p], b0, b1);
      dq4(l, cw[p] >> 16, b2, b3);
      mma_bf16(acc, xa.x, xa.y, b0, b1);
      mma_bf16(acc, xa.z, xa.w, b2, b3);
    }
  }

  // acc[0], acc[1]: batch g, rows 2t, 2t+1 of the group (acc[2..3] padding)
  red[warp][lane][0] = acc[0];
  red[warp][lane][1] = acc[1];
  __syncthreads();
  if (warp == 0) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      s0 += red[w][lane][0];
      s1 += red[w][lane][1];
    }
    if (g < B) {
      const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 8 + 2 * t;
      const uint32_t o = pack_bf16x2(s0, s1);
      if (r0 < N) y[static_cast<int64_t>(g) * N + r0] = static_cast<uint16_t>(o);
      if (r0 + 1 < N)
        y[static_cast<int64_t>(g) * N + r0 + 1] = static_cast<uint16_t>(o >> 16);
    }
  }
}

template <int BS, int QT>
cudaError_t launch_bs(const void* x, int64_t B, int64_t K, const bnb4_qstate& W,
                      int64_t N, void* y, cudaStream_t s) {
  const int64_t grid = (N + 7) / 8;
  if (W.double_quant)
    gemv4_kernel<BS, QT, true><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), static_cast<int>(B), K, W.codes,
        W.absmax, W.absmax_q, W.scale2, W.offset, N, static_cast<uint16_t*>(y));
  else
    gemv4_kernel<BS, QT, false><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), static_cast<int>(B), K, W.codes,
        W.absmax, W.absmax_q, W.scale2, W.offset, N, static_cast<uint16_t*>(y));
  return cudaGetLastError();
}

template <int QT>
cudaError_t launch_q(const void* x, int64_t B, int64_t K, const bnb4_qstate& W,
                     int64_t N, void* y, cudaStream_t s) {
  switch (W.blocksize) {
    case 32: return launch_bs<32, QT>(x, B, K, W, N, y, s);
    case 64: return launch_bs<64, QT>(x, B, K, W, N, y, s);
    case 128: return launch_bs<128, QT>(x, B, K, W, N, y, s);
    default: return launch_bs<256, QT>(x, B, K, W, N, y, s);
  }
}

}  // namespace

cudaError_t launch_gemv(const void* x, int64_t B, int64_t K,
                        const bnb4_qstate& W, int64_t N, void* y, int num_sms,
                        cudaStream_t s) {
  (void)num_sms;
  return W.qtype == kQtNF4 ? launch_q<kQtNF4>(x, B, K, W, N, y, s)
                           : launch_q<kQtFP4>(x, B, K, W, N, y, s);
}

}  // namespace bnb4
