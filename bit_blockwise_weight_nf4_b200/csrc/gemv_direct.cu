// gemv_direct.cu -- decode GEMV with 4-bit weights on sm_100a, one CTA per 16
// weight rows: the kernel behind single GEMV calls, grouped calls of two or
// three weights at B = 1 and every grouped call at B > 1 (lists of four or
// more weights at B = 1 run the persistent TMA-staged kernel of gemv.cu;
// measured side by side on B200, this one is 10-17% faster for a single
// weight at B = 1 and 28-32% at B = 8), and of single linears with 9 to 16
// rows of x when x and the codes are 32-byte aligned.
//   y[b, n] = h( sum_k x[b, k] * What[n, k] + bias[n] ),  1 <= B <= 16,
//   What[n, k] = h(RN(t[code] * a_hat))   (dequantized weight, exact),
// h = round to the 16-bit compute format, bf16 or fp16 (nearest even); the
// bias is optional.
//
// Method: bitsandbytes' gemv_4bit op (ossradar page, release notes 0.50.0)
// over the blockwise NF4 / FP4 format of the CSDN article (section
// "数学原理对比"), nested (double) quantization decoded in-kernel.
//
// Design:
//  * One CTA (8 warps) per 16 weight rows, 2 CTAs resident per SM, as many
//    CTAs as row groups: the block scheduler overlaps one CTA's start-up
//    (first loads) with other CTAs' math.  The warps split K in 256-wide
//    steps; the 4 lanes of a quad own two rows (g and g + 8) and a
//    contiguous 64-element segment of each per step (a 256-bit load per
//    row straight into registers when the codes are 32-byte aligned, else
//    two 128-bit loads); every lane keeps 2 steps of loads (codes and raw
//    scales) in flight.
//  * Per (row, quant block) a lane builds the 16-entry table of
//    h(RN(t[i] * a_hat)) and looks codes up with byte permutes (lut.cuh;
//    shift-based selectors: the multiply-high form that helps the
//    persistent kernel measured 2-6% slower here).
//  * The products run on mma.sync m16n8k16 with the weight as the A operand
//    (16 rows) and x as B (batch columns, read just in time from L1, 32
//    bytes per load when aligned): K is permuted identically in both
//    operands, which leaves the dot products unchanged; two accumulator
//    chains keep consecutive MMAs independent; batch columns beyond B read a
//    valid row whose outputs are discarded.  For 9 to 16 rows the operands
//    swap (x the A operand, each weight row set the B operand), so every
//    weight is still dequantized once.
//  * The 8 warps' partial sums are added in shared memory in a fixed order,
//    the bias (if any) added in fp32, and rounded once.
//  * In a programmatic launch (below), before waiting on the previous
//    kernel, each CTA warms L2 with its own weight rows and with the rows of
//    the CTA one wave (the CTAs resident at once) later, which starts when a
//    CTA retires: every CTA's first loads then find their codes in L2
//    (measured on B200: 2-5% faster for a single MLP weight, 7% over a 7B
//    decoder pass of single calls).
//  * Inside a captured CUDA graph, after a kernel node, the launch is a
//    programmatic dependent of that kernel (common.cuh): it may be scheduled
//    while the kernel's last wave runs and waits for it before its first
//    global access (a 7B decoder pass replayed as a graph: 2.5% faster).
#include "common.cuh"
#include "kernels.h"
#include "l2warm.cuh"
#include "lut.cuh"

namespace bnb4 {
namespace {

constexpr int kWarps = 8;       // warps per CTA; they split K of one 16-row group
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerCta = 16;
constexpr int kKStep = 256;  // K covered by one warp step (4 lanes x 64)
constexpr int kChains = 2;   // independent MMA accumulators per warp
constexpr int kDirectListMax = 32;  // weights per launch of a list

// D[16 x 8] += A[16 x 16] (weight rows) * B[16 x 8] (x columns), bf16 or
// fp16 in (format F), fp32 accumulate.
template <int F>
__device__ __forceinline__ void mma16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                      uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (F == BNB4_F16)
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Raw scale inputs of one quant block, loaded ahead and decoded when used
// (so the decode never waits on a load issued just before it).
struct RawScale {
  uint32_t u;  // absmax_q byte (double quant) or absmax bits
  float s;     // scale2 of the block's group (double quant)
};

template <bool DQ>
__device__ __forceinline__ RawScale load_scale(int64_t b, const float* absmax,
                                               const uint8_t* absmax_q,
                                               const float* scale2) {
  RawScale r;
  if constexpr (DQ) {
    r.u = __ldg(absmax_q + b);
    r.s = __ldg(scale2 + (b >> 8));
  } else {
    r.u = __float_as_uint(__ldg(absmax + b));
    r.s = 0.0f;
  }
  return r;
}

template <bool DQ>
__device__ __forceinline__ float decode(const RawScale& r, float off) {
  if constexpr (DQ)
    return __fmaf_rn(static_cast<float>(static_cast<int>(r.u) - 128), r.s, off);
  else
    return __uint_as_float(r.u);
}

// Loads of one K step of one lane: 64 codes of each of its two rows and the
// scales of their blocks, issued kDepth steps ahead of their use.
struct StepBuf {
  uint4 c[2][2];       // [row g / g+8][16-byte half]
  RawScale a[2][2];    // [row][block within the segment (blocksize 32)]
};

// The weights of a launch: problem i owns row groups [rg0, rg0 + ceil(N /
// 16)) of the grid; all share K and the batch size.
struct DirectProb {
  const uint16_t* x;
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* scale2;
  const float* offset;
  const uint16_t* bias;
  uint16_t* y;
  int64_t N;
  int rg0;
};
template <int MAXP>
struct DirectList {
  DirectProb p[MAXP];
  int count;
};

// L2 warm-up of row group `cta` of the launch (its problem found from the
// list's row-group offsets), by one warp: lanes 0-15 the codes of one row
// each (K / 2 bytes: K is a multiple of 64 and the codes 16-byte aligned),
// lanes 16-31 the group's block scales line by line.
template <int BS, bool DQ, int MAXP>
__device__ __forceinline__ void warm_rows(const DirectList<MAXP>& L, int cta, int64_t K,
                                          int lane) {
  int q = 0;
  if constexpr (MAXP > 1)
    while (q + 1 < L.count && cta >= L.p[q + 1].rg0) ++q;
  const DirectProb& P = L.p[q];
  const int64_t row0 = static_cast<int64_t>(cta - P.rg0) * kRowsPerCta;
  const int64_t rows = P.N - row0 < kRowsPerCta ? P.N - row0 : kRowsPerCta;
  if (lane < kRowsPerCta) {
    if (lane < rows) prefetch_l2_range(P.codes + (row0 + lane) * (K / 2), K / 2);
  } else {
    const int64_t b0 = row0 * K / BS, nblk = rows * K / BS;
    const char* s = DQ ? reinterpret_cast<const char*>(P.absmax_q + b0)
                       : reinterpret_cast<const char*>(P.absmax + b0);
    const int64_t bytes = DQ ? nblk : 4 * nblk;
    for (int64_t o = static_cast<int64_t>(lane - kRowsPerCta) * 128; o < bytes;
         o += (32 - kRowsPerCta) * 128)
      prefetch_l2_line(s + o);
  }
}

// V8: every x and codes array of the launch is 32-byte aligned, so a lane
// reads a row's 32 code bytes of a step, and x for two MMAs, with one 256-bit
// load each (half the load instructions and, for B > 1, half the L1 lines
// that the loads of x touch: measured 7-18% faster at B = 8, up to 15% for a
// single weight at B = 1; not used for lists at B = 1, see launch_list).
// T16 (V8 only): 9 to 16 rows of x.  The MMAs swap roles: x is the A operand
// (16 rows: the lane's rows g and g + 8 of x), each of the lane's two weight
// rows the B operand of its own MMA (rows 0-7 and 8-15 of the group, one
// accumulator each, alternating); the lane dequantizes the same two rows as
// for B <= 8.
template <int BS, int QT, bool DQ, int kDepth, int F, int MAXP, bool V8, bool T16>
__global__ void __launch_bounds__(kThreads, 2)
    gemv4_direct_kernel(const __grid_constant__ DirectList<MAXP> L, int B, int64_t K,
                        int64_t ahead) {
  static_assert(V8 || !T16, "the 16-row form reads x with 256-bit loads");
  constexpr int kAcc = T16 ? 2 : kChains;  // accumulators (4 floats each) per lane
  __shared__ float red[kWarps][32][T16 ? 8 : 4];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;  // rows g and g + 8 of the group; row(s) g (and g + 8) of x
  const int t = lane & 3;   // K segment of the step
  int pi = 0;  // this CTA's problem
  if constexpr (MAXP > 1)
    while (pi + 1 < L.count && static_cast<int>(blockIdx.x) >= L.p[pi + 1].rg0) ++pi;
  const DirectProb& P = L.p[pi];
  const uint16_t* __restrict__ x = P.x;
  const uint8_t* __restrict__ codes = P.codes;
  const float* __restrict__ absmax = P.absmax;
  const uint8_t* __restrict__ absmax_q = P.absmax_q;
  const float* __restrict__ scale2 = P.scale2;
  const float* __restrict__ offset = P.offset;
  const uint16_t* __restrict__ bias = P.bias;
  uint16_t* __restrict__ y = P.y;
  const int64_t N = P.N;
  const int64_t row0 = static_cast<int64_t>(static_cast<int>(blockIdx.x) - P.rg0) * kRowsPerCta;
  const int64_t n[2] = {row0 + g, row0 + g + 8};
  const bool ok[2] = {n[0] < N, n[1] < N};
  const int64_t steps = (K + kKStep - 1) / kKStep;
  // programmatic dependent launch (inside a captured graph after a kernel):
  // the next kernel may be scheduled now; no global access before the
  // previous kernel has completed (x may be its output)
  pdl_trigger();
  // Warm L2 (l2warm.cuh) with this CTA's weight rows, while the previous
  // kernel may still run, and with the rows of the CTA `ahead` places later,
  // which an SM will most likely start when this one (or its neighbour)
  // retires: every CTA after the first `ahead` then finds its codes in L2.
  // ahead == 0 (a plain launch): no warm-up.
  if (ahead > 0) {
    if (warp == 0) warm_rows<BS, DQ>(L, static_cast<int>(blockIdx.x), K, lane);
    if (warp == 1 && static_cast<int64_t>(blockIdx.x) + ahead < gridDim.x)
      warm_rows<BS, DQ>(L, static_cast<int>(blockIdx.x) + ahead, K, lane);
  }
  pdl_wait();
  const float off = DQ ? __ldg(offset) : 0.0f;
  const int my_steps =
      warp < steps ? static_cast<int>((steps - warp + kWarps - 1) / kWarps) : 0;
  // rows of x beyond B read row B-1 (valid memory); their outputs are never
  // stored
  const uint16_t* xrow = x + static_cast<int64_t>(g < B ? g : B - 1) * K;
  const uint16_t* xrow8 = x + static_cast<int64_t>(g + 8 < B ? g + 8 : B - 1) * K;

  auto issue = [&](int i, StepBuf& b) {
    const int64_t k0 = (static_cast<int64_t>(i) * kWarps + warp) * kKStep + 64 * t;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (ok[r] && k0 < K) {
        const uint8_t* src = codes + n[r] * (K / 2) + k0 / 2;
        if constexpr (V8) {
          const U8x32 cc = ldg_stream_v8(src);
          b.c[r][0] = make_uint4(cc.v[0], cc.v[1], cc.v[2], cc.v[3]);
          b.c[r][1] = make_uint4(cc.v[4], cc.v[5], cc.v[6], cc.v[7]);
        } else {
          b.c[r][0] = ldg_stream_v4(src);
          b.c[r][1] = ldg_stream_v4(src + 16);
        }
        const int64_t blk = (n[r] * K + k0) / BS;
        b.a[r][0] = load_scale<DQ>(blk, absmax, absmax_q, scale2);
        if constexpr (BS == 32) b.a[r][1] = load_scale<DQ>(blk + 1, absmax, absmax_q, scale2);
      } else {
        b.c[r][0] = make_uint4(0, 0, 0, 0);
        b.c[r][1] = b.c[r][0];
        b.a[r][0] = RawScale{0u, 0.0f};
        b.a[r][1] = b.a[r][0];
      }
    }
  };

  float acc[kAcc][4] = {};
  StepBuf buf[kDepth];
#pragma unroll
  for (int d = 0; d < kDepth; ++d)
    if (d < my_steps) issue(d, buf[d]);

  for (int base = 0; base < my_steps; base += kDepth) {
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      const int i = base + d;
      if (i < my_steps) {  // warp-uniform
        const int64_t k0 = (static_cast<int64_t>(i) * kWarps + warp) * kKStep + 64 * t;
        const bool seg = k0 < K;
        // past a ragged K edge or the N edge the lane's rows are zero codes
        // with a zero scale: mma.sync needs every lane of the warp
        Lut lut[2][2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          lut[r][0] = make_lut<QT, F>(ok[r] && seg ? decode<DQ>(buf[d].a[r][0], off) : 0.0f);
          lut[r][1] = BS == 32
                          ? make_lut<QT, F>(ok[r] && seg ? decode<DQ>(buf[d].a[r][1], off) : 0.0f)
                          : lut[r][0];
        }
        const int64_t kx = seg ? k0 : 0;  // x stays in bounds on a ragged edge
        U8x32 xq, xq8;  // V8: x at k0 + 8p .. +15 (rows g and g + 8)
#pragma unroll
        for (int p = 0; p < 8; ++p) {  // codes k0 + 8p .. +7 of both rows: two MMAs
          uint4 xb, xc;  // x at k0 + 8p .. +7: row g (and row g + 8)
          if constexpr (V8) {
            if ((p & 1) == 0) {
              xq = ldg_v8(xrow + kx + 8 * p);
              if constexpr (T16) xq8 = ldg_v8(xrow8 + kx + 8 * p);
            }
            const int q = (p & 1) * 4;
            xb = make_uint4(xq.v[q], xq.v[q + 1], xq.v[q + 2], xq.v[q + 3]);
            if constexpr (T16) xc = make_uint4(xq8.v[q], xq8.v[q + 1], xq8.v[q + 2], xq8.v[q + 3]);
          } else {
            xb = __ldg(reinterpret_cast<const uint4*>(xrow + kx + 8 * p));
          }
          const int h = p >> 2, wi = p & 3;
          const uint32_t w0 = wi == 0 ? buf[d].c[0][h].x : wi == 1 ? buf[d].c[0][h].y
                            : wi == 2 ? buf[d].c[0][h].z : buf[d].c[0][h].w;
          const uint32_t w1 = wi == 0 ? buf[d].c[1][h].x : wi == 1 ? buf[d].c[1][h].y
                            : wi == 2 ? buf[d].c[1][h].z : buf[d].c[1][h].w;
          const uint4 o0 = dq8(lut[0][BS == 32 ? h : 0], w0);
          const uint4 o1 = dq8(lut[1][BS == 32 ? h : 0], w1);
          if constexpr (T16) {
            mma16<F>(acc[0], xb.x, xc.x, xb.y, xc.y, o0.x, o0.y);
            mma16<F>(acc[1], xb.x, xc.x, xb.y, xc.y, o1.x, o1.y);
            mma16<F>(acc[0], xb.z, xc.z, xb.w, xc.w, o0.z, o0.w);
            mma16<F>(acc[1], xb.z, xc.z, xb.w, xc.w, o1.z, o1.w);
          } else {
            mma16<F>(acc[(2 * p) % kChains], o0.x, o1.x, o0.y, o1.y, xb.x, xb.y);
            mma16<F>(acc[(2 * p + 1) % kChains], o0.z, o1.z, o0.w, o1.w, xb.z, xb.w);
          }
        }
        if (i + kDepth < my_steps) issue(i + kDepth, buf[d]);
      }
    }
  }

  if constexpr (T16) {
    // acc[a]: rows 8a + 2t, 8a + 2t + 1 of the group (1, 3: the second) for
    // rows g (0, 1) and g + 8 (2, 3) of x
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int v = 0; v < 4; ++v) red[warp][lane][4 * a + v] = acc[a][v];
  } else {
    // acc[.]: rows g (0, 1) and g + 8 (2, 3) of the group, batch columns 2t
    // and 2t + 1
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kChains; ++c) sum += acc[c][v];
      red[warp][lane][v] = sum;
    }
  }
  __syncthreads();
  if (warp == 0) {
    if constexpr (T16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][lane][e];
        const int64_t row = row0 + 8 * (e >> 2) + 2 * t + (e & 1);
        const int xr = g + 8 * ((e >> 1) & 1);
        if (row < N && xr < B) {
          if (bias) v = __fadd_rn(v, half_to_f32<F>(bias[row]));
          const uint32_t o = pack2<F>(v, 0.0f);
          y[static_cast<int64_t>(xr) * N + row] = static_cast<uint16_t>(o);
        }
      }
    } else {
      float s[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        s[v] = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s[v] += red[w][lane][v];
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          const int bcol = 2 * t + cb;
          if (ok[r] && bcol < B) {
            float v = s[2 * r + cb];
            if (bias) v = __fadd_rn(v, half_to_f32<F>(bias[n[r]]));
            const uint32_t o = pack2<F>(v, 0.0f);
            y[static_cast<int64_t>(bcol) * N + n[r]] = static_cast<uint16_t>(o);
          }
        }
      }
    }
  }
}

template <int BS, int QT, bool DQ, int F, int MAXP>
cudaError_t launch_t(const DirectList<MAXP>& L, int64_t grid, int64_t B, int64_t K, bool v8,
                     int64_t ahead, cudaStream_t s) {
  const bool prog = programmatic_after_kernel(s);
  // L2 warm-up only in a programmatic launch, where it overlaps the previous
  // kernel: in a plain launch the first wave's prefetches of the next wave's
  // rows compete with its own first loads (measured on B200: a 7B decoder
  // pass of eager launches 2.56 -> 2.80 ms with the warm-up on)
  if (!prog) ahead = 0;
  // two K steps of loads in flight per lane (for K <= 4096 that is all of a
  // warp's share), 2 CTAs of 8 warps resident per SM
  const dim3 grd(static_cast<unsigned>(grid)), blk(kThreads);
  if constexpr (MAXP == 1) {
    if (B > 8)  // single weights only; the caller checked v8
      return launch_kernel(gemv4_direct_kernel<BS, QT, DQ, 2, F, MAXP, true, true>, grd, blk,
                           0, s, prog, L, static_cast<int>(B), K, ahead);
  }
  if (v8)
    return launch_kernel(gemv4_direct_kernel<BS, QT, DQ, 2, F, MAXP, true, false>, grd, blk, 0,
                         s, prog, L, static_cast<int>(B), K, ahead);
  return launch_kernel(gemv4_direct_kernel<BS, QT, DQ, 2, F, MAXP, false, false>, grd, blk, 0, s,
                       prog, L, static_cast<int>(B), K, ahead);
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <int MAXP>
cudaError_t launch_list(const GemvLinear* lin, int count, int64_t B, int fmt, int num_sms,
                        cudaStream_t s) {
  DirectList<MAXP> L{};
  L.count = count;
  int64_t rg = 0;
  bool v8 = true;  // every x and codes array 32-byte aligned
  for (int i = 0; i < count; ++i) {
    const GemvLinear& l = lin[i];
    v8 = v8 && aligned32(l.x) && aligned32(l.W->codes);
    DirectProb& p = L.p[i];
    p.x = static_cast<const uint16_t*>(l.x);
    p.codes = l.W->codes;
    p.absmax = l.W->absmax;
    p.absmax_q = l.W->absmax_q;
    p.scale2 = l.W->scale2;
    p.offset = l.W->offset;
    p.bias = static_cast<const uint16_t*>(l.bias);
    p.y = static_cast<uint16_t*>(l.y);
    p.N = l.N;
    p.rg0 = static_cast<int>(rg);
    rg += (l.N + kRowsPerCta - 1) / kRowsPerCta;
  }
  if (B > 8 && (MAXP != 1 || !v8)) return cudaErrorInvalidValue;  // see gemv_direct_takes
  // lists at B = 1 keep the 128-bit loads: measured on B200, 256-bit ones
  // cost them 1-3% (two 11008 x 4096 weights: 14.6 -> 15.0 us each) and a
  // 7B decoder pass 2%, while single weights gain up to 15% (4096^2: 7.1 ->
  // 6.1 us) and every B > 1 launch 7-18%
  if (MAXP != 1 && B == 1) v8 = false;
  const bnb4_qstate& W = *lin[0].W;
  const int64_t K = lin[0].K;
  // CTAs resident at once (2 per SM): the distance of the row group a CTA
  // warms L2 for, one wave ahead
  const int64_t ahead = 2 * static_cast<int64_t>(num_sms);
  const bool dq = W.double_quant != 0;
  const bool nf4 = W.qtype == kQtNF4;
  const bool f16 = fmt == BNB4_F16;
#define BNB4_DIRECT_LAUNCH(BSV)                                                                    \
  if (nf4)                                                                                         \
    return dq ? (f16 ? launch_t<BSV, kQtNF4, true, BNB4_F16, MAXP>(L, rg, B, K, v8, ahead, s)      \
                     : launch_t<BSV, kQtNF4, true, BNB4_BF16, MAXP>(L, rg, B, K, v8, ahead, s))    \
              : (f16 ? launch_t<BSV, kQtNF4, false, BNB4_F16, MAXP>(L, rg, B, K, v8, ahead, s)     \
                     : launch_t<BSV, kQtNF4, false, BNB4_BF16, MAXP>(L, rg, B, K, v8, ahead, s));  \
  return dq ? (f16 ? launch_t<BSV, kQtFP4, true, BNB4_F16, MAXP>(L, rg, B, K, v8, ahead, s)        \
                   : launch_t<BSV, kQtFP4, true, BNB4_BF16, MAXP>(L, rg, B, K, v8, ahead, s))      \
            : (f16 ? launch_t<BSV, kQtFP4, false, BNB4_F16, MAXP>(L, rg, B, K, v8, ahead, s)       \
                   : launch_t<BSV, kQtFP4, false, BNB4_BF16, MAXP>(L, rg, B, K, v8, ahead, s));
  switch (W.blocksize) {
    case 32: BNB4_DIRECT_LAUNCH(32)
    case 64: BNB4_DIRECT_LAUNCH(64)
    case 128: BNB4_DIRECT_LAUNCH(128)
    default: BNB4_DIRECT_LAUNCH(256)
  }
#undef BNB4_DIRECT_LAUNCH
}

}  // namespace

bool gemv_direct_takes(const void* x, const bnb4_qstate& W, int64_t B) {
  return B >= 1 && (B <= 8 || (B <= 16 && aligned32(x) && aligned32(W.codes)));
}

cudaError_t launch_gemv_direct(const void* x, int64_t B, int64_t K, const bnb4_qstate& W,
                               int64_t N, void* y, const void* bias, int fmt, int num_sms,
                               cudaStream_t s) {
  const GemvLinear one{x, &W, K, N, bias, y};
  return launch_list<1>(&one, 1, B, fmt, num_sms, s);
}

cudaError_t launch_gemv_direct_list(const GemvLinear* lin, int count, int64_t B, int fmt,
                                    int num_sms, cudaStream_t s) {
  if (count == 1) return launch_list<1>(lin, 1, B, fmt, num_sms, s);
  for (int i = 0; i < count; i += kDirectListMax) {
    const int c = count - i < kDirectListMax ? count - i : kDirectListMax;
    const cudaError_t e = launch_list<kDirectListMax>(lin + i, c, B, fmt, num_sms, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bnb4
