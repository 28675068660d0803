// quant.cu -- blockwise 4-bit quantization on sm_100a.
//
// Method (CSDN article on bitsandbytes, section "数学原理对比"; release notes
// 0.50.2 and 0.49.2 on the ossradar repository page):
//   per block of `blocksize` consecutive elements: a = max|x| (exact fp32);
//   r = RN(1/a) (0 for a = 0); v = RN(x * r); code = number of codebook
//   midpoints strictly below v (FP4: magnitude midpoints below |v| plus the
//   sign bit for a negative value with a non-zero magnitude); two codes per
//   byte, first element in the high nibble; the absmax store of a partial last
//   block is masked.
// Double quantization (same article, section "实际性能差异"): offset = mean of
//   absmax (fp64 sum), c = RN(a - offset), per group of 256: s = RN(max|c| /
//   127), u = clamp(rint(RN(c / s)), -127, 127) + 128.
//
// Design (HBM-bound; the instruction budget per element decides how close to
// the bound it runs): a persistent grid of 256-thread CTAs, exactly the
// resident ones (3 per SM).  Each warp streams whole tiles of 8 rows x 512
// contiguous bytes with 128-bit non-allocating loads, refilling each row's
// register slot with the next tile's row as soon as it is consumed (8 loads
// in flight per lane at all times).  Per row a lane holds one 16-byte chunk
// of a block; the block absmax is an xor-shuffle reduction among the lanes
// that hold it.  Addresses are lane pointers advanced once per tile, rows
// are immediate offsets.  The common case -- an absmax in [2^-126, 2^126),
// warp-uniformly -- takes a branch-free path:
//   * 1/a from the approximate reciprocal refined to the correctly rounded
//     value (Newton-Raphson step plus Markstein's final correction);
//   * nearest code: one FMA buckets v into 1/32-wide intervals (the integer
//     lands in the mantissa bits of 1.5 * 2^23 + v * 32), one lane-private
//     shared-memory lookup of {candidate midpoint, midpoints below the
//     bucket}, one compare;
//   * the chunk's packed word is built by a Horner chain p = 16 p + code in
//     the nibble order of the byte layout, so no shifts or ors are needed.
// Any other row group (zero, subnormal or huge absmax, infinities) and the
// one ragged tile at the end take an exact out-of-line path with the
// correctly rounded reciprocal and a clamped lookup.  The double
// quantization runs as a second, tiny kernel that first reduces the per-CTA
// fp64 partial sums in a fixed order.
#include "common.cuh"
#include "kernels.h"
#include "l2warm.cuh"

namespace bnb4 {
namespace {

constexpr int kThreads = 256;
constexpr int kCtasPerSm = 3;       // resident CTAs per SM (register cap)
constexpr int kRows = 8;            // 16-byte chunks per lane per tile
constexpr int kLutEntries = 128;    // the fast path masks the bucket to 7 bits
// v is bucketed as j = rint(32 v) + 32 with one FMA against 1.5 * 2^23 + 32:
// the integer lands in the mantissa bits.
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;
constexpr int kLutBuckets = 65;  // buckets reached by |v| <= 1 (+ rounding)

// The FP4 code of v (a finite value away from every decision point; used
// only to label the table's buckets): the magnitude midpoints strictly below
// |v|, plus the sign bit for a negative value with a non-zero magnitude.
__device__ uint32_t fp4_code_at(float v) {
  uint32_t m = 0;
  const float a = fabsf(v);
#pragma unroll
  for (int i = 0; i < 7; ++i)
    m += __fmul_rn(__fadd_rn(fp4_magnitude(i), fp4_magnitude(i + 1)), 0.5f) < a ? 1u : 0u;
  return v < 0.0f && m != 0 ? m + 8u : m;
}

// Bucket table, replicated per lane: entry (j, lane) at lut[j * 32 + lane],
// for buckets 1/32 wide over v in [-1, 1] (j = rint(32 v) + 32).  The code
// of v changes at most once inside a bucket (decision points are at least
// 0.08 apart; a bucket widened by 1e-3 on each side holds at most one), at
// the candidate cand (+inf where there is none).
//  NF4: entry {cand, base}; code = base + (v > cand), base counting the
//       midpoints below the bucket.
//  FP4: entry {cand, lo | hi << 8}; code = v > cand ? hi : lo.  Its codes
//       are sign-magnitude: a positive midpoint m changes the code where
//       v > m, a negative one (-m) where v >= -m, stored as the float just
//       below -m so that the same comparison decides.
// Entries past the reachable buckets are {+inf, 0}: only a NaN lands there,
// and its code is 0 (no midpoint is below NaN).
template <int QT>
__device__ void build_lut(uint2* lut) {
  // one thread per entry computes it into lane slot 0 ...
  if (threadIdx.x < kLutEntries) {
    const int j = threadIdx.x;
    uint32_t word = 0;
    float cand = __int_as_float(0x7f800000);
    if (j < kLutBuckets) {
      const float center = static_cast<float>(j - 32);
      const float lo = (center - 0.5f) / 32.0f - 1e-3f;
      const float hi = (center + 0.5f) / 32.0f + 1e-3f;
      if constexpr (QT == kQtNF4) {
        int base = 0;
#pragma unroll
        for (int i = 0; i < 15; ++i) {
          const float mid = __fmul_rn(__fadd_rn(nf4_value(i), nf4_value(i + 1)), 0.5f);
          if (mid < lo) ++base;
          else if (mid <= hi) cand = mid;
        }
        word = static_cast<uint32_t>(base);
      } else {
        float d = 0.0f;  // the decision point in the bucket, if any
        bool has = false;
#pragma unroll
        for (int i = 0; i < 7; ++i) {
          const float mid = __fmul_rn(__fadd_rn(fp4_magnitude(i), fp4_magnitude(i + 1)), 0.5f);
          if (mid >= lo && mid <= hi) {
            cand = mid;
            d = mid;
            has = true;
          }
          if (-mid >= lo && -mid <= hi) {  // v >= -mid  <=>  v > (the float below -mid)
            cand = __int_as_float(__float_as_int(-mid) + 1);
            d = -mid;
            has = true;
          }
        }
        // the codes on either side of the decision point (other decision
        // points are >= 0.08 away), or the bucket's one code at its center
        const uint32_t c_lo = fp4_code_at(has ? d - 1e-4f : center / 32.0f);
        const uint32_t c_hi = has ? fp4_code_at(d + 1e-4f) : c_lo;
        word = c_lo | (c_hi << 8);
      }
    }
    lut[j * 32] = make_uint2(__float_as_uint(cand), word);
  }
  __syncthreads();
  // ... and every thread replicates entries to the other lane slots
  for (int idx = threadIdx.x; idx < kLutEntries * 32; idx += blockDim.x)
    if (idx & 31) lut[idx] = lut[idx & ~31];
}

// Exact nearest code for any v (infinite and NaN included): the bucket is
// clamped in the float domain.  A NaN (maxNum drops it) lands in bucket 0,
// whose NF4 base is the NaN's code 0 (no midpoint is below NaN); FP4's
// bucket 0 holds the code of v near -1, so a NaN returns 0 first.
template <int QT>
__device__ __forceinline__ uint32_t code_of(float v, const uint2* lut_lane) {
  if constexpr (QT == kQtFP4)
    if (v != v) return 0u;
  const float f = fminf(fmaxf(__fmaf_rn(v, 32.0f, kMagic + 32.0f), kMagic),
                        kMagic + 64.0f);
  const int j = __float_as_int(f) - kMagicBits;
  const uint2 e = lut_lane[j * 32];
  const bool above = v > __uint_as_float(e.x);
  if constexpr (QT == kQtNF4)
    return e.y + (above ? 1u : 0u);
  else
    return above ? (e.y >> 8) & 0xffu : e.y & 0xffu;
}

// One Horner step of the fast path, p * 16 + code(v), for |v| <= 1 + 2^-23
// (finite block, absmax in the normal range) or NaN: the bucket index is then
// 0..64 (127 for the canonical NaN) without clamping, the 7-bit mask only
// keeps the address inside the table, and the code follows the entry as in
// code_of.  lut_addr = shared address of this lane's slot of bucket 0.
// "v > cand" is the sign bit of cand - v (exact: both are floats, the
// difference of distinct ones is never rounded to zero, an infinite cand
// gives +inf, and a NaN -- the canonical one, sign clear -- compares false),
// so the compare runs on the FMA pipe as a subtraction.  Written out in PTX:
// NF4 adds the sign bit to base + 16 p; FP4 uses it to pick the entry's lo or
// hi byte with one byte permute.
template <int QT>
__device__ __forceinline__ uint32_t horner_code(uint32_t p, float v, uint32_t lut_addr) {
  uint32_t out;
  if constexpr (QT == kQtNF4) {
    asm("{\n\t.reg .b32 f, j, a, c, b, d, s, t;\n\t"
        "fma.rn.f32 f, %1, 0f42000000, 0f4B400020;\n\t"  // v * 32 + 1.5 * 2^23 + 32
        "and.b32 j, f, 127;\n\t"
        "mad.lo.u32 a, j, 256, %2;\n\t"
        "ld.shared.v2.u32 {c, b}, [a];\n\t"
        "sub.rn.f32 d, c, %1;\n\t"    // negative exactly when v > cand
        "mad.lo.u32 t, %3, 16, b;\n\t"
        "shr.u32 s, d, 31;\n\t"
        "add.u32 %0, t, s;\n\t}"
        : "=r"(out)
        : "f"(v), "r"(lut_addr), "r"(p));
  } else {
    asm("{\n\t.reg .b32 f, j, a, c, b, d, s, k;\n\t"
        "fma.rn.f32 f, %1, 0f42000000, 0f4B400020;\n\t"  // v * 32 + 1.5 * 2^23 + 32
        "and.b32 j, f, 127;\n\t"
        "mad.lo.u32 a, j, 256, %2;\n\t"
        "ld.shared.v2.u32 {c, b}, [a];\n\t"
        "sub.rn.f32 d, c, %1;\n\t"    // negative exactly when v > cand
        "shr.u32 s, d, 31;\n\t"
        "or.b32 s, s, 0x4440;\n\t"    // byte 1 (hi) or 0 (lo) of b, upper bytes 0
        "prmt.b32 k, b, 0, s;\n\t"
        "mad.lo.u32 %0, %3, 16, k;\n\t}"
        : "=r"(out)
        : "f"(v), "r"(lut_addr), "r"(p));
  }
  return out;
}

// Correctly rounded 1/a for a in [2^-126, 2^126): the hardware approximate
// reciprocal y0 (within an ulp), one Newton-Raphson step y1 = y0 + y0 (1 -
// a y0), then Markstein's correction y1 + y1 (1 - a y1), whose residual is
// exact in one fma and whose last fma rounds once (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).  The result equals the
// correctly rounded reciprocal for every input of the range (checked
// exhaustively against the round-to-nearest division by the library's
// debug entry point bnb4_debug_check_rcp).
__device__ __forceinline__ float rcp_rn_normal(float a) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(a));
  float e = __fmaf_rn(-a, y, 1.0f);
  y = __fmaf_rn(e, y, y);
  e = __fmaf_rn(-a, y, 1.0f);
  return __fmaf_rn(e, y, y);
}

// a in [2^-126, 2^126) -- the range of rcp_rn_normal.
__device__ __forceinline__ bool normal_scale(float a) {
  return __float_as_uint(a) - 0x00800000u < 0x7e000000u;
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kPerChunk = 4;
  __device__ static float get(const uint4& c, int i) {
    const uint32_t w = i == 0 ? c.x : i == 1 ? c.y : i == 2 ? c.z : c.w;
    return __uint_as_float(w);
  }
  __device__ static uint4 load_partial(const float* x, int64_t e, int64_t n) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = e + i < n ? __float_as_uint(__ldg(x + e + i)) : 0u;
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Elem<uint16_t> {  // bf16 bit patterns
  static constexpr int kPerChunk = 8;
  __device__ static float get(const uint4& c, int i) {
    const uint32_t w = (i >> 1) == 0 ? c.x : (i >> 1) == 1 ? c.y
                       : (i >> 1) == 2 ? c.z : c.w;
    return (i & 1) ? bf16_hi(w) : bf16_lo(w);
  }
  __device__ static uint4 load_partial(const uint16_t* x, int64_t e,
                                       int64_t n) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = e + 2 * i < n ? __ldg(x + e + 2 * i) : 0u;
      const uint32_t hi = e + 2 * i + 1 < n ? __ldg(x + e + 2 * i + 1) : 0u;
      w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// fp16 input: IEEE binary16 patterns, decoded exactly to fp32.
struct Half16 {
  uint16_t bits;
};
template <>
struct Elem<Half16> {
  static constexpr int kPerChunk = 8;
  __device__ static float get(const uint4& c, int i) {
    const uint32_t w = (i >> 1) == 0 ? c.x : (i >> 1) == 1 ? c.y
                       : (i >> 1) == 2 ? c.z : c.w;
    return half_to_f32<BNB4_F16>((i & 1) ? w >> 16 : w);
  }
  __device__ static uint4 load_partial(const Half16* x, int64_t e, int64_t n) {
    return Elem<uint16_t>::load_partial(reinterpret_cast<const uint16_t*>(x), e, n);
  }
};

// Block absmax of a row group: the lane's chunk(s), then an xor-shuffle
// reduction over the lanes holding the block (for LPB = 64 the two rows of
// the group hold one block across the whole warp).
template <typename T, int LPB, int RG>
__device__ __forceinline__ float group_absmax(const uint4* ch) {
  constexpr int EPL = Elem<T>::kPerChunk;
  float m = 0.0f;
#pragma unroll
  for (int rr = 0; rr < RG; ++rr)
#pragma unroll
    for (int i = 0; i < EPL; ++i) m = fmaxf(m, fabsf(Elem<T>::get(ch[rr], i)));
  constexpr int kFirst = LPB == 64 ? 16 : LPB / 2;
#pragma unroll
  for (int o = kFirst; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// Exact path for one chunk (any absmax, any bounds): the correctly rounded
// reciprocal (0 for a zero block), the clamped lookup, padding nibbles of
// elements at or past n set to 0, and a store that stays inside the
// ceil(n/2) code bytes.  Out of line: it runs for rare row groups and the
// one ragged tile, and keeps the streaming loop small.
template <typename T, int QT>
__device__ __noinline__ void chunk_exact(uint4 ch, float m, int64_t e, int64_t n,
                                         uint8_t* codes, const uint2* lut_lane) {
  constexpr int EPL = Elem<T>::kPerChunk;
  const float inv = m == 0.0f ? 0.0f : __frcp_rn(m);
  uint32_t p = 0;
#pragma unroll
  for (int q = EPL / 2 - 1; q >= 0; --q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * q + h;
      uint32_t c = code_of<QT>(__fmul_rn(Elem<T>::get(ch, i), inv), lut_lane);
      if (e + i >= n) c = 0u;
      p = p * 16u + c;
    }
  }
  uint8_t* dst = codes + e / 2;
  if (e + EPL <= n) {
    if constexpr (EPL == 8)
      *reinterpret_cast<uint32_t*>(dst) = p;
    else
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(p);
  } else {
    const int64_t nbytes = (n + 1) / 2;
#pragma unroll
    for (int j = 0; j < EPL / 2; ++j)
      if (e / 2 + j < nbytes) dst[j] = static_cast<uint8_t>(p >> (8 * j));
  }
}

// STR: x is a row-major [n / v.cols, v.cols] view with rows v.ld elements
// apart (16-byte aligned rows, n < 2^32); blocks still run over the logical
// element order, so the results equal those of the contiguous tensor.
template <typename T, int BS, int QT, bool DQ, bool STR>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    quant4_kernel(const T* __restrict__ x, int64_t n,
                  uint8_t* __restrict__ codes, float* __restrict__ absmax,
                  double* __restrict__ partials, View2D v, bool warm) {
  constexpr int EPL = Elem<T>::kPerChunk;  // elements per 16-byte chunk
  constexpr int LPB = BS / EPL;            // lanes (chunks) per block
  constexpr int ROW = 32 * EPL;            // elements per warp row
  constexpr int TILE = kRows * ROW;        // elements per warp tile
  constexpr int RG = LPB == 64 ? 2 : 1;    // rows per block group
  static_assert(LPB == 64 || (LPB >= 4 && LPB <= 32), "blocksize");
  static_assert(TILE % BS == 0, "tile must hold whole blocks");

  extern __shared__ uint2 lut[];
  __shared__ double red[kThreads / 32];
  pdl_trigger();  // the double-quant kernel may be scheduled early
  // Warm L2 (l2warm.cuh) with the warp's first tile of x, one 128-byte line
  // per lane (a tile is 32 lanes x 8 chunks of 16 bytes), while a previous
  // kernel may still run (`warm`: a programmatic launch on device memory).
  if (!STR && warm) {
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
    if (t0 < n / TILE)
      prefetch_l2_line(reinterpret_cast<const char*>(x + t0 * TILE) + (threadIdx.x & 31) * 128);
  }
  build_lut<QT>(lut);
  __syncthreads();
  // launched programmatically (inside a captured graph after a kernel): no
  // global access before the previous kernel has completed
  pdl_wait();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint2* lut_lane = lut + lane;
  const uint32_t lut_addr = static_cast<uint32_t>(__cvta_generic_to_shared(lut_lane));
  const int64_t nb = (n + BS - 1) / BS;
  const int64_t n_full = n / TILE;  // tiles entirely inside n
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const bool writer = LPB == 64 ? lane == 0 : (lane % LPB) == 0;
  double acc = 0.0;

  int64_t tile = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
  if (tile < n_full) {
    // lane pointers at row 0 of the current tile; rows are immediate offsets
    const int64_t e0 = tile * TILE + lane * EPL;
    const T* xp = x + e0;
    uint8_t* cp = codes + e0 / 2;
    float* ap = absmax + tile * (TILE / BS) + (LPB == 64 ? 0 : lane / LPB);
    const int64_t stride = n_warps * TILE;
    uint4 c[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      c[r] = STR ? ldg_stream_v4(x + view_offset(e0 + r * ROW, v)) : ldg_stream_v4(xp + r * ROW);
    for (; tile < n_full; tile += n_warps) {
      // the last tile of the warp refills from itself (the loads are unused)
      const T* xn = tile + n_warps < n_full ? xp + stride : xp;
      const int64_t en = (tile + n_warps < n_full ? tile + n_warps : tile) * TILE + lane * EPL;
#pragma unroll
      for (int r0 = 0; r0 < kRows; r0 += RG) {
        const float m = group_absmax<T, LPB, RG>(c + r0);
        if (writer) ap[r0 * ROW / BS] = m;
        if constexpr (DQ) acc += static_cast<double>(writer ? m : 0.0f);
        if (__any_sync(0xffffffffu, !normal_scale(m))) {
#pragma unroll
          for (int rr = 0; rr < RG; ++rr)
            chunk_exact<T, QT>(c[r0 + rr], m, tile * TILE + lane * EPL + (r0 + rr) * ROW,
                               n, codes, lut_lane);
        } else {
          const float inv = rcp_rn_normal(m);
#pragma unroll
          for (int rr = 0; rr < RG; ++rr) {
            const int r = r0 + rr;
            uint32_t p = 0;
#pragma unroll
            for (int q = EPL / 2 - 1; q >= 0; --q) {
              p = horner_code<QT>(p, __fmul_rn(Elem<T>::get(c[r], 2 * q), inv), lut_addr);
              p = horner_code<QT>(p, __fmul_rn(Elem<T>::get(c[r], 2 * q + 1), inv), lut_addr);
            }
            if constexpr (EPL == 8)
              *reinterpret_cast<uint32_t*>(cp + r * ROW / 2) = p;
            else
              *reinterpret_cast<uint16_t*>(cp + r * ROW / 2) = static_cast<uint16_t>(p);
          }
        }
#pragma unroll
        for (int rr = 0; rr < RG; ++rr)
          c[r0 + rr] = STR ? ldg_stream_v4(x + view_offset(en + (r0 + rr) * ROW, v))
                           : ldg_stream_v4(xn + (r0 + rr) * ROW);
      }
      xp = xn;
      cp += stride / 2;
      ap += stride / BS;
    }
  }

  // the ragged tile (elements n_full * TILE .. n - 1) belongs to the warp
  // whose tile sequence reaches it
  if (n % TILE != 0 && tile == n_full) {
    const int64_t t0 = n_full * TILE;
#pragma unroll 1
    for (int r0 = 0; r0 < kRows; r0 += RG) {
      uint4 ch[RG];
#pragma unroll
      for (int rr = 0; rr < RG; ++rr) {
        const int64_t e = t0 + static_cast<int64_t>((r0 + rr) * 32 + lane) * EPL;
        if constexpr (STR)  // whole chunks (n and the rows are chunk multiples)
          ch[rr] = e < n ? ldg_stream_v4(x + view_offset(e, v)) : make_uint4(0, 0, 0, 0);
        else
          ch[rr] = Elem<T>::load_partial(x, e, n);
      }
      const float m = group_absmax<T, LPB, RG>(ch);
      const int64_t b = (t0 + static_cast<int64_t>(r0) * ROW) / BS +
                        (LPB == 64 ? 0 : lane / LPB);
      if (writer && b < nb) {
        absmax[b] = m;
        if constexpr (DQ) acc += static_cast<double>(m);
      }
#pragma unroll
      for (int rr = 0; rr < RG; ++rr) {
        const int64_t e = t0 + static_cast<int64_t>((r0 + rr) * 32 + lane) * EPL;
        if (e < n) chunk_exact<T, QT>(ch[rr], m, e, n, codes, lut_lane);
      }
    }
  }

  if constexpr (DQ) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double s = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) s += red[w];
      partials[blockIdx.x] = s;
    }
  }
}

// Double quantization of the absmax array: one warp per group of 256 blocks
// (grid-strided over the groups).  Every CTA first reduces the per-CTA
// partial sums of the quantize kernel in the same fixed order -- thread i
// adds partials i, i + 256, ... (independent loads, one round trip, shared
// with the loads of the warp's first group), then a fixed xor tree per warp
// and the 8 warp sums in order -- so all CTAs agree on the offset; the sum
// is exact whenever the absmax values span few enough binades, and then
// equals the oracle's sequential sum.
constexpr int kDqThreads = 256;

__global__ void __launch_bounds__(kDqThreads)
    dq_absmax_kernel(const float* __restrict__ absmax, int64_t nb,
                     const double* __restrict__ partials, int n_partials,
                     uint8_t* __restrict__ absmax_q, float* __restrict__ scale2,
                     float* __restrict__ offset) {
  __shared__ double red[kDqThreads / 32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t ng = (nb + 255) / 256;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (kDqThreads / 32);
  int64_t g = static_cast<int64_t>(blockIdx.x) * (kDqThreads / 32) + warp;
  // entries g*256 + lane + 32 j of the warp's group (coalesced); 0 past nb
  auto load_group = [&](int64_t grp, float (&a)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t b = grp * 256 + lane + 32 * j;
      a[j] = grp < ng && b < nb ? __ldg(absmax + b) : 0.0f;
    }
  };
  pdl_trigger();  // a programmatic launch after this one may be scheduled early
  pdl_wait();     // the quantize kernel's absmax and partial sums are complete
  // the warp's first group is requested together with the partial sums, so
  // the two loads share one round trip
  float a[8];
  load_group(g, a);
  double sum = 0.0;
  for (int i = threadIdx.x; i < n_partials; i += kDqThreads) sum += partials[i];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = 0.0;
#pragma unroll
  for (int w = 0; w < kDqThreads / 32; ++w) sum += red[w];
  const float off = static_cast<float>(sum / static_cast<double>(nb));
  if (blockIdx.x == 0 && threadIdx.x == 0) offset[0] = off;

  for (; g < ng; g += stride) {
    float c[8];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t b = g * 256 + lane + 32 * j;
      c[j] = b < nb ? __fsub_rn(a[j], off) : 0.0f;
      m = fmaxf(m, fabsf(c[j]));
    }
    load_group(g + stride, a);  // the next group of this warp (zeros past ng)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sg = __fdiv_rn(m, 127.0f);
    if (lane == 0) scale2[g] = sg;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t b = g * 256 + lane + 32 * j;
      if (b < nb) {
        float q = 0.0f;
        if (sg != 0.0f) q = fminf(fmaxf(rintf(__fdiv_rn(c[j], sg)), -127.0f), 127.0f);
        absmax_q[b] = static_cast<uint8_t>(static_cast<int>(q) + 128);
      }
    }
  }
}

// Every fp32 input of rcp_rn_normal's range against __frcp_rn.
constexpr uint32_t kRcpFirst = 0x00800000u;              // 2^-126
constexpr uint32_t kRcpCount = 0x7e800000u - kRcpFirst;  // up to 2^126

__global__ void check_rcp_init(unsigned long long* res) {
  res[0] = 0ull;
  res[1] = 0xffffffffull;
}

__global__ void __launch_bounds__(256) check_rcp_kernel(unsigned long long* res) {
  unsigned long long bad = 0;
  uint32_t first = 0xffffffffu;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < kRcpCount; i += stride) {
    const uint32_t bits = kRcpFirst + i;
    const float a = __uint_as_float(bits);
    if (__float_as_uint(rcp_rn_normal(a)) != __float_as_uint(__frcp_rn(a))) {
      ++bad;
      first = min(first, bits);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    bad += __shfl_xor_sync(0xffffffffu, bad, o);
    first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
  }
  if ((threadIdx.x & 31) == 0 && bad != 0) {
    atomicAdd(res, bad);
    // the low word of res[1] holds the smallest mismatching pattern; the
    // high word stays 0
    atomicMin(reinterpret_cast<unsigned long long*>(res + 1),
              static_cast<unsigned long long>(first));
  }
}

template <typename T, int BS, int QT, bool DQ>
cudaError_t launch_quant(const void* x, int64_t n, uint8_t* codes,
                         float* absmax, double* partials, int grid, const View2D* view,
                         bool warm, cudaStream_t s) {
  const size_t smem = kLutEntries * 32 * sizeof(uint2);
  const bool prog = programmatic_after_kernel(s);
  if (view)
    return launch_kernel(quant4_kernel<T, BS, QT, DQ, true>, dim3(grid), dim3(kThreads), smem,
                         s, prog, static_cast<const T*>(x), n, codes, absmax, partials, *view,
                         false);
  // the L2 warm-up only where it overlaps a previous kernel
  return launch_kernel(quant4_kernel<T, BS, QT, DQ, false>, dim3(grid), dim3(kThreads), smem, s,
                       prog, static_cast<const T*>(x), n, codes, absmax, partials, View2D{},
                       warm && prog);
}

template <typename T, int QT, bool DQ>
cudaError_t dispatch_bs(int bs, const void* x, int64_t n, uint8_t* codes,
                        float* absmax, double* partials, int grid, const View2D* view,
                        bool warm, cudaStream_t s) {
  switch (bs) {
    case 32:
      return launch_quant<T, 32, QT, DQ>(x, n, codes, absmax, partials, grid, view, warm, s);
    case 64:
      return launch_quant<T, 64, QT, DQ>(x, n, codes, absmax, partials, grid, view, warm, s);
    case 128:
      return launch_quant<T, 128, QT, DQ>(x, n, codes, absmax, partials, grid, view, warm, s);
    default:
      return launch_quant<T, 256, QT, DQ>(x, n, codes, absmax, partials, grid, view, warm, s);
  }
}

template <typename T>
cudaError_t dispatch_q(int qt, bool dq, int bs, const void* x, int64_t n,
                       uint8_t* codes, float* absmax, double* partials,
                       int grid, const View2D* view, bool warm, cudaStream_t s) {
  if (qt == kQtNF4)
    return dq ? dispatch_bs<T, kQtNF4, true>(bs, x, n, codes, absmax, partials, grid, view,
                                             warm, s)
              : dispatch_bs<T, kQtNF4, false>(bs, x, n, codes, absmax, partials, grid, view,
                                              warm, s);
  return dq ? dispatch_bs<T, kQtFP4, true>(bs, x, n, codes, absmax, partials, grid, view, warm,
                                           s)
            : dispatch_bs<T, kQtFP4, false>(bs, x, n, codes, absmax, partials, grid, view,
                                            warm, s);
}

}  // namespace

cudaError_t launch_check_rcp(void* result, cudaStream_t s) {
  auto* res = static_cast<unsigned long long*>(result);
  cudaError_t e = launch_kernel(check_rcp_init, dim3(1), dim3(1), 0, s, false, res);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  return launch_kernel(check_rcp_kernel, dim3(sms * 8), dim3(256), 0, s, false, res);
}

int quant_grid(int64_t n, int x_dtype, int num_sms) {
  const int64_t epl = x_dtype == BNB4_F32 ? 4 : 8;
  const int64_t tile = kRows * 32 * epl;
  const int64_t tiles = (n + tile - 1) / tile;
  const int64_t ctas = (tiles + kThreads / 32 - 1) / (kThreads / 32);
  int64_t g = static_cast<int64_t>(num_sms) * kCtasPerSm;
  if (ctas < g) g = ctas;
  if (g > kMaxPartials) g = kMaxPartials;
  return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_quantize(const void* x, int x_dtype, const bnb4_qstate& st,
                            void* workspace, int* err, int num_sms, cudaStream_t s,
                            const View2D* view, bool warm_x) {
  (void)err;  // no bounded waits here
  const bool dq = st.double_quant != 0;
  const int grid = quant_grid(st.n, x_dtype, num_sms);
  double* partials = static_cast<double*>(workspace);
  cudaError_t e =
      x_dtype == BNB4_F32
          ? dispatch_q<float>(st.qtype, dq, st.blocksize, x, st.n, st.codes,
                              st.absmax, partials, grid, view, warm_x, s)
      : x_dtype == BNB4_F16
          ? dispatch_q<Half16>(st.qtype, dq, st.blocksize, x, st.n, st.codes,
                               st.absmax, partials, grid, view, warm_x, s)
          : dispatch_q<uint16_t>(st.qtype, dq, st.blocksize, x, st.n, st.codes,
                                 st.absmax, partials, grid, view, warm_x, s);
  if (e != cudaSuccess || !dq) return e;
  const int64_t nb = (st.n + st.blocksize - 1) / st.blocksize;
  const int64_t ng = (nb + 255) / 256;
  const int64_t warps_per_cta = kDqThreads / 32;
  int64_t g2 = (ng + warps_per_cta - 1) / warps_per_cta;
  if (g2 > 2048) g2 = 2048;
  // programmatic: its predecessor is always the quantize kernel just launched
  return launch_kernel(dq_absmax_kernel, dim3(static_cast<unsigned>(g2)), dim3(kDqThreads),
                       0, s, true, static_cast<const float*>(st.absmax), nb,
                    static_cast<const double*>(partials), grid, st.absmax_q, st.scale2,
                    st.offset);
}

}  // namespace bnb4
