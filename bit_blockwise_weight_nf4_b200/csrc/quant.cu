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
// Design (HBM-bound): a persistent grid of 256-thread CTAs, exactly the
// resident ones (3 per SM); each warp streams tiles of 8 x 512 contiguous
// bytes with 128-bit non-allocating loads, refilling each row's register slot
// with the next tile's row as soon as it is consumed (8 loads in flight per
// lane at all times), reduces each block's absmax with xor shuffles among the
// lanes that hold it, and writes the packed codes with one coalesced
// 16/32-bit store per lane and row.  The nearest-code search is one
// fused multiply-add that buckets v into 1/32-wide intervals, one shared-
// memory lookup of {candidate midpoint, codes below it} (lane-replicated, so
// conflict free) and one compare.  The double quantization runs as a second,
// tiny kernel that first reduces the per-CTA fp64 partial sums in a fixed
// order.
#include "common.cuh"
#include "kernels.h"

namespace bnb4 {
namespace {

constexpr int kThreads = 256;
constexpr int kCtasPerSm = 3;       // resident CTAs per SM (register cap)
constexpr int kRows = 8;            // 16-byte chunks per lane per tile
constexpr int kLutBuckets = 65;     // buckets j = 0..64 reached by finite values
constexpr int kLutEntries = 128;    // the fast path masks the bucket to 7 bits
// v is bucketed as j = rint(32 v) + 32 (NF4) or rint(32 |v|) (FP4) with one
// FMA against 1.5 * 2^23 (+32): the integer lands in the mantissa bits.
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

// Bucket table, replicated per lane: entry (j, lane) at lut[j * 32 + lane].
// For every v whose bucket is j, code = base + (v > cand), where base counts
// the midpoints below the bucket and cand is the only midpoint inside it (or
// +inf).  Buckets are 1/32 wide; codebook midpoints are at least 0.08 apart, so
// a bucket widened by 1e-3 on each side holds at most one.
template <int QT>
__device__ void build_lut(uint2* lut) {
  constexpr int nm = QT == kQtNF4 ? 15 : 7;
  // one thread per bucket computes its entry into lane slot 0 (entries past
  // the last reachable bucket repeat it: only non-finite input lands there)
  if (threadIdx.x < kLutEntries) {
    const int j = threadIdx.x < kLutBuckets ? threadIdx.x : kLutBuckets - 1;
    const float center = QT == kQtNF4 ? static_cast<float>(j - 32)
                                      : static_cast<float>(j);
    const float lo = (center - 0.5f) / 32.0f - 1e-3f;
    const float hi = (center + 0.5f) / 32.0f + 1e-3f;
    int base = 0;
    float cand = __int_as_float(0x7f800000);
#pragma unroll
    for (int i = 0; i < nm; ++i) {
      const float a = QT == kQtNF4 ? nf4_value(i) : fp4_magnitude(i);
      const float b = QT == kQtNF4 ? nf4_value(i + 1) : fp4_magnitude(i + 1);
      const float mid = __fmul_rn(__fadd_rn(a, b), 0.5f);
      if (mid < lo) ++base;
      else if (mid <= hi) cand = mid;
    }
    lut[threadIdx.x * 32] = make_uint2(__float_as_uint(cand), static_cast<uint32_t>(base));
  }
  __syncthreads();
  // ... and every thread replicates entries to the other lane slots
  for (int idx = threadIdx.x; idx < kLutEntries * 32; idx += blockDim.x)
    if (idx & 31) lut[idx] = lut[idx & ~31];
}

template <int QT>
__device__ __forceinline__ uint32_t code_of(float v, const uint2* lut_lane) {
  if constexpr (QT == kQtNF4) {
    // clamp in the float domain: keeps NaN (maxNum drops it) and out-of-range
    // values inside the table, with the same result as counting midpoints.
    const float f = fminf(fmaxf(__fmaf_rn(v, 32.0f, kMagic + 32.0f), kMagic),
                          kMagic + 64.0f);
    const int j = __float_as_int(f) - kMagicBits;
    const uint2 e = lut_lane[j * 32];
    return e.y + (v > __uint_as_float(e.x) ? 1u : 0u);
  } else {
    const float a = fabsf(v);
    const float f =
        fminf(fmaxf(__fmaf_rn(a, 32.0f, kMagic), kMagic), kMagic + 32.0f);
    const int j = __float_as_int(f) - kMagicBits;
    const uint2 e = lut_lane[j * 32];
    const uint32_t m = e.y + (a > __uint_as_float(e.x) ? 1u : 0u);
    return (v < 0.0f && m != 0u) ? (m | 8u) : m;
  }
}

__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

// Fast nearest code for |v| <= 1 + 2^-23, which holds whenever the block's
// reciprocal 1/absmax is finite and the input finite: the bucket index is
// then 0..64 without clamping.  The 7-bit mask only keeps non-finite input
// inside the table (its code is unspecified).  lut_addr = shared address of
// this lane's slot of bucket 0.
template <int QT>
__device__ __forceinline__ uint32_t code_fast(float v, uint32_t lut_addr) {
  if constexpr (QT == kQtNF4) {
    const float f = __fmaf_rn(v, 32.0f, kMagic + 32.0f);
    const uint2 e = lds_v2(lut_addr + ((__float_as_uint(f) & 0x7fu) << 8));
    return e.y + (v > __uint_as_float(e.x) ? 1u : 0u);
  } else {
    const float a = fabsf(v);
    const float f = __fmaf_rn(a, 32.0f, kMagic);
    const uint2 e = lds_v2(lut_addr + ((__float_as_uint(f) & 0x7fu) << 8));
    const uint32_t m = e.y + (a > __uint_as_float(e.x) ? 1u : 0u);
    return (v < 0.0f && m != 0u) ? (m | 8u) : m;
  }
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

// One warp tile: per absmax group of rows, the block absmax (per chunk, then
// across the lanes -- and for LPB == 64 the two rows -- holding the block),
// the masked absmax store, the codes and the packed store.  As soon as a row
// is consumed its register slot is refilled with the same row of the warp's
// next tile.  FULL (the tile lies entirely inside n) removes every bounds
// check from the element loops.
template <bool FULL, typename T, int BS, int QT, bool DQ, typename LoadRow>
__device__ __forceinline__ void quant_tile(uint4 (&c)[kRows], int64_t e0, int64_t n,
                                           int64_t nb, int64_t next, int64_t n_tiles,
                                           int lane, const uint2* lut_lane, uint32_t lut_addr,
                                           uint8_t* __restrict__ codes,
                                           float* __restrict__ absmax, double& acc,
                                           const LoadRow& load_row) {
  constexpr int EPL = Elem<T>::kPerChunk;
  constexpr int LPB = BS / EPL;
  constexpr int ROW = 32 * EPL;
  constexpr int RG = LPB == 64 ? 2 : 1;
#pragma unroll
  for (int r0 = 0; r0 < kRows; r0 += RG) {
    float m = 0.0f;
#pragma unroll
    for (int rr = 0; rr < RG; ++rr)
#pragma unroll
      for (int i = 0; i < EPL; ++i) m = fmaxf(m, fabsf(Elem<T>::get(c[r0 + rr], i)));
    constexpr int kFirst = LPB == 64 ? 16 : LPB / 2;
#pragma unroll
    for (int o = kFirst; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    {
      const bool writer = LPB == 64 ? lane == 0 : (lane % LPB) == 0;
      const int64_t b = (e0 + static_cast<int64_t>(r0) * ROW) / BS +
                        (LPB == 64 ? 0 : lane / LPB);
      if (writer && (FULL || b < nb)) {
        absmax[b] = m;
        if constexpr (DQ) acc += static_cast<double>(m);
      }
    }
    const float inv = m == 0.0f ? 0.0f : __frcp_rn(m);
    // a subnormal absmax below 2^-128 makes the reciprocal infinite: such
    // rows (warp-uniform choice) take the clamped search, which reproduces
    // the midpoint count for infinite and NaN products
    const bool slow = __any_sync(0xffffffffu, isinf(inv));
#pragma unroll
    for (int rr = 0; rr < RG; ++rr) {
      const int r = r0 + rr;
      const int64_t e = e0 + static_cast<int64_t>(r * 32 + lane) * EPL;
      uint32_t packed = 0;
      if (!slow) {
#pragma unroll
        for (int i = 0; i < EPL; i += 2) {
          uint32_t c0 = code_fast<QT>(__fmul_rn(Elem<T>::get(c[r], i), inv), lut_addr);
          uint32_t c1 = code_fast<QT>(__fmul_rn(Elem<T>::get(c[r], i + 1), inv), lut_addr);
          if constexpr (!FULL) {  // padding nibbles of the ragged tail are 0
            if (e + i >= n) c0 = 0u;
            if (e + i + 1 >= n) c1 = 0u;
          }
          packed |= (c0 * 16u + c1) << (4 * i);
        }
      } else {
#pragma unroll
        for (int i = 0; i < EPL; i += 2) {
          uint32_t c0 = code_of<QT>(__fmul_rn(Elem<T>::get(c[r], i), inv), lut_lane);
          uint32_t c1 = code_of<QT>(__fmul_rn(Elem<T>::get(c[r], i + 1), inv), lut_lane);
          if constexpr (!FULL) {
            if (e + i >= n) c0 = 0u;
            if (e + i + 1 >= n) c1 = 0u;
          }
          packed |= (c0 * 16u + c1) << (4 * i);
        }
      }
      if (next < n_tiles) c[r] = load_row(next, r);
      uint8_t* dst = codes + e / 2;
      if (FULL || e + EPL <= n) {
        if constexpr (EPL == 8)
          *reinterpret_cast<uint32_t*>(dst) = packed;
        else
          *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
      } else {
        const int64_t nbytes = (n + 1) / 2;
#pragma unroll
        for (int j = 0; j < EPL / 2; ++j)
          if (e / 2 + j < nbytes) dst[j] = static_cast<uint8_t>(packed >> (8 * j));
      }
    }
  }
}

template <typename T, int BS, int QT, bool DQ>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    quant4_kernel(const T* __restrict__ x, int64_t n,
                  uint8_t* __restrict__ codes, float* __restrict__ absmax,
                  double* __restrict__ partials) {
  constexpr int EPL = Elem<T>::kPerChunk;  // elements per 16-byte chunk
  constexpr int LPB = BS / EPL;            // lanes (chunks) per block
  constexpr int ROW = 32 * EPL;            // elements per warp row
  constexpr int TILE = kRows * ROW;        // elements per warp tile
  static_assert(LPB == 64 || (LPB >= 4 && LPB <= 32), "blocksize");
  static_assert(TILE % BS == 0, "tile must hold whole blocks");

  extern __shared__ uint2 lut[];
  __shared__ double red[kThreads / 32];
  pdl_trigger();  // the double-quant kernel may be scheduled early
  build_lut<QT>(lut);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint2* lut_lane = lut + lane;
  const uint32_t lut_addr = static_cast<uint32_t>(__cvta_generic_to_shared(lut_lane));
  const int64_t nb = (n + BS - 1) / BS;
  const int64_t n_tiles = (n + TILE - 1) / TILE;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  double acc = 0.0;

  auto load_row = [&](int64_t tile, int r) -> uint4 {
    const int64_t t0 = tile * TILE;
    const int64_t e = t0 + static_cast<int64_t>(r * 32 + lane) * EPL;
    if (t0 + TILE <= n) return ldg_stream_v4(x + e);
    return Elem<T>::load_partial(x, e, n);
  };

  int64_t tile = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
  uint4 c[kRows];
  if (tile < n_tiles) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) c[r] = load_row(tile, r);
  }
  for (; tile < n_tiles; tile += n_warps) {
    const int64_t e0 = tile * TILE;
    const int64_t next = tile + n_warps;
    if (e0 + TILE <= n)
      quant_tile<true, T, BS, QT, DQ>(c, e0, n, nb, next, n_tiles, lane, lut_lane,
                                      lut_addr, codes, absmax, acc, load_row);
    else
      quant_tile<false, T, BS, QT, DQ>(c, e0, n, nb, next, n_tiles, lane, lut_lane,
                                       lut_addr, codes, absmax, acc, load_row);
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
// (grid-strided over the groups), no CTA-wide synchronization.  Every warp
// reduces the per-CTA partial sums of the quantize kernel in the same fixed
// order (lane-strided fp64 sums, then a fixed xor tree), so all agree on the
// offset; the sum is exact whenever the absmax values span few enough
// binades, and then equals the oracle's sequential sum.
constexpr int kDqThreads = 256;

__global__ void __launch_bounds__(kDqThreads)
    dq_absmax_kernel(const float* __restrict__ absmax, int64_t nb,
                     const double* __restrict__ partials, int n_partials,
                     uint8_t* __restrict__ absmax_q, float* __restrict__ scale2,
                     float* __restrict__ offset) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  pdl_wait();  // the quantize kernel's absmax and partial sums are complete
  double sum = 0.0;
  for (int i = lane; i < n_partials; i += 32) sum += partials[i];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float off = static_cast<float>(sum / static_cast<double>(nb));
  if (blockIdx.x == 0 && threadIdx.x == 0) offset[0] = off;

  const int64_t ng = (nb + 255) / 256;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (kDqThreads / 32);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * (kDqThreads / 32) + warp; g < ng;
       g += stride) {
    float c[8];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // entry g*256 + lane + 32 j (coalesced)
      const int64_t b = g * 256 + lane + 32 * j;
      c[j] = b < nb ? __fsub_rn(__ldg(absmax + b), off) : 0.0f;
      m = fmaxf(m, fabsf(c[j]));
    }
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

template <typename T, int BS, int QT, bool DQ>
cudaError_t launch_quant(const void* x, int64_t n, uint8_t* codes,
                         float* absmax, double* partials, int grid,
                         cudaStream_t s) {
  const size_t smem = kLutEntries * 32 * sizeof(uint2);
  return launch_kernel(quant4_kernel<T, BS, QT, DQ>, dim3(grid), dim3(kThreads), smem, s,
                       false, static_cast<const T*>(x), n, codes, absmax, partials);
}

template <typename T, int QT, bool DQ>
cudaError_t dispatch_bs(int bs, const void* x, int64_t n, uint8_t* codes,
                        float* absmax, double* partials, int grid,
                        cudaStream_t s) {
  switch (bs) {
    case 32: return launch_quant<T, 32, QT, DQ>(x, n, codes, absmax, partials, grid, s);
    case 64: return launch_quant<T, 64, QT, DQ>(x, n, codes, absmax, partials, grid, s);
    case 128: return launch_quant<T, 128, QT, DQ>(x, n, codes, absmax, partials, grid, s);
    default: return launch_quant<T, 256, QT, DQ>(x, n, codes, absmax, partials, grid, s);
  }
}

template <typename T>
cudaError_t dispatch_q(int qt, bool dq, int bs, const void* x, int64_t n,
                       uint8_t* codes, float* absmax, double* partials,
                       int grid, cudaStream_t s) {
  if (qt == kQtNF4)
    return dq ? dispatch_bs<T, kQtNF4, true>(bs, x, n, codes, absmax, partials, grid, s)
              : dispatch_bs<T, kQtNF4, false>(bs, x, n, codes, absmax, partials, grid, s);
  return dq ? dispatch_bs<T, kQtFP4, true>(bs, x, n, codes, absmax, partials, grid, s)
            : dispatch_bs<T, kQtFP4, false>(bs, x, n, codes, absmax, partials, grid, s);
}

}  // namespace

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
                            double* partials, int grid, cudaStream_t s) {
  const bool dq = st.double_quant != 0;
  cudaError_t e =
      x_dtype == BNB4_F32
          ? dispatch_q<float>(st.qtype, dq, st.blocksize, x, st.n, st.codes,
                              st.absmax, partials, grid, s)
          : dispatch_q<uint16_t>(st.qtype, dq, st.blocksize, x, st.n, st.codes,
                                 st.absmax, partials, grid, s);
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
