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
// Design (HBM-bound): a persistent grid of 256-thread CTAs; each warp streams
// tiles of 8 x 512 contiguous bytes with 128-bit non-allocating loads (8
// independent loads in flight per lane), reduces each block's absmax with xor
// shuffles among the lanes that hold it, and writes the packed codes with one
// coalesced 16/32-bit store per lane and row.  The nearest-code search is one
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
constexpr int kRows = 8;            // 16-byte chunks per lane per tile
constexpr int kLutEntries = 65;     // buckets j = 0..64
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
  float mid[nm];
#pragma unroll
  for (int i = 0; i < nm; ++i) {
    const float a = QT == kQtNF4 ? nf4_value(i) : fp4_magnitude(i);
    const float b = QT == kQtNF4 ? nf4_value(i + 1) : fp4_magnitude(i + 1);
    mid[i] = __fmul_rn(__fadd_rn(a, b), 0.5f);
  }
  for (int idx = threadIdx.x; idx < kLutEntries * 32; idx += blockDim.x) {
    const int j = idx >> 5;
    const float center = QT == kQtNF4 ? static_cast<float>(j - 32)
                                      : static_cast<float>(j);
    const float lo = (center - 0.5f) / 32.0f - 1e-3f;
    const float hi = (center + 0.5f) / 32.0f + 1e-3f;
    int base = 0;
    float cand = __int_as_float(0x7f800000);
#pragma unroll
    for (int i = 0; i < nm; ++i) {
      if (mid[i] < lo) ++base;
      else if (mid[i] <= hi) cand = mid[i];
    }
    lut[idx] = make_uint2(__float_as_uint(cand), static_cast<uint32_t>(base));
  }
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

template <typename T, int BS, int QT, bool DQ>
__global__ void __launch_bounds__(kThreads)
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
  build_lut<QT>(lut);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint2* lut_lane = lut + lane;
  const int64_t nb = (n + BS - 1) / BS;
  const int64_t n_tiles = (n + TILE - 1) / TILE;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  double acc = 0.0;

  for (int64_t tile = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
       tile < n_tiles; tile += n_warps) {
    const int64_t e0 = tile * TILE;
    const bool full = e0 + TILE <= n;
    uint4 c[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int64_t e = e0 + static_cast<int64_t>(r * 32 + lane) * EPL;
      if (full)
        c[r] = ldg_stream_v4(x + e);
      else
        c[r] = Elem<T>::load_partial(x, e, n);
    }
    // per-chunk absmax, then across the lanes (and rows) of each block
    float a[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) m = fmaxf(m, fabsf(Elem<T>::get(c[r], i)));
      a[r] = m;
    }
    if constexpr (LPB == 64) {
#pragma unroll
      for (int r = 0; r < kRows; r += 2) {
        float m = fmaxf(a[r], a[r + 1]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        a[r] = a[r + 1] = m;
      }
    } else {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float m = a[r];
#pragma unroll
        for (int o = LPB / 2; o >= 1; o >>= 1)
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        a[r] = m;
      }
    }
    // masked absmax store (+ fp64 partial sum for the double quantization)
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      bool writer;
      int64_t b;
      if constexpr (LPB == 64) {
        writer = (r & 1) == 0 && lane == 0;
        b = (e0 + static_cast<int64_t>(r) * ROW) / BS;
      } else {
        writer = (lane % LPB) == 0;
        b = (e0 + static_cast<int64_t>(r) * ROW) / BS + lane / LPB;
      }
      if (writer && b < nb) {
        absmax[b] = a[r];
        if constexpr (DQ) acc += static_cast<double>(a[r]);
      }
    }
    // codes
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const float inv = a[r] == 0.0f ? 0.0f : __frcp_rn(a[r]);
      const int64_t e = e0 + static_cast<int64_t>(r * 32 + lane) * EPL;
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < EPL; i += 2) {
        uint32_t c0 = code_of<QT>(__fmul_rn(Elem<T>::get(c[r], i), inv), lut_lane);
        uint32_t c1 = code_of<QT>(__fmul_rn(Elem<T>::get(c[r], i + 1), inv), lut_lane);
        if (!full) {  // padding nibbles of the ragged tail are 0
          if (e + i >= n) c0 = 0u;
          if (e + i + 1 >= n) c1 = 0u;
        }
        packed |= (c0 * 16u + c1) << (4 * i);
      }
      uint8_t* dst = codes + e / 2;
      if (full || e + EPL <= n) {
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

// Double quantization of the absmax array: one CTA per group of 256 blocks
// (grid-strided).  Every CTA reduces the per-CTA partial sums of the quantize
// kernel in the same fixed order, so all agree on the offset.
__global__ void __launch_bounds__(256)
    dq_absmax_kernel(const float* __restrict__ absmax, int64_t nb,
                     const double* __restrict__ partials, int n_partials,
                     uint8_t* __restrict__ absmax_q, float* __restrict__ scale2,
                     float* __restrict__ offset) {
  __shared__ double dred[256];
  __shared__ float fred[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < n_partials; i += 256) s += partials[i];
  dred[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w >= 1; w >>= 1) {
    if (threadIdx.x < w) dred[threadIdx.x] += dred[threadIdx.x + w];
    __syncthreads();
  }
  const float off = static_cast<float>(dred[0] / static_cast<double>(nb));
  if (blockIdx.x == 0 && threadIdx.x == 0) offset[0] = off;

  const int64_t ng = (nb + 255) / 256;
  for (int64_t g = blockIdx.x; g < ng; g += gridDim.x) {
    const int64_t b = g * 256 + threadIdx.x;
    const float cb = b < nb ? __fsub_rn(absmax[b], off) : 0.0f;
    __syncthreads();
    fred[threadIdx.x] = fabsf(cb);
    __syncthreads();
    for (int w = 128; w >= 1; w >>= 1) {
      if (threadIdx.x < w)
        fred[threadIdx.x] = fmaxf(fred[threadIdx.x], fred[threadIdx.x + w]);
      __syncthreads();
    }
    const float sg = __fdiv_rn(fred[0], 127.0f);
    if (threadIdx.x == 0) scale2[g] = sg;
    if (b < nb) {
      float q = 0.0f;
      if (sg != 0.0f) q = fminf(fmaxf(rintf(__fdiv_rn(cb, sg)), -127.0f), 127.0f);
      absmax_q[b] = static_cast<uint8_t>(static_cast<int>(q) + 128);
    }
  }
}

template <typename T, int BS, int QT, bool DQ>
cudaError_t launch_quant(const void* x, int64_t n, uint8_t* codes,
                         float* absmax, double* partials, int grid,
                         cudaStream_t s) {
  const size_t smem = kLutEntries * 32 * sizeof(uint2);
  quant4_kernel<T, BS, QT, DQ><<<grid, kThreads, smem, s>>>(
      static_cast<const T*>(x), n, codes, absmax, partials);
  return cudaGetLastError();
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
  int64_t g = static_cast<int64_t>(num_sms) * 4;
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
  const int g2 = static_cast<int>(ng < 4096 ? ng : 4096);
  dq_absmax_kernel<<<g2, 256, 0, s>>>(st.absmax, nb, partials, grid,
                                      st.absmax_q, st.scale2, st.offset);
  return cudaGetLastError();
}

}  // namespace bnb4
