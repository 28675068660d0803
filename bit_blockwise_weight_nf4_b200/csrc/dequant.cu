// dequant.cu -- blockwise 4-bit dequantization on sm_100a.
//
// Method (CSDN article on bitsandbytes, section "实际性能差异", double
// quantization; release notes 0.49.2 on the ossradar page, dequantize op):
//   a_hat = fma(u - 128, scale2[b / 256], offset) (one rounding) with double
//   quantization, the stored absmax without; w = RN(t[code] * a_hat) in fp32;
//   bf16 output = round-to-nearest-even of w.
//
// Design (HBM-bound on the output write): a persistent grid; each lane owns
// one output chunk of 16 bytes per row (4 fp32 or 8 bf16 elements), so a
// warp's code load (64 or 128 contiguous bytes) and its output store (512
// contiguous bytes) are both fully coalesced.  A warp streams whole tiles of
// 4 rows; each row's register slots -- the code word and the raw scale
// inputs of the chunk's block -- are refilled with the same row of the warp's
// next tile as soon as the row is consumed, so neither the codes nor the
// scales are waited for.  Lane pointers advance once per tile and rows are
// immediate offsets.  The 16-entry codebook sits in shared memory (one bank
// per entry, conflict free); a code's byte offset into it comes from two
// masks of the whole code word and one byte permute per element.  The one
// ragged tile at the end takes a bounds-checked path.
#include "common.cuh"
#include "kernels.h"
#include "lut.cuh"

namespace bnb4 {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 4;  // rows per tile (4 measured best of 2-16 on B200)
constexpr int kCtasPerSm = 4;  // resident CTAs per SM (64 registers)

// Output element type per format: fp32 (4 per 16-byte chunk) or a 16-bit
// pattern, bf16 or fp16 (8 per chunk).
template <int OF>
struct Out {
  using T = uint16_t;
  static constexpr int kPerChunk = 8;
};
template <>
struct Out<BNB4_F32> {
  using T = float;
  static constexpr int kPerChunk = 4;
};


// Raw scale inputs of a block: absmax_q byte and scale2 (double quant) or the
// absmax bits.
struct Raw {
  uint32_t u;
  float s;
};

template <bool DQ>
__device__ __forceinline__ Raw load_raw(int64_t b, const float* absmax,
                                        const uint8_t* absmax_q, const float* scale2) {
  if constexpr (DQ)
    return Raw{static_cast<uint32_t>(__ldg(absmax_q + b)), __ldg(scale2 + (b >> 8))};
  else
    return Raw{__float_as_uint(__ldg(absmax + b)), 0.0f};
}

template <bool DQ>
__device__ __forceinline__ float decode(Raw r, float off) {
  if constexpr (DQ)
    return __fmaf_rn(static_cast<float>(static_cast<int>(r.u) - 128), r.s, off);
  else
    return __uint_as_float(r.u);
}

// The chunk's EPL values w = RN(t[code] * ah), in element order.  cw holds
// EPL / 2 code bytes (first element in the high nibble of byte 0).
template <int EPL>
__device__ __forceinline__ void chunk_values(uint32_t cw, float ah, const float* table,
                                             float (&w)[EPL]) {
  const char* tb = reinterpret_cast<const char*>(table);
  const uint32_t evens = (cw >> 2) & 0x3c3c3c3cu;  // 4 * code of element 2j
  const uint32_t odds = (cw << 2) & 0x3c3c3c3cu;   // 4 * code of element 2j+1
#pragma unroll
  for (int j = 0; j < EPL / 2; ++j) {
    const uint32_t oe = prmt(evens, 0u, 0x4440u | j);
    const uint32_t oo = prmt(odds, 0u, 0x4440u | j);
    w[2 * j] = __fmul_rn(*reinterpret_cast<const float*>(tb + oe), ah);
    w[2 * j + 1] = __fmul_rn(*reinterpret_cast<const float*>(tb + oo), ah);
  }
}

template <int OF, int EPL>
__device__ __forceinline__ void store_chunk(typename Out<OF>::T* dst, const float (&w)[EPL]) {
  if constexpr (EPL == 4) {
    *reinterpret_cast<float4*>(dst) = make_float4(w[0], w[1], w[2], w[3]);
  } else {
    *reinterpret_cast<uint4*>(dst) =
        make_uint4(pack2<OF>(w[0], w[1]), pack2<OF>(w[2], w[3]),
                   pack2<OF>(w[4], w[5]), pack2<OF>(w[6], w[7]));
  }
}

template <int EPL>
__device__ __forceinline__ uint32_t load_codes(const uint8_t* p) {
  if constexpr (EPL == 8)
    return __ldg(reinterpret_cast<const uint32_t*>(p));
  else
    return __ldg(reinterpret_cast<const uint16_t*>(p));
}

// STR: out is a row-major [n / v.cols, v.cols] view with rows v.ld elements
// apart (16-byte aligned rows, n < 2^32); element e of the logical tensor is
// written at out + view_offset(e).
template <int OF, bool DQ, int BS, bool STR>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    dequant4_kernel(const uint8_t* __restrict__ codes, int64_t n, int qtype,
                    const float* __restrict__ absmax,
                    const uint8_t* __restrict__ absmax_q,
                    const float* __restrict__ scale2,
                    const float* __restrict__ offset,
                    typename Out<OF>::T* __restrict__ out, View2D v) {
  using TO = typename Out<OF>::T;
  constexpr int EPL = Out<OF>::kPerChunk;
  constexpr int ROW = 32 * EPL;
  constexpr int TILE = kRows * ROW;
  static_assert(TILE % BS == 0, "tile must hold whole blocks");
  __shared__ float table[16];
  if (threadIdx.x < 16) table[threadIdx.x] = code_value(qtype, threadIdx.x);
  __syncthreads();
  // programmatic dependent launch (inside a captured graph after a kernel):
  // no global access before the previous kernel has completed
  pdl_trigger();
  pdl_wait();
  const float off = DQ ? __ldg(offset) : 0.0f;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t n_full = n / TILE;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);

  int64_t tile = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
  if (tile < n_full) {
    const int64_t e0 = tile * TILE + lane * EPL;
    const uint8_t* cp = codes + e0 / 2;
    TO* op = out + e0;
    int64_t et = e0;       // logical element of the lane's chunk in row 0
    int64_t b0 = e0 / BS;  // block of the lane's chunk in row 0
    const int64_t stride = n_warps * TILE;
    // block of row r relative to row 0 (ROW may be smaller than BS)
    auto rb = [&](int r) -> int64_t {
      return static_cast<int64_t>((lane * EPL + r * ROW) / BS - (lane * EPL) / BS);
    };
    uint32_t cw[kRows];
    Raw raw[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      cw[r] = load_codes<EPL>(cp + r * ROW / 2);
      raw[r] = load_raw<DQ>(b0 + rb(r), absmax, absmax_q, scale2);
    }
    for (; tile < n_full; tile += n_warps) {
      // the last tile of the warp refills from itself (the loads are unused)
      const int64_t step = tile + n_warps < n_full ? stride : 0;
      const uint8_t* cn = cp + step / 2;
      const int64_t bn = b0 + step / BS;
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float w[EPL];
        chunk_values<EPL>(cw[r], decode<DQ>(raw[r], off), table, w);
        cw[r] = load_codes<EPL>(cn + r * ROW / 2);
        raw[r] = load_raw<DQ>(bn + rb(r), absmax, absmax_q, scale2);
        store_chunk<OF, EPL>(STR ? out + view_offset(et + r * ROW, v) : op + r * ROW, w);
      }
      cp = cn;
      b0 = bn;
      op += stride;
      et += stride;
    }
  }

  // the ragged tile (elements n_full * TILE .. n - 1) belongs to the warp
  // whose tile sequence reaches it
  if (n % TILE != 0 && tile == n_full) {
    const int64_t nbytes = (n + 1) / 2;
#pragma unroll 1
    for (int r = 0; r < kRows; ++r) {
      const int64_t e = n_full * TILE + static_cast<int64_t>(r * 32 + lane) * EPL;
      if (e >= n) break;
      uint32_t cwp = 0;
#pragma unroll
      for (int j = 0; j < EPL / 2; ++j)
        if (e / 2 + j < nbytes) cwp |= static_cast<uint32_t>(__ldg(codes + e / 2 + j)) << (8 * j);
      float w[EPL];
      chunk_values<EPL>(cwp, decode<DQ>(load_raw<DQ>(e / BS, absmax, absmax_q, scale2), off),
                        table, w);
      if (e + EPL <= n) {
        store_chunk<OF, EPL>(STR ? out + view_offset(e, v) : out + e, w);
      } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          if (e + i < n) {
            if constexpr (EPL == 4)
              out[e + i] = w[i];
            else
              out[e + i] = static_cast<uint16_t>(pack2<OF>(w[i], 0.0f) & 0xffffu);
          }
        }
      }
    }
  }
}

template <int OF, bool DQ, int BS>
cudaError_t launch(const bnb4_qstate& st, void* out, int grid, const View2D* view,
                   cudaStream_t s) {
  using TO = typename Out<OF>::T;
  if (view)
    return launch_kernel(dequant4_kernel<OF, DQ, BS, true>, dim3(grid), dim3(kThreads), 0, s,
                         programmatic_after_kernel(s), static_cast<const uint8_t*>(st.codes),
                         st.n,
                         static_cast<int>(st.qtype), static_cast<const float*>(st.absmax),
                         static_cast<const uint8_t*>(st.absmax_q),
                         static_cast<const float*>(st.scale2),
                         static_cast<const float*>(st.offset), static_cast<TO*>(out), *view);
  return launch_kernel(dequant4_kernel<OF, DQ, BS, false>, dim3(grid), dim3(kThreads), 0, s,
                       programmatic_after_kernel(s),
                       static_cast<const uint8_t*>(st.codes), st.n,
                       static_cast<int>(st.qtype), static_cast<const float*>(st.absmax),
                       static_cast<const uint8_t*>(st.absmax_q),
                       static_cast<const float*>(st.scale2),
                       static_cast<const float*>(st.offset), static_cast<TO*>(out), View2D{});
}

template <int OF, bool DQ>
cudaError_t launch_bs(const bnb4_qstate& st, void* out, int grid, const View2D* view,
                      cudaStream_t s) {
  switch (st.blocksize) {
    case 32: return launch<OF, DQ, 32>(st, out, grid, view, s);
    case 64: return launch<OF, DQ, 64>(st, out, grid, view, s);
    case 128: return launch<OF, DQ, 128>(st, out, grid, view, s);
    default: return launch<OF, DQ, 256>(st, out, grid, view, s);
  }
}

}  // namespace

int dequant_grid(int64_t n, int out_dtype, int num_sms) {
  const int64_t epl = out_dtype == BNB4_F32 ? 4 : 8;
  const int64_t tile = kRows * 32 * epl;
  const int64_t tiles = (n + tile - 1) / tile;
  const int64_t ctas = (tiles + kThreads / 32 - 1) / (kThreads / 32);
  int64_t g = static_cast<int64_t>(num_sms) * kCtasPerSm;  // resident CTAs
  if (ctas < g) g = ctas;
  return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_dequantize(const bnb4_qstate& st, void* out, int out_dtype,
                              int grid, cudaStream_t s, const View2D* view) {
  const bool dq = st.double_quant != 0;
  if (out_dtype == BNB4_F32)
    return dq ? launch_bs<BNB4_F32, true>(st, out, grid, view, s)
              : launch_bs<BNB4_F32, false>(st, out, grid, view, s);
  if (out_dtype == BNB4_F16)
    return dq ? launch_bs<BNB4_F16, true>(st, out, grid, view, s)
              : launch_bs<BNB4_F16, false>(st, out, grid, view, s);
  return dq ? launch_bs<BNB4_BF16, true>(st, out, grid, view, s)
            : launch_bs<BNB4_BF16, false>(st, out, grid, view, s);
}

}  // namespace bnb4
