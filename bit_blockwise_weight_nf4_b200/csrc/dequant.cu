// dequant.cu -- blockwise 4-bit dequantization on sm_100a.
//
// Method (CSDN article on bitsandbytes, section "实际性能差异", double
// quantization; release notes 0.49.2 on the ossradar page, dequantize op):
//   a_hat = fma(u - 128, scale2[b / 256], offset) (one rounding) with double
//   quantization, the stored absmax without; w = RN(t[code] * a_hat) in fp32;
//   bf16 output = round-to-nearest-even of w.
//
// Design (HBM-bound on the output write): persistent grid; each lane owns one
// output chunk of 16 bytes per row (4 fp32 or 8 bf16 elements), so a warp's
// codes load (64 or 128 contiguous bytes) and its output store (512 contiguous
// bytes) are both fully coalesced; 8 rows per tile keep eight independent code
// loads in flight, refilled from the next tile as rows are consumed.  The
// 16-entry codebook sits in shared memory (one bank per entry); the decoded
// scale of a chunk (all its elements share one block) comes from L1-resident
// absmax bytes.
#include "common.cuh"
#include "kernels.h"

namespace bnb4 {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 8;

template <typename TO>
struct Out;
template <>
struct Out<float> {
  static constexpr int kPerChunk = 4;
};
template <>
struct Out<uint16_t> {
  static constexpr int kPerChunk = 8;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// One warp tile.  Per row: the chunk's decoded scale, then for every code
// byte the two codebook values from the 16-entry shared table (conflict
// free: 16 entries in 16 banks) times the scale.  The byte offsets of the
// codes into the table come from two masks of the whole word (high nibbles
// = even elements, low nibbles = odd elements, both times 4) and one byte
// permute per element.  Each row's register slot is refilled with the same
// row of the warp's next tile as soon as it is consumed.  FULL (the tile
// lies entirely inside n) removes every bounds check.
template <bool FULL, typename TO, bool DQ, typename LoadRow>
__device__ __forceinline__ void dequant_tile(uint32_t (&cw)[kRows], int64_t e0, int64_t n,
                                             int64_t next, int64_t n_tiles, int lane,
                                             int bs_log2, const float* table,
                                             const float* __restrict__ absmax,
                                             const uint8_t* __restrict__ absmax_q,
                                             const float* __restrict__ scale2, float off,
                                             TO* __restrict__ out, const LoadRow& load_row) {
  constexpr int EPL = Out<TO>::kPerChunk;
  const char* tb = reinterpret_cast<const char*>(table);
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int64_t e = e0 + static_cast<int64_t>(r * 32 + lane) * EPL;
    if (!FULL && e >= n) continue;
    const float ah = decoded_absmax<DQ>(e >> bs_log2, absmax, absmax_q, scale2, off);
    const uint32_t evens = (cw[r] >> 2) & 0x3c3c3c3cu;  // 4 * code of element 2j
    const uint32_t odds = (cw[r] << 2) & 0x3c3c3c3cu;   // 4 * code of element 2j+1
    float w[EPL];
#pragma unroll
    for (int j = 0; j < EPL / 2; ++j) {
      const uint32_t oe = prmt(evens, 0u, 0x4440u | j);
      const uint32_t oo = prmt(odds, 0u, 0x4440u | j);
      w[2 * j] = __fmul_rn(*reinterpret_cast<const float*>(tb + oe), ah);
      w[2 * j + 1] = __fmul_rn(*reinterpret_cast<const float*>(tb + oo), ah);
    }
    if (next < n_tiles) cw[r] = load_row(next, r);
    TO* dst = out + e;
    if (FULL || e + EPL <= n) {
      if constexpr (EPL == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(w[0], w[1], w[2], w[3]);
      } else {
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]),
                       pack_bf16x2(w[4], w[5]), pack_bf16x2(w[6], w[7]));
      }
    } else {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        if (e + i < n) {
          if constexpr (EPL == 4)
            dst[i] = w[i];
          else
            dst[i] = static_cast<uint16_t>(pack_bf16x2(w[i], 0.0f) & 0xffffu);
        }
      }
    }
  }
}

template <typename TO, bool DQ>
__global__ void __launch_bounds__(kThreads)
    dequant4_kernel(const uint8_t* __restrict__ codes, int64_t n, int bs_log2,
                    int qtype, const float* __restrict__ absmax,
                    const uint8_t* __restrict__ absmax_q,
                    const float* __restrict__ scale2,
                    const float* __restrict__ offset, TO* __restrict__ out) {
  constexpr int EPL = Out<TO>::kPerChunk;
  constexpr int TILE = kRows * 32 * EPL;
  __shared__ float table[16];
  if (threadIdx.x < 16) table[threadIdx.x] = code_value(qtype, threadIdx.x);
  __syncthreads();
  const float off = DQ ? __ldg(offset) : 0.0f;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t n_tiles = (n + TILE - 1) / TILE;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t nbytes = (n + 1) / 2;

  auto load_row = [&](int64_t tile, int r) -> uint32_t {
    const int64_t t0 = tile * TILE;
    const int64_t e = t0 + static_cast<int64_t>(r * 32 + lane) * EPL;
    const uint8_t* src = codes + e / 2;
    if (t0 + TILE <= n) {
      if constexpr (EPL == 8)
        return __ldg(reinterpret_cast<const uint32_t*>(src));
      else
        return __ldg(reinterpret_cast<const uint16_t*>(src));
    }
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < EPL / 2; ++j)
      if (e / 2 + j < nbytes) w |= static_cast<uint32_t>(__ldg(src + j)) << (8 * j);
    return w;
  };

  int64_t tile = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
  uint32_t cw[kRows];
  if (tile < n_tiles) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) cw[r] = load_row(tile, r);
  }
  for (; tile < n_tiles; tile += n_warps) {
    const int64_t e0 = tile * TILE;
    const int64_t next = tile + n_warps;
    if (e0 + TILE <= n)
      dequant_tile<true, TO, DQ>(cw, e0, n, next, n_tiles, lane, bs_log2, table, absmax,
                                 absmax_q, scale2, off, out, load_row);
    else
      dequant_tile<false, TO, DQ>(cw, e0, n, next, n_tiles, lane, bs_log2, table, absmax,
                                  absmax_q, scale2, off, out, load_row);
  }
}

template <typename TO, bool DQ>
cudaError_t launch(const bnb4_qstate& st, void* out, int grid, cudaStream_t s) {
  const int bs_log2 = __builtin_ctz(static_cast<unsigned>(st.blocksize));
  return launch_kernel(dequant4_kernel<TO, DQ>, dim3(grid), dim3(kThreads), 0, s, false,
                    static_cast<const uint8_t*>(st.codes), st.n, bs_log2,
                    static_cast<int>(st.qtype), static_cast<const float*>(st.absmax),
                    static_cast<const uint8_t*>(st.absmax_q),
                    static_cast<const float*>(st.scale2),
                    static_cast<const float*>(st.offset), static_cast<TO*>(out));
}

}  // namespace

int dequant_grid(int64_t n, int out_dtype, int num_sms) {
  const int64_t epl = out_dtype == BNB4_F32 ? 4 : 8;
  const int64_t tile = kRows * 32 * epl;
  const int64_t tiles = (n + tile - 1) / tile;
  const int64_t ctas = (tiles + kThreads / 32 - 1) / (kThreads / 32);
  int64_t g = static_cast<int64_t>(num_sms) * 6;  // resident CTAs (48 registers)
  if (ctas < g) g = ctas;
  return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_dequantize(const bnb4_qstate& st, void* out, int out_dtype,
                              int grid, cudaStream_t s) {
  const bool dq = st.double_quant != 0;
  if (out_dtype == BNB4_F32)
    return dq ? launch<float, true>(st, out, grid, s)
              : launch<float, false>(st, out, grid, s);
  return dq ? launch<uint16_t, true>(st, out, grid, s)
            : launch<uint16_t, false>(st, out, grid, s);
}

}  // namespace bnb4
