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
// loads in flight.  The 16-entry codebook sits in shared memory; the decoded
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

  for (int64_t tile = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
       tile < n_tiles; tile += n_warps) {
    const int64_t e0 = tile * TILE;
    const bool full = e0 + TILE <= n;
    uint32_t cw[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int64_t e = e0 + static_cast<int64_t>(r * 32 + lane) * EPL;
      const uint8_t* src = codes + e / 2;
      if (full) {
        if constexpr (EPL == 8)
          cw[r] = __ldg(reinterpret_cast<const uint32_t*>(src));
        else
          cw[r] = __ldg(reinterpret_cast<const uint16_t*>(src));
      } else {
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < EPL / 2; ++j)
          if (e / 2 + j < nbytes) w |= static_cast<uint32_t>(__ldg(src + j)) << (8 * j);
        cw[r] = w;
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int64_t e = e0 + static_cast<int64_t>(r * 32 + lane) * EPL;
      if (!full && e >= n) continue;
      const float ah =
          decoded_absmax<DQ>(e >> bs_log2, absmax, absmax_q, scale2, off);
      float w[EPL];
#pragma unroll
      for (int i = 0; i < EPL; i += 2) {
        const uint32_t byte = (cw[r] >> (4 * i)) & 0xffu;
        w[i] = __fmul_rn(table[byte >> 4], ah);
        w[i + 1] = __fmul_rn(table[byte & 15u], ah);
      }
      TO* dst = out + e;
      if (full || e + EPL <= n) {
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
}

template <typename TO, bool DQ>
cudaError_t launch(const bnb4_qstate& st, void* out, int grid, cudaStream_t s) {
  const int bs_log2 = __builtin_ctz(static_cast<unsigned>(st.blocksize));
  dequant4_kernel<TO, DQ><<<grid, kThreads, 0, s>>>(
      st.codes, st.n, bs_log2, st.qtype, st.absmax, st.absmax_q, st.scale2,
      st.offset, static_cast<TO*>(out));
  return cudaGetLastError();
}

}  // namespace

int dequant_grid(int64_t n, int out_dtype, int num_sms) {
  const int64_t epl = out_dtype == BNB4_F32 ? 4 : 8;
  const int64_t tile = kRows * 32 * epl;
  const int64_t tiles = (n + tile - 1) / tile;
  const int64_t ctas = (tiles + kThreads / 32 - 1) / (kThreads / 32);
  int64_t g = static_cast<int64_t>(num_sms) * 4;
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
