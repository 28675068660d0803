// gemm.cu -- prefill GEMM with fused 4-bit weight dequantization, sm_100a:
//   Y[m, n] = bf16( sum_k X[m, k] * What[n, k] ),
//   What[n, k] = bf16(RN(t[code] * a_hat))  (exact dequantized weight),
// fp32 accumulation in tensor memory by tcgen05.mma (kind::f16, bf16 inputs).
//
// Method: the fused 4-bit dequantize + GEMM of bitsandbytes' release notes
// 0.50.0 (ossradar page), nested quantization decoded inside, over the NF4 /
// FP4 blockwise format of the CSDN article (section "数学原理对比").
//
// Design (one CTA per 256 x 256 output tile, 10 warps, 3-stage pipeline):
//  * warp 0: producer.  Lane 0 issues the TMA loads of a 64-wide K step --
//    two 128 x 64 bf16 tiles of X (128-byte swizzle) and the 256 x 32-byte
//    packed weight tile; meanwhile all 32 lanes decode the 256 block scales of
//    the step (nested quantization) into shared memory, so the dequantizers
//    never wait on a global load.  One mbarrier (32 arrivals + the TMA bytes)
//    marks the stage full.
//  * warps 2..9 (256 threads): dequantizers.  Thread r turns weight row r of
//    the stage (64 codes) into 64 bf16 values through a per-block 16-entry
//    table (byte-permute lookups, as in the GEMV) and stores them in the
//    128-byte-swizzled K-major layout the MMA reads; then fence.proxy.async
//    and an arrive on the stage's "weights ready" barrier.
//  * warp 1 (one lane): allocates 512 TMEM columns (two 128 x 256 fp32
//    accumulators), waits for both barriers of a stage, issues 2 x 4
//    tcgen05.mma (M 128, N 256, K 16) -- the dequantized tile is used by both
//    M halves, halving the dequantization work per flop -- and commits to the
//    stage's "empty" barrier.
//  * epilogue: the 8 dequant warps read the accumulators with tcgen05.ld
//    (warp w owns TMEM lanes 32 (w % 4)..+31), round to bf16 and store.
//  * Every mbarrier wait is bounded in time; on expiry the CTA sets the
//    library's device error word, drains what it started and exits.
//  No TMA multicast is used.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {
namespace {

constexpr int BM = 128;     // rows of one accumulator (M of one MMA)
constexpr int MSUB = 2;     // accumulators per CTA (M tile 256)
constexpr int BN = 256;     // weight rows per CTA (N of one MMA)
constexpr int BK = 64;      // K per stage (one 128-byte swizzle row of bf16)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int B_BYTES = BN * BK * 2;    // 32 KB
constexpr int WP_BYTES = BN * BK / 2;   // 8 KB packed codes
constexpr int STAGE_BYTES = MSUB * A_BYTES + B_BYTES + WP_BYTES;
constexpr int SCALE_FLOATS = 2 * BN;  // decoded scales of a stage (2 per row
                                      // for blocksize 32)
constexpr int kDeqWarps = 8;
constexpr int kThreads = 64 + kDeqWarps * 32;
constexpr int TMEM_COLS = 512;
constexpr int SMEM_BYTES =
    STAGES * STAGE_BYTES + STAGES * SCALE_FLOATS * 4 + 1024 /*align*/ + 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");

struct Bars {
  uint64_t full[STAGES];    // TMA bytes of the stage landed
  uint64_t bready[STAGES];  // dequantized weights of the stage written
  uint64_t empty[STAGES];   // MMAs reading the stage finished
  uint64_t accum;           // all MMAs finished
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx_only(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase of `parity`; false when the CTA is aborting or
// the time limit expired (then the device error word is set).
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, Bars* bars, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*reinterpret_cast<volatile int*>(&bars->abort)) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicExch(err, 1);
        *reinterpret_cast<volatile int*>(&bars->abort) = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map,
                                            int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), sm100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3fffu);
  d |= static_cast<uint64_t>(1u) << 16;          // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;  // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;          // descriptor version
  d |= static_cast<uint64_t>(2u) << 61;          // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::f16, D fp32, A and B bf16, both K-major,
// N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(BM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc,
                                          uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          bar)
      : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

struct Lut {
  uint32_t L[4], H[4];
};

template <int QT>
__device__ __forceinline__ Lut make_lut(float ah) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int c0 = 2 * j, c1 = 2 * j + 1;
    const float t0 = QT == kQtNF4 ? nf4_value(c0)
                                  : ((c0 & 8) ? -fp4_magnitude(c0 & 7) : fp4_magnitude(c0 & 7));
    const float t1 = QT == kQtNF4 ? nf4_value(c1)
                                  : ((c1 & 8) ? -fp4_magnitude(c1 & 7) : fp4_magnitude(c1 & 7));
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

// 8 codes of one packed 32-bit word (natural order k0..k7) -> 8 bf16 in k
// order as 4 words.
__device__ __forceinline__ uint4 dq8(const Lut& l, uint32_t w) {
  uint4 o;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t v = h ? (w >> 16) : w;
    const uint32_t sel = v & 0x7777u;
    const uint32_t mix = ((v >> 1) & 0x4444u) | 0x3210u;
    const uint32_t lo = prmt(prmt(l.L[0], l.L[1], sel), prmt(l.L[2], l.L[3], sel), mix);
    const uint32_t hi = prmt(prmt(l.H[0], l.H[1], sel), prmt(l.H[2], l.H[3], sel), mix);
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

template <int BS, int QT, bool DQ>
__global__ void __launch_bounds__(kThreads, 1)
    gemm4_kernel(const __grid_constant__ CUtensorMap map_x,
                 const __grid_constant__ CUtensorMap map_w, int M, int N, int K,
                 const float* __restrict__ absmax,
                 const uint8_t* __restrict__ absmax_q,
                 const float* __restrict__ scale2,
                 const float* __restrict__ offset, uint16_t* __restrict__ Y,
                 int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* scales = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES +
                                       STAGES * SCALE_FLOATS * 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * (BM * MSUB);
  const int n0 = blockIdx.x * BN;
  const int k_tiles = K / BK;

  auto stage_a = [&](int s, int j) { return smem + s * STAGE_BYTES + j * A_BYTES; };
  auto stage_b = [&](int s) { return smem + s * STAGE_BYTES + MSUB * A_BYTES; };
  auto stage_wp = [&](int s) {
    return smem + s * STAGE_BYTES + MSUB * A_BYTES + B_BYTES;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 32);
      mbar_init(smem_u32(&bars->bready[s]), kDeqWarps * 32);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->accum), 1);
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    const float off = DQ ? __ldg(offset) : 0.0f;
    int last_round[STAGES];
    for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
    for (int kt = 0; kt < k_tiles; ++kt) {
      const int s = kt % STAGES, round = kt / STAGES;
      if (!wait_bounded(smem_u32(&bars->empty[s]), (round & 1) ^ 1, bars, err)) break;
      const uint32_t fb = smem_u32(&bars->full[s]);
      if (lane == 0) {
        mbar_expect_tx_only(fb, MSUB * A_BYTES + WP_BYTES);
        for (int j = 0; j < MSUB; ++j)
          tma_load_2d(smem_u32(stage_a(s, j)), &map_x, kt * BK, m0 + j * BM, fb);
        tma_load_2d(smem_u32(stage_wp(s)), &map_w, kt * (BK / 2), n0, fb);
      }
      last_round[s] = round;
      float* sc = scales + s * SCALE_FLOATS;
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) {
        const int row = lane + 32 * i;
        const int64_t n = static_cast<int64_t>(n0) + row;
        float a0 = 0.0f, a1 = 0.0f;
        if (n < N) {
          const int64_t b = (n * K + static_cast<int64_t>(kt) * BK) / BS;
          a0 = decoded_absmax<DQ>(b, absmax, absmax_q, scale2, off);
          if constexpr (BS == 32) a1 = decoded_absmax<DQ>(b + 1, absmax, absmax_q, scale2, off);
        }
        sc[row] = a0;
        if constexpr (BS == 32) sc[BN + row] = a1;
      }
      mbar_arrive(fb);
    }
    // drain: every load issued has landed before the CTA may exit
    if (lane == 0)
      for (int s = 0; s < STAGES; ++s)
        if (last_round[s] >= 0)
          wait_bounded(smem_u32(&bars->full[s]), last_round[s] & 1, bars, err);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kt = 0; kt < k_tiles && ok; ++kt) {
        const int s = kt % STAGES, round = kt / STAGES;
        ok = wait_bounded(smem_u32(&bars->full[s]), round & 1, bars, err) &&
             wait_bounded(smem_u32(&bars->bready[s]), round & 1, bars, err);
        if (!ok) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t b_addr = smem_u32(stage_b(s));
#pragma unroll
        for (int j = 0; j < MSUB; ++j) {
          const uint32_t a_addr = smem_u32(stage_a(s, j));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(tmem + j * BN, sw128_desc(a_addr + 32 * k),
                      sw128_desc(b_addr + 32 * k), (kt > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&bars->empty[s]));
      }
      // completion of every MMA issued (also on the abort path, before the
      // TMEM is released)
      umma_commit(smem_u32(&bars->accum));
      wait_bounded(smem_u32(&bars->accum), 0, bars, err);
    }
  } else {
    // ------------------------------------------------- dequant + epilogue
    const int r = threadIdx.x - 64;  // weight row of the tile
    const int64_t n = static_cast<int64_t>(n0) + r;
    const bool row_ok = n < N;
    bool ok = true;
    for (int kt = 0; kt < k_tiles; ++kt) {
      const int s = kt % STAGES, round = kt / STAGES;
      if (!wait_bounded(smem_u32(&bars->full[s]), round & 1, bars, err)) {
        ok = false;
        break;
      }
      uint8_t* brow = stage_b(s) + r * 128;
      const int sw = r & 7;
      if (row_ok) {
        const uint4* wp = reinterpret_cast<const uint4*>(stage_wp(s) + r * 32);
        const uint4 c0 = wp[0], c1 = wp[1];
        const float* sc = scales + s * SCALE_FLOATS;
        const Lut l0 = make_lut<QT>(sc[r]);
        Lut l1 = l0;
        if constexpr (BS == 32) l1 = make_lut<QT>(sc[BN + r]);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const uint4 v = dq8(p < 4 ? l0 : l1, cw[p]);
          *reinterpret_cast<uint4*>(brow + ((p ^ sw) << 4)) = v;
        }
      } else {
#pragma unroll
        for (int p = 0; p < 8; ++p)
          *reinterpret_cast<uint4*>(brow + ((p ^ sw) << 4)) = make_uint4(0, 0, 0, 0);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(smem_u32(&bars->bready[s]));
    }
    // epilogue: accumulator j, TMEM lanes 32 q .. 32 q + 31, columns of half h.
    // tcgen05.ld is warp-collective, so the go / no-go decision is made
    // uniform across the warp.
    bool go = __all_sync(0xffffffffu, ok);
    if (go) {
      bool w = true;
      if (lane == 0) w = wait_bounded(smem_u32(&bars->accum), 0, bars, err);
      go = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    }
    if (go) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int q = warp & 3;
      const int h = (warp - 2) >> 2;
#pragma unroll 1
      for (int j = 0; j < MSUB; ++j) {
        const int row = m0 + j * BM + q * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int col = h * 128 + c * 32;
          uint32_t v[32];
          const uint32_t taddr =
              tmem + (static_cast<uint32_t>(q * 32) << 16) + j * BN + col;
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
              "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
              "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
              : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]),
                "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]),
                "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
                "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
                "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
                "=r"(v[30]), "=r"(v[31])
              : "r"(taddr));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          if (row < M && n0 + col < N) {
            uint16_t* dst = Y + static_cast<int64_t>(row) * N + n0 + col;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (n0 + col + 8 * i < N) {
                const uint4 o = make_uint4(
                    pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
                *reinterpret_cast<uint4*>(dst + 8 * i) = o;
              }
            }
          }
        }
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base,
                 uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BS, int QT, bool DQ>
cudaError_t launch_t(const void* X, int64_t M, int64_t K, const bnb4_qstate& W,
                     int64_t N, void* Y, int* err, cudaStream_t s) {
  static bool attr_set[64] = {};  // per device
  auto kern = gemm4_kernel<BS, QT, DQ>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap mx, mw;
  if (!make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.codes, K / 2, N, K / 2,
                   BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((N + BN - 1) / BN),
                  static_cast<unsigned>((M + BM * MSUB - 1) / (BM * MSUB)));
  kern<<<grid, kThreads, SMEM_BYTES, s>>>(mx, mw, static_cast<int>(M), static_cast<int>(N),
                                          static_cast<int>(K), W.absmax, W.absmax_q,
                                          W.scale2, W.offset, static_cast<uint16_t*>(Y), err);
  return cudaGetLastError();
}

template <int QT, bool DQ>
cudaError_t launch_bs(const void* X, int64_t M, int64_t K, const bnb4_qstate& W,
                      int64_t N, void* Y, int* err, cudaStream_t s) {
  switch (W.blocksize) {
    case 32: return launch_t<32, QT, DQ>(X, M, K, W, N, Y, err, s);
    case 64: return launch_t<64, QT, DQ>(X, M, K, W, N, Y, err, s);
    case 128: return launch_t<128, QT, DQ>(X, M, K, W, N, Y, err, s);
    default: return launch_t<256, QT, DQ>(X, M, K, W, N, Y, err, s);
  }
}

}  // namespace

cudaError_t launch_gemm(const void* X, int64_t M, int64_t K,
                        const bnb4_qstate& W, int64_t N, void* Y, int* err,
                        int num_sms, cudaStream_t s) {
  (void)num_sms;
  if (W.qtype == kQtNF4)
    return W.double_quant ? launch_bs<kQtNF4, true>(X, M, K, W, N, Y, err, s)
                          : launch_bs<kQtNF4, false>(X, M, K, W, N, Y, err, s);
  return W.double_quant ? launch_bs<kQtFP4, true>(X, M, K, W, N, Y, err, s)
                        : launch_bs<kQtFP4, false>(X, M, K, W, N, Y, err, s);
}

}  // namespace bnb4
