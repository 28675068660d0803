// gemm_small.cu -- small-M linear with fused 4-bit weight dequantization on
// sm_100a (the batch tier between the decode GEMV and the prefill GEMM):
//   Y[m, n] = h( sum_k X[m, k] * What[n, k] + bias[n] ),  1 <= M <= 256,
//   What[n, k] = h(RN(t[code] * a_hat))  (exact dequantized weight),
// h = round to the 16-bit compute format (bf16 or fp16, nearest even), bias
// optional; fp32 accumulation in tensor memory by tcgen05.mma (kind::f16,
// bf16 or fp16 inputs).
//
// Method: the fused 4-bit dequantize + matmul of bitsandbytes' release notes
// 0.50.0 (ossradar page) for few tokens, over the NF4 / FP4 blockwise format
// of the CSDN article (section "数学原理对比"), nested quantization decoded
// inside.
//
// Design.  With few tokens the weight stream is the whole cost, so every
// weight byte is read and dequantized exactly once and the tokens ride along:
//  * operands swapped: the CTA's 128 dequantized weight rows are the MMA's
//    M (128, cta_group::1), the tokens its N (M rounded up to 16); the
//    accumulator is 128 TMEM lanes (weight rows) x NT columns (tokens).
//  * split K over a cluster of S CTAs (1..8) that share the 128 rows; each
//    CTA takes a contiguous run of 64-wide K steps.  The partial accumulators
//    meet in shared memory and are summed in rank order through distributed
//    shared memory, each CTA reducing and storing a share of the tokens --
//    a fixed order, so results are bit-reproducible.  The host picks S so
//    that the clusters fill the SMs evenly.
//  * warp 0: TMA producer of X (NT x 64 16-bit values per K step, 128-byte swizzle;
//    rows past M read as zeros; 2 stages up to 96 tokens, else 4).  Warp 1:
//    allocates TMEM; one lane issues 4
//    tcgen05.mma (K 16 each) per step and commits to the stages' "empty"
//    barriers.  Warps 2..9: two groups of 4 warps (thread r owns weight row
//    r) alternate K steps; each thread loads its row's 32 code bytes and
//    block scales two of its steps ahead straight into registers (every code
//    byte is used by exactly one thread, so no staging), builds the block's
//    16-bit table, dequantizes with byte permutes into the 128-byte-swizzled
//    K-major A stage, then fence.proxy.async and one arrive per warp.
//  * epilogue: the same 8 warps read the accumulator with tcgen05.ld (warp w
//    sees TMEM lanes 32 (w mod 4) ..), either rounding and storing directly (S = 1)
//    or through the cluster reduction.
//  * every mbarrier wait is bounded in time; on expiry the CTA sets the
//    library's device error word, drains what it started and still reaches
//    both cluster barriers, so its peers never wait on it.
//  No TMA load uses cluster multicast.
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace bnb4 {
namespace {

constexpr int ROWS = 128;             // weight rows per CTA (MMA M)
constexpr int BK = 64;                // K per step (one 128-byte swizzle row)
constexpr int SA = 4;                 // dequantized weight stages
constexpr int kMaxSX = 4;             // X stages: 4, or 2 up to kTwoStageMaxNT tokens
// With 2 X stages up to 96 tokens the CTA's shared memory shrinks by 2 X
// tiles, which leaves the L1 room for the block scales' cache lines (and
// lets 2 CTAs share an SM up to 96 tokens): measured on B200, 5-26% faster
// at 32-96 tokens on the Llama-7B shapes (4096 x 11008 at 64 tokens: 40.5 ->
// 29.9 us); from 128 tokens on, 4 stages are as fast or faster.
constexpr int kTwoStageMaxNT = 96;
constexpr int NGROUPS = 2;            // dequant groups, alternating K steps
constexpr int kGroupThreads = ROWS;   // thread r of a group owns weight row r
constexpr int kFirstDeqWarp = 2;
constexpr int kDeqThreads = NGROUPS * kGroupThreads;
constexpr int kThreads = kFirstDeqWarp * 32 + kDeqThreads;  // 320
constexpr int kMaxNT = 256;           // tokens per launch (MMA N <= 256)
constexpr int kMaxCluster = 8;        // portable cluster size
constexpr int A_BYTES = ROWS * BK * 2;  // 16 KB
constexpr int OFF_A = 0;
constexpr int OFF_X = OFF_A + SA * A_BYTES;
static_assert(OFF_X % 1024 == 0, "swizzled tiles need 1024-byte alignment");

// X stage bytes for NT tokens (a multiple of 1024 since NT % 16 == 0).
__host__ __device__ constexpr int x_stage_bytes(int nt) { return nt * BK * 2; }
__host__ __device__ constexpr int bars_offset(int nt, int sx) {
  return OFF_X + sx * x_stage_bytes(nt);
}
constexpr int smem_bytes(int nt, int sx) { return bars_offset(nt, sx) + 256 + 1024 /*align*/; }
constexpr int x_stages(int nt) { return nt <= kTwoStageMaxNT ? 2 : kMaxSX; }
static_assert(smem_bytes(kMaxNT, kMaxSX) <= 232448, "shared memory budget");
// the partial accumulator (fp32, NT x 128) fits in the idle rings
static_assert(ROWS * kMaxNT * 4 <= bars_offset(kMaxNT, kMaxSX), "reduction buffer");
static_assert(ROWS * kTwoStageMaxNT * 4 <= bars_offset(kTwoStageMaxNT, 2), "reduction buffer");

struct Bars {
  uint64_t afull[SA], aempty[SA];  // dequantized stage written / consumed
  uint64_t xfull[kMaxSX], xempty[kMaxSX];  // X stage landed / consumed
  uint64_t accum;                  // all MMAs finished
  uint64_t wait_limit_ns;          // bound of every wait of this launch
  uint32_t tmem_base;
  int abort;
};

// Instruction descriptor: kind::f16, D fp32, A and B both bf16 (format code
// 1) or both fp16 (0), K-major, M = 128 (one CTA), N = nt.
__host__ __device__ constexpr uint32_t idesc_for(int nt, int fmt) {
  return (1u << 4) | (fmt == BNB4_F16 ? 0u : (1u << 7) | (1u << 10)) |
         (static_cast<uint32_t>(nt >> 3) << 17) | (static_cast<uint32_t>(ROWS >> 4) << 24);
}

__device__ __forceinline__ void umma16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on this CTA's barrier `bar` once all previously issued MMAs of the
// thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// One step's inputs of one weight row: its 64 codes and raw block scales.
struct RowStep {
  uint4 c0, c1;     // codes of K 0..31 and 32..63 of the step
  uint32_t u[2];    // absmax_q byte (double quant) or absmax bits, per block
  float g[2];       // scale2 of the block's group (double quant)
};

template <int BS, int QT, bool DQ, int F, int SX>
__global__ void __launch_bounds__(kThreads, 2)
    gemm_small_kernel(const __grid_constant__ CUtensorMap map_x, int M, int N, int K, int nt,
                      uint32_t idesc, uint32_t tmem_cols, const uint8_t* __restrict__ codes,
                      const float* __restrict__ absmax, const uint8_t* __restrict__ absmax_q,
                      const float* __restrict__ scale2, const float* __restrict__ offset,
                      const uint16_t* __restrict__ bias, uint16_t* __restrict__ Y, int* err,
                      uint64_t wait_limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic so every access stays a shared-memory access
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int xs_bytes = x_stage_bytes(nt);
  Bars* bars = reinterpret_cast<Bars*>(smem + bars_offset(nt, SX));
  // programmatic dependent launch (inside a captured graph after a kernel):
  // no global access and no tensor memory taken before the previous kernel
  // has completed
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  uint32_t csize;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));
  const int S = static_cast<int>(csize);
  const int n0 = static_cast<int>(blockIdx.x / csize) * ROWS;
  // this CTA's run of K steps: the first k_tiles % S ranks take one more
  const int k_tiles = K / BK;
  const int base = k_tiles / S, rem = k_tiles % S;
  const int r_ = static_cast<int>(rank);
  const int steps = base + (r_ < rem ? 1 : 0);
  const int kt0 = r_ * base + (r_ < rem ? r_ : rem);

  auto a_tile = [&](int s) { return smem + OFF_A + s * A_BYTES; };
  auto x_tile = [&](int s) { return smem + OFF_X + s * xs_bytes; };
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  // Dequantizing threads (warps 2..): thread r of group grp owns weight row
  // n0 + r and takes K steps i = grp (mod NGROUPS).  The codes and raw block
  // scales of its first two steps are requested here, before the setup
  // below, so their memory latency overlaps it (as does the X tensor map's).
  const bool deq = warp >= kFirstDeqWarp;
  const int dq = deq ? static_cast<int>(threadIdx.x) - kFirstDeqWarp * 32 : 0;
  const int grp = dq / kGroupThreads;
  const int r = dq % kGroupThreads;
  const int64_t n = static_cast<int64_t>(n0) + r;
  const bool row_ok = deq && n < N;
  constexpr int NBLK = BS == 32 ? 2 : 1;
  auto fetch = [&](int i, RowStep& b) {
    b.c0 = b.c1 = make_uint4(0, 0, 0, 0);
    b.u[0] = b.u[1] = 0u;
    b.g[0] = b.g[1] = 0.0f;
    if (row_ok && i < steps) {
      const int64_t k = static_cast<int64_t>(kt0 + i) * BK;
      const uint8_t* src = codes + n * (K / 2) + k / 2;
      b.c0 = ldg_stream_v4(src);
      b.c1 = ldg_stream_v4(src + 16);
      const int64_t blk = (n * K + k) / BS;
#pragma unroll
      for (int j = 0; j < NBLK; ++j) {
        if constexpr (DQ) {
          b.u[j] = __ldg(absmax_q + blk + j);
          b.g[j] = __ldg(scale2 + ((blk + j) >> 8));
        } else {
          b.u[j] = __float_as_uint(__ldg(absmax + blk + j));
        }
      }
    }
  };
  // two register sets, each refilled two of the group's steps ahead
  RowStep b0, b1;
  if (deq) {
    fetch(grp, b0);
    fetch(grp + NGROUPS, b1);
  }
  if (threadIdx.x == 0)
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x))
                 : "memory");

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(bar(bars->afull[s]), kGroupThreads / 32);
      mbar_init(bar(bars->aempty[s]), 1);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(bar(bars->xfull[s]), 1);
      mbar_init(bar(bars->xempty[s]), 1);
    }
    mbar_init(bar(bars->accum), 1);
    bars->abort = 0;
    bars->wait_limit_ns = wait_limit_ns;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = bars->tmem_base;
  bool ok = true;  // dequant / epilogue threads: no wait gave up

  if (warp == 0) {
    // ------------------------------------------------------ X producer
    if (lane == 0) {
      int last = -1;
      for (int i = 0; i < steps; ++i) {
        const int s = i % SX;
        if (!wait_bounded(bar(bars->xempty[s]), ((i / SX) & 1) ^ 1, bars, err)) break;
        const uint32_t fb = bar(bars->xfull[s]);
        mbar_arrive_expect_tx(fb, static_cast<uint32_t>(xs_bytes));
        tma_load_2d(smem_u32(x_tile(s)), &map_x, (kt0 + i) * BK, 0, fb);
        last = i;
      }
      // drain: the loads this CTA issued have landed
      for (int i = last - SX + 1 > 0 ? last - SX + 1 : 0; i <= last; ++i)
        wait_drain(bar(bars->xfull[i % SX]), (i / SX) & 1, bars);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      for (int i = 0; i < steps; ++i) {
        const int sa = i % SA, sx = i % SX;
        if (!wait_bounded(bar(bars->afull[sa]), (i / SA) & 1, bars, err) ||
            !wait_bounded(bar(bars->xfull[sx]), (i / SX) & 1, bars, err))
          break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a_addr = smem_u32(a_tile(sa));
        const uint32_t x_addr = smem_u32(x_tile(sx));
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          umma16(tmem, sw128_desc(a_addr + 32 * k), sw128_desc(x_addr + 32 * k), idesc,
                    (i > 0 || k > 0) ? 1u : 0u);
        umma_commit(bar(bars->aempty[sa]));
        umma_commit(bar(bars->xempty[sx]));
      }
      // completion of every MMA issued (also on the abort path, before the
      // TMEM is released)
      umma_commit(bar(bars->accum));
    }
  } else {
    // ------------------------------------------------------ dequantizers
    const float off = DQ ? __ldg(offset) : 0.0f;
    // one warp-uniform decision per wait: lane 0 waits, the warp follows
    auto warp_wait = [&](uint32_t b, uint32_t parity) {
      bool w = true;
      if (lane == 0) w = wait_bounded(b, parity, bars, err);
      return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    };
    auto step = [&](int i, const RowStep& b) {
      const int sa = i % SA;
      // the MMAs that read this stage last time have completed
      if (!warp_wait(bar(bars->aempty[sa]), ((i / SA) & 1) ^ 1)) return false;
      uint8_t* arow = a_tile(sa) + r * 128;
      const int swz = r & 7;
      if (row_ok) {
        float a0, a1;
        if constexpr (DQ) {
          a0 = __fmaf_rn(static_cast<float>(static_cast<int>(b.u[0]) - 128), b.g[0], off);
          a1 = __fmaf_rn(static_cast<float>(static_cast<int>(b.u[1]) - 128), b.g[1], off);
        } else {
          a0 = __uint_as_float(b.u[0]);
          a1 = __uint_as_float(b.u[1]);
        }
        const Lut l0 = make_lut<QT, F>(a0);
        Lut l1 = l0;
        if constexpr (BS == 32) l1 = make_lut<QT, F>(a1);
        const uint32_t cw[8] = {b.c0.x, b.c0.y, b.c0.z, b.c0.w, b.c1.x, b.c1.y, b.c1.z, b.c1.w};
#pragma unroll
        for (int p = 0; p < 8; ++p)
          *reinterpret_cast<uint4*>(arow + ((p ^ swz) << 4)) = dq8(p < 4 ? l0 : l1, cw[p]);
      } else {
#pragma unroll
        for (int p = 0; p < 8; ++p)
          *reinterpret_cast<uint4*>(arow + ((p ^ swz) << 4)) = make_uint4(0, 0, 0, 0);
      }
      // the stores become visible to the tensor core (async proxy), then one
      // arrive per warp
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->afull[sa]));
      return true;
    };
    for (int i = grp; i < steps && ok; i += 2 * NGROUPS) {
      ok = step(i, b0);
      fetch(i + 2 * NGROUPS, b0);
      if (ok && i + NGROUPS < steps) {
        ok = step(i + NGROUPS, b1);
        fetch(i + 3 * NGROUPS, b1);
      }
    }
    // --------------------------------------------------------- epilogue
    // warp w reads TMEM lanes 32 (w mod 4) .. + 31 (its weight rows) and
    // half h of the NT token columns; the go / no-go decision is warp-uniform
    // (tcgen05.ld is warp-collective)
    bool go = __all_sync(0xffffffffu, ok);
    if (go) go = warp_wait(bar(bars->accum), 0);
    if (go) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int q = warp & 3;
      const int h = (warp - kFirstDeqWarp) >> 2;
      const int row = q * 32 + lane;
      const int64_t nr = static_cast<int64_t>(n0) + row;
      float* red = reinterpret_cast<float*>(smem);  // [NT][128] partial sums
      const int half = nt >> 1;                     // a multiple of 8
#pragma unroll 1
      for (int c = h * half; c < (h + 1) * half; c += 8) {
        uint32_t v[8];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
              "=r"(v[6]), "=r"(v[7])
            : "r"(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (S == 1) {
          const float b = bias && nr < N ? half_to_f32<F>(bias[nr]) : 0.0f;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c + j < M && nr < N)
              Y[static_cast<int64_t>(c + j) * N + nr] = static_cast<uint16_t>(
                  pack2<F>(bias ? __fadd_rn(__uint_as_float(v[j]), b) : __uint_as_float(v[j]),
                           0.0f));
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) red[(c + j) * ROWS + row] = __uint_as_float(v[j]);
        }
      }
    }
  }

  // Every MMA of this CTA has completed before the partial sums are shared
  // and before TMEM is released, also on the abort path.
  if (warp == 1 && lane == 0) wait_drain(bar(bars->accum), 0, bars);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  cluster_sync();  // partial sums of all ranks are in their shared memory
  if (S > 1 && warp >= kFirstDeqWarp) {
    // rank s reduces tokens [s * per, (s + 1) * per): thread (r, c0) sums
    // the ranks' partials of weight row r in rank order, tokens c0, c0 + 2, ..
    const int c0 = grp;    // thread (r, c0): weight row r, tokens c0, c0 + 2, ..
    const int64_t nr = n;
    const int per = (M + S - 1) / S;
    const int t0 = r_ * per;
    const int t1 = t0 + per < M ? t0 + per : M;
    const uint32_t red0 = smem_u32(smem);
    if (nr < N) {
      const float b = bias ? half_to_f32<F>(bias[nr]) : 0.0f;
#pragma unroll 1
      for (int c = t0 + c0; c < t1; c += 2) {
        const uint32_t off = red0 + static_cast<uint32_t>((c * ROWS + r) * 4);
        float part[kMaxCluster];
#pragma unroll
        for (int s = 0; s < kMaxCluster; ++s)
          part[s] = s < S ? ld_cluster_f32(map_to(off, static_cast<uint32_t>(s))) : 0.0f;
        float sum = part[0];
#pragma unroll
        for (int s = 1; s < kMaxCluster; ++s)
          if (s < S) sum += part[s];
        if (bias) sum = __fadd_rn(sum, b);
        Y[static_cast<int64_t>(c) * N + nr] = static_cast<uint16_t>(pack2<F>(sum, 0.0f));
      }
    }
  }
  cluster_sync();  // no CTA leaves while a peer may still read its partials
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(tmem_cols));
  }
}

// Cluster size S (K slices per 128-row tile).  Cost model, in K steps of one
// CTA alone on an SM: every CTA pays kOverheadSteps (launch, first loads,
// epilogue and cluster reduction) plus its steps, stretched by
// kCoResidentStretch per extra CTA sharing the SM; CTAs beyond the resident
// slots run in further waves.  Fitted to graph-timed sweeps of S = 1..8 on
// the Llama-7B projection shapes at 16..256 tokens.
constexpr double kOverheadSteps = 11.0;
constexpr double kCoResidentStretch = 0.65;

int choose_split(int64_t tiles, int k_tiles, int num_sms, int per_sm) {
  int best = 1;
  double best_cost = 1e300;
  const int64_t slots = static_cast<int64_t>(num_sms) * per_sm;
  for (int s = 1; s <= kMaxCluster && s <= k_tiles; ++s) {
    const int64_t ctas = tiles * s;
    const int64_t waves = (ctas + slots - 1) / slots;
    const int64_t resident = ctas < slots ? ctas : slots;
    const int64_t share = (resident + num_sms - 1) / num_sms;  // CTAs per busy SM
    const double stretch = 1.0 + kCoResidentStretch * static_cast<double>(share - 1);
    const double cost = static_cast<double>(waves) *
                        (((k_tiles + s - 1) / s) * stretch + kOverheadSteps);
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

template <int BS, int QT, bool DQ, int F>
cudaError_t launch_t(const void* X, int64_t M, int64_t K, const bnb4_qstate& W, int64_t N,
                     void* Y, const void* bias, int* err, int num_sms, uint64_t wait_limit_ns,
                     cudaStream_t s) {
  // per device; a race only repeats the (idempotent) attribute call
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_relaxed)) {
    e = cudaFuncSetAttribute(gemm_small_kernel<BS, QT, DQ, F, 2>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes(kTwoStageMaxNT, 2));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_small_kernel<BS, QT, DQ, F, kMaxSX>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes(kMaxNT, kMaxSX));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  const int nt = static_cast<int>((M + 15) / 16 * 16);
  const int sx = x_stages(nt);
  auto kern = sx == 2 ? gemm_small_kernel<BS, QT, DQ, F, 2>
                      : gemm_small_kernel<BS, QT, DQ, F, kMaxSX>;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(nt)) cols <<= 1;
  CUtensorMap mx;
  if (!make_map_2d(&mx, F == BNB4_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   X, K, M, K * 2, BK, nt,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int64_t tiles = (N + ROWS - 1) / ROWS;
  const int k_tiles = static_cast<int>(K / BK);
  // CTAs per SM: shared memory allows 2 up to NT = 96, registers 2 at most
  const int per_sm_smem = 233472 / (smem_bytes(nt, sx) + 1024);
  const int per_sm = per_sm_smem < 2 ? (per_sm_smem < 1 ? 1 : per_sm_smem) : 2;
  const int S = choose_split(tiles, k_tiles, num_sms, per_sm);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * S));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes(nt, sx);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic_after_kernel(s) ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, mx, static_cast<int>(M), static_cast<int>(N),
                            static_cast<int>(K), nt, idesc_for(nt, F), cols,
                            static_cast<const uint8_t*>(W.codes),
                            static_cast<const float*>(W.absmax),
                            static_cast<const uint8_t*>(W.absmax_q),
                            static_cast<const float*>(W.scale2),
                            static_cast<const float*>(W.offset),
                            static_cast<const uint16_t*>(bias), static_cast<uint16_t*>(Y), err,
                            wait_limit_ns);
}

template <int QT, bool DQ, int F>
cudaError_t launch_bs(const void* X, int64_t M, int64_t K, const bnb4_qstate& W, int64_t N,
                      void* Y, const void* bias, int* err, int sms, uint64_t lim,
                      cudaStream_t s) {
  switch (W.blocksize) {
    case 32: return launch_t<32, QT, DQ, F>(X, M, K, W, N, Y, bias, err, sms, lim, s);
    case 64: return launch_t<64, QT, DQ, F>(X, M, K, W, N, Y, bias, err, sms, lim, s);
    case 128: return launch_t<128, QT, DQ, F>(X, M, K, W, N, Y, bias, err, sms, lim, s);
    default: return launch_t<256, QT, DQ, F>(X, M, K, W, N, Y, bias, err, sms, lim, s);
  }
}

template <int F>
cudaError_t launch_f(const void* X, int64_t M, int64_t K, const bnb4_qstate& W, int64_t N,
                     void* Y, const void* bias, int* err, int sms, uint64_t lim,
                     cudaStream_t s) {
  if (W.qtype == kQtNF4)
    return W.double_quant ? launch_bs<kQtNF4, true, F>(X, M, K, W, N, Y, bias, err, sms, lim, s)
                          : launch_bs<kQtNF4, false, F>(X, M, K, W, N, Y, bias, err, sms, lim, s);
  return W.double_quant ? launch_bs<kQtFP4, true, F>(X, M, K, W, N, Y, bias, err, sms, lim, s)
                        : launch_bs<kQtFP4, false, F>(X, M, K, W, N, Y, bias, err, sms, lim, s);
}

}  // namespace

cudaError_t launch_gemm_small(const void* X, int64_t M, int64_t K, const bnb4_qstate& W,
                              int64_t N, void* Y, const void* bias, int fmt, int* err,
                              int num_sms, cudaStream_t s, uint64_t wait_limit_ns) {
  if (M < 1 || M > kMaxNT) return cudaErrorInvalidValue;
  const uint64_t lim = wait_limit_ns ? wait_limit_ns : kWaitLimitNs;
  return fmt == BNB4_F16 ? launch_f<BNB4_F16>(X, M, K, W, N, Y, bias, err, num_sms, lim, s)
                         : launch_f<BNB4_BF16>(X, M, K, W, N, Y, bias, err, num_sms, lim, s);
}

}  // namespace bnb4
