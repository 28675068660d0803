// gemm.cu -- prefill GEMM with fused 4-bit weight dequantization, sm_100a:
//   Y[m, n] = h( sum_k X[m, k] * What[n, k] + bias[n] ),
//   What[n, k] = h(RN(t[code] * a_hat))  (exact dequantized weight),
// h = round to the 16-bit compute format (bf16 or fp16, nearest even), bias
// optional; fp32 accumulation in tensor memory by tcgen05.mma (kind::f16,
// bf16 or fp16 inputs).
//
// Method: the fused 4-bit dequantize + GEMM of bitsandbytes' release notes
// 0.50.0 (ossradar page), nested quantization decoded inside, over the NF4 /
// FP4 blockwise format of the CSDN article (section "数学原理对比").
//
// Design: CTA pairs (clusters of 2) with tcgen05.mma.cta_group::2.  A pair
// owns a 512 x 256 output tile: two M = 256 accumulators (each CTA holds 128
// rows of each in its TMEM, 2 x 256 columns) and N = 256 weight rows split in
// halves -- each CTA dequantizes only its 128 weight rows, so the
// dequantization work per flop is a quarter of a one-CTA 128 x 256 MMA.
// Per CTA, 19 warps and three smem rings:
//  * ring A (3 stages): the CTA's two 128 x 64 16-bit tiles of X per 64-wide K
//    step, TMA (128-byte swizzle) completing on the leader CTA's barrier;
//    warp 0 produces it (the leader also arms the barrier with the bytes of
//    both CTAs).
//  * ring W (4 stages, one per dequant group): the CTA's 128 x 32-byte packed weight tile (TMA) plus
//    its 128 decoded block scales (nested quantization decoded by the 32
//    lanes of warp 2, whose scale loads run two steps ahead).
//  * ring B (6 stages): the CTA's dequantized 128 x 64 16-bit weight half,
//    written by warps 3..18 in four groups of 4 warps (group g takes the K
//    steps kt = g mod 4 and owns B slot g; thread r of a group owns weight
//    row r) in the 128-byte-swizzled K-major layout, then fence.proxy.async
//    and one cluster-scope arrive per warp on the leader's barrier.
//  * warp 1: allocates 512 TMEM columns in both CTAs; in the leader one lane
//    waits for the A and B stages of both CTAs and issues 2 x 4
//    tcgen05.mma.cta_group::2 (M 256, N 256, K 16), then commits to the
//    "empty" barriers of both CTAs (multicast commit).
//  * epilogue: warps 3..18 of each CTA read its accumulator rows with
//    tcgen05.ld, add the bias, round to the compute format and store.
//  * Every mbarrier wait is bounded in time; on expiry the CTA sets the
//    library's device error word, drains what it started and exits.
//  No TMA load uses cluster multicast.
#include <atomic>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace bnb4 {
namespace {

constexpr int BM = 128;      // rows of one accumulator per CTA
constexpr int MSUB = 2;      // accumulators (M = 256 each across the pair)
constexpr int BNP = 256;     // weight rows per pair (N of one MMA)
constexpr int BNC = 128;     // weight rows per CTA
constexpr int BK = 64;       // K per stage (one 128-byte swizzle row of 16-bit values)
constexpr int SA = 3;        // X stages
// Dequantized weight stages: K step kt uses stage kt % SB, so the group that
// dequantizes step kt + 4 (4 groups take every 4th step) refills the stage
// the MMA of step kt + 4 - SB used; 6 stages give the groups 2 more MMA
// steps of slack than 4 (measured: 4% faster on all three Llama shapes).
constexpr int SB = 6;
constexpr int SW = 4;        // packed weight + scale stages (one per group)
constexpr int NGROUPS = 4;   // dequant groups (one K step each in flight)
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int A_STAGE = MSUB * A_BYTES;  // 32 KB
constexpr int B_BYTES = BNC * BK * 2;    // 16 KB
constexpr int WP_BYTES = BNC * BK / 2;   // 4 KB packed codes
constexpr int SCALE_FLOATS = 2 * BNC;    // 2 per row for blocksize 32
constexpr int Y_BOX_BYTES = BM * 64 * 2;  // 16 KB output box (128 rows x 64 values)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + SA * A_STAGE;
constexpr int OFF_W = OFF_B + SB * B_BYTES;
constexpr int OFF_S = OFF_W + SW * WP_BYTES;
constexpr int OFF_BARS = OFF_S + SW * SCALE_FLOATS * 4;
constexpr int kDeqWarps = 16;
constexpr int kGroupThreads = BNC;  // threads per group = weight rows of a CTA
constexpr int kFirstDeqWarp = 3;
constexpr int kThreads = (kFirstDeqWarp + kDeqWarps) * 32;
constexpr int TMEM_COLS = 512;
constexpr int SMEM_BYTES = OFF_BARS + 256 + 1024 /*align*/;
static_assert(OFF_B % 1024 == 0 && OFF_W % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(kDeqWarps * 32 == NGROUPS * kGroupThreads, "groups");
static_assert(SW == NGROUPS, "each group owns one packed-weight stage");
static_assert(4 * MSUB * Y_BOX_BYTES <= OFF_W, "output boxes fit in the X and B rings");

struct Bars {
  uint64_t afull[SA], aempty[SA];  // X tiles of both CTAs landed (leader) / consumed
  uint64_t wfull[SW], wempty[SW];  // codes + scales ready / read (local)
  uint64_t bfull[SB], bempty[SB];  // dequantized halves written (leader) / consumed
  uint64_t accum;                  // all MMAs finished
  uint64_t wait_limit_ns;  // bound of every wait of this launch
  uint32_t tmem_base;
  int abort;
};

// Instruction descriptor: kind::f16, D fp32, A and B both bf16 (format code
// 1) or both fp16 (0), K-major, N = 256, M = 256 (two CTAs).
template <int F>
constexpr uint32_t kIdesc = (1u << 4) | (F == BNB4_F16 ? 0u : (1u << 7) | (1u << 10)) |
                            (static_cast<uint32_t>(BNP >> 3) << 17) |
                            (static_cast<uint32_t>((2 * BM) >> 4) << 24);

template <int F>
__device__ __forceinline__ void umma16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc<F>), "r"(accumulate));
}

// Arrive on the barrier at `bar`'s offset in both CTAs of the pair once all
// previously issued MMAs have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\t"
      "mov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], m;\n\t}" ::"r"(bar)
      : "memory");
}

template <int BS, int QT, bool DQ, int F>
__global__ void __launch_bounds__(kThreads, 1)
    gemm4_kernel(const __grid_constant__ CUtensorMap map_x,
                 const __grid_constant__ CUtensorMap map_w,
                 const __grid_constant__ CUtensorMap map_y, int M, int N, int K,
                 int n_pair_cols, const float* __restrict__ absmax,
                 const uint8_t* __restrict__ absmax_q,
                 const float* __restrict__ scale2,
                 const float* __restrict__ offset, const uint16_t* __restrict__ bias,
                 int* err, uint64_t wait_limit_ns, int withhold_first_x) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic (not an integer cast) so every access stays a shared-memory
  // access rather than a generic one
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BARS);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int m_pair = (pair / n_pair_cols) * (2 * MSUB * BM);
  const int n_pair = (pair % n_pair_cols) * BNP;
  const int n0 = n_pair + static_cast<int>(rank) * BNC;  // this CTA's weight rows
  const int k_tiles = K / BK;

  auto a_tile = [&](int s, int j) { return smem + OFF_A + s * A_STAGE + j * A_BYTES; };
  auto b_tile = [&](int s) { return smem + OFF_B + s * B_BYTES; };
  auto w_tile = [&](int s) { return smem + OFF_W + s * WP_BYTES; };
  auto scales = [&](int s) {
    return reinterpret_cast<float*>(smem + OFF_S) + s * SCALE_FLOATS;
  };
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(bar(bars->afull[s]), 1);
      mbar_init(bar(bars->aempty[s]), 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(bar(bars->wfull[s]), 32);
      mbar_init(bar(bars->wempty[s]), kGroupThreads / 32);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(bar(bars->bfull[s]), 2 * kGroupThreads / 32);
      mbar_init(bar(bars->bempty[s]), 1);
    }
    mbar_init(bar(bars->accum), 1);
    bars->abort = 0;
    bars->wait_limit_ns = wait_limit_ns;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------ X producer
    if (lane == 0) {
      int last = -1;
      for (int kt = 0; kt < k_tiles; ++kt) {
        const int s = kt % SA, round = kt / SA;
        if (!wait_bounded(bar(bars->aempty[s]), (round & 1) ^ 1, bars, err)) break;
        // failure-detection diagnostic: the first X stage is never armed or
        // loaded, so the MMA's wait for it runs out (nothing else changes)
        if (withhold_first_x && kt == 0) continue;
        const uint32_t fb = bar(bars->afull[s]);
        if (leader) mbar_arrive_expect_tx(fb, 2 * A_STAGE);  // bytes of both CTAs
        const uint32_t cfb = map_to(fb, 0);
        for (int j = 0; j < MSUB; ++j)
          tma_load_2d_pair(smem_u32(a_tile(s, j)), &map_x, kt * BK,
                           m_pair + j * 2 * BM + static_cast<int>(rank) * BM, cfb);
        last = kt;
      }
      // drain: the loads this CTA issued have landed (the leader's barrier
      // completes only when both CTAs' bytes arrived)
      for (int kt = last - SA + 1 > 0 ? last - SA + 1 : 0; kt <= last; ++kt)
        if (leader) wait_drain<true>(bar(bars->afull[kt % SA]), (kt / SA) & 1, bars);
    }
  } else if (warp == 2) {
    // ------------------------------- packed weight + scale producer
    // The raw scale inputs of a step are loaded two steps ahead into one of
    // two register sets, so their latency overlaps the waits and the TMAs.
    const float off = DQ ? __ldg(offset) : 0.0f;
    constexpr int RPL = BNC / 32;  // rows per lane
    constexpr int NBLK = BS == 32 ? 2 : 1;
    auto fetch = [&](int kt, uint32_t (&u)[RPL][NBLK], float (&g)[RPL][NBLK]) {
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        const int64_t n = static_cast<int64_t>(n0) + lane + 32 * i;
#pragma unroll
        for (int j = 0; j < NBLK; ++j) {
          u[i][j] = 0u;
          g[i][j] = 0.0f;
          if (n < N && kt < k_tiles) {
            const int64_t b = (n * K + static_cast<int64_t>(kt) * BK) / BS + j;
            if constexpr (DQ) {
              u[i][j] = __ldg(absmax_q + b);
              g[i][j] = __ldg(scale2 + (b >> 8));
            } else {
              u[i][j] = __float_as_uint(__ldg(absmax + b));
            }
          }
        }
      }
    };
    // two register sets, each refilled two steps ahead of its use
    uint32_t ua[RPL][NBLK], ub[RPL][NBLK];
    float ga[RPL][NBLK], gb[RPL][NBLK];
    fetch(0, ua, ga);
    fetch(1, ub, gb);
    int last = -1;
    bool ok = true;
    auto step = [&](int kt, const uint32_t (&u)[RPL][NBLK], const float (&g)[RPL][NBLK]) {
      const int s = kt % SW, round = kt / SW;
      if (!wait_bounded(bar(bars->wempty[s]), (round & 1) ^ 1, bars, err)) {
        ok = false;
        return;
      }
      const uint32_t fb = bar(bars->wfull[s]);
      if (lane == 0) {
        mbar_expect_tx_only(fb, WP_BYTES);
        tma_load_2d(smem_u32(w_tile(s)), &map_w, kt * (BK / 2), n0, fb);
      }
      last = kt;
      float* sc = scales(s);
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        const int row = lane + 32 * i;
#pragma unroll
        for (int j = 0; j < NBLK; ++j) {
          float a;
          if constexpr (DQ)
            a = __fmaf_rn(static_cast<float>(static_cast<int>(u[i][j]) - 128), g[i][j], off);
          else
            a = __uint_as_float(u[i][j]);
          sc[j * BNC + row] = a;
        }
      }
      mbar_arrive(fb);
    };
    for (int kt = 0; kt < k_tiles && ok; kt += 2) {
      step(kt, ua, ga);
      fetch(kt + 2, ua, ga);
      if (kt + 1 < k_tiles && ok) {
        step(kt + 1, ub, gb);
        fetch(kt + 3, ub, gb);
      }
    }
    if (lane == 0)
      for (int kt = last - SW + 1 > 0 ? last - SW + 1 : 0; kt <= last; ++kt)
        wait_drain(bar(bars->wfull[kt % SW]), (kt / SW) & 1, bars);
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader CTA)
    if (leader && lane == 0) {
      for (int kt = 0; kt < k_tiles; ++kt) {
        const int sa = kt % SA, sb = kt % SB;
        if (!wait_bounded<true>(bar(bars->afull[sa]), (kt / SA) & 1, bars, err) ||
            !wait_bounded<true>(bar(bars->bfull[sb]), (kt / SB) & 1, bars, err))
          break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t b_addr = smem_u32(b_tile(sb));
#pragma unroll
        for (int j = 0; j < MSUB; ++j) {
          const uint32_t a_addr = smem_u32(a_tile(sa, j));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma16_pair<F>(tmem + j * BNP, sw128_desc(a_addr + 32 * k),
                           sw128_desc(b_addr + 32 * k), (kt > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit_pair(bar(bars->aempty[sa]));
        umma_commit_pair(bar(bars->bempty[sb]));
      }
      // completion of every MMA issued, signalled to both CTAs (also on the
      // abort path, before the TMEM is released)
      umma_commit_pair(bar(bars->accum));
    }
  } else {
    // ------------------------------------------------- dequant + epilogue
    const int dq = threadIdx.x - kFirstDeqWarp * 32;
    const int grp = dq / kGroupThreads;   // takes K steps kt = grp (mod 4)
    const int r = dq % kGroupThreads;     // weight row of this CTA's half
    const bool row_ok = static_cast<int64_t>(n0) + r < N;
    bool ok = true;
    for (int kt = grp; kt < k_tiles; kt += NGROUPS) {
      const int sw = kt % SW, sb = kt % SB;
      if (!wait_bounded(bar(bars->wfull[sw]), (kt / SW) & 1, bars, err)) {
        ok = false;
        break;
      }
      const uint4* wp = reinterpret_cast<const uint4*>(w_tile(sw) + r * 32);
      const uint4 c0 = wp[0], c1 = wp[1];
      const float* sc = scales(sw);
      const float s0 = sc[r];
      const float s1 = BS == 32 ? sc[BNC + r] : s0;
      // the next TMA load into this stage (async proxy) must not overtake
      // these shared-memory reads (generic proxy): order them before the
      // release
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->wempty[sw]));
      if (!wait_bounded(bar(bars->bempty[sb]), ((kt / SB) & 1) ^ 1, bars, err)) {
        ok = false;
        break;
      }
      uint8_t* brow = b_tile(sb) + r * 128;
      const int swz = r & 7;
      if (row_ok) {
        const Lut l0 = make_lut<QT, F>(s0);
        Lut l1 = l0;
        if constexpr (BS == 32) l1 = make_lut<QT, F>(s1);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const uint4 v = dq8(p < 4 ? l0 : l1, cw[p]);
          *reinterpret_cast<uint4*>(brow + ((p ^ swz) << 4)) = v;
        }
      } else {
#pragma unroll
        for (int p = 0; p < 8; ++p)
          *reinterpret_cast<uint4*>(brow + ((p ^ swz) << 4)) = make_uint4(0, 0, 0, 0);
      }
      // every lane makes its stores visible to the tensor core (async proxy),
      // then one cluster-scope release per warp signals the leader
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to(bar(bars->bfull[sb]), 0));
    }
    // epilogue: accumulator j, TMEM lanes 32 q .. 32 q + 31 (rows of this
    // CTA), a 64-column quarter h.  The tile goes through shared memory --
    // the X and dequantized-weight rings are idle once every MMA has
    // completed -- as 4 * MSUB boxes of 128 rows x 64 columns in the 128-byte
    // swizzled layout of the TMA store, then leaves in 4 * MSUB tensor
    // stores: whole 128-byte row segments instead of one 16-byte piece per
    // row per store instruction.  tcgen05.ld is warp-collective, so the go /
    // no-go decision is uniform across the warp; every epilogue warp reaches
    // the named barrier, go or not.
    bool go = __all_sync(0xffffffffu, ok);
    if (go) {
      bool w = true;
      if (lane == 0) w = wait_bounded(bar(bars->accum), 0, bars, err);
      go = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    }
    uint8_t* ybuf = smem + OFF_A;  // 4 * MSUB boxes of 16 KB
    if (go) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int q = warp & 3;                     // TMEM lane quarter
      const int h = (warp - kFirstDeqWarp) >> 2;  // 64-column quarter
      const int r = q * 32 + lane;                // row of the CTA's 128
#pragma unroll 1
      for (int j = 0; j < MSUB; ++j) {
        uint8_t* box = ybuf + (j * 4 + h) * Y_BOX_BYTES + r * 128;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          const uint32_t taddr =
              tmem + (static_cast<uint32_t>(q * 32) << 16) + j * BNP + h * 64 + c * 32;
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
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // 16-byte chunk c * 4 + i of the row
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * i + e]);
            // bias of the chunk's 8 columns (N % 8 == 0: a chunk is wholly
            // inside or outside the N edge)
            const int col0 = n_pair + h * 64 + c * 32 + 8 * i;
            if (bias && col0 < N) {
              const uint4 bb = __ldg(reinterpret_cast<const uint4*>(bias + col0));
              const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
              for (int e = 0; e < 8; ++e)
                f[e] = __fadd_rn(f[e], half_to_f32<F>(e & 1 ? bw[e >> 1] >> 16 : bw[e >> 1]));
            }
            const uint4 o = make_uint4(pack2<F>(f[0], f[1]), pack2<F>(f[2], f[3]),
                                       pack2<F>(f[4], f[5]), pack2<F>(f[6], f[7]));
            *reinterpret_cast<uint4*>(box + (((c * 4 + i) ^ (r & 7)) << 4)) = o;
          }
        }
      }
      // the stores become visible to the TMA (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kDeqWarps * 32) : "memory");
    if (threadIdx.x == kFirstDeqWarp * 32 && !*reinterpret_cast<volatile int*>(&bars->abort)) {
      // boxes past the M or N edge are skipped; a box that straddles an edge
      // is clipped by the TMA
#pragma unroll 1
      for (int bx = 0; bx < 4 * MSUB; ++bx) {
        const int x = n_pair + (bx & 3) * 64;
        const int y = m_pair + (bx >> 2) * 2 * BM + static_cast<int>(rank) * BM;
        if (x < N && y < M) tma_store_2d(&map_y, smem_u32(ybuf + bx * Y_BOX_BYTES), x, y);
      }
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // written before exit
    }
  }

  // Teardown: every MMA of the pair has completed (the accum barrier of this
  // CTA) before either CTA releases TMEM or exits, and neither exits while
  // the other may still arrive on its barriers.
  if (warp == 1 && lane == 0) wait_drain(bar(bars->accum), 0, bars);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS));
  }
}

template <int BS, int QT, bool DQ, int F>
cudaError_t launch_t(const void* X, int64_t M, int64_t K, const bnb4_qstate& W,
                     int64_t N, void* Y, const void* bias, int* err, uint64_t wait_limit_ns,
                     int withhold, cudaStream_t s) {
  // per device; a race only repeats the (idempotent) attribute call
  static std::atomic<bool> attr_set[64];
  auto kern = gemm4_kernel<BS, QT, DQ, F>;
  constexpr CUtensorMapDataType kT16 =
      F == BNB4_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_relaxed)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  CUtensorMap mx, mw, my;
  if (!make_map_2d(&mx, kT16, X, K, M, K * 2, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.codes, K / 2, N, K / 2,
                   BK / 2, BNC, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!make_map_2d(&my, kT16, Y, N, M, N * 2, 64, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int n_pair_cols = static_cast<int>((N + BNP - 1) / BNP);
  const int m_pairs = static_cast<int>((M + 2 * MSUB * BM - 1) / (2 * MSUB * BM));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * n_pair_cols * m_pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mx, mw, my, static_cast<int>(M), static_cast<int>(N),
                            static_cast<int>(K), n_pair_cols, W.absmax, W.absmax_q,
                            W.scale2, W.offset, static_cast<const uint16_t*>(bias), err,
                            wait_limit_ns, withhold);
}

template <int QT, bool DQ, int F>
cudaError_t launch_bs(const void* X, int64_t M, int64_t K, const bnb4_qstate& W,
                      int64_t N, void* Y, const void* bias, int* err, uint64_t lim,
                      int withhold, cudaStream_t s) {
  switch (W.blocksize) {
    case 32: return launch_t<32, QT, DQ, F>(X, M, K, W, N, Y, bias, err, lim, withhold, s);
    case 64: return launch_t<64, QT, DQ, F>(X, M, K, W, N, Y, bias, err, lim, withhold, s);
    case 128: return launch_t<128, QT, DQ, F>(X, M, K, W, N, Y, bias, err, lim, withhold, s);
    default: return launch_t<256, QT, DQ, F>(X, M, K, W, N, Y, bias, err, lim, withhold, s);
  }
}

template <int F>
cudaError_t launch_f(const void* X, int64_t M, int64_t K, const bnb4_qstate& W, int64_t N,
                     void* Y, const void* bias, int* err, uint64_t lim, int wh,
                     cudaStream_t s) {
  if (W.qtype == kQtNF4)
    return W.double_quant ? launch_bs<kQtNF4, true, F>(X, M, K, W, N, Y, bias, err, lim, wh, s)
                          : launch_bs<kQtNF4, false, F>(X, M, K, W, N, Y, bias, err, lim, wh, s);
  return W.double_quant ? launch_bs<kQtFP4, true, F>(X, M, K, W, N, Y, bias, err, lim, wh, s)
                        : launch_bs<kQtFP4, false, F>(X, M, K, W, N, Y, bias, err, lim, wh, s);
}

}  // namespace

cudaError_t launch_gemm(const void* X, int64_t M, int64_t K,
                        const bnb4_qstate& W, int64_t N, void* Y, const void* bias,
                        int fmt, int* err, int num_sms, cudaStream_t s,
                        uint64_t wait_limit_ns, int withhold_first_x) {
  (void)num_sms;
  const uint64_t lim = wait_limit_ns ? wait_limit_ns : kWaitLimitNs;
  const int wh = withhold_first_x;
  return fmt == BNB4_F16 ? launch_f<BNB4_F16>(X, M, K, W, N, Y, bias, err, lim, wh, s)
                         : launch_f<BNB4_BF16>(X, M, K, W, N, Y, bias, err, lim, wh, s);
}

}  // namespace bnb4
