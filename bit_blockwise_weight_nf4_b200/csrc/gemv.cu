// gemv.cu -- decode GEMV with 4-bit weights on sm_100a:
//   y[b, n] = h( sum_k x[b, k] * What[n, k] + bias[n] ),  1 <= B <= 8,
//   What[n, k] = h(RN(t[code] * a_hat))   (dequantized weight, exact),
// h = round to the 16-bit compute format, bf16 or fp16 (nearest even); the
// bias is optional.
//
// This kernel serves lists of four or more weights with one row of x; single
// weights, short lists and B > 1 run the one-CTA-per-16-rows kernel of
// gemv_direct.cu (faster there).
//
// Method: bitsandbytes' gemv_4bit op (ossradar page, release notes 0.50.0)
// over the blockwise NF4 / FP4 format of the CSDN article (section
// "数学原理对比"), nested (double) quantization decoded in-kernel.
//
// Design.  The exact table lookup costs about 2.5 integer-ALU operations per
// weight (byte permutes run at half the FMA rate), so on B200 the kernel is
// bound by the ALU pipe before HBM; everything else is kept off the
// per-weight path.
//  * Persistent grid, one CTA of 16 warps per SM; each CTA owns a balanced,
//    contiguous range of 16-row groups.  A work item is 16 rows x 256 K (2 KB
//    of codes); lane (g, t) of a warp owns rows g and g + 8 and the
//    64-element K segment t of the item.
//  * The CTA's items, in row-major order (row group, K chunk), are cut into
//    16 contiguous runs, one per warp.  A warp sums each row group it covers
//    in registers and stores it; only a row group that two or more warps
//    share (at most one per run boundary) goes through shared memory, added
//    after one barrier at the end in warp order -- a fixed order, so results
//    are bit-reproducible for a given problem list and SM count.
//  * Each warp streams its run through a private 4-stage ring: lane 0 starts
//    a 2-D TMA copy of the code tile (128-byte swizzle) on the stage's
//    mbarrier, the lanes copy the words holding their blocks' scales with
//    cp.async, four items ahead of the math.
//  * Dequantization by byte permutes (lut.cuh): per (row, quant block) a lane
//    builds the 16-entry table of h(RN(t[i] * a_hat)), bit-identical to
//    dequantizing every element.  Products on mma.sync m16n8k16 (weights as
//    the A operand, 16 rows; x as B, batch columns): K is permuted
//    identically in both operands, which leaves the dot products unchanged.
//    Lanes of batch columns beyond B hold zeros and load nothing.
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "lut.cuh"
#include "sm100.cuh"

namespace bnb4 {
namespace {

constexpr int kWarps = 16;                        // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;                        // ring depth per warp
constexpr int kRows = 16;                         // rows of an item (MMA M)
constexpr int kItemK = 256;                       // K of an item (4 lanes x 64)

constexpr int kTileBytes = kRows * kItemK / 2;    // packed codes of one item: 2 KB

// Per warp, a ring of kStages items: the code tile (16 rows x 128 bytes,
// written by TMA with the 128-byte swizzle: 16-byte chunk c of row r sits at
// chunk c ^ (r & 7)), the lane-major scale words and the tile's "full"
// mbarrier; and the warp's partial sums of the (at most two) row groups it
// shares with its neighbours.
struct Smem {
  uint8_t tiles[kWarps][kStages][kTileBytes];
  uint32_t sc[kWarps][kStages][4][32];  // dq: [u word g, u word g+8, scale2 g, scale2 g+8]
                                        // else [absmax g, absmax g+8, next g, next g+8]
  float4 part[2][kWarps][32];           // [0]: the warp's first row group, [1]: its last
  uint64_t full[kWarps][kStages];
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment of the tiles
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert((kStages & (kStages - 1)) == 0, "ring index by mask");
static_assert(kTileBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");

// One GEMV of a launch: y = x . What^T (+ bias) for a weight [N, K] (K is
// the launch's).
struct Prob {
  const uint16_t* x;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* scale2;
  const float* offset;
  const uint16_t* bias;
  uint16_t* y;
  int64_t nb;  // quant blocks, N * K / blocksize
  int N;
  int rg0;     // first row group of this problem in the launch's list
};

// The problems of a launch (their row groups concatenated in order), all
// with the same K, batch size B, blocksize, code table and scale format, and
// each one's tensor map of its codes viewed as uint8 [N, K / 2] (box 128
// bytes x 16 rows, 128-byte swizzle; rows past N and bytes past K / 2 read
// as zeros).
template <int MAXP>
struct Group {
  CUtensorMap maps[MAXP];
  Prob p[MAXP];
  int count;
  int B;
  int K;
  int C;      // 256-wide K chunks per row group
  int kb;     // quant blocks per row, K / blocksize
  int n_rg;   // row groups of all problems
  uint32_t k16, k31;  // 2^16 and 2^31, opaque to the compiler (see dq8_fma)
  int* err;           // the library's device error word
};
constexpr int kSmallGroup = 4;   // q/k/v, gate/up
constexpr int kLargeGroup = 32;  // a longer list is launched in parts of 32
static_assert(sizeof(Group<kLargeGroup>) <= 32000, "kernel parameter space");

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// 4-byte slot of which only the first `bytes` (1..4) are read from global
// memory, the rest zero-filled: never reads past the end of a byte array.
__device__ __forceinline__ void cp_async4_part(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

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

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Bounded wait for a code tile; on expiry the device error word is set and
// the warp goes on (its output is then wrong and reported as such; every
// barrier of the protocol is still reached, so nothing hangs).
__device__ __forceinline__ void wait_tile(uint32_t full, uint32_t parity, int* err) {
  if (mbar_try_wait<false>(full, parity)) return;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait<false>(full, parity))
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicExch(err, 1);
      return;
    }
}

// Write the fp32 sums of one row group (this lane's rows g, g + 8 and batch
// columns 2t, 2t + 1) rounded once, after the bias.
template <int F>
__device__ __forceinline__ void store_rows(const float4& v, int rl, int lane, const Prob& a,
                                           int B) {
  const int g = lane >> 2, t = lane & 3;
  const float s[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int n = rl * kRows + g + 8 * r;
    if (n >= a.N) continue;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      const int col = 2 * t + cb;
      if (col < B) {
        float val = s[2 * r + cb];
        if (a.bias) val = __fadd_rn(val, half_to_f32<F>(a.bias[n]));
        a.y[static_cast<int64_t>(col) * a.N + n] = static_cast<uint16_t>(pack2<F>(val, 0.0f));
      }
    }
  }
}

// A position in a CTA's item sequence: global row group rg, K chunk kc and
// the problem p that rg belongs to.  Stepping costs an increment and a
// compare, a new row group one more compare, a new problem one parameter
// load.
template <int MAXP>
struct Pos {
  int rg, kc, p, next_rg0;
  __device__ void seek(const Group<MAXP>& grp, int rg_, int kc_, int p_from) {
    rg = rg_;
    kc = kc_;
    p = p_from;
    while (p + 1 < grp.count && rg >= grp.p[p + 1].rg0) ++p;
    next_rg0 = p + 1 < grp.count ? grp.p[p + 1].rg0 : 0x7fffffff;
  }
  // to the next item; true when that item begins a new row group
  __device__ bool step(const Group<MAXP>& grp) {
    if (++kc < grp.C) return false;
    kc = 0;
    if (++rg >= next_rg0) {
      ++p;
      next_rg0 = p + 1 < grp.count ? grp.p[p + 1].rg0 : 0x7fffffff;
    }
    return true;
  }
};

// The copies of one warp's run of items, issued kStages items ahead of the
// math: lane 0 arms the stage's barrier and starts the TMA of the code tile;
// every lane copies the words holding its two rows' block scales.  Rows past
// N and segments past K copy no scales (the TMA fills their codes with
// zeros).
template <int BS, bool DQ, int MAXP, bool QUAD>
struct Fetch {
  const Group<MAXP>& grp;
  int lane, t;
  Pos<MAXP> pos;
  int left;             // items not yet issued
  int row0;             // first row of the row group within its problem
  int64_t blk0;         // block of row g at k = 0
  bool ok0, ok1, last;  // rows g, g + 8 exist; the problem's last row group
  // the problem's scale arrays
  const uint8_t* aq;
  const float* s2;
  int64_t nb;
  // QUAD: the row this lane copies a word of (g + 8 (t & 1)), as the
  // block at the start of the current chunk, and whether that row exists
  int64_t qb;
  bool qv;

  __device__ Fetch(const Group<MAXP>& gp, int lane_, const Pos<MAXP>& start, int count)
      : grp(gp), lane(lane_), t(lane_ & 3), pos(start), left(count) {
    enter();
  }
  __device__ void enter() {
    const Prob& a = grp.p[pos.p];
    row0 = (pos.rg - a.rg0) * kRows;
    const int n0 = row0 + (lane >> 2);
    blk0 = static_cast<int64_t>(n0) * grp.kb;
    ok0 = n0 < a.N;
    ok1 = n0 + 8 < a.N;
    last = row0 + kRows >= a.N;
    aq = a.absmax_q;
    s2 = a.scale2;
    nb = a.nb;
    qb = blk0 + static_cast<int64_t>(8 * (t & 1)) * grp.kb + pos.kc * (kItemK / BS);
    qv = (t & 1) ? ok1 : ok0;
  }

  __device__ void issue(uint8_t* tile, uint32_t* sc, uint32_t full) {
    if (left == 0) return;
    --left;
    if (lane == 0) {
      mbar_arrive_expect_tx(full, kTileBytes);
      tma_load_2d(smem_u32(tile), &grp.maps[pos.p], pos.kc * (kItemK / 2), row0, full);
    }
    if constexpr (QUAD) {
      // one word per lane, no branches: t < 2 the aligned absmax_q word of
      // its row (cut at the end of the array in the last row group), t >= 2
      // the row's scale2; a missing row copies nothing (zero-fill)
      const int64_t wb = qb & ~int64_t(3);
      const void* src = t < 2 ? static_cast<const void*>(aq + wb)
                              : static_cast<const void*>(s2 + (qb >> 8));
      uint32_t bytes = 4;
      if (t < 2 && last) {
        const int64_t rest = nb - wb;
        bytes = static_cast<uint32_t>(rest < 4 ? rest : 4);
      }
      if (!qv) {
        bytes = 0;
        src = s2;
      }
      cp_async4_part(smem_u32(sc + lane), src, bytes);
      qb += kItemK / BS;
    } else {
      const int koff = pos.kc * kItemK + 64 * t;  // the lane's K segment
      const bool seg = koff < grp.K;
      const bool v0 = seg && ok0, v1 = seg && ok1;
      const int64_t b0 = blk0 + koff / BS;
      const int64_t b1 = b0 + static_cast<int64_t>(8) * grp.kb;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (!(r ? v1 : v0)) continue;
        const int64_t b = r ? b1 : b0;
        if constexpr (DQ) {
          // the aligned 4-byte word holding u_b (and u_{b+1} at blocksize 32:
          // b is even), cut at the end of the array in the last row group
          const int64_t wb = b & ~int64_t(3);
          if (last) {
            const int64_t rest = nb - wb;
            cp_async4_part(smem_u32(sc + r * 32 + lane), aq + wb,
                           static_cast<uint32_t>(rest < 4 ? rest : 4));
          } else {
            cp_async4(smem_u32(sc + r * 32 + lane), aq + wb);
          }
          cp_async4(smem_u32(sc + (2 + r) * 32 + lane), s2 + (b >> 8));
        } else {
          const float* am = grp.p[pos.p].absmax;
          cp_async4(smem_u32(sc + r * 32 + lane), am + b);
          if constexpr (BS == 32) cp_async4(smem_u32(sc + (2 + r) * 32 + lane), am + b + 1);
        }
      }
    }
    if (pos.step(grp)) enter();
  }
};

// Decoded scale of a block from its staged words (u at byte `sh` of the u
// word); 0 for an invalid row / segment (its products are then 0 or
// discarded).
template <bool DQ>
__device__ __forceinline__ float scale_of(uint32_t w_u, uint32_t w_s, int sh, float off,
                                          bool valid) {
  if (!valid) return 0.0f;
  if constexpr (DQ) {
    const uint32_t u = prmt(w_u, 0u, 0x4440u | static_cast<uint32_t>(sh));
    return __fmaf_rn(static_cast<float>(static_cast<int>(u) - 128), __uint_as_float(w_s), off);
  } else {
    return __uint_as_float(w_u);
  }
}

// QUAD: double quant, blocksize >= 64 and K % 256 == 0 -- the blocks of one
// row of an item lie in one aligned 4-byte word of absmax_q and one scale2
// group, so the 4 lanes of a quad copy their two rows' words together (lane
// t: t = 0 the u word of row g, 1 of row g + 8, 2 / 3 their scale2), and no
// K segment is past K.
template <int BS, int QT, bool DQ, int F, int MAXP, bool QUAD>
__global__ void __launch_bounds__(kThreads, 1)
    gemv4_kernel(const __grid_constant__ Group<MAXP> grp) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // 1024-byte aligned base (the swizzled tiles), by pointer arithmetic on the
  // shared array so every access stays a shared-memory access
  const uint32_t raw = smem_u32(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int C = grp.C;
  const int rb = static_cast<int>(static_cast<int64_t>(grp.n_rg) * blockIdx.x / gridDim.x);
  const int re = static_cast<int>(static_cast<int64_t>(grp.n_rg) * (blockIdx.x + 1) / gridDim.x);
  const int64_t items = static_cast<int64_t>(re - rb) * C;
  // warp w's run of the CTA's items is [run(w), run(w + 1))
  auto run = [&](int w) { return static_cast<int>(items * w / kWarps); };
  const int i0 = run(warp), i1 = run(warp + 1);
  const int cnt = i1 - i0;
  int p_begin = 0;
  while (p_begin + 1 < grp.count && rb >= grp.p[p_begin + 1].rg0) ++p_begin;
  // programmatic dependent launch (inside a captured graph after a kernel):
  // no global access before the previous kernel has completed
  pdl_trigger();
  pdl_wait();

  if (cnt > 0) {
    uint64_t* full = sm.full[warp];
    if (lane == 0) {
      for (int d = 0; d < kStages; ++d) mbar_init(smem_u32(&full[d]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();

    Pos<MAXP> cp;  // the item the math is on
    cp.seek(grp, rb + i0 / C, i0 % C, p_begin);
    // Only the first item's copies start now: with every warp's whole ring
    // requested at once the first tiles would arrive last among them, and
    // the math waits for a tile while the rest of the ring is no use yet.
    // The other stages fill once the first tile is in (kStages - 1 empty
    // copy groups after the first keep the count of groups committed after
    // each item's at kStages - 1 when it is consumed).
    Fetch<BS, DQ, MAXP, QUAD> f(grp, lane, cp, cnt);
    f.issue(sm.tiles[warp][0], &sm.sc[warp][0][0][0], smem_u32(&full[0]));
#pragma unroll
    for (int d = 0; d < kStages; ++d) cp_async_commit();
    wait_tile(smem_u32(&full[0]), 0u, grp.err);
#pragma unroll
    for (int e = 1; e < kStages; ++e) {
      f.issue(sm.tiles[warp][e], &sm.sc[warp][e][0][0], smem_u32(&full[e]));
      cp_async_commit();
    }

    const uint32_t k16 = grp.k16, k31 = grp.k31;
    // the row group being summed: its problem, row group within the problem,
    // this lane's rows, decoded-scale offset, x row and block-index low bits
    int cur_p = 0, rl = 0;
    bool cok0 = false, cok1 = false;
    float off = 0.0f;
    const uint16_t* xrow = nullptr;
    uint32_t blk_lo = 0;
    auto enter = [&]() {
      const Prob& a = grp.p[cp.p];
      cur_p = cp.p;
      rl = cp.rg - a.rg0;
      const int n0 = rl * kRows + g;
      cok0 = n0 < a.N;
      cok1 = n0 + 8 < a.N;
      off = DQ ? __ldg(a.offset) : 0.0f;
      xrow = a.x + static_cast<int64_t>(g) * grp.K;  // read by lanes g < B only
      blk_lo = static_cast<uint32_t>(n0) * static_cast<uint32_t>(grp.kb);
    };
    enter();
    float acc[2][4] = {};
    bool first = true;  // the row group is the run's first
    uint4 xb[8];        // lanes of batch columns past B keep these zeros
#pragma unroll
    for (int q = 0; q < 8; ++q) xb[q] = make_uint4(0, 0, 0, 0);

    for (int j = 0; j < cnt; ++j) {
      const int d = j & (kStages - 1);
      const int koff = cp.kc * kItemK + 64 * t;  // the lane's K segment
      const bool seg = QUAD || koff < grp.K;
      // x of the segment (batch column g; a segment past K reads zeros)
      if (g < grp.B) {
        const uint4* xs = reinterpret_cast<const uint4*>(xrow + (seg ? koff : 0));
#pragma unroll
        for (int q = 0; q < 8; ++q) xb[q] = seg ? __ldg(xs + q) : make_uint4(0, 0, 0, 0);
      }
      wait_tile(smem_u32(&full[d]), static_cast<uint32_t>(j / kStages) & 1u, grp.err);
      cp_async_wait<kStages - 1>();  // this lane's scale copies of item j have landed
      // rows g and g + 8, 16-byte chunks 2t and 2t + 1 (swizzled by row & 7 = g)
      const uint8_t* tile = sm.tiles[warp][d];
      uint4 c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c[q] = *reinterpret_cast<const uint4*>(tile + (g + 8 * (q >> 1)) * 128 +
                                               (((2 * t + (q & 1)) ^ g) << 4));
      uint32_t sw[4];
      if constexpr (QUAD) {
        __syncwarp();  // the quad-mates' scale copies (each waited above) are visible
        const uint4 v = *reinterpret_cast<const uint4*>(&sm.sc[warp][d][0][lane & ~3]);
        sw[0] = v.x;
        sw[1] = v.y;
        sw[2] = v.z;
        sw[3] = v.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) sw[q] = sm.sc[warp][d][q][lane];
      }
      // byte of u in each staged word: the block index mod 4
      const uint32_t bl = blk_lo + static_cast<uint32_t>(koff / BS);
      const int sh0 = static_cast<int>(bl & 3u);
      const int sh1 = static_cast<int>((bl + 8u * static_cast<uint32_t>(grp.kb)) & 3u);
      const float a00 = scale_of<DQ>(sw[0], sw[2], sh0, off, seg && cok0);
      const float a10 = scale_of<DQ>(sw[1], sw[3], sh1, off, seg && cok1);
      float a01 = 0.f, a11 = 0.f;
      if constexpr (BS == 32) {  // the segment's second block (b + 1: the next byte)
        a01 = DQ ? scale_of<DQ>(sw[0], sw[2], sh0 + 1, off, seg && cok0)
                 : (seg && cok0 ? __uint_as_float(sw[2]) : 0.f);
        a11 = DQ ? scale_of<DQ>(sw[1], sw[3], sh1 + 1, off, seg && cok1)
                 : (seg && cok1 ? __uint_as_float(sw[3]) : 0.f);
      }

      // refill this stage with the item kStages ahead once every lane's reads
      // of it are done (the values above are in registers); the fence orders
      // those shared-memory reads before the TMA's writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      f.issue(sm.tiles[warp][d], &sm.sc[warp][d][0][0], smem_u32(&full[d]));
      cp_async_commit();

#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // one table per (row, quant block): blocksize 32 switches at h = 1
        Lut l0, l1;
        if (BS == 32 && h == 1) {
          l0 = make_lut<QT, F>(a01);
          l1 = make_lut<QT, F>(a11);
        } else {
          l0 = make_lut<QT, F>(a00);
          l1 = make_lut<QT, F>(a10);
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          const int p = 4 * h + wi;  // codes koff + 8p .. + 7 of both rows
          const uint4 o0 = dq8_fma(l0, word(c[h], wi), k16, k31);
          const uint4 o1 = dq8_fma(l1, word(c[2 + h], wi), k16, k31);
          mma16<F>(acc[0], o0.x, o1.x, o0.y, o1.y, xb[p].x, xb[p].y);
          mma16<F>(acc[1], o0.z, o1.z, o0.w, o1.w, xb[p].z, xb[p].w);
        }
      }

      // the end of a row group: store it, or leave it in shared memory when
      // a neighbouring run holds part of it (the run's first row group when
      // the run starts inside it, its last when the run ends inside it)
      const bool more = j + 1 < cnt;
      if (cp.step(grp) || !more) {
        const float4 v = make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1],
                                     acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
        const bool shared = (first && i0 % C != 0) || (!more && i1 % C != 0);
        if (shared)
          sm.part[first ? 0 : 1][warp][lane] = v;
        else
          store_rows<F>(v, rl, lane, grp.p[cur_p], grp.B);
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][e] = 0.f;
        first = false;
        if (more) enter();
      }
    }
    cp_async_wait<0>();
  }

  // A shared row group is added up by the warp whose run holds its last
  // item (then the row group is that run's first): the partial sums of the
  // runs that hold part of it, in warp order.
  __syncthreads();
  if (cnt > 0 && i0 % C != 0 && i1 >= (i0 / C + 1) * C) {
    const int lrg = i0 / C;  // the row group, CTA-local
    const int first_item = lrg * C;
    // the run holding its first item: the largest w with run(w) <= first_item
    const int w_lo =
        static_cast<int>((static_cast<int64_t>(first_item + 1) * kWarps - 1) / items);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    int a0 = run(w_lo);
    for (int w = w_lo; w <= warp; ++w) {
      const int a1 = run(w + 1);
      if (a1 != a0) {  // (an empty run deposited nothing)
        // a run that starts inside the row group deposited it as its first
        const float4 q = sm.part[a0 >= first_item ? 0 : 1][w][lane];
        s.x += q.x;
        s.y += q.y;
        s.z += q.z;
        s.w += q.w;
      }
      a0 = a1;
    }
    Pos<MAXP> rp;
    rp.seek(grp, rb + lrg, 0, p_begin);
    const Prob& a = grp.p[rp.p];
    store_rows<F>(s, rb + lrg - a.rg0, lane, a, grp.B);
  }
}

template <int BS, int QT, bool DQ, int F, int MAXP, bool QUAD>
cudaError_t launch_k(const Group<MAXP>& grp, int num_sms, cudaStream_t s) {
  auto kern = gemv4_kernel<BS, QT, DQ, F, MAXP, QUAD>;
  // per device; a race only repeats the (idempotent) attribute call
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_relaxed)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  const int64_t grid = grp.n_rg < num_sms ? grp.n_rg : num_sms;
  return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmemBytes, s,
                       programmatic_after_kernel(s), grp);
}

template <int BS, int QT, bool DQ, int F, int MAXP>
cudaError_t launch_t(const Group<MAXP>& grp, int num_sms, cudaStream_t s) {
  if constexpr (DQ && BS >= 64) {
    if (grp.K % kItemK == 0) return launch_k<BS, QT, DQ, F, MAXP, true>(grp, num_sms, s);
  }
  return launch_k<BS, QT, DQ, F, MAXP, false>(grp, num_sms, s);
}

// Fills the problem list from the linear layers' arguments (already checked
// by the caller) and launches the kernel of their common format.
template <int MAXP>
cudaError_t launch_group(const GemvLinear* lin, int count, int64_t B, int fmt, int num_sms,
                         int* err, cudaStream_t s) {
  Group<MAXP> grp{};
  grp.count = count;
  grp.B = static_cast<int>(B);
  grp.err = err;
  int64_t rg = 0;
  for (int i = 0; i < count; ++i) {
    const GemvLinear& l = lin[i];
    if (!make_map_2d(&grp.maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, l.W->codes,
                     static_cast<uint64_t>(l.K / 2), static_cast<uint64_t>(l.N),
                     static_cast<uint64_t>(l.K / 2), kItemK / 2, kRows,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    Prob& p = grp.p[i];
    p.x = static_cast<const uint16_t*>(l.x);
    p.absmax = l.W->absmax;
    p.absmax_q = l.W->absmax_q;
    p.scale2 = l.W->scale2;
    p.offset = l.W->offset;
    p.bias = static_cast<const uint16_t*>(l.bias);
    p.y = static_cast<uint16_t*>(l.y);
    p.nb = l.N * l.K / l.W->blocksize;
    p.N = static_cast<int>(l.N);
    p.rg0 = static_cast<int>(rg);
    rg += (l.N + kRows - 1) / kRows;
  }
  grp.K = static_cast<int>(lin[0].K);
  grp.C = static_cast<int>((lin[0].K + kItemK - 1) / kItemK);
  grp.kb = static_cast<int>(lin[0].K / lin[0].W->blocksize);
  grp.n_rg = static_cast<int>(rg);
  grp.k16 = 1u << 16;
  grp.k31 = 1u << 31;
  const bnb4_qstate& W = *lin[0].W;
  const bool dq = W.double_quant != 0;
  const bool nf4 = W.qtype == kQtNF4;
  const bool f16 = fmt == BNB4_F16;
#define BNB4_GEMV_LAUNCH(BSV)                                                              \
  if (nf4)                                                                                 \
    return dq ? (f16 ? launch_t<BSV, kQtNF4, true, BNB4_F16>(grp, num_sms, s)              \
                     : launch_t<BSV, kQtNF4, true, BNB4_BF16>(grp, num_sms, s))            \
              : (f16 ? launch_t<BSV, kQtNF4, false, BNB4_F16>(grp, num_sms, s)             \
                     : launch_t<BSV, kQtNF4, false, BNB4_BF16>(grp, num_sms, s));          \
  return dq ? (f16 ? launch_t<BSV, kQtFP4, true, BNB4_F16>(grp, num_sms, s)                \
                   : launch_t<BSV, kQtFP4, true, BNB4_BF16>(grp, num_sms, s))              \
            : (f16 ? launch_t<BSV, kQtFP4, false, BNB4_F16>(grp, num_sms, s)               \
                   : launch_t<BSV, kQtFP4, false, BNB4_BF16>(grp, num_sms, s));
  switch (W.blocksize) {
    case 32: BNB4_GEMV_LAUNCH(32)
    case 64: BNB4_GEMV_LAUNCH(64)
    case 128: BNB4_GEMV_LAUNCH(128)
    default: BNB4_GEMV_LAUNCH(256)
  }
#undef BNB4_GEMV_LAUNCH
}

}  // namespace

cudaError_t launch_gemv(const void* x, int64_t B, int64_t K, const bnb4_qstate& W,
                        int64_t N, void* y, const void* bias, int fmt, int num_sms, int* err,
                        cudaStream_t s) {
  // a single weight: the direct kernel is faster (gemv_direct.cu)
  (void)err;
  return launch_gemv_direct(x, B, K, W, N, y, bias, fmt, num_sms, s);
}

cudaError_t launch_gemv_group(const GemvLinear* lin, int count, int64_t B, int fmt,
                              int num_sms, int* err, cudaStream_t s, bool persistent) {
  // Measured on B200 (µs per weight, rotating weights larger than L2): this
  // kernel wins for single-row x over lists of 4 or more (11008 x 4096: 12.0
  // against 13.9 over 16); the one-CTA-per-16-rows kernel of gemv_direct.cu
  // wins for lists of 2 or 3 and at every size for B > 1 (16.9 against 22.8
  // for two 11008 x 4096 weights at B = 8).
  for (int i = 0; i < count; i += kLargeGroup) {
    const int c = count - i < kLargeGroup ? count - i : kLargeGroup;
    cudaError_t e;
    if (!persistent && (B > 1 || c < 4))
      e = launch_gemv_direct_list(lin + i, c, B, fmt, num_sms, s);
    else if (c <= kSmallGroup)
      e = launch_group<kSmallGroup>(lin + i, c, B, fmt, num_sms, err, s);
    else
      e = launch_group<kLargeGroup>(lin + i, c, B, fmt, num_sms, err, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bnb4
