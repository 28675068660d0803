// gemv.cu -- decode GEMV with 4-bit weights on sm_100a:
//   y[b, n] = h( sum_k x[b, k] * What[n, k] + bias[n] ),  1 <= B <= 8,
//   What[n, k] = h(RN(t[code] * a_hat))   (dequantized weight, exact),
// h = round to the 16-bit compute format, bf16 or fp16 (nearest even); the
// bias is optional.
//
// Method: bitsandbytes' gemv_4bit op (ossradar page, release notes 0.50.0)
// over the blockwise NF4 / FP4 format of the CSDN article (section
// "数学原理对比"), nested (double) quantization decoded in-kernel.
//
// Design (bound by the packed-byte stream from HBM and by instruction issue):
//  * Persistent grid, one CTA per SM; each CTA owns a contiguous, balanced
//    range of 16-row groups.  A work item is 16 rows x 256 K (2 KB of codes):
//    lane (g, t) of a warp owns rows g and g + 8 and the 64-element K segment
//    t of the item.
//  * Every consumer warp streams its items through a private ring of
//    shared-memory stages filled by cp.async, several items ahead.  Each lane
//    copies exactly the 2 x 32 code bytes and the scale words it later reads,
//    so completion is tracked per thread (cp.async.wait_group) and no lane
//    waits on another; the HBM latency is hidden without holding loads in
//    registers.
//  * Split-K mode (K of at least one item per consumer warp): the CTA's items
//    are its (row group, K chunk) pairs in row-major order, dealt to the
//    warps round-robin; a warp sums its chunks of a row group in registers
//    and hands the partial sums to a reducer warp through a double-buffered
//    shared-memory slot (named barriers FULL / EMPTY).  The reducer adds them
//    in warp order -- a fixed order, so results are bit-reproducible --,
//    adds the bias and stores y.  Short K: each warp takes whole row groups
//    and stores y itself.
//  * Dequantization by byte permutes (lut.cuh): per (row, quant block) a lane
//    builds the 16-entry table of h(RN(t[i] * a_hat)), bit-identical to
//    dequantizing every element.  Products on mma.sync m16n8k16 (weights as
//    the A operand, 16 rows; x as B, batch columns): one 128-bit load of x
//    feeds two MMAs, and K is permuted identically in both operands, which
//    leaves the dot products unchanged.  Batch columns beyond B read a valid
//    row whose outputs are never stored.
#include "common.cuh"
#include "kernels.h"
#include "lut.cuh"
#include "sm100.cuh"

namespace bnb4 {
namespace {

constexpr int kConsumers = 16;                    // warps per CTA
constexpr int kThreads = kConsumers * 32;
constexpr int kStages = 4;                        // ring depth per warp
constexpr int kRows = 16;                         // rows of an item (MMA M)
constexpr int kItemK = 256;                       // K of an item (4 lanes x 64)

constexpr int kTileBytes = kRows * kItemK / 2;    // packed codes of one item: 2 KB

// Per consumer warp, a ring of kStages items: the code tile (16 rows x 128
// bytes, written by TMA with the 128-byte swizzle: 16-byte chunk c of row r
// sits at chunk c ^ (r & 7)), the lane-major scale words (each lane copies
// the words it reads), and the tile's "full" mbarrier.
struct Smem {
  uint8_t tiles[kConsumers][kStages][kTileBytes];
  uint32_t sc[kConsumers][kStages][4][32];  // dq: [u word g, u word g+8, scale2 g, scale2 g+8]
                                            // else [absmax g, absmax g+8, next g, next g+8]
  // per item and lane, written by the fetching lane and read back by the
  // same lane when it computes the item: {row group, problem, K offset of
  // the lane's segment, flags: row g ok, row g + 8 ok, byte of u in each
  // scale word}
  int4 rec[kConsumers][kStages][32];
  float4 red[2][kConsumers][32];            // partial sums of two row groups in flight
  uint64_t full[kConsumers][kStages];
  int arrived[2];  // warps that deposited their partials in slot s
  int reduced[2];  // the CTA-local row group last reduced out of slot s
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
constexpr int kSmallGroup = 4;   // one GEMV, or q/k/v, gate/up
constexpr int kLargeGroup = 32;  // a longer list is launched in parts of 32
static_assert(sizeof(Group<kLargeGroup>) <= 32000, "kernel parameter space");

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
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
// Bounded wait until a shared-memory word equals `want` (set by another warp
// of the CTA); on expiry the device error word is set and the caller goes
// on, so nothing hangs.
__device__ __forceinline__ void wait_word(const int* word, int want, int* err) {
  if (*reinterpret_cast<const volatile int*>(word) == want) return;
  const uint64_t t0 = global_ns();
  while (*reinterpret_cast<const volatile int*>(word) != want) {
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicExch(err, 1);
      return;
    }
    __nanosleep(32);
  }
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

// The item sequence of one consumer warp and the copies of each item.  All
// state is 32-bit except the block index; advancing costs a few integer
// operations, a new row group a few more, a new problem a handful of
// parameter loads.
template <int BS, bool DQ, int MAXP>
struct Fetcher {
  const Group<MAXP>& grp;
  int lane, g, t;
  bool split;
  int nw;
  int rg, rg_end, kc, p, rl, next_rg0;  // item (global row group, chunk), problem
  int64_t blk0;                         // block of row g at k = 0
  bool ok0, ok1, last;                  // rows g, g + 8 exist; last row group
  // double quant with blocksize >= 64 and K % 256 == 0: the blocks of one
  // row of an item lie in one aligned 4-byte word of absmax_q and one scale2
  // group, so the 4 lanes of a quad copy their two rows' words together
  // (lane t: t = 0 the u word of row g, 1 of row g + 8, 2 / 3 their scale2)
  bool quad_sc;

  __device__ Fetcher(const Group<MAXP>& gp, int lane_, bool split_, int nw_, int warp,
                     int rg_begin, int rg_end_, int p_begin)
      : grp(gp), lane(lane_), g(lane_ >> 2), t(lane_ & 3), split(split_), nw(nw_),
        rg_end(rg_end_) {
    quad_sc = DQ && BS >= 64 && grp.K % kItemK == 0;
    rg = split ? rg_begin : rg_begin + warp;
    kc = split ? warp : 0;
    p = p_begin;
    set_problem();
    set_row_group();
  }
  __device__ void set_problem() {
    while (p + 1 < grp.count && rg >= grp.p[p + 1].rg0) ++p;
    next_rg0 = p + 1 < grp.count ? grp.p[p + 1].rg0 : grp.n_rg;
  }
  __device__ void set_row_group() {
    rl = rg - grp.p[p].rg0;
    const int n0 = rl * kRows + g;
    const int N = grp.p[p].N;
    blk0 = static_cast<int64_t>(n0) * grp.kb;
    ok0 = n0 < N;
    ok1 = n0 + 8 < N;
    last = (rl + 1) * kRows >= N;
  }
  __device__ bool valid() const { return rg < rg_end; }
  __device__ void advance() {
    if (split) {
      kc += nw;
      if (kc < grp.C) return;
      kc -= grp.C;
      ++rg;
    } else {
      if (++kc < grp.C) return;
      kc = 0;
      rg += nw;
    }
    if (rg >= rg_end) return;
    if (rg >= next_rg0) set_problem();
    set_row_group();
  }

  // lane 0 arms the stage's barrier and starts the TMA of the code tile;
  // every lane copies the words holding its two rows' block scales and
  // writes the item's record.  Rows past N and segments past K copy no
  // scales (the TMA fills their codes with zeros).
  __device__ void issue(uint8_t* tile, uint32_t* sc, int4* rec, uint32_t full) const {
    if (lane == 0) {
      mbar_arrive_expect_tx(full, kTileBytes);
      tma_load_2d(smem_u32(tile), &grp.maps[p], kc * (kItemK / 2), rl * kRows, full);
    }
    const int koff = kc * kItemK + 64 * t;  // the lane's K segment
    const bool seg = koff < grp.K;
    const bool v0 = seg && ok0, v1 = seg && ok1;
    const int64_t b0 = blk0 + koff / BS;
    const int64_t b1 = b0 + static_cast<int64_t>(8) * grp.kb;
    const Prob& a = grp.p[p];
    if (quad_sc) {
      const int r = t & 1;  // the row this lane copies a word of
      if (r ? v1 : v0) {
        const int64_t b = r ? b1 : b0;
        if (t < 2) {
          const int64_t wb = b & ~int64_t(3);
          if (last) {
            const int64_t left = a.nb - wb;
            cp_async4_part(smem_u32(sc + lane), a.absmax_q + wb,
                           static_cast<uint32_t>(left < 4 ? left : 4));
          } else {
            cp_async4(smem_u32(sc + lane), a.absmax_q + wb);
          }
        } else {
          cp_async4(smem_u32(sc + lane), a.scale2 + (b >> 8));
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (quad_sc || !(r ? v1 : v0)) continue;
      const int64_t b = r ? b1 : b0;
      if constexpr (DQ) {
        // the aligned 4-byte word holding u_b (and u_{b+1} at blocksize 32:
        // b is even), cut at the end of the array in the last row group
        const int64_t wb = b & ~int64_t(3);
        if (last) {
          const int64_t left = a.nb - wb;
          cp_async4_part(smem_u32(sc + r * 32 + lane), a.absmax_q + wb,
                         static_cast<uint32_t>(left < 4 ? left : 4));
        } else {
          cp_async4(smem_u32(sc + r * 32 + lane), a.absmax_q + wb);
        }
        cp_async4(smem_u32(sc + (2 + r) * 32 + lane), a.scale2 + (b >> 8));
      } else {
        cp_async4(smem_u32(sc + r * 32 + lane), a.absmax + b);
        if constexpr (BS == 32) cp_async4(smem_u32(sc + (2 + r) * 32 + lane), a.absmax + b + 1);
      }
    }
    const int flags = (v0 ? 1 : 0) | (v1 ? 2 : 0) | (static_cast<int>(b0 & 3) << 4) |
                      (static_cast<int>(b1 & 3) << 8);
    *rec = make_int4(rg, p, koff, flags);
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

template <int BS, int QT, bool DQ, int F, int MAXP>
__global__ void __launch_bounds__(kThreads, 1)
    gemv4_kernel(const __grid_constant__ Group<MAXP> grp) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // 1024-byte aligned base (the swizzled tiles), by pointer arithmetic on the
  // shared array so every access stays a shared-memory access
  const uint32_t raw = smem_u32(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rg_begin = static_cast<int>(static_cast<int64_t>(grp.n_rg) * blockIdx.x / gridDim.x);
  const int rg_end = static_cast<int>(static_cast<int64_t>(grp.n_rg) * (blockIdx.x + 1) / gridDim.x);
  const int R = rg_end - rg_begin;
  int p_begin = 0;
  while (p_begin + 1 < grp.count && rg_begin >= grp.p[p_begin + 1].rg0) ++p_begin;
  // Split K over nw consumer warps when the CTA has fewer row groups than
  // warps; else whole row groups per warp (no hand-over at all).  nw <= C in
  // split mode, so a warp's consecutive items are at most one row group
  // apart and every warp contributes to every row group.
  const bool split_k = R < kConsumers;
  const int nw = split_k ? (grp.C < kConsumers ? grp.C : kConsumers) : kConsumers;
  if (threadIdx.x == 0) {
    sm.arrived[0] = sm.arrived[1] = 0;
    sm.reduced[0] = -2;  // slot s first holds row group s
    sm.reduced[1] = -1;
  }
  __syncthreads();
  if (warp >= nw) return;

  const int g = lane >> 2, t = lane & 3;
  uint64_t* full = sm.full[warp];
  if (lane == 0) {
    for (int d = 0; d < kStages; ++d) mbar_init(smem_u32(&full[d]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();

  Fetcher<BS, DQ, MAXP> f(grp, lane, split_k, nw, warp, rg_begin, rg_end, p_begin);
#pragma unroll
  for (int d = 0; d < kStages; ++d) {
    if (f.valid()) {
      f.issue(sm.tiles[warp][d], &sm.sc[warp][d][0][0], &sm.rec[warp][d][lane],
              smem_u32(&full[d]));
      f.advance();
    } else {
      sm.rec[warp][d][lane] = make_int4(rg_end, 0, 0, 0);  // end marker
    }
    cp_async_commit();
  }

  float acc[2][4] = {};
  int cur_rg = -1, cur_p = -1;
  float off = 0.0f;
  const uint16_t* xrow = nullptr;
  const uint32_t k16 = grp.k16, k31 = grp.k31;
  const bool quad_sc = f.quad_sc;
  // split K with one chunk per warp per row group: the warp's chunk, hence
  // its slice of x, never changes -- it is loaded once per problem
  const bool x_fixed = split_k && grp.C == nw;
  uint4 xb[8];

  // Split K: the partial sums of CTA-local row group r go to slot r & 1; the
  // warp that deposits last adds the nw partials in warp order (a fixed
  // order: bit-reproducible), stores y, empties the slot and marks row group
  // r reduced, which frees the slot for row group r + 2.
  auto flush = [&]() {
    const float4 v = make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1],
                                 acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
    if (split_k) {
      const int r = cur_rg - rg_begin;
      const int s = r & 1;
      if (r >= 2) {  // the slot's previous row group has been reduced
        if (lane == 0) wait_word(&sm.reduced[s], r - 2, grp.err);
        __syncwarp();
        __threadfence_block();
      }
      sm.red[s][warp][lane] = v;
      __threadfence_block();
      __syncwarp();
      int before = 0;
      if (lane == 0) before = atomicAdd(&sm.arrived[s], 1);
      before = __shfl_sync(0xffffffffu, before, 0);
      if (before == nw - 1) {  // the last to deposit: reduce
        __threadfence_block();
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = 0; w < nw; ++w) {
          const float4 q = sm.red[s][w][lane];
          sum.x += q.x;
          sum.y += q.y;
          sum.z += q.z;
          sum.w += q.w;
        }
        store_rows<F>(sum, cur_rg - grp.p[cur_p].rg0, lane, grp.p[cur_p], grp.B);
        __threadfence_block();
        __syncwarp();
        if (lane == 0) {
          sm.arrived[s] = 0;
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&sm.reduced[s]) = r;
        }
      }
    } else {
      store_rows<F>(v, cur_rg - grp.p[cur_p].rg0, lane, grp.p[cur_p], grp.B);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[c][e] = 0.f;
  };

  // items in the order they were issued; the ring holds the next kStages
  for (int j = 0;; ++j) {
    const int d = j & (kStages - 1);
    const int4 rec = sm.rec[warp][d][lane];  // written by this lane
    if (rec.x >= rg_end) break;              // the end marker
    if (rec.x != cur_rg) {
      if (cur_rg >= 0) flush();
      if (rec.y != cur_p) {  // per-problem values
        const Prob& a = grp.p[rec.y];
        off = DQ ? __ldg(a.offset) : 0.0f;
        xrow = a.x + static_cast<int64_t>(g < grp.B ? g : grp.B - 1) * grp.K;
        cur_p = rec.y;
        if (x_fixed) {  // (a segment past a ragged K reads no x)
          const bool in_k = rec.z < grp.K;
          const uint4* xs = reinterpret_cast<const uint4*>(xrow + (in_k ? rec.z : 0));
#pragma unroll
          for (int p = 0; p < 8; ++p) xb[p] = in_k ? __ldg(xs + p) : make_uint4(0, 0, 0, 0);
        }
      }
      cur_rg = rec.x;
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
    if (quad_sc) {
      __syncwarp();  // the quad-mates' scale copies (each waited above) are visible
#pragma unroll
      for (int q = 0; q < 4; ++q) sw[q] = sm.sc[warp][d][0][(lane & ~3) | q];
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) sw[q] = sm.sc[warp][d][q][lane];
    }
    const int koff = rec.z;
    const bool ok0 = rec.w & 1, ok1 = rec.w & 2;
    const bool seg = koff < grp.K;
    const int sh0 = (rec.w >> 4) & 3, sh1 = (rec.w >> 8) & 3;
    const float a00 = scale_of<DQ>(sw[0], sw[2], sh0, off, ok0);
    const float a10 = scale_of<DQ>(sw[1], sw[3], sh1, off, ok1);
    float a01 = 0.f, a11 = 0.f;
    if constexpr (BS == 32) {  // the segment's second block (b + 1: the next byte)
      a01 = DQ ? scale_of<DQ>(sw[0], sw[2], sh0 + 1, off, ok0) : (ok0 ? __uint_as_float(sw[2]) : 0.f);
      a11 = DQ ? scale_of<DQ>(sw[1], sw[3], sh1 + 1, off, ok1) : (ok1 ? __uint_as_float(sw[3]) : 0.f);
    }

    // refill this stage with the item kStages ahead once every lane's reads
    // of it are done (the values above are in registers and used); the
    // fence orders those shared-memory reads before the TMA's writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (f.valid()) {
      f.issue(sm.tiles[warp][d], &sm.sc[warp][d][0][0], &sm.rec[warp][d][lane],
              smem_u32(&full[d]));
      f.advance();
    } else {
      sm.rec[warp][d][lane] = make_int4(rg_end, 0, 0, 0);  // end marker
    }
    cp_async_commit();

    if (!x_fixed) {
      const uint4* xs = reinterpret_cast<const uint4*>(xrow + (seg ? koff : 0));
#pragma unroll
      for (int p = 0; p < 8; ++p) xb[p] = seg ? __ldg(xs + p) : make_uint4(0, 0, 0, 0);
    }

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
  }
  cp_async_wait<0>();
  if (cur_rg >= 0) flush();
}

template <int BS, int QT, bool DQ, int F, int MAXP>
cudaError_t launch_t(const Group<MAXP>& grp, int num_sms, cudaStream_t s) {
  auto kern = gemv4_kernel<BS, QT, DQ, F, MAXP>;
  static bool attr_set[64] = {};  // per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t grid = grp.n_rg < num_sms ? grp.n_rg : num_sms;
  return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmemBytes, s,
                       false, grp);
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
  const GemvLinear one{x, &W, K, N, bias, y};
  return launch_group<kSmallGroup>(&one, 1, B, fmt, num_sms, err, s);
}

cudaError_t launch_gemv_group(const GemvLinear* lin, int count, int64_t B, int fmt,
                              int num_sms, int* err, cudaStream_t s) {
  if (count <= kSmallGroup) return launch_group<kSmallGroup>(lin, count, B, fmt, num_sms, err, s);
  for (int i = 0; i < count; i += kLargeGroup) {
    const int c = count - i < kLargeGroup ? count - i : kLargeGroup;
    const cudaError_t e = c <= kSmallGroup
                              ? launch_group<kSmallGroup>(lin + i, c, B, fmt, num_sms, err, s)
                              : launch_group<kLargeGroup>(lin + i, c, B, fmt, num_sms, err, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bnb4
