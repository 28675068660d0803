// l2warm.cuh -- L2 warm-up of bytes a kernel will read soon (sm_100a).
//
// A prefetch only places lines in L2, which every SM reads and writes
// coherently: a later write to the same bytes by another kernel still reaches
// the loads that follow it.  So a kernel may warm its read-only operands
// before waiting on the kernel it depends on (pdl_wait), and a CTA may warm
// the operands of a CTA that will start after it.  The kernels do so only in
// a programmatic launch, where the prefetches overlap the previous kernel; in
// a plain launch they would compete with the kernel's own first loads.
//
// Only for plain device memory: the linear entry points accept nothing else
// for the weight state, and the quantize entry points warm their input only
// when it is device memory (not page-locked host memory read over the bus).
#pragma once

#include <stdint.h>

namespace bnb4 {
namespace {

// Bulk form: 16-byte aligned address, size a multiple of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// One cache line around p; no alignment rule.
__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

constexpr int64_t kPrefetchChunk = 16384;  // bytes per bulk prefetch

// [p, p + bytes) in bulk prefetches of at most kPrefetchChunk bytes (p
// 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2_range(const uint8_t* p, int64_t bytes) {
  for (int64_t o = 0; o < bytes; o += kPrefetchChunk)
    prefetch_l2_bulk(p + o, static_cast<uint32_t>(bytes - o < kPrefetchChunk ? bytes - o
                                                                              : kPrefetchChunk));
}

}  // namespace
}  // namespace bnb4
