// common.cuh -- device-side constants and helpers shared by the kernels of the
// 4-bit blockwise quantization library (sm_100a).
//
// The codebooks follow the CSDN article on bitsandbytes, section "数学原理对比"
// (NF4: 16 normal-quantile values normalised to [-1, 1] with an exact 0) and
// its closing remarks (FP4: an E2M1-like format; here E2M1 magnitudes / 6 with
// a sign bit).  The NF4 values are the QLoRA quantile construction:
// positives = inverse normal CDF at 8 evenly spaced probabilities in
// (1/2, 1 - delta], negatives = the same at 7 points, mirrored, plus 0,
// all divided by the largest; delta = (1/32 + 1/30) / 2.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bnb4.h"

namespace bnb4 {

constexpr int kQtNF4 = BNB4_NF4;
constexpr int kQtFP4 = BNB4_FP4;

// NF4 codebook, ascending; index 7 is the exact zero.
__device__ __forceinline__ float nf4_value(int i) {
  constexpr float t[16] = {
      -0x1p+0f,        -0x1.647362p-1f, -0x1.0cd65cp-1f, -0x1.94653cp-2f,
      -0x1.234496p-2f, -0x1.7a6a7ap-3f, -0x1.74f0d2p-4f, 0x0p+0f,
      0x1.45f602p-4f,  0x1.4995bep-3f,  0x1.f809b4p-3f,  0x1.5a066cp-2f,
      0x1.c3496ap-2f,  0x1.200f52p-1f,  0x1.722760p-1f,  0x1p+0f};
  return t[i];
}

// FP4 magnitudes: E2M1 values {0, .5, 1, 1.5, 2, 3, 4, 6} divided by 6.
__device__ __forceinline__ float fp4_magnitude(int m) {
  constexpr float t[8] = {0x0p+0f,        0x1.555556p-4f, 0x1.555556p-3f,
                          0x1p-2f,        0x1.555556p-2f, 0x1p-1f,
                          0x1.555556p-1f, 0x1p+0f};
  return t[m];
}

// Dequantization value of 4-bit code c (FP4: bit 3 is the sign).
__device__ __forceinline__ float code_value(int qtype, int c) {
  if (qtype == kQtNF4) return nf4_value(c);
  const float m = fp4_magnitude(c & 7);
  return (c & 8) ? -m : m;
}

// Decoded absmax of block b: fma(u - 128, s, offset) rounded once with double
// quantization, the exact absmax without.
template <bool DQ>
__device__ __forceinline__ float decoded_absmax(int64_t b, const float* absmax,
                                                const uint8_t* absmax_q,
                                                const float* scale2,
                                                float offset) {
  if constexpr (DQ) {
    const int u = __ldg(absmax_q + b);
    return __fmaf_rn(static_cast<float>(u - 128), __ldg(scale2 + (b >> 8)),
                     offset);
  } else {
    return __ldg(absmax + b);
  }
}

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 256-bit loads (sm_100): the address must be 32-byte aligned.
struct U8x32 {
  uint32_t v[8];
};
__device__ __forceinline__ U8x32 ldg_v8(const void* p) {
  U8x32 r;
  asm volatile("ld.global.nc.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]), "=r"(r.v[4]),
                 "=r"(r.v[5]), "=r"(r.v[6]), "=r"(r.v[7])
               : "l"(p));
  return r;
}
__device__ __forceinline__ U8x32 ldg_stream_v8(const void* p) {
  U8x32 r;
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]), "=r"(r.v[4]),
                 "=r"(r.v[5]), "=r"(r.v[6]), "=r"(r.v[7])
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) {
  return __uint_as_float(w << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
  return __uint_as_float(w & 0xffff0000u);
}

// Two fp32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 -> packed fp16x2 (lo in bits 0..15), IEEE round to nearest even
// (infinity past the largest finite value, subnormals kept).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The 16-bit compute formats (F = BNB4_BF16 or BNB4_F16): a packed pair from
// two fp32 values, and the exact fp32 value of a 16-bit pattern.
template <int F>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (F == BNB4_F16)
    return pack_f16x2(lo, hi);
  else
    return pack_bf16x2(lo, hi);
}
template <int F>
__device__ __forceinline__ float half_to_f32(uint32_t bits16) {
  if constexpr (F == BNB4_F16) {
    float f;
    asm("{\n\t.reg .b16 h, u;\n\tmov.b32 {h, u}, %1;\n\tcvt.f32.f16 %0, h;\n\t}"
        : "=f"(f)
        : "r"(bits16));
    return f;
  } else {
    return __uint_as_float(bits16 << 16);
  }
}

// A row-major [rows, cols] view whose rows start ld elements apart (ld >=
// cols): flat element e = q * cols + c of the logical tensor lives at offset
// q * ld + c.  q = floor(e / cols) is the high half of e * magic with magic =
// ceil(2^64 / cols), exact for e < 2^32 and 2 <= cols < 2^32 (the error of
// e * magic / 2^64 is below 2^-32 < 1 / cols).
struct View2D {
  int64_t cols, ld;
  uint64_t magic;
};

__device__ __forceinline__ int64_t view_offset(int64_t e, const View2D& v) {
  const uint64_t q = __umul64hi(static_cast<uint64_t>(e), v.magic);
  return e + static_cast<int64_t>(q) * (v.ld - v.cols);
}

inline View2D make_view(int64_t cols, int64_t ld) {
  return View2D{cols, ld, ~0ull / static_cast<uint64_t>(cols) + 1ull};
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may be scheduled while the kernel before it on the stream
// finishes; it waits for that kernel with pdl_wait before touching global
// memory.  Such a launch is made only where the predecessor is known to be a
// kernel: the double-quant kernel after the quantize kernel of the same call,
// and, while a stream is being captured into a CUDA graph, a library kernel
// whose one dependency node is a kernel node (programmatic_after_kernel).
// Eager launches of a call's first kernel are plain: the caller's previous
// work on the stream may be a copy, which a programmatic launch would not
// wait for (observed on B200: a pageable host-to-device copy followed by
// programmatic launches gave intermittent mismatches).  Both device calls are
// no-ops without such a launch.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// True while `s` is being captured and its single dependency is a kernel
// node: a launch there may be programmatic (a kernel-to-kernel edge).
inline bool programmatic_after_kernel(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  const cudaGraphNode_t* deps = nullptr;
  size_t n = 0;
  if (cudaStreamGetCaptureInfo(s, &st, nullptr, nullptr, &deps, &n) != cudaSuccess) {
    cudaGetLastError();  // not fatal: launch plainly
    return false;
  }
  if (st != cudaStreamCaptureStatusActive || n != 1 || deps == nullptr) return false;
  cudaGraphNodeType t;
  if (cudaGraphNodeGetType(deps[0], &t) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return t == cudaGraphNodeTypeKernel;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, bool programmatic, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace bnb4
