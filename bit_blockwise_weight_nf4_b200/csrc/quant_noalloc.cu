// quant_noalloc.cu -- bnb_quantize_4bit_noalloc: double-quantized 4-bit
// quantization that allocates nothing and needs no caller workspace.
//
// Some callers cannot hand the library a scratch buffer or allocate one for
// it: a plugin running inside a host framework that owns every device
// allocation, a loader working under a fixed device-memory budget, or a
// latency-critical path where cudaMalloc (which may synchronize the device or
// fail under memory pressure) is not acceptable.  This entry point keeps its
// scratch -- one fp64 partial sum per CTA for the mean of the block scales and
// the exact fp32 absmax of every block, which double quantization consumes
// and nobody reads afterwards -- in a fixed array in the library's own device
// memory instead.  The caller still passes the input and the outputs (codes,
// absmax_q, scale2, offset).
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "bnb4.h"
#include "kernels.h"

namespace {

// Scratch layout: kMaxPartials fp64 partial sums (32 KiB), then up to
// BNB4_NOALLOC_MAX_BLOCKS fp32 absmax values (4 MiB).  Every GPU that loads
// the library holds this array until the process exits.
constexpr size_t kPartialsBytes = (bnb4::kDqWorkspaceBytes + 255) / 256 * 256;
constexpr size_t kScratchBytes =
    kPartialsBytes + sizeof(float) * static_cast<size_t>(BNB4_NOALLOC_MAX_BLOCKS);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Device address of the scratch array on the current device.  In host code
// `g_noalloc_scratch` names a host-side stand-in, not device memory, so the
// address is looked up once per device (with that device current) and cached.
// The lookup also loads the module holding the array on that device (lazy
// module loading), which maps its memory: that first call can therefore fail
// with BNB4_ERR_CUDA when the device is out of memory.  Two host threads may
// make their first call at once; both store the same address (atomic slot).
int scratch_address(unsigned char** out) {
  static std::atomic<unsigned char*> cache[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return BNB4_ERR_CUDA;
  unsigned char* a = cache[dev].load(std::memory_order_relaxed);
  if (a == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return BNB4_ERR_CUDA;
    }
    a = static_cast<unsigned char*>(p);
    cache[dev].store(a, std::memory_order_relaxed);
  }
  *out = a;
  return BNB4_OK;
}

int sm_count(int* out) {
  static std::atomic<int> cache[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return BNB4_ERR_CUDA;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        v <= 0)
      return BNB4_ERR_CUDA;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  *out = v;
  return BNB4_OK;
}

}  // namespace

extern "C" BNB4_API int bnb_quantize_4bit_noalloc(const void* x, int32_t x_dtype,
                                                  const bnb4_qstate* st,
                                                  void* stream) {
  if (!x || !st) return BNB4_ERR_INVALID_ARG;
  if (x_dtype != BNB4_F32 && x_dtype != BNB4_BF16 && x_dtype != BNB4_F16)
    return BNB4_ERR_UNSUPPORTED;
  if (!st->codes || st->n <= 0 || st->reserved != 0) return BNB4_ERR_INVALID_ARG;
  if (st->qtype != BNB4_NF4 && st->qtype != BNB4_FP4) return BNB4_ERR_INVALID_ARG;
  if (st->double_quant != 1) return BNB4_ERR_INVALID_ARG;
  if (st->blocksize != 32 && st->blocksize != 64 && st->blocksize != 128 &&
      st->blocksize != 256)
    return BNB4_ERR_UNSUPPORTED;
  if (!st->absmax_q || !st->scale2 || !st->offset) return BNB4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(st->codes, 16) || !aligned(st->absmax_q, 4) ||
      !aligned(st->scale2, 4) || !aligned(st->offset, 4))
    return BNB4_ERR_ALIGNMENT;
  const int64_t nb = (st->n + st->blocksize - 1) / st->blocksize;
  if (nb > BNB4_NOALLOC_MAX_BLOCKS) return BNB4_ERR_SCRATCH_LIMIT;

  int sms = 0, rc;
  if ((rc = sm_count(&sms)) != BNB4_OK) return rc;
  // x follows bnb_quantize_4bit's rules (device, managed or page-locked host
  // memory, the latter read through its device address); the outputs must
  // be device or managed memory.  A pointer query allocates nothing.
  const void* xd = nullptr;
  const void* d = nullptr;
  if ((rc = bnb4::resolve_ptr(x, bnb4::Residency::kDeviceOrPinnedHost, &xd)) != BNB4_OK)
    return rc;
  const auto out_mem = bnb4::Residency::kDeviceOrManaged;
  if ((rc = bnb4::resolve_ptr(st->codes, out_mem, &d)) != BNB4_OK ||
      (rc = bnb4::resolve_ptr(st->absmax_q, out_mem, &d)) != BNB4_OK ||
      (rc = bnb4::resolve_ptr(st->scale2, out_mem, &d)) != BNB4_OK ||
      (rc = bnb4::resolve_ptr(st->offset, out_mem, &d)) != BNB4_OK)
    return rc;
  unsigned char* scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != BNB4_OK) return rc;
  int* err = nullptr;
  if ((rc = bnb4::device_error_word(&err)) != BNB4_OK) return rc;

  bnb4_qstate s = *st;  // same kernels, with the intermediate absmax in scratch
  s.absmax = reinterpret_cast<float*>(scratch + kPartialsBytes);
  const cudaError_t e = bnb4::launch_quantize(xd, x_dtype, s, scratch, err, sms,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BNB4_OK : BNB4_ERR_CUDA;
}
