// api.cu -- the C ABI declared in include/bnb4.h: argument checks, buffer
// size queries, the device error word, and the launches on the caller's
// stream.  Nothing here allocates or synchronizes (bnb4_device_status aside).
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "bnb4.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// Set by kernels whose bounded waits expire; read by bnb4_device_status.
__device__ int g_device_error = 0;

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

bool valid_blocksize(int32_t bs) {
  return bs == 32 || bs == 64 || bs == 128 || bs == 256;
}

int64_t n_blocks(int64_t n, int64_t bs) { return (n + bs - 1) / bs; }

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices)
    return BNB4_ERR_CUDA;
  return BNB4_OK;
}

// Per-device caches of values that never change while the process runs.
// Host threads may fill them concurrently: each slot is an atomic written
// with the same value by whichever thread gets there, read relaxed.
int num_sms(int* out) {
  static std::atomic<int> cache[kMaxDevices];
  int dev;
  if (current_device(&dev) != BNB4_OK) return BNB4_ERR_CUDA;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess || v <= 0)
      return BNB4_ERR_CUDA;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  *out = v;
  return BNB4_OK;
}

int error_word(int** out) {
  static std::atomic<int*> cache[kMaxDevices];
  int dev;
  if (current_device(&dev) != BNB4_OK) return BNB4_ERR_CUDA;
  int* w = cache[dev].load(std::memory_order_relaxed);
  if (w == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess || !p)
      return BNB4_ERR_CUDA;
    w = static_cast<int*>(p);
    cache[dev].store(w, std::memory_order_relaxed);
  }
  *out = w;
  return BNB4_OK;
}

}  // namespace

int bnb4::device_error_word(int** out) { return error_word(out); }

namespace {

// Fields shared by every state check.
int check_state_common(const bnb4_qstate* st) {
  if (!st || !st->codes || st->n <= 0) return BNB4_ERR_INVALID_ARG;
  if (st->qtype != BNB4_NF4 && st->qtype != BNB4_FP4)
    return BNB4_ERR_INVALID_ARG;
  if (st->double_quant != 0 && st->double_quant != 1)
    return BNB4_ERR_INVALID_ARG;
  if (st->reserved != 0) return BNB4_ERR_INVALID_ARG;
  if (!valid_blocksize(st->blocksize)) return BNB4_ERR_UNSUPPORTED;
  if (!aligned(st->codes, 16)) return BNB4_ERR_ALIGNMENT;
  // the decode kernel copies the aligned 4-byte word holding each scale byte
  if (st->double_quant && st->absmax_q && !aligned(st->absmax_q, 4)) return BNB4_ERR_ALIGNMENT;
  return BNB4_OK;
}

// A state a consumer reads: the scales it needs must be present.
int check_state_read(const bnb4_qstate* st) {
  int rc = check_state_common(st);
  if (rc != BNB4_OK) return rc;
  if (st->double_quant) {
    if (!st->absmax_q || !st->scale2 || !st->offset) return BNB4_ERR_INVALID_ARG;
    if (!aligned(st->scale2, 4) || !aligned(st->offset, 4))
      return BNB4_ERR_ALIGNMENT;
  } else {
    if (!st->absmax) return BNB4_ERR_INVALID_ARG;
    if (!aligned(st->absmax, 4)) return BNB4_ERR_ALIGNMENT;
  }
  return BNB4_OK;
}

int check_weight(const bnb4_qstate* W, int64_t N, int64_t K) {
  int rc = check_state_read(W);
  if (rc != BNB4_OK) return rc;
  if (N <= 0 || K <= 0) return BNB4_ERR_SHAPE;
  if (N > INT64_MAX / K || W->n != N * K) return BNB4_ERR_SHAPE;
  if (K % 64 != 0 || K % W->blocksize != 0) return BNB4_ERR_SHAPE;
  return BNB4_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? BNB4_OK : BNB4_ERR_CUDA; }

}  // namespace

// Where a pointer that a kernel will dereference lives (declared in
// kernels.h, shared with the allocation-free entry point).  Device memory
// is used as it is; managed memory too where `where` allows it; page-locked
// host memory, where allowed, through the device address the runtime maps
// it to (the quantize kernels then stream it over the bus -- quantize on
// load).  Anything else, pageable host memory in particular, is refused
// before anything is launched: a kernel given a plain host address would
// fault.  *dev receives the address the device uses.
//
// The query is a host-side lookup that enqueues nothing; a caller may be in
// the middle of capturing a stream into a CUDA graph, whose default (global)
// mode forbids such calls.  The query therefore runs with this thread's
// capture interaction mode switched to relaxed and restored right after, so
// the checks behave the same inside and outside a capture.  *on_device (if
// given) tells whether p is plain device memory.
int bnb4::resolve_ptr(const void* p, Residency where, const void** dev, bool* on_device) {
  cudaPointerAttributes a;
  cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
  const bool swapped = cudaThreadExchangeStreamCaptureMode(&mode) == cudaSuccess;
  const cudaError_t q = cudaPointerGetAttributes(&a, p);
  if (swapped) cudaThreadExchangeStreamCaptureMode(&mode);
  if (q != cudaSuccess) {
    cudaGetLastError();  // clear the (non-sticky) error the failed query recorded
    return BNB4_ERR_INVALID_ARG;
  }
  if (on_device) *on_device = a.type == cudaMemoryTypeDevice;
  if (a.type == cudaMemoryTypeDevice) {
    *dev = p;
    return BNB4_OK;
  }
  if (a.type == cudaMemoryTypeManaged && where != Residency::kDevice) {
    *dev = p;
    return BNB4_OK;
  }
  if (a.type == cudaMemoryTypeHost && a.devicePointer &&
      where == Residency::kDeviceOrPinnedHost) {
    *dev = a.devicePointer;
    return BNB4_OK;
  }
  return BNB4_ERR_INVALID_ARG;
}

namespace {

// The pointers of a quantization state that a kernel touches: device or
// managed memory.  `scales_of_reader`: only the scale arrays a consumer reads
// (absmax without double quantization, the three double-quant arrays with
// it); otherwise every non-null array the quantize kernels write.
int check_state_memory(const bnb4_qstate* st, bool scales_of_reader,
                       bnb4::Residency where = bnb4::Residency::kDeviceOrManaged) {
  const void* d;
  int rc;
  if ((rc = bnb4::resolve_ptr(st->codes, where, &d)) != BNB4_OK) return rc;
  const bool want_absmax = scales_of_reader ? !st->double_quant : st->absmax != nullptr;
  const bool want_dq = st->double_quant != 0;
  if (want_absmax && (rc = bnb4::resolve_ptr(st->absmax, where, &d)) != BNB4_OK) return rc;
  if (want_dq) {
    if ((rc = bnb4::resolve_ptr(st->absmax_q, where, &d)) != BNB4_OK) return rc;
    if ((rc = bnb4::resolve_ptr(st->scale2, where, &d)) != BNB4_OK) return rc;
    if ((rc = bnb4::resolve_ptr(st->offset, where, &d)) != BNB4_OK) return rc;
  }
  return BNB4_OK;
}

// Activations, outputs and bias of the linear entry points: device memory
// (the kernels read x and write y through TMA on the larger tiers).
int check_linear_memory(const void* x, const void* y, const void* bias,
                        const bnb4_qstate* W) {
  const void* d;
  int rc;
  const auto dev = bnb4::Residency::kDevice;
  if ((rc = bnb4::resolve_ptr(x, dev, &d)) != BNB4_OK) return rc;
  if ((rc = bnb4::resolve_ptr(y, dev, &d)) != BNB4_OK) return rc;
  if (bias && (rc = bnb4::resolve_ptr(bias, dev, &d)) != BNB4_OK) return rc;
  return check_state_memory(W, true, dev);
}

// A row-major [rows, cols] view with row stride ld over a state of n = rows
// * cols elements: whole 16-byte chunks per row (cols and ld multiples of
// `epc` elements), ld >= cols, and n < 2^32 (the view's index division).
int check_view(int64_t rows, int64_t cols, int64_t ld, int64_t n, int64_t epc) {
  if (rows < 1 || cols < 1 || ld < cols) return BNB4_ERR_SHAPE;
  if (cols % epc != 0 || ld % epc != 0) return BNB4_ERR_SHAPE;
  if (rows > INT64_MAX / cols || rows * cols != n) return BNB4_ERR_SHAPE;
  if (n >= (int64_t(1) << 32)) return BNB4_ERR_SHAPE;
  return BNB4_OK;
}

int quantize_impl(const void* x, int32_t x_dtype, const bnb4_qstate* st, void* workspace,
                  size_t workspace_bytes, void* stream, const bnb4::View2D* view) {
  if (!x) return BNB4_ERR_INVALID_ARG;
  if (x_dtype != BNB4_F32 && x_dtype != BNB4_BF16 && x_dtype != BNB4_F16)
    return BNB4_ERR_UNSUPPORTED;
  int rc = check_state_common(st);
  if (rc != BNB4_OK) return rc;
  if (!st->absmax) return BNB4_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return BNB4_ERR_ALIGNMENT;
  if (!aligned(st->absmax, 4)) return BNB4_ERR_ALIGNMENT;
  if (st->double_quant) {
    if (!st->absmax_q || !st->scale2 || !st->offset) return BNB4_ERR_INVALID_ARG;
    if (!aligned(st->scale2, 4) || !aligned(st->offset, 4))
      return BNB4_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < bnb4::kDqWorkspaceBytes) return BNB4_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return BNB4_ERR_ALIGNMENT;
  }
  int sms;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  const void *xd, *ws_dev;
  bool x_dev = false;
  if ((rc = bnb4::resolve_ptr(x, bnb4::Residency::kDeviceOrPinnedHost, &xd, &x_dev)) !=
      BNB4_OK)
    return rc;
  if ((rc = check_state_memory(st, false)) != BNB4_OK) return rc;
  if (st->double_quant &&
      (rc = bnb4::resolve_ptr(workspace, bnb4::Residency::kDeviceOrManaged, &ws_dev)) !=
          BNB4_OK)
    return rc;
  int* err = nullptr;
  if (st->double_quant && (rc = error_word(&err)) != BNB4_OK) return rc;
  return from_cuda(bnb4::launch_quantize(xd, x_dtype, *st, workspace, err, sms,
                                         static_cast<cudaStream_t>(stream), view, x_dev));
}

int dequantize_impl(const bnb4_qstate* st, void* out, int32_t out_dtype, void* stream,
                    const bnb4::View2D* view) {
  if (!out) return BNB4_ERR_INVALID_ARG;
  if (out_dtype != BNB4_F32 && out_dtype != BNB4_BF16 && out_dtype != BNB4_F16)
    return BNB4_ERR_UNSUPPORTED;
  int rc = check_state_read(st);
  if (rc != BNB4_OK) return rc;
  if (!aligned(out, 16)) return BNB4_ERR_ALIGNMENT;
  int sms;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  const void* od;
  if ((rc = bnb4::resolve_ptr(out, bnb4::Residency::kDeviceOrManaged, &od)) != BNB4_OK)
    return rc;
  if ((rc = check_state_memory(st, true)) != BNB4_OK) return rc;
  const int grid = bnb4::dequant_grid(st->n, out_dtype, sms);
  return from_cuda(bnb4::launch_dequantize(*st, out, out_dtype, grid,
                                           static_cast<cudaStream_t>(stream), view));
}

// Kernel choice by the number of token rows: the mma.sync GEMV up to 8 (x
// as the MMA's B operand), and from 9 to 16 when x and the codes are 32-byte
// aligned (x as its A operand; measured faster than the small-M kernel on
// the Llama-7B shapes), the small-M tcgen05 kernel (weight rows as the MMA's
// M, K split over a cluster) up to 256, the 2-CTA tcgen05 GEMM above.
// Grouped decode calls take up to 8 rows.
constexpr int64_t kGemvMaxB = 8;
constexpr int64_t kSmallMaxM = 256;

bool use_gemv(const void* x, const bnb4_qstate& W, int64_t M) {
  return M <= kGemvMaxB || bnb4::gemv_direct_takes(x, W, M);
}

}  // namespace

extern "C" {

int bnb4_abi_version(void) { return BNB4_ABI_VERSION; }

const char* bnb4_strerror(int status) {
  switch (status) {
    case BNB4_OK: return "ok";
    case BNB4_ERR_INVALID_ARG: return "invalid argument (null pointer, n <= 0 or bad enum)";
    case BNB4_ERR_UNSUPPORTED: return "unsupported blocksize or dtype";
    case BNB4_ERR_ALIGNMENT: return "pointer misaligned (16 bytes for vector data)";
    case BNB4_ERR_SHAPE: return "shape constraint violated";
    case BNB4_ERR_WORKSPACE: return "workspace missing or too small";
    case BNB4_ERR_CUDA: return "CUDA runtime error";
    case BNB4_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    case BNB4_ERR_SCRATCH_LIMIT:
      return "input exceeds the fixed scratch of the allocation-free entry point";
    default: return "unknown status";
  }
}

int bnb4_query_sizes(int64_t n, int32_t blocksize, int32_t double_quant,
                     bnb4_sizes* out) {
  if (!out || n <= 0 || (double_quant != 0 && double_quant != 1))
    return BNB4_ERR_INVALID_ARG;
  if (!valid_blocksize(blocksize)) return BNB4_ERR_UNSUPPORTED;
  const int64_t nb = n_blocks(n, blocksize);
  const int64_t ng = n_blocks(nb, 256);
  out->codes = static_cast<size_t>((n + 1) / 2);
  out->absmax = static_cast<size_t>(4 * nb);
  out->absmax_q = double_quant ? static_cast<size_t>(nb) : 0;
  out->scale2 = double_quant ? static_cast<size_t>(4 * ng) : 0;
  out->offset = double_quant ? 4 : 0;
  out->workspace = double_quant ? bnb4::kDqWorkspaceBytes : 0;
  return BNB4_OK;
}

int bnb_quantize_4bit(const void* x, int32_t x_dtype, const bnb4_qstate* st,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return quantize_impl(x, x_dtype, st, workspace, workspace_bytes, stream, nullptr);
}

int bnb_quantize_4bit_2d(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                         int64_t ld, const bnb4_qstate* st, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (!x || !st) return BNB4_ERR_INVALID_ARG;
  if (x_dtype != BNB4_F32 && x_dtype != BNB4_BF16 && x_dtype != BNB4_F16)
    return BNB4_ERR_UNSUPPORTED;
  const int rc = check_view(rows, cols, ld, st->n, x_dtype == BNB4_F32 ? 4 : 8);
  if (rc != BNB4_OK) return rc;
  if (ld == cols)
    return quantize_impl(x, x_dtype, st, workspace, workspace_bytes, stream, nullptr);
  const bnb4::View2D v = bnb4::make_view(cols, ld);
  return quantize_impl(x, x_dtype, st, workspace, workspace_bytes, stream, &v);
}

int bnb_dequantize_4bit(const bnb4_qstate* st, void* out, int32_t out_dtype,
                        void* stream) {
  return dequantize_impl(st, out, out_dtype, stream, nullptr);
}

int bnb_dequantize_4bit_2d(const bnb4_qstate* st, void* out, int32_t out_dtype, int64_t rows,
                           int64_t cols, int64_t ld, void* stream) {
  if (!st || !out) return BNB4_ERR_INVALID_ARG;
  if (out_dtype != BNB4_F32 && out_dtype != BNB4_BF16 && out_dtype != BNB4_F16)
    return BNB4_ERR_UNSUPPORTED;
  const int rc = check_view(rows, cols, ld, st->n, out_dtype == BNB4_F32 ? 4 : 8);
  if (rc != BNB4_OK) return rc;
  if (ld == cols) return dequantize_impl(st, out, out_dtype, stream, nullptr);
  const bnb4::View2D v = bnb4::make_view(cols, ld);
  return dequantize_impl(st, out, out_dtype, stream, &v);
}

int bnb_gemv_4bit(const void* x, int64_t B, int64_t K, const bnb4_qstate* W,
                  int64_t N, void* y, void* stream) {
  if (!x || !y) return BNB4_ERR_INVALID_ARG;
  int rc = check_weight(W, N, K);
  if (rc != BNB4_OK) return rc;
  if (B < 1 || B > kSmallMaxM) return BNB4_ERR_SHAPE;
  if (N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return BNB4_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(y, 2)) return BNB4_ERR_ALIGNMENT;
  int sms;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  if ((rc = check_linear_memory(x, y, nullptr, W)) != BNB4_OK) return rc;
  int* err;
  if ((rc = error_word(&err)) != BNB4_OK) return rc;
  if (use_gemv(x, *W, B))
    return from_cuda(bnb4::launch_gemv(x, B, K, *W, N, y, nullptr, BNB4_BF16, sms, err,
                                       static_cast<cudaStream_t>(stream)));
  return from_cuda(bnb4::launch_gemm_small(x, B, K, *W, N, y, nullptr, BNB4_BF16, err, sms,
                                           static_cast<cudaStream_t>(stream)));
}

namespace {
int gemv_grouped_impl(const bnb4_gemv_problem* problems, int32_t count, int64_t B,
                      int32_t dtype, void* stream, bool persistent) {
  if (!problems || count < 1) return BNB4_ERR_INVALID_ARG;
  if (count > BNB4_GROUP_MAX) return BNB4_ERR_SHAPE;
  if (dtype != BNB4_BF16 && dtype != BNB4_F16) return BNB4_ERR_UNSUPPORTED;
  if (B < 1 || B > kGemvMaxB) return BNB4_ERR_SHAPE;
  bnb4::GemvLinear lin[BNB4_GROUP_MAX];
  const bnb4_qstate& W0 = problems[0].W;
  for (int32_t i = 0; i < count; ++i) {
    const bnb4_gemv_problem& p = problems[i];
    if (!p.x || !p.y) return BNB4_ERR_INVALID_ARG;
    int rc = check_weight(&p.W, p.N, p.K);
    if (rc != BNB4_OK) return rc;
    if (p.N >= (int64_t(1) << 31) || p.K >= (int64_t(1) << 31) || p.K != problems[0].K)
      return BNB4_ERR_SHAPE;
    if (p.W.blocksize != W0.blocksize || p.W.qtype != W0.qtype ||
        p.W.double_quant != W0.double_quant)
      return BNB4_ERR_UNSUPPORTED;
    if (!aligned(p.x, 16) || !aligned(p.y, 2) || !aligned(p.bias, 16))
      return BNB4_ERR_ALIGNMENT;
    lin[i] = bnb4::GemvLinear{p.x, &p.W, p.K, p.N, p.bias, p.y};
  }
  int sms, rc;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  for (int32_t i = 0; i < count; ++i) {
    const bnb4_gemv_problem& p = problems[i];
    if ((rc = check_linear_memory(p.x, p.y, p.bias, &p.W)) != BNB4_OK) return rc;
  }
  int* err;
  if ((rc = error_word(&err)) != BNB4_OK) return rc;
  return from_cuda(bnb4::launch_gemv_group(lin, count, B, dtype, sms, err,
                                           static_cast<cudaStream_t>(stream), persistent));
}
}  // namespace

int bnb_gemv_4bit_grouped(const bnb4_gemv_problem* problems, int32_t count, int64_t B,
                          int32_t dtype, void* stream) {
  return gemv_grouped_impl(problems, count, B, dtype, stream, false);
}

int bnb4_debug_gemv_grouped_persistent(const bnb4_gemv_problem* problems, int32_t count,
                                       int64_t B, int32_t dtype, void* stream) {
  return gemv_grouped_impl(problems, count, B, dtype, stream, true);
}

int bnb_gemm_4bit(const void* X, int64_t M, int64_t K, const bnb4_qstate* W,
                  int64_t N, void* Y, void* stream) {
  if (!X || !Y) return BNB4_ERR_INVALID_ARG;
  int rc = check_weight(W, N, K);
  if (rc != BNB4_OK) return rc;
  if (M < 1 || N % 8 != 0 || M > (int64_t(1) << 31) || N >= (int64_t(1) << 31) ||
      K >= (int64_t(1) << 31))
    return BNB4_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(Y, 16)) return BNB4_ERR_ALIGNMENT;
  int sms;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  if ((rc = check_linear_memory(X, Y, nullptr, W)) != BNB4_OK) return rc;
  int* err;
  if ((rc = error_word(&err)) != BNB4_OK) return rc;
  if (use_gemv(X, *W, M))
    return from_cuda(bnb4::launch_gemv(X, M, K, *W, N, Y, nullptr, BNB4_BF16, sms, err,
                                       static_cast<cudaStream_t>(stream)));
  if (M <= kSmallMaxM)
    return from_cuda(bnb4::launch_gemm_small(X, M, K, *W, N, Y, nullptr, BNB4_BF16, err,
                                             sms, static_cast<cudaStream_t>(stream)));
  return from_cuda(bnb4::launch_gemm(X, M, K, *W, N, Y, nullptr, BNB4_BF16, err, sms,
                                     static_cast<cudaStream_t>(stream)));
}

int bnb_linear_4bit(const void* x, int32_t dtype, int64_t M, int64_t K, const bnb4_qstate* W,
                    int64_t N, const void* bias, void* y, void* stream) {
  if (!x || !y) return BNB4_ERR_INVALID_ARG;
  if (dtype != BNB4_BF16 && dtype != BNB4_F16) return BNB4_ERR_UNSUPPORTED;
  int rc = check_weight(W, N, K);
  if (rc != BNB4_OK) return rc;
  if (M < 1 || M > (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return BNB4_ERR_SHAPE;
  if (M > kSmallMaxM && N % 8 != 0) return BNB4_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(y, M > kSmallMaxM ? 16 : 2) || !aligned(bias, 16))
    return BNB4_ERR_ALIGNMENT;
  int sms;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  if ((rc = check_linear_memory(x, y, bias, W)) != BNB4_OK) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err;
  if ((rc = error_word(&err)) != BNB4_OK) return rc;
  if (use_gemv(x, *W, M))
    return from_cuda(bnb4::launch_gemv(x, M, K, *W, N, y, bias, dtype, sms, err, s));
  if (M <= kSmallMaxM)
    return from_cuda(bnb4::launch_gemm_small(x, M, K, *W, N, y, bias, dtype, err, sms, s));
  return from_cuda(bnb4::launch_gemm(x, M, K, *W, N, y, bias, dtype, err, sms, s));
}

int bnb4_debug_gemm_withhold(const void* X, int64_t M, int64_t K,
                             const bnb4_qstate* W, int64_t N, void* Y,
                             int32_t wait_limit_us, void* stream) {
  if (!X || !Y) return BNB4_ERR_INVALID_ARG;
  int rc = check_weight(W, N, K);
  if (rc != BNB4_OK) return rc;
  if (M < 1 || N % 8 != 0 || M > (int64_t(1) << 31) || N > (int64_t(1) << 31))
    return BNB4_ERR_SHAPE;
  if (wait_limit_us < 1 || wait_limit_us > 1000000) return BNB4_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Y, 16)) return BNB4_ERR_ALIGNMENT;
  int sms;
  if ((rc = num_sms(&sms)) != BNB4_OK) return rc;
  if ((rc = check_linear_memory(X, Y, nullptr, W)) != BNB4_OK) return rc;
  int* err;
  if ((rc = error_word(&err)) != BNB4_OK) return rc;
  return from_cuda(bnb4::launch_gemm(X, M, K, *W, N, Y, nullptr, BNB4_BF16, err, sms,
                                     static_cast<cudaStream_t>(stream),
                                     static_cast<uint64_t>(wait_limit_us) * 1000u, 1));
}

int bnb4_debug_check_rcp(void* result, void* stream) {
  if (!result) return BNB4_ERR_INVALID_ARG;
  if (!aligned(result, 8)) return BNB4_ERR_ALIGNMENT;
  const void* d;
  const int rc = bnb4::resolve_ptr(result, bnb4::Residency::kDeviceOrManaged, &d);
  if (rc != BNB4_OK) return rc;
  return from_cuda(bnb4::launch_check_rcp(result, static_cast<cudaStream_t>(stream)));
}

int bnb4_device_status(void* stream, int32_t clear) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BNB4_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess)
    return BNB4_ERR_CUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
      return BNB4_ERR_CUDA;
  }
  return v ? BNB4_ERR_DEVICE_TIMEOUT : BNB4_OK;
}

}  // extern "C"
