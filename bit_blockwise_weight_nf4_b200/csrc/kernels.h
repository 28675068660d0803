// kernels.h -- internal launcher interface between the C ABI (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bnb4.h"

namespace bnb4 {

struct View2D;  // a strided 2-D view (common.cuh)

// Where a pointer a kernel dereferences may live: device memory only;
// device or managed memory; device, managed or page-locked host memory.
enum class Residency { kDevice, kDeviceOrManaged, kDeviceOrPinnedHost };

// BNB4_OK with the address the device uses in *dev, or BNB4_ERR_INVALID_ARG
// (pageable host memory, a pointer the runtime does not know, or a kind of
// memory `where` excludes).  Host-only; launches nothing.
int resolve_ptr(const void* p, Residency where, const void** dev,
                bool* on_device = nullptr);

// Upper bound on the quantize grid.  The double-quant workspace holds one
// fp64 partial sum of the blocks' absmax per CTA.
constexpr int kMaxPartials = 4096;
constexpr size_t kDqWorkspaceBytes = sizeof(double) * static_cast<size_t>(kMaxPartials);

int quant_grid(int64_t n, int x_dtype, int num_sms);
// workspace: kDqWorkspaceBytes, 16-byte aligned (double quant only); err:
// the device error word (unused: the quantize kernels have no waits).  view: x is a row-major 2-D view with a row stride
// (see View2D), or null for a contiguous x.
// warm_x: x is device memory, which the quantize kernel may warm in L2
// before waiting on the previous kernel of a programmatic launch.
cudaError_t launch_quantize(const void* x, int x_dtype, const bnb4_qstate& st,
                            void* workspace, int* err, int num_sms, cudaStream_t s,
                            const View2D* view = nullptr, bool warm_x = false);

// The library's device error word on the current device (api.cu).
int device_error_word(int** out);

int dequant_grid(int64_t n, int out_dtype, int num_sms);
cudaError_t launch_dequantize(const bnb4_qstate& st, void* out, int out_dtype,
                              int grid, cudaStream_t s, const View2D* view = nullptr);

// Compares the quantize kernel's reciprocal with the correctly rounded one
// over its whole input range; result = {u64 mismatches, u32 first, u32 0}.
cudaError_t launch_check_rcp(void* result, cudaStream_t s);

// The linear kernels take the 16-bit compute format `fmt` (BNB4_BF16 or
// BNB4_F16) of x, y and bias; bias (N elements) may be null.
// err: the device error word (set when a bounded wait of the decode kernel
// expires).
cudaError_t launch_gemv(const void* x, int64_t B, int64_t K,
                        const bnb4_qstate& W, int64_t N, void* y, const void* bias,
                        int fmt, int num_sms, int* err, cudaStream_t s);

// One decode linear of a grouped launch (x [B, K], W [N, K], bias, y [B, N]).
struct GemvLinear {
  const void* x;
  const bnb4_qstate* W;
  int64_t K, N;
  const void* bias;
  void* y;
};

// The same GEMV in a launch of its own (one CTA per 16 rows, gemv_direct.cu):
// faster than the persistent kernel for a single weight.  B <= 8, or B <= 16
// when gemv_direct_takes(x, W, B) (x and the codes 32-byte aligned).
bool gemv_direct_takes(const void* x, const bnb4_qstate& W, int64_t B);
cudaError_t launch_gemv_direct(const void* x, int64_t B, int64_t K, const bnb4_qstate& W,
                               int64_t N, void* y, const void* bias, int fmt, int num_sms,
                               cudaStream_t s);
// A list of decode linears (one K, one format, B <= 8), one CTA per 16 rows of
// any of them, in launches of up to 32 weights.
cudaError_t launch_gemv_direct_list(const GemvLinear* lin, int count, int64_t B, int fmt,
                                    int num_sms, cudaStream_t s);


// 1..BNB4_GROUP_MAX linears of one format (blocksize, code table, scale
// format) and one batch size B <= 8: the persistent kernel for B = 1 and 4 or
// more weights (or always, with `persistent`), else the one-CTA-per-16-rows
// kernel; launches of up to 32 weights.
cudaError_t launch_gemv_group(const GemvLinear* lin, int count, int64_t B, int fmt,
                              int num_sms, int* err, cudaStream_t s, bool persistent = false);

// wait_limit_ns = 0 selects the normal bound of every mbarrier wait (2 s);
// withhold_first_x != 0 is the failure-detection diagnostic (the first X
// stage is never loaded, so the kernel's waits run out).
cudaError_t launch_gemm(const void* X, int64_t M, int64_t K,
                        const bnb4_qstate& W, int64_t N, void* Y, const void* bias,
                        int fmt, int* err, int num_sms, cudaStream_t s,
                        uint64_t wait_limit_ns = 0, int withhold_first_x = 0);

// Linear layer for 1..256 tokens (the small-batch tier): weight rows on the
// MMA's M side, tokens on its N side, K split over a cluster.
cudaError_t launch_gemm_small(const void* X, int64_t M, int64_t K,
                              const bnb4_qstate& W, int64_t N, void* Y, const void* bias,
                              int fmt, int* err, int num_sms, cudaStream_t s,
                              uint64_t wait_limit_ns = 0);

}  // namespace bnb4
