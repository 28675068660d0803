"""Python binding of the bnb4 C ABI (``include/bnb4.h``).

Two layers, both argument marshalling only -- every step of the
quantize / dequantize / GEMV / GEMM path runs in the CUDA library:

* raw ctypes entry points with the C names (``bnb_quantize_4bit``,
  ``bnb_quantize_4bit_noalloc``, ``bnb_dequantize_4bit``, ``bnb_gemv_4bit``,
  ``bnb_gemv_4bit_grouped``, ``bnb_gemm_4bit``,
  ``bnb_linear_4bit``, ``bnb4_query_sizes``, ``bnb4_device_status``,
  ``bnb4_strerror``, ``bnb4_abi_version``), returning the C status;
* torch helpers (``QuantState``, ``quantize_4bit``, ``dequantize_4bit``,
  ``gemv_4bit``, ``gemv_4bit_grouped``, ``gemm_4bit``, ``linear_4bit``) that
  allocate device buffers
  with torch, call the entry points on torch's current stream and raise
  ``Bnb4Error`` on a non-zero status.

There is no CPU fallback: if ``libbnb4.so`` is missing, ``load()`` raises.
Build it with ``python -m bit_blockwise_weight_nf4_b200.build``.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbnb4.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_ALIGNMENT = -3
ERR_SHAPE = -4
ERR_WORKSPACE = -5
ERR_CUDA = -6
ERR_DEVICE_TIMEOUT = -7
ERR_SCRATCH_LIMIT = -8

NOALLOC_MAX_BLOCKS = 1 << 20

NF4 = 0
FP4 = 1
F32 = 0
BF16 = 1
F16 = 2

ABI_VERSION = 4
GROUP_MAX = 256


class QState(ctypes.Structure):
    """``bnb4_qstate``: device pointers of a quantization state."""
    _fields_ = [("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("absmax_q", ctypes.c_void_p), ("scale2", ctypes.c_void_p),
                ("offset", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("blocksize", ctypes.c_int32), ("qtype", ctypes.c_int32),
                ("double_quant", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class GemvProblem(ctypes.Structure):
    """``bnb4_gemv_problem``: one linear of a grouped decode launch."""
    _fields_ = [("x", ctypes.c_void_p), ("W", QState), ("K", ctypes.c_int64),
                ("N", ctypes.c_int64), ("bias", ctypes.c_void_p), ("y", ctypes.c_void_p)]


class Sizes(ctypes.Structure):
    """``bnb4_sizes``: byte sizes of a state's buffers."""
    _fields_ = [("codes", ctypes.c_size_t), ("absmax", ctypes.c_size_t),
                ("absmax_q", ctypes.c_size_t), ("scale2", ctypes.c_size_t),
                ("offset", ctypes.c_size_t), ("workspace", ctypes.c_size_t)]


class Bnb4Error(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__("%s failed: %s (status %d)"
                         % (what or "bnb4 call", bnb4_strerror(status), status))


_lib = None


def load():
    """Load libbnb4.so (once).  Raises if the library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libbnb4.so is missing; build it with "
            "`python -m bit_blockwise_weight_nf4_b200.build` (no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    QP = ctypes.POINTER(QState)
    sig = {
        "bnb4_query_sizes": ([i64, i32, i32, ctypes.POINTER(Sizes)], ctypes.c_int),
        "bnb_quantize_4bit": ([p, i32, QP, p, sz, p], ctypes.c_int),
        "bnb_quantize_4bit_noalloc": ([p, i32, QP, p], ctypes.c_int),
        "bnb_dequantize_4bit": ([QP, p, i32, p], ctypes.c_int),
        "bnb_quantize_4bit_2d": ([p, i32, i64, i64, i64, QP, p, sz, p], ctypes.c_int),
        "bnb_dequantize_4bit_2d": ([QP, p, i32, i64, i64, i64, p], ctypes.c_int),
        "bnb_gemv_4bit": ([p, i64, i64, QP, i64, p, p], ctypes.c_int),
        "bnb_gemm_4bit": ([p, i64, i64, QP, i64, p, p], ctypes.c_int),
        "bnb_gemv_4bit_grouped": ([ctypes.POINTER(GemvProblem), i32, i64, i32, p],
                                  ctypes.c_int),
        "bnb4_debug_gemv_grouped_persistent": ([ctypes.POINTER(GemvProblem), i32, i64, i32, p],
                                               ctypes.c_int),
        "bnb_linear_4bit": ([p, i32, i64, i64, QP, i64, p, p, p], ctypes.c_int),
        "bnb4_device_status": ([p, i32], ctypes.c_int),
        "bnb4_debug_gemm_withhold": ([p, i64, i64, QP, i64, p, i32, p], ctypes.c_int),
        "bnb4_debug_check_rcp": ([p, p], ctypes.c_int),
        "bnb4_strerror": ([ctypes.c_int], ctypes.c_char_p),
        "bnb4_abi_version": ([], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    if lib.bnb4_abi_version() != ABI_VERSION:
        raise RuntimeError("libbnb4.so ABI version mismatch")
    _lib = lib
    return lib


# ------------------------------------------------------ raw C entry points
def bnb4_abi_version():
    return load().bnb4_abi_version()


def bnb4_strerror(status):
    return load().bnb4_strerror(status).decode()


def bnb4_query_sizes(n, blocksize, double_quant):
    out = Sizes()
    rc = load().bnb4_query_sizes(n, blocksize, int(bool(double_quant)),
                                 ctypes.byref(out))
    return rc, out


def bnb_quantize_4bit(x, x_dtype, st, workspace, workspace_bytes, stream):
    return load().bnb_quantize_4bit(x, x_dtype, ctypes.byref(st), workspace,
                                    workspace_bytes, stream)


def bnb_quantize_4bit_noalloc(x, x_dtype, st, stream):
    """Allocation-free double-quantized quantize (see include/bnb4.h): the
    library keeps its scratch in its own fixed device array, so the caller
    passes no workspace and st.absmax is ignored."""
    return load().bnb_quantize_4bit_noalloc(x, x_dtype, ctypes.byref(st), stream)


def bnb_dequantize_4bit(st, out, out_dtype, stream):
    return load().bnb_dequantize_4bit(ctypes.byref(st), out, out_dtype, stream)


def bnb_quantize_4bit_2d(x, x_dtype, rows, cols, ld, st, workspace, workspace_bytes, stream):
    return load().bnb_quantize_4bit_2d(x, x_dtype, rows, cols, ld, ctypes.byref(st),
                                       workspace, workspace_bytes, stream)


def bnb_dequantize_4bit_2d(st, out, out_dtype, rows, cols, ld, stream):
    return load().bnb_dequantize_4bit_2d(ctypes.byref(st), out, out_dtype, rows, cols, ld,
                                         stream)


def bnb_gemv_4bit(x, B, K, W, N, y, stream):
    return load().bnb_gemv_4bit(x, B, K, ctypes.byref(W), N, y, stream)


def bnb_gemm_4bit(X, M, K, W, N, Y, stream):
    return load().bnb_gemm_4bit(X, M, K, ctypes.byref(W), N, Y, stream)


def bnb_gemv_4bit_grouped(problems, B, dtype, stream):
    """``problems``: a sequence of GemvProblem (or a ctypes array of them)."""
    if not isinstance(problems, ctypes.Array):
        problems = (GemvProblem * len(problems))(*problems)
    return load().bnb_gemv_4bit_grouped(problems, len(problems), B, dtype, stream)


def bnb4_debug_gemv_grouped_persistent(problems, B, dtype, stream):
    """bnb_gemv_4bit_grouped forced onto the persistent kernel (tests)."""
    if not isinstance(problems, ctypes.Array):
        problems = (GemvProblem * len(problems))(*problems)
    return load().bnb4_debug_gemv_grouped_persistent(problems, len(problems), B, dtype, stream)


def bnb_linear_4bit(x, dtype, M, K, W, N, bias, y, stream):
    return load().bnb_linear_4bit(x, dtype, M, K, ctypes.byref(W), N, bias, y, stream)


def bnb4_debug_gemm_withhold(X, M, K, W, N, Y, wait_limit_us, stream):
    """Failure-detection diagnostic (see include/bnb4.h)."""
    return load().bnb4_debug_gemm_withhold(X, M, K, ctypes.byref(W), N, Y,
                                           wait_limit_us, stream)


def bnb4_debug_check_rcp(result, stream):
    """Self-check of the quantize kernel's reciprocal over its whole input
    range (see include/bnb4.h); result = 16-byte device buffer."""
    return load().bnb4_debug_check_rcp(result, stream)


def bnb4_device_status(stream, clear=True):
    return load().bnb4_device_status(stream, int(bool(clear)))


# ------------------------------------------------------------ torch layer
def _torch():
    import torch
    return torch


def _stream():
    return _torch().cuda.current_stream().cuda_stream


def _check(rc, what):
    if rc != OK:
        raise Bnb4Error(rc, what)


class QuantState:
    """Device buffers of a quantization state of ``n`` elements (torch
    tensors) plus the matching ``bnb4_qstate`` struct."""

    def __init__(self, n, blocksize=64, qtype=NF4, double_quant=True,
                 device="cuda"):
        torch = _torch()
        rc, sz = bnb4_query_sizes(n, blocksize, double_quant)
        _check(rc, "bnb4_query_sizes")
        self.n, self.blocksize, self.qtype = n, blocksize, qtype
        self.double_quant = bool(double_quant)
        u8, f32 = torch.uint8, torch.float32
        self.codes = torch.empty(sz.codes, dtype=u8, device=device)
        self.absmax = torch.empty(sz.absmax // 4, dtype=f32, device=device)
        self.absmax_q = torch.empty(sz.absmax_q, dtype=u8, device=device) \
            if self.double_quant else None
        self.scale2 = torch.empty(sz.scale2 // 4, dtype=f32, device=device) \
            if self.double_quant else None
        self.offset = torch.empty(1, dtype=f32, device=device) \
            if self.double_quant else None
        self.workspace_bytes = sz.workspace

    @staticmethod
    def _p(t):
        return None if t is None else t.data_ptr()

    def cstruct(self):
        return QState(self._p(self.codes), self._p(self.absmax),
                      self._p(self.absmax_q), self._p(self.scale2),
                      self._p(self.offset), self.n, self.blocksize, self.qtype,
                      int(self.double_quant), 0)

    @property
    def nbytes(self):
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.absmax_q, self.scale2, self.offset)
                   if t is not None) + (0 if self.double_quant else
                                        self.absmax.numel() * 4)


_DT = {"torch.float32": F32, "torch.bfloat16": BF16, "torch.float16": F16}


def workspace_for(state):
    torch = _torch()
    if state.workspace_bytes == 0:
        return None
    return torch.empty(state.workspace_bytes, dtype=torch.uint8,
                       device=state.codes.device)


def _view_2d(t):
    """(rows, cols, ld) of a 2-D tensor whose rows are contiguous, else None."""
    if t.dim() != 2 or t.stride(1) != 1:
        return None
    return t.shape[0], t.shape[1], t.stride(0)


def quantize_4bit(x, blocksize=64, qtype=NF4, double_quant=True, state=None,
                  workspace=None):
    """Quantize an fp32 / bf16 / fp16 tensor (in its logical row-major order):
    a CUDA tensor, or a page-locked CPU tensor (``pin_memory()``), which the
    kernel reads over the bus and quantizes on the way in.  Contiguous
    tensors of any shape, or 2-D views with contiguous rows (row stride
    ``x.stride(0)``)."""
    dt = _DT.get(str(x.dtype))
    if dt is None:
        raise TypeError("quantize_4bit takes float32, bfloat16 or float16")
    if x.device.type == "cpu" and not x.is_pinned():
        raise ValueError("quantize_4bit reads CPU tensors only from page-locked memory")
    view = None if x.is_contiguous() else _view_2d(x)
    if not x.is_contiguous() and view is None:
        raise ValueError("quantize_4bit takes a contiguous tensor or a 2-D row-strided view")
    device = x.device if x.device.type == "cuda" else _torch().device("cuda")
    if state is None:
        state = QuantState(x.numel(), blocksize, qtype, double_quant, device)
    if workspace is None:
        workspace = workspace_for(state)
    st = state.cstruct()
    ws = None if workspace is None else workspace.data_ptr()
    wsb = 0 if workspace is None else workspace.numel()
    if view is None:
        rc = bnb_quantize_4bit(x.data_ptr(), dt, st, ws, wsb, _stream())
    else:
        rc = bnb_quantize_4bit_2d(x.data_ptr(), dt, *view, st, ws, wsb, _stream())
    _check(rc, "bnb_quantize_4bit")
    return state


def dequantize_4bit(state, out_dtype=None, out=None):
    """Dequantize to a flat fp32 (default), bf16 or fp16 CUDA tensor, or into
    ``out``: a contiguous tensor of state.n elements or a 2-D view with
    contiguous rows."""
    torch = _torch()
    out_dtype = out_dtype or torch.float32
    if out is None:
        out = torch.empty(state.n, dtype=out_dtype, device=state.codes.device)
    dt = _DT[str(out.dtype)]
    if out.is_contiguous():
        rc = bnb_dequantize_4bit(state.cstruct(), out.data_ptr(), dt, _stream())
    else:
        view = _view_2d(out)
        if view is None:
            raise ValueError("dequantize_4bit writes a contiguous tensor or a 2-D row-strided view")
        rc = bnb_dequantize_4bit_2d(state.cstruct(), out.data_ptr(), dt, *view, _stream())
    _check(rc, "bnb_dequantize_4bit")
    return out


def gemv_4bit(x, state, N, out=None):
    """y = x @ What^T for bf16 x [B, K], B <= 256; What is the [N, K] weight."""
    torch = _torch()
    B, K = x.shape
    if out is None:
        out = torch.empty(B, N, dtype=torch.bfloat16, device=x.device)
    rc = bnb_gemv_4bit(x.data_ptr(), B, K, state.cstruct(), N, out.data_ptr(),
                       _stream())
    _check(rc, "bnb_gemv_4bit")
    return out


def gemm_4bit(X, state, N, out=None):
    """Y = X @ What^T for bf16 X [M, K]; What is the [N, K] weight."""
    torch = _torch()
    M, K = X.shape
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    rc = bnb_gemm_4bit(X.data_ptr(), M, K, state.cstruct(), N, out.data_ptr(),
                       _stream())
    _check(rc, "bnb_gemm_4bit")
    return out


def linear_4bit(x, state, N, bias=None, out=None):
    """y = x @ What^T (+ bias) for x [M, K] in bf16 or fp16 (the compute
    type; What is the [N, K] weight dequantized in it, bias [N] of the same
    dtype or None)."""
    torch = _torch()
    M, K = x.shape
    dt = {"torch.bfloat16": BF16, "torch.float16": F16}.get(str(x.dtype))
    if dt is None:
        raise TypeError("linear_4bit takes bfloat16 or float16 activations")
    if bias is not None and bias.dtype != x.dtype:
        raise TypeError("bias must have the dtype of x")
    if out is None:
        out = torch.empty(M, N, dtype=x.dtype, device=x.device)
    rc = bnb_linear_4bit(x.data_ptr(), dt, M, K, state.cstruct(), N,
                         None if bias is None else bias.data_ptr(), out.data_ptr(),
                         _stream())
    _check(rc, "bnb_linear_4bit")
    return out


def gemv_4bit_grouped(items, outs=None, _persistent=False):
    """Several decode linears in one launch: ``items`` is a list of (x,
    state, N) or (x, state, N, bias) with x [B, K] (bf16 or fp16, the same B
    and dtype for all; x may be shared); returns the outputs [B, N] (or
    writes ``outs``).  With one row of x and four or more linears the list
    runs the persistent decode kernel (``_persistent=True`` forces it, for
    tests), whose fp32 sums may differ in the last bit from a single call's."""
    torch = _torch()
    if outs is None:
        outs = [torch.empty(it[0].shape[0], it[2], dtype=it[0].dtype, device=it[0].device)
                for it in items]
    dt = {"torch.bfloat16": BF16, "torch.float16": F16}.get(str(items[0][0].dtype))
    if dt is None:
        raise TypeError("gemv_4bit_grouped takes bfloat16 or float16 activations")
    probs = (GemvProblem * len(items))()
    for i, (it, y) in enumerate(zip(items, outs)):
        x, state, N = it[0], it[1], it[2]
        bias = it[3] if len(it) > 3 else None
        probs[i] = GemvProblem(x.data_ptr(), state.cstruct(), x.shape[1], N,
                               None if bias is None else bias.data_ptr(), y.data_ptr())
    fn = bnb4_debug_gemv_grouped_persistent if _persistent else bnb_gemv_4bit_grouped
    rc = fn(probs, items[0][0].shape[0], dt, _stream())
    _check(rc, "bnb_gemv_4bit_grouped")
    return outs


def state_from_arrays(arrs, device="cuda"):
    """A device QuantState holding copies of host arrays (numpy) with the
    keys codes / absmax / absmax_q / scale2 / offset / n / blocksize / qtype /
    double_quant -- e.g. a state computed elsewhere."""
    torch = _torch()
    st = QuantState(arrs["n"], arrs["blocksize"], arrs["qtype"],
                    arrs["double_quant"], device)
    st.codes.copy_(torch.from_numpy(arrs["codes"]))
    st.absmax.copy_(torch.from_numpy(arrs["absmax"]))
    if st.double_quant:
        st.absmax_q.copy_(torch.from_numpy(arrs["absmax_q"]))
        st.scale2.copy_(torch.from_numpy(arrs["scale2"]))
        st.offset.copy_(torch.from_numpy(arrs["offset"]))
    return st


def state_to_arrays(state):
    """Host (numpy) copies of a device QuantState's buffers."""
    d = {"n": state.n, "blocksize": state.blocksize, "qtype": state.qtype,
         "double_quant": state.double_quant,
         "codes": state.codes.cpu().numpy(), "absmax": state.absmax.cpu().numpy()}
    if state.double_quant:
        d["absmax_q"] = state.absmax_q.cpu().numpy()
        d["scale2"] = state.scale2.cpu().numpy()
        d["offset"] = state.offset.cpu().numpy()
    return d
