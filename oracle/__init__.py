"""CPU oracle for 4-bit blockwise NF4 / FP4 quantization (TEST INFRASTRUCTURE).

A thin numpy/ctypes wrapper around ``bnb4_oracle.c`` -- a plain, slow,
single-threaded C implementation of what the GPU path computes.  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package; the product library never does, and the two share no
code.  The method, the page citations and every reading taken where the pages
are silent are written out in the header comment of ``bnb4_oracle.c``.

Arrays are numpy.  bf16 data travels as ``np.uint16`` bit patterns, fp16
data as ``np.float16`` (or its ``np.uint16`` bit patterns where stated).
"""
import ctypes
import os

import numpy as np

from . import build as _build

NF4 = 0
FP4 = 1
F32 = 0
BF16 = 1
F16 = 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        lib.orc_codebook.argtypes = [i32, p]
        lib.orc_bf16_rne.argtypes = [ctypes.c_float]
        lib.orc_bf16_rne.restype = ctypes.c_uint16
        lib.orc_f16_rne.argtypes = [ctypes.c_float]
        lib.orc_f16_rne.restype = ctypes.c_uint16
        lib.orc_f16_to_float.argtypes = [ctypes.c_uint16]
        lib.orc_f16_to_float.restype = ctypes.c_float
        lib.orc_nearest_code.argtypes = [i32, ctypes.c_float]
        lib.orc_quantize_4bit.argtypes = [p, i32, i64, i32, i32, i32,
                                          p, p, p, p, p, p]
        lib.orc_dequantize_4bit.argtypes = [p, i64, i32, i32, i32,
                                            p, p, p, p, p, i32]
        lib.orc_linear_ref.argtypes = [p, i32, i64, i64, p, i64, p, i64, p, i64,
                                       p, p]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments (status %d)" % (what, rc))


def codebook(qtype):
    """The 16 fp32 dequantization values, indexed by the 4-bit code."""
    out = np.zeros(16, np.float32)
    _check(_load().orc_codebook(qtype, _ptr(out)), "codebook")
    return out


def bf16_rne(f):
    """bf16 bit pattern of fp32 value ``f`` (round to nearest even)."""
    return int(_load().orc_bf16_rne(ctypes.c_float(f)))


def f16_rne(f):
    """IEEE binary16 bit pattern of fp32 value ``f`` (round to nearest even)."""
    return int(_load().orc_f16_rne(ctypes.c_float(f)))


def f16_to_float(h):
    """Exact fp32 value of binary16 bit pattern ``h``."""
    return float(_load().orc_f16_to_float(ctypes.c_uint16(h)))


def nearest_code(qtype, v):
    """Code of one normalised fp32 value."""
    return int(_load().orc_nearest_code(qtype, ctypes.c_float(v)))


def n_blocks(n, blocksize):
    return (n + blocksize - 1) // blocksize


def quantize(x, blocksize=64, qtype=NF4, double_quant=True):
    """Quantize a flat fp32 array, bf16 bit-pattern (uint16) array or fp16
    (float16) array.

    Returns a dict with ``codes`` (uint8, ceil(n/2)), ``absmax`` (fp32, nb),
    and for double quant ``absmax_q`` (uint8, nb), ``scale2`` (fp32,
    ceil(nb/256)), ``offset`` (fp32, 1) and ``sum_exact`` (the absmax mean is
    independent of summation order).
    """
    x = np.ascontiguousarray(x).reshape(-1)
    if x.dtype == np.float32:
        xd = F32
    elif x.dtype == np.uint16:
        xd = BF16
    elif x.dtype == np.float16:
        xd = F16
        x = x.view(np.uint16)
    else:
        raise TypeError("oracle quantize takes float32, uint16 (bf16 bits) or float16")
    n = x.size
    nb = n_blocks(n, blocksize)
    st = {"n": n, "blocksize": blocksize, "qtype": qtype,
          "double_quant": bool(double_quant)}
    st["codes"] = np.zeros((n + 1) // 2, np.uint8)
    st["absmax"] = np.zeros(nb, np.float32)
    if double_quant:
        st["absmax_q"] = np.zeros(nb, np.uint8)
        st["scale2"] = np.zeros(n_blocks(nb, 256), np.float32)
        st["offset"] = np.zeros(1, np.float32)
    exact = ctypes.c_int(0)
    rc = _load().orc_quantize_4bit(
        _ptr(x), xd, n, blocksize, qtype, int(bool(double_quant)),
        _ptr(st["codes"]), _ptr(st["absmax"]), _ptr(st.get("absmax_q")),
        _ptr(st.get("scale2")), _ptr(st.get("offset")), ctypes.byref(exact))
    _check(rc, "quantize")
    st["sum_exact"] = bool(exact.value)
    return st


def dequantize(st, out_dtype=F32):
    """Dequantize a state from :func:`quantize` (or one built from GPU
    outputs) to fp32, or to bf16 / fp16 bit patterns (uint16)."""
    n = st["n"]
    out = np.zeros(n, np.float32 if out_dtype == F32 else np.uint16)
    dq = bool(st["double_quant"])
    rc = _load().orc_dequantize_4bit(
        _ptr(np.ascontiguousarray(st["codes"], np.uint8)), n, st["blocksize"],
        st["qtype"], int(dq),
        _ptr(st.get("absmax")) if not dq else None,
        _ptr(st.get("absmax_q")) if dq else None,
        _ptr(st.get("scale2")) if dq else None,
        _ptr(st.get("offset")) if dq else None,
        _ptr(out), out_dtype)
    _check(rc, "dequantize")
    return out


def linear_ref(x_bits, W_bits, rows=None, cols=None, dtype=BF16, bias_bits=None):
    """fp64 y = x . W^T (+ bias) for bit-pattern x [M, K], W [N, K] and bias
    [N] in bf16 (``dtype`` BF16) or fp16 (F16).

    ``rows`` / ``cols`` optionally select a subset of x rows / W rows; the
    result is [len(rows), len(cols)].
    """
    x_bits = np.ascontiguousarray(x_bits).view(np.uint16)
    W_bits = np.ascontiguousarray(W_bits).view(np.uint16)
    M, K = x_bits.shape
    N, K2 = W_bits.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits).view(np.uint16)
    if b is not None and b.size != N:
        raise ValueError("bias must have N entries")
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    c = None if cols is None else np.ascontiguousarray(cols, np.int64)
    nr = M if r is None else r.size
    nc = N if c is None else c.size
    y = np.zeros((nr, nc), np.float64)
    rc = _load().orc_linear_ref(_ptr(x_bits), dtype, M, K, _ptr(r), nr, _ptr(W_bits),
                                N, _ptr(c), nc, _ptr(b), _ptr(y))
    _check(rc, "linear_ref")
    return y


def bf16_bits_to_f64(bits):
    """Exact float64 values of bf16 bit patterns."""
    b = np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits):
    """Exact float64 values of fp16 bit patterns."""
    return np.ascontiguousarray(bits, np.uint16).view(np.float16).astype(np.float64)
