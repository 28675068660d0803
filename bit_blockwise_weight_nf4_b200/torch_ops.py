"""The library's calls as ``bnb4::`` torch operators, and a 4-bit linear
module -- integration glue only: every operator body calls the C ABI through
the binding in ``__init__.py`` (no computation here, no CPU fallback).

* ``torch.ops.bnb4.quantize_4bit(x, blocksize, qtype, double_quant)`` ->
  (codes, absmax, absmax_q, scale2, offset); the last three are empty
  without double quantization.
* ``torch.ops.bnb4.dequantize_4bit(codes, absmax, absmax_q, scale2, offset,
  n, blocksize, qtype, double_quant, out_dtype)`` -> flat tensor of n.
* ``torch.ops.bnb4.gemv_4bit`` / ``gemm_4bit`` (bf16) and ``linear_4bit``
  (bf16 or fp16 with an optional bias): y = x @ What^T for a weight [N, K]
  given by its state tensors.

Each operator has a fake (shape-only) implementation, so graphs that call it
can be traced (torch.compile, export) without running it.  The ossradar
page's release notes describe registering the 4-bit ops with torch.library
for torch.compile; the icman guide describes the Linear4bit module whose
weight is quantized when the module is moved to the GPU.
"""
from typing import Optional, Tuple

import torch

from . import (BF16, F16, NF4, QState, _check, _stream, bnb_dequantize_4bit, bnb_gemm_4bit,
               bnb_gemv_4bit, bnb_linear_4bit, bnb_quantize_4bit, bnb_quantize_4bit_2d,
               workspace_for, QuantState)

Tensor = torch.Tensor
_DTYPES = {torch.float32: 0, torch.bfloat16: BF16, torch.float16: F16}


def _n_blocks(n, blocksize):
    return (n + blocksize - 1) // blocksize


def _qstate(codes, absmax, absmax_q, scale2, offset, n, blocksize, qtype, double_quant):
    p = lambda t: t.data_ptr() if t is not None and t.numel() > 0 else None
    return QState(p(codes), p(absmax), p(absmax_q), p(scale2), p(offset), n, blocksize,
                  qtype, int(bool(double_quant)), 0)


# ------------------------------------------------------------------ quantize
@torch.library.custom_op("bnb4::quantize_4bit", mutates_args=())
def quantize_4bit(x: Tensor, blocksize: int, qtype: int,
                  double_quant: bool) -> Tuple[Tensor, Tensor, Tensor, Tensor, Tensor]:
    dt = _DTYPES.get(x.dtype)
    if dt is None:
        raise TypeError("bnb4::quantize_4bit takes float32, bfloat16 or float16")
    device = x.device if x.is_cuda else torch.device("cuda")
    st = QuantState(x.numel(), blocksize, qtype, double_quant, device)
    ws = workspace_for(st)
    wsp, wsb = (None, 0) if ws is None else (ws.data_ptr(), ws.numel())
    if x.is_contiguous():
        rc = bnb_quantize_4bit(x.data_ptr(), dt, st.cstruct(), wsp, wsb, _stream())
    elif x.dim() == 2 and x.stride(1) == 1:
        rc = bnb_quantize_4bit_2d(x.data_ptr(), dt, x.shape[0], x.shape[1], x.stride(0),
                                  st.cstruct(), wsp, wsb, _stream())
    else:
        raise ValueError("bnb4::quantize_4bit takes a contiguous tensor or a row-strided 2-D view")
    _check(rc, "bnb4::quantize_4bit")
    if double_quant:
        return st.codes, st.absmax, st.absmax_q, st.scale2, st.offset
    # three distinct empty outputs (operator outputs may not alias each other)
    empty = lambda dt: torch.empty(0, dtype=dt, device=device)
    return st.codes, st.absmax, empty(torch.uint8), empty(torch.float32), empty(torch.float32)


@quantize_4bit.register_fake
def _(x, blocksize, qtype, double_quant):
    n = x.numel()
    nb = _n_blocks(n, blocksize)
    dev = x.device if x.device.type != "cpu" else torch.device("cuda")
    u8 = lambda k: x.new_empty(k, dtype=torch.uint8, device=dev)
    f32 = lambda k: x.new_empty(k, dtype=torch.float32, device=dev)
    if double_quant:
        return u8((n + 1) // 2), f32(nb), u8(nb), f32(_n_blocks(nb, 256)), f32(1)
    return u8((n + 1) // 2), f32(nb), u8(0), f32(0), f32(0)


# ---------------------------------------------------------------- dequantize
@torch.library.custom_op("bnb4::dequantize_4bit", mutates_args=())
def dequantize_4bit(codes: Tensor, absmax: Tensor, absmax_q: Tensor, scale2: Tensor,
                    offset: Tensor, n: int, blocksize: int, qtype: int, double_quant: bool,
                    out_dtype: torch.dtype) -> Tensor:
    dt = _DTYPES.get(out_dtype)
    if dt is None:
        raise TypeError("bnb4::dequantize_4bit writes float32, bfloat16 or float16")
    out = torch.empty(n, dtype=out_dtype, device=codes.device)
    st = _qstate(codes, absmax, absmax_q, scale2, offset, n, blocksize, qtype, double_quant)
    _check(bnb_dequantize_4bit(st, out.data_ptr(), dt, _stream()), "bnb4::dequantize_4bit")
    return out


@dequantize_4bit.register_fake
def _(codes, absmax, absmax_q, scale2, offset, n, blocksize, qtype, double_quant, out_dtype):
    return codes.new_empty(n, dtype=out_dtype)


# --------------------------------------------------------------- linear ops
def _linear_out(x, N):
    return torch.empty(x.shape[0], N, dtype=x.dtype, device=x.device)


@torch.library.custom_op("bnb4::gemv_4bit", mutates_args=())
def gemv_4bit(x: Tensor, codes: Tensor, absmax: Tensor, absmax_q: Tensor, scale2: Tensor,
              offset: Tensor, N: int, blocksize: int, qtype: int, double_quant: bool) -> Tensor:
    B, K = x.shape
    y = _linear_out(x, N)
    st = _qstate(codes, absmax, absmax_q, scale2, offset, N * K, blocksize, qtype, double_quant)
    _check(bnb_gemv_4bit(x.data_ptr(), B, K, st, N, y.data_ptr(), _stream()), "bnb4::gemv_4bit")
    return y


@torch.library.custom_op("bnb4::gemm_4bit", mutates_args=())
def gemm_4bit(x: Tensor, codes: Tensor, absmax: Tensor, absmax_q: Tensor, scale2: Tensor,
              offset: Tensor, N: int, blocksize: int, qtype: int, double_quant: bool) -> Tensor:
    M, K = x.shape
    y = _linear_out(x, N)
    st = _qstate(codes, absmax, absmax_q, scale2, offset, N * K, blocksize, qtype, double_quant)
    _check(bnb_gemm_4bit(x.data_ptr(), M, K, st, N, y.data_ptr(), _stream()), "bnb4::gemm_4bit")
    return y


@torch.library.custom_op("bnb4::linear_4bit", mutates_args=())
def linear_4bit(x: Tensor, codes: Tensor, absmax: Tensor, absmax_q: Tensor, scale2: Tensor,
                offset: Tensor, N: int, blocksize: int, qtype: int, double_quant: bool,
                bias: Optional[Tensor]) -> Tensor:
    dt = {torch.bfloat16: BF16, torch.float16: F16}.get(x.dtype)
    if dt is None:
        raise TypeError("bnb4::linear_4bit takes bfloat16 or float16 activations")
    M, K = x.shape
    y = _linear_out(x, N)
    st = _qstate(codes, absmax, absmax_q, scale2, offset, N * K, blocksize, qtype, double_quant)
    rc = bnb_linear_4bit(x.data_ptr(), dt, M, K, st, N,
                         None if bias is None else bias.data_ptr(), y.data_ptr(), _stream())
    _check(rc, "bnb4::linear_4bit")
    return y


for _op in (gemv_4bit, gemm_4bit):
    @_op.register_fake
    def _(x, codes, absmax, absmax_q, scale2, offset, N, blocksize, qtype, double_quant):
        return x.new_empty(x.shape[0], N)


@linear_4bit.register_fake
def _(x, codes, absmax, absmax_q, scale2, offset, N, blocksize, qtype, double_quant, bias):
    return x.new_empty(x.shape[0], N)


# ------------------------------------------------------------------- module
class Linear4bit(torch.nn.Module):
    """y = x @ W^T + b with W stored 4-bit (NF4 or FP4, blockwise, optionally
    double-quantized).  The weight is held in full precision until the
    module is moved to a CUDA device, which quantizes it there (the icman
    guide's Linear4bit behaviour) and drops the full-precision copy; the
    forward pass runs the fused 4-bit linear in ``compute_dtype`` (bf16 or
    fp16) with the bias fused in."""

    def __init__(self, in_features, out_features, bias=True, qtype=NF4, blocksize=64,
                 double_quant=True, compute_dtype=torch.bfloat16):
        super().__init__()
        if compute_dtype not in (torch.bfloat16, torch.float16):
            raise TypeError("compute_dtype must be bfloat16 or float16")
        self.in_features, self.out_features = in_features, out_features
        self.qtype, self.blocksize, self.double_quant = qtype, blocksize, bool(double_quant)
        self.compute_dtype = compute_dtype
        self.weight = torch.nn.Parameter(
            torch.empty(out_features, in_features, dtype=compute_dtype), requires_grad=False)
        self.bias = torch.nn.Parameter(torch.zeros(out_features, dtype=compute_dtype),
                                       requires_grad=False) if bias else None
        for name in ("codes", "absmax", "absmax_q", "scale2", "offset"):
            self.register_buffer(name, None)

    @property
    def quantized(self):
        return self.codes is not None

    def quantize_(self):
        """Quantize the full-precision weight (on the GPU or in page-locked
        host memory) into the 4-bit state buffers and drop it."""
        codes, absmax, absmax_q, scale2, offset = torch.ops.bnb4.quantize_4bit(
            self.weight.detach(), self.blocksize, self.qtype, self.double_quant)
        self.codes, self.absmax, self.absmax_q = codes, absmax, absmax_q
        self.scale2, self.offset = scale2, offset
        self.weight = None
        return self

    def _apply(self, fn, recurse=True):
        super()._apply(fn, recurse)
        if self.weight is not None and self.weight.is_cuda:
            self.quantize_()
        return self

    def forward(self, x):
        if not self.quantized:
            raise RuntimeError("Linear4bit: move the module to a CUDA device to quantize it")
        shape = x.shape
        x2 = x.reshape(-1, self.in_features).to(self.compute_dtype).contiguous()
        bias = None if self.bias is None else self.bias.to(self.compute_dtype)
        y = torch.ops.bnb4.linear_4bit(x2, self.codes, self.absmax, self.absmax_q, self.scale2,
                                       self.offset, self.out_features, self.blocksize,
                                       self.qtype, self.double_quant, bias)
        return y.reshape(*shape[:-1], self.out_features)

    def extra_repr(self):
        return "in_features=%d, out_features=%d, qtype=%s, blocksize=%d, double_quant=%s" % (
            self.in_features, self.out_features, "nf4" if self.qtype == NF4 else "fp4",
            self.blocksize, self.double_quant)
