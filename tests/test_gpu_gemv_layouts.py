"""Decode GEMV load forms and the 9-16-row form, against the fp64 oracle.

With x and the packed codes 32-byte aligned, the decode kernel reads both
with 256-bit loads and also takes 9 to 16 rows of x (x as the MMA's A
operand, each weight row the B operand); with either one only 16-byte
aligned (the API's minimum) it reads them with 128-bit loads, and 9 to 16
rows go to the small-batch kernel instead.  Every form is checked with the
linear tolerance of the other decode tests (parity.check_linear)."""
import copy

import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


def offset_copy(t, off):
    """A copy of the 1-D device tensor ``t`` whose data pointer is ``off``
    bytes past a 32-byte boundary (off a multiple of the element size)."""
    es = t.element_size()
    buf = torch.empty(t.numel() + 64 // es, dtype=t.dtype, device=t.device)
    lead = ((off - buf.data_ptr() % 32) % 32) // es
    v = buf[lead:lead + t.numel()]
    v.copy_(t)
    assert v.data_ptr() % 32 == off
    return v


def make(N, K, bs=64, qtype=bnb4.NF4, dq=True, seed=0):
    W = synth.weight_bf16(N, K, seed=seed)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), bs, qtype, dq)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    return bnb4.state_from_arrays(st), What


def run(B, N, K, x_off=0, codes_off=0, seed=0, **fmt):
    g, What = make(N, K, seed=seed, **fmt)
    if codes_off:
        g = copy.copy(g)
        g.codes = offset_copy(g.codes, codes_off)
    x = synth.activations_bf16(B, K, seed=seed + 1)
    xd = x.cuda()
    if x_off:
        xd = offset_copy(xd.view(-1), x_off).view(B, K)
    y = bnb4.gemv_4bit(xd, g, N)
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x)
    check_linear(cpu_bits(y), oracle.linear_ref(xb, What), xb, What)
    return y


@pytest.mark.parametrize("B", [9, 12, 16])
@pytest.mark.parametrize("N,K", [(1030, 4096), (257, 1088), (16, 64)])
def test_rows_9_to_16(B, N, K):
    """The 16-row form: ragged N (a partial row group), several K steps, a
    single step."""
    run(B, N, K, seed=B + N)


@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008)])
def test_rows_16_llama_mlp(N, K):
    run(16, N, K, seed=N)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
def test_rows_9_to_16_every_format(qtype, bs, dq):
    run(13, 264, 1280, bs=bs, qtype=qtype, dq=dq, seed=bs + int(dq))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_rows_9_to_16_bias(dtype):
    """The fp16 / bf16 linear with a fused bias through the 16-row form."""
    tdt, odt = {"bf16": (torch.bfloat16, oracle.BF16), "f16": (torch.float16, oracle.F16)}[dtype]
    M, N, K = 11, 264, 1280
    W = synth.weight_bf16(N, K, seed=5).to(tdt)
    x = synth.activations_bf16(M, K, seed=6).to(tdt)
    bias = synth.normal_f32((N,), seed=7, std=1.0).to(tdt)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    st = oracle.quantize(W.view(-1).numpy() if dtype == "f16" else bits(W).reshape(-1),
                         64, bnb4.NF4, True)
    What = oracle.dequantize(st, odt).reshape(N, K)
    y64 = oracle.linear_ref(bits(x), What, dtype=odt, bias_bits=bits(bias))
    y = bnb4.linear_4bit(x.cuda(), bnb4.state_from_arrays(st), N, bias=bias.cuda())
    torch.cuda.synchronize()
    check_linear(cpu_bits(y), y64, bits(x), What, dtype=odt)


@pytest.mark.parametrize("B", [1, 8, 12])
@pytest.mark.parametrize("which", ["x", "codes", "both"])
def test_16_byte_aligned_inputs(B, which):
    """x and / or the codes 16-byte but not 32-byte aligned: the 128-bit load
    form (B <= 8) or the small-batch kernel (B = 12)."""
    run(B, 1030, 4096, x_off=16 if which != "codes" else 0,
        codes_off=16 if which != "x" else 0, seed=40 + B)


@pytest.mark.parametrize("B", [9, 16])
def test_load_forms_agree(B):
    """The same weight and x through both load forms of the B <= 8 kernel
    (bit-identical: the loads differ, not the arithmetic) and, at 9-16 rows,
    the 16-row form against the small-batch kernel (within tolerance)."""
    N, K = 1030, 4096
    g, What = make(N, K, seed=B)
    x = synth.activations_bf16(B, K, seed=B + 1).cuda()
    y_fast = bnb4.gemv_4bit(x, g, N)
    y_small = bnb4.gemv_4bit(offset_copy(x.view(-1), 16).view(B, K), g, N)
    for b in (1, 8):
        a = bnb4.gemv_4bit(x[:b].contiguous(), g, N)
        c = bnb4.gemv_4bit(offset_copy(x[:b].contiguous().view(-1), 16).view(b, K), g, N)
        assert torch.equal(a, c)
    torch.cuda.synchronize()
    d = (y_fast.float() - y_small.float()).norm() / y_small.float().norm()
    assert d.item() < 2e-3
