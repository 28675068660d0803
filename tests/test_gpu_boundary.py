"""Every entry point refuses memory a kernel cannot dereference.

A pageable host pointer (a plain CPU tensor) handed to any call must come
back as BNB4_ERR_INVALID_ARG with nothing launched, as include/bnb4.h
promises.  Each refused call is made while the stream is being captured
into a CUDA graph that is never replayed: the call returns the status the
same way, and if a check ever stopped working, the kernel it let through
would only be recorded, never run on the device.
"""
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def weight():
    """A device NF4 state of a [256, 512] weight (double quant) and a warm
    library: one real call of each kind before any capture."""
    w = synth.weight_bf16(256, 512, seed=3).cuda()
    st = bnb4.quantize_4bit(w, 64, bnb4.NF4, True)
    x = torch.ones(4, 512, dtype=torch.bfloat16, device="cuda")
    bnb4.linear_4bit(x, st, 256)
    bnb4.gemm_4bit(torch.ones(512, 512, dtype=torch.bfloat16, device="cuda"), st, 256)
    bnb4.dequantize_4bit(st, torch.bfloat16)
    torch.cuda.synchronize()
    return st


def refused(call):
    """Run call(stream) while the stream is captured into a graph that is
    dropped without replay; return the call's status."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
            rc = call(s.cuda_stream)
    del g  # never replayed
    torch.cuda.synchronize()
    return rc


def host(*shape, dtype=torch.bfloat16):
    t = torch.zeros(*shape, dtype=dtype)
    assert t.device.type == "cpu" and not t.is_pinned()
    return t


@pytest.mark.parametrize("M", [1, 16, 512])
def test_linear_entries_refuse_pageable_activations(weight, M):
    st = weight.cstruct()
    K, N = 512, 256
    xd = torch.ones(M, K, dtype=torch.bfloat16, device="cuda")
    yd = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    xh, yh, bh = host(M, K), host(M, N), host(N)
    calls = [
        lambda s: bnb4.bnb_gemm_4bit(xh.data_ptr(), M, K, st, N, yd.data_ptr(), s),
        lambda s: bnb4.bnb_gemm_4bit(xd.data_ptr(), M, K, st, N, yh.data_ptr(), s),
        lambda s: bnb4.bnb_linear_4bit(xd.data_ptr(), bnb4.BF16, M, K, st, N,
                                       bh.data_ptr(), yd.data_ptr(), s),
    ]
    if M <= 256:
        calls.append(lambda s: bnb4.bnb_gemv_4bit(xh.data_ptr(), M, K, st, N,
                                                  yd.data_ptr(), s))
    for call in calls:
        assert refused(call) == bnb4.ERR_INVALID_ARG
    assert bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == bnb4.OK


def test_linear_entries_refuse_pageable_weight_arrays(weight):
    M, K, N = 4, 512, 256
    xd = torch.ones(M, K, dtype=torch.bfloat16, device="cuda")
    yd = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    codes_h = host(weight.codes.numel(), dtype=torch.uint8)
    aq_h = host(weight.absmax_q.numel(), dtype=torch.uint8)
    for field, t in (("codes", codes_h), ("absmax_q", aq_h)):
        st = weight.cstruct()
        setattr(st, field, t.data_ptr())
        rc = refused(lambda s: bnb4.bnb_linear_4bit(xd.data_ptr(), bnb4.BF16, M, K, st, N,
                                                    None, yd.data_ptr(), s))
        assert rc == bnb4.ERR_INVALID_ARG, field


def test_dequantize_refuses_pageable_output(weight):
    out_h = host(weight.n)
    assert refused(lambda s: bnb4.bnb_dequantize_4bit(
        weight.cstruct(), out_h.data_ptr(), bnb4.BF16, s)) == bnb4.ERR_INVALID_ARG
    assert refused(lambda s: bnb4.bnb_dequantize_4bit_2d(
        weight.cstruct(), out_h.data_ptr(), bnb4.BF16, 256, 512, 512, s)) == \
        bnb4.ERR_INVALID_ARG


def test_quantize_refuses_pageable_outputs(weight):
    w = synth.weight_bf16(256, 512, seed=4).cuda()
    ws = bnb4.workspace_for(weight)
    codes_h = host(weight.codes.numel(), dtype=torch.uint8)
    st = weight.cstruct()
    st.codes = codes_h.data_ptr()
    assert refused(lambda s: bnb4.bnb_quantize_4bit(
        w.data_ptr(), bnb4.BF16, st, ws.data_ptr(), ws.numel(), s)) == bnb4.ERR_INVALID_ARG


def test_noalloc_refuses_pageable_input(weight):
    """The allocation-free quantize applies the same memory rules as the
    regular one (the pointer query allocates nothing)."""
    xh = host(256 * 512)
    st = weight.cstruct()
    st.absmax = None
    assert refused(lambda s: bnb4.bnb_quantize_4bit_noalloc(
        xh.data_ptr(), bnb4.BF16, st, s)) == bnb4.ERR_INVALID_ARG
