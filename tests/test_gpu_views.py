"""GPU parity for non-contiguous inputs and outputs and for quantize-on-load
(release notes 0.49.2: quantize / dequantize handle non-contiguous tensors;
the icman guide: bf16 / fp16 weights are quantized as they move to the
GPU).  A row-strided 2-D view quantizes bit for bit like its contiguous copy
does in the oracle; page-locked host memory is read by the kernel directly;
pageable host memory is refused before anything runs; dequantization into
a row-strided view writes exactly the view."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import GuardedState, assert_state_equal, cpu_bits

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
C_DT = {"f32": bnb4.F32, "bf16": bnb4.BF16, "f16": bnb4.F16}


def status_ok():
    torch.cuda.synchronize()
    return bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == 0


def host_for_oracle(t):
    """numpy array the oracle quantizes (fp32, bf16 bits or fp16)."""
    t = t.contiguous().view(-1)
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits(t)
    return t.numpy()


def wide(rows, ld, dtype, seed):
    """[rows, ld] tensor ~ N(0, 0.02^2) with a few x20 outliers."""
    x = synth.normal_f32((rows, ld), seed=seed, std=0.02)
    x.view(-1)[::997] *= 20.0
    return x.to(TORCH_DT[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("rows,cols,ld", [(37, 1344, 1408),   # blocks of 256 span rows
                                          (5, 72, 80),        # blocks of 64 span rows
                                          (1, 256, 264),
                                          (300, 4104, 4112),  # several tiles, ragged tail
                                          (96, 11008, 11264)])
@pytest.mark.parametrize("bs", [64, 256])
def test_quantize_row_strided_view(dtype, rows, cols, ld, bs):
    full = wide(rows, ld, dtype, seed=rows + cols + bs)
    x = full[:, :cols]
    orc = oracle.quantize(host_for_oracle(x), bs, oracle.NF4, True)
    g = GuardedState(rows * cols, bs, bnb4.NF4, True)
    xd = full.cuda()[:, :cols]  # the same view on the device: rows ld elements apart
    assert xd.stride(0) == ld
    rc = bnb4.bnb_quantize_4bit_2d(xd.data_ptr(), C_DT[dtype], rows, cols, ld, g.cstruct(),
                                   g.workspace.data_ptr(), g.workspace.numel(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == 0, bnb4.bnb4_strerror(rc)
    assert status_ok()
    assert_state_equal(g.arrays(), orc, True)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("dq", [True, False])
def test_quantize_view_fp4_and_plain_absmax(qtype, dq):
    full = wide(64, 1088, "bf16", seed=5 + qtype)
    x = full[:, :1024]
    st = bnb4.quantize_4bit(full.cuda()[:, :1024], 64, qtype, dq)
    assert status_ok()
    orc = oracle.quantize(host_for_oracle(x), 64, qtype, dq)
    got = bnb4.state_to_arrays(st)
    assert_state_equal(got, orc, dq)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("n", [4096 * 4096 + 40, 100003])
def test_quantize_on_load_from_pinned_host(dtype, n):
    """The kernel reads a page-locked host tensor over the bus: the state
    equals the oracle's and that of quantizing a device copy."""
    x = synth.normal_f32((n,), seed=n, std=0.02).to(TORCH_DT[dtype]).pin_memory()
    st_host = bnb4.quantize_4bit(x, 64, bnb4.NF4, True)
    st_dev = bnb4.quantize_4bit(x.cuda(), 64, bnb4.NF4, True)
    assert status_ok()
    orc = oracle.quantize(host_for_oracle(x), 64, oracle.NF4, True)
    a, b = bnb4.state_to_arrays(st_host), bnb4.state_to_arrays(st_dev)
    assert_state_equal(a, orc, True)
    assert_state_equal(b, orc, True)


def test_quantize_on_load_strided_pinned_view():
    """A row-strided view of a page-locked host checkpoint."""
    x = wide(200, 2112, "bf16", seed=77).pin_memory()[:, :2048]
    st = bnb4.quantize_4bit(x, 64, bnb4.NF4, True)
    assert status_ok()
    orc = oracle.quantize(host_for_oracle(x), 64, oracle.NF4, True)
    assert_state_equal(bnb4.state_to_arrays(st), orc, True)


def test_pageable_host_input_is_refused():
    """Memory the device cannot address is refused with INVALID_ARG and
    nothing is launched (the device stays healthy)."""
    x = synth.normal_f32((4096,), seed=1, std=0.02).to(torch.bfloat16)
    assert not x.is_pinned()
    st = bnb4.QuantState(4096, 64, bnb4.NF4, True)
    ws = bnb4.workspace_for(st)
    rc = bnb4.bnb_quantize_4bit(x.data_ptr(), bnb4.BF16, st.cstruct(), ws.data_ptr(),
                                ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == bnb4.ERR_INVALID_ARG
    rc = bnb4.bnb_quantize_4bit_2d(x.data_ptr(), bnb4.BF16, 64, 64, 64, st.cstruct(),
                                   ws.data_ptr(), ws.numel(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == bnb4.ERR_INVALID_ARG
    assert status_ok()
    with pytest.raises(ValueError, match="page-locked"):
        bnb4.quantize_4bit(x)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("rows,cols,ld", [(37, 1344, 1408), (3, 72, 96), (130, 4104, 4128)])
def test_dequantize_into_row_strided_view(dtype, rows, cols, ld):
    """Element (r, c) of the view receives logical element r * cols + c,
    bit-equal to the oracle; the gap columns between the rows keep their
    canary bytes."""
    x = synth.normal_f32((rows * cols,), seed=rows + ld, std=0.02).numpy()
    orc = oracle.quantize(x, 64, oracle.FP4, True)
    odt = {"f32": oracle.F32, "bf16": oracle.BF16, "f16": oracle.F16}[dtype]
    want = oracle.dequantize(orc, odt).reshape(rows, cols)
    g = bnb4.state_from_arrays(orc)
    buf = torch.full((rows, ld), -3.0, dtype=TORCH_DT[dtype], device="cuda")
    out = bnb4.dequantize_4bit(g, out=buf[:, :cols])
    assert status_ok()
    got = out.cpu()
    if dtype == "f32":
        assert got.contiguous().numpy().tobytes() == want.tobytes()
    else:
        assert np.array_equal(cpu_bits(got), want)
    assert torch.all(buf[:, cols:].cpu() == -3.0)
