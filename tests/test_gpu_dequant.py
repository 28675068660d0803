"""GPU parity of bnb_dequantize_4bit against the CPU oracle, bit for bit, in
fp32, bf16 and fp16, on a state the oracle computed (uploaded), and end to end
(GPU quantize then GPU dequantize vs oracle quantize then oracle
dequantize)."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import CANARY, GUARD, cpu_bits

pytestmark = pytest.mark.gpu


def gpu_dequant(state, n, out_dtype):
    elt = 4 if out_dtype == bnb4.F32 else 2
    buf = torch.full((n * elt + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
    rc = bnb4.bnb_dequantize_4bit(state.cstruct(), buf.data_ptr(), out_dtype,
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0, bnb4.bnb4_strerror(rc)
    host = buf.cpu().numpy()
    assert np.all(host[n * elt:] == CANARY), "write past the end of the output"
    return host[:n * elt].view(np.float32 if out_dtype == bnb4.F32 else np.uint16)


@pytest.mark.parametrize("out_dtype", [bnb4.F32, bnb4.BF16, bnb4.F16])
@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
@pytest.mark.parametrize("n", [1, 3, 64, 65, 1023, 4097, 100003])
def test_dequantize_oracle_state(out_dtype, qtype, bs, dq, n):
    x = synth.normal_f32((n,), seed=7 * n + bs, std=0.02).numpy()
    st = oracle.quantize(x, bs, qtype, dq)
    want = oracle.dequantize(st, out_dtype)
    g = bnb4.state_from_arrays(st)
    got = gpu_dequant(g, n, out_dtype)
    assert got.tobytes() == want.tobytes()


def test_roundtrip_vector_1m_end_to_end():
    """Quantize then dequantize the 2^20 fp32 vector (seed 0, bs 64, double
    quant) on the GPU; compare with the oracle doing the same."""
    x = synth.normal_f32((synth.ROUNDTRIP_N,), seed=0, std=0.02)
    orc = oracle.quantize(x.numpy(), 64, bnb4.NF4, True)
    want = oracle.dequantize(orc, oracle.F32)
    st = bnb4.quantize_4bit(x.cuda(), 64, bnb4.NF4, True)
    got = bnb4.dequantize_4bit(st, torch.float32).cpu().numpy()
    assert got.tobytes() == want.tobytes()


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
def test_matrix_4096_end_to_end_bf16(qtype):
    W = synth.weight_bf16(4096, 4096, seed=1000, outlier_frac=synth.OUTLIER_FRAC)
    orc = oracle.quantize(synth.bf16_bits(W.view(-1)), 64, qtype, True)
    want = oracle.dequantize(orc, oracle.BF16)
    st = bnb4.quantize_4bit(W.cuda().view(-1), 64, qtype, True)
    got = cpu_bits(bnb4.dequantize_4bit(st, torch.bfloat16))
    assert got.tobytes() == want.tobytes()


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
def test_matrix_4096_end_to_end_f16(qtype):
    """The fp16 compute type: an fp16 weight quantized and dequantized to fp16
    on the GPU equals the oracle doing the same, bit for bit."""
    W = synth.weight_bf16(4096, 4096, seed=1001, outlier_frac=synth.OUTLIER_FRAC)
    W = W.to(torch.float16)
    orc = oracle.quantize(W.view(-1).numpy(), 64, qtype, True)
    want = oracle.dequantize(orc, oracle.F16)
    st = bnb4.quantize_4bit(W.cuda().view(-1), 64, qtype, True)
    got = cpu_bits(bnb4.dequantize_4bit(st, torch.float16))
    assert got.tobytes() == want.tobytes()
