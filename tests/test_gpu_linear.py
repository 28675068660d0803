"""GPU parity of bnb_linear_4bit -- the fused 4-bit linear layer in both
16-bit compute types (bf16, fp16) with an optional fused bias -- against the
fp64 oracle over the weight dequantized in that compute type, with the
tolerance of the method's brief.  Every kernel tier is reached: the decode
kernel (M <= 8, and 9..16 rows with x and the codes 32-byte aligned, as
here), the small-batch kernel (up to 256) and the prefill kernel."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu

DT = {"bf16": (torch.bfloat16, oracle.BF16), "f16": (torch.float16, oracle.F16)}


def status_ok():
    torch.cuda.synchronize()
    return bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == 0


def case(M, N, K, dtype, with_bias, bs=64, qtype=bnb4.NF4, dq=True, seed=0, n_rows=None):
    tdt, odt = DT[dtype]
    W = synth.weight_bf16(N, K, seed=seed).to(tdt)
    x = synth.activations_bf16(M, K, seed=seed + 1).to(tdt)
    bias = (synth.normal_f32((N,), seed=seed + 2, std=1.0).to(tdt) if with_bias else None)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    st = oracle.quantize(W.view(-1).numpy() if dtype == "f16" else bits(W).reshape(-1),
                         bs, qtype, dq)
    What = oracle.dequantize(st, odt).reshape(N, K)
    rows = None
    if n_rows is not None and n_rows < M:
        rng = np.random.default_rng(seed)
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, n_rows - 2, replace=False)]))
    y64 = oracle.linear_ref(bits(x), What, rows=rows, dtype=odt,
                            bias_bits=None if bias is None else bits(bias))
    g = bnb4.state_from_arrays(st)
    y = bnb4.linear_4bit(x.cuda(), g, N, bias=None if bias is None else bias.cuda())
    assert status_ok()
    yb = cpu_bits(y)
    if rows is not None:
        yb = yb[rows]
    return check_linear(yb, y64, bits(x), What, rows=rows, dtype=odt)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("M", [1, 5, 8, 9, 40, 256, 257, 600])
def test_every_tier(dtype, with_bias, M):
    """Decode (1, 5, 8, 9 rows), small-batch (40, 256) and prefill (257, 600)
    kernels, ragged N (3 weight-row tiles of the small kernel, partial pair
    tiles of the prefill kernel) and several K steps."""
    case(M, 264 if M <= 256 else 520, 1280 if M <= 256 else 1024, dtype, with_bias,
         seed=M + 17 * int(with_bias))


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128])
@pytest.mark.parametrize("dq", [True, False])
@pytest.mark.parametrize("M", [3, 33, 300])
def test_fp16_every_format(qtype, bs, dq, M):
    """The fp16 tables (two per K step at blocksize 32, nested scales decoded
    in each kernel) in each tier, with a bias."""
    case(M, 136 if M <= 256 else 264, 640, "f16", True, bs, qtype, dq, seed=bs + M + qtype)


@pytest.mark.parametrize("N,K", synth.GEMM_SHAPES)
@pytest.mark.parametrize("M", [1, 16, 2048])
def test_llama_shapes_fp16_bias(N, K, M):
    """Llama-7B projection shapes in fp16 with a bias: decode, batch 16 and a
    2048-token prefill (checked on 48 sampled rows)."""
    case(M, N, K, "f16", True, seed=N + K + M, n_rows=48 if M > 64 else None)


@pytest.mark.parametrize("M", [4, 64, 512])
def test_bf16_without_bias_equals_gemm_entry(M):
    """With bf16 and no bias the linear entry runs the same kernel as
    bnb_gemm_4bit: the outputs agree bit for bit."""
    W = synth.weight_bf16(1024, 2048, seed=M).cuda().view(-1)
    st = bnb4.quantize_4bit(W, 64, bnb4.NF4, True)
    x = synth.activations_bf16(M, 2048, seed=M + 1).cuda()
    a = bnb4.linear_4bit(x, st, 1024)
    b = bnb4.gemm_4bit(x, st, 1024)
    assert status_ok()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_fp16_overflowing_weights_become_infinite():
    """fp16 dequantized weights past 65504 round to infinity (the IEEE
    rounding the oracle follows), on the GPU as in the oracle."""
    N, K = 64, 128
    W = torch.full((N, K), 1.0e5, dtype=torch.float32)
    st = bnb4.quantize_4bit(W.cuda().view(-1), 64, bnb4.NF4, False)
    w16 = bnb4.dequantize_4bit(st, torch.float16).cpu()
    assert torch.isinf(w16).all()
    orc = oracle.dequantize(oracle.quantize(W.view(-1).numpy(), 64, bnb4.NF4, False),
                            oracle.F16)
    assert np.array_equal(cpu_bits(w16), orc)
