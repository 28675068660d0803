"""The bnb4:: torch operators and the Linear4bit module on the GPU:
torch.library's operator checks (schema, fake implementation against the real
one, no aliasing), a Linear4bit built from an nn.Linear state dict and moved
to the GPU (which quantizes it) against the functional linear on the same
state and the fp64 oracle, and a traced graph calling the operators."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
from bit_blockwise_weight_nf4_b200 import torch_ops
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


def test_opcheck_every_operator():
    W = synth.weight_bf16(256, 512, seed=1).cuda()
    st = torch.ops.bnb4.quantize_4bit(W, 64, bnb4.NF4, True)
    torch.library.opcheck(torch.ops.bnb4.quantize_4bit.default, (W, 64, bnb4.NF4, True))
    torch.library.opcheck(torch.ops.bnb4.quantize_4bit.default, (W.view(-1)[:1000], 32, bnb4.FP4,
                                                                 False))
    torch.library.opcheck(torch.ops.bnb4.dequantize_4bit.default,
                          (*st, 256 * 512, 64, bnb4.NF4, True, torch.bfloat16))
    x1 = synth.activations_bf16(4, 512, seed=2).cuda()
    x2 = synth.activations_bf16(300, 512, seed=3).cuda()
    torch.library.opcheck(torch.ops.bnb4.gemv_4bit.default, (x1, *st, 256, 64, bnb4.NF4, True))
    torch.library.opcheck(torch.ops.bnb4.gemm_4bit.default, (x2, *st, 256, 64, bnb4.NF4, True))
    b = torch.randn(256, dtype=torch.float16, device="cuda")
    torch.library.opcheck(torch.ops.bnb4.linear_4bit.default,
                          (x2.half(), *st, 256, 64, bnb4.NF4, True, b))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M", [3, 40, 300])
def test_linear4bit_module(dtype, M):
    ref = torch.nn.Linear(1024, 520, bias=True)
    with torch.no_grad():
        ref.weight.copy_(synth.normal_f32((520, 1024), seed=M, std=0.02))
        ref.bias.copy_(synth.normal_f32((520,), seed=M + 1, std=1.0))
    m = torch_ops.Linear4bit(1024, 520, compute_dtype=dtype)
    m.load_state_dict({k: v.to(dtype) for k, v in ref.state_dict().items()})
    w_host = m.weight.detach().clone()
    m = m.cuda()
    assert m.quantized and m.weight is None
    x = synth.activations_bf16(M, 1024, seed=M + 2).to(dtype).cuda()
    y = m(x.view(M, 1, 1024)).view(M, 520)
    # the same state through the functional entry, bit for bit
    st = bnb4.QuantState(520 * 1024, 64, bnb4.NF4, True)
    for k in ("codes", "absmax", "absmax_q", "scale2", "offset"):
        getattr(st, k).copy_(getattr(m, k))
    y2 = bnb4.linear_4bit(x, st, 520, bias=m.bias)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    # and the oracle on the weight quantized from the same full-precision values
    odt = oracle.F16 if dtype == torch.float16 else oracle.BF16
    bits = lambda t: t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    host = w_host.view(-1).numpy() if dtype == torch.float16 else bits(w_host).reshape(-1)
    What = oracle.dequantize(oracle.quantize(host, 64, oracle.NF4, True), odt).reshape(520, 1024)
    y64 = oracle.linear_ref(bits(x), What, dtype=odt, bias_bits=bits(m.bias))
    check_linear(cpu_bits(y), y64, bits(x), What, dtype=odt)


def test_traced_graph_calls_the_operators():
    """A function calling the operators traces into one graph (torch.compile
    with the eager backend, fullgraph) and gives the eager result bit for
    bit."""
    W = synth.weight_bf16(384, 1024, seed=7).cuda()
    st = torch.ops.bnb4.quantize_4bit(W, 64, bnb4.NF4, True)
    x = synth.activations_bf16(24, 1024, seed=8).cuda()

    def f(x, codes, absmax, absmax_q, scale2, offset):
        h = torch.ops.bnb4.linear_4bit(x, codes, absmax, absmax_q, scale2, offset, 384, 64,
                                       bnb4.NF4, True, None)
        return torch.relu(h) * 2

    eager = f(x, *st)
    compiled = torch.compile(f, backend="eager", fullgraph=True)(x, *st)
    torch.cuda.synchronize()
    assert torch.equal(eager.view(torch.int16), compiled.view(torch.int16))
