"""Decode GEMVs chained through their outputs on one stream.

Each link reads the output of the link before, as a decoder's linears do.
The chain must give exactly the results of the same links run one at a time
with a synchronisation between them (the kernels are deterministic) --
eagerly, inside a CUDA graph whose first node copies the chain's input in,
and for a decoder layer's grouped lists mixing both decode kernels.  (A
launch that overlaps its predecessor, as a programmatic dependent launch
would, must still pass this.)  The last link is also checked against the
fp64 oracle."""
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu

# (N, K) of consecutive links: each K is the previous link's N
CHAIN = [(4096, 4096), (11008, 4096), (4096, 11008), (1088, 4096), (4096, 1088), (4096, 4096)]


def quantized(shapes, seed):
    out = []
    for i, (N, K) in enumerate(shapes):
        w = synth.weight_bf16(N, K, seed=seed + i, device="cuda")
        out.append(bnb4.quantize_4bit(w.view(-1), 64, bnb4.NF4, True))
    torch.cuda.synchronize()
    return out


def run_chain(x, sts, sync, outs=None):
    ys = []
    for i, (st, (N, _)) in enumerate(zip(sts, CHAIN)):
        x = bnb4.gemv_4bit(x, st, N, out=None if outs is None else outs[i])
        if sync:
            torch.cuda.synchronize()
        ys.append(x)
    return ys


def check_last_link(x_prev, st, y):
    N, K = y.shape[1], x_prev.shape[1]
    What = oracle.dequantize(bnb4.state_to_arrays(st), oracle.BF16).reshape(N, K)
    xb = cpu_bits(x_prev)
    check_linear(cpu_bits(y), oracle.linear_ref(xb, What), xb, What)


@pytest.mark.parametrize("B", [1, 5])
def test_eager_chain_equals_serialised(B):
    sts = quantized(CHAIN, seed=500 + B)
    for trial in range(4):
        x = synth.activations_bf16(B, CHAIN[0][1], seed=600 + trial, device="cuda")
        ref = run_chain(x, sts, sync=True)
        got = run_chain(x, sts, sync=False)
        torch.cuda.synchronize()
        for i, (a, b) in enumerate(zip(got, ref)):
            assert torch.equal(a, b), "link %d differs from the serialised run" % i
    check_last_link(ref[-2], sts[-1], ref[-1])


def test_graph_chain_with_input_copy():
    """The graph's first node is a copy into the chain's input buffer; the
    first decode launch must wait for it, the rest for their predecessors."""
    B = 1
    sts = quantized(CHAIN, seed=700)
    x_src = torch.empty(B, CHAIN[0][1], dtype=torch.bfloat16, device="cuda")
    x_in = torch.zeros_like(x_src)
    outs = [torch.empty(B, N, dtype=torch.bfloat16, device="cuda") for N, _ in CHAIN]
    run_chain(x_in, sts, sync=False, outs=outs)  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s), torch.cuda.graph(g, stream=s):
        x_in.copy_(x_src)
        run_chain(x_in, sts, sync=False, outs=outs)
    torch.cuda.current_stream().wait_stream(s)
    for trial in range(3):
        x_src.copy_(synth.activations_bf16(B, CHAIN[0][1], seed=800 + trial, device="cuda"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ref = run_chain(x_src.clone(), sts, sync=True)
        for i, (a, b) in enumerate(zip(outs, ref)):
            assert torch.equal(a, b), "replay %d: link %d differs" % (trial, i)
    check_last_link(ref[-2], sts[-1], outs[-1])
    del g


@pytest.mark.parametrize("B", [1, 4])
def test_decoder_layers_with_grouped_lists(B):
    """Two decoder layers: q/k/v (grouped) -> o -> a list of four (the
    persistent kernel at B = 1) -> gate/up (grouped) -> down, each list
    reading the output of the one before."""
    shapes = [(4096, 4096)] * 8 + [(11008, 4096)] * 2 + [(4096, 11008)]
    layers = [quantized(shapes, seed=900 + 20 * l) for l in range(2)]

    def layer_pass(x, sync):
        ys = []

        def step(items):
            out = bnb4.gemv_4bit_grouped(items)
            if sync:
                torch.cuda.synchronize()
            ys.extend(out)
            return out

        for w in layers:
            q = step([(x, w[i], 4096) for i in range(3)])
            o = step([(q[0], w[3], 4096)])
            l4 = step([(o[0], w[4 + i], 4096) for i in range(4)])
            gu = step([(l4[3], w[8], 11008), (l4[3], w[9], 11008)])
            x = step([(gu[1], w[10], 4096)])[0]
        torch.cuda.synchronize()
        return ys

    for trial in range(3):
        x = synth.activations_bf16(B, 4096, seed=1000 + trial, device="cuda")
        ref = layer_pass(x, sync=True)
        got = layer_pass(x, sync=False)
        for i, (a, b) in enumerate(zip(got, ref)):
            assert torch.equal(a, b), "output %d differs from the serialised run" % i


def test_graph_after_other_kernels():
    """Inside a CUDA graph the library's kernels that follow a kernel node
    are launched as programmatic dependents of it: here every input is the
    output of a torch kernel captured just before (one that never lets its
    dependents start early), so each call must still see that kernel's
    finished output -- quantize, dequantize, a decode chain and a 64-token
    linear (the small-batch kernel), compared bit for bit with the same
    calls run eagerly."""
    N, K, B = 1088, 4096, 1
    w_src = synth.weight_bf16(N, K, seed=31, device="cuda").view(-1)
    x_src = torch.empty(B, K, dtype=torch.bfloat16, device="cuda")
    X_src = torch.empty(64, K, dtype=torch.bfloat16, device="cuda")
    st = bnb4.QuantState(N * K, 64, bnb4.NF4, True)
    ws = bnb4.workspace_for(st)
    deq = torch.empty(N * K, dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty(B, N, dtype=torch.bfloat16, device="cuda")
    sts2 = quantized([(K, N)], seed=32)

    def body():
        w = w_src * 1.0                      # a torch kernel produces the weight
        bnb4.quantize_4bit(w, 64, bnb4.NF4, True, state=st, workspace=ws)
        bnb4.dequantize_4bit(st, torch.bfloat16, out=deq)
        x = x_src + 0.0                      # and another one the activations
        bnb4.gemv_4bit(x, st, N, out=y1)
        y2 = bnb4.gemv_4bit(y1, sts2[0], K)
        return y2, bnb4.gemm_4bit(X_src * 1.0, st, N)

    x_src.copy_(synth.activations_bf16(B, K, seed=33, device="cuda"))
    X_src.copy_(synth.activations_bf16(64, K, seed=34, device="cuda"))
    body()  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s), torch.cuda.graph(g, stream=s):
        y2, Y3 = body()
    torch.cuda.current_stream().wait_stream(s)
    for trial in range(3):
        x_src.copy_(synth.activations_bf16(B, K, seed=40 + trial, device="cuda"))
        X_src.copy_(synth.activations_bf16(64, K, seed=50 + trial, device="cuda"))
        w_src.mul_(-1.0 if trial % 2 else 1.0)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        got = (st.codes.clone(), st.absmax_q.clone(), deq.clone(), y1.clone(), y2.clone(),
               Y3.clone())
        ref_st = bnb4.quantize_4bit(w_src.clone(), 64, bnb4.NF4, True)
        ref_deq = bnb4.dequantize_4bit(ref_st, torch.bfloat16)
        ref_y1 = bnb4.gemv_4bit(x_src.clone(), ref_st, N)
        ref_y2 = bnb4.gemv_4bit(ref_y1, sts2[0], K)
        ref_Y3 = bnb4.gemm_4bit(X_src.clone(), ref_st, N)
        torch.cuda.synchronize()
        for name, a, b in zip(("codes", "absmax_q", "dequantized", "y1", "y2", "Y64"), got,
                              (ref_st.codes, ref_st.absmax_q, ref_deq, ref_y1, ref_y2, ref_Y3)):
            assert torch.equal(a, b), "replay %d: %s differs" % (trial, name)
    del g
