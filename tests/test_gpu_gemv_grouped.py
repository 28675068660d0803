"""Grouped decode GEMV (several linears in one launch) against the fp64
oracle over each weight's dequantized values, with the tolerance of the
single GEMV, and bit-reproducible for the same problem list.  Every test runs
the public entry (which picks the kernel by list length and B) and the same
list forced onto the persistent TMA-staged kernel."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[False, True], ids=["public", "persistent"])
def persist(request):
    return request.param


def make(N, K, bs, qtype, dq, seed):
    W = synth.weight_bf16(N, K, seed=seed)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), bs, qtype, dq)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    return bnb4.state_from_arrays(st), What, st


def run_group(shapes, B, bs=64, qtype=bnb4.NF4, dq=True, share_x=False, seed=0, persist=False):
    xs, items, refs = {}, [], []
    for i, (N, K) in enumerate(shapes):
        key = K if share_x else (K, i)
        if key not in xs:
            xs[key] = synth.activations_bf16(B, K, seed=seed + 100 + i)
        g, What, _ = make(N, K, bs, qtype, dq, seed + i)
        items.append((xs[key].cuda(), g, N))
        refs.append((xs[key], What))
    ys = bnb4.gemv_4bit_grouped(items, _persistent=persist)
    torch.cuda.synchronize()
    for y, (x, What) in zip(ys, refs):
        xb = synth.bf16_bits(x)
        check_linear(cpu_bits(y), oracle.linear_ref(xb, What), xb, What)
    return items, ys


@pytest.mark.parametrize("B", [1, 8])
def test_qkv_like_group_shares_x(B, persist):
    """q / k / v: three weights reading the same activations."""
    run_group([(1030, 4096)] * 3, B, share_x=True, seed=B, persist=persist)


@pytest.mark.parametrize("B", [1, 3])
@pytest.mark.parametrize("K", [64, 1344, 4096, 11008])
def test_mixed_rows_and_inputs(B, K, persist):
    """Different N per problem (ragged, tiny and large; one K per launch),
    separate inputs, one launch: short K with many row groups takes whole
    row groups per warp, long K splits them."""
    run_group([(4099, K), (257, K), (8, K), (1030, K)] + ([(40003, K)] if K <= 1344 else []),
              B, seed=10 + B + K, persist=persist)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
def test_every_format(qtype, bs, dq, persist):
    run_group([(259, 1280), (100, 1280), (33, 1280)], 2, bs=bs, qtype=qtype, dq=dq,
              seed=bs + int(dq), persist=persist)


def test_many_problems_large_group(persist):
    """More problems than one launch's parameter block holds (launched in
    parts of 32), each its own x."""
    shapes = [(64 + 16 * i, 576) for i in range(70)]
    run_group(shapes, 1, seed=77, persist=persist)


def test_fp16_with_bias_matches_oracle(persist):
    shapes = [(520, 1024), (264, 1024)]
    items, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weight_bf16(N, K, seed=40 + i)
        st = oracle.quantize(synth.bf16_bits(W.view(-1)), 64, oracle.NF4, True)
        W16 = oracle.dequantize(st, oracle.F16).reshape(N, K)
        x16 = synth.activations_bf16(4, K, seed=50 + i).to(torch.float16)
        b16 = synth.normal_f32((N,), seed=60 + i).to(torch.float16)
        items.append((x16.cuda(), bnb4.state_from_arrays(st), N, b16.cuda()))
        refs.append((x16, W16, b16))
    ys = bnb4.gemv_4bit_grouped(items, _persistent=persist)
    torch.cuda.synchronize()
    for y, (x16, W16, b16) in zip(ys, refs):
        bits = lambda t: t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
        y64 = oracle.linear_ref(bits(x16), W16, dtype=oracle.F16, bias_bits=bits(b16))
        check_linear(bits(y), y64, bits(x16), W16, dtype=oracle.F16)


def test_group_is_bit_reproducible(persist):
    items, ys = run_group([(11008, 4096), (4096, 4096), (4096, 4096)], 1, seed=5,
                          persist=persist)
    again = bnb4.gemv_4bit_grouped(items, _persistent=persist)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(ys, again))


def test_outputs_do_not_spill(persist):
    """Each y is written exactly within its [B, N]: canaries after each
    output survive."""
    N1, N2, K, B = 37, 100, 512, 3
    g1, W1, _ = make(N1, K, 64, bnb4.NF4, True, 1)
    g2, W2, _ = make(N2, K, 64, bnb4.NF4, True, 2)
    x = synth.activations_bf16(B, K, seed=3)
    buf = torch.full((B * N1 + 64 + B * N2 + 64,), -5.0, dtype=torch.bfloat16, device="cuda")
    y1 = buf[:B * N1].view(B, N1)
    y2 = buf[B * N1 + 64:B * N1 + 64 + B * N2].view(B, N2)
    bnb4.gemv_4bit_grouped([(x.cuda(), g1, N1), (x.cuda(), g2, N2)], outs=[y1, y2],
                           _persistent=persist)
    torch.cuda.synchronize()
    h = buf.cpu()
    assert torch.all(h[B * N1:B * N1 + 64] == -5.0)
    assert torch.all(h[B * N1 + 64 + B * N2:] == -5.0)
    xb = synth.bf16_bits(x)
    check_linear(cpu_bits(y1), oracle.linear_ref(xb, W1), xb, W1)
    check_linear(cpu_bits(y2), oracle.linear_ref(xb, W2), xb, W2)


@pytest.mark.parametrize("B", [1, 8])
def test_full_size_layer_lists(B, persist):
    """A Llama-7B layer's decode launches at full size, as the bench makes
    them: q / k / v (three 4096 x 4096, one x), gate / up (two 11008 x 4096,
    one x), and the six K = 4096 linears in one list; every output checked
    against the oracle."""
    run_group([(4096, 4096)] * 3, B, share_x=True, seed=300 + B, persist=persist)
    run_group([(11008, 4096)] * 2, B, share_x=True, seed=310 + B, persist=persist)
    run_group([(4096, 4096)] * 4 + [(11008, 4096)] * 2, B, share_x=True, seed=320 + B,
              persist=persist)
