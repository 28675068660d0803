"""GPU GEMV (decode) against the fp64 oracle over the dequantized bf16
weight: relative Frobenius error <= 2e-3, per-row max abs error <=
1e-2 ||x_b|| max|What|, and nearly every output equal to the bf16 rounding of
the exact result."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


def case(N, K, B, bs, qtype, dq, seed, path="single"):
    """path "single": one bnb_gemv_4bit call (the one-CTA-per-16-rows
    kernel); "grouped": the weight twice in one bnb_gemv_4bit_grouped call
    (that kernel over a list); "persistent": the same list forced onto the
    persistent TMA-staged kernel; every output checked."""
    W = synth.weight_bf16(N, K, seed=seed)
    x = synth.activations_bf16(B, K, seed=seed + 1)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), bs, qtype, dq)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    xb = synth.bf16_bits(x)
    y64 = oracle.linear_ref(xb, What)
    g = bnb4.state_from_arrays(st)
    if path == "single":
        return check_linear(cpu_bits(bnb4.gemv_4bit(x.cuda(), g, N)), y64, xb, What)
    xd = x.cuda()
    for y in bnb4.gemv_4bit_grouped([(xd, g, N), (xd, g, N)], _persistent=path == "persistent"):
        r = check_linear(cpu_bits(y), y64, xb, What)
    return r


PATHS = ["single", "grouped", "persistent"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("B", [1, 8])
def test_llama_mlp_shapes(N, K, B, path):
    """Decode GEMV: x bf16 [B, K] ~ N(0, 1); NF4 weight ~ N(0, 0.02^2),
    blocksize 64, double quant (Llama-7B MLP shapes)."""
    case(N, K, B, 64, bnb4.NF4, True, seed=N + K, path=path)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
@pytest.mark.parametrize("N,K,B", [(1, 256, 1), (13, 320, 3), (100, 576, 8),
                                   (257, 1024, 5), (8, 64, 2)])
@pytest.mark.parametrize("path", PATHS)
def test_small_ragged(qtype, bs, dq, N, K, B, path):
    if K % bs:
        pytest.skip("K must be a multiple of the blocksize")
    case(N, K, B, bs, qtype, dq, seed=N * 31 + K, path=path)


@pytest.mark.parametrize("N,K,B", [(4099, 4096, 1), (1030, 2112, 2), (517, 11008, 4),
                                   (30001, 256, 8), (4096, 64, 1), (22, 1344, 2),
                                   (40003, 1024, 1), (38000, 2048, 3), (2400, 4352, 8)])
@pytest.mark.parametrize("path", PATHS)
def test_row_groups_and_warp_splits(N, K, B, path):
    """16-row groups with ragged N; K split over a CTA's warps (few row
    groups per CTA: runs that start and end inside row groups, a last chunk
    with empty segments) or whole row groups per warp (short K and many row
    groups: 40003 x 1024, 38000 x 2048)."""
    case(N, K, B, 64, bnb4.NF4, True, seed=N + 3 * K + B, path=path)


@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008), (40003, 1024)])
def test_decode_is_bit_reproducible(N, K):
    """The partial sums over K are added in a fixed order: repeated launches
    give identical bits."""
    W = synth.weight_bf16(N, K, seed=9)
    g = bnb4.quantize_4bit(W.cuda().view(-1), 64, bnb4.NF4, True)
    x = synth.activations_bf16(1, K, seed=10).cuda()
    ys = [bnb4.gemv_4bit(x, g, N) for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])


@pytest.mark.parametrize("B", [9, 16, 17, 24, 32, 33, 40, 63, 64])
@pytest.mark.parametrize("N,K", [(1030, 2112), (4096, 4096)])
def test_batch_column_groups(N, K, B):
    """bnb_gemv_4bit with 9..64 rows of x (the small-batch kernel: tokens on
    the MMA's N side, padded to a multiple of 16 with zero rows)."""
    case(N, K, B, 64, bnb4.NF4, True, seed=N + 7 * K + B)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
@pytest.mark.parametrize("B", [12, 30, 64])
def test_batch_groups_every_format(qtype, bs, dq, B):
    """Every blocksize / code table / scale format through bnb_gemv_4bit
    above 8 rows, ragged N and K spanning several K steps."""
    case(259, 1280, B, bs, qtype, dq, seed=bs + 11 * B + int(dq))


def test_gpu_quantized_weight_end_to_end():
    """GPU quantize then GEMV on the GPU state (the codes equal the oracle's,
    so the same fp64 reference applies)."""
    N, K = 4096, 4096
    W = synth.weight_bf16(N, K, seed=5, outlier_frac=synth.OUTLIER_FRAC)
    x = synth.activations_bf16(1, K, seed=6)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), 64, bnb4.NF4, True)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    xb = synth.bf16_bits(x)
    y64 = oracle.linear_ref(xb, What)
    g = bnb4.quantize_4bit(W.cuda().view(-1), 64, bnb4.NF4, True)
    y = bnb4.gemv_4bit(x.cuda(), g, N)
    check_linear(cpu_bits(y), y64, xb, What)


@pytest.mark.parametrize("B", [17, 64])
def test_batch_rows_past_B_untouched(B):
    """The output rows past B (inside the last 16-token MMA column block)
    are never written: a canary row after y [B, N] keeps its bytes."""
    N, K = 520, 1024
    W = synth.weight_bf16(N, K, seed=B)
    x = synth.activations_bf16(B, K, seed=B + 1)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), 64, bnb4.NF4, True)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    g = bnb4.state_from_arrays(st)
    buf = torch.full(((B + 1) * N,), -7.0, dtype=torch.bfloat16, device="cuda")
    y = buf[:B * N].view(B, N)
    bnb4.gemv_4bit(x.cuda(), g, N, out=y)
    torch.cuda.synchronize()
    assert torch.all(buf[B * N:] == -7.0)
    check_linear(cpu_bits(y), oracle.linear_ref(synth.bf16_bits(x), What),
                 synth.bf16_bits(x), What)

