"""GPU small-batch tier (1..256 token rows: the tcgen05 kernel with the
weight rows on the MMA's M side and K split over a cluster of 1..8 CTAs)
against the fp64 oracle over the dequantized bf16 weight, with the tolerance
of the method's brief.  Reached through both linear entry points: the GEMM
for 8 < M <= 256 and the GEMV for 8 < B <= 256 (M <= 8 runs the decode
kernel, and so does 9..16 when x and the codes are 32-byte aligned: the
cases with 9..16 rows run both, the small-batch kernel on a copy of x that
is only 16-byte aligned)."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


def status_ok():
    torch.cuda.synchronize()
    return bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == 0


def case(M, N, K, bs=64, qtype=bnb4.NF4, dq=True, seed=0, entry="gemm", unaligned=False):
    W = synth.weight_bf16(N, K, seed=seed)
    X = synth.activations_bf16(M, K, seed=seed + 1)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), bs, qtype, dq)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    Xb = synth.bf16_bits(X)
    y64 = oracle.linear_ref(Xb, What)
    g = bnb4.state_from_arrays(st)
    Xd = X.cuda()
    if unaligned:  # a copy 16 bytes past a 32-byte boundary
        buf = torch.empty(M * K + 32, dtype=Xd.dtype, device="cuda")
        lead = ((16 - buf.data_ptr() % 32) % 32) // 2
        Xd = buf[lead:lead + M * K].view(M, K)
        Xd.copy_(X)
        assert Xd.data_ptr() % 32 == 16
    if entry == "gemm":
        Y = bnb4.gemm_4bit(Xd, g, N)
    else:
        Y = bnb4.gemv_4bit(Xd, g, N)
    assert status_ok()
    return check_linear(cpu_bits(Y), y64, Xb, What)


@pytest.mark.parametrize("M", [1, 2, 8, 9, 15, 16, 17, 31, 33, 48, 63, 64, 65,
                               100, 128, 129, 200, 255, 256])
def test_token_counts(M):
    """Every token count class: M <= 8 through the decode kernel, above it
    NT = M rounded up to 16 (16..256), rows past M read as zeros by the TMA
    and never stored; 9 weight-row tiles (the
    last ragged) with 33 K steps split over a 7-CTA cluster (5 or 4 steps
    per rank)."""
    case(M, 1032, 2112, seed=M)
    if 9 <= M <= 16:
        case(M, 1032, 2112, seed=M, unaligned=True)


@pytest.mark.parametrize("N,K", [(16384, 256),   # cluster of 2 / 1 (24 / 160 tokens)
                                 (8192, 512),    # 4 / 2
                                 (6144, 960),    # 5 / 3
                                 (4104, 512),    # 8 / 4, ragged N
                                 (2056, 320),    # 5: one K step per rank
                                 (512, 704),     # 6: ranks of 2 and 1 steps
                                 (264, 1280),    # 7, ragged N
                                 (1024, 1024),   # 8
                                 (128, 64)])     # one tile, one K step
@pytest.mark.parametrize("M", [24, 160])
def test_cluster_splits(N, K, M):
    """The K split over clusters of every size the launcher picks (noted per
    shape for 148 SMs: 2 CTAs per SM at 24 tokens, 1 at 160), uneven step
    counts per rank, and the rank-order reduction of the partial sums
    through distributed shared memory."""
    case(M, N, K, seed=N + K + M)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
def test_every_format(qtype, bs, dq):
    """Each blocksize / code table / scale format (two tables per K step
    for blocksize 32, nested scales decoded in the dequantizing threads)."""
    case(40, 264, 1280, bs, qtype, dq, seed=bs + 3 * qtype + int(dq))


@pytest.mark.parametrize("N,K", synth.GEMM_SHAPES)
@pytest.mark.parametrize("M", [16, 64])
def test_llama_shapes(N, K, M):
    """Llama-7B projection shapes at batch 16 and 64: X bf16 ~ N(0, 1), NF4
    weight ~ N(0, 0.02^2), blocksize 64, double quant."""
    case(M, N, K, seed=N + 5 * K + M)


@pytest.mark.parametrize("B,N", [(9, 1030), (64, 517), (256, 1030)])
def test_gemv_entry_large_batch(B, N):
    """bnb_gemv_4bit with more than 8 rows of x runs the same kernel; N need
    not be a multiple of 8 there (y is written element by element)."""
    case(B, N, 1344, seed=B + N, entry="gemv", unaligned=B <= 16)


@pytest.mark.parametrize("M", [64, 256])
def test_repeated_launches_bit_identical(M):
    """The cluster reduction sums the ranks' partials in rank order, so
    repeated launches agree bit for bit; a ring race would show up here as
    run-to-run differences."""
    W = synth.weight_bf16(4096, 4096, seed=M).cuda().view(-1)
    st = bnb4.quantize_4bit(W, 64, bnb4.NF4, True)
    X = synth.activations_bf16(M, 4096, seed=M + 1).cuda()
    outs = [bnb4.gemm_4bit(X, st, 4096) for _ in range(16)]
    assert status_ok()
    ref = outs[0].view(torch.int16)
    differing = [i for i in range(1, len(outs)) if not torch.equal(outs[i].view(torch.int16), ref)]
    assert not differing, "launches %s differ from the first" % differing


def test_rows_past_M_untouched():
    """Y is written only at rows < M and columns < N: canary values after
    the output survive."""
    M, N, K = 33, 520, 1024
    W = synth.weight_bf16(N, K, seed=9)
    X = synth.activations_bf16(M, K, seed=10)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), 64, bnb4.NF4, True)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    g = bnb4.state_from_arrays(st)
    buf = torch.full(((M + 2) * N,), -7.0, dtype=torch.bfloat16, device="cuda")
    Y = buf[:M * N].view(M, N)
    bnb4.gemm_4bit(X.cuda(), g, N, out=Y)
    assert status_ok()
    assert torch.all(buf[M * N:] == -7.0)
    check_linear(cpu_bits(Y), oracle.linear_ref(synth.bf16_bits(X), What),
                 synth.bf16_bits(X), What)
