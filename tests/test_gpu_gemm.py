"""GPU prefill GEMM (tcgen05, fused dequantization) against the fp64 oracle
over the dequantized bf16 weight, with the tolerance of the method's brief.
Full-size shapes are checked on a seeded sample of 128 rows of X (8 from
every 128-row sub-tile, its edge rows included; all columns);
small shapes, including ragged M, are checked in full."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


def case(M, N, K, bs, qtype, dq, seed, n_rows=None):
    W = synth.weight_bf16(N, K, seed=seed)
    X = synth.activations_bf16(M, K, seed=seed + 1)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), bs, qtype, dq)
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    Xb = synth.bf16_bits(X)
    rows = None
    if n_rows is not None and n_rows < M:
        # stratified: the same number of rows from every 128-row sub-tile
        # (each CTA of a pair holds 128-row sub-tiles of X), its first and
        # last row included
        rng = np.random.default_rng(seed)
        per = max(2, n_rows // -(-M // 128))
        picks = []
        for t0 in range(0, M, 128):
            t1 = min(t0 + 128, M)
            inner = np.arange(t0 + 1, t1 - 1)
            k = min(per - 2, inner.size)
            picks += [t0, t1 - 1] + list(rng.choice(inner, k, replace=False) if k > 0 else [])
        rows = np.unique(np.array(picks))
    y64 = oracle.linear_ref(Xb, What, rows=rows)
    g = bnb4.state_from_arrays(st)
    Y = bnb4.gemm_4bit(X.cuda(), g, N)
    torch.cuda.synchronize()
    assert bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == 0
    Yb = cpu_bits(Y)
    if rows is not None:
        Yb = Yb[rows]
    return check_linear(Yb, y64, Xb, What, rows=rows)


@pytest.mark.parametrize("N,K", synth.GEMM_SHAPES)
def test_prefill_shapes_nf4_bs64(N, K):
    """X bf16 [2048, K] ~ N(0, 1); NF4 weight ~ N(0, 0.02^2), blocksize 64,
    double quant."""
    case(synth.GEMM_M, N, K, 64, bnb4.NF4, True, seed=N + 3 * K, n_rows=128)


@pytest.mark.parametrize("qtype,bs", [(bnb4.NF4, 128), (bnb4.FP4, 64),
                                      (bnb4.FP4, 128)])
def test_prefill_variants(qtype, bs):
    case(synth.GEMM_M, 4096, 4096, bs, qtype, True, seed=bs + qtype, n_rows=128)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
@pytest.mark.parametrize("M,N,K", [(1, 8, 256), (100, 264, 512),
                                   (300, 520, 192), (256, 256, 64),
                                   (513, 16, 1024)])
def test_small_ragged(qtype, bs, dq, M, N, K):
    if K % bs:
        pytest.skip("K must be a multiple of the blocksize")
    case(M, N, K, bs, qtype, dq, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(1500, 4104, 512),   # several M tiles, ragged M and N
                                   (700, 2056, 320),    # ragged M, N and K steps
                                   (2048, 11008, 256)]) # more tiles than SM pairs
def test_tiles_ragged(M, N, K):
    """Partial pair tiles at the M and N edges, and more tiles than SM pairs
    (several waves)."""
    case(M, N, K, 64, bnb4.NF4, True, seed=M + 7 * N + K, n_rows=64)


@pytest.mark.parametrize("qtype,bs", [(bnb4.FP4, 64), (bnb4.NF4, 64), (bnb4.NF4, 32)])
def test_repeated_launches_bit_identical(qtype, bs):
    """The kernel's accumulation order is fixed, so repeated launches on the
    same inputs must agree bit for bit; a race between the shared-memory
    rings (a stage refilled while it is still being read) shows up here as
    run-to-run differences long before it breaks the tolerance."""
    W = synth.weight_bf16(4096, 4096, seed=bs + 11 * qtype).cuda().view(-1)
    st = bnb4.quantize_4bit(W, bs, qtype, True)
    X = synth.activations_bf16(2048, 4096, seed=bs + 11 * qtype + 1).cuda()
    outs = [bnb4.gemm_4bit(X, st, 4096) for _ in range(16)]
    torch.cuda.synchronize()
    assert bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == 0
    ref = outs[0].view(torch.int16)
    differing = [i for i in range(1, len(outs)) if not torch.equal(outs[i].view(torch.int16), ref)]
    assert not differing, "launches %s differ from the first" % differing
