"""GPU parity of bnb_quantize_4bit against the CPU oracle: codes, absmax,
absmax_q, scale2 and offset must be bit-identical, and nothing may be written
past any output buffer."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import GuardedState, assert_state_equal

pytestmark = pytest.mark.gpu


def run_both(x_cpu, bs, qtype, dq):
    """x_cpu: fp32, bf16 or fp16 CPU tensor. Returns (gpu arrays, oracle
    state)."""
    if x_cpu.dtype == torch.float32:
        host, dt = x_cpu.contiguous().view(-1).numpy(), bnb4.F32
    elif x_cpu.dtype == torch.float16:
        host, dt = x_cpu.contiguous().view(-1).numpy(), bnb4.F16
    else:
        host, dt = synth.bf16_bits(x_cpu.view(-1)), bnb4.BF16
    orc = oracle.quantize(host, bs, qtype, dq)
    g = GuardedState(host.size, bs, qtype, dq)
    g.quantize(x_cpu.cuda(), dt)
    return g.arrays(), orc


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [True, False])
@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 257, 4097, 100003])
def test_quantize_small_ragged(dtype, qtype, bs, dq, n):
    x = synth.normal_f32((n,), seed=n + bs, std=0.02)
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    elif dtype == "f16":
        x = x.to(torch.float16)
    gpu, orc = run_both(x, bs, qtype, dq)
    assert_state_equal(gpu, orc, dq)


def test_roundtrip_vector_1m():
    """fp32 vector of 2^20 ~ N(0, 0.02^2), seed 0, blocksize 64, double
    quant (mean-subtracted absmax in groups of 256)."""
    x = synth.normal_f32((synth.ROUNDTRIP_N,), seed=0, std=0.02)
    gpu, orc = run_both(x, 64, bnb4.NF4, True)
    assert orc["sum_exact"]
    assert_state_equal(gpu, orc, True)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("f16", [False, True])
def test_matrix_4096_with_outliers(qtype, f16):
    """bf16 (or, for the fp16 compute type, the same values in fp16) 4096 x
    4096 ~ N(0, 0.02^2), 0.1% of positions x20, blocksize 64, double quant."""
    W = synth.weight_bf16(4096, 4096, seed=1000, outlier_frac=synth.OUTLIER_FRAC)
    if f16:
        W = W.to(torch.float16)
    gpu, orc = run_both(W, 64, qtype, True)
    assert orc["sum_exact"]
    assert_state_equal(gpu, orc, True)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 256])
def test_exact_midpoint_ties(qtype, bs):
    """Blocks with max 2^k and the other elements exactly on fp32 codebook
    midpoints times 2^k: v lands on the midpoint, the lower code wins."""
    t = oracle.codebook(qtype).astype(np.float32)
    if qtype == bnb4.NF4:
        mids = [(t[i] + t[i + 1]) * np.float32(0.5) for i in range(15)]
    else:
        mids = [(t[i] + t[i + 1]) * np.float32(0.5) for i in range(7)]
        mids += [-m for m in mids]
    mids = np.array(mids, np.float32)
    rng = np.random.default_rng(bs)
    blocks = []
    for k in range(-20, 21, 5):
        blk = rng.choice(mids, bs).astype(np.float32) * np.float32(2.0 ** k)
        blk[rng.integers(bs)] = np.float32(2.0 ** k)
        blocks.append(blk)
    x = torch.from_numpy(np.concatenate(blocks))
    gpu, orc = run_both(x, bs, qtype, True)
    assert_state_equal(gpu, orc, True)


@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
def test_zero_tiny_and_signed_zero_blocks(qtype):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(64 * 12) * 0.02).astype(np.float32)
    x[0:64] = 0.0                                   # all-zero block
    x[64:128] = -0.0                                # all negative zero
    x[128:192] = rng.standard_normal(64) * 1e-40    # subnormal block
    x[192:256] = 0.0
    x[200] = 3e-39                                  # single tiny value
    x[256:320] = rng.standard_normal(64) * 1e30     # huge block
    gpu, orc = run_both(torch.from_numpy(x), 64, qtype, False)
    assert_state_equal(gpu, orc, False)


def test_codes_are_deterministic_and_independent_of_dq():
    x = synth.weight_bf16(512, 1024, seed=77).cuda().view(-1)
    a = bnb4.quantize_4bit(x, 64, bnb4.NF4, True)
    b = bnb4.quantize_4bit(x, 64, bnb4.NF4, False)
    c = bnb4.quantize_4bit(x, 64, bnb4.NF4, True)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.absmax, b.absmax)
    for k in ("codes", "absmax", "absmax_q", "scale2", "offset"):
        assert torch.equal(getattr(a, k), getattr(c, k))


def _special_blocks(bs, n_blocks, rng):
    """n_blocks blocks of N(0, 0.02^2) with special blocks spread through
    them: every absmax class the kernel treats apart (zero, subnormal,
    either side of 2^-126 and 2^126, near the fp32 maximum, infinite) and
    NaN elements in otherwise normal blocks."""
    x = (rng.standard_normal(bs * n_blocks) * 0.02).astype(np.float32)
    f = lambda bits: np.array([bits], np.uint32).view(np.float32)[0]
    specials = [
        lambda b: b * 0.0,                                   # all zero
        lambda b: np.full_like(b, -0.0),                     # all -0
        lambda b: b * np.float32(1e-37),                     # subnormal and tiny
        lambda b: np.where(np.arange(b.size) == 3, f(0x00800000), b * 1e-38),  # max 2^-126
        lambda b: np.where(np.arange(b.size) == 5, f(0x007fffff), b * 1e-39),  # max just below
        lambda b: np.where(np.arange(b.size) == 1, f(0x7e7fffff), b * 1e36),   # max just below 2^126
        lambda b: np.where(np.arange(b.size) == 2, f(0x7e800000), b * 1e36),   # max 2^126
        lambda b: np.where(np.arange(b.size) == 0, f(0x7f7fffff), b * 1e37),   # near FLT_MAX
        lambda b: np.where(np.arange(b.size) == 7, np.float32(np.inf), b),     # +inf
        lambda b: np.where(np.arange(b.size) == 9, np.float32(-np.inf), b),    # -inf
        lambda b: np.where(np.arange(b.size) % 5 == 0, np.float32(np.nan), b), # NaNs, finite max
    ]
    for i, blk in enumerate(range(3, n_blocks, 7)):
        sl = slice(blk * bs, (blk + 1) * bs)
        x[sl] = specials[i % len(specials)](x[sl]).astype(np.float32)
    return x


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("qtype", [bnb4.NF4, bnb4.FP4])
@pytest.mark.parametrize("bs", [32, 64, 256])
def test_special_values_in_full_tiles(dtype, qtype, bs):
    """Zero, subnormal, boundary, huge and infinite block maxima and NaN
    elements, placed inside full tiles (so the streaming loop's warp-uniform
    choice between the fast and the exact path is exercised) and in the
    ragged tail: codes and absmax equal the oracle's bit for bit."""
    rng = np.random.default_rng(bs + {"f32": 0, "bf16": 7, "f16": 11}[dtype] + 3 * qtype)
    n = 16384 * 3 + 77 * bs // 32 + 5
    nb = -(-n // bs)
    x = _special_blocks(bs, nb, rng)[:n]
    xt = torch.from_numpy(x)
    if dtype == "bf16":
        xt = xt.to(torch.bfloat16)
    elif dtype == "f16":  # the fp16 range turns the classes into 0, subnormal, inf
        xt = xt.to(torch.float16)
    gpu, orc = run_both(xt, bs, qtype, False)
    assert_state_equal(gpu, orc, False)


def test_fast_reciprocal_exhaustive():
    """The quantize kernel's reciprocal (approximation + Newton-Raphson +
    Markstein correction) equals CUDA's round-to-nearest reciprocal for every
    fp32 input in [2^-126, 2^126)."""
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    rc = bnb4.bnb4_debug_check_rcp(res.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, bnb4.bnb4_strerror(rc)
    torch.cuda.synchronize()
    mismatches, first = res.cpu().tolist()
    assert mismatches == 0, "first mismatching input bits 0x%08x" % (first & 0xffffffff)
    assert first & 0xffffffff == 0xffffffff


# ---- the grid-wide mean of double quantization: workspace reuse and replay


def _bits(x):
    return synth.bf16_bits(x.cpu().view(-1)) if x.dtype == torch.bfloat16 else \
        x.cpu().view(-1).numpy()


def _check_dq(st, x, bs=64, qtype=bnb4.NF4):
    orc = oracle.quantize(_bits(x), bs, qtype, True)
    assert orc["sum_exact"]
    assert_state_equal(bnb4.state_to_arrays(st), orc, True)


def test_workspace_reused_across_inputs_and_sizes():
    """One workspace, calls of different sizes and data in a row: no call
    takes another call's partial sums (a smaller grid leaves stale sums
    beyond its own, which it must not read)."""
    ws = None
    xs = [synth.weight_bf16(4096, 4096, seed=s, outlier_frac=synth.OUTLIER_FRAC).cuda().view(-1)
          for s in (1, 2)] + [synth.normal_f32((100003,), seed=3, std=0.02).cuda()]
    sts = []
    for x in xs + xs[::-1]:
        st = bnb4.QuantState(x.numel(), 64, bnb4.NF4, True)
        ws = ws if ws is not None else bnb4.workspace_for(st)
        sts.append((bnb4.quantize_4bit(x, 64, bnb4.NF4, True, state=st, workspace=ws), x))
    torch.cuda.synchronize()
    for st, x in sts:
        _check_dq(st, x)
    assert bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) == bnb4.OK


def test_fresh_workspace_with_arbitrary_contents():
    """A workspace's contents on first use do not matter."""
    x = synth.weight_bf16(1024, 4096, seed=8).cuda().view(-1)
    st = bnb4.QuantState(x.numel(), 64, bnb4.NF4, True)
    for fill in (0x00, 0xFF, None):
        ws = bnb4.workspace_for(st)
        if fill is None:
            ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8))
        else:
            ws.fill_(fill)
        bnb4.quantize_4bit(x, 64, bnb4.NF4, True, state=st, workspace=ws)
        torch.cuda.synchronize()
        _check_dq(st, x)


def test_graph_replay_with_new_data_each_time():
    """A quantize call captured once in a CUDA graph and replayed on new
    input values each time: every replay forms its own mean (the kernel, not
    the captured arguments, numbers the calls)."""
    n = 4096 * 1024
    x = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    st = bnb4.QuantState(n, 64, bnb4.FP4, True)
    ws = bnb4.workspace_for(st)
    x.copy_(synth.weight_bf16(4096, 1024, seed=20).view(-1))
    bnb4.quantize_4bit(x, 64, bnb4.FP4, True, state=st, workspace=ws)  # warm
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s), torch.cuda.graph(g, stream=s):
        bnb4.quantize_4bit(x, 64, bnb4.FP4, True, state=st, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    for seed in (21, 22, 23):
        src = synth.weight_bf16(4096, 1024, seed=seed, outlier_frac=synth.OUTLIER_FRAC)
        x.copy_(src.view(-1))
        g.replay()
        torch.cuda.synchronize()
        _check_dq(st, src.view(-1), qtype=bnb4.FP4)
    del g
