"""The allocation-free quantize entry point against the regular one.

bnb_quantize_4bit_noalloc serves callers that cannot allocate device memory or
hand the library a workspace (a plugin whose host framework owns every
device allocation, or a latency-critical loader that must not call
cudaMalloc).  It keeps its scratch in a fixed array inside the library, so
these tests check that two calls in a row -- the second on a different input,
after the first has left its own values in that shared array, also a small
input right after a large one -- give exactly the codes and double-quant
scales of bnb_quantize_4bit and of the CPU oracle, and that inputs larger
than the fixed scratch are refused before anything is launched.

This file is collected last (pytest orders files by name), so a run that
stops at the first failure has already run every other test; it also passes
when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth

pytestmark = pytest.mark.gpu


def _noalloc(x, dtype, blocksize, qtype):
    """Output buffers allocated by the test (the caller's side); the entry
    point itself gets no workspace and no absmax buffer."""
    n = x.numel()
    rc, sz = bnb4.bnb4_query_sizes(n, blocksize, True)
    assert rc == 0
    out = {"codes": torch.empty(sz.codes, dtype=torch.uint8, device="cuda"),
           "absmax_q": torch.empty(sz.absmax_q, dtype=torch.uint8, device="cuda"),
           "scale2": torch.empty(sz.scale2 // 4, dtype=torch.float32, device="cuda"),
           "offset": torch.empty(1, dtype=torch.float32, device="cuda")}
    st = bnb4.QState(out["codes"].data_ptr(), None, out["absmax_q"].data_ptr(),
                     out["scale2"].data_ptr(), out["offset"].data_ptr(), n,
                     blocksize, qtype, 1, 0)
    rc = bnb4.bnb_quantize_4bit_noalloc(x.data_ptr(), dtype, st,
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0, bnb4.bnb4_strerror(rc)
    return out


def _regular(x, blocksize, qtype):
    st = bnb4.quantize_4bit(x, blocksize, qtype, True)
    return {"codes": st.codes, "absmax_q": st.absmax_q, "scale2": st.scale2,
            "offset": st.offset}


CASES = [
    # (shape, dtype, blocksize, qtype): bf16 Llama-sized matrix with
    # outliers, fp32 vector, ragged bf16 length with blocksize 32, fp16
    ((4096, 4096), "bf16", 64, bnb4.NF4),
    ((1 << 20,), "f32", 64, bnb4.FP4),
    ((100003,), "bf16", 32, bnb4.NF4),
    ((3 * 65536 + 40,), "f16", 128, bnb4.FP4),
]
DT = {"f32": bnb4.F32, "bf16": bnb4.BF16, "f16": bnb4.F16}


def _input(shape, dtype, seed):
    if dtype == "f32":
        return synth.normal_f32(shape, seed=seed, std=0.02).cuda()
    if dtype == "f16":
        return synth.normal_f32(shape, seed=seed, std=0.02).to(torch.float16).cuda()
    if len(shape) == 2:
        return synth.weight_bf16(shape[0], shape[1], seed=seed,
                                 outlier_frac=synth.OUTLIER_FRAC).cuda().view(-1)
    return synth.normal_f32(shape, seed=seed, std=0.02).to(torch.bfloat16).cuda()


def _oracle(x, blocksize, qtype):
    h = x.cpu()
    if h.dtype == torch.bfloat16:
        h = synth.bf16_bits(h)
    else:
        h = h.numpy()
    return oracle.quantize(h, blocksize, qtype, True)


def _assert_equal(g, w, orc):
    for k in ("codes", "absmax_q", "scale2", "offset"):
        assert torch.equal(g[k], w[k]), k
        assert np.array_equal(g[k].cpu().numpy(), orc[k]), k


@pytest.mark.parametrize("shape,dtype,blocksize,qtype", CASES)
def test_noalloc_matches_regular_two_calls_in_a_row(shape, dtype, blocksize, qtype):
    dt = DT[dtype]
    xs = [_input(shape, dtype, seed) for seed in (21, 22)]
    got = [_noalloc(x, dt, blocksize, qtype) for x in xs]   # back to back
    want = [_regular(x, blocksize, qtype) for x in xs]
    torch.cuda.synchronize()
    for x, g, w in zip(xs, got, want):
        _assert_equal(g, w, _oracle(x, blocksize, qtype))
    # the two inputs differ, so equal outputs would mean stale scratch
    assert not torch.equal(got[0]["codes"], got[1]["codes"])


def test_noalloc_large_then_small():
    """A large call fills the shared scratch (every CTA's partial sum, every
    block's absmax); the small call right after uses a smaller grid and
    fewer blocks and must not read any of the leftovers."""
    big = _input((4096, 4096), "bf16", 31)
    small = _input((100003,), "bf16", 32)
    g_big = _noalloc(big, bnb4.BF16, 64, bnb4.NF4)
    g_small = _noalloc(small, bnb4.BF16, 64, bnb4.NF4)
    torch.cuda.synchronize()
    _assert_equal(g_big, _regular(big, 64, bnb4.NF4), _oracle(big, 64, bnb4.NF4))
    _assert_equal(g_small, _regular(small, 64, bnb4.NF4), _oracle(small, 64, bnb4.NF4))


def test_noalloc_refuses_inputs_beyond_its_scratch():
    n = (bnb4.NOALLOC_MAX_BLOCKS + 1) * 32
    st = bnb4.QState(0x10000, None, 0x20000, 0x30000, 0x40000, n, 32, bnb4.NF4, 1, 0)
    rc = bnb4.bnb_quantize_4bit_noalloc(0x50000, bnb4.BF16, st, None)
    assert rc == bnb4.ERR_SCRATCH_LIMIT
    assert "scratch" in bnb4.bnb4_strerror(rc)


def test_noalloc_requires_double_quant():
    st = bnb4.QState(0x10000, None, 0x20000, 0x30000, 0x40000, 4096, 64, bnb4.NF4, 0, 0)
    assert bnb4.bnb_quantize_4bit_noalloc(0x50000, bnb4.BF16, st, None) == \
        bnb4.ERR_INVALID_ARG
