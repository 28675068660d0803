"""Helpers shared by the GPU parity tests: unpacking, guard (canary) buffers
and the linear-layer tolerance.

Tolerance for y = bf16(fp32 sum of x * What) against the fp64 oracle y64:
  * relative Frobenius error <= 2e-3 and per-row max abs error <=
    1e-2 * ||x_b||_2 * max|What| (the method's brief).  The Frobenius bound is
    statistical -- rounding one value to bf16 alone can cost up to 2^-8
    relative -- so it is applied to outputs of at least 1024 elements;
  * for every output, the bound the arithmetic gives: the fp32 accumulation
    of exact bf16 x bf16 products errs by at most gamma * S (S = sum |x w|,
    gamma = K 2^-22, a loose bound for any summation order and for the
    tensor cores' accumulation), and the final bf16 rounding by 2^-8 of the
    value: |y - y64| <= 2^-8 (|y64| + gamma S) + gamma S;
  * with at least 1024 outputs, 98% of them equal bf16(y64) exactly (a wrong
    What, or unrounded weights, would not); 90% for fp16, whose output ulp is
    8x finer, so that the fp32 tensor-core accumulation over K = 11008 flips
    a few percent of the roundings (95.8% measured on the prefill kernel),
    while a wrong fp16 What still fails by far (bf16-rounded weights match
    ~14%, unrounded fp32 weights ~58%, on 32 x 256 outputs at K = 4096)."""
import numpy as np
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle

REL_FROB_TOL = 2e-3
MATCH_MIN = {oracle.BF16: 0.98, oracle.F16: 0.90}
MAX_ABS_FACTOR = 1e-2
CANARY = 0xA5
GUARD = 64  # bytes of canary after every output buffer


def bits_to_f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def cpu_bits(t):
    """uint16 bit patterns of a bf16 tensor (any device)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class GuardedState:
    """A device quantization state whose buffers are followed by canary
    bytes, to catch writes past the end."""

    def __init__(self, n, blocksize, qtype, dq):
        rc, sz = bnb4.bnb4_query_sizes(n, blocksize, dq)
        assert rc == 0
        self.n, self.blocksize, self.qtype, self.dq = n, blocksize, qtype, dq
        self.sizes = {"codes": sz.codes, "absmax": sz.absmax,
                      "absmax_q": sz.absmax_q, "scale2": sz.scale2,
                      "offset": sz.offset}
        self.buf = {k: torch.full((v + GUARD,), CANARY, dtype=torch.uint8,
                                  device="cuda")
                    for k, v in self.sizes.items() if v > 0}
        self.workspace = torch.empty(sz.workspace, dtype=torch.uint8,
                                     device="cuda") if sz.workspace else None

    def cstruct(self):
        p = lambda k: self.buf[k].data_ptr() if k in self.buf else None
        return bnb4.QState(p("codes"), p("absmax"), p("absmax_q"), p("scale2"),
                           p("offset"), self.n, self.blocksize, self.qtype,
                           int(self.dq), 0)

    def quantize(self, x, x_dtype):
        rc = bnb4.bnb_quantize_4bit(
            x.data_ptr(), x_dtype, self.cstruct(),
            None if self.workspace is None else self.workspace.data_ptr(),
            0 if self.workspace is None else self.workspace.numel(),
            torch.cuda.current_stream().cuda_stream)
        assert rc == 0, bnb4.bnb4_strerror(rc)
        torch.cuda.synchronize()

    def arrays(self):
        host = {k: b.cpu().numpy() for k, b in self.buf.items()}
        for k, b in host.items():
            assert np.all(b[self.sizes[k]:] == CANARY), "write past the end of " + k
        out = {"codes": host["codes"][:self.sizes["codes"]],
               "absmax": host["absmax"][:self.sizes["absmax"]].view(np.float32)}
        if self.dq:
            out["absmax_q"] = host["absmax_q"][:self.sizes["absmax_q"]]
            out["scale2"] = host["scale2"][:self.sizes["scale2"]].view(np.float32)
            out["offset"] = host["offset"][:4].view(np.float32)
        return out


def assert_state_equal(gpu, orc, dq):
    keys = ["codes", "absmax"] + (["absmax_q", "scale2", "offset"] if dq else [])
    for k in keys:
        a, b = gpu[k], orc[k]
        assert a.shape == b.shape, k
        if not np.array_equal(a.view(np.uint8), b.view(np.uint8)):
            bad = np.nonzero(a.view(np.uint8) != b.view(np.uint8))[0]
            raise AssertionError("%s differs at %d bytes, first %s" % (k, bad.size, bad[:8]))


FROB_MIN_ELEMENTS = 1024


def check_linear(y_gpu_bits, y64, x_bits, What_bits, rows=None, dtype=oracle.BF16):
    """Tolerance for y = x What^T (+ bias; rows of x optionally subsampled;
    y64 is the fp64 oracle for those rows) in the compute type ``dtype``
    (bf16 or fp16 bit patterns).  See the module docstring; for fp16 the
    final rounding costs 2^-11 instead of 2^-8."""
    to64 = oracle.f16_bits_to_f64 if dtype == oracle.F16 else bits_to_f64
    unit = 2.0 ** -11 if dtype == oracle.F16 else 2.0 ** -8
    y = to64(y_gpu_bits).reshape(y64.shape)
    err = y - y64
    rel = np.linalg.norm(err) / max(np.linalg.norm(y64), 1e-300)
    if y64.size >= FROB_MIN_ELEMENTS:
        assert rel <= REL_FROB_TOL, "relative Frobenius error %.3g" % rel
    x = to64(x_bits)
    if rows is not None:
        x = x[rows]
    W = to64(What_bits)
    wmax = np.abs(W).max()
    bound = MAX_ABS_FACTOR * np.linalg.norm(x, axis=1) * wmax
    assert np.all(np.abs(err).max(axis=1) <= bound + 1e-30), "max abs error"
    K = x.shape[1]
    gamma = K * 2.0 ** -22
    S = np.abs(x) @ np.abs(W).T
    elem = unit * (np.abs(y64) + gamma * S) + gamma * S
    bad = np.abs(err) > elem
    assert not bad.any(), "elementwise bound violated at %d outputs" % bad.sum()
    # the rounding of the exact fp64 result to the compute type is the
    # dominant error: almost every output must equal it (a wrong What would not)
    t16 = torch.float16 if dtype == oracle.F16 else torch.bfloat16
    ref16 = torch.from_numpy(y64).to(t16).view(torch.int16).numpy() \
        .view(np.uint16).reshape(-1)
    match = np.mean(ref16 == np.asarray(y_gpu_bits).reshape(-1))
    if y64.size >= FROB_MIN_ELEMENTS:
        assert match >= MATCH_MIN[dtype], \
            "only %.4f of outputs equal the rounded fp64 reference" % match
    return rel, match
