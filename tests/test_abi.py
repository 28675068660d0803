"""The C-ABI library loads, exports every entry point include/bnb4.h
declares, and rejects bad arguments with the documented status before any
CUDA call (these checks run on a machine without a GPU)."""
import ctypes
import os
import re

import pytest

import bit_blockwise_weight_nf4_b200 as bnb4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bnb4.h")


@pytest.fixture(scope="module")
def lib():
    from bit_blockwise_weight_nf4_b200 import build
    build.build()
    return bnb4.load()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"BNB4_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("bnb_quantize_4bit", "bnb_dequantize_4bit", "bnb_gemv_4bit",
              "bnb_gemm_4bit"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings(lib):
    assert bnb4.bnb4_abi_version() == bnb4.ABI_VERSION
    for s in range(-7, 1):
        assert bnb4.bnb4_strerror(s)
    assert bnb4.bnb4_strerror(-99) == "unknown status"


@pytest.mark.parametrize("n,bs,dq", [(1, 64, 1), (1 << 20, 64, 1),
                                     (4096 * 4096, 64, 1), (1000003, 32, 0),
                                     (65, 256, 1)])
def test_query_sizes(lib, n, bs, dq):
    rc, s = bnb4.bnb4_query_sizes(n, bs, dq)
    assert rc == 0
    nb = -(-n // bs)
    assert s.codes == (n + 1) // 2 and s.absmax == 4 * nb
    assert s.absmax_q == (nb if dq else 0)
    assert s.scale2 == (4 * -(-nb // 256) if dq else 0)
    assert s.offset == (4 if dq else 0)
    assert (s.workspace > 0) == bool(dq)


def test_query_sizes_errors(lib):
    assert bnb4.bnb4_query_sizes(0, 64, 1)[0] == bnb4.ERR_INVALID_ARG
    assert bnb4.bnb4_query_sizes(10, 48, 1)[0] == bnb4.ERR_UNSUPPORTED
    out = bnb4.Sizes()
    assert lib.bnb4_query_sizes(10, 64, 2, ctypes.byref(out)) == bnb4.ERR_INVALID_ARG
    assert lib.bnb4_query_sizes(10, 64, 1, None) == bnb4.ERR_INVALID_ARG


A16 = 0x10000  # fake, 16-byte aligned addresses: never dereferenced because
A4 = 0x20004   # every call below fails its argument checks first


def good_state(**kw):
    st = bnb4.QState(A16, A16 + 0x1000, A16 + 0x2000, A16 + 0x3000,
                     A16 + 0x4000, 4096, 64, bnb4.NF4, 1, 0)
    for k, v in kw.items():
        setattr(st, k, v)
    return st


@pytest.mark.parametrize("kw,x,dt,ws,wsb,want", [
    ({}, None, 1, A16, 1 << 20, bnb4.ERR_INVALID_ARG),
    ({}, A16, 7, A16, 1 << 20, bnb4.ERR_UNSUPPORTED),
    ({"blocksize": 48}, A16, 1, A16, 1 << 20, bnb4.ERR_UNSUPPORTED),
    ({"qtype": 2}, A16, 1, A16, 1 << 20, bnb4.ERR_INVALID_ARG),
    ({"n": 0}, A16, 1, A16, 1 << 20, bnb4.ERR_INVALID_ARG),
    ({"reserved": 1}, A16, 1, A16, 1 << 20, bnb4.ERR_INVALID_ARG),
    ({"codes": A16 + 8}, A16, 1, A16, 1 << 20, bnb4.ERR_ALIGNMENT),
    ({"absmax_q": A16 + 0x2001}, A16, 1, A16, 1 << 20, bnb4.ERR_ALIGNMENT),
    ({}, A16 + 4, 1, A16, 1 << 20, bnb4.ERR_ALIGNMENT),
    ({}, A16, 1, None, 0, bnb4.ERR_WORKSPACE),
    ({}, A16, 1, A16, 64, bnb4.ERR_WORKSPACE),
    ({"scale2": None}, A16, 1, A16, 1 << 20, bnb4.ERR_INVALID_ARG),
    ({"absmax": None}, A16, 1, A16, 1 << 20, bnb4.ERR_INVALID_ARG),
])
def test_quantize_argument_errors(lib, kw, x, dt, ws, wsb, want):
    assert bnb4.bnb_quantize_4bit(x, dt, good_state(**kw), ws, wsb, None) == want


def test_dequantize_argument_errors(lib):
    assert bnb4.bnb_dequantize_4bit(good_state(), None, 0, None) == bnb4.ERR_INVALID_ARG
    assert bnb4.bnb_dequantize_4bit(good_state(), A16, 5, None) == bnb4.ERR_UNSUPPORTED
    assert bnb4.bnb_dequantize_4bit(good_state(), A16 + 2, 0, None) == bnb4.ERR_ALIGNMENT
    assert bnb4.bnb_dequantize_4bit(good_state(offset=None), A16, 0, None) == \
        bnb4.ERR_INVALID_ARG
    assert bnb4.bnb_dequantize_4bit(good_state(double_quant=0, absmax=None), A16, 0,
                                    None) == bnb4.ERR_INVALID_ARG
    assert bnb4.bnb_dequantize_4bit(good_state(scale2=A4 + 1), A16, 0, None) == \
        bnb4.ERR_ALIGNMENT


def test_gemv_argument_errors(lib):
    W = good_state(n=64 * 64)
    ok = dict(x=A16, B=1, K=64, N=64, y=A16)

    def call(**kw):
        a = dict(ok, **kw)
        return bnb4.bnb_gemv_4bit(a["x"], a["B"], a["K"], kw.get("W", W), a["N"],
                                  a["y"], None)
    assert call(x=None) == bnb4.ERR_INVALID_ARG
    assert call(B=0) == bnb4.ERR_SHAPE
    assert call(B=257) == bnb4.ERR_SHAPE
    assert call(K=32, N=128) == bnb4.ERR_SHAPE          # K % 64
    assert call(N=65) == bnb4.ERR_SHAPE                 # W.n != N*K
    assert call(W=good_state(n=128 * 64, blocksize=128), N=128) == bnb4.ERR_SHAPE
    assert call(x=A16 + 8) == bnb4.ERR_ALIGNMENT
    assert call(y=A16 + 1) == bnb4.ERR_ALIGNMENT
    assert call(W=good_state(n=64 * 64, absmax_q=A16 + 0x2002)) == bnb4.ERR_ALIGNMENT


def test_grouped_gemv_argument_errors(lib):
    def prob(**kw):
        d = dict(x=A16, W=good_state(n=64 * 64), K=64, N=64, bias=None, y=A16)
        d.update(kw)
        return bnb4.GemvProblem(d["x"], d["W"], d["K"], d["N"], d["bias"], d["y"])

    def call(probs, B=1, dt=bnb4.BF16):
        return bnb4.bnb_gemv_4bit_grouped(probs, B, dt, None)
    assert lib.bnb_gemv_4bit_grouped(None, 1, 1, bnb4.BF16, None) == bnb4.ERR_INVALID_ARG
    assert call([prob()] * (bnb4.GROUP_MAX + 1)) == bnb4.ERR_SHAPE
    assert call([prob()], dt=bnb4.F32) == bnb4.ERR_UNSUPPORTED
    assert call([prob()], B=9) == bnb4.ERR_SHAPE
    assert call([prob()], B=0) == bnb4.ERR_SHAPE
    assert call([prob(), prob(x=None)]) == bnb4.ERR_INVALID_ARG
    assert call([prob(), prob(N=65)]) == bnb4.ERR_SHAPE
    assert call([prob(), prob(K=128, W=good_state(n=64 * 128))]) == bnb4.ERR_SHAPE  # K differs
    assert call([prob(K=128, W=good_state(n=64 * 128)),
                 prob(W=good_state(n=64 * 128, blocksize=128), K=128)]) == bnb4.ERR_UNSUPPORTED
    assert call([prob(), prob(W=good_state(n=64 * 64, qtype=bnb4.FP4))]) == bnb4.ERR_UNSUPPORTED
    assert call([prob(), prob(bias=A16 + 2)]) == bnb4.ERR_ALIGNMENT
    assert call([prob(x=A16 + 8)]) == bnb4.ERR_ALIGNMENT


def test_gemm_argument_errors(lib):
    W = good_state(n=64 * 64)

    def call(X=A16, M=128, K=64, N=64, Y=A16, W=W):
        return bnb4.bnb_gemm_4bit(X, M, K, W, N, Y, None)
    assert call(Y=None) == bnb4.ERR_INVALID_ARG
    assert call(M=0) == bnb4.ERR_SHAPE
    assert call(N=60, W=good_state(n=60 * 64)) == bnb4.ERR_SHAPE   # N % 8
    assert call(K=96, W=good_state(n=64 * 96)) == bnb4.ERR_SHAPE   # K % 64
    assert call(X=A16 + 2) == bnb4.ERR_ALIGNMENT
    assert call(Y=A16 + 8) == bnb4.ERR_ALIGNMENT


def test_linear_argument_errors(lib):
    W = good_state(n=64 * 64)

    def call(x=A16, dtype=bnb4.F16, M=4, K=64, N=64, bias=None, y=A16, W=W):
        return bnb4.bnb_linear_4bit(x, dtype, M, K, W, N, bias, y, None)
    assert call(x=None) == bnb4.ERR_INVALID_ARG
    assert call(y=None) == bnb4.ERR_INVALID_ARG
    assert call(dtype=bnb4.F32) == bnb4.ERR_UNSUPPORTED
    assert call(dtype=7) == bnb4.ERR_UNSUPPORTED
    assert call(M=0) == bnb4.ERR_SHAPE
    assert call(K=96, W=good_state(n=64 * 96)) == bnb4.ERR_SHAPE          # K % 64
    assert call(M=300, N=60, W=good_state(n=60 * 64)) == bnb4.ERR_SHAPE   # N % 8 above 256
    assert call(x=A16 + 2) == bnb4.ERR_ALIGNMENT
    assert call(bias=A16 + 2) == bnb4.ERR_ALIGNMENT
    assert call(y=A16 + 1) == bnb4.ERR_ALIGNMENT
    assert call(M=300, y=A16 + 2) == bnb4.ERR_ALIGNMENT                   # 16 B above 256


def test_view_argument_errors(lib):
    st = good_state(n=16 * 64)

    def q(rows=16, cols=64, ld=72, dtype=bnb4.BF16, W=st, x=A16):
        return bnb4.bnb_quantize_4bit_2d(x, dtype, rows, cols, ld, W, A16, 1 << 20, None)

    def d(rows=16, cols=64, ld=72, dtype=bnb4.BF16, W=st, out=A16):
        return bnb4.bnb_dequantize_4bit_2d(W, out, dtype, rows, cols, ld, None)
    for call in (q, d):
        assert call(rows=15) == bnb4.ERR_SHAPE                  # rows * cols != n
        assert call(ld=60) == bnb4.ERR_SHAPE                    # ld < cols
        assert call(cols=60, rows=16, W=good_state(n=16 * 60), ld=64) == bnb4.ERR_SHAPE
        assert call(ld=68) == bnb4.ERR_SHAPE                    # rows not 16-byte aligned
        assert call(dtype=9) == bnb4.ERR_UNSUPPORTED
        assert call(rows=1 << 20, cols=1 << 12, ld=1 << 12,
                    W=good_state(n=1 << 32)) == bnb4.ERR_SHAPE  # n >= 2^32
        assert call(rows=0) == bnb4.ERR_SHAPE
    # fp32 rows need only 4-element alignment
    assert q(cols=68, ld=76, dtype=bnb4.F32, W=good_state(n=16 * 68)) != bnb4.ERR_SHAPE
    assert q(x=None) == bnb4.ERR_INVALID_ARG
    assert d(out=None) == bnb4.ERR_INVALID_ARG


def test_no_cpu_fallback_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(bnb4, "_lib", None)
    monkeypatch.setattr(bnb4, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        bnb4.load()
