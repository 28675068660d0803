"""Pins for the CPU oracle: each test checks it against something other than
itself -- the closed form through a library quantile function, the values the
NF4 article prints, exact rational arithmetic, torch's bf16 cast, numpy's
IEEE binary16 conversion, numpy's matmul, or brute force on tiny inputs.  No
GPU is needed."""
import os
from fractions import Fraction
from statistics import NormalDist

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(x):
    return np.float32(x)


def frac_to_f32(fr):
    """Exact round-to-nearest-even of a rational to fp32 (normal or
    subnormal range), independent of any floating-point library."""
    if fr == 0:
        return np.float32(0.0)
    sign = -1 if fr < 0 else 1
    a = abs(Fraction(fr))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = max(e - 23, -149)
    m = a / Fraction(2) ** q
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return np.float32(sign * fl * 2.0 ** q)


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ codebooks
def test_nf4_table_matches_closed_form():
    """Normal-quantile construction (QLoRA) recomputed with the standard
    library's inverse normal CDF, cast to fp32, compared bit for bit."""
    nd = NormalDist()
    delta = 0.5 * (1 / 32 + 1 / 30)
    pmax = 1 - delta
    lin = lambda a, b, n: [a + (b - a) * i / (n - 1) for i in range(n)]
    pos = [nd.inv_cdf(p) for p in lin(0.5, pmax, 9)[1:]]
    neg = [-nd.inv_cdf(p) for p in lin(0.5, pmax, 8)[1:]]
    v = sorted(pos + neg + [0.0])
    expect = np.array([x / max(v) for x in v], np.float64).astype(np.float32)
    got = oracle.codebook(oracle.NF4)
    assert got.tobytes() == expect.tobytes()


def test_nf4_table_matches_printed_values():
    t = oracle.codebook(oracle.NF4)
    for idx, val, tol in read_golden("nf4_printed_values.txt"):
        assert abs(float(t[int(idx)]) - float(val)) <= float(tol), idx
    assert np.all(np.diff(t) > 0)
    # the printed positive 0.697 is a garble: the table is not symmetric
    assert abs(float(t[14]) - 0.697) > 0.02


def e2m1_value(bits3):
    """E2M1 magnitude from its 3 bits (2 exponent, 1 mantissa, bias 1)."""
    e, m = bits3 >> 1, bits3 & 1
    return m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)


def test_fp4_table_is_e2m1_over_6():
    t = oracle.codebook(oracle.FP4)
    for idx, val in read_golden("fp4_e2m1_magnitudes.txt"):
        assert e2m1_value(int(idx)) == float(val)
    for c in range(16):
        mag = frac_to_f32(Fraction(e2m1_value(c & 7)) / 6)
        want = -mag if c & 8 else mag
        assert t[c].tobytes() == np.float32(want).tobytes(), c
    assert np.signbit(t[8]) and t[8] == 0.0


# ------------------------------------------------------------- nearest code
def brute_nearest(qtype, v):
    """argmin |v - t[c]| in exact arithmetic, ties to the lower index (NF4)
    or to the smaller magnitude (FP4, sign bit only for a non-zero
    magnitude)."""
    t = oracle.codebook(qtype)
    fv = Fraction(float(v))
    if qtype == oracle.NF4:
        best = None
        for c in range(16):
            d = abs(fv - Fraction(float(t[c])))
            if best is None or d < best[0]:
                best = (d, c)
        return best[1]
    best = None
    for m in range(8):
        d = abs(abs(fv) - Fraction(float(t[m])))
        if best is None or d < best[0]:
            best = (d, m)
    m = best[1]
    return m | 8 if (v < 0 and m > 0) else m


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_nearest_code_brute_force(qtype):
    rng = np.random.default_rng(11)
    vals = np.concatenate([rng.uniform(-1, 1, 3000),
                           oracle.codebook(qtype).astype(np.float64),
                           [0.0, -0.0, 1.0, -1.0]]).astype(np.float32)
    for v in vals:
        assert oracle.nearest_code(qtype, float(v)) == brute_nearest(qtype, v), v


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_tie_at_fp32_midpoint_goes_to_lower(qtype):
    t = oracle.codebook(qtype)
    if qtype == oracle.NF4:
        for i in range(15):
            mid = f32(f32(t[i] + t[i + 1]) * f32(0.5))
            assert oracle.nearest_code(qtype, float(mid)) == i
            assert oracle.nearest_code(qtype, float(np.nextafter(mid, f32(2)))) == i + 1
    else:
        for i in range(7):
            mid = f32(f32(t[i] + t[i + 1]) * f32(0.5))
            assert oracle.nearest_code(qtype, float(mid)) == i
            assert oracle.nearest_code(qtype, float(-mid)) == (i | 8 if i else 0)
            up = np.nextafter(mid, f32(2))
            assert oracle.nearest_code(qtype, float(up)) == i + 1
            assert oracle.nearest_code(qtype, float(-up)) == (i + 1) | 8


# --------------------------------------------------------------- quantize
@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_codebook_times_absmax_round_trips(qtype, bs):
    """x = RN(t[c] * a) for every code c quantizes to c and dequantizes
    (no double quant) back to x exactly."""
    rng = np.random.default_rng(bs + qtype)
    t = oracle.codebook(qtype)
    codes_all = [c for c in range(16) if not (qtype == oracle.FP4 and c == 8)]
    blocks = []
    for _ in range(6):
        a = f32(rng.uniform(1e-3, 3.0))
        cs = rng.choice(codes_all, size=bs)
        cs[0] = 15  # the block max is a itself (t[15] = 1)
        blocks.append((a, cs))
    x = np.concatenate([(t[cs] * a).astype(np.float32) for a, cs in blocks])
    st = oracle.quantize(x, bs, qtype, double_quant=False)
    n = x.size
    codes = np.zeros(n, np.uint8)
    codes[0::2] = st["codes"] >> 4
    codes[1::2] = st["codes"] & 15
    want = np.concatenate([cs for _, cs in blocks]).astype(np.uint8)
    if qtype == oracle.FP4:
        want = np.where((want & 7) == 0, 0, want)  # -0 is stored as code 0
    assert np.array_equal(codes, want)
    assert np.array_equal(st["absmax"], np.array([a for a, _ in blocks], np.float32))
    back = oracle.dequantize(st, oracle.F32)
    assert back.tobytes() == x.tobytes() or np.array_equal(back, x)


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_block_max_maps_to_unit_code(qtype):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(64 * 50) * 0.02).astype(np.float32)
    st = oracle.quantize(x, 64, qtype, double_quant=False)
    codes = np.zeros(x.size, np.uint8)
    codes[0::2] = st["codes"] >> 4
    codes[1::2] = st["codes"] & 15
    for b in range(50):
        blk = x[b * 64:(b + 1) * 64]
        i = int(np.argmax(np.abs(blk)))
        c = codes[b * 64 + i]
        if qtype == oracle.NF4:
            assert c == (15 if blk[i] > 0 else 0)
        else:
            assert c == (7 if blk[i] > 0 else 15)
    if qtype == oracle.FP4:
        assert not np.any(codes == 8)


def test_packing_order_and_odd_tail():
    t = oracle.codebook(oracle.NF4)
    x = np.array([t[3], t[12], t[15], t[0], t[9]], np.float32)  # absmax 1
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=False)
    assert list(st["codes"]) == [0x3C, 0xF0, 0x90]


def test_partial_last_block():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(65).astype(np.float32)
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=False)
    assert st["absmax"].size == 2
    assert st["absmax"][0] == np.abs(x[:64]).max()
    assert st["absmax"][1] == abs(x[64])


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_all_zero_block(qtype):
    x = np.zeros(64, np.float32)
    x[1] = -0.0
    st = oracle.quantize(x, 64, qtype, double_quant=False)
    zc = 7 if qtype == oracle.NF4 else 0
    assert np.all(st["codes"] == (zc << 4 | zc))
    back = oracle.dequantize(st, oracle.F32)
    assert np.all(back == 0) and not np.any(np.signbit(back))


def test_bf16_input_is_exact_widening():
    torch.manual_seed(0)
    xb = (torch.randn(1000) * 0.02).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    a = oracle.quantize(bits, 64, oracle.NF4, double_quant=True)
    b = oracle.quantize(xb.float().numpy(), 64, oracle.NF4, double_quant=True)
    for k in ("codes", "absmax", "absmax_q", "scale2", "offset"):
        assert np.array_equal(a[k], b[k]), k


# ------------------------------------------- normalisation by the reciprocal
# Reading R5: v = RN(x * RN(1 / absmax)).  The two plausible alternatives --
# dividing, v = RN(x / absmax), or normalising in fp64 and rounding once to
# fp32 -- differ from it by at most one fp32 ulp of v, so they give a
# different code only where that ulp straddles a codebook midpoint.  The
# search below builds such (x, absmax) pairs in exact rational arithmetic
# and checks that the oracle takes the reciprocal reading on every one.

def _ulp_step(x, k):
    """The fp32 value k ulps away from fp32 x (k may be negative)."""
    v = np.float32(x)
    toward = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
    for _ in range(abs(k)):
        v = np.nextafter(v, toward)
    return v


def _r6_midpoints(qtype):
    """Reading R6's fp32 midpoints RN(RN(t[i] + t[i+1]) * 0.5), rounded here
    in exact rational arithmetic (NF4: 15 ascending; FP4: 7 magnitudes).
    Where t[i] + t[i+1] is not an fp32 number the midpoint sits an ulp off
    the exact one, so the code can differ from the exact argmin on that
    single value."""
    t = [Fraction(float(v)) for v in oracle.codebook(qtype)]
    k = 15 if qtype == oracle.NF4 else 7
    return [frac_to_f32(Fraction(float(frac_to_f32(t[i] + t[i + 1]))) / 2)
            for i in range(k)]


def r6_code(qtype, v):
    """Code of fp32 v under R6: the number of fp32 midpoints strictly below v
    (FP4: below |v|, sign bit for a negative value with a non-zero
    magnitude)."""
    mids = _r6_midpoints(qtype)
    fv = Fraction(float(v))
    if qtype == oracle.NF4:
        return sum(1 for m in mids if fv > Fraction(float(m)))
    m = sum(1 for mm in mids if abs(fv) > Fraction(float(mm)))
    return m | 8 if (fv < 0 and m > 0) else m


def test_r6_midpoints_equal_nearest_except_on_rounded_midpoints():
    """R6 against the exact argmin.  An fp32 midpoint lies within half an
    ulp of the exact one, so the fp32 values on either side of it get the
    exact nearest code; on the midpoint itself the tie rule gives the lower
    index, which is the exact nearest entry unless the fp32 midpoint was
    rounded above the exact one (then the value is strictly closer to the
    upper entry: a documented consequence of R6)."""
    rounded_up = 0
    for qtype in (oracle.NF4, oracle.FP4):
        t = oracle.codebook(qtype)
        for i, m in enumerate(_r6_midpoints(qtype)):
            exact = (Fraction(float(t[i])) + Fraction(float(t[i + 1]))) / 2
            below = np.nextafter(m, np.float32(-2))
            above = np.nextafter(m, np.float32(2))
            assert r6_code(qtype, below) == brute_nearest(qtype, below) == i
            assert r6_code(qtype, above) == brute_nearest(qtype, above) == i + 1
            assert r6_code(qtype, m) == oracle.nearest_code(qtype, float(m)) == i
            if Fraction(float(m)) > exact:
                rounded_up += 1
                assert brute_nearest(qtype, m) == i + 1
            else:
                assert brute_nearest(qtype, m) == i
    assert rounded_up > 0


def _straddle_cases(qtype, want=24, seed=21):
    """(a, x, code_reciprocal, code_division) with the two readings on
    opposite sides of a midpoint; both orientations, positive and negative
    x."""
    rng = np.random.default_rng(seed)
    mids = [Fraction(float(m)) for m in _r6_midpoints(qtype)]
    if qtype == oracle.FP4:
        mids = mids + [-m for m in mids]
    out, seen = [], set()
    tries = 0
    while len(out) < want and tries < 4000:
        tries += 1
        a = np.float32(rng.uniform(0.01, 0.09))
        fa = Fraction(float(a))
        r = frac_to_f32(1 / fa)
        # a reciprocal with a large relative error makes straddles likely
        if abs(Fraction(float(r)) * fa - 1) < Fraction(1, 2 ** 26):
            continue
        for m in mids:
            x0 = frac_to_f32(m * fa)
            for k in range(-3, 4):
                x = _ulp_step(x0, k)
                if not (abs(float(x)) < float(a)):
                    continue
                fx = Fraction(float(x))
                v_rcp = frac_to_f32(fx * Fraction(float(r)))
                v_div = frac_to_f32(fx / fa)
                c_rcp = r6_code(qtype, v_rcp)
                c_div = r6_code(qtype, v_div)
                if c_rcp != c_div:
                    key = (int(c_rcp > c_div), bool(x < 0))
                    seen.add(key)
                    out.append((a, x, c_rcp, c_div))
    return out, seen


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_normalisation_multiplies_by_rounded_reciprocal(qtype):
    cases, seen = _straddle_cases(qtype)
    assert len(cases) >= 24
    # both directions of the disagreement, and (NF4) both signs of x
    assert {k[0] for k in seen} == {0, 1}
    if qtype == oracle.NF4:
        assert {k[1] for k in seen} == {False, True}
    bs = 32
    x = np.zeros(len(cases) * bs, np.float32)
    for j, (a, xv, _, _) in enumerate(cases):
        x[j * bs] = a          # the block max, code +-1
        x[j * bs + 1] = xv     # the straddling element
    st = oracle.quantize(x, bs, qtype, double_quant=False)
    hi = st["codes"] >> 4
    lo = st["codes"] & 15
    for j, (a, xv, c_rcp, c_div) in enumerate(cases):
        assert st["absmax"][j] == a
        got = int(lo[j * bs // 2])  # element 1 of the block: low nibble of byte 0
        assert got == c_rcp, (float(a), float(xv))
        assert got != c_div
        # normalising in fp64 and rounding once lands on the division's side
        v64 = np.float32(np.float64(xv) / np.float64(a))
        assert r6_code(qtype, v64) == c_div
        assert int(hi[j * bs // 2]) == (15 if qtype == oracle.NF4 else 7)


def _r6_vectorised(qtype, v):
    """r6_code over an fp32 array (fp32 comparisons are exact)."""
    mids = np.array(_r6_midpoints(qtype), np.float32)
    if qtype == oracle.NF4:
        return (v[:, None] > mids[None, :]).sum(axis=1)
    m = (np.abs(v)[:, None] > mids[None, :]).sum(axis=1)
    return np.where((v < 0) & (m > 0), m | 8, m)


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_quantize_codes_match_reciprocal_restatement(qtype):
    """10^5 N(0, 0.02^2) elements: every code equals R6's code of
    RN(x * RN(1/a)), computed here with IEEE fp32 arithmetic (itself checked
    against exact rational rounding on a sample)."""
    rng = np.random.default_rng(23)
    n, bs = 100_000, 64
    x = (rng.standard_normal(n) * 0.02).astype(np.float32)
    st = oracle.quantize(x, bs, qtype, double_quant=False)
    codes = np.zeros(n, np.uint8)
    codes[0::2] = st["codes"] >> 4
    codes[1::2] = st["codes"] & 15
    nb = (n + bs - 1) // bs
    pad = np.zeros(nb * bs, np.float32)
    pad[:n] = x
    a = np.abs(pad.reshape(nb, bs)).max(axis=1).astype(np.float32)
    assert np.array_equal(a, st["absmax"])
    r = (np.float32(1.0) / a).astype(np.float32)
    v = (x * np.repeat(r, bs)[:n]).astype(np.float32)
    assert v.dtype == np.float32
    for i in rng.choice(n, 300, replace=False):
        b = i // bs
        assert r[b] == frac_to_f32(1 / Fraction(float(a[b])))
        assert v[i] == frac_to_f32(Fraction(float(x[i])) * Fraction(float(r[b])))
    assert np.array_equal(codes, _r6_vectorised(qtype, v).astype(np.uint8))
    # away from the rounded midpoints the codes are the exact nearest entries
    sample = rng.choice(n, 2000, replace=False)
    for i in sample:
        if v[i] not in set(_r6_midpoints(qtype)):
            assert codes[i] == brute_nearest(qtype, v[i])


# ------------------------------------------------------- double quantization
def test_double_quant_offset_is_exact_mean():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(64 * 1000) * 0.02).astype(np.float32)
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=True)
    assert st["sum_exact"]
    mean = sum(Fraction(float(a)) for a in st["absmax"]) / st["absmax"].size
    # fp64 sum is exact here, then S / nb rounds to fp64 and then to fp32
    s64 = float(sum(Fraction(float(a)) for a in st["absmax"]))
    assert st["offset"][0] == np.float32(s64 / st["absmax"].size)
    assert abs(float(st["offset"][0]) - float(mean)) <= 2 ** -20 * float(mean)


def test_double_quant_scale_and_codes_exact():
    """s = RN(M / 127), q = rint(RN(c / s)) recomputed in exact arithmetic."""
    rng = np.random.default_rng(8)
    x = (rng.standard_normal(64 * 700) * 0.02).astype(np.float32)
    x[rng.choice(x.size, 70, replace=False)] *= 20
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=True)
    off = Fraction(float(st["offset"][0]))
    a = st["absmax"]
    for g in range(st["scale2"].size):
        grp = a[g * 256:(g + 1) * 256]
        cs = [frac_to_f32(Fraction(float(v)) - off) for v in grp]
        M = max(abs(float(c)) for c in cs)
        s = frac_to_f32(Fraction(M) / 127)
        assert st["scale2"][g] == s
        for j, c in enumerate(cs):
            r = frac_to_f32(Fraction(float(c)) / Fraction(float(s)))
            q = int(np.rint(np.float64(r)))  # half-even on an exact value
            q = max(-127, min(127, q))
            assert int(st["absmax_q"][g * 256 + j]) == q + 128
    assert st["absmax_q"].min() >= 1


def test_double_quant_rint_is_half_even():
    """absmax values [0, 254, 129.5, 124.5]: mean 127, c = [-127, 127, 2.5,
    -2.5], s = 1, so q = rint(+-2.5) = +-2 under round-half-even."""
    bs = 32
    x = np.zeros(4 * bs, np.float32)
    for b, a in enumerate([0.0, 254.0, 129.5, 124.5]):
        x[b * bs] = a
        x[b * bs + 1] = a * 0.25
    st = oracle.quantize(x, bs, oracle.NF4, double_quant=True)
    assert st["offset"][0] == 127.0 and st["scale2"][0] == 1.0
    assert list(st["absmax_q"]) == [1, 255, 130, 126]


def test_double_quant_all_equal_absmax():
    x = np.tile(np.array([0.5] + [0.1] * 63, np.float32), 300)
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=True)
    assert st["offset"][0] == 0.5
    assert np.all(st["scale2"] == 0) and np.all(st["absmax_q"] == 128)
    nodq = dict(st, double_quant=False)
    assert np.array_equal(oracle.dequantize(st), oracle.dequantize(nodq))


def test_double_quant_error_bound():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(64 * 2000) * 0.02).astype(np.float32)
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=True)
    t15 = np.float32(1.0)
    # decoded absmax = dequantized value of code 15 (t = 1)
    ahat = np.array([float(oracle.dequantize(
        {"n": 1, "blocksize": 64, "qtype": 0, "double_quant": True,
         "codes": np.array([0xF0], np.uint8),
         "absmax_q": st["absmax_q"][b:b + 1],
         "scale2": st["scale2"][b // 256:b // 256 + 1],
         "offset": st["offset"]})[0]) * float(t15) for b in range(0, 2000, 97)])
    a = st["absmax"][0:2000:97].astype(np.float64)
    s = st["scale2"][np.arange(0, 2000, 97) // 256].astype(np.float64)
    assert np.all(np.abs(ahat - a) <= s / 2 + 4 * np.spacing(np.float32(a)).astype(np.float64) + 1e-12)


def test_codes_do_not_depend_on_double_quant():
    rng = np.random.default_rng(10)
    x = (rng.standard_normal(64 * 300 + 17) * 0.02).astype(np.float32)
    a = oracle.quantize(x, 64, oracle.NF4, double_quant=True)
    b = oracle.quantize(x, 64, oracle.NF4, double_quant=False)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["absmax"], b["absmax"])


def test_sum_exact_flag_detects_order_dependence():
    bs = 32
    x = np.zeros(3 * bs, np.float32)
    x[0], x[bs], x[2 * bs] = 2.0 ** 60, 1.0, 1.0
    st = oracle.quantize(x, bs, oracle.NF4, double_quant=True)
    assert not st["sum_exact"]


# ------------------------------------------------------------- dequantize
def test_decode_fma_single_rounding():
    """a_hat = fma(u - 128, s, offset) against exact arithmetic."""
    rng = np.random.default_rng(12)
    for _ in range(400):
        u = int(rng.integers(1, 256))
        s = np.float32(rng.uniform(1e-5, 1e-3))
        off = np.float32(rng.uniform(0.01, 0.1))
        st = {"n": 1, "blocksize": 64, "qtype": 0, "double_quant": True,
              "codes": np.array([0xF0], np.uint8),
              "absmax_q": np.array([u], np.uint8),
              "scale2": np.array([s], np.float32),
              "offset": np.array([off], np.float32)}
        got = oracle.dequantize(st)[0]  # t[15] = 1, so w = a_hat
        want = frac_to_f32((u - 128) * Fraction(float(s)) + Fraction(float(off)))
        assert got == want


def test_bf16_rne_matches_torch_cast():
    rng = np.random.default_rng(13)
    vals = np.concatenate([
        rng.standard_normal(5000).astype(np.float32),
        (rng.standard_normal(500) * 1e-39).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 1.0 + 2 ** -8,
                  1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20], np.float32)])
    # exact ties: low 16 bits == 0x8000
    ties = (rng.integers(0, 2 ** 15, 500).astype(np.uint32) << 16 | 0x8000) \
        .view(np.float32)
    vals = np.concatenate([vals, ties[np.isfinite(ties)]])
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want)


def test_dequant_bf16_is_rne_of_fp32():
    rng = np.random.default_rng(14)
    x = (rng.standard_normal(64 * 40 + 3) * 0.02).astype(np.float32)
    st = oracle.quantize(x, 64, oracle.FP4, double_quant=True)
    w32 = oracle.dequantize(st, oracle.F32)
    w16 = oracle.dequantize(st, oracle.BF16)
    want = torch.from_numpy(w32).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)
    assert np.array_equal(w16, want)


# --------------------------------------------------------- linear reference
def test_linear_ref_matches_numpy_matmul():
    rng = np.random.default_rng(15)
    x = torch.from_numpy(rng.standard_normal((5, 96)).astype(np.float32)) \
        .to(torch.bfloat16)
    W = torch.from_numpy((rng.standard_normal((37, 96)) * 0.02).astype(np.float32)) \
        .to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    y = oracle.linear_ref(xb, Wb)
    ref = x.double().numpy() @ W.double().numpy().T
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-15)
    rows, cols = np.array([4, 0, 2]), np.array([36, 1])
    ys = oracle.linear_ref(xb, Wb, rows, cols)
    assert np.allclose(ys, ref[np.ix_(rows, cols)], rtol=1e-13, atol=1e-15)


def test_linear_ref_one_hot_rows_copy_columns():
    rng = np.random.default_rng(16)
    x = torch.from_numpy(rng.standard_normal((3, 64)).astype(np.float32)) \
        .to(torch.bfloat16)
    W = torch.zeros(8, 64, dtype=torch.bfloat16)
    for i in range(8):
        W[i, 7 * i] = 1.0
    y = oracle.linear_ref(x.view(torch.int16).numpy().view(np.uint16),
                          W.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(y, x.double().numpy()[:, [7 * i for i in range(8)]])


# ------------------------------------------------------ method-level claim
def test_nf4_beats_int4_on_normal_weights():
    """The NF4 article's claim: on N(0, s^2) weights NF4 has lower error than
    symmetric absmax INT4 (uniform codes -7..7 times absmax/7)."""
    rng = np.random.default_rng(17)
    x = (rng.standard_normal(64 * 4000) * 0.02).astype(np.float32)
    st = oracle.quantize(x, 64, oracle.NF4, double_quant=False)
    mse_nf4 = np.mean((oracle.dequantize(st).astype(np.float64) - x) ** 2)
    blk = x.reshape(-1, 64).astype(np.float64)
    a = np.abs(blk).max(axis=1, keepdims=True)
    q = np.clip(np.rint(blk / a * 7), -7, 7)
    mse_int4 = np.mean((q * a / 7 - blk) ** 2)
    assert mse_nf4 < mse_int4


# ---- fp16 compute type and bias ---------------------------------------------

def test_f16_rne_matches_numpy_cast():
    """The oracle's binary16 rounding against numpy's IEEE float32 -> float16
    conversion (round to nearest even): random values over every exponent,
    exact ties, the subnormal range, the overflow boundary and specials."""
    rng = np.random.default_rng(21)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-5).astype(np.float32),   # subnormal f16
        (rng.standard_normal(2000) * 1e-7).astype(np.float32),   # below 2^-24
        (rng.standard_normal(2000) * 3e4).astype(np.float32),    # near overflow
        rng.integers(0, 2 ** 31, 4000, dtype=np.uint32).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65519.99, 65520.0,
                  -65520.0, 2 ** -14, 2 ** -24, 2 ** -25, 3 * 2 ** -26,
                  2 ** -25 * 1.0000001, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11,
                  6.1e-5], np.float32)])
    # exact ties at normal and subnormal spacing
    ties = (rng.integers(0x38800000 >> 13, 0x477fe000 >> 13, 500).astype(np.uint32) << 13
            | 0x1000).view(np.float32)
    sub_ties = ((rng.integers(0, 1024, 200) * 2 + 1) * 2.0 ** -25).astype(np.float32)
    vals = np.concatenate([vals, ties, sub_ties])
    vals = vals[~np.isnan(vals)]
    with np.errstate(over="ignore"):  # values past 65520 become infinity
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f16_rne(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want), np.nonzero(got != want)[0][:8]
    nan = oracle.f16_rne(float("nan"))
    assert nan & 0x7c00 == 0x7c00 and nan & 0x3ff


def test_f16_decode_is_exact_for_every_pattern():
    """All 65536 binary16 patterns decode to the value numpy assigns them."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = pats.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_to_float(int(h)) for h in pats], np.float32)
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin].view(np.uint32), want[fin].view(np.uint32))
    assert np.all(np.isnan(got[~fin]))


@pytest.mark.parametrize("qtype", [oracle.NF4, oracle.FP4])
def test_f16_input_is_exact_widening(qtype):
    """Quantizing fp16 data equals quantizing the same values as fp32."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal(64 * 33 + 5) * 0.02).astype(np.float16)
    x[::97] *= np.float16(20.0)
    a = oracle.quantize(x, 64, qtype, True)
    b = oracle.quantize(x.astype(np.float32), 64, qtype, True)
    for k in ("codes", "absmax", "absmax_q", "scale2", "offset"):
        assert np.array_equal(a[k], b[k]), k


def test_dequant_f16_is_rne_of_fp32():
    """The fp16 dequantized weight is numpy's fp16 rounding of the fp32 one."""
    rng = np.random.default_rng(23)
    x = (rng.standard_normal(64 * 40 + 3) * 0.02).astype(np.float32)
    for qtype in (oracle.NF4, oracle.FP4):
        st = oracle.quantize(x, 64, qtype, double_quant=True)
        w32 = oracle.dequantize(st, oracle.F32)
        w16 = oracle.dequantize(st, oracle.F16)
        assert np.array_equal(w16, w32.astype(np.float16).view(np.uint16))


def test_linear_ref_f16_and_bias_match_numpy_matmul():
    """fp16 operands and a bias: the fp64 reference equals numpy's float64
    matmul of the exact values plus the bias (summation order aside)."""
    rng = np.random.default_rng(24)
    x = rng.standard_normal((5, 96)).astype(np.float16)
    W = (rng.standard_normal((7, 96)) * 0.05).astype(np.float16)
    bias = rng.standard_normal(7).astype(np.float16)
    y = oracle.linear_ref(x.view(np.uint16), W.view(np.uint16), dtype=oracle.F16,
                          bias_bits=bias.view(np.uint16))
    want = x.astype(np.float64) @ W.astype(np.float64).T + bias.astype(np.float64)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
    yb = oracle.linear_ref(x.view(np.uint16), W.view(np.uint16), dtype=oracle.F16)
    np.testing.assert_allclose(y - yb, np.broadcast_to(bias.astype(np.float64), y.shape),
                               rtol=1e-12, atol=1e-12)
    # a bf16 bias is decoded as bf16
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    Wb = torch.from_numpy(W.astype(np.float32)).to(torch.bfloat16)
    bb = torch.from_numpy(bias.astype(np.float32)).to(torch.bfloat16)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    y2 = oracle.linear_ref(bits(xb), bits(Wb), bias_bits=bits(bb))
    want2 = xb.double().numpy() @ Wb.double().numpy().T + bb.double().numpy()
    np.testing.assert_allclose(y2, want2, rtol=1e-12, atol=1e-12)
