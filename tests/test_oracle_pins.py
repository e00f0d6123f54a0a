"""Pins for the CPU oracle: each check ties the oracle to something other than itself --
value sets fixed by the format definitions, brute force with exact rational arithmetic,
closed forms, invariants the pages state, and hand-worked blocks (tests/golden/).

Passages followed:
  ScaleSweep (gist.science/ko/paper/2606.07618), "Methodology": S = max|x|/(256*6), E4M3
    base scale, 126 positive finite E4M3 values, offsets [-3,+7] / [-8,+7], the bound
    ratios 12/7, 4/5, 1/2, MSE and WMSE objectives.
  Adaptive Block-Scaled Data Types (gist.science/ko/paper/2603.28765), "Methodology": IF4,
    7/6 and 6/7, indicator bit; "Problem": 4/6.
  Bridging the Gap ... Microscaling FP4 (gist.science/ko/paper/2509.23202), "Methodology":
    MXFP4, block-wise Hadamard.  TORQ (gist.science/ko/paper/2605.19561), "Method": S-step.
"""
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

import oracle as O
from fp4_block_scaled_nvfp4_b200 import synth

GRID = [Fr(0), Fr(1, 2), Fr(1), Fr(3, 2), Fr(2), Fr(3), Fr(4), Fr(6)]
f32 = np.float32


# ---------------------------------------------------------------------------------
# independent references
# ---------------------------------------------------------------------------------
def e4m3_values_from_format():
    """All E4M3FN magnitudes from the bit layout: sign | 4 exponent (bias 7) | 3 mantissa."""
    vals = {}
    for p in range(0x7F):  # 0x7F is NaN in the FN variant
        E, M = p >> 3, p & 7
        vals[p] = Fr(M, 8) * Fr(2) ** -6 if E == 0 else (1 + Fr(M, 8)) * Fr(2) ** (E - 7)
    return vals


E4M3 = e4m3_values_from_format()


def nearest_e4m3(v: Fr) -> int:
    """Brute-force nearest E4M3FN pattern, ties to the even pattern, saturating at 448."""
    if v >= 448:
        return 0x7E
    best = min(E4M3, key=lambda p: (abs(v - E4M3[p]), p & 1))
    return best


def nearest_e2m1(y: Fr) -> Fr:
    """Brute-force nearest magnitude of the E2M1 grid, ties to the even index, saturating at 6."""
    a = abs(y)
    k = min(range(8), key=lambda k: (abs(a - GRID[k]), k & 1))
    return GRID[k] if y >= 0 else -GRID[k]


# ---------------------------------------------------------------------------------
# codec
# ---------------------------------------------------------------------------------
def test_e4m3_value_set():
    pos = [p for p in range(1, 0x7F)]
    vals = [O.e4m3_value(p) for p in pos]
    assert len(set(vals)) == 126          # ScaleSweep: 126 positive finite E4M3 values
    assert max(vals) == 448.0 and min(vals) == 2.0 ** -9
    for p in range(0x7F):
        assert Fr(O.e4m3_value(p)) == E4M3[p]
    assert np.isnan(O.e4m3_value(0x7F))


def test_e4m3_roundtrip_and_ties():
    for p in range(0x7F):
        assert O.e4m3_encode(O.e4m3_value(p)) == p
    # every midpoint between consecutive patterns goes to the even pattern
    for p in range(0x7E):
        mid = (E4M3[p] + E4M3[p + 1]) / 2
        m32 = float(f32(float(mid)))
        if Fr(m32) == mid:
            assert O.e4m3_encode(m32) == (p if p % 2 == 0 else p + 1)
    assert O.e4m3_encode(448.0) == 0x7E and O.e4m3_encode(1e30) == 0x7E and O.e4m3_encode(470.0) == 0x7E


def test_e4m3_random_vs_bruteforce():
    rng = np.random.default_rng(7)
    vs = np.concatenate([np.exp(rng.uniform(np.log(1e-4), np.log(600), 3000)), rng.uniform(0, 0.02, 500)])
    for v in vs.astype(np.float32):
        assert O.e4m3_encode(float(v)) == nearest_e4m3(Fr(float(v)))


def test_e2m1_grid_ties_saturation_sign():
    for k, g in enumerate(GRID):
        assert O.e2m1_encode(float(g)) == k and O.e2m1_value(k) == float(g)
        assert O.e2m1_value(k | 8) == -float(g)
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for y, k in ties.items():
        assert O.e2m1_encode(y) == k and O.e2m1_encode(-y) == (k | 8)
    assert O.e2m1_encode(7.0) == 7 and O.e2m1_encode(1e9) == 7 and O.e2m1_encode(-100.0) == 15
    assert O.e2m1_encode(-0.0) == 8 and O.e2m1_encode(0.0) == 0 and O.e2m1_encode(-0.1) == 8
    rng = np.random.default_rng(3)
    for y in rng.uniform(-8, 8, 4000).astype(np.float32):
        code = O.e2m1_encode(float(y))
        assert Fr(O.e2m1_value(code)) == nearest_e2m1(Fr(float(y)))


# ---------------------------------------------------------------------------------
# global scale, window arithmetic
# ---------------------------------------------------------------------------------
def test_global_scale_formula():
    for amax in [1536.0, 3072.0, 1.0, 0.02, 123.456]:
        S = O.global_scale(amax)
        assert S == float(f32(amax) / f32(1536.0))     # one binary32 division
        assert abs(Fr(S) * 1536 - Fr(amax)) <= Fr(amax) * Fr(2) ** -23
    assert O.global_scale(1536.0 * 4) == 4.0


def test_window_bounds_in_bit_pattern_space():
    """ScaleSweep: the MSE optimum lies in [4/5, 12/7] s_base; the pages map that to
    bit-pattern offsets [-3, +7].  Check the mapping for every normal base pattern."""
    for p0 in range(8, 0x7F):
        e0 = E4M3[p0]
        # +7 covers every value up to 12/7 e0 (the value past the window is above the bound)
        if p0 + 8 <= 0x7E:
            assert E4M3[p0 + 8] > Fr(12, 7) * e0
        above = [p for p in range(p0, 0x7F) if E4M3[p] <= Fr(12, 7) * e0]
        assert max(above) - p0 <= 7
        # -3 covers every value down to 4/5 e0
        if p0 - 4 >= 1:
            assert E4M3[p0 - 4] < Fr(4, 5) * e0
        below = [p for p in range(1, p0 + 1) if E4M3[p] >= Fr(4, 5) * e0]
        assert p0 - min(below) <= 3
        # offsets of 8 are exact factors of two (within the normal range)
        if p0 - 8 >= 8:
            assert E4M3[p0 - 8] * 2 == e0
            assert E4M3[p0 - 8] == Fr(1, 2) * e0    # the WMSE bound 1/2 s_base is offset -8


# ---------------------------------------------------------------------------------
# exact error arithmetic (rational brute force) and the argmins
# ---------------------------------------------------------------------------------
K67 = f32(6.0) / f32(7.0)      # RN(6/7), the INT4 dequantization constant
K76 = f32(7.0) / f32(6.0)      # RN(7/6), the INT4 pre-scale


def fp4_codes_exact(xb, s):
    """E2M1 magnitudes of the binary32 quantizer y = RN(x * RN(1/s)), rounded by brute force."""
    inv = f32(1.0) / f32(s) if s else f32(0.0)
    return [abs(nearest_e2m1(Fr(float(f32(xv) * inv)))) for xv in xb]


def int4_codes_exact(xb, s):
    """|n| of the INT4 path: n = clamp(round-half-even(RN(RN(x * RN(1/s)) * RN(7/6))), -7, 7),
    the rounding done on exact rationals."""
    inv = f32(1.0) / f32(s)
    out = []
    for xv in xb:
        z = Fr(float(f32(f32(xv) * inv) * K76))
        n = round(z)                       # Python rounds halves to even
        out.append(min(abs(n), 7))
    return out


def exact_error(xb, recon):
    """sum (x - recon)^2 over exact rationals (the block MSE, the method's objective)."""
    return sum((abs(Fr(float(xv))) - r) ** 2 for xv, r in zip(xb, recon))


def sv_of(p, S):
    return float(f32(float(E4M3[p])) * f32(S)) if p else 0.0


def exact_fp4_error(xb, p, S):
    s = sv_of(p, S)
    return exact_error(xb, [m * Fr(s) for m in fp4_codes_exact(xb, s)]) if p else exact_error(xb, [0] * len(xb))


def exact_int4_error(xb, p, S):
    s = sv_of(p, S)
    if not p:
        return exact_error(xb, [0] * len(xb))
    g = Fr(float(f32(K67 * f32(s))))       # the INT4 block scale RN(RN(6/7) * sv)
    return exact_error(xb, [n * g for n in int4_codes_exact(xb, s)])


def _tensor_with(xb, amax=1536.0):
    """Place block(s) into a tensor whose extra block sets amax (so S is known)."""
    xb = np.asarray(xb, np.float32).reshape(1, -1)
    pad = np.zeros((1, 16), np.float32)
    pad[0, 0] = amax
    return np.concatenate([xb, pad], axis=1)


def _tie_heavy_blocks(seed, n=40):
    """Blocks built to tie: grid values of two scales 3/2 apart, octave pairs, zero blocks with
    one value, and plain random blocks (S = 1 through the extra block)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        kind = rng.integers(0, 4)
        e = float(E4M3[int(rng.integers(40, 80))])
        if kind == 0:      # values on {0, 1.5, 3, 6} e: exact at e and at 1.5 e alike
            v = rng.choice([0.0, 1.5, 3.0, 6.0], 16) * e * rng.choice([-1, 1], 16)
            v[0] = 6 * e
        elif kind == 1:    # octave: values on {2, 3, 4, 6} e
            v = rng.choice([0.0, 2.0, 3.0, 4.0, 6.0], 16) * e
            v[3] = 6 * e
        elif kind == 2:
            v = np.zeros(16)
            v[rng.integers(0, 16)] = rng.uniform(0.1, 300)
        else:
            v = rng.laplace(size=16) * np.exp(rng.normal(size=16)) * 3
        out.append(np.asarray(v, np.float32))
    return out


@pytest.mark.parametrize("cfg", ["cfg1", "cfg3", "cfg4"])
def test_error_and_argmin_are_exact(cfg):
    """The oracle's MSE sweep: its reported block error is the exact rational block MSE (to the
    double rounding of the report) and its choice is the exact argmin over the window, the
    lowest offset winning a tie -- strictly, no tolerance."""
    w = synth.make(cfg, rows=2, cols=512)
    x = synth.as_f32(w)
    O.inexact_count()
    r = O.nvfp4_quantize(x, "sweep_mse")
    assert O.inexact_count() == 0
    S = r["S"]
    rng = np.random.default_rng(11)
    for _ in range(14):
        row, b = rng.integers(0, x.shape[0]), rng.integers(0, x.shape[1] // 16)
        xb = x[row, b * 16:(b + 1) * 16]
        p0 = O.e4m3_encode(float(f32(np.abs(xb).max()) / (f32(6) * f32(S))))
        cands = [p for p in range(p0 - 3, p0 + 8) if 0 <= p <= 0x7E]
        ex = {p: exact_fp4_error(xb, p, S) for p in cands}
        best = min(ex.values())
        want = min(p for p in cands if ex[p] == best)
        assert int(r["p"][row, b]) == want
        assert r["err"][row, b] == float(best)
        srt = sorted(ex.values())
        assert bool(r["tie"][row, b]) == (srt[0] == srt[1])


def test_argmin_exact_on_tie_heavy_blocks():
    """Blocks whose candidates tie exactly (scales 3/2 or 2 apart reproducing the same values):
    the oracle takes the lowest offset among the exact minima and flags the tie."""
    blocks = _tie_heavy_blocks(31)
    x = np.concatenate(blocks).reshape(1, -1)
    x = _tensor_with(x)
    r = O.nvfp4_quantize(x, "sweep_mse")
    assert r["S"] == 1.0
    ties = 0
    for j, xb in enumerate(blocks):
        p0 = O.e4m3_encode(float(f32(np.abs(xb).max()) / f32(6)))
        cands = [p for p in range(p0 - 3, p0 + 8) if 0 <= p <= 0x7E]
        ex = {p: exact_fp4_error(xb, p, 1.0) for p in cands}
        best = min(ex.values())
        assert int(r["p"][0, j]) == min(p for p in cands if ex[p] == best)
        t = sorted(ex.values())[1] == best
        assert bool(r["tie"][0, j]) == t
        ties += t
    assert ties >= 4


def test_weighted_error_matches_exact():
    """WMSE is binary32 with one accumulator per candidate in element order: xhat = RN(q sv),
    d = RN(x - xhat), acc = fma(RN(w d), d, acc).  Pinned against the exact weighted MSE of the
    same codes, within the error bound of those roundings (each product and difference one
    relative 2^-24, each fma one more), and the choice against the exact weighted argmin wherever
    the exact gap exceeds twice that bound."""
    wl = synth.make("cfg2", rows=2, cols=256)
    x = synth.as_f32(wl)
    imp = wl["importance"][:256]
    r = O.nvfp4_quantize(x, "sweep_wmse", importance=imp)
    S = r["S"]
    u = Fr(1, 2 ** 24)
    for row, b in [(0, 0), (0, 5), (1, 9), (1, 15), (0, 12)]:
        xb = x[row, b * 16:(b + 1) * 16]
        wb = imp[b * 16:(b + 1) * 16]
        p0 = O.e4m3_encode(float(f32(np.abs(xb).max()) / (f32(6) * f32(S))))
        cands = [p for p in range(p0 - 8, p0 + 8) if 0 <= p <= 0x7E]
        exact, bound = {}, {}
        for p in cands:
            s = sv_of(p, S)
            m = fp4_codes_exact(xb, s) if p else [0] * 16
            e, bd = Fr(0), Fr(0)
            for xv, wv, mm in zip(xb, wb, m):
                d = abs(Fr(float(xv))) - mm * Fr(s)
                e += Fr(float(wv)) * d * d
                eps = u * (abs(mm * Fr(s)) + abs(d)) * 2       # xhat and d roundings
                bd += Fr(float(wv)) * (2 * abs(d) * eps + eps * eps) * (1 + 4 * u) + 3 * u * Fr(float(wv)) * (abs(d) + eps) ** 2
            exact[p], bound[p] = e, bd + 17 * u * e
        chosen = int(r["p"][row, b])
        assert abs(Fr(float(r["err"][row, b])) - exact[chosen]) <= bound[chosen]
        best = min(exact, key=lambda p: (exact[p], p))
        if chosen != best:
            assert exact[chosen] - exact[best] <= bound[chosen] + bound[best]


def test_bruteforce_all_126_scales_on_tiny_blocks():
    """The window's choice has the exact minimum block MSE over every E4M3 scale on random
    blocks (ScaleSweep: the optimum lies inside the narrow window)."""
    rng = np.random.default_rng(5)
    for t in range(8):
        xb = (rng.laplace(size=16) * np.exp(rng.normal(size=16))).astype(np.float32)
        x = _tensor_with(xb, amax=float(np.abs(xb).max()) * 3.0)
        r = O.nvfp4_quantize(x, "sweep_mse")
        ex = {p: exact_fp4_error(xb, p, r["S"]) for p in range(0x7F)}
        assert ex[int(r["p"][0, 0])] == min(ex.values())


@pytest.mark.parametrize("cfg,obj", [("cfg1", "sweep_mse"), ("cfg3", "sweep_mse"), ("cfg2", "sweep_wmse")])
def test_window_claim_vs_bruteforce(cfg, obj):
    """Count blocks whose all-pattern optimum lies outside the window: 0 expected for MSE
    (Lemmas 4.1/4.3); the WMSE lower bound is empirical on the page, so it is reported."""
    wl = synth.make(cfg, rows=8, cols=1024)
    x = synth.as_f32(wl)
    imp = wl.get("importance")
    imp = None if imp is None else imp[:1024]
    win = O.nvfp4_quantize(x, obj, importance=imp)
    bf = O.nvfp4_quantize(x, "brute_mse" if obj == "sweep_mse" else "brute_wmse", importance=imp)
    outside = int(np.sum(bf["err"] < win["err"]))
    if obj == "sweep_mse":
        assert outside == 0
        assert np.array_equal(bf["err"], win["err"])
    else:
        assert outside <= max(1, win["err"].size // 100)


# ---------------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("cfg", ["cfg1", "cfg3"])
def test_ordering_sweep_46_absmax(cfg):
    wl = synth.make(cfg, rows=16, cols=1024)
    x = synth.as_f32(wl)
    ea = O.nvfp4_quantize(x, "absmax")["err"]
    e46 = O.nvfp4_quantize(x, "four_over_six")
    es = O.nvfp4_quantize(x, "sweep_mse")["err"]
    assert np.all(e46["err"] <= ea)
    assert np.all(es <= e46["err"])       # p4 - p0 lies in [-3, 7] for these data
    assert np.all(es <= ea)


def test_wmse_with_unit_weights_tracks_mse():
    """With unit weights the WMSE accumulator is the block MSE in binary32: within 2^-18
    relative of the exact error of the same codes, and choosing the exact MSE optimum except on
    blocks whose two best candidates are within that rounding of each other."""
    wl = synth.make("cfg3", rows=8, cols=512)
    x = synth.as_f32(wl)
    one = np.ones(512, np.float32)
    a = O.nvfp4_quantize(x, "brute_mse")
    b = O.nvfp4_quantize(x, "brute_wmse", importance=one)
    S = a["S"]
    differ = np.argwhere(a["scales"] != b["scales"])
    assert len(differ) <= a["scales"].size // 100
    for row, j in differ:
        xb = x[row, j * 16:(j + 1) * 16]
        ea, eb = exact_fp4_error(xb, int(a["p"][row, j]), S), exact_fp4_error(xb, int(b["p"][row, j]), S)
        assert ea <= eb and float(eb - ea) <= 2.0 ** -17 * float(eb)
    rng = np.random.default_rng(4)
    for row, j in zip(rng.integers(0, 8, 12), rng.integers(0, 32, 12)):
        xb = x[row, j * 16:(j + 1) * 16]
        e = exact_fp4_error(xb, int(b["p"][row, j]), S)
        assert abs(Fr(float(b["err"][row, j])) - e) <= Fr(1, 2 ** 18) * e + Fr(1, 10 ** 40)


def test_if4_errors_are_exact():
    """IF4 at the AbsMax scale: both types' reported errors are the exact rational block MSE
    (INT4 reconstruction n * RN(RN(6/7) * sv): the integer times the block scale with the 6/7
    dequantization folded in, in binary32 like every scale),
    and INT4 is chosen exactly when its exact error is lower (a tie keeps FP4)."""
    wl = synth.make("cfg4", rows=2, cols=1024)
    x = synth.as_f32(wl)
    O.inexact_count()
    r = O.if4_quantize(x)
    assert O.inexact_count() == 0
    S = r["S"]
    rng = np.random.default_rng(8)
    picks = list(zip(rng.integers(0, 2, 24), rng.integers(0, 64, 24)))
    ints = 0
    for row, j in picks:
        xb = x[row, j * 16:(j + 1) * 16]
        p = int(r["scales"][row, j]) & 0x7F
        ef, ei = exact_fp4_error(xb, p, S), exact_int4_error(xb, p, S)
        assert r["err_fp"][row, j] == float(ef) and r["err_int"][row, j] == float(ei)
        assert bool(r["scales"][row, j] >> 7) == (ei < ef)
        ints += ei < ef
    assert 0 < ints < len(picks)


def test_if4_invariants():
    wl = synth.make("cfg4", rows=8, cols=1024)
    x = synth.as_f32(wl)
    r = O.if4_quantize(x)
    a = O.nvfp4_quantize(x, "absmax")
    ind = (r["scales"] >> 7).astype(bool)
    assert np.array_equal(r["scales"] & 0x7F, a["scales"])          # shared AbsMax scale
    # both report the exact block error: IF4's FP4 path at p0 is AbsMax itself
    assert np.array_equal(r["err_fp"], a["err"])
    assert np.all(np.where(ind, r["err_int"], r["err_fp"]) <= a["err"])   # IF4 <= AbsMax
    assert 0 < ind.mean() < 1
    # FP4 blocks carry exactly the AbsMax codes
    cf = r["codes"].reshape(8, -1, 8)[~ind]
    assert np.array_equal(cf, a["codes"].reshape(8, -1, 8)[~ind])
    # INT4 nibbles are two's complement in [-7, 7] (0x8 never used)
    ci = r["codes"].reshape(8, -1, 8)[ind]
    nib = np.concatenate([ci & 0xF, ci >> 4])
    assert not np.any(nib == 8)


def test_mx_exponent_closed_form():
    rng = np.random.default_rng(9)
    for a in np.exp(rng.uniform(-60, 60, 3000)).astype(np.float32):
        e = O.mx_exponent(float(a))
        assert Fr(float(a)) <= 6 * Fr(2) ** e and Fr(float(a)) > 6 * Fr(2) ** (e - 1)   # smallest such e
        assert 3 < float(a) / 2.0 ** e <= 6
        eo = O.mx_exponent(float(a), True)
        assert 4 <= float(a) / 2.0 ** eo < 8
    assert O.mx_exponent(0.0) == -127


def test_e8m0_roundtrip_every_exponent():
    # a block whose maximum is 6 * 2^e and whose other elements are signed E2M1 grid values
    # times 2^e selects E8M0 byte e + 127 and dequantizes exactly, for every exponent whose
    # block fits in binary32 (-127 .. 125; 2^-128 and below are exact fp32 subnormals)
    blocks = []
    exps = list(range(-127, 126))
    for e in exps:
        p = 2.0 ** e
        vals = [6 * p] + [sg * float(g) * p for g in GRID for sg in (1, -1)] + [0.0] * 15
        blocks.append(np.array(vals[:32], np.float32))
    x = np.concatenate(blocks).reshape(1, -1)
    r = O.mxfp4_quantize(x)
    assert list(r["scales"][0]) == [e + 127 for e in exps]
    xh = O.dequantize(r["codes"], r["scales"], 0.0, "mxfp4")
    assert np.array_equal(xh.view(np.uint32), x.view(np.uint32))


def _mx_blocks(seed, n):
    """Blocks of 32 from several distributions: Laplace with per-channel scales (the activation
    workload's shape), Gaussian, exact E2M1 grid values times a power of two, and blocks with one
    large outlier."""
    rng = np.random.default_rng(seed)
    lap = rng.laplace(size=(n, 32)) * np.exp(rng.normal(0, 1.5, size=(1, 32)))
    gau = rng.normal(size=(n, 32))
    grid = rng.choice(GRID, size=(n, 32)) * rng.choice([-1.0, 1.0], size=(n, 32)) * 2.0 ** rng.integers(-4, 5, (n, 1))
    out = rng.normal(size=(n, 32)) * 0.1
    out[:, 0] = rng.uniform(3, 40, n)
    return np.concatenate([lap, gau, grid, out]).astype(np.float32)


def test_mx_sweep_never_prefers_a_larger_exponent():
    # Above the max rule e_c every |x| <= 6*2^e_c, and the grid at 2^(e_c+1) restricted to
    # [0, 6*2^e_c] is {0,1,2,3,4,6}*2^e_c, a subset of the grid at 2^e_c: a larger scale can only
    # tie.  The brute-force optimum over all 255 exponents therefore never exceeds e_c.
    x = _mx_blocks(11, 500)
    rule = O.mxfp4_quantize(x, sweep="rule")["scales"].astype(int)
    brute = O.mxfp4_quantize(x, sweep="brute")["scales"].astype(int)
    assert (brute <= rule).all()


@pytest.mark.parametrize("had", [False, True])
def test_mx_sweep_window_holds_the_optimum(had):
    # The window [e_c - 2, e_c] against the brute force over every exponent, on config-shaped
    # activations (Laplace, lognormal(0,1.5) channel std, outlier channels x100) and on the
    # synthetic mixtures: the optimum is always inside, and with exact errors the sweep picks it.
    w = synth.make("cfg5", rows=64, cols=8192)
    x = np.concatenate([O.widen_bf16(w["x"]).reshape(-1, 32), _mx_blocks(12, 300)])
    rule = O.mxfp4_quantize(x, hadamard=had, sweep="rule")["scales"].astype(int)
    O.inexact_count()
    sw = O.mxfp4_quantize(x, hadamard=had, sweep="sweep")["scales"].astype(int)
    assert O.inexact_count() == 0                          # the window's sums are exact
    brute = O.mxfp4_quantize(x, hadamard=had, sweep="brute")["scales"].astype(int)
    assert ((brute >= rule - 2) & (brute <= rule)).all()
    assert ((sw >= rule - 2) & (sw <= rule)).all()
    assert np.array_equal(sw, brute)                       # exact errors: the window's pick is the optimum


def test_mx_sweep_error_never_above_either_rule():
    # the exact block error of the sweep's exponent never exceeds that of either max rule, and
    # the exact errors themselves are the rational sums over the dequantized (exact) values
    x = _mx_blocks(13, 500)
    sw = O.mxfp4_quantize(x, sweep="sweep")
    es = O.mx_block_errors(x, sw["scales"])
    xs = O.dequantize(sw["codes"], sw["scales"], 0.0, "mxfp4")
    for i in range(0, len(x), 97):
        assert es[i, 0] == float(sum((Fr(float(a)) - Fr(float(b))) ** 2 for a, b in zip(x[i], xs[i])))
    for ocp in (False, True):
        er = O.mx_block_errors(x, O.mxfp4_quantize(x, sweep="rule", ocp_floor=ocp)["scales"])
        assert (es <= er).all()
        assert (es < er).any()


def _if4_blocks(seed, n):
    """Tensors of 16-element blocks for the IF4 sweep: Student-t weights (the IF4 workload's
    shape), Laplace activations with per-channel scales, and INT4 / E2M1 grid points at random
    E4M3 scales, each tensor carrying its own S."""
    rng = np.random.default_rng(seed)
    t = (rng.standard_t(4, size=(n, 64)) * 0.02).astype(np.float32)
    lap = (rng.laplace(size=(n, 64)) * np.exp(rng.normal(0, 1.5, size=(1, 64)))).astype(np.float32)
    k67 = np.float32(6.0) / np.float32(7.0)
    ints = (rng.integers(-7, 8, size=(n, 64)).astype(np.float32) * k67).astype(np.float32)
    ints *= np.float32(2.0) ** rng.integers(-3, 3, size=(n, 4)).repeat(16, axis=1).astype(np.float32)
    return [t, lap, ints]


def test_if4_sweep_window_holds_the_optimum():
    # IF4 x ScaleSweep over the MSE window against the brute force over all 127 patterns under
    # both types, on config-shaped weights and activations and on exact INT4 grids
    w4 = synth.make("cfg4", rows=8, cols=14336)
    w3 = synth.make("cfg3", rows=8, cols=4096)
    for x in [synth.as_f32(w4), synth.as_f32(w3)] + _if4_blocks(21, 64):
        sw = O.if4_quantize(x, sweep="sweep")
        bf = O.if4_quantize(x, sweep="brute")
        a = O.if4_quantize(x)
        off = (sw["scales"] & 0x7F).astype(int) - (a["scales"] & 0x7F).astype(int)
        assert ((off >= -3) & (off <= 7)).all()
        assert np.array_equal(sw["scales"], bf["scales"])
        assert np.array_equal(sw["codes"], bf["codes"])


def test_if4_sweep_dominates_if4_and_the_nvfp4_sweep():
    # The IF4 sweep's candidate set contains the NVFP4 sweep's (same FP4 errors) and IF4's own
    # (both types at p0); with exact errors its chosen error is never larger.
    w4 = synth.make("cfg4", rows=8, cols=14336)
    for x in [synth.as_f32(w4)] + _if4_blocks(22, 32):
        sw = O.if4_quantize(x, sweep="sweep")
        chosen = np.where(sw["scales"] >> 7, sw["err_int"], sw["err_fp"])
        nv = O.nvfp4_quantize(x, "sweep_mse", S=sw["S"])
        assert (chosen <= nv["err"]).all()
        a = O.if4_quantize(x, S=sw["S"])
        at_p0 = np.minimum(a["err_fp"], a["err_int"])
        assert (chosen <= at_p0).all()
        assert (chosen < nv["err"]).any() and (chosen < at_p0).any()


@pytest.mark.parametrize("rows,J", [(128, 4), (256, 64), (200, 6), (1, 1), (130, 257)])
def test_tiled_scale_layout(rows, J):
    # The consumer layout restated as NVIDIA's block-scaled GEMMs describe it: pad to 128 x 4 tiles,
    # view each tile's 128 rows as 4 groups of 32, and store (tile row, tile column, row-in-group,
    # group, column) -- a reshape and an axis permutation, independent of the oracle's loop.
    rng = np.random.default_rng(rows * 1000 + J)
    sc = rng.integers(1, 255, size=(rows, J), dtype=np.uint8)
    got = O.tile_scales(sc)
    rt, jt = (rows + 127) // 128, (J + 3) // 4
    pad = np.zeros((rt * 128, jt * 4), np.uint8)
    pad[:rows, :J] = sc
    want = pad.reshape(rt, 4, 32, jt, 4).transpose(0, 3, 2, 1, 4).ravel()
    assert np.array_equal(got, want)
    # a bijection of the padded matrix onto the buffer: every byte placed once
    ids = np.arange(rt * 128 * jt * 4).reshape(rt * 128, jt * 4)
    placed = ids.reshape(rt, 4, 32, jt, 4).transpose(0, 3, 2, 1, 4).ravel()
    assert np.array_equal(np.sort(placed), np.arange(placed.size))


def test_nvfp4_gemm_oracle():
    # against a triple loop over exact rationals on a tiny problem, and against the float64
    # product of the dequantized operands (each dequantized value is one rounding of the exact one)
    rng = np.random.default_rng(5)
    a = rng.normal(size=(3, 32)).astype(np.float32)
    b = rng.normal(size=(2, 32)).astype(np.float32)
    ra, rb = O.nvfp4_quantize(a, "sweep_mse"), O.nvfp4_quantize(b, "sweep_mse")
    d = O.nvfp4_gemm(ra["codes"], ra["scales"], ra["S"], rb["codes"], rb["scales"], rb["S"])
    def val(codes, scales, S, r, k):
        c = (int(codes[r, k // 2]) >> (4 * (k % 2))) & 0xF
        g = GRID[c & 7] * (-1 if c & 8 else 1)
        return g * E4M3[int(scales[r, k // 16])] * Fr(S)
    for m in range(3):
        for n in range(2):
            exact = sum(val(ra["codes"], ra["scales"], ra["S"], m, k) * val(rb["codes"], rb["scales"], rb["S"], n, k)
                        for k in range(32))
            assert abs(d[m, n] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))
    da = O.dequantize(ra["codes"], ra["scales"], ra["S"], "nvfp4").astype(np.float64)
    db = O.dequantize(rb["codes"], rb["scales"], rb["S"], "nvfp4").astype(np.float64)
    mag = np.abs(da) @ np.abs(db).T
    assert np.all(np.abs(d - da @ db.T) <= 2 ** -22 * mag)


def test_batch_codec_matches_the_scalar_encoders():
    # the batch codec (E4M3 by bisection) against the scalar encoders (E4M3 by a scan over all
    # patterns): every E4M3 value and midpoint and their fp32 neighbours, both signs, and random
    # values over the whole range, subnormals, saturation and infinities included
    vals = np.array([O.lib().fp4q_o_e4m3_value(p) for p in range(127)])
    pts = np.concatenate([vals, (vals[:-1] + vals[1:]) / 2, [448.0, 464.0, 480.0, 1e30, np.inf]]).astype(np.float32)
    near = np.concatenate([np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0)), pts])
    rng = np.random.default_rng(9)
    rnd = (rng.random(200000) * 2.0 ** rng.integers(-20, 12, 200000)).astype(np.float32)
    x = np.concatenate([near, rnd]).astype(np.float32)
    x = np.concatenate([x, -x])
    got = O.encode(x, "e4m3")
    ref = np.array([(0x80 if np.signbit(v) else 0) | O.lib().fp4q_o_e4m3_encode(abs(float(v))) for v in x], np.uint8)
    assert np.array_equal(got, ref)
    got = O.encode(x, "e2m1")
    assert np.array_equal(got, np.array([O.lib().fp4q_o_e2m1_encode(float(v)) for v in x], np.uint8))


def test_mxfp4_gemm_oracle():
    # against a triple loop over exact rationals (E8M0 byte b is the power of two 2^(b - 127)),
    # and against the float64 product of the dequantized operands, plain and rotated
    rng = np.random.default_rng(6)
    a = (rng.normal(size=(3, 64)) * 3).astype(np.float32)
    b = (rng.normal(size=(2, 64)) * 0.01).astype(np.float32)
    for had in (False, True):
        ra, rb = O.mxfp4_quantize(a, hadamard=had), O.mxfp4_quantize(b, hadamard=had)
        d = O.mxfp4_gemm(ra["codes"], ra["scales"], rb["codes"], rb["scales"])
        def val(codes, scales, r, k):
            c = (int(codes[r, k // 2]) >> (4 * (k % 2))) & 0xF
            g = GRID[c & 7] * (-1 if c & 8 else 1)
            return g * Fr(2) ** (int(scales[r, k // 32]) - 127)
        for m in range(3):
            for n in range(2):
                exact = sum(val(ra["codes"], ra["scales"], m, k) * val(rb["codes"], rb["scales"], n, k) for k in range(64))
                assert abs(d[m, n] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))
        da = O.dequantize(ra["codes"], ra["scales"], 0.0, "mxfp4").astype(np.float64)
        db = O.dequantize(rb["codes"], rb["scales"], 0.0, "mxfp4").astype(np.float64)
        assert np.array_equal(d, da @ db.T)   # the dequantized values are exact here


def test_hadamard_is_normalized_sylvester():
    H = np.array([[1.0]])
    while H.shape[0] < 32:
        H = np.block([[H, H], [H, -H]])
    M = np.stack([O.hadamard32(np.eye(32, dtype=np.float32)[k]) for k in range(32)], axis=1).astype(np.float64)
    KH = float(np.float32(1 / np.sqrt(32.0)))
    assert np.array_equal(M, H * KH)
    assert np.allclose(M @ M, np.eye(32), atol=1e-6)                   # involution
    rng = np.random.default_rng(1)
    for _ in range(20):
        v = rng.normal(size=32).astype(np.float32)
        ref = (H / np.sqrt(32)) @ v.astype(np.float64)
        assert np.allclose(O.hadamard32(v), ref, rtol=1e-5, atol=1e-6)


H16 = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(16)] for i in range(16)]) / 4   # closed form


def test_hadamard16_is_normalized_sylvester():
    """The 16-point rotation NVFP4/IF4 blocks take is H_16 / 4 with H_16[i][j] =
    (-1)^popcount(i & j) (Sylvester order): checked column by column, then as a matrix
    product on integer blocks (every partial sum exact), as an involution, block by block
    along a row, and within the summation error bound on random values."""
    M = np.stack([O.hadamard16(np.eye(16, dtype=np.float32)[k]) for k in range(16)], axis=1).astype(np.float64)
    assert np.array_equal(M, H16)
    rng = np.random.default_rng(3)
    x = rng.integers(-1000, 1000, size=(5, 64)).astype(np.float32)
    rx = O.rotate16(x)
    assert np.array_equal(rx.astype(np.float64), (x.astype(np.float64).reshape(5, 4, 16) @ H16.T).reshape(5, 64))
    assert np.array_equal(O.rotate16(rx), x)
    v = rng.normal(size=(64, 16)).astype(np.float32) * np.exp(rng.uniform(-20, 20, size=(64, 1))).astype(np.float32)
    got = O.rotate16(v).astype(np.float64)
    exact = v.astype(np.float64) @ H16.T
    # four levels of binary32 additions, then an exact 1/4: |error| <= 4 u sum|v| / 4 (u = 2^-24)
    bound = 4 * 2.0 ** -24 * np.abs(v.astype(np.float64)).sum(axis=1, keepdims=True) / 4 * 1.0001
    assert np.all(np.abs(got - exact) <= bound)


def _rotated_grid_tensor(seed, rows=6, cols=128):
    """x = H y blockwise (closed-form matrix, exact: multiples of 1/8 below 2^5) with y on the
    E2M1 grid and every block's largest magnitude 6."""
    rng = np.random.default_rng(seed)
    y = rng.choice([0, .5, 1, 1.5, 2, 3, 4, 6], size=(rows, cols)) * rng.choice([-1.0, 1.0], size=(rows, cols))
    y[:, rng.integers(0, 16)::16] = 6.0 * rng.choice([-1.0, 1.0], size=(rows, cols // 16))
    x = (y.reshape(rows, -1, 16) @ H16.T).reshape(rows, cols)
    return x.astype(np.float32), y.astype(np.float32)


@pytest.mark.parametrize("method", ["absmax", "four_over_six", "sweep_mse", "if4"])
def test_hadamard16_quantize_is_exact_on_rotated_grid_values(method):
    """If H x lies on the FP4 grid at scale 1 with block maxima 6, the rotated method must
    take S = 6/1536 = 2^-8 from max|H x| (max|x| is larger), pick pattern 0x78 (e = 256,
    sv = 1) in every block with zero error, reproduce H x exactly without the inverse
    rotation and x exactly with it."""
    x, y = _rotated_grid_tensor(5)
    assert np.abs(x).max() > 6.0
    fmt = "if4" if method == "if4" else "nvfp4"
    r = O.if4_quantize(x, hadamard16=True) if fmt == "if4" else O.nvfp4_quantize(x, method, hadamard16=True)
    assert r["S"] == 2.0 ** -8
    assert np.all(r["scales"] == 0x78)
    assert np.array_equal(O.dequantize(r["codes"], r["scales"], r["S"], fmt), y)
    assert np.array_equal(O.dequantize(r["codes"], r["scales"], r["S"], fmt, inverse_hadamard=True), x)
    # and the plain path on the same tensor sees max|x|, not max|H x|
    plain = O.if4_quantize(x) if fmt == "if4" else O.nvfp4_quantize(x, method)
    assert plain["S"] == np.float32(np.float32(np.abs(x).max()) / np.float32(1536))


def test_hadamard16_spreads_an_outlier():
    """One outlier c in a block becomes c/4 at all 16 positions: S = RN(RN(c/4) / 1536)."""
    x = np.zeros((2, 32), np.float32)
    x[1, 21] = -3000.0
    x[0, 2] = 7.0
    r = O.nvfp4_quantize(x, "sweep_mse", hadamard16=True)
    assert r["S"] == np.float32(np.float32(750.0) / np.float32(1536.0))
    xr = O.rotate16(x)
    assert np.all(np.abs(xr[1, 16:]) == 750.0) and np.all(xr[1, :16] == 0)


def test_exact_roundtrip_every_e2m1_x_e4m3_value():
    """With S = 1, every value q*e(p) is reproduced bit-exactly.  AbsMax reaches patterns
    1..0x78 (a_b/(6S) <= 256 by construction): a block whose max is 6*e(p) selects p and
    every code of the grid is exact.  The top patterns 0x79..0x7E (reached only through
    sweep offsets) are checked through the dequantizer: code q at scale p gives q*e(p)."""
    blocks = []
    for p in range(1, 0x79):
        e = float(E4M3[p])
        vals = [6 * e] + [s * float(g) * e for g in GRID[:7] for s in (1, -1)] + [0.0]
        blocks.append(np.array(vals[:16], np.float32))
    x = np.concatenate(blocks).reshape(1, -1)
    assert np.abs(x).max() == 1536.0
    r = O.nvfp4_quantize(x, "absmax")
    assert r["S"] == 1.0
    assert list(r["scales"][0]) == list(range(1, 0x79))
    xh = O.dequantize(r["codes"], r["scales"], r["S"], "nvfp4")
    assert np.array_equal(xh.view(np.uint32), x.view(np.uint32))
    assert np.all(r["err"] == 0.0)                    # exactly representable: error exactly 0
    rs = O.nvfp4_quantize(x, "sweep_mse")
    assert np.all(rs["err"] == 0.0)
    assert np.array_equal(O.dequantize(rs["codes"], rs["scales"], rs["S"], "nvfp4"), x)
    for p in range(0x79, 0x7F):
        codes = np.array([[k | (k << 4) for k in range(8)] + [(k | 8) | ((k | 8) << 4) for k in range(8)]], np.uint8)
        xh = O.dequantize(codes, np.array([[p, p]], np.uint8), 1.0, "nvfp4")
        want = [float(g * E4M3[p]) for g in GRID for _ in (0, 1)] + [-float(g * E4M3[p]) for g in GRID for _ in (0, 1)]
        assert list(xh[0]) == want


def _parse_golden():
    path = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.txt")
    rows = []
    for line in open(path):
        if not line.strip() or line.startswith("#"):
            continue
        f = [t.strip() for t in line.split("|")]
        rows.append((f[0], f[1], f[2], np.array(f[3].split(), np.float32), int(f[4], 16), f[5]))
    return rows


def _golden_value(tok):
    """A golden error: a decimal, or k*2^-n written as 'k/2^n' (exact)."""
    if "/2^" in tok:
        k, n = tok.split("/2^")
        return Fr(int(k), 2 ** int(n))
    return Fr(tok)


@pytest.mark.parametrize("row", _parse_golden(), ids=lambda r: r[0])
def test_hand_worked(row):
    _, method, S, xb, scale, expect_tok = row
    if method.startswith("mxfp4"):
        expect = np.array(expect_tok.split(), np.float32)
        r = O.mxfp4_quantize(xb.reshape(1, -1), ocp_floor=method.endswith("ocp"),
                             sweep="sweep" if method.endswith("sweep") else "rule")
        assert r["scales"][0, 0] == scale
        xh = O.dequantize(r["codes"], r["scales"], 0.0, "mxfp4")
        assert np.array_equal(xh[0], expect)
        return
    expect_exact = _golden_value(expect_tok)
    if method == "if6":
        r = O.if6_quantize(_tensor_with(xb, amax=1920.0))
        assert r["S"] == float(S)
        assert r["scales"][0, 0] == scale
        err = r["err_int"][0, 0] if scale & 0x80 else r["err_fp"][0, 0]
        assert err == float(expect_exact)
        # both IF6 rows dequantize to themselves (hw16's 31 K = 7.5 - 15 * 2^-26 rounds to 7.5)
        assert np.array_equal(O.if6_dequantize(r["codes"], r["scales"], r["S"])[0, :16], xb)
        return
    x = _tensor_with(xb)
    if method.startswith("if4"):
        r = O.if4_quantize(x, sweep="sweep" if method.endswith("sweep") else "absmax")
        assert r["S"] == float(S)
        assert r["scales"][0, 0] == scale
        err = r["err_int"][0, 0] if scale & 0x80 else r["err_fp"][0, 0]
        assert err == float(expect_exact)
        xh = O.dequantize(r["codes"], r["scales"], r["S"], "if4")
        assert np.array_equal(xh[0, :16], xb)    # every hand-worked IF4 block dequantizes to itself
        return
    r = O.nvfp4_quantize(x, method)
    assert r["S"] == float(S)
    assert r["scales"][0, 0] == scale
    assert r["err"][0, 0] == float(expect_exact)     # the exact block MSE


def test_status_paths():
    x = np.zeros((2, 32), np.float32)
    r = O.nvfp4_quantize(x, "sweep_mse")
    assert r["status"] == 0 and r["S"] == 0.0 and not r["scales"].any() and not r["codes"].any()
    x[0, 3] = -0.0
    assert O.nvfp4_quantize(x, "absmax")["codes"][0, 1] == 0x80      # -0 keeps its sign bit
    x[1, 5] = np.nan
    r = O.nvfp4_quantize(x, "absmax")
    assert r["status"] == O.ST_NONFINITE and np.isnan(r["S"])
    x = np.full((1, 16), 1e-35, np.float32)
    assert O.nvfp4_quantize(x, "absmax")["status"] == O.ST_RANGE
    x = np.zeros((1, 32), np.float32)
    x[0, 20] = np.inf
    r = O.mxfp4_quantize(x)
    assert r["scales"][0, 0] == 0xFF


def _nearest_bf16_bits(v: float) -> int:
    """Brute-force bf16 rounding of a finite float32: of the two bf16 values bracketing v (the
    upper 16 bits, and that pattern plus one), the nearer over exact rationals, a tie to the even
    pattern.  As IEEE rounding does, the pattern past the largest finite value stands for 2^128
    (the next value with an unbounded exponent), so magnitudes from the midpoint up overflow."""
    u = int(np.float32(v).view(np.uint32))
    lo = u >> 16
    cands = [lo, lo + 1]
    def val(b):
        if (b & 0x7F80) == 0x7F80:
            return None if (b & 0x7F) else Fr(2) ** 128 * (-1 if b & 0x8000 else 1)
        return Fr(float(np.uint32(b << 16).view(np.float32)))
    x = Fr(float(v))
    best = min(cands, key=lambda b: (abs(val(b) - x), b & 1))
    return best


def test_f32_to_bf16_is_nearest_even():
    # The bf16 output of the dequantizer: nearest with ties to even, checked against the brute
    # force above on random values of every binade (subnormals included), on exact ties (low half
    # 0x8000) and their neighbours, both signs; NaN stays a NaN and infinities stay infinite.
    rng = np.random.default_rng(17)
    r = rng.integers(0, 0xFF000000, 40000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 0x7F7F, 4000, dtype=np.uint64).astype(np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    near = np.concatenate([ties - np.uint32(1), ties + np.uint32(1)])
    bits = np.concatenate([r, ties, near, np.array([0x7F7FFFFF, 0x7F7F7FFF, 0x7F7F8000, 1, 0x8000, 0x00018000], np.uint32)])
    bits = np.concatenate([bits, bits | np.uint32(0x80000000)])
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    got = O.f32_to_bf16(x)
    want = np.array([_nearest_bf16_bits(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, want)
    special = O.f32_to_bf16(np.array([np.inf, -np.inf, np.nan], np.float32))
    assert special[0] == 0x7F80 and special[1] == 0xFF80 and (special[2] & 0x7F80) == 0x7F80 and (special[2] & 0x7F)


def test_near_tie_statistic_on_constructed_blocks():
    # hw4's block [6, 0 x 15] at S = 1 is reproduced exactly at offsets 0 and +4: an exact tie of
    # the runner-up (gap 0); [5] x 16 has a unique zero-error candidate (offset +5), so its
    # runner-up is strictly worse; an all-zero tensor has one candidate (no runner-up).
    x = _tensor_with(np.concatenate([np.array([6.0] + [0.0] * 15, np.float32), np.full(16, 5.0, np.float32)]))
    r = O.nvfp4_quantize(x, "sweep_mse")
    assert r["tie"][0, 0] and r["gap"][0, 0] == 0.0 and r["p2"][0, 0] == r["p"][0, 0] + 4
    assert not r["tie"][0, 1] and r["gap"][0, 1] > 1e-3
    st = O.near_ties(r)
    assert st["exact"] >= 1 and st["near"] >= st["exact"]
    z = O.nvfp4_quantize(np.zeros((1, 32), np.float32), "sweep_mse")
    assert np.all(np.isinf(z["gap"])) and O.near_ties(z)["with_runner_up"] == 0


def test_if4_sweep_is_the_exact_argmin():
    # IF4 x ScaleSweep: the chosen (pattern, type) is the exact lexicographic minimum of
    # (block MSE, offset, FP4 before INT4) over the window, on sampled weight blocks
    w = synth.make("cfg4", rows=2, cols=512)
    x = synth.as_f32(w)
    O.inexact_count()                      # clears counts left by earlier brute-force checks
    r = O.if4_quantize(x, sweep="sweep")
    assert O.inexact_count() == 0
    S = r["S"]
    rng = np.random.default_rng(19)
    for row, j in zip(rng.integers(0, 2, 10), rng.integers(0, 32, 10)):
        xb = x[row, j * 16:(j + 1) * 16]
        p0 = O.e4m3_encode(float(f32(np.abs(xb).max()) / (f32(6) * f32(S))))
        keys = []
        for p in range(max(p0 - 3, 0), min(p0 + 7, 0x7E) + 1):
            keys.append((exact_fp4_error(xb, p, S), p, 0))
            keys.append((exact_int4_error(xb, p, S), p, 1))
        e, p, t = min(keys)
        assert int(r["scales"][row, j]) == (p | (0x80 if t else 0))
        assert (r["err_int"] if t else r["err_fp"])[row, j] == float(e)


# ---------------------------------------------------------------------------------
# IF6: FP6 E2M3 vs scaled INT6 (Adaptive Block-Scaled Data Types, Methodology, extensibility)
# ---------------------------------------------------------------------------------
def e2m3_values_from_format():
    """FP6 E2M3 magnitudes from the bit layout: 2 exponent bits (bias 1), 3 mantissa bits,
    exponent 0 subnormal (k/8)."""
    return [Fr(c & 7, 8) if (c >> 3) == 0 else (1 + Fr(c & 7, 8)) * Fr(2) ** ((c >> 3) - 1) for c in range(32)]


E2M3 = e2m3_values_from_format()


def nearest_e2m3(y: Fr) -> int:
    a = abs(y)
    c = min(range(32), key=lambda c: (abs(a - E2M3[c]), c & 1))
    return c | (0x20 if y < 0 else 0)


def test_e2m3_value_set_and_rounding():
    assert [Fr(O.e2m3_value(c)) for c in range(32)] == E2M3
    assert max(E2M3) == Fr(15, 2) and len(set(E2M3)) == 32
    rng = np.random.default_rng(23)
    ys = np.concatenate([rng.uniform(-9, 9, 3000), [float(m) for m in E2M3],
                         [float((E2M3[c] + E2M3[c + 1]) / 2) for c in range(31)]]).astype(np.float32)
    for y in ys:
        assert O.e2m3_encode(float(y)) == nearest_e2m3(Fr(float(y))), float(y)
    assert O.e2m3_encode(100.0) == 31 and O.e2m3_encode(-0.0) == 0x20


def _exact_if6(xb, p, S):
    s = sv_of(p, S)
    inv = f32(1.0) / f32(s)
    fp = [E2M3[nearest_e2m3(Fr(float(f32(v) * inv))) & 31] for v in xb]
    K62 = f32(62.0) / f32(15.0)
    n = [min(abs(round(Fr(float(f32(f32(v) * inv) * K62)))), 31) for v in xb]
    g = Fr(float(f32(f32(15.0) / f32(62.0)) * f32(s)))
    return exact_error(xb, [m * Fr(s) for m in fp]), exact_error(xb, [k * g for k in n])


def test_if6_errors_and_choice_are_exact():
    w = synth.make("cfg4", rows=2, cols=1024)
    x = synth.as_f32(w)
    O.inexact_count()
    r = O.if6_quantize(x)
    assert O.inexact_count() == 0
    S = r["S"]
    assert S == float(f32(np.abs(x).max()) / f32(1920.0))
    rng = np.random.default_rng(29)
    ints = 0
    for row, j in zip(rng.integers(0, 2, 20), rng.integers(0, 64, 20)):
        xb = x[row, j * 16:(j + 1) * 16]
        p0 = O.e4m3_encode(float(f32(np.abs(xb).max()) / (f32(7.5) * f32(S))))
        assert int(r["scales"][row, j]) & 0x7F == p0
        ef, ei = _exact_if6(xb, p0, S)
        assert r["err_fp"][row, j] == float(ef) and r["err_int"][row, j] == float(ei)
        assert bool(r["scales"][row, j] >> 7) == (ei < ef)
        ints += ei < ef
    assert 0 < ints < 20


def test_if6_packing_and_round_trip():
    # 6-bit fields, element i at bits 6i..6i+5 of the block's 12 bytes: the dequantized values are
    # each field decoded (FP6: the E2M3 value, sign bit 5; INT6: two's complement times the INT6
    # scale) times the block scale, checked field by field against an independent bit reader
    w = synth.make("cfg3", rows=4, cols=256)
    x = synth.as_f32(w)
    r = O.if6_quantize(x)
    xh = O.if6_dequantize(r["codes"], r["scales"], r["S"])
    bits = np.unpackbits(r["codes"].reshape(4, -1, 12), axis=2, bitorder="little").reshape(4, -1, 16, 6)
    fields = (bits * (1 << np.arange(6))).sum(axis=3)
    for row in range(4):
        for j in range(16):
            sb = int(r["scales"][row, j])
            s = f32(f32(O.e4m3_value(sb & 0x7F)) * f32(r["S"]))
            for i in range(16):
                f = int(fields[row, j, i])
                if sb & 0x80:
                    n = f - 64 if f >= 32 else f
                    want = f32(f32(n) * f32(f32(f32(15.0) / f32(62.0)) * s))
                else:
                    want = f32(f32(O.e2m3_value(f) * (-1 if f & 0x20 else 1)) * s)
                assert xh[row, 16 * j + i] == want
    # a block on the FP6 grid comes back exactly
    xb = np.array([7.5, 0.125, 3.75, -1.875, 0.5, 6, 0.625, -0.375] + [0] * 8, np.float32)
    r = O.if6_quantize(_tensor_with(xb, amax=1920.0))
    assert np.array_equal(O.if6_dequantize(r["codes"], r["scales"], r["S"])[0, :16], xb)
