"""Pins of the CPU oracle against what the pages and plain mathematics fix.

Each check compares the oracle with something other than itself: values printed on the
pages, hand-derived worked examples (tests/golden/worked_examples.txt), closed forms,
exact rational brute force on tiny inputs, independent numpy formulations of the same
rounding rule, and invariants that follow from the definitions.
"""
import math
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.txt")


# ------------------------------------------------------------------------------------
# independent helpers (no oracle code)
# ------------------------------------------------------------------------------------

def e4m3_by_hand(code):
    """E4M3 value from its bit fields, written independently of the oracle."""
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return float("nan")
    return s * (m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))


E4M3_POS = np.array([e4m3_by_hand(c) for c in range(127)], np.float32)
E2M1_POS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)


def nearest_even_argmin(z, grid):
    """Nearest grid index by full argmin (float64 distances); equidistant -> even index;
    values above the last point saturate. Vectorised over z."""
    z = np.asarray(z, np.float64)
    g = np.asarray(grid, np.float64)
    d = np.abs(z[..., None] - g[None, :])
    dmin = d.min(axis=-1, keepdims=True)
    cand = d == dmin
    idx = np.arange(len(g))
    even_pick = np.where(cand & (idx % 2 == 0), idx, len(g) + 1).min(axis=-1)
    any_pick = np.where(cand, idx, len(g) + 1).min(axis=-1)
    out = np.where(cand.sum(axis=-1) > 1, even_pick, any_pick)
    out = np.where(z >= g[-1], len(g) - 1, out)
    return out


def all_positive_bf16_as_f32():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)          # +0 .. largest finite
    return (bits << 16).view(np.float32)


def to_bf16_bits(x):
    """float32 -> bf16 bit pattern, round-to-nearest-even (inputs here are exact)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    rnd = ((u >> 16) & 1) + 0x7FFF
    return ((u + rnd) >> 16).astype(np.uint16)


def load_golden():
    cases, cur = [], {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line:
            if cur:
                cases.append(cur)
                cur = {}
            continue
        if line.startswith("#"):
            continue
        k, v = line.split(":", 1)
        cur[k.strip()] = v.strip()
    if cur:
        cases.append(cur)
    return cases


def parse_floats(s):
    return np.array([float(t) for t in s.split()], np.float32)


# ------------------------------------------------------------------------------------
# number formats
# ------------------------------------------------------------------------------------

def test_e2m1_codebook_matches_page(orc):
    # qwantize "Results", "Exotic Scales": the FP4 codebook {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
    assert orc.e2m1_table().tolist() == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert [orc.e2m1_value(8 + c) for c in range(8)] == [-v for v in [0, .5, 1, 1.5, 2, 3, 4, 6]]


def test_e4m3_table_facts(orc):
    t = orc.e4m3_table()
    pos = t[1:]
    # 126 positive finite values (qwantize "Results", "Exotic Scales"), increasing.
    assert len(pos) == 126 and np.all(np.diff(t) > 0)
    # max 448; min 2^-9 with subnormals ("Is Finer Better?", Appendix F.3).
    assert pos.max() == 448.0 and pos.min() == 2.0 ** -9
    assert orc.e4m3_value(0x38) == 1.0 and orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x08) == 2.0 ** -6                  # smallest normal
    assert math.isnan(orc.e4m3_value(0x7F)) and math.isnan(orc.e4m3_value(0xFF))
    assert orc.e4m3_value(0xB8) == -1.0
    np.testing.assert_array_equal(t, E4M3_POS)
    # values used in the worked examples
    assert orc.e4m3_value(0x22) == 0.15625 and orc.e4m3_value(0x23) == 0.171875
    assert orc.e4m3_value(0x28) == 0.25


# ------------------------------------------------------------------------------------
# exhaustive element projection against independent numpy rounding
# ------------------------------------------------------------------------------------

def test_nvfp4_projection_exhaustive_bf16(orc):
    """Every finite positive bf16 weight x every E4M3 scale: the oracle's sorted-table
    projection equals an argmin-based nearest-even rounding of the IEEE float32 quotient."""
    w = all_positive_bf16_as_f32()
    for c in range(1, 127):
        s = np.float32(E4M3_POS[c])
        q, wq = orc.project_many("nvfp4", c, w)
        with np.errstate(over="ignore"):
            z = w / s                                         # IEEE float32 division
        ref = nearest_even_argmin(z, E2M1_POS)
        np.testing.assert_array_equal(q, ref, err_msg=f"scale code {c}")
        np.testing.assert_array_equal(wq, s * E2M1_POS[ref])
        qn, _ = orc.project_many("nvfp4", c, -w)              # symmetric in sign
        np.testing.assert_array_equal(qn, q)


def test_int8_projection_exhaustive_bf16(orc):
    """INT8: q = rint(fl32(|w| / fl32(v / 127))) clipped to 127 (numpy rint is
    round-half-even), w^ = fl32(q * s_eff) -- for every finite bf16 and every scale."""
    w = all_positive_bf16_as_f32()
    for c in range(1, 127):
        s_eff = np.float32(E4M3_POS[c]) / np.float32(127.0)
        q, wq = orc.project_many("int8", c, w)
        with np.errstate(over="ignore"):
            z = w / s_eff
        ref = np.minimum(np.rint(z), 127.0).astype(np.int64)
        np.testing.assert_array_equal(q.astype(np.int64), ref, err_msg=f"scale code {c}")
        np.testing.assert_array_equal(wq, ref.astype(np.float32) * s_eff)


def test_e4m3_element_projection_exhaustive_bf16(orc):
    """E4M3 elements: nearest finite E4M3 of fl32(|w| / s) with ties to even and
    saturation at 448, against argmin over the hand-decoded table."""
    w = all_positive_bf16_as_f32()
    scales = [1.0, 0.5, 3.0, 0.0011160714, 7.25e-5, 1.37, 2.0 ** -20, 448.0 / 3]
    for s in scales:
        s = np.float32(s)
        q, wq = orc.project_e4m3_many(s, w)
        with np.errstate(over="ignore"):
            z = w / s
        ref = np.empty(len(w), np.int64)
        for i0 in range(0, len(w), 4096):
            ref[i0:i0 + 4096] = nearest_even_argmin(z[i0:i0 + 4096], E4M3_POS)
        np.testing.assert_array_equal(q.astype(np.int64), ref, err_msg=f"scale {s}")
        np.testing.assert_array_equal(wq, s * E4M3_POS[ref])


def test_e4m3_snap_matches_argmin(orc):
    """RNE onto the E4M3 grid (the naive snap) equals a full argmin with even ties on a
    dense sweep including every midpoint between neighbouring E4M3 values."""
    mids = (E4M3_POS[1:].astype(np.float64) + E4M3_POS[:-1]) / 2
    xs = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                         np.nextafter(mids.astype(np.float32), np.float32(1e9)),
                         np.geomspace(1e-5, 1e3, 20000), [448, 464, 500, 1e30, 0.0]])
    xs = xs.astype(np.float32)
    got = np.array([orc.lib().orc_e4m3_rne_code(float(x)) for x in xs])
    np.testing.assert_array_equal(got, nearest_even_argmin(xs, E4M3_POS))


# ------------------------------------------------------------------------------------
# worked examples and closed forms
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("case", load_golden(), ids=lambda c: c["case"])
def test_worked_examples(orc, case):
    fmt, mode, B = case["fmt"], case["mode"], int(case["block"])
    w = parse_floats(case["w"]).reshape(1, -1)
    if mode == "fixed":
        c = int(case["scale"], 16)
        nib = []
        for x in w[0]:
            q, _ = orc.project(fmt, c, float(x))
            nib.append((8 if math.copysign(1, x) < 0 else 0) | q)
        got = bytes((nib[2 * i] | nib[2 * i + 1] << 4) for i in range(len(nib) // 2))
        assert got.hex() == case["codes"].replace(" ", "")
        return
    h = parse_floats(case["h"]) if "h" in case else None
    sfmt = case.get("sfmt", "e4m3")
    r = orc.quantize(w, fmt, mode, B, h=h, sfmt=sfmt)
    assert int(r.scales[0, 0]) == int(case["scale"], 16)
    if "codes" in case:
        assert bytes(r.codes[0]).hex() == case["codes"].replace(" ", "")
    if "best" in case:
        assert r.best[0, 0] == float(case["best"])
    if "second" in case:
        assert r.second[0, 0] == float(case["second"])
    if "sse" in case:
        What = orc.dequant(r.codes, r.scales, fmt, B, 1, w.shape[1], sfmt=sfmt)
        m = orc.metrics(orc.error_sums(w, What))
        assert m["sse"] == float(case["sse"])
        if "weight_rel" in case:
            assert m["weight_rel"] == float(case["weight_rel"])


def test_naive_is_amax_closed_form(orc):
    """Naive NVFP4 scale = RNE_E4M3(fl32(amax / 6)); INT8 stored amax = RNE_E4M3(amax)
    ("Is Finer Better?", sec. 2.1; qwantize "Results", INT8 section)."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((32, 256)) * np.exp(rng.normal(-3, 2, (32, 1)))).astype(np.float32)
    for fmt, B, C in (("nvfp4", 16, 6.0), ("int8", 32, None)):
        r = orc.quantize(W, fmt, "naive", B)
        amax = np.abs(W.reshape(32, -1, B)).max(axis=-1)
        t = amax / np.float32(C) if C else amax
        ref = nearest_even_argmin(t.astype(np.float32), E4M3_POS)
        np.testing.assert_array_equal(r.scales.astype(np.int64), ref)
        np.testing.assert_array_equal(r.naive.astype(np.int64), ref)


def test_act_sqmean_closed_form(orc):
    """h_j = (1/R) sum_r x_rj^2 ("quantization_algorithms.txt", sec. 1), on integer data
    where every sum is exact; bf16 and float32 inputs, threaded and not."""
    rng = np.random.default_rng(1)
    X = rng.integers(-9, 10, size=(64, 48)).astype(np.float32)
    ref = (X.astype(np.float64) ** 2).sum(axis=0) / 64
    np.testing.assert_array_equal(orc.act_sqmean(X), ref.astype(np.float32))
    np.testing.assert_array_equal(orc.act_sqmean(to_bf16_bits(X)), ref.astype(np.float32))
    np.testing.assert_array_equal(orc.act_sqmean(X, n_threads=3), ref.astype(np.float32))
    # a non-power-of-two row count: exact rational mean, rounded once
    X3 = X[:37]
    s = (X3.astype(np.int64) ** 2).sum(axis=0)
    ref3 = np.array([float(Fr(int(v), 37)) for v in s], np.float64).astype(np.float32)
    np.testing.assert_array_equal(orc.act_sqmean(X3), ref3)


def test_output_error_closed_forms(orc):
    """||X What^T - X W^T||_F / ||X W^T||_F (qwantize "Results", metric definitions)."""
    X = np.array([[1, 0], [0, 1]], np.float32)
    W = np.array([[1, 2]], np.float32)
    assert orc.output_error(X, W, np.array([[1, 1]], np.float32)) == pytest.approx(1 / 5 ** .5,
                                                                                  rel=1e-15)
    rng = np.random.default_rng(2)
    X = rng.standard_normal((16, 32)).astype(np.float32)
    W = rng.standard_normal((8, 32)).astype(np.float32)
    assert orc.output_error(X, W, W) == 0.0
    assert orc.output_error(X, W, 2 * W) == pytest.approx(1.0, rel=1e-14)
    assert orc.output_error(X, W, np.zeros_like(W)) == pytest.approx(1.0, rel=1e-14)


def test_error_sums_closed_form(orc):
    W = np.array([[1, -2, 3, 0]], np.float32)
    What = np.array([[1, -1, 2, 1]], np.float32)
    h = np.array([1, 2, 3, 4], np.float32)
    s = orc.error_sums(W, What, h)
    assert s.tolist() == [0 + 1 + 1 + 1, 1 + 4 + 9, 0 + 2 + 3 + 4, 1 + 8 + 27]
    m = orc.metrics(s)
    assert m["weight_rel"] == pytest.approx((3 / 14) ** .5) and m["h_rel"] == pytest.approx(
        (9 / 36) ** .5)


# ------------------------------------------------------------------------------------
# exact rational brute force on tiny inputs
# ------------------------------------------------------------------------------------

def exact_errors_1d(w, c, fmt):
    """Every candidate's exact block error (Fractions). The only float step is the one
    the definition fixes: the IEEE float32 quotient (and, for INT8, the float32 effective
    scale and dequantised product)."""
    errs = []
    a = np.abs(w).astype(np.float32)
    for code in range(1, 127):
        if fmt == "nvfp4":
            s = np.float32(E4M3_POS[code])
            z = a / s
            q = nearest_even_argmin(z, E2M1_POS)
            wq = [Fr(float(s)) * Fr(float(E2M1_POS[i])) for i in q]   # exact: <= 6 bits
        else:
            s = np.float32(E4M3_POS[code]) / np.float32(127)
            z = a / s
            q = np.minimum(np.rint(z), 127)
            wq = [Fr(float(np.float32(qi) * s)) for qi in q]
        e = sum(Fr(float(cj)) * (Fr(float(aj)) - wj) ** 2 for aj, cj, wj in zip(a, c, wq))
        errs.append(e)
    return errs


def tiny_blocks(B, rng):
    blocks = [np.ones(B, np.float32), np.zeros(B, np.float32),
              np.array([0.5 * (i % 3) for i in range(B)], np.float32)]
    one = np.zeros(B, np.float32)
    one[3] = -0.3
    blocks.append(one)
    for _ in range(6):
        x = rng.standard_normal(B) * np.exp(rng.normal(-3, 0.5))
        blocks.append((to_bf16_bits(x.astype(np.float32)).astype(np.uint32) << 16).view(np.float32))
    return blocks


@pytest.mark.parametrize("fmt,B", [("nvfp4", 16), ("nvfp4", 32), ("int8", 32)])
@pytest.mark.parametrize("mode", ["sse", "hopt"])
def test_search_equals_exact_bruteforce(orc, fmt, B, mode):
    rng = np.random.default_rng(11 + B)
    h = np.exp(rng.normal(0, 1, B)).astype(np.float32) if mode == "hopt" else None
    c = h if h is not None else np.ones(B, np.float32)
    for blk in tiny_blocks(B, rng):
        r = orc.quantize(blk.reshape(1, -1), fmt, mode, B, h=h)
        errs = exact_errors_1d(blk, c, fmt)
        e1 = min(errs)
        star = 1 + errs.index(e1)                       # lowest index on exact ties
        rest = sorted(errs)[1]
        near = (rest - e1) <= Fr(1, 10 ** 12) * e1
        if not near:
            assert int(r.scales[0, 0]) == star
        else:                                           # exact ties must still resolve low
            ties = [i + 1 for i, e in enumerate(errs) if e == e1]
            if len(ties) > 1 and rest == e1:
                assert int(r.scales[0, 0]) == ties[0]
        assert r.best[0, 0] == pytest.approx(float(e1), rel=1e-13, abs=1e-300)


@pytest.mark.parametrize("fmt,B", [("nvfp4", 16), ("int8", 32)])
def test_window_bounds_exact(orc, fmt, B):
    """Bounded search: candidates are the E4M3 codes [c0 - w, c0 + w] clipped to [1, 126]
    around the naive code c0 (qwantize "Results", INT8 section); checked for several w
    against the exact errors of every candidate."""
    rng = np.random.default_rng(21 + B)
    c = np.ones(B, np.float32)
    for blk in tiny_blocks(B, rng)[3:]:
        errs = exact_errors_1d(blk, c, fmt)
        amax = float(np.abs(blk).max())
        c0 = orc.naive_code(fmt, amax)
        for w in (0, 1, 2, 3, 8):
            lo, hi = max(1, c0 - w), min(126, c0 + w)
            if c0 == 0:
                lo, hi = 1, max(1, w)
            sub = errs[lo - 1:hi]
            star = lo + sub.index(min(sub))
            r = orc.quantize(blk.reshape(1, -1), fmt, "sse", B, window=w)
            assert int(r.scales[0, 0]) == star, (w, c0)
            assert r.best[0, 0] == pytest.approx(float(min(sub)), rel=1e-13, abs=1e-300)


def exact_tile_errors(W, h, points, lo, hi):
    a = np.abs(W).astype(np.float32)
    amax = a.max()
    base = np.float32(amax) / np.float32(448)
    g = np.array([2.0 ** (lo + (hi - lo) * p / (points - 1)) for p in range(points)], np.float32)
    errs = []
    for p in range(points):
        s = np.float32(base * g[p])
        z = a / s
        q = nearest_even_argmin(z.ravel(), E4M3_POS).reshape(z.shape)
        wq = np.float32(s) * E4M3_POS[q]
        e = Fr(0)
        for i in range(W.shape[0]):
            for j in range(W.shape[1]):
                e += Fr(float(h[j])) * (Fr(float(a[i, j])) - Fr(float(wq[i, j]))) ** 2
        errs.append(e)
    return errs, g, base


def test_log_grid_and_tile_search_exact(orc):
    """Tile-scale search on a logarithmic grid ("quantization_algorithms.txt", sec. 1):
    grid endpoints 2^-2 and 2^2, and the searched tile scale against exact brute force."""
    g = orc.log_grid(64, -2.0, 2.0)
    assert g[0] == 0.25 and g[-1] == 4.0 and np.all(np.diff(g) > 0) and len(g) == 64
    assert g[21] == np.float32(2.0 ** (-2 + 4 * 21 / 63))
    rng = np.random.default_rng(3)
    T, P = 4, 9
    for trial in range(6):
        W = (rng.standard_t(4, (T, T)) * 0.05).astype(np.float32)
        h = np.exp(rng.normal(0, 1, T)).astype(np.float32)
        r = orc.quantize(W, "e4m3", "hopt", T, h=h, points=P, lo=-2.0, hi=2.0)
        errs, gref, base = exact_tile_errors(W, h, P, -2.0, 2.0)
        np.testing.assert_array_equal(orc.log_grid(P, -2.0, 2.0), gref)
        e1 = min(errs)
        star = errs.index(e1)
        if (sorted(errs)[1] - e1) > Fr(1, 10 ** 12) * e1:
            assert int(r.naive[0, 0]) == star
            assert r.scales[0, 0] == np.float32(base * gref[star])
        assert r.best[0, 0] == pytest.approx(float(e1), rel=1e-13)
        assert r.second[0, 0] == pytest.approx(float(sorted(errs)[1]), rel=1e-13)
        # naive tile scale: fl32(amax / 448)
        rn = orc.quantize(W, "e4m3", "naive", T)
        assert rn.scales[0, 0] == np.float32(np.abs(W).max()) / np.float32(448)


# ------------------------------------------------------------------------------------
# invariants of the definitions
# ------------------------------------------------------------------------------------

def synthetic(n, k, seed):
    rng = np.random.default_rng(seed)
    sig = np.exp(rng.normal(-3, 0.5, (n, 1)))
    W = rng.standard_normal((n, k)) * sig
    W[:, rng.permutation(k)[:2]] *= 20
    return to_bf16_bits(W.astype(np.float32))


def block_errors(orc, W, r, fmt, B, c):
    n, k = W.shape
    What = orc.dequant(r.codes, r.scales, fmt, B, n, k).astype(np.float64)
    d = orc.to_float(W).astype(np.float64) - What
    return (c[None, :] * d * d).reshape(n, k // B, B).sum(axis=-1)


@pytest.mark.parametrize("fmt,B,window", [("nvfp4", 16, -1), ("nvfp4", 32, -1),
                                          ("int8", 64, 8)])
def test_search_invariants(orc, fmt, B, window):
    W = synthetic(24, 512, 7)
    rng = np.random.default_rng(8)
    h = np.exp(rng.normal(0, 1, 512)).astype(np.float32)
    ones = np.ones(512, np.float32)
    rn = orc.quantize(W, fmt, "naive", B)
    rs = orc.quantize(W, fmt, "sse", B, window=window)
    rh = orc.quantize(W, fmt, "hopt", B, h=h, window=window)
    r1 = orc.quantize(W, fmt, "hopt", B, h=ones, window=window)
    # SSE-optimal never exceeds naive (the naive scale is a candidate).
    en = block_errors(orc, W, rn, fmt, B, ones.astype(np.float64))
    es = block_errors(orc, W, rs, fmt, B, ones.astype(np.float64))
    assert np.all(es <= en * (1 + 1e-12))
    np.testing.assert_allclose(rs.best, es, rtol=1e-12)
    # H-optimal with h = 1 is SSE-optimal, bit for bit.
    for key in ("codes", "scales", "best", "second"):
        np.testing.assert_array_equal(r1[key], rs[key])
    # H-optimal minimises the h-weighted error; SSE the plain one.
    hs = block_errors(orc, W, rs, fmt, B, h.astype(np.float64))
    hh = block_errors(orc, W, rh, fmt, B, h.astype(np.float64))
    assert np.all(hh <= hs * (1 + 1e-12))
    es_h = block_errors(orc, W, rh, fmt, B, ones.astype(np.float64))
    assert np.all(es <= es_h * (1 + 1e-12))
    # the window always contains the naive code
    if window >= 0:
        assert np.all(np.abs(rs.scales.astype(int) - rn.scales.astype(int)) <= window)


def test_window_equals_full_when_optimum_inside(orc):
    W = synthetic(32, 512, 9)
    for fmt, B in (("nvfp4", 16), ("int8", 32)):
        full = orc.quantize(W, fmt, "sse", B, window=-1)
        win = orc.quantize(W, fmt, "sse", B, window=8)
        inside = np.abs(full.scales.astype(int) - full.naive) <= 8
        assert inside.mean() > 0.5
        np.testing.assert_array_equal(win.scales[inside], full.scales[inside])
        np.testing.assert_array_equal(win.best[inside], full.best[inside])


def test_tile_h_one_equals_sse(orc):
    rng = np.random.default_rng(4)
    W = to_bf16_bits((rng.standard_t(4, (128, 128)) * 0.05).astype(np.float32))
    a = orc.quantize(W, "e4m3", "sse", 64)
    b = orc.quantize(W, "e4m3", "hopt", 64, h=np.ones(128, np.float32))
    for key in ("codes", "scales", "best", "naive"):
        np.testing.assert_array_equal(a[key], b[key])


def test_dequant_agrees_with_search_errors(orc):
    """The error the search minimised equals the error of the dequantised block."""
    W = synthetic(8, 256, 12)
    rng = np.random.default_rng(13)
    h = np.exp(rng.normal(0, 1, 256)).astype(np.float32)
    for fmt, B in (("nvfp4", 16), ("int8", 64)):
        r = orc.quantize(W, fmt, "hopt", B, h=h)
        np.testing.assert_allclose(block_errors(orc, W, r, fmt, B, h.astype(np.float64)),
                                   r.best, rtol=1e-12)


def test_zero_and_tiny_blocks(orc):
    """A naive scale that rounds to zero zeroes the block ("Is Finer Better?", App. F.3);
    an all-zero block under search ties everywhere and takes the smallest scale."""
    W = np.zeros((1, 32), np.float32)
    W[0, :16] = 1e-5
    W[0, 5] = -1e-5
    r = orc.quantize(W, "nvfp4", "naive", 16)
    assert r.scales[0, 0] == 0 and r.codes[0, 2] == 0x80 and r.codes[0, 0] == 0
    assert r.scales[0, 1] == 0 and np.all(r.codes[0, 8:] == 0)
    rs = orc.quantize(W, "nvfp4", "sse", 16)
    assert rs.scales[0, 1] == 1 and rs.best[0, 1] == 0 and rs.second[0, 1] == 0
    assert rs.scales[0, 0] >= 1
