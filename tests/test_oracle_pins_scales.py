"""Pins of the oracle's other block-scale grids (UE4M4, UE5M3, UE8M0) and INT4 elements.

Sources: qwantize "Results", sections "MXFP4 (UE8M0 power-of-2 scales)", "Exotic Scales",
"GPTQ Quantization" (the NVINT4 rows) and "Larger blocks" (INT4 symmetric 0..7); "Is Finer
Better? The Limits of Microscaling Formats in LLMs", sec. 2.1 (OCP E8M0 scales).

Each check compares the oracle with something other than itself: the values the pages
print (maxima, counts), bit-field decodings written here, an independent numpy rounding
rule, exact rational brute force on tiny blocks, and invariants (grid inclusions).
"""
import math
from fractions import Fraction as Fr

import numpy as np
import pytest

from tests.test_oracle_pins import (E2M1_POS, E4M3_POS, all_positive_bf16_as_f32,
                                    nearest_even_argmin, synthetic, to_bf16_bits)


def ue4m4_by_hand(code):
    e, m = code >> 4, code & 15
    return m / 16 * 2.0 ** -6 if e == 0 else (1 + m / 16) * 2.0 ** (e - 7)


def ue5m3_by_hand(code):
    e, m = code >> 3, code & 7
    return m / 8 * 2.0 ** -14 if e == 0 else (1 + m / 8) * 2.0 ** (e - 15)


def ue8m0_by_hand(code):
    return 2.0 ** (code - 127)


HAND = {"ue4m4": [ue4m4_by_hand(c) for c in range(256)],
        "ue5m3": [ue5m3_by_hand(c) for c in range(256)],
        "ue8m0": [ue8m0_by_hand(c) for c in range(255)],
        "e4m3": [float(v) for v in E4M3_POS]}
FIRST = {"e4m3": 1, "ue4m4": 1, "ue5m3": 1, "ue8m0": 0}
INT4_POS = np.arange(8, dtype=np.float32)


# ------------------------------------------------------------------------------------
# tables
# ------------------------------------------------------------------------------------

def test_scale_tables_match_bit_fields_and_page_facts(orc):
    for sfmt, vals in HAND.items():
        t = orc.scale_table(sfmt)
        assert t.tolist() == [float(np.float32(v)) for v in vals], sfmt
        assert np.all(np.diff(t.astype(np.float64)) > 0), sfmt          # sorted by code
    # "Exotic Scales": 255 distinct positive values each, max about 496 and 122880.
    ue44, ue53 = orc.scale_table("ue4m4"), orc.scale_table("ue5m3")
    assert (ue44 > 0).sum() == 255 and (ue53 > 0).sum() == 255
    assert ue44[-1] == 496.0 and ue53[-1] == 122880.0
    assert ue44[1] == 2.0 ** -10 and ue53[1] == 2.0 ** -17
    # "MXFP4": consecutive UE8M0 scales differ by a factor of 2; OCP E8M0 2^-127 .. 2^127.
    u8 = orc.scale_table("ue8m0").astype(np.float64)
    assert np.all(u8[1:] / u8[:-1] == 2.0) and u8[0] == 2.0 ** -127 and u8[-1] == 2.0 ** 127
    assert math.isnan(orc.scale_value("ue8m0", 255))


def test_grid_inclusions(orc):
    """UE4M4 adds a mantissa bit to E4M3 and UE5M3 an exponent bit: both contain every
    E4M3 value; E4M3's powers of two are UE8M0 values."""
    e4 = set(orc.e4m3_table().tolist())
    assert e4 <= set(orc.scale_table("ue4m4").tolist())
    assert e4 <= set(orc.scale_table("ue5m3").tolist())
    pow2 = {v for v in e4 if v > 0 and math.frexp(v)[0] == 0.5}
    assert len(pow2) == 18 and pow2 <= set(orc.scale_table("ue8m0").tolist())


# ------------------------------------------------------------------------------------
# projections (exhaustive over positive bf16 values, sampled scale codes)
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,sfmt", [("nvfp4", "ue4m4"), ("nvfp4", "ue5m3"),
                                      ("nvfp4", "ue8m0"), ("int4", "e4m3"), ("int4", "ue4m4")])
def test_projection_exhaustive_bf16(orc, fmt, sfmt):
    w = all_positive_bf16_as_f32()
    grid = E2M1_POS if fmt == "nvfp4" else INT4_POS
    tab = np.array(HAND[sfmt], np.float32)
    codes = sorted(set(range(FIRST[sfmt], len(tab), 9)) | {FIRST[sfmt], len(tab) - 1})
    for c in codes:
        s = np.float32(tab[c])
        with np.errstate(over="ignore"):
            z = w / s                                   # IEEE float32 quotient
        q_ref = nearest_even_argmin(z, grid)
        q, wq = orc.project_many(fmt, c, w, sfmt=sfmt)
        assert np.array_equal(q, q_ref), (sfmt, c)
        with np.errstate(over="ignore"):
            assert np.array_equal(wq, grid[q_ref] * s), (sfmt, c)


# ------------------------------------------------------------------------------------
# naive scales
# ------------------------------------------------------------------------------------

def test_naive_closed_forms(orc):
    amaxes = [0.0, 2.0 ** -130, 1e-30, 0.75, 1.0, 5.999, 6.0, 7.0, 7.999, 8.0, 448.0, 1e30,
              3e38]
    for a in amaxes:
        a32 = float(np.float32(a))
        # MXFP4: OCP 2^(floor(log2 amax) - 2), clamped to the E8M0 codes 0 .. 254.
        if a32 == 0:
            want = 0
        else:
            fl = math.frexp(a32)[1] - 1                 # floor(log2 a), exact
            want = min(max(fl - 2 + 127, 0), 254)
        assert orc.naive_code("nvfp4", a32, sfmt="ue8m0") == want, a
        # NVINT4: nearest E4M3 value to fl32(amax / 7); E2M1 on UE grids: amax / 6.
        z7 = np.float32(a32) / np.float32(7)
        assert orc.naive_code("int4", a32) == int(nearest_even_argmin([z7], E4M3_POS)[0])
        z6 = np.float32(a32) / np.float32(6)
        for sfmt in ("ue4m4", "ue5m3"):
            g = np.array(HAND[sfmt], np.float32)
            assert orc.naive_code("nvfp4", a32, sfmt=sfmt) == int(nearest_even_argmin([z6], g)[0])
            assert orc.naive_code("int4", a32, sfmt=sfmt) == int(nearest_even_argmin([z7], g)[0])
    assert orc.naive_code("nvfp4", 6.0, sfmt="ue8m0") == 127       # s = 1: 6 maps to 6
    assert orc.naive_code("nvfp4", 8.0, sfmt="ue8m0") == 128       # s = 2


# ------------------------------------------------------------------------------------
# exact rational brute force on tiny blocks
# ------------------------------------------------------------------------------------

def exact_errors(w, c, fmt, sfmt):
    """Every candidate's exact block error (Fractions), candidates in code order. Float
    steps: the IEEE float32 quotient only (dequantised products are exact here)."""
    grid = E2M1_POS if fmt == "nvfp4" else INT4_POS
    tab = np.array(HAND[sfmt], np.float32)
    a = np.abs(w).astype(np.float32)
    errs = []
    for code in range(FIRST[sfmt], len(tab)):
        s = np.float32(tab[code])
        with np.errstate(over="ignore"):
            q = nearest_even_argmin(a / s, grid)
        wq = [Fr(float(s)) * Fr(float(grid[i])) for i in q]
        errs.append(sum(Fr(float(cj)) * (Fr(float(aj)) - wj) ** 2
                        for aj, cj, wj in zip(a, c, wq)))
    return errs


def tiny(B, rng):
    out = [np.full(B, 2.0, np.float32), np.linspace(-1, 1, B).astype(np.float32)]
    for _ in range(5):
        x = rng.standard_normal(B) * np.exp(rng.normal(-3, 1.0))
        out.append((to_bf16_bits(x.astype(np.float32)).astype(np.uint32) << 16).view(np.float32))
    return out


@pytest.mark.parametrize("fmt,sfmt,B", [("nvfp4", "ue8m0", 16), ("nvfp4", "ue8m0", 32),
                                        ("nvfp4", "ue4m4", 16), ("nvfp4", "ue5m3", 16),
                                        ("int4", "e4m3", 16), ("int4", "ue4m4", 16)])
@pytest.mark.parametrize("mode", ["sse", "hopt"])
def test_search_equals_exact_bruteforce(orc, fmt, sfmt, B, mode):
    rng = np.random.default_rng(31 + B)
    h = np.exp(rng.normal(0, 1, B)).astype(np.float32) if mode == "hopt" else None
    c = h if h is not None else np.ones(B, np.float32)
    for blk in tiny(B, rng):
        r = orc.quantize(blk.reshape(1, -1), fmt, mode, B, h=h, sfmt=sfmt)
        errs = exact_errors(blk, c, fmt, sfmt)
        e1 = min(errs)
        star = FIRST[sfmt] + errs.index(e1)             # lowest code among exact ties
        assert int(r.scales[0, 0]) == star, (sfmt, blk[:4])
        assert r.best[0, 0] == pytest.approx(float(e1), rel=1e-13, abs=1e-300)


def test_window_in_code_space(orc):
    """A window of w codes around the naive code, clipped to the grid's candidate codes."""
    rng = np.random.default_rng(5)
    c = np.ones(16, np.float32)
    for sfmt in ("ue8m0", "ue4m4"):
        for blk in tiny(16, rng)[1:]:
            errs = exact_errors(blk, c, "nvfp4", sfmt)
            c0 = orc.naive_code("nvfp4", float(np.abs(blk).max()), sfmt=sfmt)
            for w in (0, 1, 3):
                top = len(HAND[sfmt]) - 1
                lo, hi = max(FIRST[sfmt], c0 - w), min(top, c0 + w)
                sub = errs[lo - FIRST[sfmt]:hi - FIRST[sfmt] + 1]
                r = orc.quantize(blk.reshape(1, -1), "nvfp4", "sse", 16, window=w, sfmt=sfmt)
                assert int(r.scales[0, 0]) == lo + sub.index(min(sub)), (sfmt, w)


# ------------------------------------------------------------------------------------
# invariants
# ------------------------------------------------------------------------------------

def test_denser_grids_never_lose(orc):
    """UE4M4 and UE5M3 contain every E4M3 value, so their best block error is at most
    E4M3's (the same double arithmetic on the same scale values)."""
    W = synthetic(16, 512, 17)
    h = np.exp(np.random.default_rng(18).normal(0, 1, 512)).astype(np.float32)
    for mode in ("sse", "hopt"):
        for fmt in ("nvfp4", "int4"):
            base = orc.quantize(W, fmt, mode, 16, h=h)
            for sfmt in ("ue4m4", "ue5m3"):
                r = orc.quantize(W, fmt, mode, 16, h=h, sfmt=sfmt)
                assert np.all(r.best <= base.best), (fmt, sfmt, mode)
                # and strictly better in many blocks: UE4M4 everywhere (twice as dense),
                # UE5M3 where E4M3 is subnormal (below 2^-6, spaced 2^-9)
                assert np.mean(r.best < base.best) > (0.4 if sfmt == "ue4m4" else 0.2)


def test_mxfp4_equals_e4m3_powers_of_two(orc):
    """Restricted to the scales both grids share (the powers of two 2^-9 .. 2^8), the
    UE8M0 search and a search over E4M3's power-of-two codes agree block by block."""
    W = synthetic(8, 256, 19)
    r8 = orc.quantize(W, "nvfp4", "sse", 16, sfmt="ue8m0")
    e4_pow2 = [c for c in range(1, 127) if math.frexp(float(E4M3_POS[c]))[0] == 0.5]
    Wf = orc.to_float(W)
    for i in range(W.shape[0]):
        for b in range(W.shape[1] // 16):
            blk = Wf[i, 16 * b:16 * b + 16]
            s8 = float(orc.scale_table("ue8m0")[r8.scales[i, b]])
            if not (2.0 ** -9 <= s8 <= 2.0 ** 8):
                continue
            errs = {}
            for c in e4_pow2:
                _, wq = orc.project_many("nvfp4", c, blk)
                d = np.abs(blk).astype(np.float64) - wq.astype(np.float64)
                errs[c] = float(np.sum(d * d))
            best_c = min(errs, key=lambda c: (errs[c], c))
            assert float(E4M3_POS[best_c]) == s8
            assert errs[best_c] == pytest.approx(r8.best[i, b], rel=1e-12, abs=1e-300)


def test_int4_dequant_signed_nibbles(orc):
    """INT4 codes are two's-complement nibbles: 0x9 = -7, 0xF = -1, 0x7 = 7."""
    codes = np.array([[0x97, 0x1F] + [0] * 6], np.uint8)
    scales = np.array([[0x38]], np.uint8)                 # E4M3 1.0
    out = orc.dequant(codes, scales, "int4", 16, 1, 16)
    assert out[0, :4].tolist() == [7.0, -7.0, -1.0, 1.0] and np.all(out[0, 4:] == 0)
    r = orc.quantize(out, "int4", "naive", 16)
    assert r.scales[0, 0] == 0x38 and bytes(r.codes[0]).hex() == bytes(codes[0]).hex()


def test_zero_block_takes_first_candidate(orc):
    """An all-zero block has zero error at every scale; ties go to the first candidate
    code: UE8M0 code 0 (2^-127, a nonzero scale), code 1 on grids whose code 0 is zero."""
    W = np.zeros((1, 32), np.float32)
    for fmt, sfmt, first in (("nvfp4", "ue8m0", 0), ("nvfp4", "ue4m4", 1),
                             ("nvfp4", "ue5m3", 1), ("int4", "e4m3", 1)):
        r = orc.quantize(W, fmt, "sse", 16, sfmt=sfmt)
        assert r.scales.tolist() == [[first, first]] and np.all(r.best == 0), sfmt
        assert np.all(r.codes == 0)
    rn = orc.quantize(W, "nvfp4", "naive", 16, sfmt="ue8m0")
    assert rn.scales.tolist() == [[0, 0]]


def test_swizzled_scale_layout(orc):
    """128 x 4 tiles of 512 bytes; in a tile row m, column c at (m % 32) 16 + (m / 32) 4 + c;
    tiles by row tile, then column tile; zero padding. Hand-placed entries and a bijection."""
    n, kb = 300, 10                                   # 3 row tiles, 3 column tiles (padded)
    s = (np.arange(n * kb) % 251 + 1).astype(np.uint8).reshape(n, kb)
    out = orc.swizzle_scales(s)
    assert out.size == 384 * 12
    assert out[0] == s[0, 0] and out[1] == s[0, 1] and out[3] == s[0, 3]
    assert out[16] == s[1, 0] and out[4] == s[32, 0] and out[15 * 16 + 3 * 4 + 2] == s[111, 2]
    assert out[512] == s[0, 4]                        # next column tile
    assert out[3 * 512 + 5 * 16] == s[133, 0]         # second row tile, row 5 of it
    assert out[2 * 512 + 0 * 16 + 1] == s[0, 9]       # column 9 = tile 2, column 1
    assert out[2 * 512 + 2] == 0                      # padded column 10
    nz = out[out != 0]
    assert sorted(nz.tolist()) == sorted(s.reshape(-1).tolist())
