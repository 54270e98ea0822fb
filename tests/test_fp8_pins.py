"""Pins of the oracle's FP8 (e4m3) table arithmetic and of the e4m3 input generator.

The pages store bf16 rows; e4m3 tables with one dequantisation scale per table are the
widening of the row gather taken here.  Everything below is checked against facts that do
not come from the oracle's own formula: the OCP FP8 E4M3 definition's landmark values,
torch's float8_e4m3fn conversion (a library routine), exact rational arithmetic with a
nearest-value search over every bf16, and a nearest-code search over every e4m3 code.
"""
from __future__ import annotations

import bisect
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

ALL_CODES = np.arange(256, dtype=np.uint8)


def _is_nan_code(c: int) -> bool:
    return (c & 0x7F) == 0x7F


# ------------------------------------------------------------------------ decode
def test_e4m3_landmarks_of_the_format():
    """Values fixed by the E4M3 definition (bias 7, 3 mantissa bits, no infinities)."""
    d = oracle.e4m3_to_double
    assert d(0x00) == 0.0 and d(0x80) == 0.0
    assert d(0x38) == 1.0 and d(0xB8) == -1.0              # exponent field 7 = 2^0
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0          # largest finite
    assert d(0x08) == 2.0 ** -6                            # smallest normal
    assert d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9   # subnormals
    assert d(0x40) == 2.0 and d(0x3C) == 1.5
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))


def test_e4m3_decode_matches_torch_float8():
    torch = pytest.importorskip("torch")
    if not hasattr(torch, "float8_e4m3fn"):
        pytest.skip("torch without float8_e4m3fn")
    ref = torch.from_numpy(ALL_CODES.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_double(int(c)) for c in ALL_CODES])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and nan.sum() == 2
    assert np.array_equal(ref[~nan], got[~nan])
    # the 254 finite codes are 253 distinct values (+0 and -0 compare equal) and monotone
    pos = got[:0x7F]
    assert np.all(np.diff(pos) > 0)


# ------------------------------------------------------------------------ dequantisation
def _finite_bf16_values():
    pats = np.arange(0x0000, 0x7F80, dtype=np.uint16)          # +0 .. largest finite
    vals = synth.bf16_to_float(pats).astype(np.float64)
    return [Fraction(float(v)) for v in vals], pats


_BF16_POS = None


def _nearest_bf16_exact(x: Fraction) -> int:
    """Nearest bf16 pattern to the exact rational x, ties to the even pattern."""
    global _BF16_POS
    if _BF16_POS is None:
        _BF16_POS = _finite_bf16_values()
    vals, pats = _BF16_POS
    a = abs(x)
    i = bisect.bisect_left(vals, a)
    cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
    best = min(cands, key=lambda j: (abs(vals[j] - a), int(pats[j]) & 1))
    p = int(pats[best])
    return p | 0x8000 if x < 0 else p


@pytest.mark.parametrize("scale", [1.0, 0.5, 4.3345e-3, 3.1e-2, 123.456, 2.0 ** -20 * 1.75])
def test_dequant_is_the_correctly_rounded_product(scale):
    s32 = np.float32(scale)
    for c in ALL_CODES:
        c = int(c)
        got = oracle.dequant_e4m3(c, s32)
        if _is_nan_code(c):
            assert (got & 0x7F80) == 0x7F80 and (got & 0x7F) != 0
            continue
        v = oracle.e4m3_to_double(c)
        exact = Fraction(v) * Fraction(float(s32))
        want = _nearest_bf16_exact(exact)
        if v == 0.0:
            want = 0x8000 if c & 0x80 else 0x0000
        assert got == want, (hex(c), scale, hex(got), hex(want))


def test_dequant_rounds_once_not_through_binary32():
    """Products whose binary32 rounding lands exactly on a bf16 midpoint while the exact
    product does not: rounding the exact product once and a detour through binary32 disagree
    there, and the oracle must take the former."""
    rng = np.random.default_rng(5)
    v = np.array([oracle.e4m3_to_double(int(c)) for c in range(1, 0x7F)])
    s = rng.uniform(0.5, 2.0, 40000).astype(np.float32)
    prod = v[:, None] * s.astype(np.float64)[None, :]            # exact (<= 28 significant bits)
    p32 = prod.astype(np.float32)
    u = p32.view(np.uint32)
    hit = ((u & 0xFFFF) == 0x8000) & (p32.astype(np.float64) != prod)
    ci, si = np.nonzero(hit)
    assert ci.size >= 8
    for a, b in list(zip(ci, si))[:64]:
        code = int(a) + 1
        exact = Fraction(float(v[a])) * Fraction(float(s[b]))
        want = _nearest_bf16_exact(exact)
        assert oracle.dequant_e4m3(code, s[b]) == want
    # the binary32 detour (ties to even at the midpoint) differs from one rounding in some cases
    detour = (u[hit] + 0x7FFF + ((u[hit] >> 16) & 1)) >> 16
    single = np.array([oracle.dequant_e4m3(int(a) + 1, s[b]) for a, b in zip(ci, si)])
    assert (detour != single).any()


def test_dequant_table_and_gather_agree():
    rng = np.random.default_rng(3)
    tabs = [rng.integers(0, 256, size=(97, 32), dtype=np.uint8) for _ in range(3)]
    scales = [np.float32(0.01), np.float32(0.02), np.float32(0.7)]
    idx = rng.integers(0, 97, size=(50, 3)).astype(np.uint32)
    m = oracle.gather(idx, tabs, scales)
    deq = [oracle.dequant_table(t, s) for t, s in zip(tabs, scales)]
    ref = oracle.gather(idx, deq)
    nan = np.isnan(synth.bf16_to_float(ref))
    assert np.array_equal(np.isnan(synth.bf16_to_float(m)), nan)
    assert np.array_equal(m[~nan], ref[~nan])
    # a swapped scale changes the result (the per-table scale is really applied per table)
    m2 = oracle.gather(idx, tabs, scales[::-1])
    assert not np.array_equal(m2[~nan], m[~nan])


# ------------------------------------------------------------------------ input generator
def test_generator_encoder_is_nearest_code_ties_even():
    """synth's integer e4m3 encoder returns, for every |n| < 2^17, the code whose value is
    nearest to n / 2^13, ties to the even code (brute force over all finite codes)."""
    vals = np.array([oracle.e4m3_to_double(int(c)) for c in range(0x7F)])   # +0 .. 448
    n = np.arange(-(2 ** 17) + 1, 2 ** 17, dtype=np.int64)
    codes = synth.encode_e4m3_int(n)
    a = np.abs(n) / 8192.0
    j = np.searchsorted(vals, a)
    lo = np.clip(j - 1, 0, 0x7E)
    hi = np.clip(j, 0, 0x7E)
    dlo, dhi = a - vals[lo], vals[hi] - a
    pick = np.where(dhi < dlo, hi, np.where(dlo < dhi, lo, np.where(hi % 2 == 0, hi, lo)))
    want = np.where(n < 0, pick | 0x80, pick)
    want = np.where(n == 0, 0, want).astype(np.uint8)
    assert np.array_equal(codes, want)


def test_generator_fp8_distribution_and_scales():
    wl = synth.get_workload("tiny").with_(table_dtype="fp8")
    codes = synth.fill_fp8(wl.table_spec(0), (wl.primes[0], wl.d_e))
    vals = oracle.dequant_table(codes, wl.table_scale(0))
    f = synth.bf16_to_float(vals).astype(np.float64)
    assert abs(f.std() / wl.table_sigma(0) - 1.0) < 0.02 and abs(f.mean()) < 1e-3 * wl.table_sigma(0) * 10
    # rows regenerate without the whole table, identically
    rows = np.array([0, 5, wl.primes[0] - 1])
    assert np.array_equal(synth.fill_rows_fp8(wl.table_spec(0), wl.d_e, rows), codes[rows])
    assert len({float(wl.table_scale(h)) for h in range(wl.H)}) == wl.H
    assert wl.table_bytes * 2 == wl.with_(table_dtype="bf16").table_bytes
