"""Pins of the oracle's number formats and rounding functions.

Each check compares the oracle with something other than itself: the golden
facts (cited in tests/golden), closed forms, library routines (numpy float16,
torch bf16 casting, math.frexp) or a brute-force nearest-value search over the
whole enumerated table in float64.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden_list(name):
    vals = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                vals.append(float(line))
    return vals


def _read_golden_kv(name):
    kv = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = line.split()
                kv[k] = float(v)
    return kv


# ------------------------------------------------------------------ tables

def test_e2m1_table_matches_golden(ref):
    mags = _read_golden_list("e2m1_magnitudes.txt")
    assert [ref.e2m1_value(m) for m in range(8)] == mags
    for m in range(8):
        v = ref.e2m1_value(8 | m)
        assert v == -mags[m] and math.copysign(1.0, v) == -1.0
    # the 4-over-6 page names 4 and 6 as the two largest values
    assert sorted(mags)[-2:] == [4.0, 6.0]


def test_e4m3_table_facts(ref):
    kv = _read_golden_kv("scale_format_facts.txt")
    vals = [ref.e4m3_value(c) for c in range(0x7F)]
    assert vals[0] == 0.0
    assert all(b > a for a, b in zip(vals, vals[1:])), "codes 0..0x7E must increase"
    pos = [v for v in vals if v > 0]
    assert len(pos) == kv["e4m3_positive_finite_codes"]
    assert max(pos) == kv["e4m3_max_finite"] and vals[0x7E] == kv["e4m3_max_finite"]
    assert min(pos) == kv["e4m3_min_positive"] and vals[1] == kv["e4m3_min_positive"]
    assert math.isnan(ref.e4m3_value(0x7F))
    # closed form: every positive value has at most 4 significant bits and the
    # subnormals are the multiples of 2^-9 below 2^-6
    for c, v in enumerate(vals):
        if v == 0:
            continue
        m, e = math.frexp(v)
        assert (m * 16) == int(m * 16), (c, v)
        if v < 2 ** -6:
            assert v / 2 ** -9 == int(v / 2 ** -9)
    # the set is exactly {k * 2^j : 8 <= k < 16, -9 <= j+3 ... } u subnormals
    normals = sorted({k * 2.0 ** (e - 3) for e in range(-6, 9) for k in range(8, 16)
                      if k * 2.0 ** (e - 3) <= 448})
    subn = [k * 2.0 ** -9 for k in range(1, 8)]
    assert pos == subn + normals


def test_e8m0_and_exponent(ref):
    kv = _read_golden_kv("scale_format_facts.txt")
    for b in range(255):
        assert ref.e8m0_value(b) == 2.0 ** (b - kv["e8m0_bias"])
    assert math.isnan(ref.e8m0_value(255))
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        np.float32(2.0) ** np.arange(-149, 128, dtype=np.float64).astype(np.float32),
        (rng.random(5000) * 10.0 ** rng.integers(-40, 38, 5000)).astype(np.float32),
        np.nextafter(np.float32(2.0) ** np.arange(-120, 120).astype(np.float32), np.float32(0)),
    ])
    for a in vals:
        a = float(a)
        if a == 0 or not math.isfinite(a):
            continue
        m, k = math.frexp(a)  # library routine: a = m * 2^k, m in [0.5, 1)
        want = max(-127, min(127, (k - 1) - int(kv["e2m1_emax"])))
        assert ref.e8m0_exponent(a) == want, a
    assert ref.e8m0_exponent(0.0) == -127


def test_fp16_decode_matches_numpy(ref):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float32)
    got = np.array([ref.fp16_to_float(int(b)) for b in bits], np.float32)
    finite = np.isfinite(want)
    assert np.array_equal(got[finite].view(np.uint32), want[finite].view(np.uint32))
    assert np.all(np.isnan(got[np.isnan(want)]))


def test_bf16_rounding_matches_torch(ref):
    rng = np.random.default_rng(12)
    a = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000).astype(np.float32),
        # exact ties and near ties
        (np.arange(1, 4000, dtype=np.uint32) << 15 | 0x3F800000).view(np.float32),
        np.array([3.3895314e38, 3.39e38, 3.4e38, -3.4e38, 1e-45, -1e-45, 0.0, -0.0], np.float32),
    ]).astype(np.float32)
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([ref.float_to_bf16(v) for v in a], np.uint16)
    assert np.array_equal(got, want)


# ---------------------------------------------------------- E2M1 rounding

E2M1_MAGS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _check_e2m1(u: np.ndarray, codes: np.ndarray):
    """Property check: |u| maps to a nearest magnitude (ties: even index),
    values >= 6 saturate, the sign bit is copied."""
    u = u.astype(np.float32)
    a = np.abs(u.astype(np.float64))
    m = codes & 7
    s = codes >> 3
    assert np.all(codes < 16)
    assert np.array_equal(s.astype(bool), np.signbit(u))
    d = np.abs(a[:, None] - E2M1_MAGS[None, :])
    dmin = d.min(axis=1)
    chosen = d[np.arange(len(a)), m]
    inrange = a < 6
    assert np.all(chosen[inrange] == dmin[inrange])
    ties = inrange & ((d == dmin[:, None]).sum(axis=1) > 1)
    assert np.all(m[ties] % 2 == 0)
    assert np.all(m[~inrange] == 7)


def test_e2m1_midpoints_closed_form(ref):
    # ties go to the even mantissa index; the values between neighbours are
    # the midpoints of the E2M1 grid
    table = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for u, want in table.items():
        for sgn in (1, -1):
            c = ref.rne_e2m1(sgn * u)
            assert abs(ref.e2m1_value(c)) == want and ((c >> 3) == (sgn < 0))
    assert ref.rne_e2m1(-0.1) == 0x8 and ref.rne_e2m1(0.1) == 0x0
    assert ref.rne_e2m1(-0.0) == 0x8
    assert ref.rne_e2m1(6.0) == 7 and ref.rne_e2m1(7.9) == 7 and ref.rne_e2m1(1e30) == 7
    assert ref.rne_e2m1(float("inf")) == 7 and ref.rne_e2m1(float("-inf")) == 15


def test_e2m1_all_bf16_patterns(ref):
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    u = (u.astype(np.uint32) << 16).view(np.float32)
    u = u[np.isfinite(u)]
    _check_e2m1(u, ref.rne_e2m1_array(u))


def test_e2m1_dense_near_decision_points(ref):
    pts = np.array([0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0],
                   np.float32)
    base = pts.view(np.uint32)
    offs = np.arange(-3000, 3001, dtype=np.int64)
    bits = (base[:, None].astype(np.int64) + offs[None, :]).reshape(-1).astype(np.uint32)
    u = np.concatenate([bits.view(np.float32), -bits.view(np.float32)])
    _check_e2m1(u, ref.rne_e2m1_array(u))


def test_e2m1_strided_sweep_all_patterns(ref):
    # every 65,521st bit pattern (a prime stride, hits every exponent and many mantissas)
    bits = np.arange(0, 2 ** 32, 65521, dtype=np.uint64).astype(np.uint32)
    u = bits.view(np.float32)
    u = u[np.isfinite(u)]
    _check_e2m1(u, ref.rne_e2m1_array(u))


# ---------------------------------------------------------- E4M3 rounding

def _e4m3_table(ref):
    return np.array([ref.e4m3_value(c) for c in range(0x7F)], np.float64)


def _check_e4m3(ref, v: np.ndarray, codes: np.ndarray):
    tab = _e4m3_table(ref)
    x = v.astype(np.float64)
    assert np.all(codes <= 0x7E)
    sat = x > 448
    assert np.all(codes[sat] == 0x7E)
    xi = x[~sat]
    ci = codes[~sat].astype(np.int64)
    # nearest by brute force over all 127 codes
    d = np.abs(xi[:, None] - tab[None, :])
    dmin = d.min(axis=1)
    assert np.all(d[np.arange(len(xi)), ci] == dmin)
    ties = (d == dmin[:, None]).sum(axis=1) > 1
    assert np.all(ci[ties] % 2 == 0)


def test_e4m3_closed_form_points(ref):
    assert ref.rne_e4m3_sat(448.0) == 0x7E and ref.rne_e4m3_sat(449.0) == 0x7E
    assert ref.rne_e4m3_sat(1e30) == 0x7E and ref.rne_e4m3_sat(float("inf")) == 0x7E
    assert ref.rne_e4m3_sat(2 ** -10) == 0  # tie between 0 and 2^-9 goes to even code 0
    assert ref.rne_e4m3_sat(np.nextafter(np.float32(2 ** -10), np.float32(1))) == 1
    assert ref.rne_e4m3_sat(1.0) == 0x38
    assert ref.rne_e4m3_sat(1.0625) == 0x38   # tie 1.0 / 1.125 -> even code 0x38
    assert ref.rne_e4m3_sat(1.1875) == 0x3A   # tie 1.125 / 1.25 -> even code 0x3A
    assert ref.rne_e4m3_sat(432.0) == 0x7E    # tie 416 / 448 -> even code 0x7E
    assert ref.rne_e4m3_sat(0.0) == 0 and ref.rne_e4m3_sat(-0.0) == 0


def test_e4m3_dense_and_sweep(ref):
    tab = _e4m3_table(ref).astype(np.float32)
    mids = ((tab[1:].astype(np.float64) + tab[:-1]) / 2).astype(np.float32)
    base = np.concatenate([tab, mids]).view(np.uint32)
    offs = np.arange(-200, 201, dtype=np.int64)
    bits = (base[:, None].astype(np.int64) + offs[None, :]).reshape(-1)
    bits = bits[(bits >= 0) & (bits < 0x7F800000)].astype(np.uint32)
    sweep = np.arange(0, 0x7F800001, 9973, dtype=np.uint64).astype(np.uint32)
    v = np.concatenate([bits, sweep]).view(np.float32)
    _check_e4m3(ref, v, ref.rne_e4m3_array(v))


# ---------------------------------------------------------- UE5M3 (reading)

def _ue5m3_table(ref):
    return np.array([ref.ue5m3_value(c) for c in range(0xFF)], np.float64)


def test_ue5m3_table_closed_form(ref):
    # the reading of the unsigned 5-exponent / 3-mantissa scale format: bias 15,
    # subnormals m * 2^-17, 0xFF NaN; the value set is exactly the subnormals
    # and {k * 2^(e-3): 8 <= k < 16, -14 <= e <= 16} less its top (1.875 * 2^16,
    # the NaN pattern)
    vals = list(_ue5m3_table(ref))
    assert vals[0] == 0.0 and math.isnan(ref.ue5m3_value(0xFF))
    assert all(b > a for a, b in zip(vals, vals[1:])), "codes 0..0xFE must increase"
    subn = [k * 2.0 ** -17 for k in range(1, 8)]
    normals = sorted(k * 2.0 ** (e - 3) for e in range(-14, 17) for k in range(8, 16))[:-1]
    assert vals[1:] == subn + normals
    assert vals[0xFE] == 1.75 * 2 ** 16 and vals[1] == 2.0 ** -17 and vals[8] == 2.0 ** -14
    assert ref.ue5m3_value(15 << 3) == 1.0


def _check_ue5m3(ref, v: np.ndarray, codes: np.ndarray):
    tab = _ue5m3_table(ref)
    x = v.astype(np.float64)
    assert np.all(codes <= 0xFE)
    sat = x > tab[-1]
    assert np.all(codes[sat] == 0xFE)
    xi = x[~sat]
    ci = codes[~sat].astype(np.int64)
    d = np.abs(xi[:, None] - tab[None, :])
    dmin = d.min(axis=1)
    assert np.all(d[np.arange(len(xi)), ci] == dmin)
    ties = (d == dmin[:, None]).sum(axis=1) > 1
    assert np.all(ci[ties] % 2 == 0)


def test_ue5m3_closed_form_points(ref):
    assert ref.rne_ue5m3_sat(1.0) == 0x78
    assert ref.rne_ue5m3_sat(1.0625) == 0x78        # tie 1 / 1.125 -> even code
    assert ref.rne_ue5m3_sat(1.1875) == 0x7A        # tie 1.125 / 1.25 -> even code
    assert ref.rne_ue5m3_sat(2.0 ** -18) == 0       # tie 0 / 2^-17 -> code 0
    assert ref.rne_ue5m3_sat(3 * 2.0 ** -18) == 2   # tie 2^-17 / 2^-16 -> even code 2
    assert ref.rne_ue5m3_sat(114688.0) == 0xFE and ref.rne_ue5m3_sat(1e30) == 0xFE
    assert ref.rne_ue5m3_sat(float("inf")) == 0xFE
    assert ref.rne_ue5m3_sat(0.0) == 0 and ref.rne_ue5m3_sat(-0.0) == 0


def test_ue5m3_dense_and_sweep(ref):
    tab = _ue5m3_table(ref).astype(np.float32)
    mids = ((tab[1:].astype(np.float64) + tab[:-1]) / 2).astype(np.float32)
    base = np.concatenate([tab, mids]).view(np.uint32)
    offs = np.arange(-100, 101, dtype=np.int64)
    bits = (base[:, None].astype(np.int64) + offs[None, :]).reshape(-1)
    bits = bits[(bits >= 0) & (bits < 0x7F800000)].astype(np.uint32)
    sweep = np.arange(0, 0x7F800001, 19997, dtype=np.uint64).astype(np.uint32)
    v = np.concatenate([bits, sweep]).view(np.float32)
    _check_ue5m3(ref, v, ref.rne_ue5m3_array(v))
