"""Pins that tie the CPU oracle to something other than itself.

Each ``pin_*`` function takes the oracle module and raises AssertionError when
the oracle disagrees with:

* a library conversion (torch's CPU casts to bfloat16 / float8_e4m3fn),
* brute force on tiny inputs (per-expert enumeration, per-token slot lists,
  nearest-code search over the whole FP8 code table),
* a closed form built so its exact answer is known by hand, or
* the exact result (fp64 / rational) within the fp32 error bound.

They run in the CPU suite against the real oracle, and against copies of the
oracle with a mistake planted in them (each plant must trip at least one pin).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import torch

from combine_ep_get_10_b200 import workloads as W

U32 = 2.0 ** -24  # fp32 unit roundoff
UBF = 2.0 ** -8  # bf16 unit roundoff


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _torch_bf16_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _torch_e4m3_codes(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _torch_e4m3_values():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()


# ------------------------------------------------------------------ formats
def pin_bf16_encode_vs_torch(o):
    rng = _rng(11)
    a = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(50000) * 1e30).astype(np.float32),
        (rng.standard_normal(50000) * 1e-38).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, 3.4e38, np.inf, -np.inf,
                  1e-45, -1e-45], np.float32),
    ])
    # exact ties: upper half + 0x8000 in the dropped bits
    hi = rng.integers(0, 0x7F00, size=20000, dtype=np.uint32) << 16
    ties = (hi | 0x8000).view(np.float32)
    a = np.concatenate([a, ties, -ties])
    got = o.f32_to_bf16(a)
    ref = _torch_bf16_bits(a)
    assert np.array_equal(got, ref), "bf16 RNE encoder differs from torch's cast"


def pin_bf16_decode_vs_torch(o):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = o.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def pin_e4m3_decode_vs_torch(o):
    codes = np.arange(256, dtype=np.uint8)
    got = o.e4m3_to_f32(codes)
    ref = _torch_e4m3_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}


def pin_e4m3_encode_vs_torch(o):
    """torch rounds to nearest-even and saturates below 464; above that it
    gives NaN, so this pin covers |v| < 464 (saturation has its own pin)."""
    rng = _rng(12)
    vals = _torch_e4m3_values()
    fin = np.sort(np.unique(np.abs(vals[np.isfinite(vals)])))
    mids = ((fin[1:].astype(np.float64) + fin[:-1]) / 2).astype(np.float32)  # exact in fp32
    nudged = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1000))])
    rnd = np.concatenate([rng.uniform(-463.9, 463.9, 200000), rng.standard_normal(100000) * 2.0 ** -7,
                          rng.standard_normal(100000) * 2.0 ** -11]).astype(np.float32)
    a = np.concatenate([fin, -fin, mids, -mids, nudged, -nudged, rnd,
                        np.array([448.0, 463.99997, -463.99997], np.float32)])
    got = o.f32_to_e4m3(a)
    ref = _torch_e4m3_codes(a)
    assert np.array_equal(got, ref), "e4m3 encoder differs from torch's cast"


def pin_e4m3_encode_bruteforce(o):
    """Nearest finite code by exhaustive search, ties to the even code, with
    magnitudes above 448 saturating to 448."""
    table = _torch_e4m3_values()[:0x7F].astype(np.float64)  # codes 0..126, all >= 0
    rng = _rng(13)
    a = np.concatenate([rng.uniform(0, 470, 3000), rng.uniform(0, 2.0 ** -5, 3000),
                        np.array([2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -9 * 1.5, 0.0, 500.0])]).astype(np.float32)
    a = np.concatenate([a, -a])
    got = o.f32_to_e4m3(a)
    for v, g in zip(a.astype(np.float64), got):
        m = abs(v)
        if m > 448.0:
            want = 0x7E
        else:
            d = np.abs(table - m)
            best = np.nonzero(d == d.min())[0]
            want = int(best[0]) if len(best) == 1 else int([c for c in best if c % 2 == 0][0])
        sign = 0x80 if math.copysign(1.0, v) < 0 else 0
        assert int(g) == (want | sign), (v, int(g), want | sign)


def pin_e4m3_saturation(o):
    a = np.array([448.0, 449.0, 463.9, 464.0, 465.0, 479.0, 480.0, 1e6, 3.4e38, np.inf], np.float32)
    got = o.f32_to_e4m3(a)
    assert (got == 0x7E).all()
    assert (o.f32_to_e4m3(-a) == 0xFE).all()
    assert o.f32_to_e4m3(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def pin_fp8_quant_closed_form(o):
    """Groups built from exact e4m3 values times 2^m, with one element at
    +-448*2^m: then amax = 448*2^m, scale = 2^m, 448/amax = 2^-m exactly, and
    every code must come back unchanged."""
    rng = _rng(14)
    vals = _torch_e4m3_values()
    finite_codes = np.array([c for c in range(256) if np.isfinite(vals[c]) and c not in (0x00, 0x80)], np.uint8)
    H = 128 * 6
    codes = rng.choice(finite_codes, size=H)
    exps = [0, 3, -5, -20, 40, -60]
    for g, pos in enumerate([0, 127, 64, 5, 127, 100]):  # first and last channel included
        codes[g * 128:(g + 1) * 128] &= 0xF7  # keep the rest strictly below 448 in magnitude
        codes[g * 128 + pos] = 0x7E if g % 2 == 0 else 0xFE
    xf = vals[codes].astype(np.float64)
    for g, m in enumerate(exps):
        xf[g * 128:(g + 1) * 128] *= 2.0 ** m
    xbits = _torch_bf16_bits(xf.astype(np.float32))
    assert np.array_equal(torch.from_numpy(xbits.view(np.int16)).view(torch.bfloat16).float().numpy(),
                          xf.astype(np.float32)), "construction must be exact in bf16"
    q, s = o.fp8_quant_row(xbits)
    assert np.array_equal(q, codes)
    assert np.array_equal(s, np.array([2.0 ** m for m in exps], np.float32))


def pin_fp8_quant_zero_and_tiny(o):
    H = 256
    x = np.zeros(H, np.float32)
    x[130] = 2.0 ** -130  # bf16 subnormal; 448/amax would overflow fp32
    x[131] = -2.0 ** -131
    xb = _torch_bf16_bits(x)
    xb[5] = 0x8000  # -0.0 in an all-zero group
    q, s = o.fp8_quant_row(xb)
    assert (q[:128] == 0).all() and s[0] == 0.0
    assert s[1] == np.float32(2.0 ** -130) / np.float32(448.0)
    assert not np.isnan(o.e4m3_to_f32(q[128:])).any()
    assert q[128 + 0] == 0x00 and q[130] != 0 and q[131] & 0x80


def pin_fp8_quant_error_bound(o):
    rng = _rng(15)
    H = 7168
    for trial in range(4):
        x = (rng.standard_normal(H) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        xb = _torch_bf16_bits(x)
        xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
        q, s = o.fp8_quant_row(xb)
        deq = _torch_e4m3_values()[q].astype(np.float64)
        for g in range(H // 128):
            seg = xf[g * 128:(g + 1) * 128]
            amax = np.abs(seg).max()
            assert s[g] == np.float32(np.float32(amax) / np.float32(448.0))
            approx = deq[g * 128:(g + 1) * 128] * s[g]
            bound = np.maximum(np.abs(seg) * 2.0 ** -4, 2.0 ** -10 * s[g]) * (1 + 1e-5) + 1e-6 * np.abs(seg)
            assert (np.abs(approx - seg) <= bound).all()
            top = np.argmax(np.abs(seg))
            assert q[g * 128 + top] & 0x7F == 0x7E  # the amax element lands on 448


# ------------------------------------------------ per-token and MX formats
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])  # OCP MX v1.0, FP4 E2M1 value table
MX_EMAX = {W.MXFP8_E4M3: 8, W.MXFP8_E5M2: 15, W.MXFP4_E2M1: 2}
MX_MAXFINITE = {W.MXFP8_E4M3: 448.0, W.MXFP8_E5M2: 57344.0, W.MXFP4_E2M1: 6.0}


def _torch_e5m2_values():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e5m2).to(torch.float32).numpy()


def _e2m1_value(code):
    v = E2M1_MAGNITUDES[code & 7]
    return -v if code & 8 else v


def _mx_element_values(dtype, codes):
    """Element codes of one MX format -> float64 values, decoded without the
    oracle (torch's float8 tables, the E2M1 value table)."""
    if dtype == W.MXFP8_E4M3:
        return _torch_e4m3_values()[codes].astype(np.float64)
    if dtype == W.MXFP8_E5M2:
        return _torch_e5m2_values()[codes].astype(np.float64)
    nib = np.empty(codes.size * 2, np.uint8)
    nib[0::2] = codes & 0xF
    nib[1::2] = codes >> 4
    return np.array([_e2m1_value(int(c)) for c in nib])


def pin_e5m2_decode_vs_torch(o):
    codes = np.arange(256, dtype=np.uint8)
    got = o.e5m2_to_f32(codes)
    ref = _torch_e5m2_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert ref[0x7B] == 57344.0 and np.isinf(ref[0x7C])


def pin_e5m2_encode_vs_torch(o):
    """torch rounds to nearest-even and overflows to inf from 61440 up; this
    pin covers |v| < 61440 (saturation has its own pin)."""
    rng = _rng(51)
    vals = _torch_e5m2_values()
    fin = np.sort(np.unique(np.abs(vals[np.isfinite(vals)])))
    mids = ((fin[1:].astype(np.float64) + fin[:-1]) / 2).astype(np.float32)
    nudged = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e6))])
    rnd = np.concatenate([rng.uniform(-61439, 61439, 100000), rng.standard_normal(100000) * 2.0 ** -12,
                          rng.standard_normal(100000) * 2.0 ** -17,
                          np.exp(rng.uniform(-30, 11, 100000)) * rng.choice([-1, 1], 100000)]).astype(np.float32)
    a = np.concatenate([fin, -fin, mids, -mids, nudged, -nudged, rnd, np.array([61439.996, -61439.996], np.float32)])
    got = o.f32_to_e5m2(a)
    ref = torch.from_numpy(a).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(got, ref), "e5m2 encoder differs from torch's cast"


def pin_e5m2_saturation(o):
    a = np.array([57344.0, 57345.0, 61439.0, 61440.0, 65536.0, 1e9, 3.4e38, np.inf], np.float32)
    assert (o.f32_to_e5m2(a) == 0x7B).all()
    assert (o.f32_to_e5m2(-a) == 0xFB).all()


def pin_e2m1_decode_table(o):
    got = o.e2m1_to_f32(np.arange(16, dtype=np.uint8)).astype(np.float64)
    want = np.concatenate([E2M1_MAGNITUDES, -E2M1_MAGNITUDES])
    assert np.array_equal(got, want)
    assert np.signbit(got[8])


def pin_e2m1_encode_bruteforce(o):
    """Nearest of the eight magnitudes by search, ties to the even code, above
    6 saturating to 6; the sign goes to bit 3 (negative zero included)."""
    rng = _rng(52)
    a = np.concatenate([rng.uniform(0, 7.5, 4000), rng.uniform(0, 1.2, 2000),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 7.0, 1e30, 0.0, 1e-40])])
    a = np.concatenate([a, -a]).astype(np.float32)
    got = o.f32_to_e2m1(a)
    for v, g in zip(a.astype(np.float64), got):
        m = abs(v)
        if m > 6.0:
            want = 7
        else:
            d = np.abs(E2M1_MAGNITUDES - m)
            best = np.nonzero(d == d.min())[0]
            want = int(best[0]) if len(best) == 1 else int([c for c in best if c % 2 == 0][0])
        sign = 8 if math.copysign(1.0, v) < 0 else 0
        assert int(g) == (want | sign), (v, int(g), want | sign)


def pin_int8_encode_vs_torch(o):
    """torch.round is round-half-to-even; codes are clamped to [-127, 127]."""
    rng = _rng(53)
    a = np.concatenate([rng.uniform(-140, 140, 100000), np.arange(-130, 131) + 0.5,
                        np.array([-1e9, 1e9, -127.5, 127.5, -0.5, 0.5, -0.0])]).astype(np.float32)
    ref = torch.from_numpy(a).round().clamp(-127, 127).to(torch.int8).numpy()
    assert np.array_equal(o.f32_to_int8(a), ref)


def pin_int8_quant_closed_form(o):
    """Rows of integers in [-126, 126] times 2^m with one element +-127*2^m:
    amax = 127*2^m, scale = 2^m and 127/amax = 2^-m exactly, so every code
    comes back unchanged."""
    rng = _rng(54)
    for H, m, pos in [(7168, 0, 0), (256, 7, 255), (136, -20, 70), (8, 60, 3), (1024, -100, 511)]:
        c = rng.integers(-126, 127, size=H)
        c[pos] = 127 if m % 2 == 0 else -127
        xf = c.astype(np.float64) * 2.0 ** m
        xb = _torch_bf16_bits(xf.astype(np.float32))
        assert np.array_equal(_bf16_f64(xb), xf)
        q, s = o.quant_row(W.INT8_PER_TOKEN, xb)
        assert np.array_equal(q.astype(np.int64), c), (H, m)
        assert s[0] == np.float32(2.0 ** m)


def pin_int8_quant_ties_and_bound(o):
    # amax 127 gives 127/amax = 1 exactly: x = k + 1/2 must round to even
    x = np.array([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 126.5, 1.5] + [0.0] * 7, np.float32)
    q, s = o.quant_row(W.INT8_PER_TOKEN, _torch_bf16_bits(x))
    assert q.tolist() == [127, 2, 4, -2, -4, 0, 0, 126, 2] + [0] * 7 and s[0] == 1.0
    # zero row, and amax = 2^-126, where 127/amax overflows fp32 and is
    # clamped to FLT_MAX = (2 - 2^-23) 2^127: the code is rint(-(4 - 2^-22)) = -4
    q, s = o.quant_row(W.INT8_PER_TOKEN, np.zeros(64, np.uint16))
    assert (q == 0).all() and s[0] == 0.0
    x = np.zeros(64, np.float32)
    x[9] = -2.0 ** -126
    q, s = o.quant_row(W.INT8_PER_TOKEN, _torch_bf16_bits(x))
    assert q[9] == -4 and (np.delete(q, 9) == 0).all()
    assert s[0] == np.float32(Fraction(2) ** -126 / 127)
    rng = _rng(55)
    for trial in range(4):
        H = 7168
        xb = _torch_bf16_bits((rng.standard_normal(H) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32))
        xf = _bf16_f64(xb)
        q, s = o.quant_row(W.INT8_PER_TOKEN, xb)
        amax = np.abs(xf).max()
        sc = float(s[0])
        assert abs(sc - amax / 127) <= U32 * amax / 127  # correctly rounded quotient
        assert abs(int(q[np.argmax(np.abs(xf))])) == 127
        assert (np.abs(q.astype(np.float64) * sc - xf) <= sc * (0.5 + 1e-5)).all()


def pin_fp8_pertoken_reduces_to_group(o):
    """With H = 128 the per-token FP8 row is the 128-channel FP8 row; for a
    long row built from e4m3 values times 2^m with one element +-448*2^m the
    codes come back unchanged and the scale is 2^m."""
    rng = _rng(56)
    for trial in range(20):
        xb = _torch_bf16_bits((rng.standard_normal(128) * 10.0 ** rng.uniform(-20, 20)).astype(np.float32))
        q, s = o.quant_row(W.FP8_E4M3_PER_TOKEN, xb)
        q1, s1 = o.fp8_quant_row(xb)
        assert np.array_equal(q, q1) and s[0] == s1[0]
    vals = _torch_e4m3_values()
    finite = np.array([c for c in range(256) if np.isfinite(vals[c]) and c not in (0x00, 0x80)], np.uint8)
    for H, m, pos in [(7168, 0, 7167), (512, -30, 0), (136, 25, 77)]:
        codes = rng.choice(finite, size=H) & 0xF7
        codes[pos] = 0x7E if m % 2 == 0 else 0xFE
        xf = vals[codes].astype(np.float64) * 2.0 ** m
        xb = _torch_bf16_bits(xf.astype(np.float32))
        assert np.array_equal(_bf16_f64(xb), xf)
        q, s = o.quant_row(W.FP8_E4M3_PER_TOKEN, xb)
        assert np.array_equal(q, codes) and s[0] == np.float32(2.0 ** m)
    q, s = o.quant_row(W.FP8_E4M3_PER_TOKEN, np.zeros(256, np.uint16))
    assert (q == 0).all() and s[0] == 0.0


def _floor_log2_exact(v):
    """floor(log2 v) for v > 0, exactly, from the rational value."""
    f = Fraction(float(v))
    n = f.numerator.bit_length() - f.denominator.bit_length()
    while Fraction(2) ** n > f:
        n -= 1
    while Fraction(2) ** (n + 1) <= f:
        n += 1
    return n


def pin_mx_shared_exp_exact(o):
    rng = _rng(57)
    vals = np.concatenate([np.exp2(rng.uniform(-149, 127.9, 3000)), np.array([1.0, 448.0, 447.9, 512.0, 6.0, 4.0,
                           57344.0, 2.0 ** -126, 2.0 ** -149, 2.0 ** -130, 3.4e38])]).astype(np.float32)
    for emax in (8, 15, 2):
        assert o.mx_shared_exp(0.0, emax) == -127
        for v in vals:
            want = max(-127, min(127, _floor_log2_exact(v) - emax))
            assert o.mx_shared_exp(float(v), emax) == want, (float(v), emax)


def pin_mx_closed_form_roundtrip(o):
    """Blocks of exact element values times 2^X whose largest element has the
    format's top exponent: the shared exponent must be X (scale byte X+127)
    and every code must come back unchanged."""
    rng = _rng(58)
    for dtype in (W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1):
        emax = MX_EMAX[dtype]
        if dtype == W.MXFP4_E2M1:
            allcodes = np.arange(16, dtype=np.uint8)
            vals = np.array([_e2m1_value(int(c)) for c in allcodes])
        else:
            table = _torch_e4m3_values() if dtype == W.MXFP8_E4M3 else _torch_e5m2_values()
            allcodes = np.array([c for c in range(256) if np.isfinite(table[c])], np.uint8)
            vals = table.astype(np.float64)[allcodes]
        top = allcodes[(np.abs(vals) >= 2.0 ** emax)]
        rest = allcodes[(np.abs(vals) < 2.0 ** emax)]
        nb = 6
        H = 32 * nb
        el = rng.choice(rest, size=H).astype(np.uint8)
        Xs = [0, 5, -9, -100, 90, -120 + emax]
        for g in range(nb):
            el[g * 32 + rng.integers(0, 32)] = rng.choice(top)
        value_of = {int(c): float(v) for c, v in zip(allcodes, vals)}
        xf = np.array([value_of[int(c)] for c in el])
        for g, X in enumerate(Xs):
            xf[g * 32:(g + 1) * 32] *= 2.0 ** X
        xb = _torch_bf16_bits(xf.astype(np.float32))
        assert np.array_equal(_bf16_f64(xb), xf), "construction must be exact in bf16"
        q, s = o.quant_row(dtype, xb)
        assert np.array_equal(s.astype(np.int64), np.array(Xs) + 127), dtype
        if dtype == W.MXFP4_E2M1:
            want = (el[0::2] | (el[1::2] << 4)).astype(np.uint8)
            assert np.array_equal(q, want)
        else:
            assert np.array_equal(q, el)


def pin_mx_error_bound(o):
    """Decoded codes times 2^X are within half an element-format spacing of
    x, or saturated at the format's largest value when |x| / 2^X exceeds it;
    the block's amax element decodes to at least 2^emax."""
    rng = _rng(59)
    for dtype in (W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1):
        emax, top = MX_EMAX[dtype], MX_MAXFINITE[dtype]
        mbits = {W.MXFP8_E4M3: 3, W.MXFP8_E5M2: 2, W.MXFP4_E2M1: 1}[dtype]
        emin = {W.MXFP8_E4M3: -6, W.MXFP8_E5M2: -14, W.MXFP4_E2M1: 0}[dtype]
        for trial in range(6):
            H = 32 * 64
            xb = _torch_bf16_bits((rng.standard_normal(H) * np.exp2(rng.uniform(-40, 40, H // 32)).repeat(32))
                                  .astype(np.float32))
            xf = _bf16_f64(xb)
            q, s = o.quant_row(dtype, xb)
            deq_el = _mx_element_values(dtype, q)
            for g in range(H // 32):
                X = int(s[g]) - 127
                seg = xf[g * 32:(g + 1) * 32] / 2.0 ** X
                d = deq_el[g * 32:(g + 1) * 32]
                e = np.floor(np.log2(np.maximum(np.abs(seg), 2.0 ** emin)))
                half = 2.0 ** (e - mbits - 1)
                sat = np.abs(seg) > top
                assert (np.abs(d[~sat] - seg[~sat]) <= half[~sat] * (1 + 1e-9)).all(), (dtype, g)
                assert (np.abs(d[sat]) == top).all() and (np.sign(d[sat]) == np.sign(seg[sat])).all()
                assert np.abs(d).max() >= 2.0 ** emax


def pin_mx_zero_tiny_and_packing(o):
    for dtype in (W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1):
        q, s = o.quant_row(dtype, np.zeros(64, np.uint16))
        assert (q == 0).all() and (s == 0).all()  # amax 0: X = -127
        x = np.zeros(64, np.float32)
        x[33] = 2.0 ** -133  # bf16 subnormal amax: X clamps to -127
        x[40] = -2.0 ** -131
        xb = _torch_bf16_bits(x)
        xb[0] = 0x8000  # -0.0
        q, s = o.quant_row(dtype, xb)
        assert s.tolist() == [0, 0]
        d = _mx_element_values(dtype, q)
        assert np.isfinite(d).all() and np.signbit(d[0])
        assert d[33] == x[33] * 2.0 ** 127 or dtype == W.MXFP4_E2M1
    # packing: element 2i in the low nibble
    x = np.array([1.0, 6.0, -0.5, 3.0] + [0.0] * 28, np.float32)
    q, s = o.quant_row(W.MXFP4_E2M1, _torch_bf16_bits(x))
    assert s[0] == 127 and q[0] == 0x72 and q[1] == 0x59 and (q[2:] == 0).all()


def pin_quant_dispatch_rows(o):
    """Each quantised dispatch row is the quantisation of its source row, in
    the scale layout of its format, at the row routing gives it."""
    rng = _rng(60)
    for dt in (W.INT8_PER_TOKEN, W.FP8_E4M3_PER_TOKEN, W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1):
        for mode, max_tokens in ((W.COMPACT, 0), (W.PADDED, 5)):
            T, E, R, K, H = 21, 8, 2, 3, 96
            idx = W.random_topk(rng, T, E, K, p_neg=0.2, allow_dup=True)
            x = _torch_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
            L = o.tc_layout(idx, E, R)
            D = o.tc_dispatch(x, idx, E, L, mode=mode, max_tokens=max_tokens, out_dtype=dt, want_src=True)
            seen = 0
            for e in range(E):
                pairs = [(t, k) for t in range(T) for k in range(K) if idx[t, k] == e]
                for j, (t, k) in enumerate(pairs):
                    if mode == W.PADDED and j >= max_tokens:
                        continue
                    row = _expected_row(e, j, L["expert_offsets"], mode, max_tokens)
                    qq, ss = o.quant_row(dt, x[t])
                    assert np.array_equal(D["recv"][row], qq), (dt, mode)
                    assert np.array_equal(np.atleast_1d(D["recv_scales"][row]), ss), (dt, mode)
                    assert D["recv_src"][row] == t
                    seen += 1
            assert seen == (D["recv_src"] >= 0).sum()


# ----------------------------------------------------------- token choice
def _brute_tc_layout(idx, E, R):
    T, K = idx.shape
    per = E // R
    slot = np.full((T, K), -1, np.int64)
    counts = np.zeros(E, np.int64)
    for e in range(E):
        pairs = [(t, k) for t in range(T) for k in range(K) if idx[t, k] == e]
        for j, (t, k) in enumerate(pairs):
            slot[t, k] = j
        counts[e] = len(pairs)
    in_rank = np.zeros((T, R), np.uint8)
    for t in range(T):
        for r in range(R):
            in_rank[t, r] = any(r * per <= idx[t, k] < (r + 1) * per for k in range(K))
    offsets = np.concatenate([[0], np.cumsum(counts)])
    bad = int(((idx < -1) | (idx >= E)).sum())
    return dict(slot=slot, counts=counts, offsets=offsets, in_rank=in_rank,
                rank_counts=in_rank.sum(axis=0), bad=bad)


TC_CASES = [
    # T, E, R, K, p_neg, dup, p_bad, seed
    (37, 8, 2, 2, 0.0, False, 0.0, 1),
    (64, 16, 4, 4, 0.2, False, 0.0, 2),
    (50, 12, 3, 5, 0.1, True, 0.0, 3),
    (40, 6, 6, 3, 0.3, True, 0.1, 4),
    (9, 64, 32, 40, 0.25, True, 0.05, 5),  # K > 32, R = 32
    (1, 4, 1, 4, 0.0, False, 0.0, 6),
    (20, 5, 1, 1, 1.0, False, 0.0, 7),  # nothing routed
    (0, 8, 2, 2, 0.0, False, 0.0, 8),  # empty
]


def pin_tc_layout_bruteforce(o):
    for T, E, R, K, p_neg, dup, p_bad, seed in TC_CASES:
        idx = W.random_topk(_rng(seed), T, E, K, p_neg=p_neg, allow_dup=dup, p_bad=p_bad).reshape(T, K)
        got = o.tc_layout(idx, E, R)
        ref = _brute_tc_layout(idx, E, R)
        assert np.array_equal(got["slot"], ref["slot"]), (T, E, R, K)
        assert np.array_equal(got["num_tokens_per_expert"], ref["counts"])
        assert np.array_equal(got["expert_offsets"], ref["offsets"])
        assert np.array_equal(got["is_token_in_rank"], ref["in_rank"])
        assert np.array_equal(got["num_tokens_per_rank"], ref["rank_counts"])
        assert got["bad_index_count"] == ref["bad"]


def pin_tc_layout_invariants(o):
    for cfg in (1, 3):
        inp = W.make_inputs(cfg)
        idx = inp["topk_idx"]
        E, R = inp["cfg"]["E"], inp["cfg"]["R"]
        L = o.tc_layout(idx, E, R)
        valid = (idx >= 0) & (idx < E)
        assert L["num_tokens_per_expert"].sum() == valid.sum()
        assert L["expert_offsets"][-1] == valid.sum()
        assert L["num_tokens_per_rank"].sum() == L["is_token_in_rank"].sum()
        # within an expert, (token, k) ascending with slots 0..n-1
        for e in range(E):
            t, k = np.nonzero(idx == e)
            order = np.lexsort((k, t))
            assert np.array_equal(L["slot"][t[order], k[order]], np.arange(len(t)))


def _expected_row(e, s, offsets, mode, max_tokens):
    return e * max_tokens + s if mode == W.PADDED else offsets[e] + s


def pin_tc_dispatch_bruteforce(o):
    rng = _rng(21)
    for (T, E, R, K, H, mode, max_tokens, dt) in [
        (33, 8, 2, 2, 256, W.COMPACT, 0, W.BF16),
        (40, 16, 4, 4, 384, W.PADDED, 6, W.BF16),  # some experts overflow 6 rows
        (25, 8, 8, 3, 256, W.PADDED, 32, W.FP8_E4M3),
        (25, 8, 2, 3, 128, W.COMPACT, 0, W.FP8_E4M3),
    ]:
        idx = W.random_topk(rng, T, E, K, p_neg=0.2, allow_dup=True, p_bad=0.05)
        x = _torch_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
        w = rng.random((T, K)).astype(np.float32)
        L = o.tc_layout(idx, E, R)
        D = o.tc_dispatch(x, idx, E, L, mode=mode, max_tokens=max_tokens, out_dtype=dt, topk_weights=w,
                          want_src=True, want_weights=True)
        rows_seen = set()
        overflow = 0
        for e in range(E):
            pairs = [(t, k) for t in range(T) for k in range(K) if idx[t, k] == e]
            for j, (t, k) in enumerate(pairs):
                if mode == W.PADDED and j >= max_tokens:
                    overflow += 1
                    continue
                row = _expected_row(e, j, L["expert_offsets"], mode, max_tokens)
                rows_seen.add(row)
                if dt == W.BF16:
                    assert np.array_equal(D["recv"][row], x[t])
                else:
                    q, s = o.fp8_quant_row(x[t])
                    assert np.array_equal(D["recv"][row], q) and np.array_equal(D["recv_scales"][row], s)
                assert D["recv_src"][row] == t and D["recv_weights"][row] == w[t, k]
        assert D["overflow_count"] == overflow
        untouched = [r for r in range(D["recv"].shape[0]) if r not in rows_seen]
        assert all(D["recv_src"][r] == -1 for r in untouched)


def _exact_combine(y_f64, rows_w):
    """sum of w*y over (row, w) in fp64 -- exact products, K-term sums."""
    acc = np.zeros(y_f64.shape[1], np.float64)
    mag = np.zeros(y_f64.shape[1], np.float64)
    for row, w in rows_w:
        acc += float(w) * y_f64[row]
        mag += abs(float(w)) * np.abs(y_f64[row])
    return acc, mag


def _bf16_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def pin_tc_combine_exact_bound(o):
    rng = _rng(31)
    for (T, E, R, K, H, mode, max_tokens) in [(30, 8, 2, 4, 256, W.COMPACT, 0), (24, 16, 4, 6, 128, W.PADDED, 5),
                                              (6, 64, 8, 40, 128, W.COMPACT, 0)]:
        idx = W.random_topk(rng, T, E, K, p_neg=0.25, allow_dup=True)
        L = o.tc_layout(idx, E, R)
        rows = E * max_tokens if mode == W.PADDED else int(L["expert_offsets"][-1])
        y = _torch_bf16_bits(rng.standard_normal((rows, H)).astype(np.float32))
        w = rng.standard_normal((T, K)).astype(np.float32)
        yf = _bf16_f64(y)
        for out_dtype in (W.FP32, W.BF16):
            out = o.tc_combine(y, idx, E, L, w, mode=mode, max_tokens=max_tokens, out_dtype=out_dtype)
            outf = out.astype(np.float64) if out_dtype == W.FP32 else _bf16_f64(out)
            for t in range(T):
                rw = []
                per_e = {}
                for k in range(K):
                    e = int(idx[t, k])
                    if e < 0:
                        continue
                    # rank of (t,k) inside expert e, by enumeration
                    j = sum(1 for tt in range(T) for kk in range(K) if idx[tt, kk] == e and (tt, kk) < (t, k))
                    if mode == W.PADDED and j >= max_tokens:
                        continue
                    rw.append((_expected_row(e, j, L["expert_offsets"], mode, max_tokens), w[t, k]))
                exact, mag = _exact_combine(yf, rw)
                bound = (len(rw) + 1) * U32 * mag * 1.0001
                if out_dtype == W.BF16:
                    bound = bound + UBF * np.abs(exact) * 1.0001
                if not rw:
                    assert (outf[t] == 0).all() and not np.signbit(outf[t]).any()
                assert (np.abs(outf[t] - exact) <= bound + 1e-300).all(), (t, out_dtype)


def pin_tc_combine_order_closed_form(o):
    """Two hand-computed fp32 cases.

    (a) terms 1, 2^-24, -1 in k order: an fmaf chain from 0 in ascending k
        gives 0 (1 + 2^-24 rounds to 1); descending k would give 2^-24.
    (b) terms -(1+2^-7) then (1+2^-23)*(1+2^-7): fused multiply-add keeps
        the exact residual 2^-23 + 2^-30; a rounded product would give 2^-23.
    """
    H = 8
    # case (a): three experts, one token, y rows are constants
    idx = np.array([[0, 1, 2]], np.int64)
    L = o.tc_layout(idx, 3, 1)
    y = _torch_bf16_bits(np.array([[1.0] * H, [2.0 ** -24] * H, [-1.0] * H], np.float32))
    w = np.array([[1.0, 1.0, 1.0]], np.float32)
    out = o.tc_combine(y, idx, 3, L, w, out_dtype=W.FP32)
    assert (out == 0.0).all()
    # case (b)
    idx = np.array([[0, 1]], np.int64)
    L = o.tc_layout(idx, 2, 1)
    y = _torch_bf16_bits(np.array([[-(1 + 2.0 ** -7)] * H, [1 + 2.0 ** -7] * H], np.float32))
    w = np.array([[1.0, 1.0 + 2.0 ** -23]], np.float32)
    out = o.tc_combine(y, idx, 2, L, w, out_dtype=W.FP32)
    assert (out == np.float32(2.0 ** -23 + 2.0 ** -30)).all()


def pin_tc_combine_unit_outputs(o):
    """Dispatch then combine with every expert output = 1.0 returns the sum
    of the token's valid gate weights (exact sum within the fp32 bound)."""
    inp = W.make_inputs(5, T=300)
    idx, w = inp["topk_idx"], inp["topk_weights"]
    E, R, K = 256, 8, 8
    L = o.tc_layout(idx, E, R)
    y = np.full((int(L["expert_offsets"][-1]), 128), 0x3F80, np.uint16)  # bf16 1.0
    out = o.tc_combine(y, idx, E, L, w, out_dtype=W.FP32)
    for t in range(idx.shape[0]):
        vw = [Fraction(float(w[t, k])) for k in range(K) if idx[t, k] >= 0]
        exact = float(sum(vw, Fraction(0)))
        bound = (len(vw) + 1) * U32 * sum(abs(float(v)) for v in vw)
        assert np.all(np.abs(out[t].astype(np.float64) - exact) <= bound), t
        if vw:
            assert abs(exact - 1.0) < 1e-6  # Dirichlet weights sum to one


def pin_tc_cfg1_closed_form(o):
    """Workload 1: expert e's output is its dispatched rows times (e+1), so
    combine must return x_t * sum_k w_k (e_k+1) up to the bf16 rounding of
    the expert outputs and the fp32 sum."""
    inp = W.make_inputs(1)
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    E, R = 8, 2
    L = o.tc_layout(idx, E, R)
    D = o.tc_dispatch(x, idx, E, L, want_src=True)
    recv = D["recv"]
    expert_of_row = np.searchsorted(L["expert_offsets"], np.arange(recv.shape[0]), side="right") - 1
    y = _torch_bf16_bits((_bf16_f64(recv) * (expert_of_row[:, None] + 1)).astype(np.float32))
    out = o.tc_combine(y, idx, E, L, w, out_dtype=W.FP32)
    xf = _bf16_f64(x)
    coef = (w.astype(np.float64) * (idx + 1)).sum(axis=1)
    mag = (np.abs(w.astype(np.float64)) * (idx + 1)).sum(axis=1)
    exact = xf * coef[:, None]
    bound = (UBF + 3 * U32) * np.abs(xf) * mag[:, None] * 1.0001
    assert (np.abs(out - exact) <= bound).all()


# --------------------------------------------------- per-rank (dedup) path
def _brute_rank(idx, E, R):
    """Rank r's tokens by enumeration from topk_idx itself: the tokens with
    at least one valid expert in r's block, ascending; rows laid end to end."""
    T, K = idx.shape
    per = E // R
    lists = [[t for t in range(T) if any(0 <= idx[t, k] < E and idx[t, k] // per == r for k in range(K))]
             for r in range(R)]
    offsets = np.concatenate([[0], np.cumsum([len(l) for l in lists])])
    row = np.full((T, R), -1, np.int64)
    for r in range(R):
        for j, t in enumerate(lists[r]):
            row[t, r] = offsets[r] + j
    return offsets, row


def pin_rank_layout_bruteforce(o):
    for T, E, R, K, p_neg, dup, p_bad, seed in TC_CASES:
        idx = W.random_topk(_rng(seed), T, E, K, p_neg=p_neg, allow_dup=dup, p_bad=p_bad).reshape(T, K)
        L = o.tc_layout(idx, E, R)
        got = o.rank_layout(L["is_token_in_rank"])
        offsets, row = _brute_rank(idx, E, R)
        assert np.array_equal(got["rank_offsets"], offsets), (T, E, R, K)
        assert np.array_equal(got["rank_row"], row)
        assert got["rank_offsets"][-1] == L["num_tokens_per_rank"].sum()


def pin_rank_dispatch_bruteforce(o):
    """Each (token, rank) row holds x[t] once; its K entries are the local
    ids and weights of the token's experts in that rank (-1 / 0 elsewhere);
    every valid (t, k) pair appears in exactly one received row."""
    rng = _rng(61)
    for T, E, R, K, H in [(37, 16, 4, 5, 64), (20, 8, 8, 3, 128), (9, 64, 32, 40, 32)]:
        idx = W.random_topk(rng, T, E, K, p_neg=0.2, allow_dup=True, p_bad=0.05)
        x = _torch_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
        w = rng.random((T, K)).astype(np.float32)
        L = o.tc_layout(idx, E, R)
        RL = o.rank_layout(L["is_token_in_rank"])
        D = o.rank_dispatch(x, idx, E, R, RL, w, want_src=True)
        offsets, row = _brute_rank(idx, E, R)
        per = E // R
        seen = 0
        for t in range(T):
            for r in range(R):
                rw = row[t, r]
                if rw < 0:
                    continue
                assert np.array_equal(D["recv"][rw], x[t]) and D["recv_src"][rw] == t
                for k in range(K):
                    e = int(idx[t, k])
                    if 0 <= e < E and e // per == r:
                        assert D["recv_topk_idx"][rw, k] == e - r * per and D["recv_topk_weights"][rw, k] == w[t, k]
                        seen += 1
                    else:
                        assert D["recv_topk_idx"][rw, k] == -1 and D["recv_topk_weights"][rw, k] == 0.0
        assert seen == int(((idx >= 0) & (idx < E)).sum())
        assert (D["recv_src"] >= 0).all()  # rows are dense


def pin_rank_combine_bound_and_units(o):
    rng = _rng(62)
    T, E, R, K, H = 40, 32, 8, 6, 64
    idx = W.random_topk(rng, T, E, K, p_neg=0.3)
    L = o.tc_layout(idx, E, R)
    RL = o.rank_layout(L["is_token_in_rank"])
    rows = int(RL["rank_offsets"][-1])
    offsets, row = _brute_rank(idx, E, R)
    y = _torch_bf16_bits(rng.standard_normal((rows, H)).astype(np.float32))
    yf = _bf16_f64(y)
    for out_dtype in (W.FP32, W.BF16):
        out = o.rank_combine(y, RL, out_dtype=out_dtype)
        outf = out.astype(np.float64) if out_dtype == W.FP32 else _bf16_f64(out)
        for t in range(T):
            rs = [row[t, r] for r in range(R) if row[t, r] >= 0]
            exact = yf[rs].sum(axis=0) if rs else np.zeros(H)
            mag = np.abs(yf[rs]).sum(axis=0) if rs else np.zeros(H)
            bound = len(rs) * U32 * mag * 1.0001
            if out_dtype == W.BF16:
                bound = bound + UBF * np.abs(exact) * 1.0001
            assert (np.abs(outf[t] - exact) <= bound + 1e-300).all(), t
            if not rs:
                assert (outf[t] == 0).all() and not np.signbit(outf[t]).any()
    ones = np.full((rows, 8), 0x3F80, np.uint16)  # every rank sends back 1.0
    out = o.rank_combine(ones, RL, out_dtype=W.FP32)
    assert np.array_equal(out[:, 0], L["is_token_in_rank"].sum(axis=1).astype(np.float32))


def pin_rank_combine_order_closed_form(o):
    """One token in ranks 0, 1, 2 returning 1, 2^-24, -1: ascending-rank fp32
    addition gives exactly 0 (1 + 2^-24 rounds to 1); any other order that
    adds 2^-24 last, or first to -1, does not."""
    idx = np.array([[0, 1, 2]], np.int64)
    L = o.tc_layout(idx, 3, 3)
    RL = o.rank_layout(L["is_token_in_rank"])
    assert RL["rank_row"].tolist() == [[0, 1, 2]]
    y = _torch_bf16_bits(np.array([[1.0] * 4, [2.0 ** -24] * 4, [-1.0] * 4], np.float32))
    assert (o.rank_combine(y, RL, out_dtype=W.FP32) == 0.0).all()
    y = _torch_bf16_bits(np.array([[-1.0] * 4, [2.0 ** -24] * 4, [1.0] * 4], np.float32))
    assert (o.rank_combine(y, RL, out_dtype=W.FP32) == np.float32(2.0 ** -24)).all()


def pin_rank_path_matches_expert_path(o):
    """Rank dispatch, a per-rank weighted sum over the local experts (each
    expert returning its input unchanged), then rank combine equals the
    per-expert dispatch + weighted combine within the fp32 bound: both are
    sum_k w_k x_t."""
    inp = W.make_inputs(2, T=64)
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    E, R, K = 256, 8, 8
    L = o.tc_layout(idx, E, R)
    RL = o.rank_layout(L["is_token_in_rank"])
    D = o.rank_dispatch(x, idx, E, R, RL, w)
    xr = _bf16_f64(D["recv"])
    yr = (xr * D["recv_topk_weights"].astype(np.float64).sum(axis=1)[:, None]).astype(np.float32)
    out_rank = o.rank_combine(_torch_bf16_bits(yr), RL, out_dtype=W.FP32).astype(np.float64)
    out_exp = o.tc_combine(o.tc_dispatch(x, idx, E, L)["recv"], idx, E, L, w, out_dtype=W.FP32).astype(np.float64)
    xf = _bf16_f64(x)
    mag = np.abs(xf) * np.abs(w.astype(np.float64)).sum(axis=1)[:, None]
    bound = (2 * UBF + (K + R + 2) * U32) * mag * 1.0001
    assert (np.abs(out_rank - out_exp) <= bound + 1e-300).all()


# ----------------------------------------------------------- expert choice
def _brute_ec(ti, T, R):
    E, C = ti.shape
    per = E // R
    flat = ti.reshape(-1)
    lists = [[s for s in range(E * C) if flat[s] == t] for t in range(T)]
    offsets = np.concatenate([[0], np.cumsum([len(l) for l in lists])])
    slots = np.array([s for l in lists for s in l], np.int64)
    counts = np.array([int(((ti[e] >= 0) & (ti[e] < T)).sum()) for e in range(E)])
    in_rank = np.zeros((T, R), np.uint8)
    for t in range(T):
        for s in lists[t]:
            in_rank[t, (s // C) // per] = 1
    bad = int(((flat < -1) | (flat >= T)).sum())
    return dict(offsets=offsets, slots=slots, counts=counts, in_rank=in_rank, bad=bad)


EC_CASES = [
    # T, E, C, R, p_neg, p_bad, seed
    (50, 8, 16, 2, 0.0, 0.0, 1),
    (20, 16, 8, 4, 0.2, 0.05, 2),
    (5, 40, 6, 8, 0.1, 0.0, 3),  # few tokens, many picks each
    (300, 4, 5, 1, 0.0, 0.0, 4),  # most tokens unpicked
    (1, 3, 2, 3, 0.5, 0.0, 5),
]


def pin_ec_layout_bruteforce(o):
    for T, E, C, R, p_neg, p_bad, seed in EC_CASES:
        ti = W.random_token_indices(_rng(seed), T, E, C, p_neg=p_neg, p_bad=p_bad)
        got = o.ec_layout(ti, T, R)
        ref = _brute_ec(ti, T, R)
        n = int(ref["offsets"][-1])
        assert np.array_equal(got["token_offsets"], ref["offsets"])
        assert np.array_equal(got["token_slots"][:n], ref["slots"])
        assert np.array_equal(got["num_tokens_per_expert"], ref["counts"])
        assert np.array_equal(got["is_token_in_rank"], ref["in_rank"])
        assert np.array_equal(got["num_tokens_per_rank"], ref["in_rank"].sum(axis=0))
        assert got["bad_index_count"] == ref["bad"]


def pin_ec_dispatch_bruteforce(o):
    rng = _rng(41)
    T, E, C, H = 30, 6, 7, 128
    ti = W.random_token_indices(rng, T, E, C, p_neg=0.2, p_bad=0.1)
    x = _torch_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    sentinel = np.full((E * C, H), 0x7FC1, np.uint16)
    recv = o.ec_dispatch(x, ti, recv=sentinel.copy())
    for e in range(E):
        for c in range(C):
            t = ti[e, c]
            if 0 <= t < T:
                assert np.array_equal(recv[e * C + c], x[t])
            else:
                assert (recv[e * C + c] == 0x7FC1).all()


def pin_ec_combine_bound(o):
    rng = _rng(42)
    for (T, E, C, R) in [(40, 8, 12, 2), (6, 48, 4, 4)]:
        ti = W.random_token_indices(rng, T, E, C, p_neg=0.15)
        L = o.ec_layout(ti, T, R)
        y = _torch_bf16_bits(rng.standard_normal((E * C, 64)).astype(np.float32))
        w = rng.standard_normal((E, C)).astype(np.float32)
        yf = _bf16_f64(y)
        flat = ti.reshape(-1)
        for out_dtype in (W.FP32, W.BF16):
            out = o.ec_combine(y, L, w, T, out_dtype=out_dtype)
            outf = out.astype(np.float64) if out_dtype == W.FP32 else _bf16_f64(out)
            for t in range(T):
                rw = [(s, w.reshape(-1)[s]) for s in range(E * C) if flat[s] == t]
                exact, mag = _exact_combine(yf, rw)
                bound = (len(rw) + 1) * U32 * mag * 1.0001
                if out_dtype == W.BF16:
                    bound = bound + UBF * np.abs(exact) * 1.0001
                if not rw:
                    assert (outf[t] == 0).all()
                assert (np.abs(outf[t] - exact) <= bound + 1e-300).all()


def pin_ec_order_closed_form(o):
    """Token 0 picked in slots 0, 1, 2 (ascending s) with products 1, 2^-24,
    -1: ascending-slot fmaf chain gives exactly 0; and a fused-residual case
    as in the token-choice order pin."""
    ti = np.array([[0], [0], [0]], np.int32)  # E=3, C=1
    L = o.ec_layout(ti, 1, 1)
    y = _torch_bf16_bits(np.array([[1.0] * 4, [2.0 ** -24] * 4, [-1.0] * 4], np.float32))
    w = np.ones((3, 1), np.float32)
    assert (o.ec_combine(y, L, w, 1, out_dtype=W.FP32) == 0.0).all()
    # fused: -(1+2^-7) + (1+2^-23)(1+2^-7) keeps the residual 2^-23 + 2^-30
    ti = np.array([[0], [0]], np.int32)
    L = o.ec_layout(ti, 1, 1)
    y = _torch_bf16_bits(np.array([[-(1 + 2.0 ** -7)] * 4, [1 + 2.0 ** -7] * 4], np.float32))
    w = np.array([[1.0], [1.0 + 2.0 ** -23]], np.float32)
    assert (o.ec_combine(y, L, w, 1, out_dtype=W.FP32) == np.float32(2.0 ** -23 + 2.0 ** -30)).all()


def pin_ec_workload_unit_weights(o):
    """Workload 4 (reduced T): with unit expert outputs, every picked token's
    combine equals the sum of its softmax weights, i.e. 1 within the bound."""
    inp = W.make_inputs(4, T=1024)
    ti, w = inp["token_indices"], inp["expert_weights"]
    L = o.ec_layout(ti, 1024, 1)
    y = np.full((ti.size, 8), 0x3F80, np.uint16)
    out = o.ec_combine(y, L, w, 1024, out_dtype=W.FP32)
    deg = np.diff(L["token_offsets"])
    assert deg.max() > 32  # popular tokens exceed the 32-pick token-choice limit
    picked = deg > 0
    assert np.all(np.abs(out[picked] - 1.0) <= (deg[picked, None] + 2) * 2.0 ** -23)
    assert (out[~picked] == 0).all()


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
