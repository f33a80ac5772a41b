"""Host checks of the arithmetic the FP8 quantisation kernel uses in place of
IEEE division (csrc/fp8_quant.cu), against the oracle's codes
(oracle/fp8_quant.py, which divides with IEEE fp32 and rounds to nearest even).

The kernel computes, for a group with max|x| = A (a bf16 value):
  * scale = RN(p + RN(A - 448 p) c) with c = RN(1/448), p = RN(A c), which
    must equal the IEEE quotient RN(A / 448);
  * with y = RN(1 / scale) (an approximate reciprocal and one Newton step on
    the device, checked there by test_gpu_fp8_quant.py through the test
    build): n0 = RN(x (-y)), n = RN(n0 + RN(x + n0 scale) (-y)) when
    A >= 2^-80, else n = RN(x / -scale) (the first step of Markstein's
    division, "IA-64 and Elementary Functions"), and the code of x / scale is
    the code of n with the sign flipped; the magnitudes are those of the plain
    form q = RN(q0 + RN(|x| - q0 scale) y), q0 = RN(|x| y), since every step
    is symmetric under negation, so the checks below run the plain form on |x|;
  * the E4M3 rounding is the hardware conversion (round to nearest even); here
    the oracle's encoder stands in for it, so these checks show that the
    quotient gives the oracle's code. The device tests check the codes the
    conversion produces.
The fp32 fused multiply-add is emulated exactly: the product of two fp32
values is exact in fp64, TwoSum gives the rounding error of the fp64 sum, and
a sum that lands exactly on an fp32 midpoint is pushed to the side its error
points to.

The default run samples the (A, x) pairs. FBK_EXHAUSTIVE=1 runs every
positive finite bf16 A with every bf16 x in [0, A] (532.7M pairs); it ran with
no mismatch and takes a few minutes. The scale check always covers every A.
"""
import os

import numpy as np
import pytest

from oracle import fp8_quant as fq

f32, f64 = np.float32, np.float64
EXHAUSTIVE = os.environ.get("FBK_EXHAUSTIVE") == "1"
FMA_DIV_MIN = f32(2.0 ** -80)


def fma32(a, b, c):
    """RN_fp32(a * b + c) for fp32 arrays, exactly."""
    a64, b64, c64 = a.astype(f64), b.astype(f64), c.astype(f64)
    p = a64 * b64                          # exact: 24 + 24 significant bits
    s = p + c64
    bb = s - p
    err = (p - (s - bb)) + (c64 - bb)      # TwoSum: p + c = s + err exactly
    r = s.astype(f32)
    lo = np.where(np.abs(r.astype(f64)) > np.abs(s), np.nextafter(r, f32(0)), r)
    hi = np.nextafter(lo, np.where(s >= 0, f32(np.inf), f32(-np.inf)))
    at_mid = (s == (lo.astype(f64) + hi.astype(f64)) / 2) & (err != 0)
    if at_mid.any():
        away = (err > 0) == (s > 0)
        r = np.where(at_mid, np.where(away, hi, lo), r)
    return r


def kernel_quotient(ax, scale, amax):
    """The kernel's |x| / scale (see the module docstring)."""
    ok = amax >= FMA_DIV_MIN
    y = (f32(1) / np.where(ok, scale, f32(1))).astype(f32)
    q0 = (ax * y).astype(f32)
    q = fma32(fma32(-q0, scale, ax), y, q0)
    return np.where(ok, q, (ax / scale).astype(f32))


def oracle_magnitude(q):
    """E4M3 exponent and mantissa fields of q >= 0, rounded to nearest even
    (the oracle's encoder, standing in for the device's conversion)."""
    return (fq.e4m3_rne_bits(np.minimum(q, f32(448))) & 0x7F).astype(np.uint8)


def kernel_scale(A):
    """The kernel's scale: one correction step from RN(A RN(1/448))."""
    c = np.full_like(A, f32(1) / f32(448))
    p = (A * c).astype(f32)
    return fma32(fma32(-p, np.full_like(A, f32(448)), A), c, p)


def test_kernel_scale_equals_ieee_quotient_for_every_bf16():
    A = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(f32)  # every positive finite bf16
    np.testing.assert_array_equal(kernel_scale(A).view(np.uint32), (A / f32(448)).astype(f32).view(np.uint32))


def test_negative_control_scale_without_correction():
    """RN(A RN(1/448)) alone differs from the quotient for many A."""
    A = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(f32)
    assert int(((A * (f32(1) / f32(448))).astype(f32) != (A / f32(448)).astype(f32)).sum()) > 1000


def test_fma_emulation_on_known_cases():
    one = np.ones(1, f32)
    eps = f32(2.0 ** -23)
    # (1 + 2^-23)^2 - 1 = 2^-22 + 2^-46: a separate multiply would lose the 2^-46
    x = one + eps
    assert fma32(x, x, -one)[0] == f32(2.0 ** -22 + 2.0 ** -46)
    # (1 + 2^-23) * 2^-24 (1 - 2^-23) = 2^-24 - 2^-70; plus c = 1 + 2^-23 the
    # exact sum lies 2^-70 below the fp32 midpoint 1 + 2^-23 + 2^-24, but its
    # fp64 sum is that midpoint, whose tie would go up to the even 1 + 2^-22
    a = np.array([1 + 2.0 ** -23], f32)
    b = np.array([2.0 ** -24 * (1 - 2.0 ** -23)], f32)
    c = np.array([1 + 2.0 ** -23], f32)
    assert (a.astype(f64) * b.astype(f64) + c.astype(f64))[0] == 1 + 2.0 ** -23 + 2.0 ** -24
    assert fma32(a, b, c)[0] == f32(1 + 2.0 ** -23)


def check_pairs(a_bits):
    """Every bf16 x in [0, A] for each A in a_bits: kernel codes == oracle codes."""
    xs = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(f32)
    bad = total = 0
    for i in range(0, len(a_bits), 64):
        A = (a_bits[i:i + 64].astype(np.uint32) << 16).view(f32)
        scale = (A / f32(448)).astype(f32)
        n = np.searchsorted(xs, A, side="right")
        Ar, sr = np.repeat(A, n), np.repeat(scale, n)
        xr = np.concatenate([xs[:k] for k in n])
        got = oracle_magnitude(kernel_quotient(xr, sr, Ar))
        want = fq.e4m3_rne_bits(np.clip((xr / sr).astype(f32), f32(-448), f32(448))) & 0x7F
        bad += int((got != want).sum())
        total += len(xr)
    return bad, total


def test_kernel_codes_equal_oracle_codes():
    a_bits = np.arange(1, 0x7F80)
    if not EXHAUSTIVE:
        r = np.random.Generator(np.random.PCG64(8))
        a_bits = np.unique(np.concatenate([r.choice(a_bits, 600, replace=False),
                                           [1, 2, 0x0080, 0x2180, 0x2200, 0x3F80, 0x43E0, 0x7F7F]]))
    bad, total = check_pairs(a_bits)
    assert total > 0 and bad == 0, f"{bad} of {total} codes differ"


def test_negative_control_without_correction():
    """q0 alone (no residual correction) gives different codes somewhere."""
    def q0_only(ax, scale, amax):
        y = (f32(1) / scale).astype(f32)
        return (ax * y).astype(f32)
    xs = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(f32)
    r = np.random.Generator(np.random.PCG64(9))
    bad = 0
    for a in r.choice(np.arange(0x3000, 0x5000), 200, replace=False):
        A = np.array([a], np.uint32) << 16
        A = A.view(f32)
        scale = (A / f32(448)).astype(f32)
        x = xs[: np.searchsorted(xs, A[0], side="right")]
        got = oracle_magnitude(q0_only(x, np.repeat(scale, len(x)), None))
        want = fq.e4m3_rne_bits(np.clip((x / scale[0]).astype(f32), f32(-448), f32(448))) & 0x7F
        bad += int((got != want).sum())
    assert bad > 0
