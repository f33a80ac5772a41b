"""CPU oracle for per-group FP8 quantisation of activations.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) may import this
module. It shares no code with the CUDA library and imports nothing from the
``cached_block_attention_b200`` package.

What is computed (LaCache, "Exact Caching and Precision-Adaptive Inference
for Diffusion Large Language Models", §3.4 Mixed precision strategy, Eq. 7-8):
the activation matrix x [rows, cols] is cut into groups of 1 x 128 consecutive
elements of a row; each group g gets the scale

    scale_g = max_{i in g} |x_i| / Q_max                          (Eq. 8)

and each element the code

    x'_i = clip(x_i / scale_g, Q_min, Q_max),  i in g             (Eq. 7)

stored in the FP8 E4M3 format, so that x_i ~ x'_i * scale_g.

Readings taken where the passage is silent:
  * the low-precision format is E4M3 with Q_max = 448 = -Q_min (the FP8 format
    whose tensor-core GEMMs the passage uses for activations);
  * x is bf16 and the arithmetic is fp32: scale_g = fp32(amax / 448) and
    x_i / scale_g are IEEE fp32 divisions (correctly rounded), and the quotient
    is rounded to E4M3 to nearest, ties to even (clip first, so no overflow);
  * a group whose elements are all zero has scale 0 and keeps its zeros
    (with their signs) as codes: Eq. 8 gives scale 0 and Eq. 7 is 0 / 0 there.
"""
from __future__ import annotations

import numpy as np

__all__ = ["GROUP", "Q_MAX", "e4m3_value", "e4m3_rne_bits", "bf16_bits_to_f32", "fp8_group_quant",
           "fp8_dequant"]

GROUP = 128
Q_MAX = 448.0

# E4M3 (OCP FP8): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
# infinities; exponent field 0 holds the subnormals m/8 * 2^-6; the largest
# finite value is 1.75 * 2^8 = 448 (code 0x7E); codes 0x7F / 0xFF are NaN.
_MIN_NORMAL = 2.0 ** -6
_SUB_QUANTUM = 2.0 ** -9


def e4m3_value(code) -> np.ndarray:
    """The real value of E4M3 codes (uint8), NaN for 0x7F / 0xFF."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * _MIN_NORMAL, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 7 == 7), np.nan, mag)
    return s * mag


def e4m3_rne_bits(v) -> np.ndarray:
    """Round values with |v| <= 448 to E4M3, nearest with ties to even, and
    return the codes (uint8). The sign of zero is kept.

    The representable magnitudes below 2^-6 are multiples of 2^-9; in
    [2^e, 2^(e+1)) for e >= -6 they are multiples of 2^(e-3). Dividing by that
    power of two and rounding with rint (half to even) is exact in fp64.
    """
    v = np.asarray(v, dtype=np.float64)
    assert np.all(np.abs(v) <= Q_MAX), "clip before rounding"
    a = np.abs(v)
    _, E = np.frexp(np.where(a > 0, a, 1.0))        # a = f * 2^E, f in [0.5, 1)
    e = E - 1                                        # a in [2^e, 2^(e+1))
    quantum = np.where(a < _MIN_NORMAL, _SUB_QUANTUM, np.exp2(e - 3.0))
    r = np.rint(a / quantum) * quantum               # the rounded magnitude (may carry to 2^(e+1))
    # encode the rounded magnitude
    sub = r < _MIN_NORMAL
    _, Er = np.frexp(np.where(r > 0, r, 1.0))
    er = Er - 1
    e_field = np.where(sub, 0, er + 7)
    m_field = np.where(sub, np.rint(r / _SUB_QUANTUM), np.rint((r / np.exp2(er) - 1.0) * 8.0))
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = code | np.where(np.signbit(v), 0x80, 0)
    return code.astype(np.uint8)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns to their (exact) fp32 values."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def fp8_group_quant(x_bits, group: int = GROUP):
    """Eq. 7-8 on a bf16 matrix [rows, cols] (uint16 bit patterns), cols a
    multiple of `group`. Returns (codes uint8 [rows, cols], scales fp32
    [rows, cols // group])."""
    x = bf16_bits_to_f32(x_bits)
    rows, cols = x.shape
    assert cols % group == 0
    xg = x.reshape(rows, cols // group, group)
    amax = np.abs(xg).max(axis=2)                                   # exact in fp32
    scale = (amax / np.float32(Q_MAX)).astype(np.float32)           # Eq. 8, one fp32 division
    nz = amax > 0
    with np.errstate(invalid="ignore", divide="ignore"):
        q = (xg / np.where(nz, scale, np.float32(1))[..., None]).astype(np.float32)  # Eq. 7, fp32 division
    q = np.where(nz[..., None], q, xg)                              # all-zero group: its zeros
    q = np.clip(q, np.float32(-Q_MAX), np.float32(Q_MAX))           # Eq. 7's clip
    return e4m3_rne_bits(q).reshape(rows, cols), scale


def fp8_dequant(codes, scales, group: int = GROUP) -> np.ndarray:
    """x'_i * scale_g in fp64 (the value the quantised tensor stands for)."""
    c = np.asarray(codes)
    rows, cols = c.shape
    return (e4m3_value(c).reshape(rows, cols // group, group)
            * np.asarray(scales, dtype=np.float64)[..., None]).reshape(rows, cols)
