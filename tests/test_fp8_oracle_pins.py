"""Pins for the per-group FP8 quantisation oracle (LaCache §3.4, Eq. 7-8):
the E4M3 format table, round trips and ties, agreement with torch's own fp32 ->
float8_e4m3fn conversion, a hand-computed fixture, invariants of Eq. 7-8, and
negative controls that plant mistakes in copies of the oracle (on the CPU)."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import fp8_quant as fq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x):
    """fp32 values that are exact in bf16 -> their bit patterns."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all(b & 0xFFFF == 0), "value is not exact in bf16"
    return (b >> 16).astype(np.uint16)


def rand_bf16(shape, seed, scale=1.0):
    r = np.random.Generator(np.random.PCG64(seed))
    x = (r.standard_normal(shape) * scale).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 pattern is fine


# ------------------------------------------------------------------ the E4M3 format

def check_table(value):
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3C: 1.5,
             0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0, 0x77: 240.0}
    for c, v in known.items():
        assert value(c) == v, hex(c)
    assert np.signbit(value(0x80)) and value(0x80) == 0
    assert np.isnan(value(0x7F)) and np.isnan(value(0xFF))
    pos = value(np.arange(0x7F))
    assert np.all(np.diff(pos) > 0)          # codes 0x00..0x7E increase strictly


def test_e4m3_table():
    check_table(fq.e4m3_value)


def check_round_trip_and_ties(encode):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(encode(fq.e4m3_value(codes)), codes)
    # the midpoint of two neighbours goes to the even mantissa, and one fp32
    # step to either side goes to the nearer neighbour
    lo = np.arange(0x00, 0x7E)
    a, b = fq.e4m3_value(lo), fq.e4m3_value(lo + 1)
    mid = ((a + b) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (a + b) / 2)          # exact in fp32
    even = np.where(lo % 2 == 0, lo, lo + 1)
    np.testing.assert_array_equal(encode(mid), even.astype(np.uint8))
    np.testing.assert_array_equal(encode(-mid), (even | 0x80).astype(np.uint8))
    up = np.nextafter(mid, np.float32(np.inf))
    down = np.nextafter(mid, np.float32(0))
    np.testing.assert_array_equal(encode(up), (lo + 1).astype(np.uint8))
    np.testing.assert_array_equal(encode(down), lo.astype(np.uint8))


def test_e4m3_round_trip_and_ties_to_even():
    check_round_trip_and_ties(fq.e4m3_rne_bits)


def test_e4m3_matches_torch_conversion():
    """torch's fp32 -> float8_e4m3fn conversion (round to nearest even) on
    every fp32 value of a bf16 pattern within +-448 and on random fp32."""
    allb = np.arange(1 << 16, dtype=np.uint32)
    x = (allb << 16).view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448)]
    r = np.random.Generator(np.random.PCG64(5)).uniform(-448, 448, 200_000).astype(np.float32)
    tiny = np.random.Generator(np.random.PCG64(6)).uniform(-2 ** -5, 2 ** -5, 200_000).astype(np.float32)
    for v in (x, r, tiny):
        want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        np.testing.assert_array_equal(fq.e4m3_rne_bits(v), want)


# ------------------------------------------------------------------ Eq. 7-8

def check_golden(quant):
    with open(os.path.join(GOLDEN, "fp8_group_quant.json")) as f:
        g = json.load(f)
    x = np.zeros((g["rows"], g["cols"]), dtype=np.float32)
    want = np.zeros(x.shape, dtype=np.uint8)
    for e in g["elements"]:
        x[e["row"], e["col"]] = e["x"]
        want[e["row"], e["col"]] = e["code"]
    codes, scales = quant(bf16_bits(x))
    np.testing.assert_array_equal(scales, np.asarray(g["scales"], dtype=np.float32))
    np.testing.assert_array_equal(codes, want)


def test_group_quant_golden():
    check_golden(fq.fp8_group_quant)


def check_invariants(quant):
    xb = rand_bf16((6, 512), 11)
    codes, scales = quant(xb)
    x = fq.bf16_bits_to_f32(xb).astype(np.float64)
    xg = x.reshape(6, 4, 128)
    cg = codes.reshape(6, 4, 128)
    # the largest |x| of every group is coded +-448
    k = np.abs(xg).argmax(axis=2)
    top = np.take_along_axis(cg, k[..., None], axis=2)[..., 0]
    np.testing.assert_array_equal(top & 0x7F, np.full(top.shape, 0x7E, dtype=np.uint8))
    np.testing.assert_array_equal(top >> 7, (np.take_along_axis(xg, k[..., None], 2)[..., 0] < 0).astype(np.uint8))
    # scale is max|x| / 448 to within fp32 rounding
    np.testing.assert_allclose(scales, np.abs(xg).max(axis=2) / 448, rtol=2 ** -24)
    # dequantisation error: half a quantum of x / scale, plus the fp32 division's rounding
    v = xg / scales[..., None].astype(np.float64)
    deq = fq.e4m3_value(cg)
    quantum = np.where(np.abs(v) < 2 ** -6, 2.0 ** -9, np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-30))) - 3))
    assert np.all(np.abs(deq - v) <= quantum / 2 + np.abs(v) * 2 ** -23)
    # scaling a row by 2^k scales its scales by 2^k and leaves the codes alone
    for kexp in (-20, -3, 5, 30):
        xb2 = bf16_bits(fq.bf16_bits_to_f32(xb) * np.float32(2.0 ** kexp))
        c2, s2 = quant(xb2)
        np.testing.assert_array_equal(c2, codes)
        np.testing.assert_array_equal(s2, scales * np.float32(2.0 ** kexp))
    # groups are independent: permuting rows and swapping group columns permutes the result
    perm = np.array([3, 0, 5, 1, 4, 2])
    swapped = xb.reshape(6, 4, 128)[perm][:, [2, 0, 3, 1]].reshape(6, 512)
    c3, s3 = quant(swapped)
    np.testing.assert_array_equal(c3, codes.reshape(6, 4, 128)[perm][:, [2, 0, 3, 1]].reshape(6, 512))
    np.testing.assert_array_equal(s3, scales[perm][:, [2, 0, 3, 1]])


def test_group_quant_invariants():
    check_invariants(fq.fp8_group_quant)


def test_all_zero_group_keeps_signed_zeros():
    x = np.zeros((1, 256), dtype=np.float32)
    x[0, 7] = -0.0
    x[0, 200] = 1.0
    codes, scales = fq.fp8_group_quant(bf16_bits(x))
    assert scales[0, 0] == 0 and scales[0, 1] == np.float32(1 / 448)
    assert codes[0, 7] == 0x80 and np.count_nonzero(codes[0, :128]) == 1
    assert codes[0, 200] == 0x7E


def test_dequant_of_golden():
    codes = np.array([[0x7E, 0x38, 0x80] + [0] * 125], dtype=np.uint8)
    deq = fq.fp8_dequant(codes, np.array([[0.5]], dtype=np.float32))
    assert deq[0, 0] == 224.0 and deq[0, 1] == 0.5 and deq[0, 2] == 0 and np.signbit(deq[0, 2])


# ------------------------------------------------------------------ negative controls

def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def _quant_variant(qmax=448.0, mode="rne", absmax=True, invert=False):
    def quant(x_bits, group=128):
        x = fq.bf16_bits_to_f32(x_bits)
        rows, cols = x.shape
        xg = x.reshape(rows, cols // group, group)
        amax = (np.abs(xg) if absmax else xg).max(axis=2)
        scale = (amax / np.float32(qmax)).astype(np.float32)
        nz = amax > 0
        with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
            s = np.where(nz, scale, np.float32(1))[..., None]
            q = (xg * s if invert else xg / s).astype(np.float32)
        q = np.where(nz[..., None], q, xg)
        q = np.clip(np.nan_to_num(q), -448, 448).astype(np.float32)
        if mode == "rtz":
            codes = fq.e4m3_rne_bits(q)
            back = fq.e4m3_value(codes)
            down = np.abs(back) > np.abs(q)                       # rounded away from zero: step back
            codes = np.where(down & (codes & 0x7F > 0), codes - 1, codes).astype(np.uint8)
        else:
            codes = fq.e4m3_rne_bits(q)
        return codes.reshape(rows, cols), scale
    return quant


def test_negative_controls():
    for bad in (_quant_variant(qmax=240.0), _quant_variant(mode="rtz"), _quant_variant(absmax=False),
                _quant_variant(invert=True)):
        _fails(check_golden, bad)
    _fails(check_invariants, _quant_variant(qmax=240.0))
    _fails(check_invariants, _quant_variant(absmax=False))

    def truncating_encoder(v):
        v = np.asarray(v, dtype=np.float64)
        codes = fq.e4m3_rne_bits(v)
        back = fq.e4m3_value(codes)
        return np.where(np.abs(back) > np.abs(v), codes - 1, codes).astype(np.uint8)
    _fails(check_round_trip_and_ties, truncating_encoder)
