"""Pins for the sparse block-external attention with a cached residual
(FlashBlock, Abstract: combined with sparse attention as residual reuse; the
reading is fixed in oracle/sparse_residual.py): page scores against brute
force, the selection's order and ties, and the two cases where the
approximation must be exact (every page kept; the dense step itself), checked
against the pinned full-attention oracle. Planted mistakes fail a pin."""
import math

import numpy as np
import pytest

from oracle import fbk_oracle as orc
from oracle import sparse_residual as sr


def rnd(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def make_case(seed, b=2, Hq=4, Hkv=2, d=8, B=3, lens=(37, 20), scale=0.8):
    q = rnd((b, B, Hq, d), seed, scale)
    kb, vb = rnd((b, B, Hkv, d), seed + 1, scale), rnd((b, B, Hkv, d), seed + 2)
    kp = [rnd((Hkv, L, d), seed + 10 + i, scale) for i, L in enumerate(lens)]
    vp = [rnd((Hkv, L, d), seed + 20 + i) for i, L in enumerate(lens)]
    return q, kb, vb, kp, vp, np.array(lens)


def test_page_scores_brute_force():
    q, _, _, kp, _, L = make_case(1)
    got = sr.page_scores(q, kp, L, 2, 0.7, 1e4, page=8)
    for bi in range(2):
        n_pages = math.ceil(L[bi] / 8)
        assert len(got[bi]) == n_pages
        for p in range(n_pages):
            best = -math.inf
            for h in range(4):
                g = h * 2 // 4
                keys = kp[bi][g, p * 8:min(L[bi], p * 8 + 8)]
                kbar = [math.fsum(keys[j, i] for j in range(len(keys))) / len(keys) for i in range(8)]
                for t in range(3):
                    qt = orc.rope(q[bi, t, h], L[bi] + t, 1e4)
                    best = max(best, 0.7 * math.fsum(qt[i] * kbar[i] for i in range(8)))
            assert abs(got[bi][p] - best) <= 1e-12 * max(1.0, abs(best))


def test_select_pages_order_and_ties():
    sel = sr.select_pages([np.array([1.0, 3.0, 3.0, 0.5, 2.0])], 3)
    np.testing.assert_array_equal(sel[0], [1, 2, 4])
    sel = sr.select_pages([np.array([2.0, 2.0, 2.0])], 2)
    np.testing.assert_array_equal(sel[0], [0, 1])
    sel = sr.select_pages([np.array([0.1, 0.2])], 5)
    np.testing.assert_array_equal(sel[0], [0, 1])


def check_exact_cases(approx, res_fn=sr.residual):
    page, tau, base = 8, 0.9, 1e4
    q0, kb0, vb0, kp, vp, L = make_case(30)
    q1, kb1, vb1, _, _, _ = make_case(40)
    dense0 = orc.prefix_partial(q0, kp, vp, L, 2, tau, base)
    # (1) every page kept: exact at any step
    allp = [np.arange(math.ceil(x / page)) for x in L]
    res_all = res_fn(dense0, sr.sparse_prefix_partial(q0, kp, vp, L, allp, page, 2, tau, base))
    got, lse = approx(q1, kb1, vb1, kp, vp, L, allp, page, res_all, 2, tau, base)
    full, full_lse = orc.full_attention(q1, kb1, vb1, kp, vp, L, 2, tau, base)
    np.testing.assert_allclose(got, full, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, rtol=1e-12, atol=1e-12)
    # (2) two of five pages kept: exact at the dense step itself, not at another step
    pages = sr.select_pages(sr.page_scores(q0, kp, L, 2, tau, base, page), 2)
    res = res_fn(dense0, sr.sparse_prefix_partial(q0, kp, vp, L, pages, page, 2, tau, base))
    got0, _ = approx(q0, kb0, vb0, kp, vp, L, pages, page, res, 2, tau, base)
    full0, _ = orc.full_attention(q0, kb0, vb0, kp, vp, L, 2, tau, base)
    np.testing.assert_allclose(got0, full0, rtol=1e-10, atol=1e-12)
    got1, _ = approx(q1, kb1, vb1, kp, vp, L, pages, page, res, 2, tau, base)
    assert np.abs(got1 - full).max() > 1e-4     # an approximation elsewhere
    assert np.all(np.isfinite(got1))


def test_exact_cases():
    check_exact_cases(sr.approx_step_output)


def test_empty_prefix_is_block_attention():
    q, kb, vb, kp, vp, L = make_case(50, lens=(0, 12))
    dense = orc.prefix_partial(q, kp, vp, L, 2, 1.0, 1e4)
    pages = [np.zeros(0, dtype=np.int64), np.array([0])]
    res = sr.residual(dense, sr.sparse_prefix_partial(q, kp, vp, L, pages, 8, 2, 1.0, 1e4))
    got, _ = sr.approx_step_output(q, kb, vb, kp, vp, L, pages, 8, res, 2, 1.0, 1e4)
    blk, _ = orc.finalize(orc.block_partial(q, kb, vb, L, 2, 1.0, 1e4))
    np.testing.assert_allclose(got[0], blk[0], rtol=1e-12, atol=1e-14)
    assert np.all(np.isfinite(got))


def test_negative_controls():
    def flipped(dense, sparse):
        r_o, r_l, e = sr.residual(dense, sparse)
        return -r_o, -r_l, e

    def state_space(dense, sparse):       # subtracts states with different maxima
        _, _, e = sr.residual(dense, sparse)
        return dense[0] / dense[2][..., None] - sparse[0] / dense[2][..., None], dense[1] - sparse[1], e
    for bad in (flipped, state_space):
        with pytest.raises(AssertionError):
            check_exact_cases(sr.approx_step_output, bad)
