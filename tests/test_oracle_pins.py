"""Pins for the fp64 oracle: closed forms, invariants, brute force and a
hand-computed fixture, plus negative controls that plant mistakes in copies of
oracle functions (on the CPU) and check that a pin fails.

Citations: LaCache ("Exact Caching and Precision-Adaptive Inference for
Diffusion Large Language Models") §3.3.2 (RoPECache, Eq. 1), §3.3.3 (FACache,
Eq. 2-6), §3.1 (mathematically equivalent output), App. J (FACache pseudocode:
initialise with cache, final normalisation and logsumexp); FlashBlock
("Attention Caching for Efficient Long-Context Block Diffusion"), Abstract.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fbk_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def make_case(seed, b=2, Hq=4, Hkv=2, d=8, B=3, lens=(5, 0), scale=1.0):
    q = rnd((b, B, Hq, d), seed, scale)
    kb = rnd((b, B, Hkv, d), seed + 1, scale)
    vb = rnd((b, B, Hkv, d), seed + 2)
    kp = [rnd((Hkv, L, d), seed + 10 + i, scale) for i, L in enumerate(lens)]
    vp = [rnd((Hkv, L, d), seed + 20 + i) for i, L in enumerate(lens)]
    return q, kb, vb, kp, vp, np.array(lens)


# ------------------------------------------------------------------ RoPE

def check_rope_closed_form(rope):
    # d = 2: theta_0 = 1, so RoPE is the plane rotation by `pos` radians.
    x = np.array([0.3, -1.7])
    for pos in (0.0, 1.0, 2.5, 131071.0):
        c, s = math.cos(pos), math.sin(pos)
        want = np.array([c * 0.3 - s * (-1.7), s * 0.3 + c * (-1.7)])
        np.testing.assert_allclose(rope(x, pos, 10000.0), want, rtol=0, atol=1e-12)
    # d = 4, base 16: theta = (1, 1/4); pair (1, 3) turns by pos/4.
    e1 = np.array([0.0, 1.0, 0.0, 0.0])
    got = rope(e1, 2.0, 16.0)
    np.testing.assert_allclose(got, [0.0, math.cos(0.5), 0.0, math.sin(0.5)], atol=1e-15)


def test_rope_closed_form():
    check_rope_closed_form(orc.rope)


def test_rope_identity_norm_relative():
    x = rnd((5, 64), 3)
    np.testing.assert_array_equal(orc.rope(x, 0, 1e4), x)
    for base in (1e4, 1e6):
        y = orc.rope(x, np.arange(5) * 977 + 131000, base)
        np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    q, k = rnd(64, 4), rnd(64, 5)
    ref = orc.rope(q, 17, 1e4) @ orc.rope(k, 5, 1e4)
    for c in (1, 100, 4096, 131000):
        np.testing.assert_allclose(orc.rope(q, 17 + c, 1e4) @ orc.rope(k, 5 + c, 1e4), ref, rtol=0,
                                   atol=1e-10)


# ------------------------------------------------------------------ softmax state

def check_golden_pow2(softmax_partial, merge):
    g = json.load(open(os.path.join(GOLDEN, "pow2_softmax.json")))
    s = np.array(g["scores_ln2"], dtype=np.float64) * math.log(2.0)
    v = np.array(g["v"], dtype=np.float64)
    o, m, l = softmax_partial(s, v)
    ex = g["expected"]
    f = lambda a: np.array([[float(Fraction(t)) for t in r] for r in a])
    np.testing.assert_allclose(m / math.log(2.0), ex["m_over_ln2"], atol=1e-14)
    np.testing.assert_allclose(l, [float(Fraction(t)) for t in ex["l"]], rtol=1e-14)
    np.testing.assert_allclose(o, f(ex["o_unnorm"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(o / l[:, None], f(ex["o"]), rtol=1e-14, atol=1e-15)
    li, ri = g["split"]["left"], g["split"]["right"]
    a = softmax_partial(s[:, li], v[li])
    b = softmax_partial(s[:, ri], v[ri])
    for mo, mm, ml in (merge(a, b), merge(b, a)):
        np.testing.assert_allclose(mm, m, atol=1e-14)
        np.testing.assert_allclose(ml, l, rtol=1e-14)
        np.testing.assert_allclose(mo, o, rtol=1e-14, atol=1e-15)


def test_golden_pow2():
    check_golden_pow2(orc.softmax_partial, orc.merge)


def check_online_matches_two_pass(online_partial):
    s = rnd((6, 200), 7, 3.0)
    v = rnd((200, 5), 8)
    o, m, l = orc.softmax_partial(s, v)
    for tile in (1, 3, 64, 200, 512):
        oo, mm, ll = online_partial(s, v, tile)
        np.testing.assert_allclose(mm, m, rtol=0, atol=0)
        np.testing.assert_allclose(ll, l, rtol=1e-12)
        np.testing.assert_allclose(oo, o, rtol=1e-12, atol=1e-13)


def test_online_recurrence_matches_two_pass():
    check_online_matches_two_pass(orc.online_partial)


def test_split_invariance_any_partition_and_order():
    s = rnd((4, 97), 9, 5.0)
    v = rnd((97, 6), 10)
    whole = orc.softmax_partial(s, v)
    rng = np.random.Generator(np.random.PCG64(11))
    for trial in range(6):
        cuts = np.sort(rng.choice(np.arange(1, 97), size=trial + 1, replace=False))
        parts = [orc.softmax_partial(s[:, a:b], v[a:b])
                 for a, b in zip(np.r_[0, cuts], np.r_[cuts, 97])]
        parts.append(orc.softmax_partial(s[:, :0], v[:0]))  # an empty split
        left = parts[0]
        for p in parts[1:]:
            left = orc.merge(left, p)
        right = parts[-1]
        for p in reversed(parts[:-1]):
            right = orc.merge(p, right)
        for st in (left, right):
            np.testing.assert_allclose(st[1], whole[1], atol=1e-13)
            np.testing.assert_allclose(st[2], whole[2], rtol=1e-12)
            np.testing.assert_allclose(st[0], whole[0], rtol=1e-12, atol=1e-13)


def test_empty_state_is_identity_of_merge():
    s = rnd((3, 10), 12)
    v = rnd((10, 4), 13)
    st = orc.softmax_partial(s, v)
    empty = orc.softmax_partial(s[:, :0], v[:0])
    assert np.all(np.isneginf(empty[1])) and np.all(empty[2] == 0) and np.all(empty[0] == 0)
    for mo, mm, ml in (orc.merge(st, empty), orc.merge(empty, st)):
        np.testing.assert_array_equal(mm, st[1])
        np.testing.assert_array_equal(ml, st[2])
        np.testing.assert_array_equal(mo, st[0])
    both = orc.merge(empty, empty)
    assert np.all(np.isneginf(both[1])) and np.all(both[2] == 0) and not np.any(np.isnan(both[0]))


# ------------------------------------------------------------------ full attention

def brute_full(q, kb, vb, kp, vp, lens, Hkv, tau, base):
    """Pure-Python loops: per-element rotation, softmax without max shift, fsum."""
    b, B, Hq, d = q.shape
    half = d // 2
    out = np.zeros((b, B, Hq, d))

    def rot(x, pos):
        y = [0.0] * d
        for i in range(half):
            a = pos * base ** (-2.0 * i / d)
            c, s = math.cos(a), math.sin(a)
            y[i] = x[i] * c - x[i + half] * s
            y[i + half] = x[i + half] * c + x[i] * s
        return y

    for bi in range(b):
        L = int(lens[bi])
        for h in range(Hq):
            g = h * Hkv // Hq
            keys = [list(kp[bi][g, j]) for j in range(L)] + [rot(list(kb[bi, t, g]), L + t) for t in range(B)]
            vals = [list(vp[bi][g, j]) for j in range(L)] + [list(vb[bi, t, g]) for t in range(B)]
            for t in range(B):
                qq = rot(list(q[bi, t, h]), L + t)
                w = [math.exp(tau * math.fsum(qq[i] * k[i] for i in range(d))) for k in keys]
                den = math.fsum(w)
                for c in range(d):
                    out[bi, t, h, c] = math.fsum(w[j] * vals[j][c] for j in range(len(keys))) / den
    return out


@pytest.mark.parametrize("d,lens,B", [(4, (0, 3), 1), (8, (5, 1), 3), (4, (2, 4), 2), (8, (0, 0), 2)])
def test_full_attention_brute_force(d, lens, B):
    q, kb, vb, kp, vp, L = make_case(30 + d + B, d=d, B=B, lens=lens)
    got, _ = orc.full_attention(q, kb, vb, kp, vp, L, 2, 0.9, 100.0)
    want = brute_full(q, kb, vb, kp, vp, L, 2, 0.9, 100.0)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_rows_sum_to_one_and_uniform_when_q_zero():
    q, kb, vb, kp, vp, L = make_case(40, lens=(6, 2))
    ones_p = [np.ones_like(x) for x in vp]
    out, _ = orc.full_attention(q, kb, np.ones_like(vb), kp, ones_p, L, 2, 1.3, 1e4)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-15)
    # q = 0: every logit is 0, so O is the plain mean of the values.
    out, lse = orc.full_attention(np.zeros_like(q), kb, vb, kp, vp, L, 2, 1.3, 1e4)
    for bi in range(2):
        for h in range(4):
            g = h * 2 // 4
            vals = np.concatenate([vp[bi][g], vb[bi, :, g]], axis=0)
            np.testing.assert_allclose(out[bi, :, h], np.broadcast_to(vals.mean(0), (3, 8)), atol=1e-15)
            np.testing.assert_allclose(lse[bi, h], math.log(vals.shape[0]), atol=1e-14)


def test_dominant_logit_selects_its_value():
    # one query row (B = 1); the prefix key j* is 60 / |q^|^2 * q^, all others 0
    d, L = 8, 6
    q = rnd((1, 1, 1, d), 50)
    qh = orc.rope(q[0, 0, 0], L, 1e4)
    kp = np.zeros((1, L, d))
    kp[0, 2] = 60.0 / (qh @ qh) * qh
    vp = rnd((1, L, d), 51)
    kb = np.zeros((1, 1, 1, d))
    vb = rnd((1, 1, 1, d), 52)
    out, lse = orc.full_attention(q, kb, vb, [kp], [vp], np.array([L]), 1, 1.0, 1e4)
    e = math.exp(60.0)
    others = vp[0].sum(0) - vp[0, 2] + vb[0, 0, 0]
    want = (e * vp[0, 2] + others) / (e + L)
    np.testing.assert_allclose(out[0, 0, 0], want, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(out[0, 0, 0], vp[0, 2], rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(lse[0, 0], 60.0 + math.log1p(L / e), atol=1e-13)


# ------------------------------------------------------------------ lossless claim

def check_lossless(prefix_partial, block_partial, merge, finalize, scale=1.0, tau=0.7):
    q, kb, vb, kp, vp, L = make_case(60, lens=(7, 0), scale=scale)
    full, lse = orc.full_attention(q, kb, vb, kp, vp, L, 2, tau, 1e4)
    st = merge(prefix_partial(q, kp, vp, L, 2, tau, 1e4), block_partial(q, kb, vb, L, 2, tau, 1e4))
    out, lse2 = finalize(st)
    np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("scale,tau", [(1.0, 0.7), (3.0, 1.0), (1.0, 1 / math.sqrt(8))])
def test_cached_merge_equals_full_attention(scale, tau):
    check_lossless(orc.prefix_partial, orc.block_partial, orc.merge, orc.finalize, scale, tau)


def test_empty_prefix_reduces_to_block_attention():
    q, kb, vb, kp, vp, L = make_case(70, lens=(0, 0))
    pfx = orc.prefix_partial(q, kp, vp, L, 2, 1.0, 1e4)
    assert np.all(np.isneginf(pfx[1])) and np.all(pfx[2] == 0)
    a, _ = orc.finalize(orc.merge(pfx, orc.block_partial(q, kb, vb, L, 2, 1.0, 1e4)))
    b, _ = orc.finalize(orc.block_partial(q, kb, vb, L, 2, 1.0, 1e4))
    np.testing.assert_array_equal(a, b)


def test_single_key_gives_its_value():
    q, kb, vb, kp, vp, L = make_case(71, b=1, B=1, lens=(0,))
    out, lse = orc.full_attention(q, kb, vb, kp, vp, L, 2, 1.0, 1e4)
    for h in range(4):
        np.testing.assert_allclose(out[0, 0, h], vb[0, 0, h * 2 // 4], rtol=1e-15)


def check_gqa_equals_repeated_mha(full_attention):
    q, kb, vb, kp, vp, L = make_case(80, Hq=6, Hkv=2, lens=(4, 9))
    gqa, _ = full_attention(q, kb, vb, kp, vp, L, 2, 1.0, 1e4)
    rep = np.array([0, 0, 0, 1, 1, 1])  # contiguous groups of Hq/Hkv = 3
    mha, _ = full_attention(q, kb[:, :, rep], vb[:, :, rep], [k[rep] for k in kp],
                            [v[rep] for v in vp], L, 6, 1.0, 1e4)
    np.testing.assert_allclose(gqa, mha, rtol=1e-14, atol=1e-15)


def test_gqa_equals_repeated_mha():
    check_gqa_equals_repeated_mha(orc.full_attention)


# ------------------------------------------------------------------ paged cache and commit

def test_paged_gather_equals_contiguous_any_permutation():
    from cached_block_attention_b200 import synth
    ks = [synth.gen_random((2, L, 8), 90 + L) for L in (70, 0, 129)]
    vs = [synth.gen_random((2, L, 8), 95 + L) for L in (70, 0, 129)]
    lens = np.array([70, 0, 129])
    for seed in (1, 2):
        kp, vp, table = synth.paged_cache(ks, vs, 2, 8, 64, 5, seed)
        gk = orc.gather_paged(kp, table, lens)
        gv = orc.gather_paged(vp, table, lens)
        for i in range(3):
            np.testing.assert_array_equal(gk[i], ks[i])
            np.testing.assert_array_equal(gv[i], vs[i])


def test_bf16_rounding_known_values():
    one = 1.0
    cases = {
        one: one,
        one + 2 ** -8: one,                       # tie -> even mantissa
        one + 3 * 2 ** -8: one + 2 ** -6,         # tie -> even mantissa
        one + 2 ** -8 + 2 ** -40: one + 2 ** -7,  # just above the tie (fp32 detour would give 1.0)
        -(2.0 ** -130): -(2.0 ** -130),           # subnormal, exact
        3.0 * 2 ** -134: 2.0 ** -132,             # subnormal tie -> even (1.5 -> 2 units)
        255.0 / 128 * 2 ** 20: 255.0 / 128 * 2 ** 20,  # largest mantissa, exact
        65504.0 * 1024: 2.0 ** 26,                # rounds up across the binade
    }
    for x, y in cases.items():
        got = orc.bits_to_f64(orc.bf16_rne_bits(np.array([x])))[0]
        assert got == y, (x, got, y)
    # on fp32-exact inputs it agrees with torch's fp32 -> bf16 rounding
    x = rnd(20000, 91, 3.0).astype(np.float32).astype(np.float64)
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.bf16_rne_bits(x), t)


def test_commit_contiguous_and_paged():
    from cached_block_attention_b200 import synth
    b, Hkv, d, B, cap = 2, 2, 8, 3, 16
    lens = np.array([0, 5])
    ks = [synth.gen_random((Hkv, L, d), 100 + L) for L in lens]
    vs = [synth.gen_random((Hkv, L, d), 110 + L) for L in lens]
    kc, vc = synth.contiguous_cache(ks, vs, Hkv, d, cap)
    kb = synth.gen_random((b, B, Hkv, d), 120)
    vb = synth.gen_random((b, B, Hkv, d), 121)
    kc2, vc2, lens2 = orc.commit_contiguous(kc, vc, orc.bits_to_f64(kb), vb, lens, 1e4)
    np.testing.assert_array_equal(lens2, lens + B)
    for bi in range(b):
        L = lens[bi]
        np.testing.assert_array_equal(vc2[bi, :, L:L + B], np.transpose(vb[bi], (1, 0, 2)))
        np.testing.assert_array_equal(kc2[bi, :, :L], kc[bi, :, :L])        # untouched
        np.testing.assert_array_equal(kc2[bi, :, L + B:], kc[bi, :, L + B:])
        np.testing.assert_array_equal(vc2[bi, :, L + B:], vc[bi, :, L + B:])
    # position 0 has angle 0: the stored K is the input K, bit for bit
    np.testing.assert_array_equal(kc2[0, :, 0], kb[0, 0])
    # elsewhere K is bf16(RoPE(k)) within half a bf16 ulp of the fp64 rotation
    rot = orc.rope(orc.bits_to_f64(kb[1, :, 0]), 5 + np.arange(B), 1e4)
    np.testing.assert_allclose(orc.bits_to_f64(kc2[1, 0, 5:8]), rot, rtol=2 ** -8, atol=0)
    # the paged layout holds the same logical cache
    kp, vp, table = synth.paged_cache(ks, vs, Hkv, d, 4, B, 7)
    kp2, vp2, lp2 = orc.commit_paged(kp, vp, table, orc.bits_to_f64(kb), vb, lens, 1e4)
    np.testing.assert_array_equal(lp2, lens2)
    gk, gv = orc.gather_paged(kp2, table, lp2), orc.gather_paged(vp2, table, lp2)
    for bi in range(b):
        np.testing.assert_array_equal(gk[bi], kc2[bi, :, :lens2[bi]])
        np.testing.assert_array_equal(gv[bi], vc2[bi, :, :lens2[bi]])


def test_commit_then_attention_over_cache_matches_step_output():
    """After commit the block's K/V are part of the cache: attention of the same
    block queries (still at positions L..L+B-1) over the L+B cached keys equals
    the step's merged output, up to the bf16 rounding of the committed K."""
    from cached_block_attention_b200 import synth
    b, Hq, Hkv, d, B, L = 1, 4, 2, 16, 4, 9
    lens = np.array([L])
    ks = [synth.gen_random((Hkv, L, d), 130, 0.5)]
    vs = [synth.gen_random((Hkv, L, d), 131)]
    kc, vc = synth.contiguous_cache(ks, vs, Hkv, d, 16)
    q = orc.bits_to_f64(synth.gen_random((b, B, Hq, d), 132, 0.5))
    kb = orc.bits_to_f64(synth.gen_random((b, B, Hkv, d), 133, 0.5))
    vb = synth.gen_random((b, B, Hkv, d), 134)
    kpf, vpf = [orc.bits_to_f64(kc[0, :, :L])], [orc.bits_to_f64(vc[0, :, :L])]
    step, _ = orc.step_output(orc.prefix_partial(q, kpf, vpf, lens, Hkv, 1.0, 1e4),
                              q, kb, orc.bits_to_f64(vb), lens, Hkv, 1.0, 1e4)
    kc2, vc2, lens2 = orc.commit_contiguous(kc, vc, kb, vb, lens, 1e4)
    assert lens2[0] == L + B
    allk, allv = orc.bits_to_f64(kc2[0, :, :L + B]), orc.bits_to_f64(vc2[0, :, :L + B])
    got = np.zeros_like(step)
    for h in range(Hq):
        g = orc.kv_head_of(h, Hq, Hkv)
        qh = orc.rope(q[0, :, h, :], L + np.arange(B), 1e4)
        o, m, l = orc.softmax_partial(qh @ allk[g].T, allv[g])
        got[0, :, h, :] = o / l[:, None]
    err = np.abs(got - step)
    assert err.max() < 1e-2 * np.abs(step).max()
    assert err.mean() < 2e-3 * np.abs(step).mean()
    assert err.max() > 0  # the rounding of committed K is visible, so the test is not vacuous


# ------------------------------------------------------------------ reuse schedule

def test_block_schedule_first_step_is_exact():
    q, kb, vb, kp, vp, L = make_case(140, lens=(6, 3))
    q2, kb2, vb2, _, _, _ = make_case(150, lens=(6, 3))
    outs = orc.block_schedule([(q, kb, vb), (q2, kb2, vb2)], kp, vp, L, 2, 1.0, 1e4)
    full, lse = orc.full_attention(q, kb, vb, kp, vp, L, 2, 1.0, 1e4)
    np.testing.assert_allclose(outs[0][0], full, rtol=1e-12, atol=1e-13)
    # the second step reuses step 1's prefix state: equal to full attention with
    # step-1 queries on the prefix part, by construction of merge + partials
    pfx = orc.prefix_partial(q, kp, vp, L, 2, 1.0, 1e4)
    want = orc.finalize(orc.merge(pfx, orc.block_partial(q2, kb2, vb2, L, 2, 1.0, 1e4)))
    np.testing.assert_allclose(outs[1][0], want[0], rtol=1e-14)


# ------------------------------------------------------------------ refresh interval (LaCache App. C)

def _steps(seed0, n, q_from=None):
    """n steps of fresh (q, k_blk, v_blk); q_from[s] = s' makes step s reuse step s' queries."""
    out = []
    for s in range(n):
        q, kb, vb, _, _, _ = make_case(seed0 + 10 * s, lens=(6, 3))
        out.append([q, kb, vb])
    for s, src in enumerate(q_from or []):
        out[s][0] = out[src][0]
    return [tuple(t) for t in out]


def check_refresh_schedule(refresh_schedule):
    _, _, _, kp, vp, L = make_case(160, lens=(6, 3))
    full = lambda st: orc.full_attention(st[0], st[1], st[2], kp, vp, L, 2, 1.0, 1e4)
    # r = 1: every step recomputes, so every step is exact full attention
    steps = _steps(170, 4)
    for st, (o, lse) in zip(steps, refresh_schedule(steps, kp, vp, L, 2, 1.0, 1e4, 1)):
        np.testing.assert_allclose(o, full(st)[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, full(st)[1], rtol=1e-12, atol=1e-13)
    # r >= S: the reuse schedule
    for r in (4, 7):
        for a, b in zip(refresh_schedule(steps, kp, vp, L, 2, 1.0, 1e4, r),
                        orc.block_schedule(steps, kp, vp, L, 2, 1.0, 1e4)):
            np.testing.assert_allclose(a[0], b[0], rtol=1e-14, atol=0)
    # r = 3 over 7 steps whose queries change only at steps 0, 3 and 6: every
    # step's prefix state was refreshed with its own queries, so all are exact
    steps = _steps(200, 7, q_from=[0, 0, 0, 3, 3, 3, 6])
    for st, (o, _) in zip(steps, refresh_schedule(steps, kp, vp, L, 2, 1.0, 1e4, 3)):
        np.testing.assert_allclose(o, full(st)[0], rtol=1e-12, atol=1e-13)
    # queries that change between refreshes (steps 1, 2, 4, 5) are not exact:
    # there the state of the latest refresh step is reused
    steps = _steps(300, 6)
    outs = refresh_schedule(steps, kp, vp, L, 2, 1.0, 1e4, 3)
    for s in (1, 2, 4, 5):
        assert np.abs(outs[s][0] - full(steps[s])[0]).max() > 1e-3
        pfx = orc.prefix_partial(steps[3 * (s // 3)][0], kp, vp, L, 2, 1.0, 1e4)
        want = orc.step_output(pfx, *steps[s], L, 2, 1.0, 1e4)
        np.testing.assert_allclose(outs[s][0], want[0], rtol=1e-14, atol=0)


def test_refresh_interval_schedule():
    check_refresh_schedule(orc.refresh_schedule)


def test_refresh_interval_rejects_zero():
    with pytest.raises(ValueError):
        orc.refresh_schedule(_steps(400, 2), [], [], np.array([0, 0]), 2, 1.0, 1e4, 0)


# ------------------------------------------------------------------ negative controls

def _fails(fn, *args, **kw):
    with pytest.raises(AssertionError):
        fn(*args, **kw)


def test_negative_control_merge_without_rescale():
    def bad_merge(a, b):
        return a[0] + b[0], np.maximum(a[1], b[1]), a[2] + b[2]
    _fails(check_lossless, orc.prefix_partial, orc.block_partial, bad_merge, orc.finalize)
    _fails(check_golden_pow2, orc.softmax_partial, bad_merge)


def test_negative_control_rope_position_off_by_one():
    # Shifting block Q and K together leaves block logits unchanged (RoPE is
    # relative), so the planted mistakes move only one side: rotations compose,
    # so rope(x, 1) feeds a vector that ends up one position late.
    def late_block_keys(q, kb, vb, lens, Hkv, tau, base, heads=None, batches=None):
        return orc.block_partial(q, orc.rope(kb, 1, base), vb, lens, Hkv, tau, base, heads, batches)

    def late_prefix_queries(q, kp, vp, lens, Hkv, tau, base, heads=None, batches=None):
        return orc.prefix_partial(orc.rope(q, 1, base), kp, vp, lens, Hkv, tau, base, heads, batches)
    _fails(check_lossless, orc.prefix_partial, late_block_keys, orc.merge, orc.finalize)
    _fails(check_lossless, late_prefix_queries, orc.block_partial, orc.merge, orc.finalize)


def test_negative_control_prefix_omitted():
    def no_prefix(q, kp, vp, lens, Hkv, tau, base, heads=None, batches=None):
        return orc.prefix_partial(q, kp, vp, np.zeros_like(lens), Hkv, tau, base, heads, batches)
    _fails(check_lossless, no_prefix, orc.block_partial, orc.merge, orc.finalize)


def test_negative_control_wrong_kv_head_map():
    real = orc.kv_head_of

    def bad_full(*a, **k):
        orc.kv_head_of = lambda h, Hq, Hkv: h % Hkv
        try:
            return orc.full_attention(*a, **k)
        finally:
            orc.kv_head_of = real
    _fails(check_gqa_equals_repeated_mha, bad_full)


def test_negative_control_rope_sign():
    def bad_rope(x, pos, base):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        ang = np.asarray(pos, dtype=np.float64)[..., None] * orc.rope_freqs(d, base)
        c, s = np.cos(ang), np.sin(ang)
        x1, x2 = x[..., : d // 2], x[..., d // 2:]
        return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)
    _fails(check_rope_closed_form, bad_rope)


def test_negative_control_online_without_alpha():
    def bad_online(s, v, tile):
        R, N = s.shape
        m = np.full(R, -np.inf); l = np.zeros(R); o = np.zeros((R, v.shape[1]))
        for j0 in range(0, N, tile):
            t = s[:, j0:j0 + tile]
            m = np.maximum(m, t.max(1))
            p = np.exp(t - m[:, None])
            l = l + p.sum(1)
            o = o + p @ v[j0:j0 + tile]
        return o, m, l
    _fails(check_online_matches_two_pass, bad_online)


def test_negative_control_refresh_off_by_one():
    def late_refresh(steps, kp, vp, lens, Hkv, tau, base, r, heads=None, batches=None):
        outs, pfx = [], None
        for s, (q, k, v) in enumerate(steps):
            if s % r == min(1, r - 1):
                pfx = orc.prefix_partial(q, kp, vp, lens, Hkv, tau, base)
            if pfx is None:
                pfx = orc.prefix_partial(q, kp, vp, lens, Hkv, tau, base)
            outs.append(orc.step_output(pfx, q, k, v, lens, Hkv, tau, base))
        return outs

    def previous_queries(steps, kp, vp, lens, Hkv, tau, base, r, heads=None, batches=None):
        outs, pfx = [], None
        for s, (q, k, v) in enumerate(steps):
            if s % r == 0:
                pfx = orc.prefix_partial(steps[max(s - 1, 0)][0], kp, vp, lens, Hkv, tau, base)
            outs.append(orc.step_output(pfx, q, k, v, lens, Hkv, tau, base))
        return outs
    _fails(check_refresh_schedule, late_refresh)
    _fails(check_refresh_schedule, previous_queries)
