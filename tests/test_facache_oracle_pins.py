"""Pins for the full-sequence FACache oracle (LaCache §3.3.3, App. J): every
output of a cached step equals plain softmax attention over the whole
sequence (the lossless claim of §3.1), which is itself checked against
pure-Python brute force; with no masked suffix the block rows equal the
block-attention oracle; planted mistakes (on the CPU) fail a pin."""
import math

import numpy as np
import pytest

from oracle import facache as fc
from oracle import fbk_oracle as orc


def rnd(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def make_sequence(seed=5, b=2, N=23, B=4, c0=9, Hq=4, Hkv=2, d=8, base=1e4, scale=0.7):
    """Raw (pre-RoPE) Q/K/V of a whole sequence, split into U (rotated, as
    RoPECache keeps it) and the block C (raw)."""
    q, k, v = rnd((b, N, Hq, d), seed, scale), rnd((b, N, Hkv, d), seed + 1, scale), rnd((b, N, Hkv, d), seed + 2)
    pos = np.arange(N)
    q_rot, k_rot = orc.rope(q, pos[None, :, None], base), orc.rope(k, pos[None, :, None], base)
    up = fc.u_positions(N - B, c0, B)
    cp = c0 + np.arange(B)
    seq = dict(q_rot=q_rot, k_rot=k_rot, v=v, up=up, cp=cp, c0=c0, Hkv=Hkv, base=base)
    u = (q_rot[:, up], k_rot[:, up], v[:, up])
    c = (q[:, cp], k[:, cp], v[:, cp])
    return seq, u, c


def check_lossless(step_fn, state_fn=fc.uu_state, tau=0.8, **kw):
    seq, (qu, ku, vu), (qc, kc, vc) = make_sequence(**kw)
    ref, ref_lse = fc.full_sequence_attention(seq["q_rot"], seq["k_rot"], seq["v"], seq["Hkv"], tau)
    st = state_fn(qu, ku, vu, seq["Hkv"], tau)
    (ou, lu), (oc, lc) = step_fn(st, qu, ku, vu, qc, kc, vc, seq["c0"], seq["Hkv"], tau, seq["base"])
    np.testing.assert_allclose(ou, ref[:, seq["up"]], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(oc, ref[:, seq["cp"]], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lu, ref_lse[:, :, seq["up"]], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lc, ref_lse[:, :, seq["cp"]], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kw", [
    dict(),                                    # prompt before, masked suffix after
    dict(c0=0),                                # the block opens the sequence: U is all suffix
    dict(N=20, B=4, c0=16),                    # no suffix: U is the prefix
    dict(B=1, c0=5, Hq=6, Hkv=3),              # one-token block, GQA 2
    dict(N=40, B=8, c0=17, Hq=4, Hkv=1, d=16), # MQA, longer
    dict(scale=3.0),                           # large logits
])
def test_cached_step_equals_full_sequence_attention(kw):
    check_lossless(fc.facache_step, **kw)


def test_state_is_reused_across_steps():
    """Two steps of one block: the block's Q/K/V change, U and its state do not;
    both steps are exact."""
    seq, (qu, ku, vu), _ = make_sequence(7)
    st = fc.uu_state(qu, ku, vu, 2, 1.0)
    for s in range(2):
        _, _, (qc, kc, vc) = make_sequence(100 + s)
        q_all = fc.assemble_sequence(qu, orc.rope(qc, seq["cp"][None, :, None], 1e4), seq["c0"])
        k_all = fc.assemble_sequence(ku, orc.rope(kc, seq["cp"][None, :, None], 1e4), seq["c0"])
        v_all = fc.assemble_sequence(vu, vc, seq["c0"])
        ref, _ = fc.full_sequence_attention(q_all, k_all, v_all, 2, 1.0)
        (ou, _), (oc, _) = fc.facache_step(st, qu, ku, vu, qc, kc, vc, seq["c0"], 2, 1.0, 1e4)
        np.testing.assert_allclose(ou, ref[:, seq["up"]], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(oc, ref[:, seq["cp"]], rtol=1e-11, atol=1e-13)


def test_no_suffix_block_rows_equal_block_attention_oracle():
    """With the block at the end of the sequence, its rows are the cached block
    attention of the other oracle: prefix keys U, block keys at L + t."""
    N, B, Hkv = 21, 5, 2
    seq, (qu, ku, vu), (qc, kc, vc) = make_sequence(11, N=N, B=B, c0=N - B, Hkv=Hkv)
    st = fc.uu_state(qu, ku, vu, Hkv, 1.0)
    _, (oc, lc) = fc.facache_step(st, qu, ku, vu, qc, kc, vc, N - B, Hkv, 1.0, 1e4)
    kp = [np.transpose(ku[i], (1, 0, 2)) for i in range(ku.shape[0])]   # [Hkv, L, d]
    vp = [np.transpose(vu[i], (1, 0, 2)) for i in range(vu.shape[0])]
    lens = np.full(ku.shape[0], N - B)
    ref, ref_lse = orc.full_attention(qc, kc, vc, kp, vp, lens, Hkv, 1.0, 1e4)
    np.testing.assert_allclose(oc, ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lc, ref_lse, rtol=1e-12, atol=1e-12)


def brute_sequence(q, k, v, Hkv, tau):
    """Per-row, per-key loops with math.fsum and no max shift."""
    b, N, Hq, d = q.shape
    out = np.zeros((b, N, Hq, d))
    for bi in range(b):
        for h in range(Hq):
            g = h * Hkv // Hq
            for i in range(N):
                w = [math.exp(tau * math.fsum(q[bi, i, h, t] * k[bi, j, g, t] for t in range(d))) for j in range(N)]
                den = math.fsum(w)
                for t in range(d):
                    out[bi, i, h, t] = math.fsum(w[j] * v[bi, j, g, t] for j in range(N)) / den
    return out


def test_full_sequence_attention_brute_force():
    q, k, v = rnd((1, 7, 4, 4), 1, 0.8), rnd((1, 7, 2, 4), 2, 0.8), rnd((1, 7, 2, 4), 3)
    got, _ = fc.full_sequence_attention(q, k, v, 2, 0.9)
    np.testing.assert_allclose(got, brute_sequence(q, k, v, 2, 0.9), rtol=1e-12, atol=1e-14)


def test_u_positions():
    np.testing.assert_array_equal(fc.u_positions(6, 2, 3), [0, 1, 5, 6, 7, 8])
    np.testing.assert_array_equal(fc.u_positions(4, 0, 2), [2, 3, 4, 5])
    np.testing.assert_array_equal(fc.u_positions(4, 4, 2), [0, 1, 2, 3])


# ------------------------------------------------------------------ negative controls

def _fails(fn, *a, **kw):
    with pytest.raises(AssertionError):
        fn(*a, **kw)


def test_negative_controls():
    def u_rows_skip_block(st, qu, ku, vu, qc, kc, vc, c0, Hkv, tau, base):
        good_u, good_c = fc.facache_step(st, qu, ku, vu, qc, kc, vc, c0, Hkv, tau, base)
        return orc.finalize(st), good_c

    def c_rows_block_only(st, qu, ku, vu, qc, kc, vc, c0, Hkv, tau, base):
        good_u, _ = fc.facache_step(st, qu, ku, vu, qc, kc, vc, c0, Hkv, tau, base)
        pos = (c0 + np.arange(qc.shape[1]))[None, :, None]
        only_block = fc._state(orc.rope(qc, pos, base), orc.rope(kc, pos, base), vc, Hkv, tau)
        return good_u, orc.finalize(only_block)

    def block_one_late(st, qu, ku, vu, qc, kc, vc, c0, Hkv, tau, base):
        return fc.facache_step(st, qu, ku, vu, qc, kc, vc, c0 + 1, Hkv, tau, base)

    def state_over_all_keys_of_u_rows_twice(qu, ku, vu, Hkv, tau):
        o, m, l = fc.uu_state(qu, ku, vu, Hkv, tau)
        return 2 * o, m, l   # O~ not matching l

    for bad in (u_rows_skip_block, c_rows_block_only, block_one_late):
        _fails(check_lossless, bad)
    _fails(check_lossless, fc.facache_step, state_fn=state_over_all_keys_of_u_rows_twice)
