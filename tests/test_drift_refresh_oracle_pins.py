"""Pins for the adaptive-refresh oracle (oracle/drift_refresh.py): the two
limits that reduce to pinned schedules, brute force for the prefix share,
closed forms for the query drift, the depth-aware rule, and negative controls
that plant a mistake in a copy of the oracle and check that a pin catches it.

Citations: Elastic-Cache, Abstract (attention-aware drift test; depth-aware
refresh from a chosen layer onward); LaCache App. C (cache update interval);
FlashBlock, Abstract (cached block-external attention).
"""
import numpy as np
import pytest

from oracle import drift_refresh as dr
from oracle import fbk_oracle as orc


def rnd(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def make_layer(seed, S=4, b=2, Hq=4, Hkv=2, d=8, B=3, lens=(6, 0), moving=True, tau=0.5):
    kp = [rnd((Hkv, L, d), seed + 10 + i) for i, L in enumerate(lens)]
    vp = [rnd((Hkv, L, d), seed + 20 + i) for i, L in enumerate(lens)]
    q0 = rnd((b, B, Hq, d), seed)
    steps = []
    for s in range(S):
        q = rnd((b, B, Hq, d), seed + 100 + s) if moving else q0
        steps.append((q, rnd((b, B, Hkv, d), seed + 200 + s), rnd((b, B, Hkv, d), seed + 300 + s)))
    return {"steps": steps, "k_pfx": kp, "v_pfx": vp, "lens": np.array(lens), "n_kv_heads": Hkv,
            "tau": tau, "base": 1e4}


def same_outputs(a, b, tol=1e-12):
    for (oa, la), (ob, lb) in zip(a, b):
        assert np.allclose(oa, ob, atol=tol, rtol=tol) and np.allclose(la, lb, atol=tol, rtol=tol)


def test_theta_zero_is_refresh_every_step():
    layers = [make_layer(1), make_layer(2)]
    outs, drift, ref = dr.adaptive_schedule(layers, 0.0)
    assert ref.all()
    for li, L in enumerate(layers):
        r1 = orc.refresh_schedule(L["steps"], L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"], L["tau"],
                                  L["base"], 1)
        same_outputs(outs[li], r1)
        # every step with state from its own queries is uncached attention
        for s, (q, k, v) in enumerate(L["steps"]):
            full = orc.full_attention(q, k, v, L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"], L["tau"],
                                      L["base"])
            same_outputs([outs[li][s]], [full], 1e-10)


def test_theta_infinite_is_the_reuse_schedule():
    layers = [make_layer(3), make_layer(4)]
    outs, drift, ref = dr.adaptive_schedule(layers, np.inf)
    assert ref[0].all() and not ref[1:].any()
    assert (drift[:-1] > 0).all()  # the queries moved: there was drift to ignore
    for li, L in enumerate(layers):
        same_outputs(outs[li], orc.block_schedule(L["steps"], L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"],
                                                  L["tau"], L["base"]))


def test_static_queries_never_drift():
    L = make_layer(5, moving=False)
    outs, drift, ref = dr.adaptive_schedule([L], 0.0)
    assert np.all(drift == 0) and ref[0].all() and not ref[1:].any()
    # the reused state was computed from the very queries of every step: exact
    same_outputs(outs[0], orc.refresh_schedule(L["steps"], L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"],
                                               L["tau"], L["base"], 1), 1e-12)


def test_depth_aware_refresh_covers_deeper_layers_only():
    moving, static = make_layer(6), make_layer(7, moving=False)
    _, drift, ref = dr.adaptive_schedule([moving, static], 0.0)
    assert ref[1:, 0].all() and ref[1:, 1].all()  # the deeper static layer follows the shallow one
    assert np.all(drift[:, 1] == 0)
    _, drift, ref = dr.adaptive_schedule([static, moving], 0.0)
    assert not ref[1:, 0].any() and ref[1:, 1].all()  # a deeper trigger leaves the shallower layer alone


def test_refresh_pattern_matches_the_schedule_and_forcing_reproduces_it():
    layers = [make_layer(8, S=6), make_layer(9, S=6, moving=False), make_layer(10, S=6)]
    _, drift0, _ = dr.adaptive_schedule(layers, np.inf)
    theta = float(np.median(drift0[:-1, 0]))  # some steps over, some under
    outs, drift, ref = dr.adaptive_schedule(layers, theta)
    assert 0 < ref[1:].sum() < ref[1:].size
    np.testing.assert_array_equal(ref, dr.refresh_pattern(drift, theta))
    outs_f, drift_f, ref_f = dr.adaptive_schedule(layers, theta, forced=ref)
    np.testing.assert_array_equal(ref_f, ref)
    np.testing.assert_array_equal(drift_f, drift)
    for a, b in zip(outs, outs_f):
        same_outputs(a, b, 0.0)


def brute_prefix_share(q, k, v, kp, vp, lens, Hkv, tau, base):
    """Softmax over [prefix ; block] keys written out, prefix weights summed."""
    b, B, Hq, d = q.shape
    out = np.zeros((b, Hq, B))
    for bi in range(b):
        L = int(lens[bi])
        pos = L + np.arange(B)
        for h in range(Hq):
            g = orc.kv_head_of(h, Hq, Hkv)
            qh = orc.rope(q[bi, :, h, :], pos, base)
            keys = np.concatenate([kp[bi][g], orc.rope(k[bi, :, g, :], pos, base)], axis=0)
            s = tau * qh @ keys.T
            w = np.exp(s - s.max(axis=1, keepdims=True))
            w /= w.sum(axis=1, keepdims=True)
            out[bi, h] = w[:, :L].sum(axis=1)
    return out


def test_prefix_share_equals_brute_force():
    L = make_layer(11, lens=(7, 0))
    q, k, v = L["steps"][0]
    pfx = orc.prefix_partial(q, L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"], L["tau"], L["base"])
    blk = orc.block_partial(q, k, v, L["lens"], L["n_kv_heads"], L["tau"], L["base"])
    got = dr.prefix_share(pfx, blk)
    ref = brute_prefix_share(q, k, v, L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"], L["tau"], L["base"])
    assert np.max(np.abs(got - ref)) < 1e-14
    assert np.all(got[1] == 0)  # the empty prefix carries no mass


def test_query_drift_closed_forms_and_rotation_invariance():
    x = rnd((1, 1, 1, 8), 12)
    y = rnd((1, 1, 1, 8), 13)
    y = y - (np.sum(x * y) / np.sum(x * x)) * x  # orthogonal to x
    assert abs(dr.query_drift(x, 3.0 * x)[0, 0, 0]) < 1e-15
    assert abs(dr.query_drift(x, -x)[0, 0, 0] - 2.0) < 1e-15
    assert abs(dr.query_drift(x, y)[0, 0, 0] - 1.0) < 1e-14
    assert dr.query_drift(x, np.zeros_like(x))[0, 0, 0] == 0.0
    assert dr.query_drift(x, x.copy())[0, 0, 0] == 0.0  # exactly, not up to rounding
    q, r = rnd((2, 3, 4, 8), 14), rnd((2, 3, 4, 8), 15)
    pos = np.arange(3)[None, :, None] + 37
    a = dr.query_drift(q, r)
    b_ = dr.query_drift(orc.rope(q, pos, 1e4), orc.rope(r, pos, 1e4))
    assert np.max(np.abs(a - b_)) < 1e-13


# ------------------------------------------------------------------ negative controls

def test_negative_control_share_without_rescale_fails():
    """Summing l1 and l2 without the e^(m - M) factors is a plausible mistake."""
    L = make_layer(16, lens=(7, 0), tau=4.0)
    q, k, v = L["steps"][0]
    pfx = orc.prefix_partial(q, L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"], L["tau"], L["base"])
    blk = orc.block_partial(q, k, v, L["lens"], L["n_kv_heads"], L["tau"], L["base"])
    bad = pfx[2] / (pfx[2] + blk[2])
    ref = brute_prefix_share(q, k, v, L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"], L["tau"], L["base"])
    assert np.max(np.abs(bad[0] - ref[0])) > 1e-3


def test_negative_control_refresh_only_the_triggering_layer_fails():
    """Refreshing only the layer whose drift exceeded theta (no depth rule)
    breaks the depth-aware pin."""
    drift = np.array([[0.5, 0.0], [0.0, 0.0]])
    pat = dr.refresh_pattern(drift, 0.1)
    only_own = np.vstack([np.ones(2, dtype=np.int64), (drift[0] > 0.1).astype(np.int64)])
    assert pat[1, 1] == 1 and only_own[1, 1] == 0
    assert not np.array_equal(pat, only_own)
