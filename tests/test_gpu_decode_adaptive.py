"""GPU parity of fbk_decode_block_adaptive: every denoising step of a block for
several layers with the drift-triggered, depth-aware refresh (Elastic-Cache,
Abstract; the rule is oracle/drift_refresh.py's reading).

The refresh decisions are taken on the device in fp32. The tests therefore
check (a) that the device followed its own rule exactly on its own statistics,
(b) that those statistics match the oracle's, and (c) every output row against
the oracle run with the device's decisions; at the two limits (threshold 0 and
+inf) the decisions are checked against the oracle's outright, and the outputs
bit for bit against fbk_decode_block with refresh interval 1 and steps.
"""
import math

import numpy as np
import pytest
import torch

from oracle import drift_refresh as dr
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import fbk  # noqa: F401  (fails loudly if not built)
    yield


def make_layers(cfg, moving, steps, seed):
    """One uploaded Case and LayerBlock per layer; a layer whose `moving` entry
    is False repeats step 0's queries at every step."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, lens, ps, tau, base = cfg
    cases, blocks = [], []
    for i, mv in enumerate(moving):
        c = H.make_case(b, hq, hkv, d, blk, lens, ps, tau, base=base, seed=seed + 37 * i, steps=steps)
        if not mv:
            q0 = c.steps_bits[0][0]
            c.steps_bits = [(q0.copy(), kk, vv) for (_, kk, vv) in c.steps_bits]
        c.upload()
        q = torch.stack([st[0] for st in c.dev["steps"]])
        k = torch.stack([st[1] for st in c.dev["steps"]])
        v = torch.stack([st[2] for st in c.dev["steps"]])
        out = torch.stack([c.out_tensor() for _ in range(steps)])
        lse = torch.empty(steps, b, hq, blk, dtype=torch.float32, device="cuda")
        cases.append(c)
        blocks.append(fbk.LayerBlock(q, k, v, c.dev["cache"], fbk.Partial.empty(c.shape), out, 1, lse))
    return cases, blocks


def oracle_layers(cases, steps):
    return [{"steps": [c.step_f64(s) for s in range(steps)], "k_pfx": c.k_pfx(), "v_pfx": c.v_pfx(),
             "lens": c.lens, "n_kv_heads": c.hkv, "tau": c.tau, "base": c.base} for c in cases]


def run(cases, blocks, theta, steps, commit=True):
    from cached_block_attention_b200 import fbk
    pol = fbk.DriftPolicy.empty(theta, len(blocks), steps)
    fbk.decode_block_adaptive(cases[0].shape, blocks, pol, cases[0].workspace(0), commit=commit)
    torch.cuda.synchronize()
    return pol.drift.cpu().numpy().astype(np.float64), pol.refreshed.cpu().numpy().astype(np.int64)


# (batch, hq, hkv, d, blk, lens, page_size, tau, base), moving queries per layer, steps
CASES = [
    ((2, 4, 4, 64, 16, (100, 37), 0, 1.0, 1e4), (True, False, True), 5),          # MHA, a static middle layer
    ((2, 8, 2, 128, 32, (300, 64), 16, 1 / math.sqrt(128), 1e6), (False, True), 4),  # GQA, pages
    ((3, 28, 4, 128, 32, (0, 129, 700), 0, 1.0, 1e4), (True, True), 4),             # two M-tiles, empty prefix
]


@pytest.mark.parametrize("cfg,moving,steps", CASES)
@pytest.mark.parametrize("theta_kind", ["zero", "mid", "inf"])
def test_adaptive_block_matches_oracle(cfg, moving, steps, theta_kind):
    seed = CASES.index((cfg, moving, steps)) * 1000 + 7
    cases, blocks = make_layers(cfg, moving, steps, seed)
    ol = oracle_layers(cases, steps)
    _, drift_inf, _ = dr.adaptive_schedule(ol, np.inf)
    theta = {"zero": 0.0, "inf": math.inf,
             "mid": float(np.median(drift_inf[:-1][drift_inf[:-1] > 0]))}[theta_kind]
    drift, refreshed = run(cases, blocks, theta, steps)
    # (a) the device followed the rule on its own statistics
    np.testing.assert_array_equal(refreshed, dr.refresh_pattern(drift, theta))
    # (b) its statistics are the oracle's (fp32 from bf16 merges against fp64);
    # a static layer's are exactly zero
    outs, drift_ref, ref_pattern = dr.adaptive_schedule(ol, theta, forced=refreshed)
    assert np.abs(drift - drift_ref).max() <= 2e-3 * max(drift_ref.max(), 1e-3) + 1e-6, (drift, drift_ref)
    for li, mv in enumerate(moving):
        if not mv:
            assert np.all(drift[:, li] == 0.0), drift[:, li]
    if theta_kind != "mid":  # far from every statistic: the decisions are the oracle's outright
        _, _, own = dr.adaptive_schedule(ol, theta)
        np.testing.assert_array_equal(refreshed, own)
    # (c) every row of every step against the oracle with the device's decisions
    for li, blk in enumerate(blocks):
        for s in range(steps):
            H.assert_close(H.host_f64(blk.out[s]), outs[li][s][0], "bf16", f"layer {li} step {s}")
            assert np.abs(H.host_f64(blk.lse[s]) - outs[li][s][1]).max() <= 2e-2
        lens_after = cases[li].dev["cache"].prefix_lens.cpu().numpy()
        np.testing.assert_array_equal(lens_after, cases[li].lens + cases[li].blk)
        assert int(cases[li].dev["cache"].error_flags.item()) == 0


@pytest.mark.parametrize("theta,interval", [(0.0, 1), (math.inf, None)])
def test_limits_equal_fixed_intervals_bit_for_bit(theta, interval):
    """threshold 0 (every layer's queries move at every step) issues the
    refreshes of interval 1, threshold +inf those of one refresh per block:
    the outputs equal fbk_decode_block's bit for bit."""
    from cached_block_attention_b200 import fbk
    cfg, moving, steps = (2, 8, 2, 128, 32, (300, 64), 16, 1.0, 1e4), (True, True, True), 4
    ca, ba = make_layers(cfg, moving, steps, seed=99)
    cb, bb = make_layers(cfg, moving, steps, seed=99)
    _, refreshed = run(ca, ba, theta, steps)
    r = interval or steps
    assert refreshed.sum() == (refreshed.size if r == 1 else len(ba))
    for L in bb:
        L.refresh_interval = r
    fbk.decode_block(cb[0].shape, bb, cb[0].workspace(0), commit=True)
    torch.cuda.synchronize()
    for li, (a, b) in enumerate(zip(ba, bb)):
        assert torch.equal(a.out, b.out), f"layer {li} outputs"
        assert torch.equal(a.lse, b.lse), f"layer {li} lse"


def test_adaptive_block_as_a_cuda_graph():
    """The decisions live on the device, so the whole block is one graph:
    replaying it gives the eager call's outputs and decisions."""
    from cached_block_attention_b200 import fbk
    cfg, moving, steps = (2, 4, 4, 64, 16, (100, 37), 0, 1.0, 1e4), (True, False, True), 5
    cases, blocks = make_layers(cfg, moving, steps, seed=314)
    ol = oracle_layers(cases, steps)
    _, drift_inf, _ = dr.adaptive_schedule(ol, np.inf)
    theta = float(np.median(drift_inf[:-1][drift_inf[:-1] > 0]))
    pol = fbk.DriftPolicy.empty(theta, len(blocks), steps)
    ws = cases[0].workspace(0)
    fbk.decode_block_adaptive(cases[0].shape, blocks, pol, ws, commit=False)
    torch.cuda.synchronize()
    eager = [b.out.clone() for b in blocks]
    eager_ref, eager_drift = pol.refreshed.clone(), pol.drift.clone()
    for b in blocks:
        b.out.zero_()
    pol.refreshed.fill_(-1)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
            fbk.decode_block_adaptive(cases[0].shape, blocks, pol, ws, commit=False, stream=st)
    g.replay()
    torch.cuda.synchronize()
    for e, b in zip(eager, blocks):
        assert torch.equal(e, b.out)
    assert torch.equal(eager_ref, pol.refreshed) and torch.equal(eager_drift, pol.drift)
