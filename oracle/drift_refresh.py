"""fp64 CPU oracle: adaptive refresh of the cached block-external state.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` may import this module. It shares no code with the CUDA library.

Elastic-Cache ("Elastic-Cache", Abstract) decides *when* to refresh cached
attention state with an attention-aware drift test, and *where* with a
depth-aware rule that recomputes from a chosen layer onward while the
shallower layers keep their caches. LaCache App. C instead refreshes at a fixed
interval per layer (``fbk_oracle.refresh_schedule``). This module is the
adaptive variant of that schedule for the state cached here, the block queries'
prefix state (FlashBlock, Abstract: cached block-external attention).

Reading (the pages give the idea, not a formula). The state of a layer was
computed from the block queries of the step at which the layer was last
refreshed (q_ref). Reusing it at the next step s + 1 is exact when the queries
of s + 1 equal q_ref, and its error matters only in proportion to the
attention mass the prefix carries in the row. The drift statistic of a layer
at step s, for the decision about step s + 1, is

    delta_s = max over the block's query rows of
              pi_ext,s * (1 - cos(q_{s+1}, q_ref))

with pi_ext,s the share of the row's softmax mass on the prefix keys at step
s (from the merge of the reused state with the fresh block state) and cos the
cosine between the row's pre-RoPE query vectors (both would be rotated by the
same angle at the same position, so it is also the cosine of the rotated
vectors). 1 - cos is evaluated as |q/|q| - r/|r||^2 / 2, which is exactly 0
for equal vectors; a zero vector counts as no drift. When delta_s > theta,
that layer and every deeper layer recompute their state at step s + 1
(depth-aware); step 0 computes every layer's state; the last step takes no
decision. The queries of step s + 1 are known at step s: a block's denoising
inputs are all in memory when the block runs.

theta = 0 refreshes a layer at every step whose queries differ from its
state's (with queries drawn afresh at every step that is refresh interval 1);
theta = inf never refreshes after step 0, which is the reuse schedule.
"""
from __future__ import annotations

import numpy as np

from . import fbk_oracle as orc


def prefix_share(pfx_state, blk_state):
    """Share of each row's softmax mass on the prefix keys: e^(m1-M) l1 /
    (e^(m1-M) l1 + e^(m2-M) l2), M = max(m1, m2); 0 for an empty prefix.
    Arrays [b, Hq, B]."""
    _, m1, l1 = (np.asarray(t, dtype=np.float64) for t in pfx_state)
    _, m2, l2 = (np.asarray(t, dtype=np.float64) for t in blk_state)
    M = np.maximum(m1, m2)
    M = np.where(np.isneginf(M), 0.0, M)
    w1 = np.where(np.isneginf(m1), 0.0, np.exp(np.where(np.isneginf(m1), 0.0, m1 - M))) * l1
    w2 = np.where(np.isneginf(m2), 0.0, np.exp(np.where(np.isneginf(m2), 0.0, m2 - M))) * l2
    tot = w1 + w2
    return np.where(tot > 0, w1 / np.where(tot > 0, tot, 1.0), 0.0)


def query_drift(q, q_ref):
    """1 - cos(q, q_ref) per row, q and q_ref [b, B, Hq, d] -> [b, Hq, B],
    as |q/|q| - r/|r||^2 / 2; 0 where either vector is zero."""
    q = np.asarray(q, dtype=np.float64)
    q_ref = np.asarray(q_ref, dtype=np.float64)
    nq = np.sqrt(np.einsum("bthd,bthd->bth", q, q))[..., None]
    nr = np.sqrt(np.einsum("bthd,bthd->bth", q_ref, q_ref))[..., None]
    ok = (nq > 0) & (nr > 0)
    diff = np.where(ok, q / np.where(nq > 0, nq, 1.0) - q_ref / np.where(nr > 0, nr, 1.0), 0.0)
    return np.transpose(0.5 * np.einsum("bthd,bthd->bth", diff, diff), (0, 2, 1))


def drift_statistic(pfx_state, blk_state, q_next, q_ref):
    """delta = max over rows of prefix_share * (1 - cos(q_next, q_ref))."""
    return float(np.max(prefix_share(pfx_state, blk_state) * query_drift(q_next, q_ref)))


def adaptive_schedule(layers, theta, forced=None):
    """Every step of one block for several layers with drift-triggered refresh.

    layers: list over layers of dicts with keys steps (list of (q, k_blk,
    v_blk)), k_pfx, v_pfx, lens, n_kv_heads, tau, base. All layers have the
    same number of steps.
    forced: optional [steps, layers] 0/1 array of refresh decisions to follow
    instead of the rule (so that a run whose fp32 statistics decided the
    refreshes can be reproduced exactly); the statistics are still computed.

    Returns (outs, drift, refreshed): outs[l][s] = (O, lse), drift [steps,
    layers] (delta_s; the last step's row is 0: it decides nothing),
    refreshed [steps, layers] (1 where the layer recomputed its state at that
    step).
    """
    n = len(layers)
    S = len(layers[0]["steps"])
    outs = [[None] * S for _ in range(n)]
    drift = np.zeros((S, n))
    refreshed = np.zeros((S, n), dtype=np.int64)
    state = [None] * n
    q_ref = [None] * n
    want = np.ones(n, dtype=bool)  # step 0 computes every layer's state
    for s in range(S):
        nxt = np.zeros(n, dtype=bool)
        for li, L in enumerate(layers):
            q, k, v = L["steps"][s]
            do = bool(forced[s, li]) if forced is not None else bool(want[li])
            if s == 0 and not do:
                raise ValueError("step 0 must compute every layer's state")
            if do:
                state[li] = orc.prefix_partial(q, L["k_pfx"], L["v_pfx"], L["lens"], L["n_kv_heads"],
                                               L["tau"], L["base"])
                q_ref[li] = np.asarray(q, dtype=np.float64)
                refreshed[s, li] = 1
            blk = orc.block_partial(q, k, v, L["lens"], L["n_kv_heads"], L["tau"], L["base"])
            outs[li][s] = orc.finalize(orc.merge(state[li], blk))
            if s + 1 < S:  # the decision about the next step, from its queries
                drift[s, li] = drift_statistic(state[li], blk, L["steps"][s + 1][0], q_ref[li])
                if drift[s, li] > theta:
                    nxt[li:] = True  # this layer and every deeper one
        want = nxt
    return outs, drift, refreshed


def refresh_pattern(drift, theta):
    """The refresh decisions the rule takes from given statistics: step 0
    refreshes every layer; layer l refreshes at s + 1 when some layer l' <= l
    had drift > theta at step s."""
    drift = np.asarray(drift, dtype=np.float64)
    S, n = drift.shape
    pat = np.zeros((S, n), dtype=np.int64)
    pat[0, :] = 1
    for s in range(S - 1):
        over = drift[s] > theta
        pat[s + 1] = np.maximum.accumulate(over).astype(np.int64)
    return pat
