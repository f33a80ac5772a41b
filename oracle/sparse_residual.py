"""CPU oracle for sparse block-external attention with a cached residual.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) may import this
module. It shares no code with the CUDA library and imports nothing from the
``cached_block_attention_b200`` package.

What is computed. FlashBlock ("Attention Caching for Efficient Long-Context
Block Diffusion", Abstract) notes that its cached block-external attention can
be combined with sparse attention as a complementary residual reuse. The
pages give the idea only; this module fixes one plain reading of it:

* page selection: the prefix of sequence b is cut into pages of P tokens
  (the last one may be partial). A page's score is the largest
  tau * <RoPE(q_t, L_b + t), kbar> over the block's rows t and the query heads,
  where kbar is the mean of the page's keys of the query head's kv-head. The
  k pages with the highest scores are kept (ties to the lower page index),
  the same pages for every head of the sequence (k >= 1);
* at a dense step s0 the block-external attention is computed twice, over
  all prefix keys (dense) and over the kept pages (sparse), both as normalised
  outputs with their logsumexp. The residual is their difference,
  R_O = O_dense - O_sparse and R_lse = lse_dense - lse_sparse, per row;
* at a later step s the block-external part is the sparse attention of step
  s's queries over the same pages, plus the cached residual:
  O_ext = O_sparse(s) + R_O, lse_ext = lse_sparse(s) + R_lse. It is merged
  with the fresh in-block attention by logsumexp, as the exact path merges
  the prefix state.

At s = s0, or with every page kept, the result is the exact attention of
that step (dense prefix). The residual is in normalised-output space because
states with different maxima cannot be subtracted. A sequence with no prefix
has no block-external part: its rows are plain in-block attention.
"""
from __future__ import annotations

import numpy as np

from oracle.fbk_oracle import block_partial, finalize, kv_head_of, merge, rope, softmax_partial

__all__ = ["page_scores", "select_pages", "sparse_prefix_partial", "external_output", "residual",
           "approx_step_output"]


def page_scores(q, k_pfx, lens, n_kv_heads, tau, base, page):
    """Score of every page of every sequence: a list over b of arrays [n_pages]."""
    q = np.asarray(q, dtype=np.float64)
    b, B, Hq, d = q.shape
    out = []
    for bi in range(b):
        L = int(lens[bi])
        n_pages = (L + page - 1) // page
        pos = L + np.arange(B)
        sc = np.full(n_pages, -np.inf)
        for h in range(Hq):
            g = kv_head_of(h, Hq, n_kv_heads)
            qh = rope(q[bi, :, h, :], pos, base)
            for p in range(n_pages):
                kbar = np.asarray(k_pfx[bi][g, p * page:min(L, (p + 1) * page)], dtype=np.float64).mean(axis=0)
                sc[p] = max(sc[p], float((tau * (qh @ kbar)).max()))
        out.append(sc)
    return out


def select_pages(scores, k_pages):
    """The k highest-scoring pages of each sequence (ties to the lower index),
    in increasing page order."""
    sel = []
    for sc in scores:
        order = sorted(range(len(sc)), key=lambda p: (-sc[p], p))
        sel.append(np.array(sorted(order[:k_pages]), dtype=np.int64))
    return sel


def _keep_keys(k_pfx, v_pfx, lens, pages, page):
    """Per sequence, the keys and values of the kept pages (in page order)."""
    kk, vv, ll = [], [], []
    for bi in range(len(lens)):
        L = int(lens[bi])
        idx = np.concatenate([np.arange(p * page, min(L, (p + 1) * page)) for p in pages[bi]]) \
            if len(pages[bi]) else np.zeros(0, dtype=np.int64)
        kk.append(np.asarray(k_pfx[bi])[:, idx])
        vv.append(np.asarray(v_pfx[bi])[:, idx])
        ll.append(len(idx))
    return kk, vv, np.array(ll)


def sparse_prefix_partial(q, k_pfx, v_pfx, lens, pages, page, n_kv_heads, tau, base):
    """State of the block's rows over the kept pages' keys only. The rows are
    rotated at their true positions L_b + t (prefix keys are stored rotated)."""
    kk, vv, _ = _keep_keys(k_pfx, v_pfx, lens, pages, page)
    q = np.asarray(q, dtype=np.float64)
    b, B, Hq, d = q.shape
    o = np.zeros((b, Hq, B, d))
    m = np.full((b, Hq, B), -np.inf)
    l = np.zeros((b, Hq, B))
    for bi in range(b):
        pos = int(lens[bi]) + np.arange(B)
        for h in range(Hq):
            g = kv_head_of(h, Hq, n_kv_heads)
            qh = rope(q[bi, :, h, :], pos, base)
            o[bi, h], m[bi, h], l[bi, h] = softmax_partial(tau * (qh @ kk[bi][g].T), vv[bi][g])
    return o, m, l


def external_output(state):
    """Normalised block-external output O~/l [b, Hq, B, d] and its logsumexp."""
    o, m, l = state
    return o / l[..., None], m + np.log(l)


def residual(dense_state, sparse_state):
    """(R_O, R_lse, empty) = dense minus sparse, in normalised-output space;
    `empty` marks rows whose prefix has no keys (no block-external part)."""
    empty = np.isneginf(np.asarray(dense_state[1]))
    with np.errstate(invalid="ignore", divide="ignore"):
        od, ld = external_output(dense_state)
        os_, ls = external_output(sparse_state)
        return np.where(empty[..., None], 0.0, od - os_), np.where(empty, 0.0, ld - ls), empty


def approx_step_output(q, k_blk, v_blk, k_pfx, v_pfx, lens, pages, page, res, n_kv_heads, tau, base):
    """One step: sparse block-external attention plus the cached residual,
    merged with the fresh in-block attention. Returns (O [b, B, Hq, d], lse)."""
    sp = sparse_prefix_partial(q, k_pfx, v_pfx, lens, pages, page, n_kv_heads, tau, base)
    r_o, r_lse, empty = res
    with np.errstate(invalid="ignore", divide="ignore"):
        o_s, lse_s = external_output(sp)
        # as a state relative to m = lse_ext: O~ = O_ext, l = 1 (empty rows: no external part)
        ext_state = (np.where(empty[..., None], 0.0, o_s + r_o), np.where(empty, -np.inf, lse_s + r_lse),
                     np.where(empty, 0.0, 1.0))
    blk = block_partial(q, k_blk, v_blk, lens, n_kv_heads, tau, base)
    return finalize(merge(ext_state, blk))
