"""CPU oracle for LaCache's FACache over a full sequence (first-layer attention
of full-sequence semi-autoregressive decoding).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) may import this
module. It shares no code with the CUDA library and imports nothing from the
``cached_block_attention_b200`` package.

What is computed (LaCache, "Exact Caching and Precision-Adaptive Inference for
Diffusion Large Language Models"):

* the sequence has N tokens; the current block C is the B positions
  c0 .. c0+B-1, and U holds every other position: the prompt and the blocks
  before C, and the masked suffix after it (§3.3.1). Every row attends
  bidirectionally to all N keys;
* Q and K of the tokens in U are kept after RoPE, at their own positions
  (RoPECache, §3.3.2 Eq. 1), and so are their V; they do not change within
  the block. The block's Q, K and V change at every step and are given
  before RoPE, which is applied at c0 + t;
* FACache (§3.3.3, Eq. 2-6, and App. J): the online-softmax state (O~, m, l)
  of the query rows in U over the keys in U is computed once per block and
  kept; at every step a row in U starts from it and streams only the block's
  keys, and a row in C streams all keys. Every output equals full attention
  over the whole sequence (the method is exact).

Readings taken where the pages are silent:
  * scores are ``tau * <q, k>`` (the pages write S = Q K^T, i.e. tau = 1);
  * RoPE is the rotate-half form with positions 0-based, as in
    ``fbk_oracle.rope``; the GQA head map is kv_head = floor(h * Hkv / Hq);
  * the rows of U are stored in sequence order with the block removed: row i
    of U is position i for i < c0 and position i + B after it.

Layouts: q_u [b, U, Hq, d], k_u / v_u [b, U, Hkv, d] (q_u, k_u after RoPE);
q_c [b, B, Hq, d], k_c / v_c [b, B, Hkv, d] (q_c, k_c before RoPE);
states O~ [b, Hq, rows, d], m and l [b, Hq, rows]; outputs [b, rows, Hq, d].
"""
from __future__ import annotations

import numpy as np

from oracle.fbk_oracle import finalize, kv_head_of, merge, rope, softmax_partial

__all__ = ["u_positions", "uu_state", "facache_step", "full_sequence_attention", "assemble_sequence"]


def u_positions(n_u: int, c0: int, blk: int) -> np.ndarray:
    """Sequence positions of the rows of U: 0 .. c0-1, then c0+B .. N-1."""
    i = np.arange(n_u)
    return np.where(i < c0, i, i + blk)


def _state(q_rows, keys, vals, n_kv_heads, tau):
    """State of query rows [b, R, Hq, d] over keys / values [b, K, Hkv, d]."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    b, R, Hq, d = q_rows.shape
    o = np.zeros((b, Hq, R, d))
    m = np.full((b, Hq, R), -np.inf)
    l = np.zeros((b, Hq, R))
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, n_kv_heads)
            s = tau * (q_rows[bi, :, h, :] @ np.asarray(keys[bi, :, g, :], dtype=np.float64).T)
            o[bi, h], m[bi, h], l[bi, h] = softmax_partial(s, np.asarray(vals[bi, :, g, :], dtype=np.float64))
    return o, m, l


def uu_state(q_u, k_u, v_u, n_kv_heads, tau):
    """FACache's cached state: the rows of U over the keys of U (LaCache §3.3.3,
    the state after streaming the KV blocks fully inside U)."""
    return _state(q_u, k_u, v_u, n_kv_heads, tau)


def facache_step(state_uu, q_u, k_u, v_u, q_c, k_c, v_c, c0, n_kv_heads, tau, base):
    """One denoising step (LaCache §3.3.3 and App. J). Rows of U: the cached
    state merged with their state over the block's keys. Rows of C: the state
    over all keys (U's and the block's). Returns ((O_u, lse_u), (O_c, lse_c))."""
    blk = np.asarray(q_c).shape[1]
    pos_c = c0 + np.arange(blk)
    qc = rope(q_c, pos_c[None, :, None], base)
    kc = rope(k_c, pos_c[None, :, None], base)
    vc = np.asarray(v_c, dtype=np.float64)
    rows_u = merge(state_uu, _state(q_u, kc, vc, n_kv_heads, tau))
    rows_c = merge(_state(qc, k_u, v_u, n_kv_heads, tau), _state(qc, kc, vc, n_kv_heads, tau))
    return finalize(rows_u), finalize(rows_c)


def assemble_sequence(x_u, x_c_rot, c0):
    """The full sequence [b, N, H, d] from U's rows and the block's rows."""
    x_u = np.asarray(x_u, dtype=np.float64)
    return np.concatenate([x_u[:, :c0], np.asarray(x_c_rot, dtype=np.float64), x_u[:, c0:]], axis=1)


def full_sequence_attention(q, k, v, n_kv_heads, tau):
    """Plain bidirectional softmax attention of every row over every key:
    q [b, N, Hq, d], k / v [b, N, Hkv, d] (after RoPE) -> O [b, N, Hq, d],
    lse [b, Hq, N]. Two-pass max/exp/sum in fp64; no state, no merge."""
    q = np.asarray(q, dtype=np.float64)
    b, N, Hq, d = q.shape
    out = np.zeros((b, N, Hq, d))
    lse = np.zeros((b, Hq, N))
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, n_kv_heads)
            s = tau * (q[bi, :, h, :] @ np.asarray(k[bi, :, g, :], dtype=np.float64).T)
            mx = s.max(axis=1)
            p = np.exp(s - mx[:, None])
            den = p.sum(axis=1)
            out[bi, :, h, :] = (p @ np.asarray(v[bi, :, g, :], dtype=np.float64)) / den[:, None]
            lse[bi, h] = mx + np.log(den)
    return out, lse
