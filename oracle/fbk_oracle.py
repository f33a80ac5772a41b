"""fp64 CPU oracle for cached block attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) may import this
module. It shares no code with the CUDA library, imports nothing from the
``cached_block_attention_b200`` package, and is slow and plain on purpose: each
function is the definition it names, written out with numpy in fp64.

What is computed (one attention layer of one denoising step of block diffusion
decoding):

* the current block of B query tokens of sequence b sits at absolute positions
  L_b .. L_b+B-1 after a cached prefix of L_b tokens (LaCache, "Exact Caching and
  Precision-Adaptive Inference for Diffusion Large Language Models", §3.3.1
  Notation and App. B.1 semi-autoregressive decoding);
* its queries attend bidirectionally to the cached prefix keys and to the block's
  own keys, with no mask inside the block (FlashBlock, "Attention Caching for
  Efficient Long-Context Block Diffusion", Abstract: block-internal attention);
* the prefix contribution is the FlashAttention online-softmax state (m, l, O~)
  restricted to the prefix keys (LaCache §3.3.3 FACache, Eq. 2-6), and the final
  output is the row-normalised merge O = O~ / l with logsumexp m + log l
  (LaCache App. J, the FACache pseudocode, final normalisation and LSE);
* RoPE is applied to block Q and K at their absolute positions, while prefix K
  in the cache is stored already rotated (LaCache §3.3.2 RoPECache, Eq. 1).

Readings taken where the pages are silent:
  * scores are ``tau * <RoPE(q), k>`` with tau an explicit argument (the pages
    write S = Q K^T, i.e. tau = 1);
  * RoPE is the rotate-half form: pairs (i, i + d/2), theta_i = base^(-2i/d),
    positions 0-based;
  * the GQA head map is kv_head = floor(h * Hkv / Hq);
  * an empty key set gives the state (O~ = 0, l = 0, m = -inf).

Layouts (same as the device buffers, fp64 here):
  q [b, B, Hq, d] (pre-RoPE), k_blk / v_blk [b, B, Hkv, d] (pre-RoPE K),
  prefix K / V: list over b of [Hkv, L_b, d] (K post-RoPE),
  partial: O~ [b, Hq, B, d], m [b, Hq, B], l [b, Hq, B],
  output O [b, B, Hq, d], lse [b, Hq, B].
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "kv_head_of", "rope_freqs", "rope", "softmax_partial", "online_partial",
    "merge", "finalize", "prefix_partial", "block_partial", "full_attention",
    "step_output", "block_schedule", "refresh_schedule", "bf16_rne_bits", "bits_to_f64",
    "commit_contiguous", "commit_paged", "gather_paged",
]


# ------------------------------------------------------------------ basics

def kv_head_of(h: int, n_q_heads: int, n_kv_heads: int) -> int:
    """Query head h reads kv-head floor(h * Hkv / Hq): contiguous groups (GQA)."""
    return (h * n_kv_heads) // n_q_heads


def rope_freqs(d: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d), i = 0 .. d/2-1 (RoFormer rotary embedding)."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def rope(x, pos, base: float) -> np.ndarray:
    """Rotate pairs (x_i, x_{i+d/2}) by angle pos * theta_i (LaCache §3.3.2, Eq. 1).

    x: [..., d]; pos: broadcastable to x.shape[:-1]. All in fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_freqs(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) to their exact fp64 values."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_rne_bits(x) -> np.ndarray:
    """Round fp64 values straight to bf16 (8 significant bits), ties to even.

    |x| in [2^(e-1), 2^e) has bf16 spacing 2^(e-8); below the normal range the
    spacing stays 2^-133. rint() rounds half to even, and every step is exact in
    fp64, so this is a single rounding from fp64 (no fp32 detour).
    """
    x = np.asarray(x, dtype=np.float64)
    assert np.all(np.isfinite(x))
    _, e = np.frexp(x)
    q = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(x, -q)), q)
    return (np.ascontiguousarray(y.astype(np.float32)).view(np.uint32) >> 16).astype(np.uint16)


# ------------------------------------------------------------------ softmax state

def softmax_partial(scores, v):
    """Online-softmax state of one row block over one key set, two-pass form.

    scores [R, N], v [N, d] -> (O~ [R, d], m [R], l [R]) with m = rowmax(scores),
    l = rowsum(exp(scores - m)), O~ = exp(scores - m) @ v: the state that the
    recurrence of LaCache §3.3.3 (Eq. 2-6) holds after streaming all N keys.
    N = 0 gives (0, -inf, 0).
    """
    scores = np.asarray(scores, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    R, N = scores.shape
    d = v.shape[1]
    if N == 0:
        return np.zeros((R, d)), np.full(R, -np.inf), np.zeros(R)
    m = scores.max(axis=1)
    p = np.exp(scores - m[:, None])
    return p @ v, m, p.sum(axis=1)


def online_partial(scores, v, tile: int):
    """The FlashAttention recurrence of LaCache §3.3.3, Eq. 2-6, over key tiles.

    Starts from (m, l, O~) = (-inf, 0, 0) and, for each tile j of `tile` keys:
      m_j = max(m_{j-1}, rowmax S_j)          (Eq. 2)
      alpha_j = exp(m_{j-1} - m_j)            (Eq. 3)
      P_j = exp(S_j - m_j)                    (Eq. 4)
      l_j = alpha_j * l_{j-1} + rowsum P_j    (Eq. 5)
      O_j = alpha_j * O_{j-1} + P_j V_j       (Eq. 6)
    """
    scores = np.asarray(scores, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    R, N = scores.shape
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    o = np.zeros((R, v.shape[1]))
    for j0 in range(0, N, tile):
        s = scores[:, j0:j0 + tile]
        m_new = np.maximum(m, s.max(axis=1))
        alpha = np.exp(m - m_new)
        p = np.exp(s - m_new[:, None])
        l = alpha * l + p.sum(axis=1)
        o = alpha[:, None] * o + p @ v[j0:j0 + tile]
        m = m_new
    return o, m, l


def merge(a, b):
    """Combine two states over disjoint key sets (LSE merge).

    Initialising the recurrence of Eq. 2-6 with a cached state and streaming
    the remaining keys (LaCache App. J, FACache pseudocode: initialise with
    cache) is, by associativity, this merge: m = max(m_a, m_b),
    l = e^(m_a-m) l_a + e^(m_b-m) l_b, O~ = e^(m_a-m) O~_a + e^(m_b-m) O~_b.
    An empty side (m = -inf) contributes nothing.
    """
    oa, ma, la = (np.asarray(t, dtype=np.float64) for t in a)
    ob, mb, lb = (np.asarray(t, dtype=np.float64) for t in b)
    m = np.maximum(ma, mb)
    m_ref = np.where(np.isneginf(m), 0.0, m)
    fa = np.where(np.isneginf(ma), 0.0, np.exp(np.where(np.isneginf(ma), 0.0, ma - m_ref)))
    fb = np.where(np.isneginf(mb), 0.0, np.exp(np.where(np.isneginf(mb), 0.0, mb - m_ref)))
    o = fa[..., None] * oa + fb[..., None] * ob
    return o, m, fa * la + fb * lb


def finalize(state):
    """O = diag(l)^-1 O~ and L = m + log l (LaCache App. J, final normalisation).

    state arrays are [b, Hq, B, d] / [b, Hq, B]; returns O [b, B, Hq, d] and
    lse [b, Hq, B].
    """
    o, m, l = state
    out = o / l[..., None]
    return np.transpose(out, (0, 2, 1, 3)).copy(), m + np.log(l)


# ------------------------------------------------------------------ per-layer ops

def _heads(Hq, heads):
    return range(Hq) if heads is None else heads


def _batches(b, batches):
    return range(b) if batches is None else batches


def prefix_partial(q, k_pfx, v_pfx, lens, n_kv_heads, tau, base, heads=None, batches=None):
    """State (O~, m, l) of the block queries over the cached prefix keys only.

    This is FACache's cached state (LaCache §3.3.3) for the block's own query
    rows, the "block-external attention" that FlashBlock caches and reuses
    across the denoising steps of a block (FlashBlock, Abstract).
    Rows not in heads/batches are left as the empty state.
    """
    q = np.asarray(q, dtype=np.float64)
    b, B, Hq, d = q.shape
    o = np.zeros((b, Hq, B, d))
    m = np.full((b, Hq, B), -np.inf)
    l = np.zeros((b, Hq, B))
    for bi in _batches(b, batches):
        L = int(lens[bi])
        pos = L + np.arange(B)
        for h in _heads(Hq, heads):
            g = kv_head_of(h, Hq, n_kv_heads)
            qh = rope(q[bi, :, h, :], pos, base)
            kk = np.asarray(k_pfx[bi][g, :L], dtype=np.float64)
            vv = np.asarray(v_pfx[bi][g, :L], dtype=np.float64)
            o[bi, h], m[bi, h], l[bi, h] = softmax_partial(tau * (qh @ kk.T), vv)
    return o, m, l


def block_partial(q, k_blk, v_blk, lens, n_kv_heads, tau, base, heads=None, batches=None):
    """State of the block queries over the block's own keys (bidirectional, no mask).

    Both Q and K of the block are rotated at positions L_b + t (LaCache §3.3.2).
    """
    q = np.asarray(q, dtype=np.float64)
    k_blk = np.asarray(k_blk, dtype=np.float64)
    v_blk = np.asarray(v_blk, dtype=np.float64)
    b, B, Hq, d = q.shape
    o = np.zeros((b, Hq, B, d))
    m = np.full((b, Hq, B), -np.inf)
    l = np.zeros((b, Hq, B))
    for bi in _batches(b, batches):
        pos = int(lens[bi]) + np.arange(B)
        for h in _heads(Hq, heads):
            g = kv_head_of(h, Hq, n_kv_heads)
            qh = rope(q[bi, :, h, :], pos, base)
            kh = rope(k_blk[bi, :, g, :], pos, base)
            o[bi, h], m[bi, h], l[bi, h] = softmax_partial(tau * (qh @ kh.T), v_blk[bi, :, g, :])
    return o, m, l


def full_attention(q, k_blk, v_blk, k_pfx, v_pfx, lens, n_kv_heads, tau, base,
                   heads=None, batches=None):
    """Uncached softmax attention of the block queries over [prefix ; block] keys.

    The plain definition, two-pass in fp64, sharing no step with the partial
    and merge functions: keys = [cached prefix rows 0..L_b-1 ; RoPE(k_blk)],
    O = softmax(tau * q^ K^T) V. This is what FACache claims to reproduce
    exactly (LaCache §3.1: mathematically equivalent output).
    Returns O [b, B, Hq, d] and lse [b, Hq, B]; unselected rows are NaN.
    """
    q = np.asarray(q, dtype=np.float64)
    k_blk = np.asarray(k_blk, dtype=np.float64)
    v_blk = np.asarray(v_blk, dtype=np.float64)
    b, B, Hq, d = q.shape
    out = np.full((b, B, Hq, d), np.nan)
    lse = np.full((b, Hq, B), np.nan)
    for bi in _batches(b, batches):
        L = int(lens[bi])
        pos = L + np.arange(B)
        for h in _heads(Hq, heads):
            g = kv_head_of(h, Hq, n_kv_heads)
            qh = rope(q[bi, :, h, :], pos, base)
            keys = np.concatenate([np.asarray(k_pfx[bi][g, :L], dtype=np.float64),
                                   rope(k_blk[bi, :, g, :], pos, base)], axis=0)
            vals = np.concatenate([np.asarray(v_pfx[bi][g, :L], dtype=np.float64),
                                   v_blk[bi, :, g, :]], axis=0)
            s = tau * (qh @ keys.T)
            mx = s.max(axis=1)
            p = np.exp(s - mx[:, None])
            den = p.sum(axis=1)
            out[bi, :, h, :] = (p @ vals) / den[:, None]
            lse[bi, h] = mx + np.log(den)
    return out, lse


def step_output(pfx_state, q, k_blk, v_blk, lens, n_kv_heads, tau, base, heads=None, batches=None):
    """One cached denoising step: merge(cached prefix state, fresh block state), normalised."""
    blk = block_partial(q, k_blk, v_blk, lens, n_kv_heads, tau, base, heads, batches)
    return finalize(merge(pfx_state, blk))


def block_schedule(steps, k_pfx, v_pfx, lens, n_kv_heads, tau, base, heads=None, batches=None):
    """The reuse schedule over one block: the prefix state is computed once, from
    the first step's block queries, and merged with a fresh block state at every
    step (FlashBlock, Abstract: cached block-external attention).

    steps: list of (q, k_blk, v_blk). Returns a list of (O, lse), one per step.
    """
    q0 = steps[0][0]
    pfx = prefix_partial(q0, k_pfx, v_pfx, lens, n_kv_heads, tau, base, heads, batches)
    return [step_output(pfx, q, k, v, lens, n_kv_heads, tau, base, heads, batches)
            for (q, k, v) in steps]


def refresh_schedule(steps, k_pfx, v_pfx, lens, n_kv_heads, tau, base, interval,
                     heads=None, batches=None):
    """The block schedule with a cache update interval r (LaCache App. C: the
    interval trades speed for accuracy when the cached state is reused across
    steps). Steps are numbered from 0 inside the block; at steps 0, r, 2r, ...
    the prefix state is computed afresh from that step's block queries, and the
    steps in between reuse the latest one.

    r = 1 recomputes at every step, so every step is exact full attention;
    r >= len(steps) is block_schedule. Returns a list of (O, lse), one per step.
    """
    if interval < 1:
        raise ValueError("refresh interval must be >= 1")
    outs, pfx = [], None
    for s, (q, k, v) in enumerate(steps):
        if s % interval == 0:
            pfx = prefix_partial(q, k_pfx, v_pfx, lens, n_kv_heads, tau, base, heads, batches)
        outs.append(step_output(pfx, q, k, v, lens, n_kv_heads, tau, base, heads, batches))
    return outs


# ------------------------------------------------------------------ commit

def commit_contiguous(k_cache_bits, v_cache_bits, k_blk, v_blk_bits, lens, base):
    """Append a finished block to a contiguous cache [b, Hkv, cap, d] (bf16 bits).

    RoPECache keeps post-RoPE K of unchanged tokens (LaCache §3.3.2, Eq. 1), so
    the finished block's K is rotated at positions L_b + t, rounded once to
    bf16 (nearest even), and stored at slots L_b .. L_b+B-1; V is stored as
    given. Returns new (k_cache, v_cache, lens + B).
    """
    kc = np.array(k_cache_bits, dtype=np.uint16, copy=True)
    vc = np.array(v_cache_bits, dtype=np.uint16, copy=True)
    k_blk = np.asarray(k_blk, dtype=np.float64)
    vb = np.asarray(v_blk_bits, dtype=np.uint16)
    b, B, Hkv, d = k_blk.shape
    new_lens = np.array(lens, dtype=np.int64, copy=True)
    for bi in range(b):
        L = int(lens[bi])
        pos = L + np.arange(B)
        for g in range(Hkv):
            kc[bi, g, L:L + B] = bf16_rne_bits(rope(k_blk[bi, :, g, :], pos, base))
            vc[bi, g, L:L + B] = vb[bi, :, g, :]
        new_lens[bi] = L + B
    return kc, vc, new_lens


def commit_paged(k_pages_bits, v_pages_bits, page_table, k_blk, v_blk_bits, lens, base):
    """Same append into a paged cache [P, Hkv, page, d]: token position p of
    sequence b lives in page page_table[b, p // page] at offset p % page."""
    kp = np.array(k_pages_bits, dtype=np.uint16, copy=True)
    vp = np.array(v_pages_bits, dtype=np.uint16, copy=True)
    k_blk = np.asarray(k_blk, dtype=np.float64)
    vb = np.asarray(v_blk_bits, dtype=np.uint16)
    b, B, Hkv, d = k_blk.shape
    ps = kp.shape[2]
    new_lens = np.array(lens, dtype=np.int64, copy=True)
    for bi in range(b):
        L = int(lens[bi])
        for t in range(B):
            p = L + t
            page = int(page_table[bi, p // ps])
            for g in range(Hkv):
                kp[page, g, p % ps] = bf16_rne_bits(rope(k_blk[bi, t, g, :], p, base))
                vp[page, g, p % ps] = vb[bi, t, g, :]
        new_lens[bi] = L + B
    return kp, vp, new_lens


def gather_paged(pages, page_table, lens):
    """Logical per-sequence view [Hkv, L_b, d] of a paged cache."""
    pages = np.asarray(pages)
    ps = pages.shape[2]
    out = []
    for bi in range(len(lens)):
        pos = np.arange(int(lens[bi]))
        rows = pages[np.asarray(page_table)[bi, pos // ps], :, pos % ps, :]  # [L, Hkv, d]
        out.append(np.transpose(rows, (1, 0, 2)))
    return out
