"""GPU parity of a whole FACache step over a sequence (LaCache §3.3.1-§3.3.3,
App. J), composed from the library's calls:
  * U's cached state over U's keys: fbk_prefix_partial_at over chunks of U's
    rows (pre-RoPE queries at their own positions; no chunk crosses the block);
  * U's rows at a step: fbk_facache_unchanged_rows with that state;
  * the block's rows: fbk_prefix_partial_at (keys = U, including the masked
    suffix; queries at c0 + t), then fbk_block_attn_merge.
Checked against the oracle (oracle/facache.py), which is pinned to plain
full-sequence attention.

Runs only on a machine with a CUDA GPU and the built library (marker `gpu`).
"""
import math

import numpy as np
import pytest
import torch

from cached_block_attention_b200 import synth
from oracle import facache as fc
from oracle import fbk_oracle as orc
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import fbk  # noqa: F401  (fails loudly if not built)
    yield


def bf16(x):
    return synth.bf16_bits(np.asarray(x, dtype=np.float64))


def make_sequence(b, hq, hkv, d, blk, n, c0s, base, seed):
    """Raw bf16 Q/K/V of every position, plus U's K after RoPE (bf16, what
    RoPECache keeps) in U's row order."""
    r = np.random.Generator(np.random.PCG64(seed))
    sc = 1.0 / math.sqrt(d)
    q = bf16(r.standard_normal((b, n, hq, d)) * sc)
    k = bf16(r.standard_normal((b, n, hkv, d)) * sc)
    v = bf16(r.standard_normal((b, n, hkv, d)) * sc)
    nu = n - blk
    up = [fc.u_positions(nu, c0s[bi], blk) for bi in range(b)]
    cp = [c0s[bi] + np.arange(blk) for bi in range(b)]
    f = orc.bits_to_f64
    ku_rot = np.stack([bf16(orc.rope(f(k[bi, up[bi]]), up[bi][:, None], base)) for bi in range(b)])
    qu_rot = np.stack([bf16(orc.rope(f(q[bi, up[bi]]), up[bi][:, None], base)) for bi in range(b)])
    seq = dict(q=q, k=k, v=v, up=up, cp=cp, ku_rot=ku_rot, qu_rot=qu_rot,
               qu_raw=np.stack([q[bi, up[bi]] for bi in range(b)]),
               vu=np.stack([v[bi, up[bi]] for bi in range(b)]),
               qc=np.stack([q[bi, cp[bi]] for bi in range(b)]),
               kc=np.stack([k[bi, cp[bi]] for bi in range(b)]),
               vc=np.stack([v[bi, cp[bi]] for bi in range(b)]))
    return seq


def u_cache(seq, hkv, d):
    """U's K (after RoPE) and V as a contiguous cache [b, Hkv, U, d], lengths U."""
    from cached_block_attention_b200 import fbk
    b, nu = seq["ku_rot"].shape[:2]
    kc = np.ascontiguousarray(np.transpose(seq["ku_rot"], (0, 2, 1, 3)))
    vc = np.ascontiguousarray(np.transpose(seq["vu"], (0, 2, 1, 3)))
    lens = torch.full((b,), nu, dtype=torch.int32, device="cuda")
    return fbk.KVCache(H.dev_bf16(kc), H.dev_bf16(vc), lens, None, torch.zeros(1, dtype=torch.int32, device="cuda"))


def state_by_chunks(seq, hq, hkv, d, blk, c0s, tau, base):
    """U's state over U's keys, chunk by chunk through fbk_prefix_partial_at."""
    from cached_block_attention_b200 import fbk
    b, nu = seq["qu_raw"].shape[:2]
    G = hq // hkv
    cmax = min(256 // G, 256)
    o = torch.empty(b, hq, nu, d, dtype=torch.float32, device="cuda")
    m = torch.empty(b, hq, nu, dtype=torch.float32, device="cuda")
    l = torch.empty(b, hq, nu, dtype=torch.float32, device="cuda")
    cache = u_cache(seq, hkv, d)
    ws = torch.empty(fbk.prefix_workspace_bytes(fbk.Shape(1, hq, hkv, d, cmax, tau, base), None, 0),
                     dtype=torch.uint8, device="cuda")
    for bi in range(b):
        one = fbk.KVCache(cache.k[bi:bi + 1], cache.v[bi:bi + 1], cache.prefix_lens[bi:bi + 1], None,
                          cache.error_flags)
        for lo, hi in ((0, c0s[bi]), (c0s[bi], nu)):      # rows before and after the block
            for i0 in range(lo, hi, cmax):
                rows = min(cmax, hi - i0)
                pos0 = i0 if i0 < c0s[bi] else i0 + blk
                shape = fbk.Shape(1, hq, hkv, d, rows, tau, base)
                part = fbk.Partial.empty(shape)
                qd = H.dev_bf16(np.ascontiguousarray(seq["qu_raw"][bi:bi + 1, i0:i0 + rows]))
                pos = torch.tensor([pos0], dtype=torch.int32, device="cuda")
                fbk.prefix_partial_at(shape, qd, pos, one, part, ws)
                o[bi, :, i0:i0 + rows] = part.o_unnorm[0]
                m[bi, :, i0:i0 + rows] = part.m[0]
                l[bi, :, i0:i0 + rows] = part.l[0]
    torch.cuda.synchronize()
    assert int(cache.error_flags.item()) == 0
    return fbk.Partial(o, m, l)


# (b, hq, hkv, d, blk, n, c0 per sequence, base, tau)
CASES = [
    (1, 4, 4, 128, 32, 300, (100,), 1e4, 1.0),
    (2, 8, 2, 128, 32, 261, (0, 229), 1e4, 1.0),              # block first; block last
    (1, 28, 4, 128, 32, 400, (150,), 1e6, 1 / math.sqrt(128)),
    (1, 4, 2, 64, 16, 333, (77,), 1e4, 1.0),
]


@pytest.mark.parametrize("cfg", CASES)
def test_uu_state_by_chunks(cfg):
    b, hq, hkv, d, blk, n, c0s, base, tau = cfg
    seq = make_sequence(b, hq, hkv, d, blk, n, c0s, base, seed=CASES.index(cfg))
    st = state_by_chunks(seq, hq, hkv, d, blk, list(c0s), tau, base)
    f = orc.bits_to_f64
    for bi in range(b):
        pos = seq["up"][bi][None, :, None]
        ref = fc.uu_state(orc.rope(f(seq["qu_raw"][bi:bi + 1]), pos, base), f(seq["ku_rot"][bi:bi + 1]),
                          f(seq["vu"][bi:bi + 1]), hkv, tau)
        got = tuple(H.host_f64(x[bi:bi + 1]) for x in (st.o_unnorm, st.m, st.l))
        H.check_partial(got, ref, "bf16", f"U state, sequence {bi}")


@pytest.mark.parametrize("cfg", CASES)
def test_full_step_equals_full_sequence_attention(cfg):
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, n, c0s, base, tau = cfg
    seq = make_sequence(b, hq, hkv, d, blk, n, c0s, base, seed=100 + CASES.index(cfg))
    st = state_by_chunks(seq, hq, hkv, d, blk, list(c0s), tau, base)
    nu = n - blk
    shape = fbk.Shape(b, hq, hkv, d, blk, tau, base)
    pos = torch.tensor(list(c0s), dtype=torch.int32, device="cuda")
    kc, vc, qc = H.dev_bf16(seq["kc"]), H.dev_bf16(seq["vc"]), H.dev_bf16(seq["qc"])
    # U's rows
    out_u = torch.empty(b, nu, hq, d, dtype=torch.bfloat16, device="cuda")
    fbk.facache_unchanged_rows(shape, H.dev_bf16(seq["qu_rot"]), st, kc, vc, pos, out_u)
    # the block's rows: their state over U's keys, then the step kernel
    cache = u_cache(seq, hkv, d)
    pfx = fbk.Partial.empty(shape)
    ws = torch.empty(fbk.prefix_workspace_bytes(shape, cache, 0), dtype=torch.uint8, device="cuda")
    fbk.prefix_partial_at(shape, qc, pos, cache, pfx, ws)
    out_c = torch.empty(b, blk, hq, d, dtype=torch.bfloat16, device="cuda")
    fbk.block_attn_merge(shape, qc, kc, vc, pos, pfx, out_c)
    torch.cuda.synchronize()
    f = orc.bits_to_f64
    for bi in range(b):
        pos_all = np.arange(n)[None, :, None]
        ref, _ = fc.full_sequence_attention(orc.rope(f(seq["q"][bi:bi + 1]), pos_all, base),
                                            orc.rope(f(seq["k"][bi:bi + 1]), pos_all, base),
                                            f(seq["v"][bi:bi + 1]), hkv, tau)
        H.assert_close(H.host_f64(out_u[bi:bi + 1]), ref[:, seq["up"][bi]], "bf16", f"U rows, sequence {bi}")
        H.assert_close(H.host_f64(out_c[bi:bi + 1]), ref[:, seq["cp"][bi]], "bf16", f"block rows, sequence {bi}")


@pytest.mark.parametrize("cfg", CASES)
def test_refresh_and_step_entry_points(cfg):
    """The same step through fbk_facache_refresh and fbk_facache_step: the state
    equals the chunk-by-chunk composition's, and both halves of the output equal
    full-sequence attention."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, n, c0s, base, tau = cfg
    seq = make_sequence(b, hq, hkv, d, blk, n, c0s, base, seed=200 + CASES.index(cfg))
    nu = n - blk
    shape = fbk.Shape(b, hq, hkv, d, blk, tau, base)
    cache = u_cache(seq, hkv, d)
    ws = torch.empty(fbk.facache_workspace_bytes(shape, nu, 0), dtype=torch.uint8, device="cuda")
    st = fbk.Partial(torch.empty(b, hq, nu, d, device="cuda"), torch.empty(b, hq, nu, device="cuda"),
                     torch.empty(b, hq, nu, device="cuda"))
    fbk.facache_refresh(shape, H.dev_bf16(seq["qu_raw"]), list(c0s), cache, st, ws)
    ref_st = state_by_chunks(seq, hq, hkv, d, blk, list(c0s), tau, base)
    for x, y in ((st.o_unnorm, ref_st.o_unnorm), (st.m, ref_st.m), (st.l, ref_st.l)):
        assert torch.equal(x, y)
    pos = torch.tensor(list(c0s), dtype=torch.int32, device="cuda")
    out_u = torch.empty(b, nu, hq, d, dtype=torch.bfloat16, device="cuda")
    out_c = torch.empty(b, blk, hq, d, dtype=torch.bfloat16, device="cuda")
    fbk.facache_step(shape, H.dev_bf16(seq["qu_rot"]), st, H.dev_bf16(seq["qc"]), H.dev_bf16(seq["kc"]),
                     H.dev_bf16(seq["vc"]), pos, cache, out_u, out_c, ws)
    torch.cuda.synchronize()
    f = orc.bits_to_f64
    for bi in range(b):
        pos_all = np.arange(n)[None, :, None]
        ref, _ = fc.full_sequence_attention(orc.rope(f(seq["q"][bi:bi + 1]), pos_all, base),
                                            orc.rope(f(seq["k"][bi:bi + 1]), pos_all, base),
                                            f(seq["v"][bi:bi + 1]), hkv, tau)
        H.assert_close(H.host_f64(out_u[bi:bi + 1]), ref[:, seq["up"][bi]], "bf16", f"U rows, sequence {bi}")
        H.assert_close(H.host_f64(out_c[bi:bi + 1]), ref[:, seq["cp"][bi]], "bf16", f"block rows, sequence {bi}")
