"""GPU parity of fbk_decode_block: every denoising step of a block for several
attention layers in one call, with a cache update interval per layer
(LaCache App. C), against the oracle's refresh schedule; bit for bit against
the same launches issued one entry point at a time; and as a CUDA graph.

Runs only on a machine with a CUDA GPU and the built library (marker `gpu`).
"""
import math

import numpy as np
import pytest
import torch

from oracle import fbk_oracle as orc
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import fbk  # noqa: F401  (fails loudly if not built)
    yield


def make_layers(cfg, intervals, steps, seed):
    """One uploaded Case per layer (own cache and inputs) and its LayerBlock."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, lens, ps, tau, base, mode = cfg
    cases, blocks = [], []
    for i, r in enumerate(intervals):
        c = H.make_case(b, hq, hkv, d, blk, lens, ps, tau, base=base, seed=seed + 37 * i, steps=steps,
                        mode=mode).upload()
        q = torch.stack([st[0] for st in c.dev["steps"]])
        k = torch.stack([st[1] for st in c.dev["steps"]])
        v = torch.stack([st[2] for st in c.dev["steps"]])
        out = torch.stack([c.out_tensor() for _ in range(steps)])
        lse = torch.empty(steps, b, hq, blk, dtype=torch.float32, device="cuda")
        cases.append(c)
        blocks.append(fbk.LayerBlock(q, k, v, c.dev["cache"], fbk.Partial.empty(c.shape), out, r, lse))
    return cases, blocks


def workspace(case):
    return case.workspace(0)


def check_commit(case, steps):
    """The layer's cache after the commit of its last step's K/V, bit for bit."""
    cache = case.dev["cache"]
    lens_after = cache.prefix_lens.cpu().numpy()
    np.testing.assert_array_equal(lens_after, case.lens + case.blk)
    kb = case.step_f64(steps - 1)[1]
    for b in range(case.batch):
        L = int(case.lens[b])
        pos = L + np.arange(case.blk)
        if case.page_size:
            pt = cache.page_table[b].cpu().numpy()
            rows_k = H.host_bits(cache.k[pt[pos // case.page_size], :, pos % case.page_size])
            rows_v = H.host_bits(cache.v[pt[pos // case.page_size], :, pos % case.page_size])
        else:
            rows_k = H.host_bits(cache.k[b, :, L:L + case.blk].transpose(0, 1))
            rows_v = H.host_bits(cache.v[b, :, L:L + case.blk].transpose(0, 1))
        np.testing.assert_array_equal(rows_k, orc.bf16_rne_bits(orc.rope(kb[b], pos[:, None], case.base)))
        np.testing.assert_array_equal(rows_v, case.steps_bits[steps - 1][2][b])
    assert int(cache.error_flags.item()) == 0


# (batch, hq, hkv, d, blk, lens, page_size, tau, base, mode), intervals per layer, steps
CASES = [
    ((2, 4, 4, 64, 16, (100, 37), 0, 1.0, 1e4, 0), (1, 2, 5), 5),                       # MHA, contiguous
    ((2, 8, 2, 128, 32, (300, 64), 16, 1 / math.sqrt(128), 1e6, 0), (3, 1), 4),         # GQA, 16-token pages
    ((3, 28, 4, 128, 32, (0, 129, 700), 0, 1.0, 1e4, 0), (2, 7), 3),                    # two M-tiles, empty prefix
    ((1, 4, 2, 128, 32, (200,), 0, 1.0, 1e4, 1), (2, 4), 3),                            # fp32 check mode
]


@pytest.mark.parametrize("cfg,intervals,steps", CASES)
def test_decode_block_matches_refresh_schedule(cfg, intervals, steps):
    """Every row of every step of every layer against the oracle's refresh
    schedule with that layer's interval, then each layer's commit."""
    from cached_block_attention_b200 import fbk
    cases, blocks = make_layers(cfg, intervals, steps, seed=CASES.index((cfg, intervals, steps)) * 1000)
    mode = "fp32" if cfg[-1] == 1 else "bf16"
    fbk.decode_block(cases[0].shape, blocks, workspace(cases[0]), commit=True)
    torch.cuda.synchronize()
    for li, (case, blk) in enumerate(zip(cases, blocks)):
        ref = orc.refresh_schedule([case.step_f64(s) for s in range(steps)], case.k_pfx(), case.v_pfx(),
                                   case.lens, case.hkv, case.tau, case.base, blk.refresh_interval)
        for s in range(steps):
            H.assert_close(H.host_f64(blk.out[s]), ref[s][0], mode, f"layer {li} step {s}")
            lse_tol = 2e-2 if mode == "bf16" else 1e-5
            assert np.abs(H.host_f64(blk.lse[s]) - ref[s][1]).max() <= lse_tol, f"layer {li} step {s} lse"
        check_commit(case, steps)


def test_decode_block_equals_single_calls():
    """The one-call loop issues exactly the launches of the single entry points
    (same kernels, same order, same pointers): outputs, lse, prefix states and
    caches agree bit for bit."""
    from cached_block_attention_b200 import fbk
    cfg, intervals, steps = (2, 8, 2, 128, 32, (300, 64), 16, 1.0, 1e4, 0), (3, 1, 2), 5
    ca, ba = make_layers(cfg, intervals, steps, seed=4242)
    cb, bb = make_layers(cfg, intervals, steps, seed=4242)
    ws_a, ws_b = workspace(ca[0]), workspace(cb[0])
    fbk.decode_block(ca[0].shape, ba, ws_a, commit=True)
    shape = cb[0].shape
    for s in range(steps):
        for L in bb:
            if s % L.refresh_interval == 0:
                fbk.prefix_partial(shape, L.q[s], L.cache, L.prefix, ws_b)
            fbk.block_attn_merge(shape, L.q[s], L.k[s], L.v[s], L.cache.prefix_lens, L.prefix, L.out[s], L.lse[s])
    for L in bb:
        fbk.commit_block_rope_append(shape, L.k[steps - 1], L.v[steps - 1], L.cache)
    torch.cuda.synchronize()
    for li, (a, b) in enumerate(zip(ba, bb)):
        assert torch.equal(a.out, b.out), f"layer {li} outputs"
        assert torch.equal(a.lse, b.lse), f"layer {li} lse"
        for x, y in ((a.prefix.o_unnorm, b.prefix.o_unnorm), (a.prefix.m, b.prefix.m), (a.prefix.l, b.prefix.l)):
            assert torch.equal(x, y), f"layer {li} prefix state"
        assert torch.equal(a.cache.k, b.cache.k) and torch.equal(a.cache.v, b.cache.v), f"layer {li} cache"
        assert torch.equal(a.cache.prefix_lens, b.cache.prefix_lens)


def test_decode_block_graph_replay_matches_eager():
    """A whole block for all layers captured as one CUDA graph and replayed
    (after resetting the lengths) reproduces the eager call bit for bit."""
    from cached_block_attention_b200 import fbk
    cfg, intervals, steps = (1, 8, 2, 128, 32, (513,), 0, 1.0, 1e4, 0), (1, 3, 4), 4
    cases, blocks = make_layers(cfg, intervals, steps, seed=777)
    ws = workspace(cases[0])
    lens0 = [L.cache.prefix_lens.clone() for L in blocks]
    fbk.decode_block(cases[0].shape, blocks, ws, commit=True)
    torch.cuda.synchronize()
    eager = [(L.out.clone(), L.lse.clone(), L.cache.k.clone()) for L in blocks]
    for L, l0 in zip(blocks, lens0):
        L.cache.prefix_lens.copy_(l0)
        L.out.zero_()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
            fbk.decode_block(cases[0].shape, blocks, ws, commit=True)
    torch.cuda.synchronize()
    for _ in range(2):
        for L, l0 in zip(blocks, lens0):
            L.cache.prefix_lens.copy_(l0)
        g.replay()
        torch.cuda.synchronize()
        for li, (L, (o, lse, k)) in enumerate(zip(blocks, eager)):
            assert torch.equal(L.out, o) and torch.equal(L.lse, lse), f"layer {li}"
            assert torch.equal(L.cache.k, k), f"layer {li} cache"
            assert torch.equal(L.cache.prefix_lens, lens0[li] + 32)
    del g


def test_decode_block_llada8b_layers():
    """Four LLaDA-8B-shaped layers (32 heads, d 128, prefix 4096, block 32),
    eight steps, intervals 1, 3, 8 and 5: every row of every step against the
    oracle, in the launch configuration the bench uses (one share per SM)."""
    from cached_block_attention_b200 import fbk
    cfg = (1, 32, 32, 128, 32, (4096,), 0, 1.0, 1e4, 0)
    intervals, steps = (1, 3, 8, 5), 8
    cases, blocks = make_layers(cfg, intervals, steps, seed=9000)
    fbk.decode_block(cases[0].shape, blocks, workspace(cases[0]), commit=True)
    torch.cuda.synchronize()
    for li, (case, blk) in enumerate(zip(cases, blocks)):
        ref = orc.refresh_schedule([case.step_f64(s) for s in range(steps)], case.k_pfx(), case.v_pfx(),
                                   case.lens, case.hkv, 1.0, case.base, blk.refresh_interval)
        for s in range(steps):
            H.assert_close(H.host_f64(blk.out[s]), ref[s][0], "bf16", f"layer {li} step {s}")
        check_commit(case, steps)


def test_decode_block_rejects_before_launch():
    """A bad second layer is refused with nothing enqueued: the first layer's
    outputs and lengths stay untouched."""
    from cached_block_attention_b200 import fbk
    cfg = (1, 4, 2, 64, 16, (50,), 0, 1.0, 1e4, 0)
    cases, blocks = make_layers(cfg, (1, 2), 2, seed=31)
    for L in blocks:
        L.out.fill_(7.0)
    blocks[1].refresh_interval = 0
    with pytest.raises(fbk.FbkError) as e:
        fbk.decode_block(cases[0].shape, blocks, workspace(cases[0]), commit=True)
    assert e.value.status == -1
    blocks[1].refresh_interval = 1
    blocks[1].cache.prefix_lens = blocks[0].cache.prefix_lens   # shared lengths with commit
    with pytest.raises(fbk.FbkError):
        fbk.decode_block(cases[0].shape, blocks, workspace(cases[0]), commit=True)
    torch.cuda.synchronize()
    assert bool((blocks[0].out == 7.0).all())
    assert blocks[0].cache.prefix_lens.tolist() == [50]
