"""GPU parity: every entry point of the C ABI against the fp64 oracle on the
same seeded inputs, element by element, at sizes that span several 64-key
tiles, both 128-row M-tiles and ragged tails, in both arithmetic modes.

Runs only on a machine with a CUDA GPU and the built library (marker `gpu`).
"""
import math

import numpy as np
import pytest
import torch

from oracle import fbk_oracle as orc
from tests import harness as H

pytestmark = pytest.mark.gpu

MODES = [(0, "bf16"), (1, "fp32")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import fbk  # noqa: F401  (fails loudly if not built)
    yield


def oracle_step(case, s, pfx_step=0):
    """Oracle output of step s with the prefix state from step pfx_step's queries."""
    qp = case.step_f64(pfx_step)[0]
    pfx = orc.prefix_partial(qp, case.k_pfx(), case.v_pfx(), case.lens, case.hkv, case.tau, case.base)
    q, k, v = case.step_f64(s)
    return orc.step_output(pfx, q, k, v, case.lens, case.hkv, case.tau, case.base)


def oracle_full(case, s):
    q, k, v = case.step_f64(s)
    return orc.full_attention(q, k, v, case.k_pfx(), case.v_pfx(), case.lens, case.hkv, case.tau, case.base)


# (batch, hq, hkv, d, blk, lens, page_size, tau)
SMALL_CASES = [
    (1, 2, 2, 64, 32, (256,), 0, 1.0),             # the tiny workload's shape
    (1, 4, 4, 128, 32, (1000,), 0, 1.0),           # ragged tail, d = 128
    (2, 28, 4, 128, 32, (300, 777), 0, 1.0),       # GQA G*B = 224: two M-tiles, padding rows
    (1, 32, 8, 128, 64, (517,), 0, 1 / math.sqrt(128)),   # G*B = 256, B = 64
    (3, 8, 2, 64, 16, (0, 65, 130), 0, 1.0),       # empty prefix in a batch, d = 64
    (2, 4, 2, 128, 8, (63, 64), 64, 1.0),          # paged, page = tile
    (2, 4, 2, 128, 32, (200, 100), 16, 1.0),       # paged, 16-token pages
    (2, 8, 8, 128, 32, (333, 129), 128, 1.0),      # paged, 128-token pages, MHA
    (1, 2, 1, 128, 1, (70,), 0, 1.0),              # B = 1 (single query row per head)
]


@pytest.mark.parametrize("mode,mname", MODES)
@pytest.mark.parametrize("cfg", SMALL_CASES)
def test_prefix_partial_matches_oracle(cfg, mode, mname):
    b, hq, hkv, d, blk, lens, ps, tau = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, ps, tau, seed=SMALL_CASES.index(cfg), mode=mode).upload()
    q = case.dev["steps"][0][0]
    got = H.partial_to_host(H.run_prefix(case, q))
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, hkv, tau, case.base)
    H.check_partial(got, ref, mname)
    assert int(case.dev["cache"].error_flags.item()) == 0


@pytest.mark.parametrize("mode,mname", MODES)
@pytest.mark.parametrize("cfg", SMALL_CASES)
def test_step_output_matches_full_attention(cfg, mode, mname):
    """Lossless: cached prefix state merged with the block state = uncached attention."""
    b, hq, hkv, d, blk, lens, ps, tau = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, ps, tau, seed=100 + SMALL_CASES.index(cfg), mode=mode).upload()
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    out, lse = H.run_step(case, pfx, 0)
    ref, ref_lse = oracle_full(case, 0)
    H.assert_close(H.host_f64(out), ref, mname, "O")
    assert np.abs(H.host_f64(lse) - ref_lse).max() <= (2e-2 if mode == 0 else 1e-5)
    # the uncached device reference agrees too
    fo, flse = H.run_full_ref(case, 0)
    H.assert_close(H.host_f64(fo), ref, mname, "full_ref O")
    assert np.abs(H.host_f64(flse) - ref_lse).max() <= (2e-2 if mode == 0 else 1e-5)


@pytest.mark.parametrize("mode,mname", MODES)
def test_reuse_schedule_over_steps(mode, mname):
    """Prefix state from step 0's queries, reused by later steps (new Q/K/V each)."""
    case = H.make_case(2, 8, 2, 128, 32, (450, 190), 0, 1.0, seed=11, steps=4, mode=mode).upload()
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    for s in range(4):
        out, lse = H.run_step(case, pfx, s)
        ref, ref_lse = oracle_step(case, s, 0)
        H.assert_close(H.host_f64(out), ref, mname, f"step {s}")


def _stress_case(mode, block_scale):
    """Growing logits: key tile t is scaled so the score spread rises from ~0.1
    to ~4 along the prefix, and the running max climbs by more than 8 log2
    units after the first tile, which drives the tensor-core kernel's rescale
    of the TMEM accumulator. Q is unit-scale; the block keys are multiplied by
    block_scale."""
    from cached_block_attention_b200 import synth
    case = H.make_case(1, 8, 2, 128, 32, (700,), 0, 1.0, scale=1.0, seed=21, mode=mode)
    k = orc.bits_to_f64(case.k_pfx_bits[0])
    ramp = 0.01 + 0.034 * (np.arange(k.shape[1]) // 64)
    case.k_pfx_bits[0] = synth.bf16_bits(k * ramp[None, :, None])
    qb, kb, vb = case.steps_bits[0]
    case.steps_bits[0] = (qb, synth.bf16_bits(orc.bits_to_f64(kb) * block_scale), vb)
    return case.upload()


def test_stress_logits_and_rescale_bf16():
    """Large prefix logits in the bf16 path. The block keys are scaled by 0.01,
    which keeps the in-block logits O(0.1) like the workloads': with unit-scale
    block Q and K the in-block logits reach ~30, and rounding Q^ and K^ to bf16
    (relative 2^-9 each) moves such a logit by ~0.06 (sum over d of |q_i k_i|
    times 2^-8), a relative weight change of 6%, which no bf16 tolerance
    absorbs. That limit belongs to the bf16 arithmetic, not to the method; the
    fp32 check-mode test below runs the unit-scale block."""
    case = _stress_case(0, 0.01)
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, 2, 1.0, case.base)
    assert np.isfinite(ref[1]).all() and ref[1].max() > 6.0  # the test really has large logits
    H.check_partial(H.partial_to_host(pfx), ref, "bf16")
    out, _ = H.run_step(case, pfx, 0)
    H.assert_close(H.host_f64(out), oracle_full(case, 0)[0], "bf16", "O")


def test_stress_logits_and_rescale_fp32_unit_block():
    """The same prefix in fp32 check mode with unit-scale block Q and K: the
    in-block logits reach 10-30 and exercise the step kernel's max
    subtraction and merge. fp32 rounding of a score s moves a softmax weight
    by about |s| 2^-24 sqrt(d), so the 1e-5 bounds are scaled by the largest
    |logit| of the step (the state's m over prefix and block)."""
    case = _stress_case(1, 1.0)
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, 2, 1.0, case.base)
    assert np.isfinite(ref[1]).all() and ref[1].max() > 6.0
    H.check_partial(H.partial_to_host(pfx), ref, "fp32", f32_scale=float(np.abs(ref[1]).max()))
    full, full_lse = oracle_full(case, 0)
    q, k, v = case.step_f64(0)
    blk = orc.block_partial(q, k, v, case.lens, case.hkv, 1.0, case.base)
    assert np.nanmax(blk[1]) > 10.0  # in-block logits are really large
    scale = float(max(np.abs(ref[1]).max(), np.nanmax(np.abs(blk[1]))))
    out, lse = H.run_step(case, pfx, 0)
    H.assert_close(H.host_f64(out), full, "fp32", "O", f32_scale=scale)
    assert np.abs(H.host_f64(lse) - full_lse).max() <= 1e-5 * scale


@pytest.mark.parametrize("splits", [1, 3, 7, 64, 148, 1000])
def test_share_count_does_not_change_result(splits):
    case = H.make_case(3, 16, 4, 128, 32, (999, 64, 2500), 0, 1.0, seed=31, mode=1).upload()
    got = H.partial_to_host(H.run_prefix(case, case.dev["steps"][0][0], num_splits=splits))
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, 4, 1.0, case.base)
    H.check_partial(got, ref, "fp32")


@pytest.mark.parametrize("cfg,splits", [
    ((2, 28, 4, 128, 32, (2000, 3000)), 0),     # ~2 tiles per share: short pieces, two M-tiles
    ((1, 32, 32, 128, 32, (4096,)), 0),         # one real warp per M-tile (MHA, 32 rows)
    ((2, 28, 4, 128, 32, (2000, 3000)), 300),   # mostly 1-tile pieces
    ((3, 8, 2, 64, 16, (100, 0, 333)), 7),      # several pieces per share, empty sequence
])
def test_deterministic_run_to_run(cfg, splits):
    """Repeated calls give bit-identical states (fixed reduction order, no
    races between the kernel's warp roles), each within tolerance of the oracle."""
    b, hq, hkv, d, blk, lens = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, 0, 1.0, seed=41).upload()
    q = case.dev["steps"][0][0]
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, hkv, 1.0, case.base)
    first = H.run_prefix(case, q, num_splits=splits)
    H.check_partial(H.partial_to_host(first), ref, "bf16")
    for _ in range(8):
        again = H.run_prefix(case, q, num_splits=splits)
        for x, y in zip((first.o_unnorm, first.m, first.l), (again.o_unnorm, again.m, again.l)):
            assert torch.equal(x, y)
    oa, _ = H.run_step(case, first, 0)
    ob, _ = H.run_step(case, first, 0)
    assert torch.equal(oa, ob)
    assert int(case.dev["cache"].error_flags.item()) == 0


def test_graph_capture_of_block_loop_matches_eager():
    """partial + S steps + commit captured in one CUDA graph: the graph reads
    prefix_lens on the device, so replaying it equals the eager calls."""
    from cached_block_attention_b200 import fbk
    case = H.make_case(2, 8, 2, 128, 32, (300, 500), 0, 1.0, seed=51, steps=3, cap_extra=64).upload()
    cache = case.dev["cache"]
    lens0 = cache.prefix_lens.clone()
    k0, v0 = cache.k.clone(), cache.v.clone()
    pfx = fbk.Partial.empty(case.shape)
    ws = case.workspace()
    outs = [case.out_tensor() for _ in range(3)]

    def block():
        fbk.prefix_partial(case.shape, case.dev["steps"][0][0], cache, pfx, ws)
        for s in range(3):
            q, k, v = case.dev["steps"][s]
            fbk.block_attn_merge(case.shape, q, k, v, cache.prefix_lens, pfx, outs[s])
        q, k, v = case.dev["steps"][2]
        fbk.commit_block_rope_append(case.shape, k, v, cache)

    block()
    eager = [o.clone() for o in outs]
    eager_k, eager_lens = cache.k.clone(), cache.prefix_lens.clone()
    cache.prefix_lens.copy_(lens0)
    cache.k.copy_(k0)
    cache.v.copy_(v0)
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
            block()
    cache.prefix_lens.copy_(lens0)
    cache.k.copy_(k0)
    cache.v.copy_(v0)
    g.replay()
    torch.cuda.synchronize()
    for e, o in zip(eager, outs):
        assert torch.equal(e, o)
    assert torch.equal(eager_k, cache.k) and torch.equal(eager_lens, cache.prefix_lens)
    np.testing.assert_array_equal(H.host_f64(cache.prefix_lens), case.lens + 32)


# ------------------------------------------------------------------ commit

@pytest.mark.parametrize("ps,base", [(0, 1e4), (64, 1e4), (16, 1e6), (128, 1e4)])
def test_commit_bit_exact(ps, base):
    from cached_block_attention_b200 import fbk
    case = H.make_case(3, 8, 4, 128, 32, (0, 100, 1000), ps, 1.0, base=base, seed=61, cap_extra=40).upload()
    cache = case.dev["cache"]
    k_before, v_before = H.host_bits(cache.k), H.host_bits(cache.v)
    q, k, v = case.dev["steps"][0]
    fbk.commit_block_rope_append(case.shape, k, v, cache)
    torch.cuda.synchronize()
    kb = case.step_f64(0)[1]
    vb_bits = case.steps_bits[0][2]
    if ps:
        table = cache.page_table.cpu().numpy()
        ref_k, ref_v, ref_lens = orc.commit_paged(k_before, v_before, table, kb, vb_bits, case.lens, base)
    else:
        ref_k, ref_v, ref_lens = orc.commit_contiguous(k_before, v_before, kb, vb_bits, case.lens, base)
    np.testing.assert_array_equal(cache.prefix_lens.cpu().numpy(), ref_lens)
    np.testing.assert_array_equal(H.host_bits(cache.v), ref_v)  # V and every untouched slot
    got_k = H.host_bits(cache.k)
    diff = got_k != ref_k
    assert diff.sum() == 0, f"{int(diff.sum())} K elements differ"
    assert int(cache.error_flags.item()) == 0


def test_commit_capacity_overflow_is_flagged_and_skipped():
    from cached_block_attention_b200 import fbk
    case = H.make_case(2, 4, 2, 64, 32, (10, 20), 0, 1.0, seed=71).upload()  # capacity 20 + 32
    cache = case.dev["cache"]
    cache.prefix_lens.copy_(torch.tensor([10, 30], dtype=torch.int32))  # 30 + 32 > 52
    k_before = cache.k.clone()
    q, k, v = case.dev["steps"][0]
    fbk.commit_block_rope_append(case.shape, k, v, cache)
    torch.cuda.synchronize()
    assert cache.prefix_lens.tolist() == [42, 30]
    assert int(cache.error_flags.item()) & fbk.DEVERR_COMMIT
    assert torch.equal(cache.k[1], k_before[1])


@pytest.mark.parametrize("mode,mname", MODES)
def test_all_prefixes_empty(mode, mname):
    """No sequence has a committed token: every row of the state is (0, -inf, 0),
    the step output is plain in-block attention, and a normal call that follows
    still works (the prefix kernels return before any tile work)."""
    case = H.make_case(2, 8, 2, 128, 32, (0, 0), 0, 1.0, seed=90, mode=mode).upload()
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    torch.cuda.synchronize()
    assert torch.isneginf(pfx.m).all() and (pfx.l == 0).all() and (pfx.o_unnorm == 0).all()
    out, lse = H.run_step(case, pfx, 0)
    H.assert_close(H.host_f64(out), oracle_full(case, 0)[0], mname, "empty-prefix step")
    nxt = H.make_case(1, 4, 4, 128, 32, (300,), 0, 1.0, seed=91, mode=mode).upload()
    got = H.partial_to_host(H.run_prefix(nxt, nxt.dev["steps"][0][0]))
    ref = orc.prefix_partial(nxt.step_f64(0)[0], nxt.k_pfx(), nxt.v_pfx(), nxt.lens, 4, 1.0, nxt.base)
    H.check_partial(got, ref, mname)
    assert int(case.dev["cache"].error_flags.item()) == 0


@pytest.mark.parametrize("page_size", [0, 16])
def test_maximum_batch(page_size):
    """b = 1024, the largest batch the shared-memory tile scan takes, with
    ragged short prefixes (a fifth of them empty): every sequence's prefix
    state, one step against uncached attention, and the commit's lengths."""
    from cached_block_attention_b200 import fbk
    rng = np.random.Generator(np.random.PCG64(1024))
    lens = rng.integers(0, 140, size=1024)
    lens[rng.random(1024) < 0.2] = 0
    case = H.make_case(1024, 2, 1, 64, 8, tuple(lens), page_size, 1.0, seed=1024).upload()
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, 1, 1.0, case.base)
    H.check_partial(H.partial_to_host(pfx), ref, "bf16", "b=1024")
    out, _ = H.run_step(case, pfx, 0)
    H.assert_close(H.host_f64(out), oracle_full(case, 0)[0], "bf16", "b=1024 step")
    q, k, v = case.dev["steps"][0]
    fbk.commit_block_rope_append(case.shape, k, v, case.dev["cache"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(case.dev["cache"].prefix_lens.cpu().numpy(), case.lens + 8)
    assert int(case.dev["cache"].error_flags.item()) == 0


def test_bad_prefix_len_and_page_are_flagged_not_read():
    from cached_block_attention_b200 import fbk
    case = H.make_case(2, 4, 2, 128, 16, (100, 100), 64, 1.0, seed=81).upload()
    cache = case.dev["cache"]
    cache.prefix_lens.copy_(torch.tensor([-5, 100], dtype=torch.int32))
    cache.page_table[1, 1] = 10 ** 6  # out of range page id
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    torch.cuda.synchronize()
    flags = int(cache.error_flags.item())
    assert flags & fbk.DEVERR_PREFIX_LEN and flags & fbk.DEVERR_PAGE_ID
    assert torch.isneginf(pfx.m[0]).all()  # the bad sequence is treated as empty
    assert not (flags & fbk.DEVERR_TIMEOUT)


# ------------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("name", ["tiny", "llada8b", "dream7b_gqa", "long131k", "ragged_paged"])
def test_workload_parity(name):
    """Full-size workloads in the bench's launch configuration (0 = one share
    per SM): the prefix state from step 1's queries, every row of every
    denoising step against the oracle's reuse schedule, step 1 against
    uncached attention, then the commit of the last step's K/V."""
    from cached_block_attention_b200 import fbk, synth
    wl = synth.WORKLOADS[name]
    case = H.case_from_workload(wl).upload()
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    kp, vp = case.k_pfx(), case.v_pfx()
    q0 = case.step_f64(0)[0]
    ref_pfx = orc.prefix_partial(q0, kp, vp, case.lens, case.hkv, 1.0, case.base)
    H.check_partial(H.partial_to_host(pfx), ref_pfx, "bf16", name)
    for s in range(wl.steps):
        out, _ = H.run_step(case, pfx, s)
        q, k, v = case.step_f64(s)
        ref, _ = orc.step_output(ref_pfx, q, k, v, case.lens, case.hkv, 1.0, case.base)
        H.assert_close(H.host_f64(out), ref, "bf16", f"{name} step {s}")
        if s == 0:
            full, _ = orc.full_attention(q, k, v, kp, vp, case.lens, case.hkv, 1.0, case.base)
            H.assert_close(H.host_f64(out), full, "bf16", f"{name} step 1 vs uncached")
    cache = case.dev["cache"]
    q, k, v = case.dev["steps"][wl.steps - 1]
    fbk.commit_block_rope_append(case.shape, k, v, cache)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cache.prefix_lens.cpu().numpy(), case.lens + wl.block_len)
    kb = case.step_f64(wl.steps - 1)[1]
    pos_t = np.arange(wl.block_len)
    for b in range(case.batch):
        L = int(case.lens[b])
        pos = L + pos_t
        if case.page_size:
            pt = cache.page_table[b].cpu().numpy()
            rows_k = H.host_bits(cache.k[pt[pos // case.page_size], :, pos % case.page_size])
            rows_v = H.host_bits(cache.v[pt[pos // case.page_size], :, pos % case.page_size])
        else:
            rows_k = H.host_bits(cache.k[b, :, L:L + wl.block_len].transpose(0, 1))
            rows_v = H.host_bits(cache.v[b, :, L:L + wl.block_len].transpose(0, 1))
        # rows_*: [B, Hkv, d]
        want_k = orc.bf16_rne_bits(orc.rope(kb[b], pos[:, None], case.base))
        np.testing.assert_array_equal(rows_k, want_k)
        np.testing.assert_array_equal(rows_v, case.steps_bits[wl.steps - 1][2][b])
    assert int(cache.error_flags.item()) == 0


# ------------------------------------------------------------------ fp32 check mode at workload scale

def check_mode_workload(name):
    """The workload itself for tiny and llada8b; for the three long ones the
    same shape, seeds and value recipe with the prefix shortened to 4096
    tokens (ragged_paged: lengths uniform in [256, 4096]), so that the fp64
    oracle of every step stays within seconds."""
    from dataclasses import replace

    from cached_block_attention_b200 import synth
    wl = synth.WORKLOADS[name]
    if name in ("dream7b_gqa", "long131k"):
        return replace(wl, name=name + "_L4096", prefix_len=4096)
    if name == "ragged_paged":
        return replace(wl, name=name + "_L4096", len_range=(256, 4096))
    return wl


@pytest.mark.parametrize("name", ["tiny", "llada8b", "dream7b_gqa", "long131k", "ragged_paged"])
def test_workload_parity_check_mode(name):
    """fp32 check mode at workload scale, against the fp64 oracle at 1e-5:
    the prefix state from step 1's queries (every row), every row of every
    denoising step against the oracle's reuse schedule, step 1 and step S
    against uncached attention with that step's queries as the state's, and
    the lse of every step."""
    wl = check_mode_workload(name)
    case = H.case_from_workload(wl, mode=1).upload()
    kp, vp = case.k_pfx(), case.v_pfx()
    q0 = case.step_f64(0)[0]
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    ref_pfx = orc.prefix_partial(q0, kp, vp, case.lens, case.hkv, 1.0, case.base)
    H.check_partial(H.partial_to_host(pfx), ref_pfx, "fp32", wl.name)
    for s in range(wl.steps):
        out, lse = H.run_step(case, pfx, s)
        q, k, v = case.step_f64(s)
        ref, ref_lse = orc.step_output(ref_pfx, q, k, v, case.lens, case.hkv, 1.0, case.base)
        H.assert_close(H.host_f64(out), ref, "fp32", f"{wl.name} step {s + 1}")
        assert np.abs(H.host_f64(lse) - ref_lse).max() <= 1e-5, f"{wl.name} step {s + 1} lse"
    # steps 1 and S with their own queries' state equal uncached attention
    for s in sorted({0, wl.steps - 1}):
        own = H.run_prefix(case, case.dev["steps"][s][0])
        out, _ = H.run_step(case, own, s)
        q, k, v = case.step_f64(s)
        full, _ = orc.full_attention(q, k, v, kp, vp, case.lens, case.hkv, 1.0, case.base)
        H.assert_close(H.host_f64(out), full, "fp32", f"{wl.name} step {s + 1} vs uncached")
    assert int(case.dev["cache"].error_flags.item()) == 0


@pytest.mark.parametrize("mode,mname", MODES)
@pytest.mark.parametrize("page_size", [0, 16, 64])
def test_memory_past_the_prefix_is_never_read(page_size, mode, mname):
    """Cache slots past each sequence's committed length hold NaN bit patterns
    (a cache allocated without initialisation may hold anything there). The
    prefix lengths are not multiples of 8, so the last tile of every unit is
    partial: the state and the step output must still be finite and match the
    oracle, which never looks past L_b."""
    case = H.make_case(3, 8, 2, 128, 32, (77, 203, 1001), page_size, 1.0, seed=131, mode=mode,
                       cap_extra=200).upload()
    cache = case.dev["cache"]
    nan = torch.tensor(0x7FC1, dtype=torch.int16).view(torch.bfloat16)
    for bi, L in enumerate(case.lens):
        if page_size:
            table = cache.page_table[bi].cpu().numpy()
            for lp, pid in enumerate(table):
                if pid < 0:
                    continue
                lo = max(0, int(L) - lp * page_size)  # first unused slot of this page
                if lo < page_size:
                    cache.k[pid, :, lo:] = nan
                    cache.v[pid, :, lo:] = nan
        else:
            cache.k[bi, :, int(L):] = nan
            cache.v[bi, :, int(L):] = nan
    pfx = H.run_prefix(case, case.dev["steps"][0][0])
    got = H.partial_to_host(pfx)
    assert np.isfinite(got[0]).all() and np.isfinite(got[2]).all()
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, case.hkv, 1.0, case.base)
    H.check_partial(got, ref, mname, f"page {page_size}")
    out, _ = H.run_step(case, pfx, 0)
    H.assert_close(H.host_f64(out), oracle_full(case, 0)[0], mname, f"page {page_size} step")
    assert int(cache.error_flags.item()) == 0
