"""GPU parity of sparse block-external attention with a cached residual
(FlashBlock, Abstract; the reading in oracle/sparse_residual.py): page means,
the top-k page selection, the sparse state through fbk_prefix_partial_at over
the kept pages, and an approximate step (residual from a dense step, applied
at a later step, merged by fbk_block_attn_merge), against the oracle.

Runs only on a machine with a CUDA GPU and the built library (marker `gpu`).
"""
import numpy as np
import pytest
import torch

from oracle import fbk_oracle as orc
from oracle import sparse_residual as sr
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import fbk  # noqa: F401  (fails loudly if not built)
    yield


# (batch, hq, hkv, d, blk, lens, page_size, k kept pages)
CASES = [
    (2, 8, 2, 128, 32, (700, 333), 64, 4),
    (1, 4, 4, 64, 16, (517,), 16, 7),
    (3, 28, 4, 128, 32, (1000, 64, 129), 64, 2),
]


def logical_pages(table_row, kept_row, n_kept):
    """Logical page indices of the kept physical pages."""
    where = {int(pid): lp for lp, pid in enumerate(table_row)}
    return np.array(sorted(where[int(p)] for p in kept_row[:n_kept]), dtype=np.int64)


def run_selection(case, k):
    from cached_block_attention_b200 import fbk
    cache = case.dev["cache"]
    b, maxp = cache.page_table.shape
    means = torch.zeros(b, maxp, case.hkv, case.d, dtype=torch.float32, device="cuda")
    fbk.page_means(case.shape, cache, means)
    kept = torch.empty(b, k, dtype=torch.int32, device="cuda")
    kept_lens = torch.empty(b, dtype=torch.int32, device="cuda")
    ws = torch.empty(fbk.select_pages_workspace_bytes(case.shape, cache), dtype=torch.uint8, device="cuda")
    fbk.select_pages(case.shape, case.dev["steps"][0][0], cache, means, k, kept, kept_lens, ws)
    torch.cuda.synchronize()
    return means, kept, kept_lens


@pytest.mark.parametrize("cfg", CASES)
def test_page_means_and_selection(cfg):
    b, hq, hkv, d, blk, lens, ps, k = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, ps, 1.0, seed=CASES.index(cfg), steps=1).upload()
    means, kept, kept_lens = run_selection(case, k)
    table = case.dev["cache"].page_table.cpu().numpy()
    kp = case.k_pfx()
    for bi in range(b):
        L = int(lens[bi])
        n_pages = (L + ps - 1) // ps
        for lp in range(n_pages):
            want = kp[bi][:, lp * ps:min(L, lp * ps + ps)].mean(axis=1)      # [Hkv, d]
            np.testing.assert_allclose(means[bi, lp].cpu().numpy(), want, rtol=1e-5, atol=1e-6)
    q0 = case.step_f64(0)[0]
    scores = sr.page_scores(q0, kp, case.lens, hkv, 1.0, case.base, ps)
    want_sel = sr.select_pages(scores, k)
    kept_np, kl = kept.cpu().numpy(), kept_lens.cpu().numpy()
    for bi in range(b):
        n_pages = len(scores[bi])
        n_kept = min(k, n_pages)
        got = logical_pages(table[bi], kept_np[bi], n_kept)
        assert np.all(kept_np[bi][n_kept:] == -1)
        L = int(lens[bi])
        assert kl[bi] == sum(min(ps, L - p * ps) for p in got)
        if not np.array_equal(got, want_sel[bi]):
            # only near-ties at the k-th score may differ (fp32 scores against fp64)
            kth = np.sort(scores[bi])[::-1][n_kept - 1]
            for p in set(got) ^ set(want_sel[bi]):
                assert abs(scores[bi][p] - kth) <= 1e-4 * max(1.0, abs(kth)), (bi, p)


def selection_near_ties_only(got, want, scores_b, n_kept):
    """The device's selection equals the oracle's, except for pages whose fp64
    score lies within fp32 rounding of the k-th score."""
    if np.array_equal(got, want):
        return
    kth = np.sort(scores_b)[::-1][n_kept - 1]
    for p in set(got) ^ set(want):
        assert abs(scores_b[p] - kth) <= 1e-4 * max(1.0, abs(kth)), p


def test_selection_with_exact_ties_takes_the_lower_pages():
    """Six full pages whose every key is one large vector x (per kv-head) tie
    exactly on both sides: their mean is x exactly, so their scores are equal
    bit for bit, and they are the best pages. With k = 3 the three lowest
    logical indices among them are kept."""
    b, hq, hkv, d, blk, ps = 2, 8, 2, 128, 16, 64
    lens = (64 * 40, 64 * 23 + 5)
    case = H.make_case(b, hq, hkv, d, blk, lens, ps, 1.0, seed=41, steps=1)
    rng = np.random.Generator(np.random.PCG64(4141))
    copies = {}
    for bi in range(b):
        x = (rng.standard_normal((hkv, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        n_full = lens[bi] // ps
        tied = sorted(int(p) for p in rng.choice(n_full, size=6, replace=False))
        for p in tied:
            case.k_pfx_bits[bi][:, p * ps:(p + 1) * ps, :] = x[:, None, :]
        copies[bi] = tied
    q0 = case.step_f64(0)[0]
    case.upload()
    k = 3
    _, kept, kept_lens = run_selection(case, k)
    table = case.dev["cache"].page_table.cpu().numpy()
    kept_np = kept.cpu().numpy()
    scores = sr.page_scores(q0, case.k_pfx(), case.lens, hkv, 1.0, case.base, ps)
    want = sr.select_pages(scores, k)
    for bi in range(b):
        tied = copies[bi]
        assert len({float(scores[bi][p]) for p in tied}) == 1 and scores[bi][tied[0]] == scores[bi].max()
        got = logical_pages(table[bi], kept_np[bi], k)
        np.testing.assert_array_equal(got, tied[:k])
        np.testing.assert_array_equal(want[bi], tied[:k])
        assert int(kept_lens[bi]) == k * ps


@pytest.mark.parametrize("k", [1, 1000, 3004])
def test_selection_over_thousands_of_pages(k):
    """3001 pages of 16 tokens (a partial last page), several pages per thread
    in the selection, several score tiles: the selection follows the oracle's,
    and k at or above the page count keeps every page."""
    b, hq, hkv, d, blk, ps = 1, 4, 2, 64, 16, 16
    L = 16 * 3000 + 7
    case = H.make_case(b, hq, hkv, d, blk, (L,), ps, 1.0, seed=43, steps=1).upload()
    _, kept, kept_lens = run_selection(case, k)
    table = case.dev["cache"].page_table.cpu().numpy()
    kept_np = kept.cpu().numpy()
    q0 = case.step_f64(0)[0]
    scores = sr.page_scores(q0, case.k_pfx(), case.lens, hkv, 1.0, case.base, ps)
    n_pages = len(scores[0])
    n_kept = min(k, n_pages)
    got = logical_pages(table[0], kept_np[0], n_kept)
    assert np.all(np.diff(got) > 0) and np.all(kept_np[0][n_kept:] == -1)
    assert int(kept_lens[0]) == sum(min(ps, L - p * ps) for p in got)
    if k >= n_pages:
        np.testing.assert_array_equal(got, np.arange(n_pages))
    selection_near_ties_only(got, sr.select_pages(scores, k)[0], scores[0], n_kept)


@pytest.mark.parametrize("cfg", CASES)
def test_sparse_state_and_approximate_step(cfg):
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, lens, ps, k = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, ps, 1.0, seed=10 + CASES.index(cfg), steps=2).upload()
    _, kept, kept_lens = run_selection(case, k)
    cache = case.dev["cache"]
    table = cache.page_table.cpu().numpy()
    kept_np = kept.cpu().numpy()
    pages = [logical_pages(table[bi], kept_np[bi], min(k, (int(lens[bi]) + ps - 1) // ps)) for bi in range(b)]
    sparse_cache = fbk.KVCache(cache.k, cache.v, kept_lens, kept, cache.error_flags)
    shape = case.shape
    ws = case.workspace()
    q0, q1 = case.dev["steps"][0][0], case.dev["steps"][1][0]

    def sparse_state(q):
        part = fbk.Partial.empty(shape)
        fbk.prefix_partial_at(shape, q, cache.prefix_lens, sparse_cache, part, ws)
        return part
    sp0 = sparse_state(q0)
    dense0 = fbk.Partial.empty(shape)
    fbk.prefix_partial(shape, q0, cache, dense0, ws)
    r_o = torch.empty(b, hq, blk, d, dtype=torch.float32, device="cuda")
    r_lse = torch.empty(b, hq, blk, dtype=torch.float32, device="cuda")
    fbk.residual_capture(shape, dense0, sp0, r_o, r_lse)
    sp1 = sparse_state(q1)
    ext = fbk.Partial.empty(shape)
    fbk.residual_apply(shape, sp1, r_o, r_lse, ext)
    _, kb1, vb1 = case.dev["steps"][1]
    out = case.out_tensor()
    fbk.block_attn_merge(shape, q1, kb1, vb1, cache.prefix_lens, ext, out)
    torch.cuda.synchronize()
    assert int(cache.error_flags.item()) == 0

    kp, vp = case.k_pfx(), case.v_pfx()
    qf0, qf1 = case.step_f64(0)[0], case.step_f64(1)
    ref_sp0 = sr.sparse_prefix_partial(qf0, kp, vp, case.lens, pages, ps, hkv, 1.0, case.base)
    H.check_partial(H.partial_to_host(sp0), ref_sp0, "bf16", "sparse state")
    ref_dense0 = orc.prefix_partial(qf0, kp, vp, case.lens, hkv, 1.0, case.base)
    res = sr.residual(ref_dense0, ref_sp0)
    want, _ = sr.approx_step_output(qf1[0], qf1[1], qf1[2], kp, vp, case.lens, pages, ps, res, hkv, 1.0, case.base)
    H.assert_close(H.host_f64(out), want, "bf16", "approximate step")
