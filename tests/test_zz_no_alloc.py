"""fbk_prefix_partial_static_scratch: the prefix partial with the library's
built-in scratch array instead of a caller workspace.

The GPU tests call it through the C ABI twice in a row and compare each result
with fbk_prefix_partial (caller workspace) on the same inputs. Both calls run
the same kernels with the same share count and a fixed-order reduction, so the
states must be bit-identical: a scratch-aliasing fault that moved a value by
less than the parity tolerance would still fail. Each result is also checked
within the parity tolerance, as the other tests check states. This file is
named to be collected last, so it also runs after every other test has used
the library in the same process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import harness as H


@pytest.fixture(scope="module")
def fbk():
    from cached_block_attention_b200 import build
    build.build()
    from cached_block_attention_b200 import fbk as m
    return m


def _call_static(fbk, case, q, out, num_splits=0):
    cs, cc, po = case.shape.c(), case.dev["cache"].c(), out.c()
    return fbk.lib.fbk_prefix_partial_static_scratch(
        ctypes.byref(cs), ctypes.c_void_p(q.data_ptr()), ctypes.byref(cc), ctypes.byref(po),
        num_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _compare(got, ref, mname, what):
    """Bit equality of O~, m and l with the workspace call, then the parity
    tests' comparison: empty rows exactly (0, -inf, 0), the rest through O~/l,
    m + log l and m."""
    for name in ("o_unnorm", "m", "l"):
        a, b = getattr(got, name), getattr(ref, name)
        assert torch.equal(a, b), f"{what}: {name} differs from the workspace call " \
            f"({int((a != b).sum())} elements)"
    H.check_partial(H.partial_to_host(got), H.partial_to_host(ref), mname, what)


# (batch, hq, hkv, d, blk, lens, page_size)
CASES = [
    (2, 28, 4, 128, 32, (300, 777), 0),   # GQA, two M-tiles, ragged tails
    (2, 4, 2, 128, 32, (200, 100), 16),   # paged, 16-token pages
    (3, 8, 2, 64, 16, (0, 65, 130), 0),   # an empty prefix in the batch, d = 64
]


@pytest.mark.gpu
@pytest.mark.parametrize("mode,mname", [(0, "bf16"), (1, "fp32")])
@pytest.mark.parametrize("cfg", CASES)
def test_static_scratch_matches_workspace_call(fbk, cfg, mode, mname):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    b, hq, hkv, d, blk, lens, ps = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, ps, seed=40 + CASES.index(cfg), mode=mode).upload()
    q = case.dev["steps"][0][0]
    ref = H.run_prefix(case, q)
    outs = []
    for _ in range(2):  # two calls in a row reuse the same scratch
        out = fbk.Partial.empty(case.shape)
        out.o_unnorm.fill_(float("nan"))
        assert _call_static(fbk, case, q, out) == fbk.OK
        outs.append(out)
    torch.cuda.synchronize()
    for i, out in enumerate(outs):
        _compare(out, ref, mname, f"call {i}")
    assert int(case.dev["cache"].error_flags.item()) == 0


@pytest.mark.gpu
def test_static_scratch_back_to_back_shapes_and_workload(fbk):
    """Two different problems one after the other (the second must not see the
    first's scratch contents), the second at the LLaDA-8B-shaped layer size."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import synth
    a = H.make_case(1, 4, 4, 128, 32, (1000,), 0, seed=50).upload()
    w = H.case_from_workload(synth.WORKLOADS["llada8b"], steps=1).upload()
    refs = [H.run_prefix(c, c.dev["steps"][0][0]) for c in (a, w)]
    outs = []
    for c in (a, w):
        out = fbk.Partial.empty(c.shape)
        fbk.prefix_partial_static_scratch(c.shape, c.dev["steps"][0][0], c.dev["cache"], out)
        outs.append(out)
    torch.cuda.synchronize()
    for out, ref, what in zip(outs, refs, ("small", "llada8b")):
        _compare(out, ref, "bf16", what)


def test_static_scratch_rejects_oversize_on_host(fbk):
    """A call needing more than the built-in array is refused before any CUDA call."""
    s = fbk.CShape(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, block_len=32,
                   softmax_scale=1.0, rope_base=1e4, mode=0)
    c = fbk.CCache(k=0x10000, v=0x20000, paged=0, page_size=0, max_pages_per_seq=0,
                   capacity_tokens=1024, num_pages=0, page_table=None, prefix_lens=0x30000,
                   error_flags=None)
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    # 64 rows x (128 + 2) fp32 per slot: 2000 shares need ~66 MB
    need = fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), ctypes.byref(c), 2000)
    assert need > fbk.STATIC_SCRATCH_BYTES
    st = fbk.lib.fbk_prefix_partial_static_scratch(ctypes.byref(s), ctypes.c_void_p(0x70000),
                                                   ctypes.byref(c), ctypes.byref(p), 2000, None)
    assert st == -6
    assert "32 MiB" in fbk.status_string(-6)
    # argument errors still come first
    assert fbk.lib.fbk_prefix_partial_static_scratch(None, None, None, None, 0, None) == -1
    bad = fbk.CShape(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=96, block_len=32,
                     softmax_scale=1.0, rope_base=1e4, mode=0)
    assert fbk.lib.fbk_prefix_partial_static_scratch(ctypes.byref(bad), ctypes.c_void_p(0x70000),
                                                     ctypes.byref(c), ctypes.byref(p), 4, None) == -2
    assert np.isfinite(need)
