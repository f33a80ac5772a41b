"""Bounded device waits: a wait that runs out ends the kernel with an error
flag and leaves the device usable.

The tensor-core prefix kernel bounds every mbarrier wait; when one runs out it
flags FBK_DEVERR_TIMEOUT, every warp role leaves its loop, the producers wait
(with the same bound) for their own loads in flight, the tensor memory is
freed and the kernel returns. Nothing faults or hangs: the test library
(libfbk_testhooks.so, include/fbk_test_hooks.h) shortens the bound to ~1e5
clocks and has block 0's K producer skip one stage, a load that never lands.
The test checks the flag, then runs normal calls on the same device, through
the test library and through the library proper, and checks them against the
oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import fbk_oracle as orc
from tests import harness as H

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT = 2_000_000_000  # the library's bound, in SM clocks


@pytest.fixture(scope="module")
def hooks():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import build, fbk
    build.build()
    lib = ctypes.CDLL(build.TEST_LIB)
    lib.fbk_test_set_wait_fault.argtypes = [ctypes.c_longlong, ctypes.c_int]
    lib.fbk_test_set_wait_fault.restype = ctypes.c_int
    lib.fbk_prefix_partial.argtypes = fbk.lib.fbk_prefix_partial.argtypes
    lib.fbk_prefix_partial.restype = ctypes.c_int
    yield lib
    lib.fbk_test_set_wait_fault(DEFAULT_LIMIT, -1)


def _prefix(lib, case, num_splits):
    """fbk_prefix_partial of the given library on the case's step-0 queries."""
    from cached_block_attention_b200 import fbk
    out = fbk.Partial.empty(case.shape)
    ws = case.workspace(num_splits)
    cs, cc, po = case.shape.c(), case.dev["cache"].c(), out.c()
    st = lib.fbk_prefix_partial(ctypes.byref(cs), ctypes.c_void_p(case.dev["steps"][0][0].data_ptr()),
                                ctypes.byref(cc), ctypes.byref(po), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                num_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    return out


@pytest.mark.parametrize("cfg,stage", [
    ((2, 28, 4, 128, 32, (1000, 1000)), 1),   # two M-tiles: both softmax warpgroups give up
    ((1, 4, 4, 128, 32, (700,)), 0),          # one M-tile, the very first stage withheld
])
def test_wait_runs_out_flags_timeout_and_device_recovers(hooks, cfg, stage):
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, lens = cfg
    case = H.make_case(b, hq, hkv, d, blk, lens, 0, 1.0, seed=123).upload()
    ref = orc.prefix_partial(case.step_f64(0)[0], case.k_pfx(), case.v_pfx(), case.lens, hkv, 1.0, case.base)
    err = case.dev["cache"].error_flags

    assert hooks.fbk_test_set_wait_fault(100_000, stage) == 0
    _prefix(hooks, case, 4)  # 4 shares: block 0 holds several stages
    torch.cuda.synchronize()
    assert int(err.item()) & fbk.DEVERR_TIMEOUT, "the withheld stage did not time out"

    # the device and both libraries still work: fresh flags, normal bound
    assert hooks.fbk_test_set_wait_fault(DEFAULT_LIMIT, -1) == 0
    err.zero_()
    got = _prefix(hooks, case, 4)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    H.check_partial(H.partial_to_host(got), ref, "bf16", "test library after the timeout")
    got = H.run_prefix(case, case.dev["steps"][0][0])
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    H.check_partial(H.partial_to_host(got), ref, "bf16", "library after the timeout")
