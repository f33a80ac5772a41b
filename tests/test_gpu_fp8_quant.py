"""GPU parity of fbk_fp8_group_quant (LaCache §3.4, Eq. 7-8) against the
oracle: E4M3 codes and fp32 scales bit for bit, on random activations with
outlier channels, on hand-built special values (ties, subnormal codes and
inputs, signed zeros, all-zero groups, the bf16 range's ends), on the
hand-computed fixture, and at the LLaDA-8B FFN shapes in full.

Runs only on a machine with a CUDA GPU and the built library (marker `gpu`).
"""
import json
import os

import numpy as np
import pytest
import torch

from cached_block_attention_b200 import synth
from oracle import fp8_quant as fq

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cached_block_attention_b200 import fbk  # noqa: F401  (fails loudly if not built)
    yield


def run_gpu(x_bits):
    from cached_block_attention_b200 import fbk
    rows, cols = x_bits.shape
    x = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()
    codes = torch.full((rows, cols), 0x7F, dtype=torch.uint8, device="cuda")      # NaN code as poison
    scales = torch.full((rows, cols // 128), float("nan"), dtype=torch.float32, device="cuda")
    fbk.fp8_group_quant(x, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def check(x_bits, what, chunk=512):
    got_c, got_s = run_gpu(x_bits)
    for r0 in range(0, x_bits.shape[0], chunk):
        want_c, want_s = fq.fp8_group_quant(x_bits[r0:r0 + chunk])
        gs = got_s[r0:r0 + chunk]
        assert np.array_equal(gs.view(np.uint32), want_s.view(np.uint32)), \
            f"{what}: {int((gs.view(np.uint32) != want_s.view(np.uint32)).sum())} scales differ"
        diff = got_c[r0:r0 + chunk] != want_c
        assert not diff.any(), f"{what}: {int(diff.sum())} codes differ, first at {np.argwhere(diff)[0] + [r0, 0]}"


@pytest.mark.parametrize("rows,cols", [(1, 128), (3, 128), (7, 384), (33, 4096), (130, 1280), (257, 12288)])
def test_random_activations(rows, cols):
    """N(0,1) activations with 1% outlier channels (x20); odd group counts
    leave the last half-warp of the last warp without a group."""
    check(synth.gen_activations(rows, cols, seed=rows * 7 + cols), f"{rows}x{cols}")


def test_special_values():
    r = np.random.Generator(np.random.PCG64(3))
    rows = []
    # all-zero groups, with and without negative zeros
    rows.append(np.zeros(128, np.float32))
    z = np.zeros(128, np.float32); z[::3] = -0.0; rows.append(z)
    # amax 7 gives scale 7/448 = 2^-6 exactly, so x / scale = 64 x: every E4M3
    # midpoint (a tie), and the bf16 values just above and below each one
    lo = np.arange(0x00, 0x7E)
    mids = ((fq.e4m3_value(lo) + fq.e4m3_value(lo + 1)) / 2 * 2.0 ** -6).astype(np.float32)
    mid_bits = mids.view(np.uint32) >> 16
    assert np.all(mids.view(np.uint32) & 0xFFFF == 0)            # the midpoints are exact in bf16
    sign = np.where(np.arange(126) % 2, -1, 1).astype(np.float32)
    for bits in (mid_bits, mid_bits + 1, mid_bits - 1):
        g = np.zeros(128, np.float32)
        g[0] = 7.0
        g[1:127] = (bits.astype(np.uint32) << 16).view(np.float32) * sign
        rows.append(g)
    # bf16 subnormal inputs (and a group made only of them)
    sub = (r.integers(1, 0x7F, 128).astype(np.uint32) << 16).view(np.float32) * np.where(r.random(128) < .5, -1, 1)
    rows.append(sub.astype(np.float32))
    mixed = r.standard_normal(128).astype(np.float32) * 1e-3; mixed[:16] = sub[:16]; rows.append(mixed)
    # the largest finite bf16 magnitudes, and one huge value among tiny ones
    big = np.full(128, 3.3895314e38, np.float32) * np.where(np.arange(128) % 2, -1, 1); rows.append(big)
    spike = r.standard_normal(128).astype(np.float32) * 1e-30; spike[77] = -1e30; rows.append(spike)
    # one group where every value is the same (all coded +-448)
    rows.append(np.full(128, -0.3, np.float32))
    x = np.stack(rows).astype(np.float32)                  # every value is exact in fp32
    assert x.shape == (len(rows), 128)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)   # truncation to bf16 patterns
    check(bits, "special values")


def test_every_scale():
    """Every positive finite bf16 max|x| A (so every scale the kernel can
    meet), twice: a group of A and its 127 bf16 predecessors (quotients in the
    densest code range below 448) and a group of A and 127 random bf16 values
    below it; signs alternate. Exercises the shared-reciprocal division at
    every scale, the IEEE division of tiny groups, tiny elements of normal
    groups, and the subnormal codes."""
    r = np.random.Generator(np.random.PCG64(17))
    A = np.arange(1, 0x7F80, dtype=np.int64)                       # bf16 bit patterns of A > 0
    pred = np.maximum(A[:, None] - np.arange(1, 128)[None, :], 0)  # 127 predecessors (0 below the bottom)
    rand = (r.random((len(A), 127)) * A[:, None]).astype(np.int64)  # random patterns below A
    sign = np.where(np.arange(127) % 2, 0x8000, 0)[None, :]
    g1 = np.concatenate([A[:, None], pred | sign], axis=1)
    g2 = np.concatenate([A[:, None] | 0x8000, rand | sign], axis=1)
    bits = np.concatenate([g1, g2], axis=0).astype(np.uint16)      # [2 * 32639, 128]
    check(bits, "every scale", chunk=8192)


def test_hand_computed_fixture():
    """The hand-computed fixture through the kernel: codes and scales equal the
    values worked out from Eq. 7-8 and the E4M3 format by hand."""
    with open(os.path.join(GOLDEN, "fp8_group_quant.json")) as f:
        g = json.load(f)
    x = np.zeros((g["rows"], g["cols"]), dtype=np.float32)
    want = np.zeros(x.shape, dtype=np.uint8)
    for e in g["elements"]:
        x[e["row"], e["col"]] = e["x"]
        want[e["row"], e["col"]] = e["code"]
    codes, scales = run_gpu((x.view(np.uint32) >> 16).astype(np.uint16))
    np.testing.assert_array_equal(codes, want)
    np.testing.assert_array_equal(scales, np.asarray(g["scales"], dtype=np.float32))


@pytest.mark.parametrize("cols", [4096, 12288])
def test_llada8b_ffn_shapes(cols):
    """The bench's workloads in full (4128 tokens: prefix 4096 + block 32;
    LLaDA-8B hidden width 4096 and FFN width 12288), every code and scale."""
    check(synth.gen_activations(4128, cols, seed=cols), f"4128x{cols}")


def test_empty_is_a_no_op():
    from cached_block_attention_b200 import fbk
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    codes = torch.empty(0, 256, dtype=torch.uint8, device="cuda")
    scales = torch.empty(0, 2, dtype=torch.float32, device="cuda")
    fbk.fp8_group_quant(x, codes, scales)
    torch.cuda.synchronize()


def test_scale_step_is_exact_for_every_group_max():
    """The kernel's per-group scale step (test build entry point, run on the
    device): for every positive finite bf16 max|x| A the scale is the IEEE
    quotient RN(A / 448), and where A >= 2^-80 the reciprocal that the
    quotient steps use is the correctly rounded RN(1 / scale)."""
    import ctypes
    from cached_block_attention_b200 import build
    build.build()
    lib = ctypes.CDLL(build.TEST_LIB)
    lib.fbk_test_fp8_group_scale.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    lib.fbk_test_fp8_group_scale.restype = ctypes.c_int
    A = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    a_d = torch.from_numpy(A).cuda()
    s_d, y_d = torch.empty_like(a_d), torch.empty_like(a_d)
    assert lib.fbk_test_fp8_group_scale(ctypes.c_void_p(a_d.data_ptr()), ctypes.c_void_p(s_d.data_ptr()),
                                        ctypes.c_void_p(y_d.data_ptr()), len(A)) == 0
    s, y = s_d.cpu().numpy(), y_d.cpu().numpy()
    want_s = (A / np.float32(448)).astype(np.float32)        # IEEE fp32 division on the host
    np.testing.assert_array_equal(s.view(np.uint32), want_s.view(np.uint32))
    big = A >= np.float32(2.0 ** -80)
    want_y = (np.float32(1) / want_s[big]).astype(np.float32)
    np.testing.assert_array_equal(y[big].view(np.uint32), want_y.view(np.uint32))
    assert np.all(y[~big] == np.float32(1))
