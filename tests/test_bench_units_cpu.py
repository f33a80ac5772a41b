"""bench.py's algorithmic units, the numerators of every roofline fraction it
reports, against the closed forms of the measurement contract: the prefix
kernel reads each committed K and V row once per kv-head (4 * Hkv * d bytes
per token), does 4 * Hq * B * d flops per token (QK^T and PV), and the step
kernel reads the block Q/K/V and the prefix state and writes O. The values
for the fixed-length workloads are written out as numbers."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from cached_block_attention_b200 import synth  # noqa: E402

# (kv bytes, prefix flops, step bytes) for the workloads whose prefix lengths are fixed
FIXED = {
    "tiny": (131_072, 4_194_304, 49_664),
    "llada8b": (67_108_864, 2_147_483_648, 1_581_056),
    "dream7b_gqa": (536_870_912, 120_259_084_288, 7_921_664),
    "long131k": (536_870_912, 137_438_953_472, 2_375_680),
}


@pytest.mark.parametrize("name", list(FIXED))
def test_units_of_fixed_workloads(name):
    u = bench.algorithmic_units(synth.WORKLOADS[name])
    assert (u["kv_bytes"], u["pfx_flops"], u["step_bytes"]) == FIXED[name]


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER)
def test_units_follow_the_closed_forms(name):
    wl = synth.WORKLOADS[name]
    L = sum(int(x) for x in wl.prefix_lens())
    b, hq, hkv, d, blk = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.block_len
    u = bench.algorithmic_units(wl)
    assert u["kv_bytes"] == 2 * 2 * hkv * d * L                # K and V, bf16, once per kv-head
    assert u["pfx_flops"] == 2 * 2 * hq * blk * d * L          # two products, two flops per multiply-add
    q_bytes = b * blk * hq * d * 2
    kv_blk = 2 * b * blk * hkv * d * 2
    state = b * hq * blk * (d + 2) * 4                         # O~, m, l in fp32
    assert u["step_bytes"] == q_bytes + kv_blk + state + q_bytes
    assert wl.kv_bytes() == u["kv_bytes"] and wl.prefix_flops() == u["pfx_flops"]


def test_ragged_lengths_are_the_seeded_draw():
    wl = synth.WORKLOADS["ragged_paged"]
    lens = wl.prefix_lens()
    assert len(lens) == 16 and lens.min() >= 1024 and lens.max() <= 16384
    assert (lens == synth.WORKLOADS["ragged_paged"].prefix_lens()).all()  # deterministic


def test_facache_units():
    # 5120 unchanged rows x 32 heads x (2d + 4(d + 2) + 2d) bytes, plus the block's K and V once per kv-head
    assert bench.facache_bytes(1, 32, 32, 128, 32, 5120) == 5120 * 32 * (256 + 520 + 256) + 2 * 32 * 32 * 128 * 2
    # the whole step adds U's K and V once per kv-head, the block rows' Q and O and their state twice
    assert bench.facache_step_bytes(1, 32, 32, 128, 32, 5120) == (
        bench.facache_bytes(1, 32, 32, 128, 32, 5120) + 2 * 32 * 5120 * 128 * 2 + 2 * 32 * 32 * 128 * 2
        + 2 * 32 * 32 * 130 * 4)
