"""GPU parity of fbk_facache_unchanged_rows (LaCache §3.3.3 FACache over a
whole sequence): the rows outside the current block merge their cached state
over the unchanged keys with their state over the block's keys. Checked
against the oracle's FACache step (which is pinned to full-sequence
attention), with the cached state from the oracle, and at the LLaDA-8B shape
with a synthetic state.

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


def make_rows_case(b, hq, hkv, d, blk, n, c0s, base, seed, scale=None):
    """A sequence of n tokens per batch entry with the block at c0s[bi]: U's
    q and k after RoPE at their positions, rounded to bf16 (what RoPECache
    holds), V, and the block's raw bf16 Q/K/V."""
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    r = np.random.Generator(np.random.PCG64(seed))
    nu = n - blk
    qu = np.zeros((b, nu, hq, d), np.uint16)
    ku = np.zeros((b, nu, hkv, d), np.uint16)
    for bi in range(b):
        pos = fc.u_positions(nu, c0s[bi], blk)[:, None]
        qu[bi] = bf16(orc.rope(r.standard_normal((nu, hq, d)) * scale, pos, base))
        ku[bi] = bf16(orc.rope(r.standard_normal((nu, hkv, d)) * scale, pos, base))
    vu = bf16(r.standard_normal((b, nu, hkv, d)) * scale)
    kc = bf16(r.standard_normal((b, blk, hkv, d)) * scale)
    vc = bf16(r.standard_normal((b, blk, hkv, d)) * scale)
    qc = bf16(r.standard_normal((b, blk, hq, d)) * scale)
    return qu, ku, vu, qc, kc, vc


def run_rows(shape, qu, state, kc, vc, c0s):
    from cached_block_attention_b200 import fbk
    dev = lambda bits: H.dev_bf16(bits)
    b, nu, hq, d = qu.shape
    st = fbk.Partial(torch.from_numpy(np.ascontiguousarray(state[0], np.float32)).cuda(),
                     torch.from_numpy(np.ascontiguousarray(state[1], np.float32)).cuda(),
                     torch.from_numpy(np.ascontiguousarray(state[2], np.float32)).cuda())
    out = torch.full((b, nu, hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((b, hq, nu), float("nan"), dtype=torch.float32, device="cuda")
    pos = torch.tensor(c0s, dtype=torch.int32, device="cuda")
    fbk.facache_unchanged_rows(shape, dev(qu), st, dev(kc), dev(vc), pos, out, lse)
    torch.cuda.synchronize()
    return H.host_f64(out), H.host_f64(lse)


# (b, hq, hkv, d, blk, n, c0 per sequence, base, tau)
CASES = [
    (2, 8, 2, 128, 32, 300, (100, 0), 1e4, 1.0),               # prompt + suffix; block first
    (1, 4, 4, 64, 16, 200, (184,), 1e4, 1 / math.sqrt(64)),     # block last: no suffix
    (3, 28, 4, 128, 32, 161, (7, 64, 129), 1e6, 1.0),           # GQA 7, ragged 16-row tail
    (1, 8, 1, 128, 64, 333, (200,), 1e4, 1.0),                  # MQA, B = 64
    (2, 4, 2, 128, 1, 70, (3, 69), 1e4, 1.0),                   # one-token block
]


@pytest.mark.parametrize("cfg", CASES)
def test_unchanged_rows_match_oracle_step(cfg):
    """The cached state of U over U's keys from the oracle (fp64, stored as
    fp32); the step's U rows against the oracle's FACache step, which equals
    full-sequence attention."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, n, c0s, base, tau = cfg
    qu, ku, vu, qc, kc, vc = make_rows_case(b, hq, hkv, d, blk, n, c0s, base, seed=CASES.index(cfg))
    f = orc.bits_to_f64
    state = fc.uu_state(f(qu), f(ku), f(vu), hkv, tau)
    shape = fbk.Shape(b, hq, hkv, d, blk, tau, base)
    got, got_lse = run_rows(shape, qu, state, kc, vc, list(c0s))
    for bi in range(b):
        sl = slice(bi, bi + 1)
        (ou, lu), _ = fc.facache_step(tuple(x[sl] for x in state), f(qu)[sl], f(ku)[sl], f(vu)[sl],
                                      f(qc)[sl], f(kc)[sl], f(vc)[sl], c0s[bi], hkv, tau, base)
        H.assert_close(got[sl], ou, "bf16", f"sequence {bi}")
        assert np.abs(got_lse[sl] - lu).max() <= 2e-2, f"sequence {bi} lse"


def test_empty_state_rows_are_block_attention():
    """Rows whose cached state is empty (O~ = 0, m = -inf, l = 0) get plain
    attention over the block's keys."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, n = 1, 4, 2, 128, 32, 100
    qu, ku, vu, qc, kc, vc = make_rows_case(b, hq, hkv, d, blk, n, (10,), 1e4, seed=77)
    nu = n - blk
    state = (np.zeros((b, hq, nu, d)), np.full((b, hq, nu), -np.inf), np.zeros((b, hq, nu)))
    shape = fbk.Shape(b, hq, hkv, d, blk, 1.0, 1e4)
    got, _ = run_rows(shape, qu, state, kc, vc, [10])
    f = orc.bits_to_f64
    (ou, _), _ = fc.facache_step(state, f(qu), f(ku), f(vu), f(qc), f(kc), f(vc), 10, hkv, 1.0, 1e4)
    H.assert_close(got, ou, "bf16", "empty state")


def test_llada8b_shape_with_synthetic_state():
    """32 heads, d 128, block 32, 5120 unchanged rows (prompt 4096 and a
    1024-token masked suffix), with a seeded synthetic state (m, l > 0, O~):
    every row against the oracle's merge of that state with the block."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, n, c0 = 1, 32, 32, 128, 32, 4096 + 32 + 1024, 4096
    qu, ku, vu, qc, kc, vc = make_rows_case(b, hq, hkv, d, blk, n, (c0,), 1e4, seed=123)
    nu = n - blk
    r = np.random.Generator(np.random.PCG64(5))
    m = r.uniform(-0.5, 0.5, (b, hq, nu))
    l = r.uniform(1.0, 6000.0, (b, hq, nu))
    o = r.standard_normal((b, hq, nu, d)) * 0.05 * l[..., None]
    state = (o.astype(np.float32).astype(np.float64), m.astype(np.float32).astype(np.float64),
             l.astype(np.float32).astype(np.float64))
    shape = fbk.Shape(b, hq, hkv, d, blk, 1.0, 1e4)
    got, got_lse = run_rows(shape, qu, state, kc, vc, [c0])
    f = orc.bits_to_f64
    (ou, lu), _ = fc.facache_step(state, f(qu), f(ku), f(vu), f(qc), f(kc), f(vc), c0, hkv, 1.0, 1e4)
    H.assert_close(got, ou, "bf16", "llada8b shape")
    assert np.abs(got_lse - lu).max() <= 2e-2


def test_block_position_near_int32_max():
    """block_pos c0 = 2^31 - 6: the block's keys sit at c0 + t, past 2^31 for
    t >= 6. Positions are formed in 64 bits, so the rows still match the
    oracle, which rotates at the exact positions."""
    from cached_block_attention_b200 import fbk
    b, hq, hkv, d, blk, n = 1, 4, 2, 128, 32, 132
    c0 = 2 ** 31 - 6
    qu, ku, vu, qc, kc, vc = make_rows_case(b, hq, hkv, d, blk, n, (c0,), 1e4, seed=88)
    f = orc.bits_to_f64
    state = fc.uu_state(f(qu), f(ku), f(vu), hkv, 1.0)
    shape = fbk.Shape(b, hq, hkv, d, blk, 1.0, 1e4)
    got, got_lse = run_rows(shape, qu, state, kc, vc, [c0])
    (ou, lu), _ = fc.facache_step(state, f(qu), f(ku), f(vu), f(qc), f(kc), f(vc), c0, hkv, 1.0, 1e4)
    H.assert_close(got, ou, "bf16", "block at 2^31 - 6")
    assert np.abs(got_lse - lu).max() <= 2e-2
