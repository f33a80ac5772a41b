"""Seeded synthetic inputs for cached block attention (shared by tests and bench).

This module is the only code that both the CPU oracle (``oracle/``) and the CUDA
path consume. It holds none of the method's arithmetic: it draws Gaussian
numbers, rounds them to bf16 and lays them out, nothing else.

Workloads follow the shapes the pages describe for LLaDA / Dream-class block
diffusion decoding (LaCache, "Exact Caching and Precision-Adaptive Inference for
Diffusion Large Language Models", §4.1 and Table 9; FlashBlock abstract). The
models and datasets themselves are not used: only their attention shapes.

Recipe (per workload):
  * prefix K/V: ``Generator(PCG64(prefix_seed))``; for each sequence b in order,
    draw K as [Hkv, L_b, d] then V as [Hkv, L_b, d] from N(0, 1); if the
    workload has heavy hitters, then draw ``round(frac * L_b)`` distinct token
    positions and multiply those K rows (all kv-heads) by ``gain``; finally
    multiply by ``value_scale`` and round to bf16 (fp64 -> fp32 -> bf16, both
    round-to-nearest-even). Prefix K is treated as already rotated (its
    distribution is rotation invariant).
  * denoising step s: ``Generator(PCG64(step_seeds[s]))`` draws Q [b,B,Hq,d],
    then K [b,B,Hkv,d], then V [b,B,Hkv,d] from N(0,1), times ``value_scale``,
    rounded to bf16. Block Q and K are pre-RoPE.
  * ragged lengths: ``Generator(PCG64(len_seed)).integers(lo, hi + 1, size=b)``.
  * paged layout: pages of ``page_size`` tokens, room for one more block per
    sequence; physical page ids are ``Generator(PCG64(page_seed)).permutation``
    of the logical pages.
  * FFN activations for the per-group FP8 quantisation (LaCache §3.4, whose
    Fig. 4 shows activation peaks): ``Generator(PCG64(seed))`` draws x
    [rows, cols] from N(0, 1), then picks ``round(0.01 * cols)`` distinct
    outlier columns and multiplies them by 20; rounded to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_len: int
    steps: int
    rope_base: float
    value_scale: float
    prefix_seed: int
    step_seeds: tuple
    prefix_len: int = 0              # uniform prefix length (when len_range is None)
    len_range: tuple | None = None   # (lo, hi) inclusive, ragged lengths
    len_seed: int = 0
    heavy_frac: float = 0.0
    heavy_gain: float = 1.0
    page_size: int = 0               # 0: contiguous cache
    page_seed: int = 0
    description: str = ""

    def prefix_lens(self) -> np.ndarray:
        if self.len_range is None:
            return np.full(self.batch, self.prefix_len, dtype=np.int64)
        lo, hi = self.len_range
        rng = np.random.Generator(np.random.PCG64(self.len_seed))
        return rng.integers(lo, hi + 1, size=self.batch).astype(np.int64)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def kv_bytes(self) -> int:
        """Bytes of prefix K and V (bf16) one prefix-partial pass must stream."""
        return int(4 * self.n_kv_heads * self.head_dim * int(self.prefix_lens().sum()))

    def prefix_flops(self) -> int:
        """QK^T plus PV multiply-adds (x2) of the prefix partial."""
        return int(4 * self.n_q_heads * self.block_len * self.head_dim * int(self.prefix_lens().sum()))


def _d(n):
    return 1.0 / math.sqrt(n)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, block_len=32,
        steps=1, rope_base=1e4, value_scale=_d(64), prefix_seed=1001, step_seeds=(0,),
        prefix_len=256,
        description="tiny single layer: b1, 2 heads MHA, d64, prefix 256, block 32, one step"),
    "llada8b": Workload(
        name="llada8b", batch=1, n_q_heads=32, n_kv_heads=32, head_dim=128, block_len=32,
        steps=32, rope_base=1e4, value_scale=_d(128), prefix_seed=1002,
        step_seeds=tuple(range(1, 33)), prefix_len=4096,
        description="LLaDA-8B-shaped layer: b1, 32 heads MHA, d128, prefix 4096, block 32, 32 steps"),
    "dream7b_gqa": Workload(
        name="dream7b_gqa", batch=8, n_q_heads=28, n_kv_heads=4, head_dim=128, block_len=32,
        steps=16, rope_base=1e6, value_scale=_d(128), prefix_seed=1003,
        step_seeds=tuple(range(1, 17)), prefix_len=32768, heavy_frac=0.01, heavy_gain=8.0,
        description="Dream-7B-shaped GQA layer: b8, 28/4 heads, d128, prefix 32768, block 32, "
                    "1% heavy-hitter key rows x8, 16 steps, RoPE base 1e6"),
    "long131k": Workload(
        name="long131k", batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, block_len=64,
        steps=8, rope_base=1e4, value_scale=_d(128), prefix_seed=1004,
        step_seeds=tuple(range(1, 9)), prefix_len=131072,
        description="long-context layer: b1, 32/8 heads, d128, prefix 131072, block 64, 8 steps"),
    "ragged_paged": Workload(
        name="ragged_paged", batch=16, n_q_heads=32, n_kv_heads=8, head_dim=128, block_len=32,
        steps=32, rope_base=1e4, value_scale=_d(128), prefix_seed=1005,
        step_seeds=tuple(range(1, 33)), len_range=(1024, 16384), len_seed=2000,
        page_size=64, page_seed=2001,
        description="ragged serving batch: 16 sequences, prefix U[1024,16384], 32/8 heads, d128, "
                    "block 32, 64-token pages with a random page table, 32 steps"),
}

# order of the five shapes as listed for this hot path
WORKLOAD_ORDER = ("tiny", "llada8b", "dream7b_gqa", "long131k", "ragged_paged")


# ---------------------------------------------------------------- bf16 packing

def bf16_bits(x) -> np.ndarray:
    """Round to bf16: fp64 -> fp32 (RNE, numpy) -> bf16 (RNE on the fp32 bits)."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- generators

def gen_prefix(wl: Workload, lens=None):
    """Prefix K and V per sequence: lists of uint16 [Hkv, L_b, d] (bf16 bits)."""
    lens = wl.prefix_lens() if lens is None else np.asarray(lens)
    rng = np.random.Generator(np.random.PCG64(wl.prefix_seed))
    ks, vs = [], []
    for b in range(wl.batch):
        L = int(lens[b])
        k = rng.standard_normal((wl.n_kv_heads, L, wl.head_dim))
        v = rng.standard_normal((wl.n_kv_heads, L, wl.head_dim))
        if wl.heavy_frac > 0.0 and L > 0:
            n = int(round(wl.heavy_frac * L))
            pos = rng.choice(L, size=n, replace=False)
            k[:, pos, :] *= wl.heavy_gain
        ks.append(bf16_bits(k * wl.value_scale))
        vs.append(bf16_bits(v * wl.value_scale))
    return ks, vs


def gen_step(wl: Workload, s: int):
    """Block Q, K, V (bf16 bits) of denoising step s (0-based index into step_seeds)."""
    rng = np.random.Generator(np.random.PCG64(wl.step_seeds[s]))
    b, B, d = wl.batch, wl.block_len, wl.head_dim
    q = rng.standard_normal((b, B, wl.n_q_heads, d))
    k = rng.standard_normal((b, B, wl.n_kv_heads, d))
    v = rng.standard_normal((b, B, wl.n_kv_heads, d))
    sc = wl.value_scale
    return bf16_bits(q * sc), bf16_bits(k * sc), bf16_bits(v * sc)


def gen_random(shape, seed, scale=1.0):
    """Generic bf16 Gaussian tensor (for edge-case tests)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return bf16_bits(rng.standard_normal(shape) * scale)


# ---------------------------------------------------------------- layouts

def gen_activations(rows: int, cols: int, seed: int, outlier_frac: float = 0.01,
                    outlier_gain: float = 20.0) -> np.ndarray:
    """FFN input activations [rows, cols] (bf16 bits) with outlier channels."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    n_out = int(round(outlier_frac * cols))
    if n_out:
        x[:, rng.choice(cols, size=n_out, replace=False)] *= np.float32(outlier_gain)
    return bf16_bits(x)


def contiguous_cache(ks, vs, n_kv_heads, head_dim, capacity):
    """Pack per-sequence prefixes into [b, Hkv, capacity, d] (zeros past L_b)."""
    b = len(ks)
    kc = np.zeros((b, n_kv_heads, capacity, head_dim), dtype=np.uint16)
    vc = np.zeros_like(kc)
    for i in range(b):
        L = ks[i].shape[1]
        assert L <= capacity
        kc[i, :, :L] = ks[i]
        vc[i, :, :L] = vs[i]
    return kc, vc


def paged_cache(ks, vs, n_kv_heads, head_dim, page_size, extra_tokens, page_seed):
    """Scatter per-sequence prefixes into pages [P, Hkv, page_size, d].

    Sequence b owns ceil((L_b + extra_tokens) / page_size) pages; physical ids are
    a seeded permutation of the logical pages. Unused table entries hold -1.
    """
    b = len(ks)
    need = [-(-(ks[i].shape[1] + extra_tokens) // page_size) for i in range(b)]
    total = int(sum(need))
    perm = np.random.Generator(np.random.PCG64(page_seed)).permutation(total).astype(np.int32)
    maxp = max(need) if b else 0
    table = np.full((b, maxp), -1, dtype=np.int32)
    kp = np.zeros((total, n_kv_heads, page_size, head_dim), dtype=np.uint16)
    vp = np.zeros_like(kp)
    off = 0
    for i in range(b):
        L = ks[i].shape[1]
        for p in range(need[i]):
            phys = int(perm[off + p])
            table[i, p] = phys
            lo, hi = p * page_size, min(L, (p + 1) * page_size)
            if hi > lo:
                kp[phys, :, : hi - lo] = ks[i][:, lo:hi]
                vp[phys, :, : hi - lo] = vs[i][:, lo:hi]
        off += need[i]
    return kp, vp, table
