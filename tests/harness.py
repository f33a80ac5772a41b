"""Test-side harness: seeded inputs -> device buffers for the CUDA library and
fp64 arrays for the oracle, plus the comparison metrics the parity tests use.

Tolerances (bf16 production path): max |err| <= 2e-2 and mean |err| <= 2e-3
(absolute), plus relative l2 ||err|| / ||ref|| <= 1e-2, because at these input
scales |O| is ~1e-3 and the absolute bounds alone would accept an all-zero
output. The relative bound comes from the arithmetic: block Q after RoPE and
P~ enter the tensor-core products rounded to bf16 (relative 2^-9 each) and O
is stored in bf16 (2^-9), i.e. a few 1e-3 in l2. fp32 check mode: max |err|
<= 1e-5 and relative l2 <= 1e-5 (fp32 accumulation over <= 131k keys).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from cached_block_attention_b200 import synth
from oracle import fbk_oracle as orc

BF16_MAX_ABS, BF16_MEAN_ABS, BF16_REL = 2e-2, 2e-3, 1e-2
F32_MAX_ABS, F32_REL = 1e-5, 1e-5


def dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    a = np.ascontiguousarray(bits).view(np.int16)
    return torch.from_numpy(a).view(torch.bfloat16).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return orc.bits_to_f64(host_bits(t))
    return t.detach().cpu().double().numpy()


def rel_l2(got, ref) -> float:
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def assert_close(got, ref, mode, what="", f32_scale=1.0):
    """f32_scale widens the fp32 check-mode bounds for inputs whose logits are
    far from the workloads' O(0.1): fp32 rounding of a score s perturbs the
    softmax weights by about |s| * 2^-24 * sqrt(d), so the bound grows with
    the largest |logit| (tests pass that as f32_scale)."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    r = rel_l2(got, ref)
    if mode == "bf16":
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs {err.max():.3e}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs {err.mean():.3e}"
        assert r <= BF16_REL, f"{what}: rel l2 {r:.3e}"
    else:
        assert err.max() <= F32_MAX_ABS * f32_scale, f"{what}: max abs {err.max():.3e}"
        assert r <= F32_REL * f32_scale, f"{what}: rel l2 {r:.3e}"
    return float(err.max()), r


@dataclass
class Case:
    """One attention layer: cache + block inputs, on the device and for the oracle."""
    batch: int
    hq: int
    hkv: int
    d: int
    blk: int
    lens: np.ndarray
    page_size: int
    tau: float
    base: float
    k_pfx_bits: list
    v_pfx_bits: list
    steps_bits: list                     # [(q, k, v) uint16]
    cap_extra: int = 0
    mode: int = 0
    dev: dict = field(default_factory=dict)

    @property
    def shape(self):
        from cached_block_attention_b200 import fbk
        return fbk.Shape(self.batch, self.hq, self.hkv, self.d, self.blk, self.tau, self.base, self.mode)

    # ---------------------------------------------------------- oracle views
    def k_pfx(self):
        return [orc.bits_to_f64(k) for k in self.k_pfx_bits]

    def v_pfx(self):
        return [orc.bits_to_f64(v) for v in self.v_pfx_bits]

    def step_f64(self, s):
        q, k, v = self.steps_bits[s]
        return orc.bits_to_f64(q), orc.bits_to_f64(k), orc.bits_to_f64(v)

    # ---------------------------------------------------------- device side
    def upload(self, device="cuda"):
        from cached_block_attention_b200 import fbk
        extra = self.cap_extra + self.blk
        if self.page_size:
            kp, vp, table = synth.paged_cache(self.k_pfx_bits, self.v_pfx_bits, self.hkv, self.d,
                                              self.page_size, extra, 77)
            k, v = dev_bf16(kp, device), dev_bf16(vp, device)
            pt = torch.from_numpy(table).to(device)
        else:
            cap = int(max(self.lens.max(), 1)) + extra
            kc, vc = synth.contiguous_cache(self.k_pfx_bits, self.v_pfx_bits, self.hkv, self.d, cap)
            k, v = dev_bf16(kc, device), dev_bf16(vc, device)
            pt = None
        lens = torch.from_numpy(self.lens.astype(np.int32)).to(device)
        err = torch.zeros(1, dtype=torch.int32, device=device)
        self.dev["cache"] = fbk.KVCache(k, v, lens, pt, err)
        self.dev["steps"] = [tuple(dev_bf16(x, device) for x in st) for st in self.steps_bits]
        return self

    def workspace(self, num_splits=0):
        from cached_block_attention_b200 import fbk
        n = fbk.prefix_workspace_bytes(self.shape, self.dev["cache"], num_splits)
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def out_tensor(self):
        dt = torch.float32 if self.mode == 1 else torch.bfloat16
        return torch.empty(self.batch, self.blk, self.hq, self.d, dtype=dt, device="cuda")


def make_case(batch=1, hq=2, hkv=2, d=64, blk=32, lens=(256,), page_size=0, tau=1.0, base=1e4,
              scale=None, seed=0, steps=1, heavy=None, cap_extra=0, mode=0) -> Case:
    """Seeded Gaussian case (values ~ N(0,1) * scale, default 1/sqrt(d)).

    heavy=(frac, gain): that fraction of prefix key rows multiplied by gain.
    """
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    lens = np.asarray(lens, dtype=np.int64)
    assert len(lens) == batch
    rng = np.random.Generator(np.random.PCG64(seed + 5000))
    ks, vs = [], []
    for b in range(batch):
        L = int(lens[b])
        k = rng.standard_normal((hkv, L, d))
        v = rng.standard_normal((hkv, L, d))
        if heavy and L:
            pos = rng.choice(L, size=max(1, int(heavy[0] * L)), replace=False)
            k[:, pos] *= heavy[1]
        ks.append(synth.bf16_bits(k * scale))
        vs.append(synth.bf16_bits(v * scale))
    st = []
    for s in range(steps):
        r = np.random.Generator(np.random.PCG64(seed + 6000 + s))
        st.append(tuple(synth.bf16_bits(r.standard_normal(sh) * scale)
                        for sh in ((batch, blk, hq, d), (batch, blk, hkv, d), (batch, blk, hkv, d))))
    return Case(batch, hq, hkv, d, blk, lens, page_size, tau, base, ks, vs, st, cap_extra, mode)


def case_from_workload(wl: synth.Workload, steps=None, mode=0) -> Case:
    lens = wl.prefix_lens()
    ks, vs = synth.gen_prefix(wl, lens)
    n = wl.steps if steps is None else steps
    st = [synth.gen_step(wl, s) for s in range(n)]
    return Case(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.block_len, lens,
                wl.page_size, 1.0, wl.rope_base, ks, vs, st, 0, mode)


# ------------------------------------------------------------------ GPU runs

def run_prefix(case: Case, q_dev, num_splits=0):
    from cached_block_attention_b200 import fbk
    pfx = fbk.Partial.empty(case.shape)
    ws = case.workspace(num_splits)
    fbk.prefix_partial(case.shape, q_dev, case.dev["cache"], pfx, ws, num_splits)
    return pfx


def run_step(case: Case, pfx, s, with_lse=True):
    from cached_block_attention_b200 import fbk
    q, k, v = case.dev["steps"][s]
    out = case.out_tensor()
    lse = torch.empty(case.batch, case.hq, case.blk, dtype=torch.float32, device="cuda") if with_lse else None
    fbk.block_attn_merge(case.shape, q, k, v, case.dev["cache"].prefix_lens, pfx, out, lse)
    return out, lse


def run_full_ref(case: Case, s):
    from cached_block_attention_b200 import fbk
    q, k, v = case.dev["steps"][s]
    out = case.out_tensor()
    lse = torch.empty(case.batch, case.hq, case.blk, dtype=torch.float32, device="cuda")
    fbk.full_ref_attn(case.shape, q, k, v, case.dev["cache"], out, lse)
    return out, lse


def partial_to_host(p):
    return host_f64(p.o_unnorm), host_f64(p.m), host_f64(p.l)


def check_partial(got, ref, mode, what="partial", rows=None, f32_scale=1.0):
    """Compare two states through what is unique about them: the normalised
    output O~/l and the logsumexp m + log l, plus m itself; empty rows must be
    (0, -inf, 0) exactly."""
    go, gm, gl = got
    ro, rm, rl = ref
    empty = np.isneginf(rm)
    assert np.array_equal(np.isneginf(gm), empty), f"{what}: empty rows differ"
    assert np.all(go[empty] == 0) and np.all(gl[empty] == 0), f"{what}: empty rows not zero"
    full = ~empty
    if not full.any():
        return
    gn = go[full] / gl[full][:, None]
    rn = ro[full] / rl[full][:, None]
    assert_close(gn, rn, mode, what + " O~/l", f32_scale)
    lse_tol = 2e-2 if mode == "bf16" else 1e-5 * f32_scale
    assert np.abs((gm[full] + np.log(gl[full])) - (rm[full] + np.log(rl[full]))).max() <= lse_tol, \
        f"{what}: lse"
    assert np.abs(gm[full] - rm[full]).max() <= lse_tol + (1e-2 if mode == "bf16" else 1e-6) * np.abs(rm[full]).max(), \
        f"{what}: m"
