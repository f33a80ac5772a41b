"""Benchmark: cached block attention denoising steps per second on B200.

One bench step = one block of block-diffusion decoding on the chosen workload
(default: the LLaDA-8B-shaped layer, b1, 32 heads, d128, prefix 4096, block 32,
32 denoising steps):
    fbk_prefix_partial        (prefix state from the block's first queries)
    32 x fbk_block_attn_merge (one per denoising step, fresh block Q/K/V each)
    fbk_commit_block_rope_append (RoPE + append the finished block)
The value is denoising steps per second over all ranks. Inputs are resident in
HBM; the block is replayed as CUDA graphs; L2 is flushed (a 2x-L2 memset)
before every timed block and the flush is outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

For N > 1 (torchrun), every rank runs an independent replica (no collective;
weak scaling) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cached block-attn denoising steps/s + KV GB/s & TFLOP/s vs roofline (1×B200)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long131k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--keep", type=float, default=0.125,
                    help="--op sparse_prefix: fraction of each sequence's prefix pages kept (top-k)")
    ap.add_argument("--op", default="attention",
                    choices=["attention", "fp8_group_quant", "facache_rows", "facache_step", "sparse_prefix"],
                    help="attention: the cached block attention block (default); fp8_group_quant: the "
                         "per-group FP8 activation quantisation on the FP8_WORKLOADS shapes; facache_rows: "
                         "the FACache step of a whole sequence's unchanged rows (FACACHE_WORKLOADS); "
                         "facache_step: the whole FACache step, unchanged rows and block rows")
    ap.add_argument("--layers", type=int, default=1,
                    help="attention layers per block; > 1 runs the whole block through fbk_decode_block")
    ap.add_argument("--adaptive", default="",
                    help="with --layers: comma-separated drift thresholds; each is also timed through "
                         "fbk_decode_block_adaptive (drift-triggered, depth-aware refresh) and reported in "
                         "adaptive_sweep")
    ap.add_argument("--refresh-interval", default="",
                    help="cache update interval(s) for --layers, comma-separated; the first is the "
                         "reported value, every one is timed and its error against interval 1 reported "
                         "(default: the workload's step count, i.e. the reuse schedule)")
    return ap.parse_args()


# DRAM traffic per launch of the dominant kernels, from ncu captures
# (dram__bytes_read.sum + dram__bytes_write.sum). An entry counts only while the
# kernel's sources hash to the value recorded with it; otherwise traffic is null.
TRAFFIC_FILE = os.path.join(ROOT, "cached_block_attention_b200", "ncu_traffic.json")
KERNEL_SOURCES = {
    "block_merge_mma_kernel": ["block_merge.cu", "common.cuh", "tc.cuh", "launch.h"],
    "prefix_tc_kernel": ["prefix_tc.cu", "common.cuh", "tc.cuh", "launch.h"],
    "fp8_group_quant_kernel": ["fp8_quant.cu", "common.cuh", "launch.h"],
}
API_KERNEL = {"fbk_block_attn_merge": "block_merge_mma_kernel", "fbk_prefix_partial": "prefix_tc_kernel"}


def sources_hash(kernel):
    """Hash of the kernel's source files with comments and blank space removed,
    so that a comment edit does not orphan a capture of unchanged code."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "cached_block_attention_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", " ", text).strip().encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel, workload):
    try:
        with open(TRAFFIC_FILE) as f:
            entries = json.load(f)
    except (OSError, ValueError):
        return None
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and e.get("sources") == sources_hash(kernel):
            return e
    return None


def load_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ roofline

def algorithmic_units(wl):
    """Algorithmic bytes / flops of one launch of each kernel on the workload:
    the prefix kernel reads K and V of every committed token once (and does
    4 * Hq * B * d flops per token: QK^T and PV); the step kernel reads the
    block Q/K/V and the prefix state and writes O."""
    L_sum = int(wl.prefix_lens().sum())
    rows = wl.batch * wl.n_q_heads * wl.block_len
    return {
        "kv_bytes": 4 * wl.n_kv_heads * wl.head_dim * L_sum,
        "pfx_flops": 4 * wl.n_q_heads * wl.block_len * wl.head_dim * L_sum,
        "step_bytes": (rows * wl.head_dim * 2                                      # Q
                       + 2 * wl.batch * wl.block_len * wl.n_kv_heads * wl.head_dim * 2  # K, V
                       + rows * (wl.head_dim + 2) * 4                              # prefix state read
                       + rows * wl.head_dim * 2),                                  # O write
    }


def dominant_roofline(wl, pfx_total_ms, pfx_launch_ms, steps_total_ms, step_launch_ms):
    """Roofline of the kernel with the larger share of the timed region. The
    timed region is a few milliseconds, so the tensor peak is the burst one.
    The prefix call's binding roofline is the slower of its bytes at the HBM
    peak and its flops at that tensor peak; frac = that time / the measured
    launch time. The step kernel's is its bytes at the HBM peak."""
    hbm_gbs, tflops, tflops_sus, peak_kind = load_peaks()
    u = algorithmic_units(wl)
    units = {
        "fbk_block_attn_merge": (steps_total_ms, u["step_bytes"], step_launch_ms),
        "fbk_prefix_partial": (pfx_total_ms, u["kv_bytes"], pfx_launch_ms),
    }
    dom = max(units, key=lambda k: units[k][0])
    _, dom_bytes, dom_launch_ms = units[dom]
    tr = measured_traffic(API_KERNEL[dom], wl.name)
    t_hbm = dom_bytes / (hbm_gbs * 1e9)
    t_tensor = u["pfx_flops"] / (tflops * 1e12) if dom == "fbk_prefix_partial" else 0.0
    if t_tensor > t_hbm:
        achieved = u["pfx_flops"] / (dom_launch_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tflops, "unit": "TFLOP/s",
                    "frac": achieved / tflops, "peak_kind": f"{peak_kind} bf16_tflops (burst)",
                    "frac_of_sustained": achieved / tflops_sus,
                    "algorithmic_flops_per_launch": u["pfx_flops"]}
    else:
        achieved = dom_bytes / (dom_launch_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                    "frac": achieved / hbm_gbs, "peak_kind": f"{peak_kind} hbm_gbs"}
    roofline.update({"traffic": tr["dram_bytes_per_launch"] if tr else None,
                     "traffic_key": ({"kernel": tr["kernel"], "workload": tr["workload"], "sources": tr["sources"]}
                                     if tr else None),
                     "kernel": dom, "algorithmic_bytes_per_launch": dom_bytes,
                     "launch_us": dom_launch_ms * 1e3,
                     "roofline_us": max(t_hbm, t_tensor) * 1e6,
                     "hbm_frac": dom_bytes / (dom_launch_ms * 1e-3) / 1e9 / hbm_gbs})
    if dom == "fbk_prefix_partial":
        roofline["tensor_frac_burst"] = u["pfx_flops"] / (dom_launch_ms * 1e-3) / 1e12 / tflops
    return roofline, u


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world, cuda=True):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    """The largest x over all ranks (each rank's device-timed milliseconds)."""
    import torch
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_steps_per_s(world, blocks, steps_per_block, max_ms):
    """Whole-job throughput: every rank decodes `blocks` blocks of its own
    replica of the workload (weak scaling) in at most max_ms."""
    return world * blocks * steps_per_block / (max_ms * 1e-3)


# ------------------------------------------------------------------ oracle timing

def oracle_block(case, steps):
    """The oracle's reuse schedule for one block (prefix state once, `steps`
    denoising steps, commit): fp64 numpy on the host cores."""
    from oracle import fbk_oracle as orc
    kp, vp = case["kp"], case["vp"]
    lens, hkv, base = case["lens"], case["hkv"], case["base"]
    q0 = case["steps"][0][0]
    pfx = orc.prefix_partial(q0, kp, vp, lens, hkv, 1.0, base)
    for s in range(steps):
        q, k, v = case["steps"][s % len(case["steps"])]
        orc.step_output(pfx, q, k, v, lens, hkv, 1.0, base)
    q, k, v = case["steps"][(steps - 1) % len(case["steps"])]
    orc.commit_contiguous(case["kc"], case["vc"], k, case["vbits"], lens, base)


def oracle_case(wl, n_step_inputs=2):
    from cached_block_attention_b200 import synth
    from oracle import fbk_oracle as orc
    lens = wl.prefix_lens()
    ks, vs = synth.gen_prefix(wl, lens)
    kc, vc = synth.contiguous_cache(ks, vs, wl.n_kv_heads, wl.head_dim, int(lens.max()) + wl.block_len)
    steps = []
    vbits = None
    for s in range(min(n_step_inputs, wl.steps)):
        q, k, v = synth.gen_step(wl, s)
        steps.append((orc.bits_to_f64(q), orc.bits_to_f64(k), orc.bits_to_f64(v)))
        vbits = v
    return {"kp": [orc.bits_to_f64(k) for k in ks], "vp": [orc.bits_to_f64(v) for v in vs],
            "lens": lens, "hkv": wl.n_kv_heads, "base": wl.rope_base, "steps": steps,
            "kc": kc, "vc": vc, "vbits": vbits}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=12.0):
    """Time the oracle as it stands on a bounded sample: whole blocks of the
    workload's reuse schedule, as many as fit in about `budget_s` seconds."""
    case = oracle_case(wl)
    t0 = time.perf_counter()
    oracle_block(case, wl.steps)
    one = time.perf_counter() - t0
    n = max(1, min(20, int(budget_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(n):
        oracle_block(case, wl.steps)
    dt = time.perf_counter() - t0
    out = {"value": n * wl.steps / dt, "unit": "denoising steps/s", "cores": blas_threads(),
           "kind": "oracle",
           "sample": f"{n} whole blocks of {wl.name} ({wl.steps} steps each, prefix state once, "
                     f"commit), fp64 numpy"}
    try:  # the same block on one host thread
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            oracle_block(case, wl.steps)
            t1 = time.perf_counter() - t0
        out["single_thread"] = {"value": wl.steps / t1, "cores": 1, "sample": f"one whole block of {wl.name}"}
    except ImportError:
        pass
    return out


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    case = oracle_case(wl)
    # each bench step is a bounded sample: one block with at most 8 denoising steps
    s = min(wl.steps, 8)
    for _ in range(args.warmup):
        oracle_block(case, s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_block(case, s)
    dt = time.perf_counter() - t0
    v = args.steps * s / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "denoising steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "description": wl.description,
                       "bench_step": f"one block sample: prefix state + {s} denoising steps + commit"},
            "cpu_baseline": {"value": v, "unit": "denoising steps/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": f"one block with {s} of {wl.steps} steps per bench step"},
            "e2e": {"value": v, "unit": "denoising steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def run_ours(args, wl, rank, world, local):
    import torch
    from cached_block_attention_b200 import fbk, synth

    dev = torch.device("cuda", local)
    S = wl.steps
    lens_np = wl.prefix_lens()
    ks, vs = synth.gen_prefix(wl, lens_np)
    extra = wl.block_len
    if wl.page_size:
        kp, vp, table = synth.paged_cache(ks, vs, wl.n_kv_heads, wl.head_dim, wl.page_size, extra, wl.page_seed)
        k_cache = torch.from_numpy(kp.view(np.int16)).view(torch.bfloat16).to(dev)
        v_cache = torch.from_numpy(vp.view(np.int16)).view(torch.bfloat16).to(dev)
        page_table = torch.from_numpy(table).to(dev)
    else:
        kc, vc = synth.contiguous_cache(ks, vs, wl.n_kv_heads, wl.head_dim, int(lens_np.max()) + extra)
        k_cache = torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16).to(dev)
        v_cache = torch.from_numpy(vc.view(np.int16)).view(torch.bfloat16).to(dev)
        page_table = None
    del ks, vs
    lens0 = torch.from_numpy(lens_np.astype(np.int32)).to(dev)
    lens = lens0.clone()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cache = fbk.KVCache(k_cache, v_cache, lens, page_table, err)
    shape = fbk.Shape(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.block_len, 1.0, wl.rope_base,
                      fbk.BF16)
    host_steps = [synth.gen_step(wl, s) for s in range(S)]
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
    h_q = torch.stack([pin(q) for q, _, _ in host_steps])
    h_k = torch.stack([pin(k) for _, k, _ in host_steps])
    h_v = torch.stack([pin(v) for _, _, v in host_steps])
    h_q, h_k, h_v = h_q.pin_memory(), h_k.pin_memory(), h_v.pin_memory()
    d_q, d_k, d_v = h_q.to(dev), h_k.to(dev), h_v.to(dev)
    pfx = fbk.Partial.empty(shape, dev)
    ws = torch.empty(fbk.prefix_workspace_bytes(shape, cache, 0), dtype=torch.uint8, device=dev)
    outs = torch.empty(S, wl.batch, wl.block_len, wl.n_q_heads, wl.head_dim, dtype=torch.bfloat16, device=dev)
    h_out = torch.empty(outs.shape, dtype=torch.bfloat16).pin_memory()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def seg_prefix():
        lens.copy_(lens0)  # every bench step decodes the same block position
        fbk.prefix_partial(shape, d_q[0], cache, pfx, ws)

    def seg_steps():
        for s in range(S):
            fbk.block_attn_merge(shape, d_q[s], d_k[s], d_v[s], lens, pfx, outs[s])

    def seg_commit():
        fbk.commit_block_rope_append(shape, d_k[S - 1], d_v[S - 1], cache)

    def seg_recompute():
        lens.copy_(lens0)
        for s in range(S):
            fbk.prefix_partial(shape, d_q[s], cache, pfx, ws)
            fbk.block_attn_merge(shape, d_q[s], d_k[s], d_v[s], lens, pfx, outs[s])
        fbk.commit_block_rope_append(shape, d_k[S - 1], d_v[S - 1], cache)

    # eager warm-up (also sets kernel attributes before capture)
    for _ in range(2):
        seg_prefix(); seg_steps(); seg_commit()
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"

    def seg_block():
        seg_prefix(); seg_steps(); seg_commit()

    st = torch.cuda.Stream(dev)
    st.wait_stream(torch.cuda.current_stream(dev))
    graphs = []
    with torch.cuda.stream(st):
        for fn in (seg_block, seg_prefix, seg_steps, seg_commit, seg_recompute):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
                fn()
            graphs.append(g)
    torch.cuda.synchronize()
    g_block, g_pfx, g_steps, g_commit, g_recomp = graphs

    def timed_blocks(n):
        """n blocks, each after an L2 flush; one graph per block between two events."""
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(st)
                g_block.replay()
                e[1].record(st)
                evs.append(e)
        return evs

    def segment_blocks(n):
        """Per-segment breakdown: the same block as three graphs with events between."""
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                e[0].record(st)
                g_pfx.replay()
                e[1].record(st)
                g_steps.replay()
                e[2].record(st)
                g_commit.replay()
                e[3].record(st)
                evs.append(e)
        return evs

    timed_blocks(args.warmup)
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    evs = timed_blocks(args.steps)
    barrier(world)
    clock_info = clocks.stop()
    t_blocks = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(sum(t_blocks), world)
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"
    sevs = segment_blocks(max(3, args.steps))
    torch.cuda.synchronize()
    t_pfx = [e[0].elapsed_time(e[1]) for e in sevs]
    t_steps = [e[1].elapsed_time(e[2]) for e in sevs]
    t_commit = [e[2].elapsed_time(e[3]) for e in sevs]

    # recompute-every-step schedule, same flush discipline
    rec = []
    with torch.cuda.stream(st):
        for _ in range(max(3, args.steps // 2)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            g_recomp.replay()
            b.record(st)
            rec.append((a, b))
    torch.cuda.synchronize()
    rec_ms = statistics.mean(a.elapsed_time(b) for a, b in rec)

    # end to end through the public API: every block's inputs go host -> device
    # from pinned memory and its outputs come back, eager API calls. Three
    # streams pipeline the blocks (copy-in of block k+1 and copy-out of block
    # k-1 overlap the compute of block k), double-buffered on the device.
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dq2 = [d_q, torch.empty_like(d_q)]
    dk2 = [d_k, torch.empty_like(d_k)]
    dv2 = [d_v, torch.empty_like(d_v)]
    do2 = [outs, torch.empty_like(outs)]
    ho2 = [h_out, torch.empty(outs.shape, dtype=torch.bfloat16).pin_memory()]
    layer2 = [fbk.LayerBlock(dq2[j], dk2[j], dv2[j], cache, pfx, do2[j], S) for j in range(2)]
    e2e_flush = wl.kv_bytes() < flush.numel()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_back = [torch.cuda.Event() for _ in range(2)]

    def e2e_blocks(n):
        for k in range(n):
            j = k % 2
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev_done[j])  # block k-2 no longer reads buffer j
                dq2[j].copy_(h_q, non_blocking=True)
                dk2[j].copy_(h_k, non_blocking=True)
                dv2[j].copy_(h_v, non_blocking=True)
                ev_in[j].record(s_in)
            with torch.cuda.stream(st):
                st.wait_event(ev_in[j])
                if k >= 2:
                    st.wait_event(ev_back[j])  # block k-2's outputs have left buffer j
                if e2e_flush:  # a prefix larger than twice the L2 evicts itself; a smaller one is flushed
                    flush.zero_()
                lens.copy_(lens0)
                # the whole block (prefix state, S steps, commit) through one API call
                fbk.decode_block(shape, [layer2[j]], ws, commit=True, stream=st)
                ev_done[j].record(st)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                ho2[j].copy_(do2[j], non_blocking=True)
                ev_back[j].record(s_out)

    e2e_blocks(2)
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(4, args.steps // 2)
    a.record(s_in)
    st.wait_event(a)
    s_out.wait_event(a)
    e2e_blocks(n_e2e)
    st.wait_event(ev_back[(n_e2e - 1) % 2])
    st.wait_event(ev_back[(n_e2e - 2) % 2])
    b.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)
    h2d = (h_q.numel() + h_k.numel() + h_v.numel()) * 2
    d2h = h_out.numel() * 2

    hbm_gbs, tflops, tflops_sus, _ = load_peaks()
    mean = lambda x: sum(x) / len(x)
    pfx_ms, steps_ms, commit_ms = mean(t_pfx), mean(t_steps), mean(t_commit)
    step_launch_ms = steps_ms / S
    roofline, u = dominant_roofline(wl, pfx_ms, pfx_ms, steps_ms, step_launch_ms)
    kv_bytes, pfx_flops = u["kv_bytes"], u["pfx_flops"]
    pfx_gbs = kv_bytes / (pfx_ms * 1e-3) / 1e9
    pfx_tfs = pfx_flops / (pfx_ms * 1e-3) / 1e12
    n_per_block = 3 + S + 2  # prefix (query rotation, share kernel, reduce), S steps, commit (rows, lengths)

    value = aggregate_steps_per_s(world, args.steps, S, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "denoising steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "description": wl.description,
                   "bench_step": f"one block: prefix state once + {S} denoising steps + commit, "
                                 "one CUDA graph per block",
                   "breakdown": "prefix_partial.us / step_us / commit_us from the same block run as three "
                                "graphs with events between (includes graph-launch gaps)",
                   "l2": "flushed (2x L2 memset) before every timed block, outside the events",
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "schedule": "reuse (prefix state computed once per block)"},
        "roofline": roofline,
        "prefix_partial": {"us": pfx_ms * 1e3, "kv_gbs": pfx_gbs, "tflops": pfx_tfs,
                           "hbm_frac": pfx_gbs / hbm_gbs, "tensor_frac_sustained": pfx_tfs / tflops_sus,
                           "tensor_frac_burst": pfx_tfs / tflops,
                           "kv_bytes": kv_bytes, "flops": pfx_flops},
        "step_us": step_launch_ms * 1e3, "commit_us": commit_ms * 1e3,
        "recompute_schedule": {"value": world * S / (rec_ms * 1e-3), "unit": "denoising steps/s",
                               "ms_per_block": rec_ms,
                               # reuse over recompute, both from the per-block device times
                               "reuse_speedup": rec_ms / (sum(t_blocks) / len(t_blocks))},
        "e2e": {"value": aggregate_steps_per_s(world, 1, S, e2e_ms), "unit": "denoising steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "one fbk_decode_block call per block (prefix state, S steps, commit); each block's "
                        "inputs H2D from pinned host and its outputs D2H inside the timed region, pipelined "
                        "over three streams (copy-in / compute / copy-out, double-buffered); L2 flushed "
                        "before each block's compute when the prefix K/V are smaller than twice the L2 "
                        "(larger ones evict themselves)",
                "l2_flushed": bool(e2e_flush)},
        "gpu_launches": n_per_block * args.steps,
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, g_block, g_pfx, g_steps, g_commit, g_recomp


# ------------------------------------------------------------------ many layers per block

def oracle_layer_block(case, steps, interval):
    """One layer's block under the refresh schedule, fp64 numpy (the oracle)."""
    from oracle import fbk_oracle as orc
    st = [case["steps"][s % len(case["steps"])] for s in range(steps)]
    orc.refresh_schedule(st, case["kp"], case["vp"], case["lens"], case["hkv"], 1.0, case["base"], interval)
    q, k, v = st[-1]
    orc.commit_contiguous(case["kc"], case["vc"], k, case["vbits"], case["lens"], case["base"])


def run_reference_layers(args, wl, rank):
    """The oracle on a bounded sample of the many-layer block: one layer's
    block (at most 8 steps) per bench step; a denoising step of the whole
    model counts args.layers layer-steps."""
    if rank != 0:
        return
    r = intervals_of(args, wl)[0]
    case = oracle_case(wl)
    s = min(wl.steps, 8)
    for _ in range(args.warmup):
        oracle_layer_block(case, s, r)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_layer_block(case, s, r)
    dt = time.perf_counter() - t0
    v = args.steps * s / dt / args.layers
    sample = f"one layer's block with {s} of {wl.steps} steps (interval {r}) per bench step; value / {args.layers} layers"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "denoising steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "layers": args.layers, "refresh_interval": r,
                       "description": wl.description},
            "cpu_baseline": {"value": v, "unit": "denoising steps/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "denoising steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_layers(args, wl, rank, world, local):
    """N attention layers x S denoising steps per block through one
    fbk_decode_block call, replayed as one CUDA graph per block, with a cache
    update interval r (LaCache App. C): each layer recomputes its prefix state
    at steps 0, r, 2r, ... Every layer has its own cache, block inputs and
    outputs (same synthetic content, separate buffers)."""
    import torch
    from cached_block_attention_b200 import fbk, synth

    dev = torch.device("cuda", local)
    S, N = wl.steps, args.layers
    intervals = intervals_of(args, wl)
    lens_np = wl.prefix_lens()
    ks, vs = synth.gen_prefix(wl, lens_np)
    extra = wl.block_len
    if wl.page_size:
        kp, vp, table = synth.paged_cache(ks, vs, wl.n_kv_heads, wl.head_dim, wl.page_size, extra, wl.page_seed)
        kh, vh, page_table = kp, vp, torch.from_numpy(table).to(dev)
    else:
        kh, vh = synth.contiguous_cache(ks, vs, wl.n_kv_heads, wl.head_dim, int(lens_np.max()) + extra)
        page_table = None
    del ks, vs
    k_src = torch.from_numpy(kh.view(np.int16)).view(torch.bfloat16).to(dev)
    v_src = torch.from_numpy(vh.view(np.int16)).view(torch.bfloat16).to(dev)
    del kh, vh
    lens0 = torch.from_numpy(np.tile(lens_np.astype(np.int32), (N, 1))).to(dev)  # [N, b]
    lens = lens0.clone()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    shape = fbk.Shape(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.block_len, 1.0, wl.rope_base,
                      fbk.BF16)
    host_steps = [synth.gen_step(wl, s) for s in range(S)]
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    h_q = torch.stack([pin(q) for q, _, _ in host_steps]).pin_memory()
    h_k = torch.stack([pin(k) for _, k, _ in host_steps]).pin_memory()
    h_v = torch.stack([pin(v) for _, _, v in host_steps]).pin_memory()
    caches, ins, pfxs, outs = [], [], [], []
    for l in range(N):
        caches.append(fbk.KVCache(k_src.clone(), v_src.clone(), lens[l], page_table, err))
        ins.append((h_q.to(dev), h_k.to(dev), h_v.to(dev)))
        pfxs.append(fbk.Partial.empty(shape, dev))
        outs.append(torch.empty(S, wl.batch, wl.block_len, wl.n_q_heads, wl.head_dim, dtype=torch.bfloat16,
                                device=dev))
    del k_src, v_src
    ws = torch.empty(fbk.prefix_workspace_bytes(shape, caches[0], 0), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def blocks_for(r):
        return [fbk.LayerBlock(ins[l][0], ins[l][1], ins[l][2], caches[l], pfxs[l], outs[l], r) for l in range(N)]

    def run_block(r):
        lens.copy_(lens0)  # every bench step decodes the same block position
        fbk.decode_block(shape, blocks_for(r), ws, commit=True)

    def seg_prefix():  # one refresh of every layer
        for l in range(N):
            fbk.prefix_partial(shape, ins[l][0][0], caches[l], pfxs[l], ws)

    def seg_step():  # one denoising step of every layer
        for l in range(N):
            fbk.block_attn_merge(shape, ins[l][0][0], ins[l][1][0], ins[l][2][0], lens[l], pfxs[l], outs[l][0])

    for r in intervals:
        for _ in range(2):
            run_block(r)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"

    # accuracy of each interval against interval 1 (every step exact up to kernel rounding)
    run_block(1)
    torch.cuda.synchronize()
    exact = torch.stack(outs).float()
    acc = {}
    for r in intervals:
        run_block(r)
        torch.cuda.synchronize()
        d = (torch.stack(outs).float() - exact)
        acc[r] = {"max_abs_vs_interval_1": float(d.abs().max()),
                  "rel_l2_vs_interval_1": float(d.norm() / exact.norm())}
    del exact

    st = torch.cuda.Stream(dev)
    st.wait_stream(torch.cuda.current_stream(dev))
    graphs = {}
    with torch.cuda.stream(st):
        for key, fn in [(("block", r), (lambda r=r: run_block(r))) for r in intervals] + \
                       [(("prefix", 0), seg_prefix), (("step", 0), seg_step)]:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
                fn()
            graphs[key] = g
    torch.cuda.synchronize()

    def timed(g, n):
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(st)
                g.replay()
                e[1].record(st)
                evs.append(e)
        return evs

    main_r = intervals[0]
    timed(graphs[("block", main_r)], args.warmup)
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    evs = timed(graphs[("block", main_r)], args.steps)
    barrier(world)
    clock_info = clocks.stop()
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), world)
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"

    sweep = []
    for r in intervals:
        ev = timed(graphs[("block", r)], max(3, args.steps // 2))
        torch.cuda.synchronize()
        ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        sweep.append({"refresh_interval": r, "value": S / (ms * 1e-3), "unit": "denoising steps/s",
                      "ms_per_block": ms, "refreshes_per_layer": -(-S // r), **acc[r]})
    # the adaptive refresh: one graph per threshold (the decisions are taken on
    # the device, so the block stays one graph); refreshes and accuracy from a
    # run of the same block
    adaptive = []
    thetas = [float(x) for x in args.adaptive.split(",")] if args.adaptive else []
    for theta in thetas:
        pol = fbk.DriftPolicy.empty(theta, N, S, dev)

        def run_adaptive(pol=pol):
            lens.copy_(lens0)
            fbk.decode_block_adaptive(shape, blocks_for(1), pol, ws, commit=True)

        run_adaptive()
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"device error flags {int(err.item())}"
        n_refresh = int(pol.refreshed.sum())
        dmax = float(pol.drift.max())
        run_block(1)
        torch.cuda.synchronize()
        exact = torch.stack(outs).float()
        run_adaptive()
        torch.cuda.synchronize()
        diff = torch.stack(outs).float() - exact
        ga = torch.cuda.CUDAGraph()
        with torch.cuda.stream(st):
            with torch.cuda.graph(ga, stream=st, capture_error_mode="thread_local"):
                run_adaptive()
        torch.cuda.synchronize()
        ev = timed(ga, max(3, args.steps // 2))
        torch.cuda.synchronize()
        ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        adaptive.append({"threshold": theta, "value": S / (ms * 1e-3), "unit": "denoising steps/s",
                         "ms_per_block": ms, "refreshes": n_refresh, "refreshes_per_layer": n_refresh / N,
                         "max_drift": dmax, "max_abs_vs_interval_1": float(diff.abs().max()),
                         "rel_l2_vs_interval_1": float(diff.norm() / exact.norm())})
        del ga, exact, diff
    ev_p = timed(graphs[("prefix", 0)], max(3, args.steps // 2))
    ev_s = timed(graphs[("step", 0)], max(3, args.steps // 2))
    torch.cuda.synchronize()
    pfx_launch_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_p) / N
    step_launch_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_s) / N
    n_ref = -(-S // main_r)
    roofline, u = dominant_roofline(wl, n_ref * N * pfx_launch_ms, pfx_launch_ms, S * N * step_launch_ms,
                                    step_launch_ms)

    # end to end through the public API: each block's inputs for every layer
    # go host -> device from pinned memory and every layer's outputs come back
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h_out = [torch.empty(outs[0].shape, dtype=torch.bfloat16).pin_memory() for _ in range(N)]
    ev_in, ev_done, ev_back = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()

    def e2e_blocks(n):
        for k in range(n):
            with torch.cuda.stream(s_in):
                if k:
                    s_in.wait_event(ev_done)  # the previous block no longer reads the inputs
                for l in range(N):
                    for dst, src in zip(ins[l], (h_q, h_k, h_v)):
                        dst.copy_(src, non_blocking=True)
                ev_in.record(s_in)
            with torch.cuda.stream(st):
                st.wait_event(ev_in)
                if k:
                    st.wait_event(ev_back)  # the previous outputs have left the device buffers
                flush.zero_()
                lens.copy_(lens0)
                fbk.decode_block(shape, blocks_for(main_r), ws, commit=True, stream=st)
                ev_done.record(st)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done)
                for l in range(N):
                    h_out[l].copy_(outs[l], non_blocking=True)
                ev_back.record(s_out)

    e2e_blocks(1)
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 4)
    a.record(s_in)
    st.wait_event(a)
    s_out.wait_event(a)
    e2e_blocks(n_e2e)
    st.wait_event(ev_back)
    b.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)
    h2d = N * (h_q.numel() + h_k.numel() + h_v.numel()) * 2
    d2h = N * outs[0].numel() * 2

    n_launch = N * (3 * n_ref + S + 2)
    value = aggregate_steps_per_s(world, args.steps, S, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "denoising steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": N, "refresh_interval": main_r,
                   "description": wl.description,
                   "bench_step": f"one block of {N} layers x {S} denoising steps through one fbk_decode_block "
                                 f"call (prefix state refreshed every {main_r} steps, then the commit), "
                                 "one CUDA graph per block; a denoising step counts all layers",
                   "l2": "flushed (2x L2 memset) before every timed block, outside the events",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roofline,
        "prefix_us": pfx_launch_ms * 1e3, "step_us": step_launch_ms * 1e3,
        "interval_sweep": sweep,
        **({"adaptive_sweep": adaptive} if adaptive else {}),
        "e2e": {"value": aggregate_steps_per_s(world, 1, S, e2e_ms), "unit": "denoising steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "one fbk_decode_block call per block; every layer's inputs H2D from pinned host and "
                        "outputs D2H inside the timed region (copy-out of a block overlaps copy-in of the next)"},
        "gpu_launches": n_launch * args.steps,
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        case = oracle_case(wl)
        s = min(wl.steps, 8)
        t0 = time.perf_counter()
        oracle_layer_block(case, s, main_r)
        one = time.perf_counter() - t0
        n = max(1, min(20, int(12.0 / max(one, 1e-3))))
        t0 = time.perf_counter()
        for _ in range(n):
            oracle_layer_block(case, s, main_r)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n * s / dt / N, "unit": "denoising steps/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{n} blocks of one layer ({s} steps, interval {main_r}, commit), "
                                          f"fp64 numpy; value / {N} layers"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    graphs.clear()


# ------------------------------------------------------------------ per-group FP8 quantisation

# FFN activations of the LLaDA-8B-shaped sequence (prefix 4096 + block 32 tokens):
# the gate-up input (hidden width 4096) and the ffout input (FFN width 12288).
FP8_WORKLOADS = {
    "ffn_out_llada8b": (4128, 12288, 12288),   # rows, cols, seed
    "ffn_in_llada8b": (4128, 4096, 4096),
}
FP8_METRIC = "per-group FP8 (E4M3, 1x128) activation quantisation, algorithmic GB/s (1×B200)"


def fp8_bytes(rows, cols):
    """Algorithmic bytes of one quantisation: bf16 in, E4M3 codes and fp32 scales out."""
    return rows * cols * 2 + rows * cols + rows * (cols // 128) * 4


def oracle_fp8_sample(x_bits, budget_s=10.0):
    """The oracle on repeated 256-row samples for about budget_s seconds: GB/s."""
    from oracle import fp8_quant as fq
    sample = x_bits[:256]
    t0 = time.perf_counter()
    fq.fp8_group_quant(sample)
    one = time.perf_counter() - t0
    n = max(1, min(50, int(budget_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(n):
        fq.fp8_group_quant(sample)
    dt = time.perf_counter() - t0
    return n * fp8_bytes(*sample.shape) / dt / 1e9, n


def run_fp8_reference(args, name, rank):
    if rank != 0:
        return
    from cached_block_attention_b200 import synth
    rows, cols, seed = FP8_WORKLOADS[name]
    x = synth.gen_activations(rows, cols, seed)
    from oracle import fp8_quant as fq
    sample = x[:256]
    for _ in range(args.warmup):
        fq.fp8_group_quant(sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fq.fp8_group_quant(sample)
    dt = time.perf_counter() - t0
    v = args.steps * fp8_bytes(*sample.shape) / dt / 1e9
    line = {"impl": "reference", "metric": FP8_METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": name, "rows": rows, "cols": cols},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"256 of the {rows} rows per bench step, numpy"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_fp8(args, name, rank, world, local):
    """One bench step = one fbk_fp8_group_quant launch over the whole activation
    matrix, resident in HBM, after an L2 flush (the input alone fits in L2)."""
    import torch
    from cached_block_attention_b200 import fbk, synth
    dev = torch.device("cuda", local)
    rows, cols, seed = FP8_WORKLOADS[name]
    x_bits = synth.gen_activations(rows, cols, seed)
    h_x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    x = h_x.to(dev)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
    scales = torch.empty(rows, cols // 128, dtype=torch.float32, device=dev)
    h_codes = torch.empty(rows, cols, dtype=torch.uint8).pin_memory()
    h_scales = torch.empty(rows, cols // 128, dtype=torch.float32).pin_memory()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream(dev)
    nbytes = fp8_bytes(rows, cols)

    def timed(n):
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(st)
                fbk.fp8_group_quant(x, codes, scales, stream=st)
                e[1].record(st)
                evs.append(e)
        return evs

    timed(max(3, args.warmup))
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    evs = timed(args.steps)
    barrier(world)
    clock_info = clocks.stop()
    t = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(sum(t), world)
    launch_ms = sum(t) / len(t)

    # end to end: the activations H2D from pinned memory, the launch, codes and scales D2H
    def e2e(n):
        with torch.cuda.stream(st):
            for _ in range(n):
                x.copy_(h_x, non_blocking=True)
                fbk.fp8_group_quant(x, codes, scales, stream=st)
                h_codes.copy_(codes, non_blocking=True)
                h_scales.copy_(scales, non_blocking=True)
    e2e(1)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    a.record(st)
    e2e(n_e2e)
    b.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)

    hbm_gbs, _, _, peak_kind = load_peaks()
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    tr = measured_traffic("fp8_group_quant_kernel", name)
    line = {
        "metric": FP8_METRIC, "value": world * args.steps * nbytes / (total_ms * 1e-3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": name, "rows": rows, "cols": cols, "group": 128,
                   "description": "bf16 activations N(0,1) with 1% outlier columns x20 -> E4M3 codes + fp32 "
                                  "scales per 1x128 group (LaCache §3.4 Eq. 7-8)",
                   "bench_step": "one fbk_fp8_group_quant launch over the whole matrix",
                   "l2": "flushed (2x L2 memset) before every timed launch, outside the events",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                     "frac": achieved / hbm_gbs, "peak_kind": f"{peak_kind} hbm_gbs",
                     "traffic": tr["dram_bytes_per_launch"] if tr else None,
                     "traffic_key": ({"kernel": tr["kernel"], "workload": tr["workload"],
                                      "sources": tr["sources"]} if tr else None),
                     "kernel": "fbk_fp8_group_quant", "algorithmic_bytes_per_launch": nbytes,
                     "launch_us": launch_ms * 1e3},
        "elements_per_s": rows * cols / (launch_ms * 1e-3),
        "e2e": {"value": world * nbytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": rows * cols * 2, "d2h_bytes_per_step": rows * cols + rows * (cols // 128) * 4,
                "note": "activations H2D from pinned host, the launch, codes and scales D2H, one stream"},
        "gpu_launches": args.steps,
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n = oracle_fp8_sample(x_bits)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n} x 256 of the {rows} rows, numpy"}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ FACache over a whole sequence

# (b, Hq, Hkv, d, B, unchanged rows, c0, seed): a LLaDA-8B-shaped layer over a
# 4096-token prompt, the 32-token block and a 1024-token masked suffix
FACACHE_WORKLOADS = {
    "llada8b_seq": (1, 32, 32, 128, 32, 4096 + 1024, 4096, 31),
}
FACACHE_METRIC = "FACache step of a sequence's unchanged rows, algorithmic GB/s (1×B200)"


def facache_bytes(b, hq, hkv, d, blk, rows):
    """Algorithmic bytes of one step of the unchanged rows: each row and head
    reads q (bf16) and its state (fp32 O~, m, l) and writes O (bf16); the
    block's K and V are read once per kv-head."""
    return b * rows * hq * (2 * d + 4 * (d + 2) + 2 * d) + 2 * b * blk * hkv * d * 2


def facache_inputs(name):
    """Seeded inputs (host): q_u bf16 bits, a synthetic state (fp32; m, l > 0),
    block K/V bf16 bits."""
    from cached_block_attention_b200 import synth
    b, hq, hkv, d, blk, rows, c0, seed = FACACHE_WORKLOADS[name]
    r = np.random.Generator(np.random.PCG64(seed))
    sc = 1.0 / np.sqrt(d)
    q = synth.bf16_bits(r.standard_normal((b, rows, hq, d), dtype=np.float32) * np.float32(sc))
    m = r.uniform(-0.5, 0.5, (b, hq, rows)).astype(np.float32)
    l = r.uniform(1.0, 6000.0, (b, hq, rows)).astype(np.float32)
    o = (r.standard_normal((b, hq, rows, d), dtype=np.float32) * np.float32(0.05)) * l[..., None]
    kb = synth.bf16_bits(r.standard_normal((b, blk, hkv, d), dtype=np.float32) * np.float32(sc))
    vb = synth.bf16_bits(r.standard_normal((b, blk, hkv, d), dtype=np.float32) * np.float32(sc))
    return q, (o, m, l), kb, vb


def oracle_facache_sample(name, n_rows=256, budget_s=10.0):
    """The oracle's step for the first n_rows unchanged rows, repeated for
    about budget_s seconds: GB/s in the same algorithmic units."""
    from oracle import facache as fc
    from oracle import fbk_oracle as orc
    b, hq, hkv, d, blk, rows, c0, seed = FACACHE_WORKLOADS[name]
    q, (o, m, l), kb, vb = facache_inputs(name)
    qs, st = orc.bits_to_f64(q[:, :n_rows]), (o[:, :, :n_rows], m[:, :, :n_rows], l[:, :, :n_rows])
    kf, vf = orc.bits_to_f64(kb), orc.bits_to_f64(vb)

    def one():
        pos = c0 + np.arange(blk)
        kr = orc.rope(kf, pos[None, :, None], 1e4)
        return orc.finalize(orc.merge(st, fc._state(qs, kr, vf, hkv, 1.0)))
    t0 = time.perf_counter()
    one()
    n = max(1, min(50, int(budget_s / max(time.perf_counter() - t0, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(n):
        one()
    dt = time.perf_counter() - t0
    return n * facache_bytes(b, hq, hkv, d, blk, n_rows) / dt / 1e9, n, dt / n


def run_facache_reference(args, name, rank):
    if rank != 0:
        return
    v, n, per = oracle_facache_sample(name, budget_s=max(1.0, 0.5 * args.steps))
    line = {"impl": "reference", "metric": FACACHE_METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": n, "warmup": args.warmup, "ms_per_step": 1e3 * per, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{n} runs of the step for 256 of the unchanged rows, numpy"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_facache(args, name, rank, world, local):
    """One bench step = one fbk_facache_unchanged_rows launch over every
    unchanged row, inputs resident in HBM, after an L2 flush."""
    import torch
    from cached_block_attention_b200 import fbk
    dev = torch.device("cuda", local)
    b, hq, hkv, d, blk, rows, c0, seed = FACACHE_WORKLOADS[name]
    q, (o, m, l), kb, vb = facache_inputs(name)
    to_bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    h_q = to_bf16(q).pin_memory()
    d_q, d_k, d_v = h_q.to(dev), to_bf16(kb).to(dev), to_bf16(vb).to(dev)
    state = fbk.Partial(torch.from_numpy(o).to(dev), torch.from_numpy(m).to(dev), torch.from_numpy(l).to(dev))
    pos = torch.full((b,), c0, dtype=torch.int32, device=dev)
    out = torch.empty(b, rows, hq, d, dtype=torch.bfloat16, device=dev)
    h_out = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    shape = fbk.Shape(b, hq, hkv, d, blk, 1.0, 1e4)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream(dev)
    nbytes = facache_bytes(b, hq, hkv, d, blk, rows)

    def timed(n):
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(st)
                fbk.facache_unchanged_rows(shape, d_q, state, d_k, d_v, pos, out, stream=st)
                e[1].record(st)
                evs.append(e)
        return evs

    timed(max(3, args.warmup))
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    evs = timed(args.steps)
    barrier(world)
    clock_info = clocks.stop()
    t = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(sum(t), world)
    launch_ms = sum(t) / len(t)

    # end to end: the rows' queries H2D (the state stays resident across the
    # block's steps), the launch, the outputs D2H
    def e2e(n):
        with torch.cuda.stream(st):
            for _ in range(n):
                d_q.copy_(h_q, non_blocking=True)
                fbk.facache_unchanged_rows(shape, d_q, state, d_k, d_v, pos, out, stream=st)
                h_out.copy_(out, non_blocking=True)
    e2e(1)
    torch.cuda.synchronize()
    a, bev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    a.record(st)
    e2e(n_e2e)
    bev.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(bev) / n_e2e, world)

    hbm_gbs, _, _, peak_kind = load_peaks()
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    line = {
        "metric": FACACHE_METRIC, "value": world * args.steps * nbytes / (total_ms * 1e-3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": name, "batch": b, "q_heads": hq, "kv_heads": hkv, "head_dim": d, "block": blk,
                   "unchanged_rows": rows, "block_pos": c0,
                   "description": "LLaDA-8B-shaped layer, 4096-token prompt + 32-token block + 1024-token "
                                  "masked suffix; synthetic cached state",
                   "bench_step": "one fbk_facache_unchanged_rows launch",
                   "l2": "flushed (2x L2 memset) before every timed launch, outside the events",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                     "frac": achieved / hbm_gbs, "peak_kind": f"{peak_kind} hbm_gbs", "traffic": None,
                     "traffic_key": None,
                     "kernel": "fbk_facache_unchanged_rows", "algorithmic_bytes_per_launch": nbytes,
                     "launch_us": launch_ms * 1e3},
        "e2e": {"value": world * nbytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h_q.numel() * 2, "d2h_bytes_per_step": h_out.numel() * 2,
                "note": "the rows' queries H2D, the launch, the outputs D2H, one stream"},
        "gpu_launches": args.steps,
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, _ = oracle_facache_sample(name)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n} runs of the step for 256 of the {rows} unchanged rows, numpy"}
    if rank == 0:
        print(json.dumps(line), flush=True)


FACACHE_STEP_METRIC = "FACache over a whole sequence: denoising steps/s (1×B200)"


def facache_step_inputs(name):
    """Seeded inputs (host) of a whole FACache step: U's queries, U's keys (after
    RoPE) and values in cache layout [b, Hkv, U, d], the block's Q/K/V (bf16 bits)."""
    from cached_block_attention_b200 import synth
    b, hq, hkv, d, blk, rows, c0, seed = FACACHE_WORKLOADS[name]
    q, _, kb, vb = facache_inputs(name)
    r = np.random.Generator(np.random.PCG64(seed + 1))
    sc = np.float32(1.0 / np.sqrt(d))
    ku = synth.bf16_bits(r.standard_normal((b, hkv, rows, d), dtype=np.float32) * sc)
    vu = synth.bf16_bits(r.standard_normal((b, hkv, rows, d), dtype=np.float32) * sc)
    qc = synth.bf16_bits(r.standard_normal((b, blk, hq, d), dtype=np.float32) * sc)
    return q, ku, vu, qc, kb, vb


def facache_step_bytes(b, hq, hkv, d, blk, rows):
    """Algorithmic bytes of one whole step: the unchanged rows (facache_bytes),
    U's K and V read once per kv-head for the block's rows, the block's queries
    and outputs (bf16) and the block rows' state written and read back (fp32)."""
    return (facache_bytes(b, hq, hkv, d, blk, rows) + 2 * b * hkv * rows * d * 2 + 2 * b * blk * hq * d * 2
            + 2 * b * hq * blk * (d + 2) * 4)


def oracle_facache_step_sample(name, n_rows=256, budget_s=10.0):
    """The oracle's whole step (the block's rows attend to all of U's keys) with
    n_rows and with 1 of the unchanged rows, repeated for about budget_s seconds;
    the unchanged rows' time is scaled from the difference to all of them.
    Returns (steps/s, runs)."""
    from oracle import facache as fc
    from oracle import fbk_oracle as orc
    b, hq, hkv, d, blk, rows, c0, seed = FACACHE_WORKLOADS[name]
    q, ku, vu, qc, kb, vb = facache_step_inputs(name)
    _, (o, m, l), _, _ = facache_inputs(name)
    f = orc.bits_to_f64
    ku_s, vu_s = np.transpose(f(ku), (0, 2, 1, 3)), np.transpose(f(vu), (0, 2, 1, 3))  # [b, U, Hkv, d]
    st = (o[:, :, :n_rows], m[:, :, :n_rows], l[:, :, :n_rows])
    st1 = (o[:, :, :1], m[:, :, :1], l[:, :, :1])
    qs, qcf, kbf, vbf = f(q[:, :n_rows]), f(qc), f(kb), f(vb)
    t_many = t_one = 0.0
    n = 0
    t_end = time.perf_counter() + budget_s
    while n == 0 or time.perf_counter() < t_end:
        t0 = time.perf_counter()
        fc.facache_step(st, qs, ku_s, vu_s, qcf, kbf, vbf, c0, hkv, 1.0, 1e4)
        t1 = time.perf_counter()
        fc.facache_step(st1, qs[:, :1], ku_s, vu_s, qcf, kbf, vbf, c0, hkv, 1.0, 1e4)
        t2 = time.perf_counter()
        t_many += t1 - t0
        t_one += t2 - t1
        n += 1
    # the block's rows and one unchanged row, plus the other unchanged rows at the sample's rate
    per_row = max(0.0, (t_many - t_one) / (n_rows - 1)) / n
    per = t_one / n + per_row * (rows - 1)
    return 1.0 / per, n


def run_facache_step(args, name, rank, world, local):
    """One bench step = one fbk_facache_step (the unchanged rows and the block's
    rows) on a LLaDA-8B-shaped sequence, one CUDA graph, inputs resident in HBM,
    L2 flushed before it. The U x U state comes from fbk_facache_refresh (once per
    block), timed separately as refresh_us."""
    import torch
    from cached_block_attention_b200 import fbk
    dev = torch.device("cuda", local)
    b, hq, hkv, d, blk, rows, c0, seed = FACACHE_WORKLOADS[name]
    q, ku, vu, qc, kb, vb = facache_step_inputs(name)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    cache = fbk.KVCache(to(ku), to(vu), torch.full((b,), rows, dtype=torch.int32, device=dev), None,
                        torch.zeros(1, dtype=torch.int32, device=dev))
    d_q, d_qc, d_kb, d_vb = to(q), to(qc), to(kb), to(vb)
    h_qc, h_kb, h_vb = (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
                        for a in (qc, kb, vb))
    state = fbk.Partial(torch.empty(b, hq, rows, d, device=dev), torch.empty(b, hq, rows, device=dev),
                        torch.empty(b, hq, rows, device=dev))
    pos = torch.full((b,), c0, dtype=torch.int32, device=dev)
    out_u = torch.empty(b, rows, hq, d, dtype=torch.bfloat16, device=dev)
    out_c = torch.empty(b, blk, hq, d, dtype=torch.bfloat16, device=dev)
    h_ou = torch.empty(out_u.shape, dtype=torch.bfloat16).pin_memory()
    h_oc = torch.empty(out_c.shape, dtype=torch.bfloat16).pin_memory()
    shape = fbk.Shape(b, hq, hkv, d, blk, 1.0, 1e4)
    ws = torch.empty(fbk.facache_workspace_bytes(shape, rows, 0), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    nbytes = facache_step_bytes(b, hq, hkv, d, blk, rows)

    def refresh():
        fbk.facache_refresh(shape, d_q, [c0] * b, cache, state, ws)

    def step():
        fbk.facache_step(shape, d_q, state, d_qc, d_kb, d_vb, pos, cache, out_u, out_c, ws)

    for _ in range(2):
        refresh()
        step()
    torch.cuda.synchronize()
    assert int(cache.error_flags.item()) == 0, "device error flags"
    st = torch.cuda.Stream(dev)
    st.wait_stream(torch.cuda.current_stream(dev))
    graphs = []
    with torch.cuda.stream(st):
        for fn in (step, refresh):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
                fn()
            graphs.append(g)
    torch.cuda.synchronize()
    g_step, g_refresh = graphs

    def timed(g, n):
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(st)
                g.replay()
                e[1].record(st)
                evs.append(e)
        return evs

    timed(g_step, max(3, args.warmup))
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    evs = timed(g_step, args.steps)
    barrier(world)
    clock_info = clocks.stop()
    t = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(sum(t), world)
    step_ms = sum(t) / len(t)
    rev = timed(g_refresh, max(3, args.steps // 2))
    torch.cuda.synchronize()
    refresh_ms = statistics.mean(a.elapsed_time(c) for a, c in rev)

    # end to end: the block's Q/K/V H2D, the step through the API, both outputs D2H
    def e2e(n):
        with torch.cuda.stream(st):
            for _ in range(n):
                d_qc.copy_(h_qc, non_blocking=True)
                d_kb.copy_(h_kb, non_blocking=True)
                d_vb.copy_(h_vb, non_blocking=True)
                fbk.facache_step(shape, d_q, state, d_qc, d_kb, d_vb, pos, cache, out_u, out_c, ws, stream=st)
                h_ou.copy_(out_u, non_blocking=True)
                h_oc.copy_(out_c, non_blocking=True)
    e2e(1)
    torch.cuda.synchronize()
    a, bev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    a.record(st)
    e2e(n_e2e)
    bev.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(bev) / n_e2e, world)

    hbm_gbs, _, _, peak_kind = load_peaks()
    achieved = nbytes / (step_ms * 1e-3) / 1e9
    line = {
        "metric": FACACHE_STEP_METRIC, "value": world * args.steps / (total_ms * 1e-3), "unit": "denoising steps/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": name, "batch": b, "q_heads": hq, "kv_heads": hkv, "head_dim": d, "block": blk,
                   "unchanged_rows": rows, "block_pos": c0,
                   "description": "LLaDA-8B-shaped layer, 4096-token prompt + 32-token block + 1024-token "
                                  "masked suffix; the U x U state from fbk_facache_refresh",
                   "bench_step": "one fbk_facache_step (unchanged rows + the block's rows over all keys), "
                                 "one CUDA graph",
                   "l2": "flushed (2x L2 memset) before every timed step, outside the events",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "refresh_us": refresh_ms * 1e3,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                     "frac": achieved / hbm_gbs, "peak_kind": f"{peak_kind} hbm_gbs", "traffic": None,
                     "traffic_key": None, "kernel": "fbk_facache_step (all launches)",
                     "algorithmic_bytes_per_launch": nbytes, "launch_us": step_ms * 1e3},
        "e2e": {"value": world / (e2e_ms * 1e-3), "unit": "denoising steps/s",
                "h2d_bytes_per_step": (h_qc.numel() + h_kb.numel() + h_vb.numel()) * 2,
                "d2h_bytes_per_step": (h_ou.numel() + h_oc.numel()) * 2,
                "note": "the block's Q/K/V H2D, the API call, both outputs D2H, one stream"},
        "gpu_launches": 5 * args.steps,  # unchanged rows (1), the block rows' prefix (3), the step kernel (1)
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n = oracle_facache_step_sample(name)
        line["cpu_baseline"] = {"value": v, "unit": "denoising steps/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n} runs of the step with 256 of the {rows} unchanged rows (their "
                                          f"time scaled to all rows) and the block's rows over all keys, numpy"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_facache_step_reference(args, name, rank):
    if rank != 0:
        return
    v, n = oracle_facache_step_sample(name, budget_s=max(1.0, 0.5 * args.steps))
    line = {"impl": "reference", "metric": FACACHE_STEP_METRIC, "value": v, "unit": "denoising steps/s",
            "n_gpus": args.gpus, "steps": n, "warmup": args.warmup, "ms_per_step": 1e3 / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name},
            "cpu_baseline": {"value": v, "unit": "denoising steps/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{n} runs of the step with 256 unchanged rows (scaled) and the block's "
                                       "rows, numpy"},
            "e2e": {"value": v, "unit": "denoising steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ sparse prefix + cached residual

SPARSE_METRIC = "sparse block-external attention with a cached residual: denoising steps/s (1×B200)"


def oracle_sparse_block(case, steps, keep, page):
    """The oracle's sparse schedule for one block (FlashBlock, Abstract; the
    reading of oracle/sparse_residual.py): page scores and the top-k pages from
    step 0's queries, the dense and the sparse state and their residual at step
    0 (whose output is exact), then `steps` - 1 steps of sparse attention plus
    the residual: fp64 numpy on the host cores."""
    from oracle import fbk_oracle as orc
    from oracle import sparse_residual as sr
    kp, vp, lens, hkv, base = case["kp"], case["vp"], case["lens"], case["hkv"], case["base"]
    pages = (np.asarray(lens) + page - 1) // page
    k = max(1, int(round(keep * float(pages.mean()))))
    q0, k0, v0 = case["steps"][0]
    sel = sr.select_pages(sr.page_scores(q0, kp, lens, hkv, 1.0, base, page), k)
    dense = orc.prefix_partial(q0, kp, vp, lens, hkv, 1.0, base)
    res = sr.residual(dense, sr.sparse_prefix_partial(q0, kp, vp, lens, sel, page, hkv, 1.0, base))
    orc.step_output(dense, q0, k0, v0, lens, hkv, 1.0, base)
    for s_ in range(1, steps):
        q, kb, vb = case["steps"][s_ % len(case["steps"])]
        sr.approx_step_output(q, kb, vb, kp, vp, lens, sel, page, res, hkv, 1.0, base)


def run_sparse_reference(args, wl, rank):
    """The reference arm of --op sparse_prefix: the oracle's sparse schedule on
    a bounded sample, one block with at most 4 denoising steps per bench step."""
    if rank != 0:
        return
    case = oracle_case(wl)
    page = wl.page_size or 64
    s = min(wl.steps, 4)
    for _ in range(args.warmup):
        oracle_sparse_block(case, s, args.keep, page)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sparse_block(case, s, args.keep, page)
    dt = time.perf_counter() - t0
    v = args.steps * s / dt
    sample = f"one block with {s} of {wl.steps} steps per bench step (keep {args.keep}, {page}-token pages)"
    line = {"impl": "reference", "metric": SPARSE_METRIC, "value": v, "unit": "denoising steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "keep": args.keep, "page_size": page},
            "cpu_baseline": {"value": v, "unit": "denoising steps/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "denoising steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_sparse(args, wl, rank, world, local):
    """One bench step = one block of the sparse schedule (FlashBlock, Abstract:
    sparse attention with complementary residual reuse; the reading of
    oracle/sparse_residual.py): at step 0 the page means, the top-k pages by
    the block queries' scores, the dense and the sparse prefix state and the
    residual between them; at every step the sparse state over the kept pages
    with that step's queries, the residual applied, and the step kernel. One
    CUDA graph per block, L2 flushed before it. Contiguous workloads are laid
    out in 64-token pages for this (the page table is what the sparse state
    reads through)."""
    import dataclasses
    import torch
    from cached_block_attention_b200 import fbk, synth
    if not wl.page_size:
        wl = dataclasses.replace(wl, page_size=64, page_seed=4242)
    dev = torch.device("cuda", local)
    S = wl.steps
    lens_np = wl.prefix_lens()
    ks, vs = synth.gen_prefix(wl, lens_np)
    kp, vp, table = synth.paged_cache(ks, vs, wl.n_kv_heads, wl.head_dim, wl.page_size, wl.block_len, wl.page_seed)
    del ks, vs
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    lens = torch.from_numpy(lens_np.astype(np.int32)).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cache = fbk.KVCache(to(kp), to(vp), lens, torch.from_numpy(table).to(dev), err)
    del kp, vp
    shape = fbk.Shape(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.block_len, 1.0, wl.rope_base)
    steps = [tuple(to(x) for x in synth.gen_step(wl, s)) for s in range(S)]
    b, maxp = table.shape
    pages = (lens_np + wl.page_size - 1) // wl.page_size
    k = max(1, int(round(args.keep * float(pages.mean()))))
    means = torch.zeros(b, maxp, wl.n_kv_heads, wl.head_dim, dtype=torch.float32, device=dev)
    kept = torch.empty(b, k, dtype=torch.int32, device=dev)
    kept_lens = torch.empty(b, dtype=torch.int32, device=dev)
    sel_ws = torch.empty(fbk.select_pages_workspace_bytes(shape, cache), dtype=torch.uint8, device=dev)
    sparse_cache = fbk.KVCache(cache.k, cache.v, kept_lens, kept, err)
    ws = torch.empty(fbk.prefix_workspace_bytes(shape, cache, 0), dtype=torch.uint8, device=dev)
    dense, sparse, ext = (fbk.Partial.empty(shape, dev) for _ in range(3))
    r_o = torch.empty(b, wl.n_q_heads, wl.block_len, wl.head_dim, dtype=torch.float32, device=dev)
    r_lse = torch.empty(b, wl.n_q_heads, wl.block_len, dtype=torch.float32, device=dev)
    out = torch.empty(S, b, wl.block_len, wl.n_q_heads, wl.head_dim, dtype=torch.bfloat16, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def seg_select():
        fbk.page_means(shape, cache, means)
        fbk.select_pages(shape, steps[0][0], cache, means, k, kept, kept_lens, sel_ws)

    def seg_dense():
        fbk.prefix_partial(shape, steps[0][0], cache, dense, ws)

    def seg_sparse(s=0):
        fbk.prefix_partial_at(shape, steps[s][0], lens, sparse_cache, sparse, ws)

    def block():
        seg_select()
        seg_dense()
        seg_sparse(0)
        fbk.residual_capture(shape, dense, sparse, r_o, r_lse)
        fbk.block_attn_merge(shape, steps[0][0], steps[0][1], steps[0][2], lens, dense, out[0])
        for s in range(1, S):
            seg_sparse(s)
            fbk.residual_apply(shape, sparse, r_o, r_lse, ext)
            fbk.block_attn_merge(shape, steps[s][0], steps[s][1], steps[s][2], lens, ext, out[s])

    for _ in range(2):
        block()
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"
    st = torch.cuda.Stream(dev)
    st.wait_stream(torch.cuda.current_stream(dev))
    graphs = {}
    with torch.cuda.stream(st):
        for name, fn in (("block", block), ("select", seg_select), ("dense", seg_dense), ("sparse", seg_sparse)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
                fn()
            graphs[name] = g
    torch.cuda.synchronize()

    def timed(g, n):
        evs = []
        with torch.cuda.stream(st):
            for _ in range(n):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(st)
                g.replay()
                e[1].record(st)
                evs.append(e)
        return evs

    timed(graphs["block"], args.warmup)
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    evs = timed(graphs["block"], args.steps)
    barrier(world)
    clock_info = clocks.stop()
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), world)
    part = {}
    for name in ("select", "dense", "sparse"):
        ev = timed(graphs[name], max(3, args.steps // 2))
        torch.cuda.synchronize()
        part[name] = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    kept_tokens = int(kept_lens.sum())
    hbm_gbs, _, _, peak_kind = load_peaks()
    sparse_bytes = 4 * wl.n_kv_heads * wl.head_dim * kept_tokens
    achieved = sparse_bytes / (part["sparse"] * 1e-3) / 1e9
    line = {
        "metric": SPARSE_METRIC, "value": aggregate_steps_per_s(world, args.steps, S, total_ms),
        "unit": "denoising steps/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "keep": args.keep, "kept_pages_per_sequence": k,
                   "page_size": wl.page_size, "kept_tokens": kept_tokens, "prefix_tokens": int(lens_np.sum()),
                   "bench_step": f"one block of the sparse schedule ({S} steps), one CUDA graph",
                   "l2": "flushed (2x L2 memset) before every timed block, outside the events",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                     "frac": achieved / hbm_gbs, "peak_kind": f"{peak_kind} hbm_gbs", "traffic": None,
                     "traffic_key": None, "kernel": "fbk_prefix_partial_at (kept pages)",
                     "algorithmic_bytes_per_launch": sparse_bytes, "launch_us": part["sparse"] * 1e3},
        "select_us": part["select"] * 1e3, "dense_prefix_us": part["dense"] * 1e3,
        "sparse_prefix_us": part["sparse"] * 1e3,
        # per block: means (1), selection (rotation, scores, top-k: 3), dense and sparse prefix (3 + 3),
        # residual capture (1) and step (1) at step 0; then sparse prefix (3), residual apply (1), step (1)
        "gpu_launches": (12 + 5 * (S - 1)) * args.steps,
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        case = oracle_case(wl)
        s_o = min(S, 4)
        t0 = time.perf_counter()
        oracle_sparse_block(case, s_o, args.keep, wl.page_size)
        v_o = s_o / (time.perf_counter() - t0)
        line["cpu_baseline"] = {"value": v_o, "unit": "denoising steps/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"one block with {s_o} of {S} steps (keep {args.keep}), fp64 numpy"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    graphs.clear()


def layer_mode(args):
    return args.layers > 1 or bool(args.refresh_interval)


def intervals_of(args, wl):
    return [int(x) for x in args.refresh_interval.split(",")] if args.refresh_interval else [wl.steps]


def main():
    args = parse()
    from cached_block_attention_b200 import synth
    if args.op == "facache_rows":
        name = args.workload if args.workload in FACACHE_WORKLOADS else "llada8b_seq"
        if args.impl == "reference":
            run_facache_reference(args, name, int(os.environ.get("RANK", "0")))
            return
        rank, world, local = dist_setup(args.gpus)
        try:
            run_facache(args, name, rank, world, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    if args.op == "facache_step":
        name = args.workload if args.workload in FACACHE_WORKLOADS else "llada8b_seq"
        if args.impl == "reference":
            run_facache_step_reference(args, name, int(os.environ.get("RANK", "0")))
            return
        rank, world, local = dist_setup(args.gpus)
        try:
            run_facache_step(args, name, rank, world, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    if args.op == "fp8_group_quant":
        name = args.workload if args.workload in FP8_WORKLOADS else "ffn_out_llada8b"
        if args.impl == "reference":
            run_fp8_reference(args, name, int(os.environ.get("RANK", "0")))
            return
        rank, world, local = dist_setup(args.gpus)
        try:
            run_fp8(args, name, rank, world, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    wl = synth.WORKLOADS[args.workload]
    if args.op == "sparse_prefix":
        if args.impl == "reference":
            run_sparse_reference(args, wl, int(os.environ.get("RANK", "0")))
            return
        rank, world, local = dist_setup(args.gpus)
        try:
            run_sparse(args, wl, rank, world, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if layer_mode(args):
            run_reference_layers(args, wl, rank)
        else:
            run_reference(args, wl, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        if layer_mode(args):
            run_layers(args, wl, rank, world, local)
        else:
            run_ours(args, wl, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
