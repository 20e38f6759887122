#!/usr/bin/env python
"""Benchmark of the paged-KV hot path on B200: store_kvcache + paged decode
(+ varlen prefill), through the C ABI of libpagedattn.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step = one attention-layer call of the Qwen3-0.6B-like decode workload
(batch 64, context lengths U[100, 1024], 16 q / 8 kv heads, head_dim 128,
block_size 256): the store of the 64 new K/V rows and the paged decode, in
one launch (pa_store_kv_decode; the two-launch form, pa_store_kv then
pa_decode, is timed beside it).  `value` is decode tokens/s over all ranks (each rank runs
its own replica: the path shards by sequence with no exchange, so scaling is
weak).  Inputs are resident in HBM; L2 is flushed (256 MiB write) before
every timed step; each step is timed with CUDA events on the launching
stream.  The same line carries the long-context, prefix-sharing and varlen
prefill workloads (at N=1), the roofline of the dominant kernel, an end-to-end
figure through the C ABI with host buffers, the CPU oracle baseline and the
SM clocks sampled during the timed region.

For N > 1 launch with torch.distributed.run (one rank per GPU, NCCL); rank 0
prints the single JSON line.  ``--impl reference`` times the CPU oracle (the
reference arm): rank 0 only, a bounded sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode tokens/s and KV HBM GB/s (% of B200 peak); prefill TFLOP/s"
PRIMARY = "qwen3_0.6b_decode"
PRIMARY_DESC = ("Qwen3-0.6B-like decode layer call: batch 64, context_lens U[100,1024], 16 q / 8 kv heads, "
                "head_dim 128, block_size 256, shuffled blocks; store of the 64 new K/V rows + paged decode "
                "(pa_store_kv_decode, one launch)")
FLUSH_BYTES = 256 << 20
SECONDARY_STEPS = 50        # timed runs per secondary measurement (median reported)
CLOCK_SOAK_S = 0.6          # untimed steps on each side of the primary timed region, for the clock sampler
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers --

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(relpath):
    with open(os.path.join(ROOT, relpath), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.txt), or None
    when the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        m = re.match(r"\s*(\S+)\s+source=(\S+)\s+sha=(\w+)\s+bytes_per_launch=(\d+)", line)
        if m and m.group(1) == kernel and source_sha(m.group(2)) == m.group(3):
            return int(m.group(4))
    return None


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        mhz, mx, reasons = [], None, set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                mhz.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[2:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch N>1 with torch.distributed.run")
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """Maximum of a per-rank float over all ranks (the only collective, outside timing)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(local_time_s: float, local_units: float, world: int, device):
    """Whole-job throughput: units of all ranks / the slowest rank's time."""
    t = max_over_ranks(local_time_s, world, device)
    u = sum_over_ranks(local_units, world, device)
    return u / t, t


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


_CASES = {}


def get_case(name):
    """The workload's CPU tensors in their timing form (unused slots filled with N(0,1)), built once and
    shared by the GPU legs and the CPU-oracle baseline."""
    from paged_kv_cache_325_b200 import workloads as W
    if name not in _CASES:
        _CASES[name] = W.WORKLOADS[name](poison=False, keep_contiguous=False)
    return _CASES[name]


# ----------------------------------------------------------- native timing --

class Timer:
    """Per-step CUDA events on the current (launching) stream, L2 flushed between steps."""

    def __init__(self, device):
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def run(self, parts, steps, flush=True):
        """parts: list of callables run in order each step; returns per-part lists of seconds."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)] for _ in range(steps)]
        for i in range(steps):
            if flush:
                self.flush.zero_()
            ev[i][0].record()
            for j, p in enumerate(parts):
                p()
                ev[i][j + 1].record()
        torch.cuda.synchronize()
        return [[ev[i][j].elapsed_time(ev[i][j + 1]) * 1e-3 for i in range(steps)] for j in range(len(parts))]


def capture(fn):
    """Capture fn into a CUDA graph (after one eager call); returns graph.replay."""
    fn()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g.replay, g


def count_kernels(fn):
    """Kernel launches one call of fn makes: fn is captured on a side stream with the runtime API (nothing runs)
    and the kernel nodes of the captured graph are counted."""
    from cuda.bindings import runtime as rt
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        (err,) = rt.cudaStreamBeginCapture(s.cuda_stream, rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
        assert err == rt.cudaError_t.cudaSuccess, err
        try:
            fn()
        finally:
            err, graph = rt.cudaStreamEndCapture(s.cuda_stream)
    assert err == rt.cudaError_t.cudaSuccess, err
    try:
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        assert err == rt.cudaError_t.cudaSuccess, err
        kernels = 0
        for node in nodes[:n]:
            err, ty = rt.cudaGraphNodeGetType(node)
            kernels += int(ty == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
        return kernels
    finally:
        rt.cudaGraphDestroy(graph)


class DecodeBench:
    def __init__(self, case, device):
        import paged_kv_cache_325_b200 as pa
        from paged_kv_cache_325_b200.workloads import DecodeCase  # noqa: F401
        self.pa = pa
        self.case = case
        self.dev = device
        c = case
        self.k_cache = c.k_cache.to(device)
        self.v_cache = c.v_cache.to(device)
        self.k_new = c.k_new.to(device)
        self.v_new = c.v_new.to(device)
        self.q = c.q.to(device)
        self.slot = torch.as_tensor(c.slot_mapping).to(device)
        self.bt = torch.as_tensor(c.block_table).to(device)
        self.ctx = torch.as_tensor(c.context_lens).to(device)
        self.out = torch.empty_like(self.q)
        self.mcl = c.max_context_len
        self.ws = pa.alloc_decode_workspace(self.q, c.num_kv_heads, self.mcl, c.block_size)
        self.splits = self.ws.numel() > 1

    def store(self):
        self.pa.pa_store_kv(self.k_new, self.v_new, self.slot, self.k_cache, self.v_cache)

    def decode(self):
        c = self.case
        self.pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.bt, self.ctx, self.mcl, c.softmax_scale,
                          workspace=self.ws)

    def store_decode(self):
        """The step as one launch: this step's K/V rows stored inside the decode kernel."""
        c = self.case
        self.pa.pa_store_kv_decode(self.k_new, self.v_new, self.slot, self.out, self.q, self.k_cache, self.v_cache,
                                   self.bt, self.ctx, self.mcl, c.softmax_scale, workspace=self.ws)

    def alg_bytes_decode(self):
        c = self.case
        return c.kv_bytes_read() + 2 * self.q.numel() * 2 + c.batch * 4 + self.bt.numel() * 4

    def alg_bytes_store(self):
        return 2 * 2 * self.k_new.numel() * 2 + self.slot.numel() * 4


def bench_primary(args, world, rank, device, pk):
    from paged_kv_cache_325_b200 import workloads as W
    case = get_case(PRIMARY)
    b = DecodeBench(case, device)
    # the step: store + decode in one launch (pa_store_kv_decode); the cache rows it writes are the same
    # every step, so every step does the same work
    step_replay, _g0 = capture(b.store_decode)
    timer = Timer(device)

    def soak(seconds):
        # untimed steps of the same loop (flush + step), so that the clock sampler, whose period is far
        # longer than the timed region, sees the GPU under this load on both sides of it
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            timer.run([step_replay], 50)

    with ClockSampler(local_gpu_index(device)) as clk:
        t_win = time.perf_counter()
        timer.run([step_replay], max(args.warmup, 3))
        soak(CLOCK_SOAK_S)
        barrier(world)
        torch.cuda.synchronize()
        (t_step,) = timer.run([step_replay], args.steps)
        torch.cuda.synchronize()
        barrier(world)
        soak(CLOCK_SOAK_S)
        t_win = time.perf_counter() - t_win
    value, t_max = aggregate(sum(t_step), args.steps * case.batch, world, device)
    step_mean = statistics.mean(t_step)
    clocks = clk.summary()
    clocks["window_s"] = round(t_win, 3)
    clocks["how"] = ("nvidia-smi every 50 ms over a window of the same step loop (L2 flush + graph replay) "
                     f"that brackets the timed steps: warm-up and {CLOCK_SOAK_S} s of untimed steps on each side")
    alg = b.alg_bytes_decode() + b.alg_bytes_store()
    achieved = alg / step_mean / 1e9
    res = {
        "value": value, "ms_per_step": t_max / args.steps * 1e3,
        "kv_gbps": case.kv_bytes_read() / step_mean / 1e9,
        "kv_hbm_frac_of_measured": case.kv_bytes_read() / step_mean / 1e9 / pk["hbm_gbs"],
        "kv_hbm_frac_of_8tbs": case.kv_bytes_read() / step_mean / 1e9 / 8000.0,
        "store_decode_us": step_mean * 1e6, "step_us_median": statistics.median(t_step) * 1e6,
        "roofline": {"kernel": "decode_split_kernel<128, 1> (store fused)", "bound": "hbm",
                     "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                     "traffic": recorded_traffic("store_decode_qwen3_0.6b"), "alg_bytes_per_launch": alg},
        # per step: the kernels of one pa_store_kv_decode call (planning, decode with the store fused in, and a
        # combine only when pairs have many splits), counted from a captured graph of the call
        "gpu_launches": count_kernels(b.store_decode) * args.steps,
        "clocks": clocks,
    }
    # the same step as two launches (pa_store_kv, then pa_decode), for comparison; rank 0 at N=1
    if world == 1:
        st_replay, _g1 = capture(b.store)
        dec_replay, _g2 = capture(b.decode)
        timer.run([st_replay, dec_replay], 5)
        steps2 = max(args.secondary_steps, min(args.steps, 500))
        t_store, t_dec = timer.run([st_replay, dec_replay], steps2)
        res["separate_launches"] = {"store_us": statistics.median(t_store) * 1e6,
                                    "decode_us": statistics.median(t_dec) * 1e6,
                                    "tokens_per_s": case.batch / (statistics.median(t_store) +
                                                                  statistics.median(t_dec)),
                                    "steps": steps2, "statistic": "median"}
    res["e2e"] = bench_e2e(b, args, world, device)
    return case, res


def bench_e2e(b, args, world, device):
    """Same metric through the public API with pinned host buffers: per step, the H2D copy of the step's
    inputs, store + decode, the D2H copy of the output, all inside the timed region.  As a serving loop
    would, the step's inputs (q, the new K/V rows, slot_mapping, block_table, context_lens) live in one
    pinned host buffer and one device buffer of the same layout, so they cross in one copy, and the
    pa_store_kv_decode call on the device buffer's views is a captured CUDA graph (the engine's decode
    graph, whose static inputs each step refills)."""
    names = ("q", "k_new", "v_new", "slot", "bt", "ctx")
    offs, off = {}, 0
    for name in names:
        t = getattr(b, name)
        offs[name] = off
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    host_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
    dev_buf = torch.empty(off, dtype=torch.uint8, device=device)

    def view(buf, name):
        t = getattr(b, name)
        n = t.numel() * t.element_size()
        return buf[offs[name]:offs[name] + n].view(t.dtype).view(t.shape)

    for name in names:
        view(host_buf, name).copy_(getattr(b, name).cpu())
    for name in names:                      # the graph below reads the step's inputs from the device buffer
        setattr(b, name, view(dev_buf, name))
    dev_buf.copy_(host_buf)
    replay, _graph = capture(b.store_decode)
    out_h = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()
    h2d = off
    d2h = out_h.numel() * out_h.element_size()

    def step():
        dev_buf.copy_(host_buf, non_blocking=True)
        replay()
        out_h.copy_(b.out, non_blocking=True)

    timer = Timer(device)
    timer.run([step], max(args.warmup, 3))
    steps = max(1, min(args.steps, 500))
    barrier(world)
    (ts,) = timer.run([step], steps)
    barrier(world)
    value, _ = aggregate(sum(ts), steps * b.case.batch, world, device)
    return {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "how": "one pinned H2D copy of the step's inputs, a graph replay of "
                                   "pa_store_kv_decode, one D2H copy of the output"}


def bench_secondary(args, device, pk, names):
    """Long-context and prefix-sharing decode, varlen prefill: rank 0 at N=1."""
    import paged_kv_cache_325_b200 as pa
    from paged_kv_cache_325_b200 import workloads as W
    timer = Timer(device)
    out = {}
    steps = args.secondary_steps
    for name in [n for n in names if n in ("long_context_decode", "prefix_sharing_decode")]:
        case = get_case(name)
        b = DecodeBench(case, device)
        b.store()
        dec_replay, _g = capture(b.decode)
        timer.run([dec_replay], 5)
        (t,) = timer.run([dec_replay], steps)
        tm = statistics.median(t)
        ach = b.alg_bytes_decode() / tm / 1e9
        r = {"decode_us": tm * 1e6, "tokens_per_s": case.batch / tm,
             "kv_gbps_logical": case.kv_bytes_read() / tm / 1e9,
             "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": ach / pk["hbm_gbs"], "frac_of_8tbs": ach / 8000.0}}
        if name == "prefix_sharing_decode":
            uniq = case.kv_bytes_unique() + 2 * b.q.numel() * 2
            r["kv_gbps_unique"] = case.kv_bytes_unique() / tm / 1e9
            r["roofline"] = {"bound": "hbm", "achieved": uniq / tm / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": uniq / tm / 1e9 / pk["hbm_gbs"], "bytes": "unique"}
            (tw,) = timer.run([dec_replay], steps, flush=False)
            r["decode_us_warm_l2"] = statistics.median(tw) * 1e6
            # the shared-prefix path: the 16 common blocks read once per KV head
            P = case.shared_prefix_blocks
            sws = pa.alloc_shared_prefix_workspace(b.q, case.num_kv_heads, b.mcl, case.block_size, P)

            def shared():
                pa.pa_decode_shared_prefix(b.out, b.q, b.k_cache, b.v_cache, b.bt, b.ctx, b.mcl, case.softmax_scale,
                                           P, sws)

            sh_replay, _g3 = capture(shared)
            timer.run([sh_replay], 5)
            (ts,) = timer.run([sh_replay], steps)
            tsm = statistics.median(ts)
            r["shared_prefix_path"] = {
                "decode_us": tsm * 1e6, "tokens_per_s": case.batch / tsm,
                "kv_gbps_unique": case.kv_bytes_unique() / tsm / 1e9,
                "roofline": {"bound": "hbm", "achieved": uniq / tsm / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": uniq / tsm / 1e9 / pk["hbm_gbs"], "bytes": "unique"}}
        out[name] = r
        del b, dec_replay, _g
        torch.cuda.empty_cache()
    if "block_size_sweep" in names:
        out["block_size_sweep"] = block_size_sweep(device, pk, timer, steps)
    if "mixed_batch" in names:
        out["mixed_batch"] = mixed_batch(device, timer, steps)
    if "varlen_prefill" not in names:
        return out
    case = get_case("varlen_prefill")
    dev = device
    kc, vc = case.k_cache.to(dev), case.v_cache.to(dev)
    kn, vn, q = case.k_new.to(dev), case.v_new.to(dev), case.q.to(dev)
    slot = torch.as_tensor(case.slot_mapping).to(dev)
    bt = torch.as_tensor(case.block_table).to(dev)
    cq = torch.as_tensor(case.cu_seqlens_q).to(dev)
    ck = torch.as_tensor(case.cu_seqlens_k).to(dev)
    o = torch.empty_like(q)
    pws = pa.alloc_prefill_workspace(q, case.num_kv_heads, case.batch, case.max_seqlen_q)

    def st():
        pa.pa_store_kv(kn, vn, slot, kc, vc)

    def pf():
        pa.pa_prefill_varlen(o, q, kc, vc, cq, ck, case.max_seqlen_q, case.max_seqlen_k, bt, case.softmax_scale,
                             workspace=pws)

    def fused():
        pa.pa_store_kv_prefill_varlen(kn, vn, slot, o, q, kc, vc, cq, ck, case.max_seqlen_q, case.max_seqlen_k, bt,
                                      case.softmax_scale, workspace=pws)

    st_replay, _g1 = capture(st)
    pf_replay, _g2 = capture(pf)
    fu_replay, _g3 = capture(fused)
    timer.run([st_replay, pf_replay], 5)
    ts, tp = timer.run([st_replay, pf_replay], steps)
    tpm, tsm = statistics.median(tp), statistics.median(ts)
    timer.run([fu_replay], 5)
    (tf,) = timer.run([fu_replay], steps)
    tfm = statistics.median(tf)
    fl = case.causal_flops()
    ach = fl / tpm / 1e12
    store_bytes = 2 * 2 * kn.numel() * 2
    out["varlen_prefill"] = {
        "prefill_us": tpm * 1e6, "store_us": tsm * 1e6, "causal_tflop": fl / 1e12,
        "store_prefill_fused_us": tfm * 1e6, "store_prefill_fused_tflops": fl / tfm / 1e12,
        "tflops": ach, "new_tokens": case.total_q, "prefill_tokens_per_s": case.total_q / (tpm + tsm),
        "store_gbps": store_bytes / tsm / 1e9,
        "roofline": {"kernel": "prefill_kernel<128, 0, 0>", "bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                     "frac_of_sustained": ach / pk["bf16_tflops_sustained"],
                     "traffic": recorded_traffic("prefill_varlen")},
    }
    return out


def mixed_batch(device, timer, steps):
    """A step that mixes 64 decode rows (one new token after 512..4096 cached tokens) with 4 prompts of
    512 new tokens, Qwen3-class heads (32 q / 8 kv, D 128, B 256): the whole batch through the prefill
    kernel (pa_prefill_varlen) against the one-token rows routed to the decode kernel
    (pa_prefill_varlen_mixed).  The store of the step's rows is done before, outside the timing."""
    import paged_kv_cache_325_b200 as pa
    from paged_kv_cache_325_b200 import workloads as W
    rng = np.random.Generator(np.random.PCG64(1006))
    blocks = rng.integers(2, 17, size=64)
    L = [int(b) * 256 + 1 for b in blocks] + [512] * 4
    c = [int(b) * 256 for b in blocks] + [0] * 4
    case = W.make_prefill_case(L, c, 32, 8, 128, 256, seed=2006, poison=False, keep_contiguous=False)
    dev = device
    kc, vc, q = case.k_cache.to(dev), case.v_cache.to(dev), case.q.to(dev)
    bt = torch.as_tensor(case.block_table).to(dev)
    cq = torch.as_tensor(case.cu_seqlens_q).to(dev)
    ck = torch.as_tensor(case.cu_seqlens_k).to(dev)
    o = torch.empty_like(q)
    pa.pa_store_kv(case.k_new.to(dev), case.v_new.to(dev), torch.as_tensor(case.slot_mapping).to(dev), kc, vc)
    pws = pa.alloc_prefill_workspace(q, 8, case.batch, case.max_seqlen_q)
    mws = pa.alloc_mixed_workspace(q, 8, case.batch, case.max_seqlen_q, case.max_seqlen_k)

    def pf():
        pa.pa_prefill_varlen(o, q, kc, vc, cq, ck, case.max_seqlen_q, case.max_seqlen_k, bt, case.softmax_scale,
                             workspace=pws)

    def mx():
        pa.pa_prefill_varlen_mixed(o, q, kc, vc, cq, ck, case.max_seqlen_q, case.max_seqlen_k, bt,
                                   case.softmax_scale, workspace=mws)

    r1, _g1 = capture(pf)
    r2, _g2 = capture(mx)
    timer.run([r1, r2], 5)
    t1, t2 = timer.run([r1, r2], steps)
    del r1, r2, _g1, _g2
    return {"decode_rows": 64, "prompt_tokens": 4 * 512, "prefill_kernel_only_us": statistics.median(t1) * 1e6,
            "routed_us": statistics.median(t2) * 1e6}


def block_size_sweep(device, pk, timer, steps):
    """Decode (Qwen3-0.6B-like shape) and varlen prefill at several block sizes: the same token
    counts, more and smaller pages (more block-table reads, smaller TMA boxes)."""
    import paged_kv_cache_325_b200 as pa
    from paged_kv_cache_325_b200 import workloads as W
    res = {"decode": {}, "prefill": {}}
    ctx = np.random.Generator(np.random.PCG64(1002)).integers(100, 1025, size=64).astype(np.int32)
    for B in (16, 32, 64, 128, 256):
        case = W.make_decode_case(ctx, 16, 8, 128, B, seed=2002, poison=False, keep_contiguous=False)
        b = DecodeBench(case, device)
        b.store()
        rep, _g = capture(b.decode)
        timer.run([rep], 5)
        (t,) = timer.run([rep], steps)
        tm = statistics.median(t)
        res["decode"][str(B)] = {"decode_us": tm * 1e6, "kv_gbps": case.kv_bytes_read() / tm / 1e9,
                                 "frac": b.alg_bytes_decode() / tm / 1e9 / pk["hbm_gbs"]}
        del b, rep, _g
    base = get_case("varlen_prefill")
    for B in (16, 32, 64, 128, 256):
        c = W.make_prefill_case(base.prompt_lens, base.cached_lens, 32, 8, 128, B, seed=2005, poison=False,
                                keep_contiguous=False)
        kc, vc = c.k_cache.to(device), c.v_cache.to(device)
        q = c.q.to(device)
        o = torch.empty_like(q)
        args = [torch.as_tensor(x).to(device) for x in (c.cu_seqlens_q, c.cu_seqlens_k, c.block_table)]
        ws = pa.alloc_prefill_workspace(q, 8, c.batch, c.max_seqlen_q)
        pa.pa_store_kv(c.k_new.to(device), c.v_new.to(device), torch.as_tensor(c.slot_mapping).to(device), kc, vc)

        def pf():
            pa.pa_prefill_varlen(o, q, kc, vc, args[0], args[1], c.max_seqlen_q, c.max_seqlen_k, args[2],
                                 c.softmax_scale, workspace=ws)

        rep, _g = capture(pf)
        timer.run([rep], 5)
        (t,) = timer.run([rep], steps)
        tm = statistics.median(t)
        res["prefill"][str(B)] = {"prefill_us": tm * 1e6, "tflops": c.causal_flops() / tm / 1e12}
        del rep, _g
    torch.cuda.empty_cache()
    return res


def local_gpu_index(device):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    idx = device.index or 0
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if idx < len(ids) and ids[idx].isdigit():
            return int(ids[idx])
    return idx


# ------------------------------------------------------------ CPU oracle --

def _median_s(fn, reps=3):
    """Wall-clock median of `reps` calls of fn (seconds)."""
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t0)
    return statistics.median(ts)


def oracle_store_s(case, reps=3):
    """Wall-clock median of the oracle's row scatter of the step's new K/V rows, written in place into a
    copy of the cache made once outside the timing (the rows it writes are the same every call)."""
    import oracle
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    return _median_s(lambda: oracle.store_inplace(case.k_new, case.v_new, case.slot_mapping, kc, vc), reps)


def oracle_decode_s(case, seqs=None, reps=3):
    """Wall-clock median of the oracle's decode of the given sequences (every q-head; all when None),
    on the cache after the step's store (done once, outside the timing)."""
    import oracle
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    oracle.store_inplace(case.k_new, case.v_new, case.slot_mapping, kc, vc)
    if seqs is None:
        call = lambda: oracle.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale)
    else:
        si = np.repeat(np.asarray(seqs), case.num_q_heads)
        hi = np.tile(np.arange(case.num_q_heads), len(seqs))
        call = lambda: oracle.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale,
                                     seq_idx=si, head_idx=hi)
    return _median_s(call, reps)


def cpu_baseline(names, rows_frac_prefill=1.0 / 8):
    """The fp64 CPU oracle as it stands, timed per workload and per call (store, decode, prefill) on this
    host's cores: wall-clock median of 3 calls each.  Every decode call covers the whole batch; the
    prefill is timed on a random 1/8 of its (token, head) rows and extrapolated to all of them (its cost
    per row is what the row's key count makes it, and the sample is uniform over rows)."""
    import oracle
    res = {}
    case = get_case(PRIMARY)
    st, dec = oracle_store_s(case), oracle_decode_s(case)
    res[PRIMARY] = {"store_s": st, "decode_s": dec, "tokens_per_s": case.batch / (st + dec),
                    "kv_gbps": case.kv_bytes_read() / dec / 1e9, "sample": "whole batch"}
    case = get_case("tiny_decode")
    st, dec = oracle_store_s(case), oracle_decode_s(case)
    res["tiny_decode"] = {"store_s": st, "decode_s": dec, "tokens_per_s": case.batch / (st + dec),
                          "sample": "whole batch"}
    for name in [n for n in ("long_context_decode", "prefix_sharing_decode") if n in names]:
        case = get_case(name)
        st, dec = oracle_store_s(case), oracle_decode_s(case)
        res[name] = {"store_s": st, "decode_s": dec, "tokens_per_s": case.batch / dec,
                     "kv_gbps": case.kv_bytes_read() / dec / 1e9, "sample": "whole batch"}
    if "varlen_prefill" in names:
        case = get_case("varlen_prefill")
        st = oracle_store_s(case)
        kc, vc = case.k_cache.clone(), case.v_cache.clone()
        oracle.store_inplace(case.k_new, case.v_new, case.slot_mapping, kc, vc)
        rng = np.random.default_rng(0)
        nrows = case.total_q * case.num_q_heads
        pick = rng.choice(nrows, size=max(1, int(nrows * rows_frac_prefill)), replace=False)
        ti, hi = pick // case.num_q_heads, pick % case.num_q_heads
        t = _median_s(lambda: oracle.prefill(case.q, kc, vc, case.cu_seqlens_q, case.cu_seqlens_k,
                                             case.block_table, case.softmax_scale, tok_idx=ti, head_idx=hi))
        full = t * nrows / len(pick)
        res["varlen_prefill"] = {"store_s": st, "store_rows": int(case.total_q),
                                 "prefill_s_sample": t, "prefill_s_extrapolated": full,
                                 "tflops": case.causal_flops() / full / 1e12,
                                 "sample": f"{len(pick)} of {nrows} (token, head) rows, uniformly at random; "
                                           f"time x {nrows / len(pick):.2f}"}
    p = res[PRIMARY]
    return {"value": p["tokens_per_s"], "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"{PRIMARY}: oracle store of the 64 new rows (in place) + fp64 decode of all 64 "
                       f"sequences x 16 q-heads, wall-clock median of 3; per_config: every other workload, "
                       f"median of 3 per call"),
            "per_config": res}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle as it stands, a bounded sample per step (rank 0 only): the
    store of the step's 64 new rows (in place) and the fp64 decode of a random subset of sequences."""
    if rank != 0:
        return
    import oracle
    case = get_case(PRIMARY)
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    rng = np.random.default_rng(0)

    def step(n_seq):
        seqs = rng.choice(case.batch, size=n_seq, replace=False)
        si = np.repeat(seqs, case.num_q_heads)
        hi = np.tile(np.arange(case.num_q_heads), n_seq)
        t0 = time.perf_counter()
        oracle.store_inplace(case.k_new, case.v_new, case.slot_mapping, kc, vc)
        oracle.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale,
                      seq_idx=si, head_idx=hi)
        return time.perf_counter() - t0

    t1 = step(1)
    per_step_budget = 90.0 / max(1, args.steps + args.warmup)
    n_seq = int(max(1, min(case.batch, per_step_budget / max(t1, 1e-3))))
    for _ in range(args.warmup):
        step(n_seq)
    ts = [step(n_seq) for _ in range(args.steps)]
    value = n_seq * args.steps / sum(ts)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(ts) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PRIMARY_DESC, "parallelism": "replicas", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"per step: oracle store of the 64 new rows (in place) + fp64 decode of "
                                       f"{n_seq} random sequences x 16 heads of the {PRIMARY} workload"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main --

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--secondary",
                    default="long_context_decode,prefix_sharing_decode,varlen_prefill,mixed_batch,block_size_sweep",
                    help="comma list of extra workloads to time at N=1 ('none' for none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--secondary-steps", type=int, default=SECONDARY_STEPS,
                    help="timed runs per secondary measurement (median reported)")
    ap.add_argument("--secondary-only", action="store_true",
                    help="time only the --secondary workloads (no primary line; for profiling one workload)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return 0

    import paged_kv_cache_325_b200 as pa
    pa.load_library()            # fails loudly when the CUDA library is missing
    if not torch.cuda.is_available():
        raise SystemExit("no CUDA device: the native arm has no CPU path")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    pk, peak_src = peaks()
    if args.secondary_only:
        if world != 1:
            raise SystemExit("--secondary-only runs on one GPU")
        names = [n for n in args.secondary.split(",") if n and n != "none"]
        print(json.dumps({"secondary_only": True, "peak_source": peak_src,
                          "workloads": bench_secondary(args, device, pk, names)}), flush=True)
        return 0
    try:
        case, res = bench_primary(args, world, rank, device, pk)
        secondary = None
        names = [n for n in args.secondary.split(",") if n and n != "none"]
        if world == 1 and names:
            secondary = bench_secondary(args, device, pk, names)
        cpu = None
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(names)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    if rank != 0:
        return 0
    rf = res["roofline"]
    rf["peak_source"] = peak_src
    line = {
        "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": PRIMARY_DESC, "parallelism": f"replicas x{world}",
                   "l2": "flushed between timed steps (256 MiB write)",
                   "timing": "per-step CUDA events around a CUDA-graph replay of pa_store_kv_decode"},
        "kv_gbps": res["kv_gbps"], "kv_hbm_frac_of_measured": res["kv_hbm_frac_of_measured"],
        "kv_hbm_frac_of_8tbs": res["kv_hbm_frac_of_8tbs"], "store_decode_us": res["store_decode_us"],
        "separate_launches": res.get("separate_launches"), "roofline": rf, "cpu_baseline": cpu, "e2e": res["e2e"],
        "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
    }
    if secondary is not None:
        line["workloads"] = secondary
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
