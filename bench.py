"""Benchmark of the HGA routed-attention hot path on B200.

One step = one pass of the whole path over the query segment of the
Qwen3-30B-A3B-shaped 64K workload (32 query heads, 4 KV heads, d=128, bf16,
last 2048 of 65536 tokens as 32 query blocks, sink 64, local 512, top-32
chunks then top-64 groups): summaries of the segment's chunks/groups, chunk
routing, group routing and gathered exact-token attention.  The 64K history
(K/V and its summaries) is committed once before timing, like a KV cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hga|reference]

Prints one JSON line (rank 0).  N > 1 runs independent replicas, one per GPU
(the path has no exchange step), timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import hga_inputs as gi  # noqa: E402

METRIC = "routed-attn query tokens/s @64K ctx; % of HBM/tensor roofline"
UNIT = "query tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


ATTEND_SOURCES = ("attend_tc.cuh", "tc.cuh", "common.cuh")


def profiled_traffic(workload: str, kernel: str = "attend_tc", sources=ATTEND_SOURCES):
    """DRAM bytes per launch from the committed ncu summary of `kernel` on
    `workload`, or None when there is none or the kernel's sources changed
    since the counters were taken (the summary records their sha256)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith(" "):
                key, _, val = line.partition(":")
                fields[key.strip()] = val.strip()
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "long_context_hga_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if fields.get("kernel_sources_sha256") != h.hexdigest():
        return None
    try:
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- dist

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"hga_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload

def algorithmic_counts(w: gi.Workload, group_cnt: np.ndarray):
    """Exact algorithmic work of one pass from the routed counts.
    attention flops: 4*d per (query row, attended token), causal-exact;
    routing flops: 2*d per (query row, candidate summary);
    attention bytes: Q + O once, plus the routed K/V working set per
    (block, KV head), plus summaries read."""
    d, G, B, g, C = w.head_dim, w.G, w.qblock, w.group, w.chunk
    nb = -(-w.Tq // B)
    att_pairs = 0
    ws_tokens = 0
    route_chunk_pairs = 0
    route_group_pairs = 0
    for b in range(nb):
        b0 = w.q0 + b * B
        b1 = min(b0 + B, w.T)
        sink = min(w.sink, b0)
        loc = b0 - max(sink, b0 - w.local)
        hi = (b0 - w.local) // C if b0 - w.local > 0 else 0
        n_cand = max(0, hi - w.sink // C)
        kc = n_cand if w.top_chunks <= 0 else min(w.top_chunks, n_cand)
        for h in range(w.n_kv_heads):
            routed = int(group_cnt[h, b]) * g
            hist = sink + routed + loc
            for pos in range(b0, b1):
                att_pairs += G * (hist + pos - b0 + 1)
            ws_tokens += hist + (b1 - b0)
            route_chunk_pairs += (b1 - b0) * G * n_cand
            route_group_pairs += (b1 - b0) * G * kc * (C // g)
    esz = 2 if w.dtype == "bf16" else 4
    att_flops = 4 * d * att_pairs
    att_bytes = (2 * w.Tq * w.n_q_heads * d + ws_tokens * 2 * d) * esz
    return {"attn_flops": att_flops, "attn_bytes": att_bytes,
            "route_chunk_flops": 2 * d * route_chunk_pairs,
            "route_group_flops": 2 * d * route_group_pairs,
            "density": att_pairs / (G * w.n_kv_heads * sum(
                p + 1 for p in range(w.q0, w.T)))}


def dense_causal_flops(w) -> float:
    """4*d flops per (query row, attended key) of dense causal attention with
    the causal diagonal aligned to the end of the context (bottom right)."""
    keys = sum(p + 1 for p in range(w.q0, w.T))
    return 4.0 * w.head_dim * w.n_q_heads * keys


def _time_fn(f, steps):
    f()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        f()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def dense_candidates(w, q, k, v, steps=5):
    """Same-shape dense causal attention (bf16, GQA, the causal diagonal at the
    end of the context), timed on every library kernel that accepts it: torch
    SDPA with each backend forced in turn, and the flash_attn package.  Returns
    {name: ms} for the ones that ran (errors as strings)."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    from torch.nn.attention.bias import causal_lower_right
    out = {}
    qt = q.permute(1, 0, 2).unsqueeze(0)                    # [1][Hq][Tq][d]
    kt = k[:, :w.T].unsqueeze(0)
    vt = v[:, :w.T].unsqueeze(0)
    mask = causal_lower_right(w.Tq, w.T)
    for name, be in (("torch_sdpa_cudnn", SDPBackend.CUDNN_ATTENTION),
                     ("torch_sdpa_flash", SDPBackend.FLASH_ATTENTION),
                     ("torch_sdpa_efficient", SDPBackend.EFFICIENT_ATTENTION)):
        def f(be=be):
            with sdpa_kernel([be]):
                if w.q0 == 0:
                    return torch.nn.functional.scaled_dot_product_attention(
                        qt, kt, vt, is_causal=True, enable_gqa=True)
                return torch.nn.functional.scaled_dot_product_attention(
                    qt, kt, vt, attn_mask=mask, enable_gqa=True)
        try:
            out[name] = _time_fn(f, steps)
        except Exception as exc:
            out[name] = f"error: {str(exc).splitlines()[0][:120]}"
    try:
        from flash_attn import flash_attn_func              # bottom-right causal, native GQA
        qf = q.unsqueeze(0)                                 # [1][Tq][Hq][d]
        kf = k[:, :w.T].permute(1, 0, 2).unsqueeze(0).contiguous()
        vf = v[:, :w.T].permute(1, 0, 2).unsqueeze(0).contiguous()
        out["flash_attn"] = _time_fn(lambda: flash_attn_func(qf, kf, vf, causal=True), steps)
    except Exception as exc:
        out["flash_attn"] = f"error: {str(exc).splitlines()[0][:120]}"
    return out


def dense_sdpa_time(w, q, k, v, steps=5):
    """The fastest dense candidate: (ms, name, {name: ms or error})."""
    cands = dense_candidates(w, q, k, v, steps)
    ok = {n: t for n, t in cands.items() if isinstance(t, float)}
    if not ok:
        raise RuntimeError(f"no dense kernel ran: {cands}")
    best = min(ok, key=ok.get)
    return ok[best], best, cands


def cpu_baseline(w: gi.Workload, inp: gi.Inputs, budget_s: float = 15.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    the workload's (block, KV head) units (plus the summaries it needs)."""
    from oracle import hga_oracle as ho
    p = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group,
                  w.qblock, w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    q = gi.to_f64(inp.q)
    k = gi.to_f64(inp.k)
    v = gi.to_f64(inp.v)
    csum, gsum = ho.build_summaries(k, p, 0, w.T)
    t_setup = time.perf_counter() - t0
    nb = -(-w.Tq // w.qblock)
    units = [(b, h) for b in range(nb) for h in range(w.n_kv_heads)]
    done = 0
    t1 = time.perf_counter()
    for (b, h) in units:
        ho.hga_forward(q, k, v, w.q0, p, units=[(b, h)], csum=csum, gsum=gsum)
        done += 1
        if time.perf_counter() - t1 > budget_s:
            break
    dt = time.perf_counter() - t1
    q_tokens = done * w.qblock / w.n_kv_heads     # one unit = 64 positions x 1/Hkv of the heads
    return {"value": q_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} of {len(units)} (block, KV head) units of {w.name} "
                      f"(routing + attention, float64 NumPy); history summaries "
                      f"({t_setup:.1f} s) excluded as commit cost"}


# ---------------------------------------------------------------- main arm

def step_names(args) -> list:
    """The library calls of one step, in launch order."""
    route = ["route"] if args.route == "fused" else ["route_chunks", "route_groups"]
    return ["commit"] + route + ["attend"]


def workload_config(w: gi.Workload, world: int, v16: bool, names) -> dict:
    """The `config` of the JSON line: the workload and how a step is timed
    (the same dict on the GPU arm and the reference arm)."""
    return {"workload": w.name, "T": w.T, "q0": w.q0, "query_tokens": w.Tq,
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "head_dim": w.head_dim,
            "routing": f"chunk {w.chunk}, group {w.group}, sink {w.sink}, "
                       f"local {w.local}, top {w.top_chunks} chunks / "
                       f"{w.top_groups} groups",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every step, outside the events: 256 MiB "
                  "written, then another 256 MiB read (no dirty lines left)",
            "v_storage": ("fp16 (history converted at commit; the segment's "
                          "V converted inside every step)" if v16 else
                          "bf16 (converted per tile on chip)"),
            "timing": f"step: one CUDA graph of the {len(names)} calls "
                      f"({', '.join(names)}) between two event nodes; "
                      "kernel_us: a second graph with an event node between "
                      "every two kernels"}


def run_hga(args, world, rank, local):
    from long_context_hga_b200 import hga
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = gi.WORKLOADS[args.workload]
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    q = inp.q.to(dev)
    k = inp.k.to(dev)
    v = inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    stream = torch.cuda.current_stream()
    # V storage: fp16 (converted once per token as it is committed; the
    # segment's own tokens are converted inside every step) or bf16 (each
    # attention tile is converted on chip)
    v16 = args.v_storage == "f16"
    # q_ready: the routing and attention calls below each follow one of the
    # library's own kernels in the stream (the step starts with commit), and
    # those let the next kernel start only after their own wait, so q is
    # complete by then and may be requested before that wait
    pq = dataclasses.replace(p, q_ready=True)
    p_att = dataclasses.replace(pq, v_f16=True) if v16 else pq
    v_att = torch.empty(v.shape, dtype=torch.float16, device=dev) if v16 else v
    # commit the history once (setup, not timed)
    hga.commit(p, k, v, 0, w.q0, bufs.chunk_sum, bufs.group_sum, v_att if v16 else None)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    # commit of the segment: its summaries and (fp16 V storage) its V in fp16,
    # one launch
    calls = [
        ("commit",
         lambda: hga.commit(p, k, v, w.q0, w.T, bufs.chunk_sum, bufs.group_sum,
                            v_att if v16 else None)),
    ] + ([
        ("route",
         lambda: hga.route(pq, q, w.q0, bufs.chunk_sum, bufs.group_sum, w.T, bufs.chunk_idx,
                           bufs.chunk_cnt, bufs.group_idx, bufs.group_cnt)),
    ] if args.route == "fused" else [
        ("route_chunks",
         lambda: hga.route_chunks(pq, q, w.q0, bufs.chunk_sum, w.T, bufs.chunk_idx,
                                  bufs.chunk_cnt)),
        ("route_groups",
         lambda: hga.route_groups(pq, q, w.q0, bufs.group_sum, w.T, bufs.chunk_idx,
                                  bufs.chunk_cnt, bufs.group_idx, bufs.group_cnt)),
    ]) + [
        ("attend",
         lambda: hga.attend(p_att, q, w.q0, k, v_att, bufs.group_idx, bufs.group_cnt, bufs.o,
                            bufs.lse)),
    ]
    names = [n for n, _ in calls]

    def step():
        for _, call in calls:
            call()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert hga.check() == 0
    counts = algorithmic_counts(w, bufs.group_cnt.cpu().numpy())

    # Two CUDA graphs of one step.  `whole` has event nodes only at its two
    # ends: the step time, with the kernels back to back and each launch
    # overlapping the previous kernel's tail.  `split` has an event node
    # between every two kernels: the per-kernel device times.
    n_kern = len(calls)
    ev_w = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_kern + 1)]
    whole, split = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    launches_cap0 = hga.launch_count()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(whole, stream=cap):
            ev_w[0].record()
            step()
            ev_w[1].record()
    launches_per_step = hga.launch_count() - launches_cap0
    with torch.cuda.stream(cap):
        with torch.cuda.graph(split, stream=cap):
            ev[0].record()
            for j, (_, call) in enumerate(calls):
                call()
                ev[j + 1].record()
    stream.wait_stream(cap)
    torch.cuda.synchronize()

    def replay_for(seconds):
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            for _ in range(20):
                whole.replay()
            torch.cuda.synchronize()

    def cold_l2():
        # outside the events: evict the step's data, then replace the dirty
        # lines of the write with clean ones so that no write-back of the
        # flush lands inside the timed step
        flush.zero_()
        torch.sum(flush_rd, 0, out=flush_sink)

    clocks = ClockSampler(local)
    clocks.start()
    replay_for(args.clock_window)          # load before the timed region (clock samples)
    step_ms = np.zeros(args.steps)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        cold_l2()
        whole.replay()
        torch.cuda.synchronize()
        step_ms[i] = ev_w[0].elapsed_time(ev_w[1])
    torch.cuda.synchronize()
    barrier(world)
    t_wall = time.perf_counter() - t_wall0
    per_kernel = np.zeros((args.steps, n_kern))
    for i in range(args.steps):
        cold_l2()
        split.replay()
        torch.cuda.synchronize()
        per_kernel[i] = [ev[j].elapsed_time(ev[j + 1]) for j in range(n_kern)]   # ms
    replay_for(args.clock_window)          # load after the timed region
    clk = clocks.stop()
    launches = launches_per_step * args.steps
    ms_local = float(step_ms.mean())
    ms = max_over_ranks(ms_local, world, dev)
    assert hga.check() == 0

    # end-to-end through the public API with host buffers: every step copies
    # its Q and the segment's K/V in from pinned host memory and reads its O
    # back.  As a serving loop would, the copies run on their own streams and
    # overlap the neighbouring steps' compute: two device state sets (K/V
    # caches with the committed history, summaries, index lists, O)
    # alternate, and events order each set's uses.
    q_h = inp.q.pin_memory()
    kseg_h = inp.k[:, w.q0:].contiguous().pin_memory()
    vseg_h = inp.v[:, w.q0:].contiguous().pin_memory()
    o_h = [torch.empty(bufs.o.shape, dtype=bufs.o.dtype).pin_memory() for _ in range(2)]
    sets = []
    for _ in range(2):
        bb = hga.allocate(p, w.T, w.Tq, device=dev)
        bb.chunk_sum.copy_(bufs.chunk_sum)
        bb.group_sum.copy_(bufs.group_sum)
        kb, vb = k.clone(), v.clone()
        sets.append((torch.empty_like(q), kb, vb, v_att.clone() if v16 else vb, bb))
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        x = i % 2
        q_d, kb, vb, vab, bb = sets[x]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[x])          # step i-2 has consumed this set
            q_d.copy_(q_h, non_blocking=True)
            kb[:, w.q0:].copy_(kseg_h, non_blocking=True)
            vb[:, w.q0:].copy_(vseg_h, non_blocking=True)
            ev_in[x].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[x])
            if i >= 2:
                s_cmp.wait_event(ev_out[x])         # step i-2's O has been read back
            hga.commit(p, kb, vb, w.q0, w.T, bb.chunk_sum, bb.group_sum, vab if v16 else None)
            hga.route_chunks(pq, q_d, w.q0, bb.chunk_sum, w.T, bb.chunk_idx, bb.chunk_cnt)
            hga.route_groups(pq, q_d, w.q0, bb.group_sum, w.T, bb.chunk_idx, bb.chunk_cnt,
                             bb.group_idx, bb.group_cnt)
            hga.attend(p_att, q_d, w.q0, kb, vab, bb.group_idx, bb.group_cnt, bb.o, bb.lse)
            ev_cmp[x].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[x])
            o_h[x].copy_(bb.o, non_blocking=True)
            ev_out[x].record(s_out)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(6, args.steps)
    es.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    ee.record(s_out)
    torch.cuda.synchronize()
    assert hga.check() == 0
    e2e_ms = max_over_ranks(es.elapsed_time(ee) / e2e_steps, world, dev)
    # the read-back O equals the device-timed step's O (same inputs, same kernels)
    e2e_same = bool(torch.equal(o_h[(e2e_steps - 1) % 2], bufs.o.cpu()))
    h2d = q_h.numel() * q_h.element_size() + 2 * kseg_h.numel() * kseg_h.element_size()
    d2h = o_h[0].numel() * o_h[0].element_size()
    del sets

    dense_ms, dense_name, dense_all = None, None, None
    if not args.no_dense:
        try:
            dense_ms, dense_name, dense_all = dense_sdpa_time(w, q, k, v)
        except Exception as exc:  # comparator only
            print(f"dense comparator failed: {exc}", file=sys.stderr)

    peaks, peak_kind = load_peaks()
    col = {n: j for j, n in enumerate(names)}
    att_ms = float(per_kernel[:, col["attend"]].mean())
    att_tflops = counts["attn_flops"] / (att_ms * 1e-3) / 1e12
    peak_tf = peaks["bf16_tflops"]
    out = None
    if rank == 0:
        n_tok = w.Tq * world
        value = n_tok / (ms * 1e-3)
        kernels = {name: round(float(per_kernel[:, j].mean()) * 1e3, 2)
                   for j, name in enumerate(names)}
        # information, not a target: planted needle groups the routing kept for
        # the block each was planted for (read after the timed region)
        g_idx, g_cnt = bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy()
        found = sum(int(j in g_idx[h, b, :g_cnt[h, b]]) for (h, j, b) in inp.needles)
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) Q/K/V, RoPE, planted needles)",
            "config": workload_config(w, world, v16, names),
            "kernel_us": kernels,
            "kernel_sum_us": round(float(per_kernel.sum(axis=1).mean()) * 1e3, 2),
            "attn_tflops": att_tflops,
            "route_tflops": (counts["route_chunk_flops"] + counts["route_group_flops"]) /
                            (float(sum(per_kernel[:, col[n]] for n in col if n.startswith("route")).mean())
                             * 1e-3) / 1e12,
            "density": counts["density"],
            "step_ms_percentiles": {k_: float(np.percentile(step_ms, q_))
                                    for k_, q_ in (("p10", 10), ("p50", 50), ("p90", 90))},
            "needle_recall": {"found": found, "planted": len(inp.needles),
                              "recall": found / max(1, len(inp.needles))},
            "roofline": {"bound": "tensor", "kernel": "hga_attend",
                         "achieved": att_tflops, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": att_tflops / peak_tf,
                         "traffic": profiled_traffic(w.name),
                         "peak_source": f"{peak_kind} bf16 burst",
                         "algorithmic_flops": counts["attn_flops"],
                         "algorithmic_bytes": counts["attn_bytes"],
                         "hbm_frac": counts["attn_bytes"] / (att_ms * 1e-3) / 1e9 /
                                     peaks["hbm_gbs"]},
            "e2e": {"value": n_tok / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "output_matches_device_step": e2e_same,
                    "pipeline": "per step: pinned H2D of Q and the segment's K/V, "
                                "commit, route_chunks, route_groups, attend, D2H of O; "
                                "copies on their own "
                                "streams overlap the neighbouring steps (2 state sets)"},
            "gpu_launches": int(launches),
            "clocks": clk,
            "dense_sdpa": None if dense_ms is None else {
                "value": w.Tq / (dense_ms * 1e-3), "unit": UNIT, "ms": dense_ms,
                "kernel": dense_name,
                "tflops": dense_causal_flops(w) / (dense_ms * 1e-3) / 1e12,
                "candidates_ms": dense_all},
            "wall_s_timed_region": t_wall,
        }
    return out, w, inp


# ---------------------------------------------------------------- other configs

def _time_graph(fn, steps, warmup, flush_w, flush_r, sink):
    """Device time of fn() as one CUDA graph, cold L2 before each replay."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            e0.record()
            fn()
            e1.record()
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush_w.zero_()
        torch.sum(flush_r, 0, out=sink)
        g.replay()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    del g
    return float(np.mean(ts))


def measure_config(w, args, dev, flush_w, flush_r, sink, dense=True, inp=None):
    """Whole-step throughput of one workload (inputs resident), with the same
    step as the headline line: commit of the segment (summaries, and V to
    fp16 for bf16 workloads, one launch), chunk and group routing, attention."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = inp if inp is not None else gi.make_inputs(w)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    v16 = w.dtype == "bf16"
    p_att = dataclasses.replace(p, v_f16=True) if v16 else p
    v_att = torch.empty(v.shape, dtype=torch.float16, device=dev) if v16 else v
    if w.q0 > 0:
        hga.commit(p, k, v, 0, w.q0, bufs.chunk_sum, bufs.group_sum, v_att if v16 else None)

    def step():
        hga.commit(p, k, v, w.q0, w.T, bufs.chunk_sum, bufs.group_sum, v_att if v16 else None)
        hga.route_chunks(p, q, w.q0, bufs.chunk_sum, w.T, bufs.chunk_idx, bufs.chunk_cnt)
        hga.route_groups(p, q, w.q0, bufs.group_sum, w.T, bufs.chunk_idx, bufs.chunk_cnt,
                         bufs.group_idx, bufs.group_cnt)
        hga.attend(p_att, q, w.q0, k, v_att, bufs.group_idx, bufs.group_cnt, bufs.o, bufs.lse)

    ms = _time_graph(step, 10, 3, flush_w, flush_r, sink)
    assert hga.check() == 0
    counts = algorithmic_counts(w, bufs.group_cnt.cpu().numpy())
    peaks, kind = load_peaks()
    flops = counts["attn_flops"] + counts["route_chunk_flops"] + counts["route_group_flops"]
    out = {"workload": w.name, "T": w.T, "query_tokens": w.Tq, "dtype": w.dtype,
           "top_chunks": w.top_chunks, "top_groups": w.top_groups,
           "ms_per_step": ms, "query_tokens_per_s": w.Tq / (ms * 1e-3),
           "attended_fraction_of_causal": counts["density"],
           "step_tflops": flops / (ms * 1e-3) / 1e12,
           "step_frac_of_tensor_peak": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "peak_source": f"{kind} bf16 burst"}
    if dense and w.dtype == "bf16":
        try:
            dms, dname, dall = dense_sdpa_time(w, q, k, v)
            out["dense_sdpa"] = {"ms": dms, "query_tokens_per_s": w.Tq / (dms * 1e-3),
                                 "kernel": dname,
                                 "tflops": dense_causal_flops(w) / (dms * 1e-3) / 1e12,
                                 "candidates_ms": dall}
        except Exception as exc:  # comparator only
            out["dense_sdpa"] = {"error": str(exc)[:200]}
    return out, (p, inp, q, k, v, bufs)


def dense_reference_fp32(w, q, k, v, rows=1024):
    """Dense causal attention of the segment in fp32 on the GPU, in slices of
    query rows (a full score matrix of a 32K prefill would not fit)."""
    G, d, Hkv = w.G, w.head_dim, w.n_kv_heads
    out = torch.empty(w.Tq, w.n_q_heads, d, dtype=torch.float32, device=q.device)
    kf, vf = k[:, :w.T].float(), v[:, :w.T].float()
    for r0 in range(0, w.Tq, rows):
        r1 = min(w.Tq, r0 + rows)
        n, last = r1 - r0, w.q0 + r1                 # keys [0, last)
        qh = q[r0:r1].float().view(n, Hkv, G, d).permute(1, 2, 0, 3)
        s = torch.einsum("hgrd,htd->hgrt", qh, kf[:, :last]) / math.sqrt(d)
        pos = w.q0 + torch.arange(r0, r1, device=q.device)
        s.masked_fill_(torch.arange(last, device=q.device)[None, :] > pos[:, None], float("-inf"))
        o = torch.einsum("hgrt,htd->hgrd", torch.softmax(s, dim=-1), vf[:, :last])
        out[r0:r1] = o.permute(2, 0, 1, 3).reshape(n, w.n_q_heads, d)
        del s, o
    return out


def measure_tiered(w, dev, flush_w, flush_r, sink, steps=5):
    """Tiered step of the 128K workload: history K/V and group summaries in
    pinned host memory, an HBM cache for a quarter of the group summaries,
    routed history groups gathered over PCIe on a side stream."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    q = inp.q.to(dev)
    full = hga.allocate(p, w.T, w.Tq, device=dev)
    k_seg = inp.k.to(dev)                      # for the history summaries (commit)
    hga.build_summaries(p, k_seg, 0, w.q0, full.chunk_sum, full.group_sum)
    tier = hga.make_host_tier(p, inp.k.pin_memory(), inp.v.pin_memory(),
                              full.group_sum.cpu().pin_memory(), t_hist=w.q0)
    del k_seg
    k_dev = torch.zeros(w.n_kv_heads, w.T, w.head_dim, dtype=torch.bfloat16, device=dev)
    v_dev = torch.zeros_like(k_dev)
    k_dev[:, w.q0:] = inp.k[:, w.q0:].to(dev)
    v_dev[:, w.q0:] = inp.v[:, w.q0:].to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    bufs.chunk_sum.copy_(full.chunk_sum)
    side = torch.cuda.Stream()
    hga.tiered_step(p, q, w.q0, tier, k_dev, v_dev, bufs, side)    # cold cache
    torch.cuda.synchronize()
    cold = tier.stats.tolist()
    ts = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0 = int(tier.bytes.item())
    for _ in range(steps):
        flush_w.zero_()
        torch.sum(flush_r, 0, out=sink)
        e0.record()
        hga.tiered_step(p, q, w.q0, tier, k_dev, v_dev, bufs, side)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    assert hga.check() == 0
    warm = (tier.stats - torch.tensor(cold, device=tier.stats.device)).tolist()
    ms = float(np.mean(ts))
    return {"workload": w.name, "T": w.T, "query_tokens": w.Tq,
            "ms_per_step": ms, "query_tokens_per_s": w.Tq / (ms * 1e-3),
            "timing": "eager tiered_step between CUDA events (host launch gaps included)",
            "history_on_host": "K/V and group summaries, pinned",
            "group_cache_slots_fraction": 0.25,
            "cold_step_hits_misses": cold,
            "warm_hit_rate": warm[0] / max(1, warm[0] + warm[1]),
            "pcie_bytes_per_step": (int(tier.bytes.item()) - b0) / steps}


def _filesystem_of(path):
    """(mount point, type, device) of the filesystem holding path."""
    best = ("?", "?", "?")
    try:
        real = os.path.realpath(path)
        for line in open("/proc/mounts"):
            dev_, mnt, typ = line.split()[:3]
            if (real == mnt or real.startswith(mnt.rstrip("/") + "/")) and \
                    len(mnt) >= len(best[0].replace("?", "")):
                best = (mnt, typ, dev_)
    except OSError:
        pass
    return {"mount": best[0], "type": best[1], "device": best[2]}


def measure_store(w, dev, cold_steps=3, warm_steps=5, page_tokens=64, io_threads=16):
    """Tiered step of the 128K workload with the history's K/V in a file
    (pages of 64 tokens of one KV head, K then V) read through a page cache
    in pinned RAM bounded to the pages one step needs (found by a first step
    with room for the whole history); group summaries as in the RAM tier.
    Cold steps start with an empty cache and read with O_DIRECT when the
    filesystem allows it (so the OS page cache does not serve them); warm
    steps find every page cached.  Wall-clock per step (the host waits for
    the routing and fills the cache inside the step)."""
    import shutil
    import tempfile
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    q = inp.q.to(dev)
    full = hga.allocate(p, w.T, w.Tq, device=dev)
    k_seg = inp.k.to(dev)
    hga.build_summaries(p, k_seg, 0, w.q0, full.chunk_sum, full.group_sum)
    del k_seg
    tier = hga.make_host_tier(p, None, None, full.group_sum.cpu().pin_memory(), t_hist=w.q0)
    k_dev = torch.zeros(w.n_kv_heads, w.T, w.head_dim, dtype=torch.bfloat16, device=dev)
    v_dev = torch.zeros_like(k_dev)
    k_dev[:, w.q0:] = inp.k[:, w.q0:].to(dev)
    v_dev[:, w.q0:] = inp.v[:, w.q0:].to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    bufs.chunk_sum.copy_(full.chunk_sum)
    tmp = tempfile.mkdtemp(prefix="hga_store_")
    path = os.path.join(tmp, "kv.bin")
    try:
        hist_pages = w.n_kv_heads * (-(-w.q0 // page_tokens))
        direct = True
        try:
            store = hga.KVStore(p, path, w.T, page_tokens, hist_pages, direct=True)
        except hga.HgaError:
            direct = False
            store = hga.KVStore(p, path, w.T, page_tokens, hist_pages, direct=False)
        t0 = time.perf_counter()
        store.append(inp.k[:, :w.q0].contiguous(), inp.v[:, :w.q0].contiguous())
        with open(path, "rb+") as f:
            os.fsync(f.fileno())
        write_s = time.perf_counter() - t0

        def one():
            torch.cuda.synchronize()
            t = time.perf_counter()
            st = hga.store_step(p, q, w.q0, tier, store, k_dev, v_dev, bufs, io_threads)
            torch.cuda.synchronize()
            st["ms"] = (time.perf_counter() - t) * 1e3
            return st

        store.reset_cache()
        cache_pages = one()["pages_needed"]          # probe: the bound for the cache
        cold = []
        for _ in range(cold_steps):
            store.reset_cache(cache_pages)
            cold.append(one())
        warm = [one() for _ in range(warm_steps)]
        assert hga.check() == 0
        # the step's output against the all-HBM path (same inputs, HBM-resident history)
        k_all, v_all = inp.k.to(dev), inp.v.to(dev)
        hga.forward(p, q, w.q0, k_all, v_all, full)
        same = bool(torch.equal(full.o, bufs.o))
        del k_all, v_all
        store.close()
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    med = lambda xs: float(np.median(xs))
    c0 = cold[-1]
    cold_ms = med([c["ms"] for c in cold])
    cold_prep = med([c["prepare_s"] for c in cold])
    return {"workload": w.name, "store": {
        "file": {"bytes": hist_pages * store.page_bytes, "page_bytes": store.page_bytes,
                 "o_direct_reads": direct, "filesystem": _filesystem_of(tmp),
                 "append_and_fsync_s": write_s},
        "cache_pages": cache_pages, "history_pages": hist_pages,
        "io_threads": io_threads,
        "pages_needed_per_step": c0["pages_needed"],
        "cold": {"ms_per_step": cold_ms, "query_tokens_per_s": w.Tq / (cold_ms * 1e-3),
                 "bytes_read": c0["bytes_read"], "prepare_ms": cold_prep * 1e3,
                 "read_GBps": c0["bytes_read"] / max(cold_prep, 1e-9) / 1e9},
        "warm": {"ms_per_step": med([c["ms"] for c in warm]),
                 "query_tokens_per_s": w.Tq / (med([c["ms"] for c in warm]) * 1e-3),
                 "hits": warm[-1]["hits"], "misses": warm[-1]["misses"],
                 "prepare_ms": med([c["prepare_s"] for c in warm]) * 1e3},
        "output_equals_all_hbm_step": same,
        "timing": "wall clock per store_step with a device synchronise on both sides"}}


def measure_all_configs(args, dev):
    """Every other workload, briefly (the headline line times the 64K one)."""
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    res = []
    for w in (gi.TINY_FP32, gi.QWEN3_8B_16K):
        try:
            res.append(measure_config(w, args, dev, flush_w, flush_r, sink)[0])
        except Exception as exc:
            res.append({"workload": w.name, "error": str(exc)[:300]})
    try:
        res.append(measure_tiered(gi.TIERED_128K, dev, flush_w, flush_r, sink))
    except Exception as exc:
        res.append({"workload": gi.TIERED_128K.name, "error": str(exc)[:300]})
    try:
        res.append(measure_store(gi.TIERED_128K, dev))
    except Exception as exc:
        res.append({"workload": gi.TIERED_128K.name, "store": {"error": str(exc)[:300]}})
    # budget sweep at 32K: sparsity vs throughput vs max error against dense
    sweep = []
    dense_o = None
    sweep_inp = gi.make_inputs(gi.SWEEP_32K)        # the budgets do not change the inputs
    for kc in gi.SWEEP_BUDGETS:
        w = gi.SWEEP_32K.with_(top_chunks=kc, top_groups=2 * kc)
        try:
            r, (p, inp, q, k, v, bufs) = measure_config(w, args, dev, flush_w, flush_r, sink,
                                                          dense=dense_o is None, inp=sweep_inp)
            if dense_o is None:
                dense_o = dense_reference_fp32(w, q, k, v)
            err = (bufs.o.float() - dense_o).abs()
            r["max_abs_err_vs_dense"] = float(err.max())
            r["mean_abs_err_vs_dense"] = float(err.mean())
            # elementwise test of the stated tolerance (bf16: 2e-3 + 1e-2 |ref|)
            r["worst_excess_vs_dense"] = float((err - (2e-3 + 1e-2 * dense_o.abs())).max())
            if kc == 0:
                r["all_point_matches_dense"] = r["worst_excess_vs_dense"] <= 0
            sweep.append(r)
            del p, inp, q, k, v, bufs
        except Exception as exc:
            sweep.append({"workload": w.name, "top_chunks": kc, "error": str(exc)[:300]})
    res.append({"workload": gi.SWEEP_32K.name, "budget_sweep": sweep})
    try:
        res.append(measure_decode(gi.QWEN3_30B_64K, dev, flush_w, flush_r, sink))
    except Exception as exc:
        res.append({"workload": gi.QWEN3_30B_64K.name, "decode": {"error": str(exc)[:300]}})
    try:
        res.append(measure_backward(gi.QWEN3_30B_64K, dev, flush_w, flush_r, sink))
    except Exception as exc:
        res.append({"workload": gi.QWEN3_30B_64K.name, "backward": {"error": str(exc)[:300]}})
    try:
        res.append(measure_causal(gi.QWEN3_30B_64K, dev, flush_w, flush_r, sink))
    except Exception as exc:
        res.append({"workload": gi.QWEN3_30B_64K.name,
                    "causal_routing": {"error": str(exc)[:300]}})
    del flush_w, flush_r
    torch.cuda.empty_cache()
    return res


def measure_one(name, args, dev):
    """One per-workload measurement of measure_all_configs, alone."""
    if name == "configs":
        return measure_all_configs(args, dev)
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    if name == "backward":
        return measure_backward(gi.QWEN3_30B_64K, dev, flush_w, flush_r, sink)
    if name == "tiered":
        return measure_tiered(gi.TIERED_128K, dev, flush_w, flush_r, sink)
    if name == "store":
        return measure_store(gi.TIERED_128K, dev)
    if name == "decode":
        return measure_decode(gi.QWEN3_30B_64K, dev, flush_w, flush_r, sink)
    if name == "causal":
        return measure_causal(gi.QWEN3_30B_64K, dev, flush_w, flush_r, sink)
    if name == "sweep":
        inp = gi.make_inputs(gi.SWEEP_32K)
        return [measure_config(gi.SWEEP_32K.with_(top_chunks=kc, top_groups=2 * kc), args, dev,
                               flush_w, flush_r, sink, dense=False, inp=inp)[0]
                for kc in gi.SWEEP_BUDGETS]
    raise ValueError(name)


def measure_decode(w, dev, flush_w, flush_r, sink, n_req=8, reps=6):
    """Generation steps at the 64K context: n_req requests, each with its own
    K/V cache (copies of the 64K workload's inputs), history committed; one
    step decodes the token at the 32nd position of every request's last query
    block (the block's routing recomputed on its 32 queries).  Timed two ways,
    each as one CUDA graph with a cold L2: one hga_decode_step per request,
    and the requests in lockstep as the heads of a single call.  Tokens/s =
    n_req per step.  HBM bytes the method must read per new token: candidate
    chunk summaries, the kept chunks' group summaries and the attended K/V of
    every KV head."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    pos = w.q0 + 31
    reqs = []
    for _ in range(n_req):
        k, v = inp.k.to(dev), inp.v.to(dev)
        q = inp.q[:w.qblock].to(dev)                 # queries of the last block so far
        v16 = torch.empty(v.shape, dtype=torch.float16, device=dev)
        bufs = hga.allocate(p, w.T, p.qblock, device=dev)
        hga.commit(p, k, v, 0, w.q0, bufs.chunk_sum, bufs.group_sum, v16)
        reqs.append((q, k, v, v16, bufs))

    def step():
        for q, k, v, v16, bufs in reqs:
            hga.decode_step(p, q, pos, k, v, bufs, v_f16=v16)

    ms = _time_graph(step, reps, 3, flush_w, flush_r, sink)
    assert hga.check() == 0
    gc = reqs[0][4].group_cnt.cpu().numpy()
    # the same requests in lockstep (one position for all) as extra heads of
    # one call: request r's KV heads are heads r*Hkv .. r*Hkv+Hkv-1 of one
    # cache, its query heads r*Hq .. (r+1)*Hq-1 (units stay independent)
    pb = dataclasses.replace(p, n_q_heads=n_req * p.n_q_heads, n_kv_heads=n_req * p.n_kv_heads)
    kb = torch.cat([r[1] for r in reqs], 0)
    vb = torch.cat([r[2] for r in reqs], 0)
    v16b = torch.empty(vb.shape, dtype=torch.float16, device=dev)
    qb = torch.cat([r[0] for r in reqs], 1).contiguous()
    bb = hga.allocate(pb, w.T, p.qblock, device=dev)
    hga.commit(pb, kb, vb, 0, w.q0, bb.chunk_sum, bb.group_sum, v16b)
    ms_b = _time_graph(lambda: hga.decode_step(pb, qb, pos, kb, vb, bb, v_f16=v16b), reps, 3,
                       flush_w, flush_r, sink)
    assert hga.check() == 0
    o_b = bb.o[pos % p.qblock]
    same = all(torch.equal(o_b[r * p.n_q_heads:(r + 1) * p.n_q_heads],
                           reqs[r][4].o[pos % p.qblock]) for r in range(n_req))
    del kb, vb, v16b, qb, bb
    b0 = pos - pos % p.qblock
    n_cand = max(0, (b0 - w.local) // w.chunk - w.sink // w.chunk)
    kept_chunks = min(w.top_chunks, n_cand) if w.top_chunks > 0 else n_cand
    routed_groups = float(gc.mean())
    per_head = (n_cand * w.head_dim * 2                                   # chunk summaries
                + 8 * kept_chunks * w.head_dim * 2                        # group summaries
                + (w.sink + routed_groups * w.group + w.local + (pos - b0 + 1))
                * w.head_dim * 2 * 2)                                     # attended K and V
    bytes_per_tok = per_head * w.n_kv_heads
    peaks, kind = load_peaks()
    achieved = n_req * bytes_per_tok / (ms * 1e-3) / 1e9
    achieved_b = n_req * bytes_per_tok / (ms_b * 1e-3) / 1e9
    out = {"workload": w.name, "decode": {
        "requests": n_req, "position": pos, "hbm_bytes_per_token": bytes_per_tok,
        "lockstep_as_heads": {
            "ms_per_step": ms_b, "tokens_per_s": n_req / (ms_b * 1e-3),
            "launches_per_step": 4, "outputs_equal_per_request_steps": same,
            "roofline": {"bound": "hbm", "achieved": achieved_b, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved_b / peaks["hbm_gbs"],
                         "peak_source": f"{kind} copy"}},
        "per_request": {
            "ms_per_step": ms, "tokens_per_s": n_req / (ms * 1e-3),
            "launches_per_step": 4 * n_req,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "peak_source": f"{kind} copy"}},
        "form": "hga_decode_step (commit, route chunks, route groups, attend on the "
                "token's block so far); lockstep requests batched as heads of one "
                "call, else one call per request"}}
    return out


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flops x 1965 MHz
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def measure_backward(w, dev, flush_w, flush_r, sink, reps=6):
    """Backward of the gathered attention (routing of the forward held fixed):
    device time of hga_attend_backward on the segment with a cold L2, and its
    algorithmic flops (10 d per (query row, attended token): the S and dP
    products and the dQ, dK, dV accumulations).  bf16 runs on the tensor
    cores (against the bf16 peak); the fp32 CUDA-core kernel (variant 1) is
    timed beside it on the same inputs.  The call also zeroes dK and dV on
    the context's tokens (2 Hkv T d 4 bytes each), timed inside."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
    hga.forward(p, q, w.q0, k, v, bufs)
    g = torch.Generator().manual_seed(17)
    d_o = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    d_q = torch.empty(q.shape, dtype=torch.float32, device=dev)
    d_k = torch.empty(k.shape, dtype=torch.float32, device=dev)
    d_v = torch.empty(v.shape, dtype=torch.float32, device=dev)

    def timed(variant):
        hga.set_kernel_variant(variant)
        try:
            ts = []
            for i in range(reps + 2):
                flush_w.zero_()
                torch.sum(flush_r, 0, out=sink)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                hga.attend_backward(p, q, w.q0, k, v, bufs.group_idx, bufs.group_cnt, bufs.o,
                                    bufs.lse, d_o, d_q, d_k, d_v)
                e1.record()
                torch.cuda.synchronize()
                if i >= 2:
                    ts.append(e0.elapsed_time(e1))
        finally:
            hga.set_kernel_variant(0)
        assert hga.check() == 0
        return float(np.median(ts))

    counts = algorithmic_counts(w, bufs.group_cnt.cpu().numpy())
    flops = counts["attn_flops"] * 10 / 4
    peaks, kind = load_peaks()
    ms = timed(0)
    ms_cc = timed(1) if w.dtype == "bf16" else None
    tf = flops / (ms * 1e-3) / 1e12
    out = {"ms": ms, "query_tokens_per_s": w.Tq / (ms * 1e-3),
           "algorithmic_flops": flops, "tflops": tf}
    if w.dtype == "bf16":
        out["roofline"] = {"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                           "frac": tf / peaks["bf16_tflops"],
                           "peak_source": f"{kind} bf16 burst"}
        out["kernel"] = ("tcgen05: D = rowsum(dO o), dK/dV per (K/V tile, unit) with one "
                         "float4 atomic flush per tile, dQ per 128-row tile")
        out["fp32_cuda_core_kernel_ms"] = ms_cc
    else:
        out["roofline"] = {"bound": "alu", "peak": FP32_ALU_PEAK_TFLOPS, "unit": "TFLOP/s",
                           "frac": tf / FP32_ALU_PEAK_TFLOPS,
                           "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz"}
        out["kernel"] = "fp32 CUDA cores, one CTA per 128-row slice, 16-byte atomics for dK/dV"
    return {"workload": w.name, "backward": out}


def measure_causal(w, dev, flush_w, flush_r, sink, reps=6):
    """Strictly causal routing variant (each block routed on the block before
    it) against the block-shared routing, same inputs: device time of
    hga_forward_causal and hga_forward (segment summaries, both routings,
    attention; bf16 V) with a cold L2, eager launches between CUDA events."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    q_ext = torch.cat([gi.make_q_before(w), inp.q]).to(dev)
    q = q_ext[w.qblock:]
    k, v = inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)

    def timed(fn):
        ts = []
        for i in range(reps + 2):
            flush_w.zero_()
            torch.sum(flush_r, 0, out=sink)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        assert hga.check() == 0
        return float(np.median(ts))

    ms_shared = timed(lambda: hga.forward(p, q, w.q0, k, v, bufs))
    o_shared = bufs.o.clone()
    ms_causal = timed(lambda: hga.forward_causal(p, q_ext, w.q0, k, v, bufs))
    return {"workload": w.name, "causal_routing": {
        "ms": ms_causal, "query_tokens_per_s": w.Tq / (ms_causal * 1e-3),
        "block_shared_ms": ms_shared, "ratio_to_block_shared": ms_causal / ms_shared,
        "max_abs_diff_vs_block_shared": float((bufs.o.float() - o_shared.float()).abs().max()),
        "timing": "eager launches between CUDA events, cold L2, median of 6"}}


REF_UNITS_PER_STEP = 32


def run_reference(args, world, rank):
    """The oracle as the reference arm, on the host cores.  One step is a
    fixed sample of REF_UNITS_PER_STEP (query block, KV head) units of the
    workload (routing + attention, float64 NumPy), rotating so that
    consecutive steps cover different units; every step is timed whole, so
    ms_per_step x steps is the time the timed steps took.  The history's
    summaries are built once before timing (commit cost, as on the GPU arm)."""
    if rank != 0:
        return None
    from oracle import hga_oracle as ho
    w = gi.WORKLOADS[args.workload]
    inp = gi.make_inputs(w)
    p = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group,
                  w.qblock, w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    t0 = time.perf_counter()
    q, k, v = gi.to_f64(inp.q), gi.to_f64(inp.k), gi.to_f64(inp.v)
    csum, gsum = ho.build_summaries(k, p, 0, w.T)
    t_setup = time.perf_counter() - t0
    nb = -(-w.Tq // w.qblock)
    units = [(b, h) for b in range(nb) for h in range(w.n_kv_heads)]
    per = min(REF_UNITS_PER_STEP, len(units))

    def step(i):
        first = (i * per) % len(units)
        sel = [units[(first + x) % len(units)] for x in range(per)]
        ho.hga_forward(q, k, v, w.q0, p, units=sel, csum=csum, gsum=gsum)

    for i in range(args.warmup):
        step(i)
    times = []
    for i in range(args.steps):
        t1 = time.perf_counter()
        step(args.warmup + i)
        times.append(time.perf_counter() - t1)
    ms = float(np.mean(times)) * 1e3
    q_tokens = per * w.qblock / w.n_kv_heads     # a unit: 64 positions x 1/Hkv of the heads
    value = q_tokens / (ms * 1e-3)
    try:
        from threadpoolctl import threadpool_info
        blas = max((x.get("num_threads", 1) for x in threadpool_info()), default=1)
    except Exception:
        blas = None
    cores = len(os.sched_getaffinity(0))
    sample = (f"each step: {per} of {len(units)} (block, KV head) units of {w.name}, "
              f"rotating (routing + attention, float64 NumPy; BLAS threads {blas}); "
              f"history summaries ({t_setup:.1f} s) built once before timing")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) Q/K/V, RoPE, planted needles)",
            "config": workload_config(w, world, args.v_storage == "f16", step_names(args)),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s_timed_region": float(sum(times))}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--workload", default=gi.QWEN3_30B_64K.name, choices=sorted(gi.WORKLOADS))
    ap.add_argument("--v-storage", default="f16", choices=["f16", "bf16"],
                    help="V cache type read by the attention (f16: converted once per token)")
    ap.add_argument("--route", default="split", choices=["fused", "split"],
                    help="chunk + group routing in one kernel (fused) or two")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the brief per-workload report of the other configurations")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--only", default=None,
                    choices=["backward", "tiered", "store", "decode", "causal", "sweep", "configs"],
                    help="run one of the per-workload measurements alone and print its "
                         "JSON (for profiling); no headline line")
    ap.add_argument("--clock-window", type=float, default=0.6,
                    help="seconds of untimed replays on each side of the timed "
                         "region while nvidia-smi samples the clocks")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "hga":
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.only is not None:
        print(json.dumps(measure_one(args.only, args, torch.device("cuda", local))), flush=True)
        return
    if args.impl == "reference":
        out = run_reference(args, world, rank)
    else:
        out, w, inp = run_hga(args, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(w, inp, budget_s=args.cpu_seconds)
        if rank == 0 and world == 1 and not args.no_configs:
            out["configs"] = measure_all_configs(args, torch.device("cuda", local))
    if out is not None:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
