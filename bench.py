#!/usr/bin/env python
"""Benchmark: MoE-layer tokens/s on B200 and the roofline fraction of the dominant kernel.

Workload (headline): the DeepSeek-V4-Flash-shaped MoE layer -- hidden 4096, expert FFN
2048 (SwiGLU), 256 experts, top-6, MXFP4 expert weights (E2M1 codes uniform over the 16
codes, one E8M0 scale per 32 elements uniform on 2^-8..2^-4) -- on an 8192-token prefill
batch (x ~ N(0,1) bf16).  This is the largest layer shape that runs on one GPU.  One step
= one pass of the whole hot path: route (fp32 logits + top-k + gates), permute (counting
sort + row gather), grouped gate/up GEMM with fused SwiGLU, grouped down GEMM, combine.
The expert weights (3.42 GB) and the permuted activations exceed the 126 MB L2, so every
step streams from HBM without an explicit flush.  Decode batches of the same layer (1 and
8 tokens) are reported in an extra object, timed while rotating over 4 weight copies so
that no batch finds its experts in L2.  By default the line also carries the other layer
shapes (Qwen3-A3B-shaped BF16 with a Zipf-skewed router, Gemma-4-26B-A4B-shaped with a
shared expert, the tiny layer: prefill and decode) and the expert-offload stack (8
DSV4-Flash-shaped layers served from pinned host memory); --no-extra / --no-stack skip them.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extra] [--no-stack]

Multi-GPU: the layer forward does not shard (one GPU per layer by construction), so
N > 1 runs N independent replicas, one process per GPU under torchrun; value is the
sum over ranks of tokens / max-over-ranks step time ("weak" scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_offload_serving_router_b200 import inputs  # noqa: E402

WORKLOAD = "dsv4_flash"
PREFILL_T = 8192
PREFILL_SIZES = {"qwen3_a3b": 4096, "dsv4_flash": 8192, "gemma4_26b_a4b": 2048, "tiny": 64}
METRIC = "MoE-layer tokens/s (decode & prefill) and % of HBM / tensor-core roofline"
LAUNCHES_PER_STEP = 3 + 3 + 1 + 1 + 1   # router (plane split, GEMM, top-k), permute (count/scan/scatter), gate/up, down, combine


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def sources_sha1(sources) -> str:
    """sha1 over the listed csrc files, in order (the sources a profiled kernel is built from)."""
    import hashlib
    h = hashlib.sha1()
    for src in sources:
        h.update(open(os.path.join(ROOT, "expert_offload_serving_router_b200", "csrc", src), "rb").read())
    return h.hexdigest()


def recorded_traffic(summary: str, sources):
    """DRAM bytes (read + write) per launch from a committed ncu summary under profiles/,
    or None when the summary is missing or the kernel's sources changed since the capture."""
    import re
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    try:
        sha = sources_sha1(sources)
    except OSError:
        return None
    fields = {}
    for line in open(p):
        m = re.match(r"\s*-?\s*(dram_bytes_per_launch|kernel_sources_sha1):\s*`?([0-9a-fA-F.]+)`?", line)
        if m:
            fields[m.group(1)] = m.group(2)
    if fields.get("kernel_sources_sha1") != sha:
        return None
    try:
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [c.strip() for c in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle timing
def oracle_tokens_per_s(cfg, layer_np, n_tokens, seed, threads):
    import oracle
    x = inputs.make_tokens(cfg, n_tokens, seed=seed, stream=77)
    shape = dict(hidden=cfg.hidden, ffn=cfg.ffn, num_experts=cfg.num_experts, top_k=cfg.top_k,
                 num_shared=cfg.num_shared, wdtype=cfg.wdtype)
    t0 = time.perf_counter()
    oracle.full_layer(shape, x, layer_np["w_router"], layer_np["bias"], layer_np, n_threads=threads)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def cpu_baseline(cfg, layer_np, budget_s=15.0):
    threads = os.cpu_count() or 1
    _, dt1 = oracle_tokens_per_s(cfg, layer_np, max(threads, 8), 0, threads)   # calibration
    per_tok = dt1 / max(threads, 8)
    n = int(min(4096, max(threads, budget_s / max(per_tok, 1e-6))))
    tps, dt = oracle_tokens_per_s(cfg, layer_np, n, 1, threads)
    return {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} tokens of the {PREFILL_T}-token {WORKLOAD} prefill (fp64 C oracle, OpenMP over tokens, "
                      f"{dt:.1f} s)"}


def max_over_ranks(torch, dist, ms, device="cuda"):
    """The slowest replica's device-timed milliseconds, returned on every rank."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_rank, ms_max):
    """Whole-job throughput of `world` replicas that each process tokens_per_rank tokens per
    step, timed by the slowest one (weak scaling: per-GPU work is fixed)."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def overlap_efficiency(copy_ms: float, compute_ms: float, layers: int, wall_ms: float) -> float:
    """Double-buffered layer streaming: the ideal wall time is the first layer's copy, then per
    layer the longer of the next layer's copy and this layer's compute (the last layer has no
    next copy).  Returns ideal / measured (1.0 = copies and compute overlap perfectly)."""
    ideal = copy_ms + (layers - 1) * max(copy_ms, compute_ms) + compute_ms
    return ideal / wall_ms


def run_reference(args, rank):
    """Reference arm: the fp64 CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    cfg = inputs.CONFIGS[WORKLOAD]
    layer_np = inputs.make_layer(cfg, seed=0)
    threads = os.cpu_count() or 1
    n = max(16, min(2 * threads, 512))
    for w in range(args.warmup):
        oracle_tokens_per_s(cfg, layer_np, n, 100 + w, threads)
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle_tokens_per_s(cfg, layer_np, n, 200 + s, threads)
    dt = time.perf_counter() - t0
    v = args.steps * n / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": f"{WORKLOAD} MoE layer prefill, {n}-token sample of the {PREFILL_T}-token batch",
                       "hidden": cfg.hidden, "ffn": cfg.ffn, "experts": cfg.num_experts, "top_k": cfg.top_k},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} tokens per step"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
class Layer:
    """One layer's weights resident on the GPU, plus the ABI structs."""
    KEYS = ("w13", "w13_scale", "w2", "w2_scale", "shared_w13", "shared_w13_scale", "shared_w2", "shared_w2_scale")

    def __init__(self, torch, F, cfg, layer_np):
        self.cfg = cfg
        self.np = layer_np
        self.t = {k: self.dev(torch, v) for k, v in layer_np.items() if v is not None}
        self.shape = F.make_shape(cfg.hidden, cfg.ffn, cfg.num_experts, cfg.top_k, cfg.num_shared, cfg.wdtype)
        self.weights = self.struct(F, self.t)

    @staticmethod
    def dev(torch, a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        return torch.from_numpy(a).cuda()

    def struct(self, F, t):
        return F.make_weights(*[t.get(k) for k in self.KEYS[:4]], None, *[t.get(k) for k in self.KEYS[4:]])

    def copy_weights(self, F):
        """A second copy of the routed expert weights (for L2-defeating rotation)."""
        t = dict(self.t)
        for k in self.KEYS[:4]:
            if k in t:
                t[k] = t[k].clone()
        return self.struct(F, t), t

    def expert_bytes(self):
        c = self.cfg
        hf = c.hidden * c.ffn
        return 3 * hf * 2 if c.wdtype == inputs.WDTYPE_BF16 else 3 * hf // 2 + 3 * hf // 32


def measure_prefill(torch, F, L, T, steps, warmup, stream, rank, clock_index=None):
    """Stepwise prefill through the public stage entry points, CUDA events between stages."""
    cfg = L.cfg
    H, Fd, E, k, S = cfg.hidden, cfg.ffn, cfg.num_experts, cfg.top_k, cfg.num_shared
    R, G = T * k + (T if S else 0), E + (1 if S else 0)
    x = Layer.dev(torch, inputs.make_tokens(cfg, T, seed=0, stream=rank))
    ws_bytes = F.ft_moe_workspace_bytes(L.shape, T)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    F.ft_moe_workspace_init(ws)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty(G + 1, dtype=torch.int32, device="cuda")
    sf = torch.empty(R, dtype=torch.int32, device="cuda")
    inv = torch.empty(R, dtype=torch.int32, device="cuda")
    xs = torch.empty((R, H), dtype=torch.int16, device="cuda")
    hbuf = torch.empty((R, Fd), dtype=torch.int16, device="cuda")
    o = torch.empty((R, H), dtype=torch.int16, device="cuda")
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    nst = 5

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        F.ft_moe_route(L.shape, T, x, L.t["w_router"], L.t.get("bias"), idx, gw, None, ws, ws_bytes, stream)
        mark(1)
        F.ft_moe_permute(L.shape, T, idx, x, off, sf, inv, xs, ws, ws_bytes, stream)
        mark(2)
        F.ft_moe_experts_gateup(L.shape, T, L.weights, xs, off, hbuf, ws, ws_bytes, stream)
        mark(3)
        F.ft_moe_experts_down(L.shape, T, L.weights, hbuf, off, o, ws, ws_bytes, stream)
        mark(4)
        F.ft_moe_combine(L.shape, T, o, inv, gw, y, stream)
        mark(5)

    for _ in range(warmup):
        step()
    F.ft_moe_check(ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(steps)]
    clk = ClockSampler(clock_index) if clock_index is not None else None
    torch.cuda.synchronize()
    if clk:
        clk.start()
        time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop() if clk else None
    F.ft_moe_check(ws)
    total_ms = t0.elapsed_time(t1)
    stage = np.zeros(nst)
    for s in range(steps):
        for i in range(nst):
            stage[i] += evs[s][i].elapsed_time(evs[s][i + 1])
    stage /= steps
    n_rows = int(off[G].item())
    gu_flops = 2.0 * n_rows * (2 * Fd) * H
    dn_flops = 2.0 * n_rows * Fd * H
    touched = int((off[1:] - off[:-1] > 0).sum().item())
    wbytes = touched * L.expert_bytes()
    names = ["route", "permute", "gateup_gemm", "down_gemm", "combine"]
    return dict(T=T, ms_step=total_ms / steps, total_ms=total_ms, stage_ms={n: float(v) for n, v in zip(names, stage)},
                gateup_tflops=gu_flops / (stage[2] * 1e-3) / 1e12, down_tflops=dn_flops / (stage[3] * 1e-3) / 1e12,
                gateup_flops=gu_flops, down_flops=dn_flops, experts_touched=touched, weight_bytes=wbytes,
                clocks=clocks, ctx=dict(x=x, ws=ws, ws_bytes=ws_bytes, y=y))


def measure_decode(torch, F, L, tokens, rank, hbm_gbs, nrot=4):
    """Decode batches through the whole-layer call, rotating over nrot weight copies so no
    batch finds its experts in L2.  Timed as plain launches and as a replayed CUDA graph
    of nrot calls (one per weight copy)."""
    cfg = L.cfg
    H, E, k = cfg.hidden, cfg.num_experts, cfg.top_k
    rot, keep = [L.weights], []
    for _ in range(1, nrot):
        wstruct, t = L.copy_weights(F)
        rot.append(wstruct)
        keep.append(t)
    stream = torch.cuda.current_stream()
    out = {}
    for Td in tokens:
        xd = Layer.dev(torch, inputs.make_tokens(cfg, Td, seed=5, stream=rank))
        yd = torch.empty((Td, H), dtype=torch.int16, device="cuda")
        idd = torch.empty((Td, k), dtype=torch.int32, device="cuda")
        ws_bytes = F.ft_moe_workspace_bytes(L.shape, Td)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        F.ft_moe_workspace_init(ws)

        def call(i, st):
            F.ft_moe_layer_forward(L.shape, Td, xd, L.t["w_router"], L.t.get("bias"), rot[i % nrot], yd, idd, None,
                                   ws, ws_bytes, st)

        for i in range(8):
            call(i, stream)
        torch.cuda.synchronize()
        n_it = 200
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for i in range(n_it):
            call(i, stream)
        d1.record(stream)
        torch.cuda.synchronize()
        us_plain = d0.elapsed_time(d1) * 1e3 / n_it
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            for i in range(nrot):
                call(i, cs)
        cs.synchronize()
        with torch.cuda.graph(g, stream=cs):
            for i in range(nrot):
                call(i, cs)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        reps = n_it // nrot
        d0.record()
        for _ in range(reps):
            g.replay()
        d1.record()
        torch.cuda.synchronize()
        us_graph = d0.elapsed_time(d1) * 1e3 / (reps * nrot)
        del g
        n_uniq = len(np.unique(idd.cpu().numpy()))
        algo_bytes = (n_uniq + cfg.num_shared) * L.expert_bytes() + E * H * 4 + 2 * Td * H * 2
        n_kern = F.ft_moe_decode_kernels(L.shape, Td)      # the library's own count for this path
        out[f"T{Td}"] = {"us_graph": us_graph, "us_plain": us_plain, "tokens_per_s": Td / (us_graph * 1e-6),
                         "experts_touched": n_uniq, "algorithmic_bytes": algo_bytes,
                         "achieved_gbs": algo_bytes / (us_graph * 1e-6) / 1e9,
                         "frac_hbm": algo_bytes / (us_graph * 1e-6) / 1e9 / hbm_gbs,
                         "launches_per_call": n_kern,
                         "timing": f"whole layer call ({n_kern} kernels), CUDA graph replay; "
                                   "us_plain = back-to-back plain launches"}
        F.ft_moe_check(ws)
    return out


def guarded(name, fn):
    """Run one auxiliary measurement (rank-local: no collectives inside) so that a failure is
    reported in the line, as {"error": ...}, instead of ending the run before the headline prints."""
    try:
        return fn()
    except Exception as ex:  # the headline line must still be printed
        print(f"bench: {name} failed: {ex!r}", file=sys.stderr, flush=True)
        return {"error": f"{type(ex).__name__}: {ex}"}


def measure_e2e(torch, dist, F, L, ctx, T, steps, warmup, world):
    """Same metric through the public whole-layer call with pinned host buffers: every step
    copies x host->device, runs ft_moe_layer_forward and copies y device->host.  The copies
    run on their own streams, double buffered, so step i's x upload and step i-1's y download
    overlap step i's layer (the serving pattern); the timed region spans the first upload to
    the last download."""
    H = L.cfg.hidden
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    x, ws, ws_bytes = ctx["x"], ctx["ws"], ctx["ws_bytes"]
    x_host = x.cpu().pin_memory()
    y_host = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
    xe = [torch.empty_like(x) for _ in range(2)]
    yb = [torch.empty((T, H), dtype=torch.int16, device="cuda") for _ in range(2)]
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def run(n, e0=None, e1=None):
        if e0 is not None:
            e0.record(s_in)
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(comp_done[b])          # xe[b] no longer read by step i-2
            with torch.cuda.stream(s_in):
                xe[b].copy_(x_host, non_blocking=True)
            in_done[b].record(s_in)
            comp.wait_event(in_done[b])
            if i >= 2:
                comp.wait_event(out_done[b])           # yb[b] downloaded for step i-2
            F.ft_moe_layer_forward(L.shape, T, xe[b], L.t["w_router"], L.t.get("bias"), L.weights, yb[b], None,
                                   None, ws, ws_bytes, comp)
            comp_done[b].record(comp)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                y_host[b].copy_(yb[b], non_blocking=True)
            out_done[b].record(s_out)
        if e1 is not None:
            e1.record(s_out)

    run(warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, e0, e1)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    if world > 1:
        ms = max_over_ranks(torch, dist, ms)
    return {"value": job_tokens_per_s(world, T, ms), "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
            "d2h_bytes_per_step": T * H * 2, "ms_per_step": ms,
            "timing": "x upload and y download on their own streams, double buffered, overlapping the layer"}


def summarize_prefill(p, hbm_gbs, tc_peak):
    t_gemm = (p["stage_ms"]["gateup_gemm"] + p["stage_ms"]["down_gemm"]) * 1e-3
    return {"T": p["T"], "ms_step": p["ms_step"], "tokens_per_s": p["T"] / (p["ms_step"] * 1e-3),
            "stage_ms": p["stage_ms"], "gateup_tflops": p["gateup_tflops"], "down_tflops": p["down_tflops"],
            "gateup_frac_tc": p["gateup_tflops"] / tc_peak,
            "experts_frac_tc": (p["gateup_flops"] + p["down_flops"]) / t_gemm / 1e12 / tc_peak,
            "experts_frac_hbm": p["weight_bytes"] / t_gemm / 1e9 / hbm_gbs, "experts_touched": p["experts_touched"]}


def measure_stack(torch, F, rank, hbm_gbs):
    """Expert-offload stack: 8 DSV4-Flash-shaped MXFP4 layers in pinned host memory, an
    8192-token prefill streamed with full-layer double buffering, then 256 single-token
    decode steps through 32 HBM expert slots per layer (cold start)."""
    st = inputs.STACK
    cfg = inputs.CONFIGS[st["layer"]]
    nl, slots = st["num_layers"], st["slots_per_layer"]
    H = cfg.hidden
    shape = F.make_shape(cfg.hidden, cfg.ffn, cfg.num_experts, cfg.top_k, 0, cfg.wdtype)
    hl = (F.ft_moe_weights * nl)()
    pinned, routers = [], []
    t_gen = time.perf_counter()
    for l in range(nl):
        d = inputs.make_layer(cfg, seed=0, layer=l, zipf=True, config_id=st["config_id"])
        ph = {}
        for key in ("w13", "w13_scale", "w2", "w2_scale"):
            a = np.ascontiguousarray(d[key])
            t = torch.empty(a.nbytes, dtype=torch.uint8, pin_memory=True)
            t.numpy()[:] = a.view(np.uint8).ravel()
            ph[key] = t
        pinned.append(ph)
        hl[l] = F.make_weights(ph["w13"], ph["w13_scale"], ph["w2"], ph["w2_scale"])
        routers.append((Layer.dev(torch, d["w_router"]), Layer.dev(torch, d["bias"])))
        del d
    t_gen = time.perf_counter() - t_gen
    cfgs = F.ft_stream_cfg(nl, slots, shape, hl, None, 0, 20000)
    n = F.ft_expert_stream_arena_bytes(cfgs)
    arena = torch.empty(n, dtype=torch.uint8, device="cuda")
    cfgs.hbm_arena, cfgs.hbm_arena_bytes = arena.data_ptr(), n
    handle = F.ft_expert_stream_create(cfgs)
    copy_stream = torch.cuda.Stream()
    out = {"host_bytes": int(sum(v.numel() for ph in pinned for v in ph.values())), "arena_bytes": n,
           "input_generation_s": t_gen}
    try:
        # pinned host -> device bandwidth probe (one 1 GiB copy, best of 3)
        probe_h = pinned[0]["w13"][: 1 << 30]
        probe_d = torch.empty(probe_h.numel(), dtype=torch.uint8, device="cuda")
        best = 0.0
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            probe_d.copy_(probe_h, non_blocking=True)
            e1.record()
            torch.cuda.synchronize()
            best = max(best, probe_h.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
        out["h2d_probe_gbs"] = best
        del probe_d
        # prefill: all layers, double buffered
        Tp = st["prefill_tokens"]
        x = Layer.dev(torch, inputs.make_tokens(cfg, Tp, seed=0, stream=500))
        wsb = F.ft_moe_workspace_bytes(shape, Tp)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        F.ft_moe_workspace_init(ws)
        yl = torch.empty((nl, Tp, H), dtype=torch.int16, device="cuda")
        xl = torch.empty((nl, Tp, H), dtype=torch.int16, device="cuda")
        wr = [r[0] for r in routers]
        bs = [r[1] for r in routers]
        F.ft_expert_stream_prefill(handle, Tp, x, wr, bs, yl, xl, ws, copy_stream=copy_stream)   # warm-up
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        F.ft_expert_stream_prefill(handle, Tp, x, wr, bs, yl, xl, ws, copy_stream=copy_stream)
        e1.record()
        torch.cuda.synchronize()
        pf_ms = e0.elapsed_time(e1)
        layer_bytes = out["host_bytes"] / nl
        out["prefill"] = {"T": Tp, "ms": pf_ms, "tokens_per_s": Tp / (pf_ms * 1e-3),
                          "h2d_gbs": out["host_bytes"] / (pf_ms * 1e-3) / 1e9,
                          "frac_of_h2d_probe": out["host_bytes"] / (pf_ms * 1e-3) / 1e9 / best,
                          "layer_copy_ms_at_probe": layer_bytes / (best * 1e9) * 1e3}
        # the same prefill streaming only each layer's routed experts (no copy/compute overlap)
        F.ft_expert_stream_reset_cache(handle)
        e0.record()
        F.ft_expert_stream_prefill_routed(handle, Tp, x, wr, bs, yl, xl, ws, copy_stream=copy_stream)
        e1.record()
        torch.cuda.synchronize()
        rt_ms = e0.elapsed_time(e1)
        out["prefill_routed"] = {"T": Tp, "ms": rt_ms, "tokens_per_s": Tp / (rt_ms * 1e-3),
                                 "h2d_bytes": F.ft_expert_stream_stats(handle, -1)[2]}
        del ws, yl, xl
        # a short prompt: whole layers vs routed experts only
        Ts = 64
        xsm = Layer.dev(torch, inputs.make_tokens(cfg, Ts, seed=0, stream=501))
        ws = torch.empty(F.ft_moe_workspace_bytes(shape, Ts), dtype=torch.uint8, device="cuda")
        F.ft_moe_workspace_init(ws)
        yl = torch.empty((nl, Ts, H), dtype=torch.int16, device="cuda")
        xl = torch.empty((nl, Ts, H), dtype=torch.int16, device="cuda")
        small = {"T": Ts}
        for mode, fn in (("full_layer", F.ft_expert_stream_prefill), ("routed_only", F.ft_expert_stream_prefill_routed)):
            fn(handle, Ts, xsm, wr, bs, yl, xl, ws, copy_stream=copy_stream)       # warm-up
            torch.cuda.synchronize()
            F.ft_expert_stream_reset_cache(handle)
            e0.record()
            fn(handle, Ts, xsm, wr, bs, yl, xl, ws, copy_stream=copy_stream)
            e1.record()
            torch.cuda.synchronize()
            small[mode] = {"ms": e0.elapsed_time(e1), "h2d_bytes": F.ft_expert_stream_stats(handle, -1)[2]}
        out["prefill_short_prompt"] = small
        del ws, yl, xl
        # decode: cold cache, 256 single-token steps, first with a cache per layer, then with
        # the same total slot count pooled across layers (global LRU at equal capacity)
        steps = st["decode_steps"]
        wsb = F.ft_moe_workspace_bytes(shape, 1)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        F.ft_moe_workspace_init(ws)
        yl = torch.empty((nl, 1, H), dtype=torch.int16, device="cuda")
        xl = torch.empty((nl, 1, H), dtype=torch.int16, device="cuda")
        xs = [Layer.dev(torch, inputs.make_tokens(cfg, 1, seed=1, stream=600 + s)) for s in range(steps)]

        def decode_run(h):
            F.ft_expert_stream_reset_cache(h)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            for s in range(steps):
                F.ft_expert_stream_decode_step(h, 1, xs[s], wr, bs, yl, xl, ws, copy_stream=copy_stream)
            torch.cuda.synchronize()
            dec_s = time.perf_counter() - t0
            st_all = F.ft_expert_stream_stats(h, -1)
            hits, misses = st_all[0], st_all[1]
            return {"steps": steps, "layers": nl, "s_total": dec_s,
                    "steps_per_s": steps / dec_s, "ms_per_step": 1e3 * dec_s / steps,
                    "hits": hits, "misses": misses, "miss_rate": misses / max(1, hits + misses),
                    "h2d_bytes": st_all[2], "wait_us_total": st_all[5],
                    "timing": "host wall clock around the 256 steps (each step waits for its routed ids)"}

        out["decode"] = dict(decode_run(handle), slots_per_layer=slots, cache="per layer")
        F.ft_moe_check(ws)
        F.ft_expert_stream_destroy(handle)
        handle = None
        cfgs.cache_policy = F.FT_CACHE_GLOBAL
        handle = F.ft_expert_stream_create(cfgs)
        out["decode_global_cache"] = dict(decode_run(handle), slots_total=nl * slots,
                                          cache="one LRU over all layers' slots (same capacity)")
        F.ft_moe_check(ws)
    finally:
        if handle is not None:
            F.ft_expert_stream_destroy(handle)
    return out


def measure_tma_reads(torch, F, reps=5):
    """Rate of TMA loads of 128-byte rows into a shared-memory ring (the library's TMA read probe,
    one CTA per SM): whole 128-row tiles against tile::gather4 loads of the same rows, and gather4
    loads of hashed rows inside a 64 MiB region (permuted token rows as a grouped GEMM would read
    them in place; the region fits in L2), with tile loads of that region for reference.  GB/s
    counts the bytes landed in shared memory; median of `reps` launches."""
    gib, region = 1 << 30, 64 << 20
    buf = torch.empty(gib // 4, dtype=torch.float32, device="cuda").normal_()
    small = buf[: region // 4]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    cases = [("tiles, 1 GiB", 0, buf, gib, 0), ("gather4 consecutive rows, 1 GiB", 1, buf, gib, 0),
             ("gather4 hashed rows in 64 MiB", 2, buf, gib, region), ("tiles, 64 MiB", 0, small, region, 0)]
    out = []
    for name, mode, b, nbytes, reg in cases:
        landed = (nbytes // 128 // 128 // nsm) * nsm * 128 * 128
        times = []
        for _ in range(reps + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            F.ft_tma_read_probe(mode, b, nbytes, reg, status, torch.cuda.current_stream())
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3)
        st = int(status.item())
        us = float(np.median(times[1:]))
        out.append({"case": name, "us": us, "gbs": landed / (us * 1e-6) / 1e9, "status": st})
    return out


def measure_hbm_ceiling(torch, F, sizes_mb=(8, 16, 32, 64, 76, 128, 256, 512, 1024, 2048), iters=20):
    """Streaming throughput of a plain read (the library's 16-byte-load probe kernel, best of 1,
    2, 4 and 8 CTAs per SM) and of a device-to-device copy for transfers of a given size,
    rotating over enough buffers (>= 1 GiB together) that L2 never holds the next one, replayed
    back to back from a CUDA graph.  GB/s counts the bytes read (read) or read + written (copy)."""
    out = []
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    for mb in sizes_mb:
        n = mb << 20
        k = max(4, -(-(1 << 30) // n))
        bufs = [torch.empty(n // 4, dtype=torch.float32, device="cuda").normal_() for _ in range(k)]
        dst = torch.empty(n // 4, dtype=torch.float32, device="cuda")
        row = {"mbytes": mb}
        variants = [("read", c) for c in (1, 2, 4, 8)] + [("copy", 0)]
        for kind, cps in variants:
            def op(i):
                if kind == "read":
                    F.ft_hbm_read_probe(bufs[i % k], n, sink, cps, torch.cuda.current_stream())
                else:
                    dst.copy_(bufs[i % k])
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                for i in range(3):
                    op(i)
            side.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                for i in range(iters):
                    op(i)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / iters
            del g
            moved = n if kind == "read" else 2 * n
            res = {"us": us, "gbs": moved / (us * 1e-6) / 1e9}
            if kind == "read":
                res["ctas_per_sm"] = cps
                if "read" not in row or res["gbs"] > row["read"]["gbs"]:
                    row["read"] = res
            else:
                row["copy"] = res
        out.append(row)
        del bufs, dst
        torch.cuda.empty_cache()
    return out


EXTRA_WORKLOADS = [("qwen3_a3b", [1, 4, 8, 16, 32]), ("gemma4_26b_a4b", [1, 4, 8, 16, 32]), ("tiny", [])]
HEADLINE_DECODE = [1, 4, 8, 16, 32]
ROOFLINE_SUMMARY = ("moe_gemm_mxfp4_dsv4_flash_T8192.md", ("gemm_mx_sm100.cu", "gemm_common.cuh", "sm100.cuh"))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-batch measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-extra", action="store_true", help="skip the other layer shapes")
    ap.add_argument("--no-stack", action="store_true", help="skip the expert-offload stack")
    ap.add_argument("--decode-tokens", default=None, help="decode batch sizes to time (comma list)")
    ap.add_argument("--decode-only", default=None, metavar="CONFIG",
                    help="time only decode batches of this layer shape (for profiling)")
    ap.add_argument("--prefill-only", default=None, metavar="CONFIG",
                    help="time only prefill steps of this layer shape at its prefill size (for profiling)")
    ap.add_argument("--prefill-tokens", type=int, default=None,
                    help="with --prefill-only: the batch size (default: the shape's prefill size)")
    ap.add_argument("--decode-rotations", type=int, default=4,
                    help="with --decode-only: weight copies rotated between calls (1 for small ncu captures)")
    ap.add_argument("--block-scaled-decode", default=None, choices=["0", "1", "2"],
                    help="MXFP4 decode on the block-scaled tensor cores: 0 never, 1 always, 2 from 4 tokens (default)")
    ap.add_argument("--tma-probe", action="store_true",
                    help="only time TMA tile loads against tile::gather4 row gathers")
    ap.add_argument("--hbm-ceiling", action="store_true",
                    help="only time plain streaming reads and copies of decode-sized transfers")
    args = ap.parse_args()
    dec_tokens = None if args.decode_tokens is None else [int(v) for v in args.decode_tokens.split(",") if v]
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import torch
    import torch.distributed as dist
    from expert_offload_serving_router_b200 import build as ftbuild
    from expert_offload_serving_router_b200 import ftmoe as F

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    if not os.path.exists(F.LIB_PATH):
        ftbuild.build()
    F.lib()
    hbm_gbs, tc_burst, tc_sus, peak_src = peaks()

    if args.tma_probe:
        if rank == 0:
            print(json.dumps({"mode": "tma-probe", "reads": measure_tma_reads(torch, F)}), flush=True)
        return

    if args.hbm_ceiling:
        if rank == 0:
            print(json.dumps({"mode": "hbm-ceiling", "peak_gbs": hbm_gbs, "peak_source": peak_src,
                              "sizes": measure_hbm_ceiling(torch, F)}), flush=True)
        return

    if args.block_scaled_decode is not None:
        F.ft_set_block_scaled_decode(int(args.block_scaled_decode))

    if args.decode_only:
        cfg = inputs.CONFIGS[args.decode_only]
        L = Layer(torch, F, cfg, inputs.make_layer(cfg, seed=0))
        dec = measure_decode(torch, F, L, dec_tokens or list(cfg.decode_tokens), rank, hbm_gbs,
                             nrot=args.decode_rotations)
        if rank == 0:
            print(json.dumps({"mode": "decode-only", "workload": f"{cfg.name} decode", "decode": dec}), flush=True)
        return

    if args.prefill_only:
        cfg = inputs.CONFIGS[args.prefill_only]
        Lp = Layer(torch, F, cfg, inputs.make_layer(cfg, seed=0))
        Tp = args.prefill_tokens or PREFILL_SIZES[args.prefill_only]
        px = measure_prefill(torch, F, Lp, Tp, args.steps, args.warmup, torch.cuda.current_stream(), rank)
        if rank == 0:
            print(json.dumps({"mode": "prefill-only", "workload": f"{cfg.name} prefill, T={Tp}",
                              "prefill": summarize_prefill(px, hbm_gbs, tc_burst)}), flush=True)
        return

    cfg = inputs.CONFIGS[WORKLOAD]
    layer_np = inputs.make_layer(cfg, seed=0)
    L = Layer(torch, F, cfg, layer_np)
    T = PREFILL_T
    if world > 1:
        dist.barrier()
    pre = measure_prefill(torch, F, L, T, args.steps, args.warmup, torch.cuda.current_stream(), rank, local)
    ms_step = pre["ms_step"]
    if world > 1:
        ms_step = max_over_ranks(torch, dist, ms_step)
        dist.barrier()
    value = job_tokens_per_s(world, T, ms_step)
    tc_peak = tc_sus if pre["total_ms"] > 1000.0 else tc_burst
    traffic = recorded_traffic(*ROOFLINE_SUMMARY)
    e2e = None if args.no_e2e else measure_e2e(torch, dist, F, L, pre["ctx"], T, args.steps, args.warmup, world)
    decode = None if args.no_decode else guarded(
        "decode", lambda: measure_decode(torch, F, L, dec_tokens or HEADLINE_DECODE, rank, hbm_gbs))
    headline_ms = pre["ms_step"]
    del L, pre["ctx"]
    torch.cuda.empty_cache()
    extra = None
    if not args.no_extra:
        extra = {}
        for name, Tds in EXTRA_WORKLOADS:
            def one(name=name, Tds=Tds):
                c = inputs.CONFIGS[name]
                Lx = Layer(torch, F, c, inputs.make_layer(c, seed=0))
                px = measure_prefill(torch, F, Lx, PREFILL_SIZES[name], 10, 3, torch.cuda.current_stream(), rank)
                out = {"prefill": summarize_prefill(px, hbm_gbs, tc_burst)}
                if Tds and not args.no_decode:
                    out["decode"] = measure_decode(torch, F, Lx, Tds, rank, hbm_gbs)
                return out
            extra[name] = guarded(name, one)
            torch.cuda.empty_cache()
    stack = None if args.no_stack else guarded("offload stack", lambda: measure_stack(torch, F, rank, hbm_gbs))
    if stack and "prefill" in stack:
        # copy time per layer from the pinned-copy probe, compute time per layer from the same
        # layer shape measured resident (the headline DSV4-Flash-shaped prefill at the stack's T)
        pf = stack["prefill"]
        pf["layer_compute_ms_resident"] = headline_ms
        pf["overlap_efficiency"] = overlap_efficiency(pf["layer_copy_ms_at_probe"], headline_ms,
                                                      inputs.STACK["num_layers"], pf["ms"])

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    cpu = None
    if world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cfg, layer_np)
    sp = summarize_prefill(pre, hbm_gbs, tc_peak)
    launches = LAUNCHES_PER_STEP * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy: MXFP4 codes uniform over the 16 E2M1 codes, E8M0 scales 2^-8..2^-4, "
                "N(0,1) bf16 tokens, N(0,0.02^2) fp32 router)",
        "config": {"workload": f"{WORKLOAD} MoE layer prefill, T={T}", "hidden": cfg.hidden, "ffn": cfg.ffn,
                   "experts": cfg.num_experts, "top_k": cfg.top_k, "tokens": T,
                   "weights": "mxfp4 (E2M1 + E8M0 per 32, dequantised exactly to bf16 in the GEMM load path)",
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (3.42 GB weights + 403 MB permuted rows per step), no flush"},
        "roofline": {"bound": "tensor", "kernel": "grouped GEMM (MXFP4 weights) gate/up + SwiGLU",
                     "achieved": pre["gateup_tflops"], "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": pre["gateup_tflops"] / tc_peak,
                     "peak_source": f"{peak_src} bf16 {'sustained' if tc_peak == tc_sus else 'burst'}",
                     "algorithmic_flops_per_launch": pre["gateup_flops"], "traffic": traffic},
        "stages_ms": sp["stage_ms"], "down_gemm_tflops": pre["down_tflops"],
        "experts_frac_of_peak": sp["experts_frac_tc"], "experts_frac_of_hbm": sp["experts_frac_hbm"],
        "e2e": e2e, "gpu_launches": launches, "clocks": pre["clocks"],
        "cpu_baseline": cpu, "decode": decode, "other_workloads": extra, "offload_stack": stack,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
