#!/usr/bin/env python
"""Benchmark: MoE-layer tokens/s on B200 and the roofline fraction of the dominant kernel.

Workload (default): the Qwen3-A3B-shaped MoE layer -- hidden 2048, expert FFN 768
(SwiGLU), 128 experts, top-8 with a Zipf(s=1) rank-scaled router bias, BF16 weights
N(0, 0.02^2) -- on a 4096-token prefill batch (x ~ N(0,1) bf16).  One step = one pass of
the whole hot path: route (fp32 logits + top-k + gates), permute (counting sort + row
gather), grouped gate/up GEMM with fused SwiGLU, grouped down GEMM, combine.  Weights
(1.21 GB) and the permuted activations exceed the 126 MB L2, so every step streams
from HBM without an explicit flush.  Decode batches (1/4/16 tokens) are reported in
an extra object, timed while rotating over 4 weight copies so that no batch finds its
experts in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

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

WORKLOAD = "qwen3_a3b"
PREFILL_T = 4096
METRIC = "MoE-layer tokens/s (decode & prefill) and % of HBM / tensor-core roofline"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def recorded_traffic(summary: str, source: str):
    """DRAM bytes (read + write) per launch from a committed ncu summary under profiles/,
    or None when the summary is missing or the kernel source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "expert_offload_serving_router_b200", "csrc", source)
    if not os.path.exists(p) or not os.path.exists(src):
        return None
    fields = {}
    for line in open(p):
        if ":" in line and line.strip().startswith(("dram_bytes_per_launch", "kernel_source_sha1")):
            k_, v_ = line.split(":", 1)
            fields[k_.strip()] = v_.strip().strip("`")
    if fields.get("kernel_source_sha1") != hashlib.sha1(open(src, "rb").read()).hexdigest():
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
def measure_e2e(args, torch, dist, F, world, shape, weights, Wt, x, x_np, y, ws, ws_bytes, stream, T, H):
    """Same metric through the public whole-layer call with pinned host buffers: every step
    copies x host->device, runs ft_moe_layer_forward and copies y device->host."""
    x_host = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    y_host = torch.empty((T, H), dtype=torch.int16).pin_memory()
    xe = torch.empty_like(x)

    def e2e_step():
        xe.copy_(x_host, non_blocking=True)
        F.ft_moe_layer_forward(shape, T, xe, Wt["w_router"], Wt.get("bias"), weights, y, None, None, ws, ws_bytes,
                               stream)
        y_host.copy_(y, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e = {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
           "d2h_bytes_per_step": T * H * 2, "ms_per_step": e2e_ms}

    return e2e


def measure_decode(torch, F, cfg, shape, weights, Wt, ws, ws_bytes, stream, rank, hbm_gbs, dev, tokens):
    """Decode batches through the whole-layer call, rotating over 4 weight copies (4.8 GB) so
    no batch finds its experts in L2.  Timed as plain launches and as a replayed CUDA graph
    of 4 calls (one per weight copy)."""
    H, Fd, E, k = cfg.hidden, cfg.ffn, cfg.num_experts, cfg.top_k
    nrot = 4
    rot = [weights]
    keep = []
    for _ in range(1, nrot):
        w13c, w2c = Wt["w13"].clone(), Wt["w2"].clone()
        keep += [w13c, w2c]
        rot.append(F.make_weights(w13c, None, w2c, None))
    out = {}
    for Td in tokens:
        xd = dev(inputs.make_tokens(cfg, Td, seed=5, stream=rank))
        yd = torch.empty((Td, H), dtype=torch.int16, device="cuda")
        idd = torch.empty((Td, k), dtype=torch.int32, device="cuda")

        def call(i, st):
            F.ft_moe_layer_forward(shape, Td, xd, Wt["w_router"], Wt.get("bias"), rot[i % nrot], yd, idd, None, ws,
                                   ws_bytes, st)

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
        # the same calls captured once into a graph and replayed
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
        algo_bytes = n_uniq * 3 * H * Fd * 2 + E * H * 4 + 2 * Td * H * 2
        out[f"T{Td}"] = {"us_graph": us_graph, "us_plain": us_plain, "tokens_per_s": Td / (us_graph * 1e-6),
                         "experts_touched": n_uniq, "algorithmic_bytes": algo_bytes,
                         "achieved_gbs": algo_bytes / (us_graph * 1e-6) / 1e9,
                         "frac_hbm": algo_bytes / (us_graph * 1e-6) / 1e9 / hbm_gbs,
                         "launches_per_call": 3, "timing": "whole layer call (memset + 3 kernels), CUDA graph replay; "
                                                          "us_plain = back-to-back plain launches"}
    F.ft_moe_check(ws)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-batch measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--decode-tokens", default="1,4,16", help="decode batch sizes to time (comma list)")
    ap.add_argument("--decode-only", action="store_true", help="time only the decode batches (for profiling)")
    args = ap.parse_args()
    args.decode_tokens = [int(v) for v in args.decode_tokens.split(",") if v]
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

    cfg = inputs.CONFIGS[WORKLOAD]
    T = PREFILL_T
    H, Fd, E, k = cfg.hidden, cfg.ffn, cfg.num_experts, cfg.top_k
    R = T * k
    layer_np = inputs.make_layer(cfg, seed=0)

    def dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        return torch.from_numpy(a).cuda()

    Wt = {kk: dev(v) for kk, v in layer_np.items() if v is not None}
    shape = F.make_shape(H, Fd, E, k, cfg.num_shared, cfg.wdtype)
    weights = F.make_weights(Wt["w13"], None, Wt["w2"], None)
    x_np = inputs.make_tokens(cfg, T, seed=0, stream=rank)
    x = dev(x_np)
    ws_bytes = F.ft_moe_workspace_bytes(shape, T)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    F.ft_moe_workspace_init(ws)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sf = torch.empty(R, dtype=torch.int32, device="cuda")
    inv = torch.empty(R, dtype=torch.int32, device="cuda")
    xs = torch.empty((R, H), dtype=torch.int16, device="cuda")
    hbuf = torch.empty((R, Fd), dtype=torch.int16, device="cuda")
    o = torch.empty((R, H), dtype=torch.int16, device="cuda")
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    stream = torch.cuda.current_stream()
    if args.decode_only:
        hbm_gbs = peaks()[0]
        decode = measure_decode(torch, F, cfg, shape, weights, Wt, ws, ws_bytes, stream, rank, hbm_gbs, dev,
                                args.decode_tokens)
        if rank == 0:
            print(json.dumps({"mode": "decode-only", "workload": f"{WORKLOAD} decode", "decode": decode}), flush=True)
        return
    NST = 5
    LAUNCHES_PER_STEP = 1 + 3 + 1 + 1 + 1   # route, permute (count/scan/scatter), gate/up, down, combine

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        F.ft_moe_route(shape, T, x, Wt["w_router"], Wt.get("bias"), idx, gw, None, ws, ws_bytes, stream)
        mark(1)
        F.ft_moe_permute(shape, T, idx, x, off, sf, inv, xs, ws, ws_bytes, stream)
        mark(2)
        F.ft_moe_experts_gateup(shape, T, weights, xs, off, hbuf, ws, ws_bytes, stream)
        mark(3)
        F.ft_moe_experts_down(shape, T, weights, hbuf, off, o, ws, ws_bytes, stream)
        mark(4)
        F.ft_moe_combine(shape, T, o, inv, gw, y, stream)
        mark(5)

    for _ in range(args.warmup):
        step()
    F.ft_moe_check(ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(NST + 1)] for _ in range(args.steps)]
    clk = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop()
    F.ft_moe_check(ws)
    total_ms = t_start.elapsed_time(t_end)
    stage_ms = np.zeros(NST)
    for s in range(args.steps):
        for i in range(NST):
            stage_ms[i] += evs[s][i].elapsed_time(evs[s][i + 1])
    stage_ms /= args.steps
    ms_step = total_ms / args.steps
    if world > 1:
        t = torch.tensor([ms_step], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())
    value = world * T / (ms_step * 1e-3)

    hbm_gbs, tc_burst, tc_sus, peak_src = peaks()
    timed_s = total_ms * 1e-3
    tc_peak = tc_sus if timed_s > 1.0 else tc_burst
    gu_flops = 2.0 * R * (2 * Fd) * H          # algorithmic FLOPs of one gate/up launch
    dn_flops = 2.0 * R * Fd * H
    gu_tflops = gu_flops / (stage_ms[2] * 1e-3) / 1e12
    dn_tflops = dn_flops / (stage_ms[3] * 1e-3) / 1e12
    traffic = recorded_traffic("moe_gemm_gateup_qwen3_a3b_T4096.md", "gemm_sm100.cu")

    # ---------------- end to end through the public call, host buffers
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, torch, dist, F, world, shape, weights, Wt, x, x_np, y, ws, ws_bytes, stream, T, H)

    # ---------------- decode batches (rotating weight copies so L2 never holds the experts)
    decode = None
    if not args.no_decode:
        decode = measure_decode(torch, F, cfg, shape, weights, Wt, ws, ws_bytes, stream, rank, hbm_gbs, dev,
                                args.decode_tokens)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    cpu = None
    if world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cfg, layer_np)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded numpy: N(0,0.02^2) bf16 weights, "
                                                       "N(0,1) bf16 tokens, Zipf(1) router bias)",
        "config": {"workload": f"{WORKLOAD} MoE layer prefill, T={T}", "hidden": H, "ffn": Fd, "experts": E,
                   "top_k": k, "tokens": T, "weights": "bf16", "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (1.21 GB weights + 134 MB permuted rows per step), no flush"},
        "roofline": {"bound": "tensor", "kernel": "moe_gemm_kernel<bf16> gate/up + SwiGLU",
                     "achieved": gu_tflops, "peak": tc_peak, "unit": "TFLOP/s", "frac": gu_tflops / tc_peak,
                     "peak_source": f"{peak_src} bf16 {'sustained' if tc_peak == tc_sus else 'burst'}",
                     "algorithmic_flops_per_launch": gu_flops, "traffic": traffic},
        "stages_ms": {"route": stage_ms[0], "permute": stage_ms[1], "gateup_gemm": stage_ms[2],
                      "down_gemm": stage_ms[3], "combine": stage_ms[4]},
        "down_gemm_tflops": dn_tflops,
        "experts_frac_of_peak": (gu_flops + dn_flops) / ((stage_ms[2] + stage_ms[3]) * 1e-3) / 1e12 / tc_peak,
        "e2e": e2e, "gpu_launches": LAUNCHES_PER_STEP * args.steps, "clocks": clocks,
        "cpu_baseline": cpu, "decode": decode,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
