"""Benchmark of one routed MoE layer forward (tokens/s) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = the whole hot path over one batch of T tokens: gating GEMM -> top-K
route -> count/scan -> permute -> grouped gate/up (SwiGLU) -> grouped down ->
combine (plus the latent projections for the latent layer).  Inputs are seeded
synthetic tensors resident in HBM; L2 is flushed (a 256 MiB write) before every
timed step, outside its events.  Under torchrun each rank runs an independent
replica of the layer on its own GPU (no data-path collective: the layer is
single-GPU by design), ranks meet at barriers around the timed region, and the
slowest rank's time is reported.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from routing_dispatch_grouped_top_b200 import config as CFG  # noqa: E402
from routing_dispatch_grouped_top_b200 import inputs  # noqa: E402

METRIC = "MoE layer tokens/s; grouped-GEMM % of bf16 peak; permute/combine % of HBM BW"
UNIT = "tokens/s"
DEFAULT_CONFIG = "qwen3"       # Qwen3-30B-A3B-shaped prefill layer
FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", default=DEFAULT_CONFIG)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    return p.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return dict(hbm=float(m["hbm_gbs"]), bf16=float(m["bf16_tflops"]),
                    bf16_sustained=float(m.get("bf16_tflops_sustained", m["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_oracle_rate(cfg, seconds: float, seed_tokens: int = 16):
    """The oracle (as it stands) on bounded samples of the workload: tokens/s on the host."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle
    # Only the experts the sample needs are materialised on the host.
    x_all = inputs.make_tokens(cfg, "cpu")
    w_g, bias = inputs.make_router(cfg, "cpu")
    w_dp, w_upp = inputs.make_latent(cfg, "cpu")
    g = torch.Generator().manual_seed(cfg.seed + 5)
    n_tok = 0
    runs = 0
    busy = 0.0                     # oracle compute time only (input preparation excluded)
    expert_cache = {}

    def expert(e):
        if e not in expert_cache:
            ge = torch.Generator().manual_seed(10_000 + e)
            F, H = cfg.F, cfg.H
            expert_cache[e] = tuple(inputs.to_bits((torch.randn(s, generator=ge) * std).to(torch.bfloat16))
                                    for s, std in (((F, H), H ** -0.5), ((F, H), H ** -0.5), ((H, F), F ** -0.5)))
        return expert_cache[e]

    w_g_np = w_g.numpy()
    bias_np = None if bias is None else bias.numpy()
    w_dp_b = None if w_dp is None else inputs.to_bits(w_dp)
    w_upp_b = None if w_upp is None else inputs.to_bits(w_upp)
    while True:
        idx = torch.randperm(cfg.T, generator=g)[:seed_tokens]
        xs = inputs.to_bits(x_all[idx])
        t0 = time.perf_counter()
        z = oracle.dense_bf16(xs, w_dp_b) if w_dp_b is not None else xs
        logits = oracle.gating_logits(z, w_g_np, bias_np)
        ids, w = oracle.route(logits, cfg.K, cfg.renormalize)
        cs = oracle.count_scan(ids, cfg.E, cfg.P)
        xp, _ = oracle.permute(z, cs["row_of_assign"], ids, w, cfg.E, cfg.P)
        busy += time.perf_counter() - t0
        for e in np.nonzero(cs["counts"])[0]:
            expert(int(e))                 # materialise the weights outside the clock
        t0 = time.perf_counter()
        off = cs["offsets"]
        h = np.zeros((xp.shape[0], cfg.F), np.uint16)
        y = np.zeros((xp.shape[0], cfg.H), np.uint16)
        for e in np.nonzero(cs["counts"])[0]:
            lo, hi = off[e], off[e + 1]
            h[lo:hi], y[lo:hi] = oracle.ffn_rows(xp[lo:hi], *expert(int(e)))
        out = oracle.combine(y, cs["row_of_assign"], w)
        if w_upp_b is not None:
            oracle.dense_bf16(out, w_upp_b)
        busy += time.perf_counter() - t0
        n_tok += seed_tokens
        runs += 1
        if len(expert_cache) > 64:
            expert_cache.clear()
        if busy >= seconds:
            break
    el = busy
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dict(value=n_tok / el, unit=UNIT, cores=int(threads), kind="oracle",
                sample=f"{runs} runs x {seed_tokens} random tokens of {cfg.name} through the whole layer "
                       f"(numpy float64, {el:.1f} s of oracle compute; weights prepared outside the clock)")


def run_reference(args, cfg):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    steps = []
    for _ in range(args.warmup):
        cpu_oracle_rate(cfg, 0.0)
    rates = [cpu_oracle_rate(cfg, max(1.0, args.cpu_seconds / max(args.steps, 1))) for _ in range(args.steps)]
    val = statistics.mean(r["value"] for r in rates)
    cb = dict(rates[-1])
    cb["value"] = val
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * 16 / val, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "K": cfg.K,
                                            "F": cfg.F, "P": cfg.P, "d_model": cfg.d_model},
            "cpu_baseline": cb, "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    cfg = CFG.get(args.config)
    if args.impl == "reference":
        return run_reference(args, cfg)

    from routing_dispatch_grouped_top_b200 import binding as B

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    dev = torch.device("cuda", local)
    d = B.dims_of(cfg)
    inp = inputs.make_layer(cfg, dev)
    w = B.pack_layer_weights(d, inp["w_g"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"], inp["w_dp"],
                             inp["w_upp"])
    bufs = B.alloc_layer_buffers(d, dev)
    ws = B.make_workspace(d, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    n_ev = B.MOE_NUM_STAGE_EVENTS

    def step(evs=None):
        B.moe_layer_forward(inp["x"], w, d, bufs, ws, stage_events=evs)

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    if B.read_device_status(ws) != 0:
        raise RuntimeError("device status set during warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(1)
            step(events[i])
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    if B.read_device_status(ws) != 0:
        raise RuntimeError("device status set during the timed steps")
    step_ms = [ev[0].elapsed_time(ev[-1]) for ev in events]
    stage_ms = [[ev[j].elapsed_time(ev[j + 1]) for ev in events] for j in range(n_ev - 1)]
    total_ms = sum(step_ms)
    if dist:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * cfg.T / (ms_per_step / 1e3)

    # end to end through the host-buffer entry point (pinned host x in, host out back)
    d_in = cfg.d_model or cfg.H
    xh = inp["x"].cpu().pin_memory()
    oh = torch.empty((cfg.T, d_in), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(inp["x"])
    for _ in range(3):
        B.moe_layer_forward_host(xh, xd, w, d, bufs, ws, oh)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for a, b in e2e_ev:
        flush.fill_(1)
        a.record(stream)
        B.moe_layer_forward_host(xh, xd, w, d, bufs, ws, oh)
        b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)
    if dist:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * cfg.T / (e2e_ms / args.steps / 1e3)

    if rank == 0:
        peaks = measured_peaks()
        names = ["latent_down", "gating", "route", "count_scan", "permute", "gate_up", "down", "combine",
                 "latent_up_and_skew"]
        stage_mean = {n: statistics.mean(v) for n, v in zip(names, stage_ms)}
        long_run = total_ms > 1000.0
        bf16_peak = peaks["bf16_sustained"] if long_run else peaks["bf16"]
        gate_up_tflops = cfg.gate_up_flops() / (stage_mean["gate_up"] / 1e3) / 1e12
        down_tflops = cfg.down_flops() / (stage_mean["down"] / 1e3) / 1e12
        ffn_ms = stage_mean["gate_up"] + stage_mean["down"]
        ffn_tflops = cfg.expert_flops() / (ffn_ms / 1e3) / 1e12
        perm_bytes = cfg.T * cfg.H * 2 + cfg.TK * cfg.H * 2
        perm_gbs = perm_bytes / (stage_mean["permute"] / 1e3) / 1e9
        comb_gbs = perm_bytes / (stage_mean["combine"] / 1e3) / 1e9
        dominant = max(("gate_up", "down"), key=lambda n: stage_mean[n])
        dom_tf = gate_up_tflops if dominant == "gate_up" else down_tflops
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "K": cfg.K, "F": cfg.F,
                       "P": cfg.P, "d_model": cfg.d_model, "parallelism": f"replicas{world}",
                       "l2": "flushed (256 MiB write) before every timed step, outside its events"},
            "roofline": {"bound": "tensor", "kernel": f"grouped_gemm<{dominant}>", "achieved": dom_tf,
                         "peak": bf16_peak, "unit": "TFLOP/s", "frac": dom_tf / bf16_peak, "traffic": None,
                         "peak_source": f"{peaks['source']} bf16 {'sustained' if long_run else 'burst'}"},
            "stages_ms": stage_mean,
            "fractions": {"grouped_gemm_tflops": ffn_tflops, "grouped_gemm_frac_bf16": ffn_tflops / bf16_peak,
                          "permute_gbs": perm_gbs, "permute_frac_hbm": perm_gbs / peaks["hbm"],
                          "combine_gbs": comb_gbs, "combine_frac_hbm": comb_gbs / peaks["hbm"]},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": cfg.T * d_in * 2,
                    "d2h_bytes_per_step": cfg.T * d_in * 2},
            "gpu_launches": (7 + (2 if cfg.d_model else 0)) * args.steps,
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_oracle_rate(cfg, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
