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
DEFAULT_CONFIG = "r1_prefill"  # DeepSeek-R1-shaped prefill layer: the largest single-GPU workload
FLUSH_BYTES = 256 << 20
E2E_LANES = 3


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--config", default=DEFAULT_CONFIG)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--group-limit", type=int, default=0,
                   help="node-limited routing: experts from the M best partitions (0 = off)")
    p.add_argument("--shared-expert", type=int, default=0, metavar="F_SHARED",
                   help="add a shared expert of this width, run on a second stream beside the routed path")
    p.add_argument("--fp8-dispatch", action="store_true",
                   help="dispatch E4M3 rows with per-token scales and run gate/up on E4M3 weights")
    p.add_argument("--gather", action="store_true",
                   help="bf16 dispatch without the permuted copy: the gate/up GEMM gathers each row's token "
                        "in place (saves the xp buffer; slower on B200, its 4-row TMA gathers bound the loads)")
    p.add_argument("--shape", action="append", default=[], metavar="FIELD=INT",
                   help="override one integer field of the workload (T, E, H, F, K, P); for reduced-size "
                        "profiling captures of a workload's kernels, e.g. --shape T=1024 --shape E=32")
    return p.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, dist=None, device="cpu") -> float:
    """Largest value over all ranks (the slowest rank's time); identity without a process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return dict(hbm=float(m["hbm_gbs"]), bf16=float(m["bf16_tflops"]),
                    bf16_sustained=float(m.get("bf16_tflops_sustained", m["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """Samples the SM clock and clock-event (throttle) reasons through NVML (read-only
    queries, the interface nvidia-smi reads) in a thread while the timed region runs."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device: int):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None

    def _handle(self, nv):
        try:
            props = torch.cuda.get_device_properties(self.device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.device)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nvml = nv
            self._h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._nvml = None
        return self

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=2)
        if self._nvml:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
        nv = self._nvml
        reasons = set()
        for _, rs in self.samples:
            for name, const in self.REASONS:
                if nv is not None and rs & getattr(nv, const, 0):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


class GpuLocalCpus:
    """Runs the enclosed host work on the CPUs of the GPU's own NUMA node (from sysfs), so that
    pinned buffers first touched there sit next to the GPU's PCIe root; the previous affinity is
    restored on exit.  A no-op where the node or the call is unavailable."""

    def __init__(self, device: int):
        self.device = device
        self.saved = None

    def _local(self):
        p = torch.cuda.get_device_properties(self.device)
        bus = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        cpus = set()
        with open(f"/sys/bus/pci/devices/{bus}/local_cpulist") as f:
            for part in f.read().strip().split(","):
                lo, _, hi = part.partition("-")
                cpus.update(range(int(lo), int(hi or lo) + 1))
        return cpus & os.sched_getaffinity(0)

    def __enter__(self):
        try:
            local = self._local()
            if local:
                self.saved = os.sched_getaffinity(0)
                os.sched_setaffinity(0, local)
        except Exception:
            self.saved = None
        return self

    def __exit__(self, *a):
        if self.saved:
            try:
                os.sched_setaffinity(0, self.saved)
            except Exception:
                pass


def code_fingerprint(path: str) -> str:
    """sha256[:12] of a CUDA source with its // comments and blank lines removed: a comment
    edit keeps the fingerprint, any change to the code changes it."""
    import hashlib
    lines = []
    for ln in open(path, encoding="utf-8"):
        cut = ln.find("//")
        if cut >= 0 and ln[:cut].count('"') % 2 == 0:
            ln = ln[:cut]
        ln = ln.rstrip()
        if ln:
            lines.append(ln)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:12]


def kernel_traffic(workload: str, stage: str):
    """DRAM bytes per launch of one kernel from a committed ncu summary, or None when the
    kernel's code changed since the counters were taken (the summary records its fingerprint)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for ln in open(path):
        f = ln.split("#")[0].split()
        if len(f) >= 4 and f[0] == workload and f[1] == stage:
            src = os.path.join(ROOT, "routing_dispatch_grouped_top_b200", "csrc", f[3].split(":")[0])
            if not os.path.exists(src):
                return None
            return float(f[2]) if code_fingerprint(src) == f[3].split(":")[1] else None
    return None


def oracle_sample_tokens(cfg) -> int:
    """Tokens per oracle sample: 16 for the small layers, fewer for the wide ones, so that one
    sample (its K experts' weights made on the host, then the float64 layer) stays within seconds."""
    return max(1, min(16, int(1.5e9 // (6 * cfg.H * cfg.F * cfg.K))))


class OracleSampler:
    """The oracle (as it stands) on bounded samples of the workload, for the host-side baseline.
    The host copies of the tokens, router and latent weights are made once; each expert's
    weights are made when a sample first needs them and kept (the 64 most recent)."""

    def __init__(self, cfg, seed_tokens: int = 0):
        import collections

        import oracle
        self.cfg, self.oracle = cfg, oracle
        self.seed_tokens = seed_tokens or oracle_sample_tokens(cfg)
        self.x_all = inputs.make_tokens(cfg, "cpu")
        w_g, bias = inputs.make_router(cfg, "cpu")
        w_dp, w_upp = inputs.make_latent(cfg, "cpu")
        self.w_g = w_g.numpy()
        self.bias = None if bias is None else bias.numpy()
        self.w_dp = None if w_dp is None else inputs.to_bits(w_dp)
        self.w_upp = None if w_upp is None else inputs.to_bits(w_upp)
        sh = inputs.make_shared_expert(cfg, "cpu")
        self.shared = None if sh is None else tuple(inputs.to_bits(t) for t in sh)
        self.g = torch.Generator().manual_seed(cfg.seed + 5)
        self.experts = collections.OrderedDict()

    def expert(self, e):
        cfg, oracle = self.cfg, self.oracle
        if e in self.experts:
            self.experts.move_to_end(e)
            return self.experts[e]
        ge = torch.Generator().manual_seed(10_000 + e)
        F, H = cfg.F, cfg.H
        wts = tuple(inputs.to_bits((torch.randn(s, generator=ge) * std).to(torch.bfloat16))
                    for s, std in (((F, H), H ** -0.5), ((F, H), H ** -0.5), ((H, F), F ** -0.5)))
        if cfg.fp8_dispatch:   # one-time weight preparation, like the GPU's
            (qg, sg), (qu, su) = oracle.quantize_rows_fp8(wts[0]), oracle.quantize_rows_fp8(wts[1])
            wts = (qg, sg, qu, su, wts[2])
        self.experts[e] = wts
        if len(self.experts) > 64:
            self.experts.popitem(last=False)
        return wts

    def rate(self, seconds: float) -> dict:
        """Tokens/s of the oracle over samples of seed_tokens random tokens, until `seconds` of
        oracle compute have passed (at least one sample)."""
        import numpy as np
        from threadpoolctl import threadpool_info
        cfg, oracle = self.cfg, self.oracle
        n_tok = runs = 0
        busy = 0.0                     # oracle compute time only (input preparation excluded)
        while True:
            idx = torch.randperm(cfg.T, generator=self.g)[:self.seed_tokens]
            xs = inputs.to_bits(self.x_all[idx])
            t0 = time.perf_counter()
            z = oracle.dense_bf16(xs, self.w_dp) if self.w_dp is not None else xs
            logits = oracle.gating_logits(z, self.w_g, self.bias)
            if cfg.group_limit:
                ids, w = oracle.route_limited(logits, cfg.K, cfg.P, cfg.group_limit, cfg.renormalize)
            else:
                ids, w = oracle.route(logits, cfg.K, cfg.renormalize)
            cs = oracle.count_scan(ids, cfg.E, cfg.P)
            xp, _ = oracle.permute(z, cs["row_of_assign"], ids, w, cfg.E, cfg.P)
            busy += time.perf_counter() - t0
            touched = [int(e) for e in np.nonzero(cs["counts"])[0]]
            wts = {e: self.expert(e) for e in touched}    # weights made outside the clock
            t0 = time.perf_counter()
            off = cs["offsets"]
            h = np.zeros((xp.shape[0], cfg.F), np.uint16)
            y = np.zeros((xp.shape[0], cfg.H), np.uint16)
            if cfg.fp8_dispatch:
                xq, xsc = oracle.dispatch_fp8(z, cs["row_of_assign"], cfg.K)
            for e in touched:
                lo, hi = off[e], off[e + 1]
                if cfg.fp8_dispatch:
                    h[lo:hi], y[lo:hi] = oracle.ffn_rows_fp8(xq[lo:hi], xsc[lo:hi], *wts[e])
                else:
                    h[lo:hi], y[lo:hi] = oracle.ffn_rows(xp[lo:hi], *wts[e])
            y_sh = None if self.shared is None else oracle.ffn_rows(z, *self.shared)[1]
            out = oracle.combine(y, cs["row_of_assign"], w, y_sh)
            if self.w_upp is not None:
                oracle.dense_bf16(out, self.w_upp)
            busy += time.perf_counter() - t0
            n_tok += self.seed_tokens
            runs += 1
            if busy >= seconds:
                break
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        return dict(value=n_tok / busy, unit=UNIT, cores=int(threads), kind="oracle",
                    sample=f"{runs} runs x {self.seed_tokens} random tokens of {cfg.name} through the whole layer "
                           f"(numpy float64, {busy:.1f} s of oracle compute; weights prepared outside the clock)")


def cpu_oracle_rate(cfg, seconds: float, seed_tokens: int = 0):
    """The oracle (as it stands) on bounded samples of the workload: tokens/s on the host."""
    return OracleSampler(cfg, seed_tokens).rate(seconds)


def shared_expert_overlap(cfg, inp, w, bufs, ws, flush, stream, n, dev) -> dict:
    """How much of the shared expert the auxiliary stream hides behind the routed path: the
    routed-only layer, the shared expert alone (one-group FFN over all T rows) and the whole
    layer, each timed on its own (mean of n L2-flushed runs; not part of the timed value)."""
    from routing_dispatch_grouped_top_b200 import binding as B
    d, d0 = B.dims_of(cfg), B.dims_of(cfg.with_(F_shared=0))
    ds = B.dims(T=cfg.T, H=cfg.H, E=1, K=1, F=cfg.F_shared)
    w0 = dict(w, w_shared_gate=None, w_shared_up=None, w_shared_down=None)
    off = torch.tensor([0, cfg.T], dtype=torch.int32, device=dev)
    rows = bufs["z"] if cfg.d_model else inp["x"]
    sg, su, sd = w["w_shared_gate"], w["w_shared_up"], w["w_shared_down"]
    runs = {
        "layer": lambda: B.moe_layer_forward(inp["x"], w, d, bufs, ws),
        "routed_only": lambda: B.moe_layer_forward(inp["x"], w0, d0, bufs, ws),
        "shared_alone": lambda: B.moe_grouped_ffn(rows, off, sg, su, sd, ds, bufs["h_shared"], bufs["y_shared"], ws),
    }
    ms = {}
    for name, fn in runs.items():
        fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        ms[name] = statistics.mean(a.elapsed_time(b) for a, b in ev)
    if B.read_device_status(ws) != 0:
        raise RuntimeError("device status set during the shared-expert pass")
    hidden = (ms["routed_only"] + ms["shared_alone"] - ms["layer"]) / ms["shared_alone"]
    return {"F_shared": cfg.F_shared, "layer_ms": ms["layer"], "routed_only_ms": ms["routed_only"],
            "shared_alone_ms": ms["shared_alone"], "hidden_frac": hidden,
            "stream": "shared expert on an auxiliary stream, forked after the latent down-projection"}


def fp8_accuracy(cfg, inp, bufs, dev) -> dict:
    """What FP8 dispatch changes: the layer output against the bf16 layer on the same inputs
    (relative Frobenius error, tokens whose expert set differs = 0 since routing precedes the
    dispatch) and the dispatch payload."""
    from routing_dispatch_grouped_top_b200 import binding as B
    c16 = cfg.with_(fp8_dispatch=False)
    d16 = B.dims_of(c16)
    w16 = B.pack_layer_weights(d16, inp["w_g"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"],
                               inp["w_dp"], inp["w_upp"], shared=inp["shared"])
    b16 = B.alloc_layer_buffers(d16, dev)
    ws16 = B.make_workspace(d16, dev)
    B.moe_layer_forward(inp["x"], w16, d16, b16, ws16)
    torch.cuda.synchronize()
    key = "final_out" if cfg.d_model else "out"
    a, b = bufs[key].double(), b16[key].double()
    rel = float(torch.linalg.norm(a - b) / torch.linalg.norm(b))
    rel_h = float(torch.linalg.norm(bufs["h"].double() - b16["h"].double()) / torch.linalg.norm(b16["h"].double()))
    same_routing = bool(torch.equal(bufs["topk_ids"], b16["topk_ids"]))
    del w16, b16, ws16
    torch.cuda.empty_cache()
    return {"out_rel_frob_vs_bf16_layer": rel, "h_rel_frob_vs_bf16_layer": rel_h, "same_routing": same_routing,
            "dispatch_bytes": cfg.dispatch_bytes_actual(), "bf16_dispatch_bytes": cfg.dispatch_bytes(2),
            "format": "E4M3 codes, one fp32 scale per token (amax/448); gate/up weights E4M3 per output feature"}


def gathers(cfg, args) -> bool:
    """bf16 dispatch without the permuted copy: the gate/up GEMM gathers the token rows."""
    return not cfg.fp8_dispatch and getattr(args, "gather", False)


def config_dict(cfg, world: int, gather: bool = False) -> dict:
    return {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "K": cfg.K, "F": cfg.F, "P": cfg.P,
            "d_model": cfg.d_model, "group_limit": cfg.group_limit, "F_shared": cfg.F_shared,
            "fp8_dispatch": cfg.fp8_dispatch,
            "dispatch": ("e4m3 rows permuted with per-row scales" if cfg.fp8_dispatch else
                         "token rows gathered by the gate/up GEMM (no permuted copy)" if gather else
                         "bf16 rows permuted into an expert-major copy"),
            "parallelism": f"replicas{world}",
            "l2": "flushed (256 MiB write) before every timed step, outside its events"}


def run_reference(args, cfg):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    steps = []
    sampler = OracleSampler(cfg)
    for _ in range(args.warmup):
        sampler.rate(0.0)
    rates = [sampler.rate(max(0.5, args.cpu_seconds / max(args.steps, 1))) for _ in range(args.steps)]
    val = statistics.mean(r["value"] for r in rates)
    cb = dict(rates[-1])
    cb["value"] = val
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * oracle_sample_tokens(cfg) / val,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_dict(cfg, ws, gathers(cfg, args)),
            "cpu_baseline": cb, "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    cfg = CFG.get(args.config)
    if args.group_limit:
        cfg = cfg.with_(group_limit=args.group_limit, name=f"{cfg.name}_node_limited_M{args.group_limit}")
    for kv in args.shape:
        k, v = kv.split("=")
        if k not in ("T", "E", "H", "F", "K", "P"):
            raise SystemExit(f"--shape: unknown field {k}")
        cfg = cfg.with_(**{k: int(v)})
    if args.shape:
        cfg = cfg.with_(name=f"{cfg.name}_reshaped_" + "_".join(args.shape).replace("=", ""))
    if args.fp8_dispatch:
        cfg = cfg.with_(fp8_dispatch=True, name=f"{cfg.name}_fp8_dispatch")
    if args.shared_expert:
        cfg = cfg.with_(F_shared=args.shared_expert, name=f"{cfg.name}_shared_expert_Fs{args.shared_expert}")
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
                             inp["w_upp"], shared=inp["shared"])
    gather = gathers(cfg, args)
    bufs = B.alloc_layer_buffers(d, dev, gather=gather)
    if cfg.F_shared:
        B.attach_aux_stream(bufs, torch.cuda.Stream(dev))
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

    # Timed region: one CUDA event pair per step, plus a pair around the gate/up GEMM (the
    # dominant kernel of every workload) for the roofline; nothing else is recorded between
    # the layer's kernels, so their programmatic dependent launches stay overlapped.
    GATE_UP = 5
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    ev_gu = [[torch.cuda.Event(enable_timing=True) if j in (GATE_UP, GATE_UP + 1) else None for j in range(n_ev)]
             for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(1)
            ev_step[i][0].record(stream)
            step(ev_gu[i])
            ev_step[i][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    if B.read_device_status(ws) != 0:
        raise RuntimeError("device status set during the timed steps")
    step_ms = [a.elapsed_time(b) for a, b in ev_step]
    gate_up_ms_timed = statistics.mean(e[GATE_UP].elapsed_time(e[GATE_UP + 1]) for e in ev_gu)
    total_ms = reduce_max(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    value = world * cfg.T / (ms_per_step / 1e3)

    # Per-stage breakdown (not part of the timed value): events between every stage.
    n_diag = min(args.steps, 20)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(n_diag)]
    for i in range(n_diag):
        flush.fill_(1)
        step(events[i])
    torch.cuda.synchronize()
    stage_ms = [[ev[j].elapsed_time(ev[j + 1]) for ev in events] for j in range(n_ev - 1)]
    shared_diag = shared_expert_overlap(cfg, inp, w, bufs, ws, flush, stream, n_diag, dev) if cfg.F_shared else None
    fp8_diag = fp8_accuracy(cfg, inp, bufs, dev) if cfg.fp8_dispatch else None

    # End to end through the host-buffer entry point: every step copies its x from pinned host
    # memory and its output back, inside the timed region.  Steps rotate over E2E_LANES streams,
    # each with its own device buffers and workspace, so the copies of some steps overlap the
    # kernels of another (the copy engines and the SMs work at the same time).  On one stream a
    # step is copy-in, kernels, copy-out in order, so with two lanes a lane's next copy-in waits
    # for its copy-out and the copies are only half hidden; three lanes keep the SMs busy.
    d_in = cfg.d_model or cfg.H
    lanes = []
    with GpuLocalCpus(local) as numa:  # the pinned host buffers on the GPU's NUMA node
        for i in range(E2E_LANES):
            lb = bufs if i == 0 else B.alloc_layer_buffers(d, dev, gather=gather)
            if cfg.F_shared and i > 0:
                B.attach_aux_stream(lb, torch.cuda.Stream(dev))
            lanes.append(dict(stream=torch.cuda.Stream(dev), bufs=lb,
                              ws=ws if i == 0 else B.make_workspace(d, dev), xd=torch.empty_like(inp["x"]),
                              oh=torch.empty((cfg.T, d_in), dtype=torch.bfloat16).pin_memory()))
        xh = inp["x"].cpu().pin_memory()

    def e2e_step(j):
        ln = lanes[j % E2E_LANES]
        with torch.cuda.stream(ln["stream"]):
            B.moe_layer_forward_host(xh, ln["xd"], w, d, ln["bufs"], ln["ws"], ln["oh"], stream=ln["stream"])

    for j in range(2 * E2E_LANES):
        e2e_step(j)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for ln in lanes:
        ln["stream"].wait_event(e_start)
    for j in range(args.steps):
        e2e_step(j)
    for ln in lanes:
        ev = torch.cuda.Event()
        ev.record(ln["stream"])
        stream.wait_event(ev)
    e_end.record(stream)
    torch.cuda.synchronize()
    for ln in lanes:
        if B.read_device_status(ln["ws"]) != 0:
            raise RuntimeError("device status set during the end-to-end steps")
    for ln in lanes[1:]:
        if not torch.equal(lanes[0]["oh"].view(torch.int16), ln["oh"].view(torch.int16)):
            raise RuntimeError("the end-to-end lanes disagree")
    e2e_ms = reduce_max(e_start.elapsed_time(e_end), dist, dev)
    e2e_value = world * cfg.T / (e2e_ms / args.steps / 1e3)

    if rank == 0:
        peaks = measured_peaks()
        clocks = clk.summary()
        names = ["latent_down", "gating", "route", "count_scan", "permute", "gate_up", "down", "combine",
                 "latent_up_and_skew"]
        stage_mean = {n: statistics.mean(v) for n, v in zip(names, stage_ms)}
        # The burst bf16 peak is a GEMM timed alone at full clock; the sustained one a GEMM loop
        # held under the 1 kW power cap.  A timed region longer than a second, or one whose clock
        # record shows the power cap, is compared with the sustained figure.
        sustained = total_ms > 1000.0 or "sw_power_cap" in clocks["reasons"]
        bf16_peak = peaks["bf16_sustained"] if sustained else peaks["bf16"]
        n_touched = int((bufs["counts"] > 0).sum().item())
        T, H, F, TK = cfg.T, cfg.H, cfg.F, cfg.TK
        # algorithmic work per launch: (flops, HBM bytes)
        fp8 = cfg.fp8_dispatch
        xb = 1 if fp8 else 2            # bytes per dispatched activation element and gate/up weight
        # gathered rows: each token's row need cross HBM once (T H 2), the permute step only
        # reads the ranks and ids and writes rows and metadata
        work = {
            "gate_up": (4 * H * F * TK, 2 * H * F * xb * n_touched + (T * H * 2 if gather else TK * H * xb)
                        + TK * F * 2 + (2 * F * 4 * n_touched + TK * 4 if fp8 else 0)),
            "down": (2 * H * F * TK, H * F * 2 * n_touched + TK * F * 2 + TK * H * 2),
            "permute": (0, (0 if gather else T * H * 2 + TK * H * xb) + TK * (4 + 8 + 16) + (TK * 4 if fp8 else 0)),
            "combine": (0, TK * H * 2 + T * H * 2 + TK * 8),
            "gating": (2 * T * H * cfg.E * 3, T * H * 2 + 3 * cfg.E * H * 2 + T * cfg.E * 4),
            "route": (0, T * cfg.E * 4 + TK * 8),
        }
        dominant = max(work, key=lambda n: stage_mean[n])
        fl, by = work[dominant]
        # the gate/up time comes from the timed region itself
        t_s = (gate_up_ms_timed if dominant == "gate_up" else stage_mean[dominant]) / 1e3
        # E4M3 gate/up: the measured bf16 peak times the nominal dense fp8 / bf16 ratio (4.5 / 2.25)
        tc_peak = 2.0 * bf16_peak if (fp8 and dominant == "gate_up") else bf16_peak
        hbm_time, tc_time = by / (peaks["hbm"] * 1e9), fl / (tc_peak * 1e12)
        if hbm_time >= tc_time:
            roof = {"bound": "hbm", "achieved": by / t_s / 1e9, "peak": peaks["hbm"], "unit": "GB/s"}
        else:
            roof = {"bound": "tensor", "achieved": fl / t_s / 1e12, "peak": tc_peak, "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = kernel_traffic(cfg.name, dominant)
        roof["kernel"] = dominant
        roof["algorithmic_bytes"] = by
        roof["algorithmic_flops"] = fl
        roof["peak_source"] = (f"{peaks['source']} " + ("HBM copy" if roof["bound"] == "hbm" else
                                                         f"bf16 {'sustained' if sustained else 'burst'}"
                                                         + (" x 2 (nominal fp8/bf16)" if tc_peak != bf16_peak
                                                            else "")))
        roof["timing"] = ("CUDA events around every gate/up launch of the timed steps" if dominant == "gate_up"
                          else "CUDA events of the per-stage pass")
        ffn_ms = stage_mean["gate_up"] + stage_mean["down"]
        ffn_tflops = cfg.expert_flops() / (ffn_ms / 1e3) / 1e12
        ffn_bytes = work["gate_up"][1] + work["down"][1]
        frac = {n: {"ms": stage_mean[n],
                    "tflops": (work[n][0] / (stage_mean[n] / 1e3) / 1e12) if work[n][0] else None,
                    "gbs": work[n][1] / (stage_mean[n] / 1e3) / 1e9} for n in work}
        for n in frac:
            frac[n]["frac_hbm"] = frac[n]["gbs"] / peaks["hbm"]
            if frac[n]["tflops"]:
                frac[n]["frac_bf16"] = frac[n]["tflops"] / bf16_peak
                frac[n]["frac_bf16_burst"] = frac[n]["tflops"] / peaks["bf16"]
        frac["grouped_ffn"] = {"ms": ffn_ms, "tflops": ffn_tflops, "frac_bf16": ffn_tflops / bf16_peak,
                               "frac_bf16_burst": ffn_tflops / peaks["bf16"],
                               "bf16_peak": "sustained" if sustained else "burst",
                               "gbs": ffn_bytes / (ffn_ms / 1e3) / 1e9,
                               "frac_hbm": ffn_bytes / (ffn_ms / 1e3) / 1e9 / peaks["hbm"],
                               "roofline_ms": 1e3 * max(ffn_bytes / (peaks["hbm"] * 1e9),
                                                        cfg.expert_flops() / (bf16_peak * 1e12))}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 gate/up, bf16 elsewhere" if fp8 else "bf16", "data": "synthetic",
            "config": config_dict(cfg, world, gather),
            "roofline": roof,
            "stages_ms": stage_mean,
            **({"shared_expert": shared_diag} if shared_diag else {}),
            **({"fp8_dispatch": fp8_diag} if fp8_diag else {}),
            "fractions": frac,
            "e2e": {"value": e2e_value, "unit": UNIT, "streams": E2E_LANES, "h2d_bytes_per_step": cfg.T * d_in * 2,
                    "d2h_bytes_per_step": cfg.T * d_in * 2, "pinned_on_gpu_numa_node": numa.saved is not None},
            "gpu_launches": (7 + (2 if cfg.d_model else 0) + (2 if cfg.F_shared else 0)) * args.steps,
            "clocks": clocks,
            "skew_max_over_mean": float(bufs["skew"].item()),
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
