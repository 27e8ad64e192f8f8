"""Benchmark of the DSpark per-step hot path on B200.

One step = dspark_draft_markov (K sequential positions) ->
dspark_confidence_prefix -> dspark_verify over one batch of the workload.
Metric: draft+verify tokens/s = B*K per step / step time (whole job: summed
over ranks for N > 1; every rank runs its own replica of the workload, there
is no data-path collective, so scaling is weak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...   # the CPU oracle on host cores

The default workload is stress (V=151936, r=256, B=512, K=16, scheduler on),
the largest configuration at the metric's vocabulary.  Its steps are
sequential decode steps: each step draws fresh uniforms (the run's per-step
sets, copied into the step's input buffers before its timed region) and
takes as previous token the token the step before emitted last, copied on
the device inside the step's graph.  The logits stay fixed for the run.

Timing: every step is replayed from CUDA graphs and timed with CUDA events
on the launching stream; a 256 MB scratch write between steps flushes L2
(outside the timed events).  Prints one JSON line (rank 0).  With --gpus N
and no launcher environment (WORLD_SIZE unset) the script starts N ranks
itself through torch.distributed.run.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft+verify tokens/s (B×K per step) at V=151936; % of HBM / tensor roofline"
UNIT = "tokens/s"
DEFAULT_CONFIG = "stress"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    # smaller shapes of a workload (profiling captures, parity spot checks);
    # the line's config reports the sizes that ran
    ap.add_argument("--B", type=int, default=0)
    ap.add_argument("--K", type=int, default=0)
    ap.add_argument("--V", type=int, default=0)
    return ap.parse_args()


def workload_of(args):
    """The workload named by --config with any --B / --K / --V override."""
    from speculative_decoding_05_b200 import workloads as WL
    over = {k: v for k, v in (("B", args.B), ("K", args.K), ("V", args.V)) if v}
    return WL.get(args.config, **over)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


def algorithmic(w, L, reproject: bool = True):
    """Algorithmic bytes / flops of one step (W counted once per step).

    The verify reads every verified target row and, per request, one more
    row of draft logits for the residual; W (and the residual's flops) only
    when it re-projects that row (without the draft's bias rows)."""
    V, r, B, K = w.V, w.r, w.B, w.K
    uw = 2 if w.uw_bf16 else 4
    draft_bytes = uw * r * V + B * K * 4 * V + B * K * uw * r
    verify_bytes = sum(int(l) + 1 for l in L) * 4 * V + B * 4 * V
    if reproject:
        verify_bytes += uw * r * V
    draft_flops = 2.0 * B * K * r * V
    verify_flops = 2.0 * B * r * V if reproject else 0.0
    return dict(draft_bytes=draft_bytes, verify_bytes=verify_bytes,
                step_bytes=draft_bytes + verify_bytes, draft_flops=draft_flops,
                verify_flops=verify_flops)


# ------------------------------------------------------------ multi-rank --

def reduce_max(value: float, device=None) -> float:
    """Max of a per-rank value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


# ---------------------------------------------------------------- traffic --

def source_closure(root=None) -> list:
    """The CUDA sources a kernel is built from: its header (or each of a
    list of headers) and every file they include, transitively (each
    kernel's header also holds its launcher); every source when no header is
    named."""
    import glob
    import re
    csrc = os.path.join(ROOT, "speculative_decoding_05_b200", "csrc")
    if root is None:
        return sorted(glob.glob(os.path.join(csrc, "*")))
    roots = [root] if isinstance(root, str) else list(root)
    seen, todo = set(), [os.path.join(csrc, r) for r in roots]
    while todo:
        f = os.path.normpath(todo.pop())
        if f in seen or not os.path.exists(f):
            continue
        seen.add(f)
        for line in open(f):
            m = re.match(r'\s*#include\s+"([^"]+)"', line)
            if m:
                todo.append(os.path.join(os.path.dirname(f), m.group(1)))
    return sorted(seen)


def source_digest(root=None) -> str:
    """Hash of the sources a stored DRAM-traffic figure depends on (see
    source_closure).  A figure is only valid for the kernel code it was
    measured on."""
    import hashlib
    h = hashlib.sha256()
    for f in source_closure(root):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def launches_per_step(draft_path: str, verify_path: str, K: int,
                      prefix_path: str = "single-cta") -> int:
    """Kernels one step launches: the draft (one persistent launch, else a
    projection and a sampler per position), the prefix cut (one, or a
    survival and a rank kernel), the verify (one single-launch kernel, else
    statistics, accept, residual and sample)."""
    draft = 1 if draft_path.startswith(("persistent", "tcgen05-persistent")) else 2 * K
    prefix = 2 if prefix_path == "multi-cta" else 1
    verify = 1 if verify_path == "single-launch" else 4
    return draft + prefix + verify


def kernel_name(path: str, call: str, w) -> str:
    if call != "dspark_draft_markov":
        return "dspark_verify kernels"
    if path == "persistent-cuda-core":
        return f"draft_gemv_kernel<{w.B}>"
    if path == "tcgen05-persistent":
        return "draft_persist_kernel"
    if path == "tcgen05":
        return "proj_tc_kernel<false> + draft_sample2_kernel"
    return "draft_proj_simt_kernel + draft_sample_kernel"


def measured_traffic(kernel: str, workload: str):
    """dram bytes (read + write) per launch from the committed ncu summary,
    or None when absent or measured on other kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(f"{kernel}|{workload}")
    except ValueError:
        return None
    if not d or d.get("source_digest") != source_digest(d.get("root")):
        return None
    return d.get("dram_bytes_per_launch")


# --------------------------------------------------------------- clocks --

class ClockSampler:
    """SM clock and throttle reasons sampled every few milliseconds by a
    host thread through NVML while the timed region runs (read only: no
    setting of the GPU is touched)."""
    # clocks-event reason bits of NVML
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, dev_id, period_s=0.005):
        self.dev_id = str(dev_id)
        self.period = period_s
        self.samples = []
        self.mask = 0
        self.max_mhz = None
        self.thread = None
        self.nvml = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        self.nvml = pynvml
        if self.dev_id.startswith(("GPU-", "MIG-")):
            return pynvml.nvmlDeviceGetHandleByUUID(self.dev_id)
        return pynvml.nvmlDeviceGetHandleByIndex(int(self.dev_id))

    def start(self):
        try:
            h = self._handle()
            self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(h, self.nvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
            return
        self.stop_evt = threading.Event()

        def loop():
            nv = self.nvml
            while not self.stop_evt.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    self.mask |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                except Exception:
                    pass
                self.stop_evt.wait(self.period)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_evt.set()
        self.thread.join(timeout=5)
        try:
            self.nvml.nvmlShutdown()
        except Exception:
            pass
        reasons = sorted(n for n, bit in self.REASONS.items() if self.mask & bit)
        sm = statistics.median(self.samples) if self.samples else None
        return dict(sm_mhz=sm, sm_max_mhz=self.max_mhz, reasons=reasons,
                    samples=len(self.samples), source="nvml, 5 ms period")


# ------------------------------------------------------------ reference --

def run_reference(args, w, rank, world):
    """The CPU oracle (double precision, OpenMP across requests) as the
    reference arm: rank 0 only, each step a bounded sample of requests."""
    if rank != 0:
        return None
    import numpy as np
    import torch
    from oracle import oracle
    from speculative_decoding_05_b200 import workloads as WL
    oracle.build()
    inp = WL.make_inputs(w, device="cpu")
    h = {k: (v.numpy() if v.dtype != torch.bfloat16 else None) for k, v in inp.items()}
    U, W = WL.host_uw(inp["U"]), WL.host_uw(inp["W"])
    n_req = max(1, min(w.B, int(os.environ.get("DSPARK_REF_REQUESTS", "2"))))
    req = np.arange(n_req)
    pr = oracle.prefix(h["z"], h["temps"], h["cost_tokens"], h["cost_ms"], enable=w.scheduler)
    L = pr["L"][req]

    def one_step():
        oracle.prefix(h["z"], h["temps"], h["cost_tokens"], h["cost_ms"], enable=w.scheduler)
        d = oracle.draft(h["base"][req], U, W, h["prev_token"][req], h["u_draft"][req],
                         inv_temp=h["inv_temp"][req])
        rows = np.concatenate([np.arange(h["row_start"][b], h["row_start"][b] + L[i] + 1)
                               for i, b in enumerate(req)])
        rs = np.concatenate([[0], np.cumsum(L + 1)[:-1]]).astype(np.int64)
        oracle.verify(h["target"][rows], rs, L, h["base"][req], U, W, h["prev_token"][req],
                      d["tokens"], d["p_tok"], h["u_accept"][req], h["u_res"][req],
                      inv_temp=h["inv_temp"][req])

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = (time.perf_counter() - t0) / args.steps
    units = n_req * w.K
    value = units / dt
    cores = min(oracle.num_threads(), n_req)
    sample = f"{n_req} of {w.B} requests of the {w.name} workload per step (full K={w.K}, V={w.V})"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "V": w.V, "r": w.r, "B": w.B, "K": w.K,
                   "sampled_requests": n_req},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def cpu_baseline(w, inp_dev, seconds):
    """The oracle timed on host cores on a bounded sample of the workload."""
    import numpy as np
    import torch
    from oracle import oracle
    from speculative_decoding_05_b200 import workloads as WL
    oracle.build()
    n_req = min(w.B, max(1, oracle.num_threads()))
    req = torch.arange(n_req, device=inp_dev["base"].device)
    host = lambda t: t.index_select(0, req).cpu().numpy()
    base, prev, it = host(inp_dev["base"]), host(inp_dev["prev_token"]), host(inp_dev["inv_temp"])
    ud, ua, ur = host(inp_dev["u_draft"]), host(inp_dev["u_accept"]), host(inp_dev["u_res"])
    U, W = WL.host_uw(inp_dev["U"]), WL.host_uw(inp_dev["W"])
    K = w.K
    rows = torch.cat([torch.arange(int(inp_dev["row_start"][b]), int(inp_dev["row_start"][b]) + K + 1)
                      for b in range(n_req)]).to(inp_dev["target"].device)
    tgt = inp_dev["target"].index_select(0, rows).cpu().numpy()
    rs = (np.arange(n_req) * (K + 1)).astype(np.int64)
    L = np.full(n_req, K, np.int32)
    steps, t0 = 0, time.perf_counter()
    while True:
        d = oracle.draft(base, U, W, prev, ud, inv_temp=it)
        oracle.verify(tgt, rs, L, base, U, W, prev, d["tokens"], d["p_tok"], ua, ur, inv_temp=it)
        steps += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = (time.perf_counter() - t0) / steps
    return {"value": n_req * K / dt, "unit": UNIT, "cores": min(oracle.num_threads(), n_req),
            "kind": "oracle",
            "sample": f"{steps} oracle steps of {n_req} request(s) x K={K} at V={w.V} "
                      f"(full-block verify), {dt:.2f} s each"}


# ----------------------------------------------------------------- main --

def step_uniform_sets(w, inp, rank: int = 0):
    """The uniforms of every step of one run of the workload, stacked on the
    device: step 0 takes the workload's own draw (already in `inp`), step
    s > 0 the fresh set WL.step_uniforms draws for it.  A one-step workload
    has one set."""
    import torch
    from speculative_decoding_05_b200 import workloads as WL
    dev = inp["u_draft"].device
    sets = [dict(u_draft=inp["u_draft"].clone(), u_accept=inp["u_accept"].clone(),
                 u_res=inp["u_res"].clone())]
    for s in range(1, max(1, w.steps)):
        sets.append(WL.step_uniforms(w, s, device=dev, seed=w.seed + 1000 * rank))
    return {k: torch.stack([d[k] for d in sets]) for k in ("u_draft", "u_accept", "u_res")}


STS_METRIC = ("calibration score entries fitted per second (sequential temperature "
              "scaling of the confidence head, N x K per fit)")
STS_UNIT = "entries/s"
STS_LAUNCHES = 1 + 2 * 42 + 4  # init, (derivative + update) x (2 bounds + 40 steps), ECE


def sts_alg_bytes(c, passes: int) -> int:
    """Bytes one fit reads: each of its passes reads all scores and accepted
    lengths once (the fit reports how many passes its search took)."""
    return passes * (c.N * c.K * 4 + c.N * 4)


def sts_oracle_sample(c, z, n_acc, seconds: float):
    """The oracle on the leading sequences of the set, sized to about
    ``seconds`` of CPU work: (entries/s, sequences, seconds of the fit)."""
    from oracle import oracle
    n = min(c.N, 20_000)
    t0 = time.perf_counter()
    oracle.sts_fit(z[:n], n_acc[:n])
    dt = time.perf_counter() - t0
    n2 = min(c.N, int(n * seconds / max(dt, 1e-3)))
    if n2 > n:
        t0 = time.perf_counter()
        oracle.sts_fit(z[:n2], n_acc[:n2])
        dt, n = time.perf_counter() - t0, n2
    return n * c.K / dt, n, dt


def run_calibration(args, c, rank, world):
    """Bench line of the temperature fit on one calibration set per rank."""
    import torch
    import torch.distributed as dist
    from speculative_decoding_05_b200 import build as BLD
    from speculative_decoding_05_b200 import dspark as D
    from speculative_decoding_05_b200 import workloads as WL

    if args.impl == "reference":
        if rank != 0:
            return
        from oracle import oracle
        d = WL.make_calibration(c, device="cpu")
        z, n_acc = d["z"].numpy(), d["n_acc"].numpy()
        n_ref = min(c.N, int(os.environ.get("DSPARK_REF_SEQUENCES", "50000")))
        for _ in range(args.warmup):
            oracle.sts_fit(z[:n_ref], n_acc[:n_ref])
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle.sts_fit(z[:n_ref], n_acc[:n_ref])
        dt = (time.perf_counter() - t0) / args.steps
        value = n_ref * c.K / dt
        sample = f"{n_ref} of {c.N} sequences of the {c.name} set per fit (K={c.K})"
        print(json.dumps({
            "impl": "reference", "metric": STS_METRIC, "value": value, "unit": STS_UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": c.name, "N": c.N, "K": c.K, "requests": n_ref},
            "cpu_baseline": {"value": value, "unit": STS_UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": STS_UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return

    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    if rank == 0:
        BLD.build()
    if world > 1:
        dist.barrier()
    D.load()
    d = WL.make_calibration(c, device=dev, seed=c.seed + 1000 * rank)
    z, n_acc = d["z"], d["n_acc"]
    ws = torch.zeros(D.dspark_sts_workspace_size(c.N, c.K), dtype=torch.uint8, device=dev)
    temps = torch.empty(c.K, dtype=torch.float32, device=dev)
    ece = torch.empty(2, dtype=torch.float32, device=dev)
    passes = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def fit():
        D.dspark_sts_fit(z, n_acc, temps, ece, ws, passes=passes, stream=stream)

    with torch.cuda.stream(stream):
        fit()
    torch.cuda.synchronize()
    flags = D.dspark_get_device_flags(ws, stream)
    if flags:
        raise RuntimeError(f"device status flags after warm-up: {flags}")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fit()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    dev_id = os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local_rank)
    clocks = ClockSampler(dev_id)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev), dev)
    units = c.N * c.K
    value = whole_job_rate(units, world, ms)
    pk = peaks()
    n_pass = int(passes.item())
    alg = sts_alg_bytes(c, n_pass)
    achieved = alg / (ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": None,
                "kernel": f"sts_grad_kernel + sts_update_kernel ({n_pass - 2} passes), "
                          "sts_ece_kernel (2 passes)",
                "call": "dspark_sts_fit", "peak_source": pk["src"] + " (burst copy)",
                "algorithmic_bytes_per_launch": alg}

    host_z = z.cpu().pin_memory()
    host_n = n_acc.cpu().pin_memory()
    host_t = torch.empty(c.K, dtype=torch.float32, pin_memory=True)
    host_e = torch.empty(2, dtype=torch.float32, pin_memory=True)
    n_e2e = max(1, min(args.e2e_steps, args.steps))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_e2e)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(n_e2e):
            flush.zero_()
            e2e_ev[i][0].record(stream)
            z.copy_(host_z, non_blocking=True)
            n_acc.copy_(host_n, non_blocking=True)
            g.replay()
            host_t.copy_(temps, non_blocking=True)
            host_e.copy_(ece, non_blocking=True)
            e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in e2e_ev), dev)
    e2e = {"value": whole_job_rate(units, world, e2e_ms), "unit": STS_UNIT,
           "h2d_bytes_per_step": host_z.numel() * 4 + host_n.numel() * 4,
           "d2h_bytes_per_step": c.K * 4 + 8, "ms_per_step": e2e_ms}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, dt = sts_oracle_sample(c, host_z.numpy(), host_n.numpy(), args.cpu_seconds)
        cpu = {"value": v, "unit": STS_UNIT, "cores": 1, "kind": "oracle",
               "sample": f"one fit on the first {n} of {c.N} sequences (K={c.K}), {dt:.2f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": STS_METRIC, "value": value, "unit": STS_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": c.name, "N": c.N, "K": c.K,
                   "l2": "flushed by a 256 MB write between steps",
                   "parallelism": f"replicas x{world}", "graphs": True},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": STS_LAUNCHES * args.steps, "clocks": clk, "passes": n_pass,
        "temps": [round(float(t), 4) for t in temps.cpu()],
        "ece_before_after": [float(e) for e in ece.cpu()]}), flush=True)


def launcher_argv(n: int, argv: list, port: int) -> list:
    """The command that runs this script as n ranks on one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def check_world(gpus: int, env) -> int:
    """World size of this process; --gpus must match the launcher's."""
    world = int(env.get("WORLD_SIZE", "1"))
    if world != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but the launcher started {world} rank(s)")
    return world


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # no launcher: start the ranks here (one process per GPU), with a
        # bound on the whole run
        import socket
        import subprocess
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        rc = subprocess.call(launcher_argv(args.gpus, sys.argv[1:], port))
        sys.exit(rc)
    rank = int(os.environ.get("RANK", "0"))
    world = check_world(args.gpus, os.environ)
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from speculative_decoding_05_b200 import workloads as WL
    if args.config in WL.CALIBRATIONS:
        run_calibration(args, WL.CALIBRATIONS[args.config], rank, world)
        return
    w = workload_of(args)

    if args.impl == "reference":
        out = run_reference(args, w, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import numpy as np
    import torch
    import torch.distributed as dist
    from speculative_decoding_05_b200 import build as BLD
    from speculative_decoding_05_b200 import dspark as D
    from speculative_decoding_05_b200.step import DSparkStep

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        BLD.build()
    if world > 1:
        dist.barrier()
    D.load()

    inp = WL.make_inputs(w, device=dev, seed=w.seed + 1000 * rank)
    n_rows = inp["target"].shape[0]
    step = DSparkStep(w.V, w.r, w.B, w.K, n_rows, inp["U"].dtype, dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    uni = step_uniform_sets(w, inp, rank)
    # the inputs are drawn on the default stream and the steps run on
    # `stream`: finish the draws (and the allocator's reuse of the blocks
    # they freed) before the first step
    torch.cuda.synchronize()

    # eager warm-up (sets kernel attributes), then capture each call in a graph
    with torch.cuda.stream(stream):
        step.run(inp, enable_prefix=w.scheduler)
    torch.cuda.synchronize()
    flags = step.flags(stream)
    if any(flags.values()):
        raise RuntimeError(f"device status flags after warm-up: {flags}")
    # one graph per call (breakdown pass) and one graph for the whole step (timed)
    graphs = []
    for fn in (lambda: step.draft(inp), lambda: step.prefix(inp, w.scheduler),
               lambda: step.verify(inp)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        graphs.append(g)
    # timed: the draft call and the rest of the step (prefix + verify, then
    # the emitted last token copied into prev_token for the next step) as two
    # graphs, so the draft's own time comes from the same timed region
    g_draft = graphs[0]
    g_rest = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_rest, stream=stream):
        step.prefix(inp, w.scheduler)
        step.verify(inp)
        if w.steps > 1:
            inp["prev_token"].copy_(step.last_token)
    torch.cuda.synchronize()
    n_set = [0]

    def next_uniforms():
        """Copy the next step's uniforms into the captured input buffers."""
        i = n_set[0] % len(uni["u_draft"])
        n_set[0] += 1
        for k in ("u_draft", "u_accept", "u_res"):
            inp[k].copy_(uni[k][i], non_blocking=True)

    def replay():
        g_draft.replay()
        g_rest.replay()

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            next_uniforms()
            replay()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    dev_id = os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local_rank)
    clocks = ClockSampler(dev_id)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.zero_()
            next_uniforms()
            ev[i][0].record(stream)
            g_draft.replay()
            ev[i][1].record(stream)
            g_rest.replay()
            ev[i][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    t_step = [e[0].elapsed_time(e[2]) for e in ev]
    t_draft_timed = [e[0].elapsed_time(e[1]) for e in ev]
    ms = reduce_max(sum(t_step) / len(t_step), dev)
    units_per_rank = w.B * w.K
    value = whole_job_rate(units_per_rank, world, ms)

    # per-call breakdown (untimed pass, same flushing)
    n_bd = max(3, min(args.steps, 50))
    bd = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_bd)]
    with torch.cuda.stream(stream):
        for i in range(n_bd):
            flush.zero_()
            for j, g in enumerate(graphs):
                bd[i][j].record(stream)
                g.replay()
            bd[i][3].record(stream)
    torch.cuda.synchronize()
    t_draft = [e[0].elapsed_time(e[1]) for e in bd]
    t_prefix = [e[1].elapsed_time(e[2]) for e in bd]
    t_verify = [e[2].elapsed_time(e[3]) for e in bd]

    L = step.verify_len.cpu().tolist()
    na = step.n_accepted.cpu()
    alg = algorithmic(w, L, reproject=step.draft_bias is None)
    pk = peaks()
    md, mv = statistics.mean(t_draft_timed), statistics.mean(t_verify)
    # dominant part: the draft call (K projection + sampler launches) or the verify call
    if md >= mv:
        dom, dom_ms, dom_bytes = "dspark_draft_markov", md, alg["draft_bytes"]
    else:
        dom, dom_ms, dom_bytes = "dspark_verify", mv, alg["verify_bytes"]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    kern = kernel_name(step.path, dom, w)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": measured_traffic(kern, w.name),
                "kernel": kern, "call": dom, "peak_source": pk["src"] + " (burst copy)",
                "algorithmic_bytes_per_launch": dom_bytes,
                "step_frac": alg["step_bytes"] / (ms * 1e-3) / 1e9 / pk["hbm"]}

    # end to end: every step copies its inputs in from pinned host memory
    # (the logits, temperatures, confidences and row offsets, and that step's
    # uniforms) and its results out; the previous token of a multi-step run
    # stays on the device (the graph carries it), that of a one-step run is
    # copied in too.  With the scheduler on, the target rows come in after
    # the cut, and only the verified ones (each request's first L_b + 1
    # rows, packed, with their row offsets): the rows a target model would
    # compute for that verify.  The host waits for the cut inside the timed
    # region.
    e2e = None
    if rank == 0 or world > 1:
        K1 = w.K + 1
        names_in = ["base", "inv_temp", "z"] + ([] if w.scheduler else ["target", "row_start"])
        if w.steps <= 1:
            names_in.append("prev_token")
        host_in = {k: inp[k].cpu().pin_memory() for k in names_in}
        host_tgt = inp["target"].cpu().pin_memory() if w.scheduler else None
        host_rs = torch.empty(w.B, dtype=torch.int64, pin_memory=True)
        host_vl = torch.empty(w.B, dtype=torch.int32, pin_memory=True)
        host_uni = {k: v.cpu().pin_memory() for k, v in uni.items()}
        outs = [step.n_accepted, step.out_tokens, step.last_token]
        host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        h2d_fixed = sum(t.numel() * t.element_size() for t in host_in.values()) + \
            sum(t[0].numel() * t.element_size() for t in host_uni.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        row_bytes = w.V * inp["target"].element_size()
        n_e2e = max(1, min(args.e2e_steps, args.steps))
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n_e2e)]
        h2d_steps = []
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(n_e2e):
                flush.zero_()
                j = i % host_uni["u_draft"].shape[0]
                e2e_ev[i][0].record(stream)
                for k in names_in:
                    inp[k].copy_(host_in[k], non_blocking=True)
                for k, v in host_uni.items():
                    inp[k].copy_(v[j], non_blocking=True)
                h2d = h2d_fixed
                if w.scheduler:
                    graphs[0].replay()
                    graphs[1].replay()
                    host_vl.copy_(step.verify_len, non_blocking=True)
                    stream.synchronize()
                    rows = host_vl.numpy().clip(0, w.K).astype(np.int64) + 1
                    rs = host_rs.numpy()
                    rs[0] = 0
                    np.cumsum(rows[:-1], out=rs[1:])
                    for bb in range(w.B):
                        o, n = int(rs[bb]), int(rows[bb])
                        inp["target"][o:o + n].copy_(host_tgt[bb * K1:bb * K1 + n],
                                                     non_blocking=True)
                    off = int(rs[-1] + rows[-1])
                    inp["row_start"].copy_(host_rs, non_blocking=True)
                    h2d += off * row_bytes + host_rs.numel() * 8
                    d2h_cut = host_vl.numel() * 4
                    graphs[2].replay()
                    if w.steps > 1:
                        inp["prev_token"].copy_(step.last_token)
                else:
                    d2h_cut = 0
                    replay()
                for o, ho in zip(outs, host_out):
                    ho.copy_(o, non_blocking=True)
                e2e_ev[i][1].record(stream)
                h2d_steps.append(h2d)
        torch.cuda.synchronize()
        if w.scheduler:
            # the packed layout is what the device buffers now hold; put the
            # full-batch layout back for anything that runs after this
            inp["target"].copy_(host_tgt)
            inp["row_start"].copy_(torch.arange(w.B, dtype=torch.int64) * K1)
            torch.cuda.synchronize()
        e2e_ms = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in e2e_ev), dev)
        e2e = {"value": whole_job_rate(units_per_rank, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": statistics.mean(h2d_steps),
               "d2h_bytes_per_step": d2h + d2h_cut, "ms_per_step": e2e_ms,
               "target_rows": "verified rows only, after the cut" if w.scheduler else "all"}
        del host_in, host_uni, host_tgt

    vpath = D.dspark_verify_path(w.V, w.r, w.B, w.K, inp["U"].dtype, step.draft_bias is not None)
    n_launch = launches_per_step(step.path, vpath, w.K, D.dspark_prefix_path(w.B, w.K, w.scheduler))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inp, args.cpu_seconds)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "V": w.V, "r": w.r, "B": w.B, "K": w.K,
                   "uw": "bf16" if w.uw_bf16 else "f32", "scheduler": w.scheduler,
                   "draft_path": step.path, "l2": "flushed by a 256 MB write between steps",
                   "parallelism": f"replicas x{world}", "graphs": True,
                   "steps_per_run": w.steps,
                   "sequential": ("fresh uniforms every step; prev_token = the previous step's "
                                  "last emitted token, carried on the device")
                   if w.steps > 1 else "one step replayed"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": n_launch * args.steps,
        "clocks": clk,
        "breakdown_ms": {"draft": md, "prefix": statistics.mean(t_prefix), "verify": mv,
                         "note": "separate graphs per call, untimed pass"},
        "accepted_mean": float(na.float().mean()), "verify_len_mean": sum(L) / len(L),
        "latency_per_emitted_token_us": ms * 1e3 / (float(na.float().sum()) + w.B),
        "wall_s": wall,
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
