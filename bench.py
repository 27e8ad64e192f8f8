"""Benchmark of the DSpark per-step hot path on B200.

One step = dspark_draft_markov (K sequential positions) ->
dspark_confidence_prefix -> dspark_verify over one batch of the workload.
Metric: draft+verify tokens/s = B*K per step / step time (whole job: summed
over ranks for N > 1; every rank runs its own replica of the workload, there
is no data-path collective, so scaling is weak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...   # the CPU oracle on host cores

Timing: every step is replayed from CUDA graphs and timed with CUDA events
on the launching stream; a 256 MB scratch write between steps flushes L2
(outside the timed events).  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft+verify tokens/s (B×K per step) at V=151936; % of HBM / tensor roofline"
UNIT = "tokens/s"
DEFAULT_CONFIG = "single"


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
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


def algorithmic(w, L):
    """Algorithmic bytes / flops of one step (W counted once per step)."""
    V, r, B, K = w.V, w.r, w.B, w.K
    uw = 2 if w.uw_bf16 else 4
    draft_bytes = uw * r * V + B * K * 4 * V + B * K * uw * r
    verify_bytes = sum(int(l) + 1 for l in L) * 4 * V + B * 4 * V + uw * r * V
    draft_flops = 2.0 * B * K * r * V
    verify_flops = 2.0 * B * r * V
    return dict(draft_bytes=draft_bytes, verify_bytes=verify_bytes,
                step_bytes=draft_bytes + verify_bytes, draft_flops=draft_flops,
                verify_flops=verify_flops)


# --------------------------------------------------------------- clocks --

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_id):
        self.dev_id = dev_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev_id)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = [l.split(",") for l in open(self.path).read().strip().splitlines() if l.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in rows:
            row = [x.strip() for x in row]
            if len(row) < 9:
                continue
            try:
                sm.append(float(row[1]))
                mx = float(row[2])
            except ValueError:
                continue
            for n, v in zip(names, row[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=mx, reasons=sorted(reasons), samples=0)
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=mx, reasons=sorted(reasons),
                    samples=len(sm))


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

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from speculative_decoding_05_b200 import workloads as WL
    w = WL.get(args.config)

    if args.impl == "reference":
        out = run_reference(args, w, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

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

    # eager warm-up (sets kernel attributes), then capture each call in a graph
    with torch.cuda.stream(stream):
        step.run(inp, enable_prefix=w.scheduler)
    torch.cuda.synchronize()
    flags = step.flags(stream)
    if any(flags.values()):
        raise RuntimeError(f"device status flags after warm-up: {flags}")
    graphs = []
    for fn in (lambda: step.draft(inp), lambda: step.prefix(inp, w.scheduler),
               lambda: step.verify(inp)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        graphs.append(g)
    torch.cuda.synchronize()

    def replay():
        for g in graphs:
            g.replay()

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            replay()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
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
            e = ev[i]
            e[0].record(stream)
            graphs[0].replay()
            e[1].record(stream)
            graphs[1].replay()
            e[2].record(stream)
            graphs[2].replay()
            e[3].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()

    t_step = [e[0].elapsed_time(e[3]) for e in ev]
    t_draft = [e[0].elapsed_time(e[1]) for e in ev]
    t_prefix = [e[1].elapsed_time(e[2]) for e in ev]
    t_verify = [e[2].elapsed_time(e[3]) for e in ev]
    ms = sum(t_step) / len(t_step)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    units_per_rank = w.B * w.K
    value = units_per_rank * world / (ms * 1e-3)

    L = step.verify_len.cpu().tolist()
    na = step.n_accepted.cpu()
    alg = algorithmic(w, L)
    pk = peaks()
    md, mv = statistics.mean(t_draft), statistics.mean(t_verify)
    # dominant part: the draft call (K projection + sampler launches) or the verify call
    if md >= mv:
        dom, dom_ms, dom_bytes = "dspark_draft_markov", md, alg["draft_bytes"]
    else:
        dom, dom_ms, dom_bytes = "dspark_verify", mv, alg["verify_bytes"]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": None,
                "kernel": dom, "peak_source": pk["src"] + " (burst copy)",
                "algorithmic_bytes_per_launch": dom_bytes,
                "step_frac": alg["step_bytes"] / (ms * 1e-3) / 1e9 / pk["hbm"]}

    # end to end: inputs from pinned host memory, outputs back, every step
    e2e = None
    if rank == 0 or world > 1:
        names_in = ["base", "target", "prev_token", "inv_temp", "u_draft", "u_accept", "u_res",
                    "z", "row_start"]
        host_in = {k: inp[k].cpu().pin_memory() for k in names_in}
        outs = [step.n_accepted, step.out_tokens, step.last_token]
        host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        n_e2e = max(1, min(args.e2e_steps, args.steps))
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n_e2e)]
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(n_e2e):
                flush.zero_()
                e2e_ev[i][0].record(stream)
                for k in names_in:
                    inp[k].copy_(host_in[k], non_blocking=True)
                replay()
                for o, ho in zip(outs, host_out):
                    ho.copy_(o, non_blocking=True)
                e2e_ev[i][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in e2e_ev)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": units_per_rank * world / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    launches_per_step = 2 * w.K + 1 + 4
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
                   "parallelism": f"replicas x{world}", "graphs": True},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "breakdown_ms": {"draft": md, "prefix": statistics.mean(t_prefix), "verify": mv},
        "accepted_mean": float(na.float().mean()), "verify_len_mean": sum(L) / len(L),
        "latency_per_emitted_token_us": ms * 1e3 / (float(na.float().sum()) + w.B),
        "wall_s": wall,
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
