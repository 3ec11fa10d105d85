"""Benchmark of MoE expert-parallel token routing on B200.

One step = the whole hot path over one batch: balanced plan (histogram, stable
counting sort, replica tables) -> dispatch of bf16 rows into the R ranks' receive
partitions -> combine of the identity expert's rows back into token order.

Default workload: R=8 simulated EP ranks, E=64 experts, S=4096 tokens per rank, K=8,
H=7168 bf16 (N = 262,144 token-slots per step). Inputs (x 470 MB, receive buffer
3.76 GB) are larger than the 126 MB L2, so no flush is needed between steps.

Prints one JSON line (rank 0). `value` = token-slots of all ranks per second of the
slowest rank's device time. With --gpus N > 1 (torchrun), every rank routes its own
independent batch on its own GPU (no data-path collective: weak scaling).
`--impl reference` times the oracle (plain single-threaded C) on the host instead.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

import synth

METRIC = "dispatch+combine token-slots/s and achieved HBM GB/s (% of peak), 1 B200"
UNIT = "token-slots/s"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ clock sampler

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML during the timed region."""

    REASONS = {
        0x0000000000000008: "hw_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000004: "sw_power_cap",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, index: int, period_s: float = 0.02):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self._thr = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if self.nv is None or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- byte accounting

def algorithmic_bytes(w):
    """Minimum bytes each kernel must move per launch (per step)."""
    row = 2 * w.H
    disp = w.T * row + w.N * row + 4 * w.N                 # read x once, write K copies, read pos
    comb = w.N * row + w.T * row + 8 * w.N                 # read K rows, write x, read pos+gates
    plan = 3 * 4 * w.N + 4 * w.N                           # 3 passes over ids, write pos
    return {"plan": plan, "dispatch": disp, "combine": comb}


# ------------------------------------------------------------------- oracle timing

def oracle_sample(w, S_sample):
    """Time the oracle (as it stands) on a bounded sample: the same workload with S
    reduced to S_sample tokens per rank. Returns (token-slots/s, description)."""
    import oracle

    ws = synth.scaled(w, S=S_sample)
    ids, gates = synth.router(ws)
    x = synth.hidden(ws).view(torch.int16).numpy().view(np.uint16)
    oracle.lib()
    t0 = time.perf_counter()
    p = oracle.plan_balanced(ids, ws.R, ws.E, ws.S, ws.K)
    t1 = time.perf_counter()
    y = oracle.dispatch(x, p.pos, ws.K, ws.N)
    t2 = time.perf_counter()
    oracle.combine(y, p.pos, gates, ws.K)
    t3 = time.perf_counter()
    dt = t3 - t0
    desc = (f"oracle plan+dispatch+combine on R={ws.R} E={ws.E} S={ws.S} K={ws.K} H={ws.H} "
            f"({ws.N} token-slots; S reduced from {w.S}); plan {t1 - t0:.3f}s dispatch "
            f"{t2 - t1:.3f}s combine {t3 - t2:.3f}s")
    return ws.N / dt, desc, dt


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    S_sample = max(1, w.S // args.ref_div)
    for _ in range(args.warmup):
        oracle_sample(w, S_sample)
    vals, tot = [], 0.0
    desc = ""
    for _ in range(args.steps):
        v, desc, dt = oracle_sample(w, S_sample)
        vals.append(v)
        tot += dt
    value = float(np.mean(vals))
    ws = synth.scaled(w, S=S_sample)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * tot / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "R": w.R, "E": w.E, "S": w.S, "K": w.K, "H": w.H,
                   "sample_S": S_sample, "seed": w.seed},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ multi-rank

def rank_workload(w, rank: int):
    """The batch one rank routes: the same shapes, its own seed (independent data)."""
    return synth.scaled(w, seed=w.seed + 1000 * rank) if rank else w


def max_over_ranks(value: float, pg, device) -> float:
    """Max of a per-rank timing over all ranks (the slowest rank sets the job time)."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------- GPU bench

def run_gpu(args, w):
    import dispatch_combine_topk_b200 as mep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    # every rank routes its own independent batch (different seed)
    wr = rank_workload(w, rank)
    ids, gates = synth.router(wr)
    x = synth.hidden(wr)
    stream = torch.cuda.Stream(dev)
    ids_d = torch.from_numpy(ids).to(dev).view(-1)
    g_d = torch.from_numpy(gates).to(dev).view(-1)
    x_d = x.to(dev)
    pb = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev)
    recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()

    def step(s, ev=None):
        if ev is not None:
            ev[0].record(s)
        mep.mep_plan(ids_d, w.R, w.E, w.S, w.K, pb, stream=s)
        if ev is not None:
            ev[1].record(s)
        mep.mep_dispatch(x_d, pb.pos, w.K, recv, stream=s)
        if ev is not None:
            ev[2].record(s)
        mep.mep_combine(recv, pb.pos, g_d, w.K, out, stream=s)
        if ev is not None:
            ev[3].record(s)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step(stream)
    stream.synchronize()
    mep.mep_get_error(clear=True)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(args.steps):
                step(stream, evs[i])
            end.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    ms = start.elapsed_time(end)
    err = mep.mep_get_error(clear=True)
    if err:
        raise RuntimeError(f"device error word {err:#x} after the timed steps")
    t_plan = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_disp = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    t_comb = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    ms_max = max_over_ranks(ms, pg, dev)
    ms_step = ms_max / args.steps

    # end to end: pinned host inputs -> device -> step -> result back to the host
    x_h = x.pin_memory()
    ids_h = torch.from_numpy(ids).view(-1).pin_memory()
    g_h = torch.from_numpy(gates).view(-1).pin_memory()
    out_h = torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step(s):
        ids_d.copy_(ids_h, non_blocking=True)
        g_d.copy_(g_h, non_blocking=True)
        x_d.copy_(x_h, non_blocking=True)
        step(s)
        out_h.copy_(out, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step(stream)
    stream.synchronize()
    if pg:
        pg.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step(stream)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, pg, dev)
    # identity expert + gates summing to 1: the result equals the input (as values)
    ok = torch.equal(out.float(), x_d.float())
    h2d = x_h.numel() * 2 + ids_h.numel() * 4 + g_h.numel() * 4
    d2h = out_h.numel() * 2

    if rank == 0:
        peak, peak_kind = load_peaks()
        ab = algorithmic_bytes(w)
        dom = "dispatch" if t_disp >= t_comb else "combine"
        t_dom = t_disp if dom == "dispatch" else t_comb
        achieved = ab[dom] / (t_dom * 1e-3) / 1e9
        dc_gbs = (ab["dispatch"] + ab["combine"]) / ((t_disp + t_comb) * 1e-3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, desc, _ = oracle_sample(w, w.S)
            cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc}
        line = {
            "metric": METRIC,
            "value": world * w.N / (ms_step * 1e-3),
            "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "R": w.R, "E": w.E, "S": w.S, "K": w.K, "H": w.H,
                       "token_slots_per_gpu": w.N, "seed": w.seed, "parallelism": f"replicas{world}",
                       "l2": f"inputs larger than L2 (x {w.T * w.H * 2 / 1e6:.0f} MB, recv "
                             f"{w.N * w.H * 2 / 1e9:.2f} GB; L2 126 MB): no flush"},
            "breakdown_ms": {"plan": t_plan, "dispatch": t_disp, "combine": t_comb},
            "dispatch_combine": {"token_slots_per_s": w.N / ((t_disp + t_comb) * 1e-3),
                                 "hbm_gbs": dc_gbs, "frac_of_peak": dc_gbs / peak,
                                 "frac_of_8tbs_nominal": dc_gbs / 8000.0},
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "algorithmic_bytes": ab[dom], "traffic": None},
            "cpu_baseline": cpu,
            "e2e": {"value": world * w.N / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "result_matches_input": bool(ok)},
            "gpu_launches": 6 * args.steps,
            "clocks": clk.summary(),
            "plan_stats": pb.stats_dict(),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mep", choices=["mep", "reference"])
    ap.add_argument("--workload", default="r8")
    ap.add_argument("--ref-div", type=int, default=8,
                    help="the oracle routes S/ref_div tokens per rank per step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens-per-rank", type=int, default=0,
                    help="override S (a smaller case of the same workload, e.g. for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = synth.get(args.workload)
    if args.tokens_per_rank:
        w = synth.scaled(w, S=args.tokens_per_rank)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
