"""Benchmark of MoE expert-parallel token routing on B200.

One step = the whole hot path over one batch: balanced plan (histogram, stable
counting sort, replica tables) -> dispatch of the token rows into the R ranks' receive
partitions -> combine of the identity expert's rows back into token order.

Default workload (the headline): R=32 simulated EP ranks, E=256 experts, S=8192 tokens
per rank, K=8, H=7168, with per-token dynamic int8 dispatch and the combine of the int8
rows (N = 2,097,152 token-slots per step). Inputs (x 3.76 GB, receive buffer 15 GB) are
larger than the 126 MB L2, so no flush is needed between steps. After it, the other four
workloads (tiny, r8, map, skew), r8 and int8 in the expert-parallel layout, and int8 with
per-expert smoothing scales are measured the same way, more briefly, and reported in the
same line under `per_workload`.

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
L2_BYTES = 126 << 20
UNIT = "token-slots/s"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------- captured traffic

CSRC = os.path.join(ROOT, "dispatch_combine_topk_b200", "csrc")


def _device_functions():
    """name -> source text of every function defined in the library's CUDA headers."""
    import re

    import glob

    funcs = {}
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cuh"))):
        src = open(path).read()
        for m in re.finditer(r"\n(?:template <[^>]*>\n)?(?:__global__|__device__|__host__ __device__)\b", src):
            brace = src.find("{", m.end())
            if brace < 0 or src.find(";", m.end(), brace) >= 0:    # a variable, not a function
                continue
            depth, end = 0, -1
            for i in range(brace, len(src)):                       # the matching closing brace
                if src[i] == "{":
                    depth += 1
                elif src[i] == "}":
                    depth -= 1
                    if depth == 0:
                        end = i
                        break
            if end < 0:
                continue
            header = re.sub(r"__launch_bounds__\s*\([^)]*\)", "", src[m.end():brace])
            name = re.search(r"(\w+)\s*\(", header)
            if name:
                funcs.setdefault(name.group(1), src[m.start():end + 1])
    return funcs


def kernel_source_hash(name: str) -> str:
    """sha256 of a kernel's source text and of every library function it calls (found
    by name, transitively), so that a captured traffic figure is only reported for the
    code it was measured on."""
    import hashlib
    import re

    funcs = _device_functions()
    if name not in funcs:
        return ""
    seen, todo = set(), [name]
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.add(f)
        for ident in set(re.findall(r"\b(\w+)\s*[<(]", funcs[f])):
            if ident in funcs and ident not in seen:
                todo.append(ident)
    h = hashlib.sha256()
    for f in sorted(seen):
        h.update(funcs[f].encode())
    return h.hexdigest()[:16]


# dram__bytes_read.sum + dram__bytes_write.sum per launch, from one ncu capture of the
# kernel on a smaller case of the same workload (inputs larger than L2), scaled to the
# full workload by the rows routed: a capture on 1/4 or 1/16 of the tokens per rank
# routes that share of the rows. "src" is the kernel's source hash when captured.
_TRAFFIC_METRICS = "dram__bytes_read.sum + dram__bytes_write.sum"
TRAFFIC = {
    ("k_dispatch_warp", "r8_e64_s4096_k8_h7168"): {
        "bytes": 4 * 997.452e6, "src": "f2dc9831a61b7e83", "case_S": 1024, "case_mb": 997.452},
    ("k_combine_v8", "r8_e64_s4096_k8_h7168"): {
        "bytes": 4 * 1005.611e6, "src": "75f948c1d2f4d491", "case_S": 1024, "case_mb": 1005.611},
    ("k_dispatch_int8_staged", "int8_r32_e256_s8192_k8_h7168"): {
        "bytes": 16 * 1116.515e6, "src": "0909085f8f5d1cb1", "case_S": 512, "case_mb": 1116.515},
    ("k_combine_int8_warp", "int8_r32_e256_s8192_k8_h7168"): {
        "bytes": 16 * 1117.508e6, "src": "528f2068b9109630", "case_S": 512, "case_mb": 1117.508},
    ("k_dispatch_warp", "skew_r64_e512_s2048_k8_h4096"): {
        "bytes": 4 * 2357.469e6, "src": "f2dc9831a61b7e83", "case_S": 512, "case_mb": 2357.469},
    ("k_combine_v8", "skew_r64_e512_s2048_k8_h4096"): {
        "bytes": 4 * 2364.012e6, "src": "75f948c1d2f4d491", "case_S": 512, "case_mb": 2364.012},
    ("k_dispatch_int8_smooth_grouped", "int8_r32_e256_s8192_k8_h7168"): {
        "bytes": 16 * 1151.300e6, "src": "77b03711df0d65be", "case_S": 512, "case_mb": 1151.300},
}


def captured_traffic(kernel: str, workload: str):
    """(bytes per full launch, capture descriptor), or (None, None) when the kernel has
    no capture for this workload or its source changed since the capture."""
    t = TRAFFIC.get((kernel, workload))
    if not t or kernel_source_hash(kernel) != t["src"]:
        return None, None
    w = synth.get(workload)
    return t["bytes"], {"kernel": kernel, "workload": workload, "case_tokens_per_rank": t["case_S"],
                        "metrics": _TRAFFIC_METRICS, "case_mb": t["case_mb"],
                        "scale": w.S // t["case_S"], "kernel_src": t["src"]}


def host_info() -> dict:
    """The host the CPU baseline runs on: logical CPUs and the CPU model name."""
    model = None
    try:
        import subprocess
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    if model is None:
        try:
            for line in open("/proc/cpuinfo"):
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
        except OSError:
            pass
    mem_gb = None
    try:
        mem_gb = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES") / 2**30
    except (ValueError, OSError):
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model, "host_mem_gib": mem_gb}


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


# ------------------------------------------------------------------- oracle timing

_SAMPLES = {}


def oracle_sample(w, S_sample):
    """Time the oracle (as it stands) on a bounded sample: the same workload with S
    reduced to S_sample tokens per rank. The timed steps are those of the GPU step
    (mapping and grouped plan, or the balanced plan; dispatch, bf16 or int8; combine,
    of the int8 rows on the int8 workload). The sample's inputs are drawn once and
    reused by later calls (drawing them is not timed).
    Returns (token-slots/s, description, seconds)."""
    import oracle

    ws = synth.scaled(w, S=S_sample)
    if ws not in _SAMPLES:
        ids, gates = synth.router(ws)
        x = synth.hidden(ws).view(torch.int16).numpy().view(np.uint16)
        _SAMPLES.clear()
        _SAMPLES[ws] = (ids, gates, x)
    ids, gates, x = _SAMPLES[ws]
    oracle.lib()
    parts = {}
    t0 = time.perf_counter()
    if ws.mapping:
        table, thr, active = synth.mapping_inputs(ws)
        bi = np.empty_like(ids)
        bm = np.empty(ids.shape, bool)
        for r in range(ws.R):
            sl = slice(r * ws.S, (r + 1) * ws.S)
            bi[sl], bm[sl] = oracle.update_expert(ids[sl], table, gates[sl], thr, active[sl], r, ws.R, 0)
        p = oracle.plan_grouped(bi, bm, ws.R, ws.R * ws.place_per_rank, ws.place_per_rank, ws.S, ws.K)
    else:
        p = oracle.plan_balanced(ids, ws.R, ws.E, ws.S, ws.K)
    t1 = time.perf_counter()
    parts["plan"] = t1 - t0
    rows = p.n_kept
    if ws.quant:
        q, sc = oracle.dispatch_int8(x, p.pos, ws.K, rows)
        t2 = time.perf_counter()
        oracle.combine_int8(q, sc, p.pos, gates, ws.K)
    else:
        y = oracle.dispatch(x, p.pos, ws.K, rows)
        t2 = time.perf_counter()
        oracle.combine(y, p.pos, gates, ws.K)
    t3 = time.perf_counter()
    parts["dispatch"] = t2 - t1
    parts["combine"] = t3 - t2
    dt = parts["plan"] + parts["dispatch"] + parts["combine"]
    desc = (f"oracle {'mapping+grouped plan' if ws.mapping else 'plan'}+"
            f"{'int8 ' if ws.quant else ''}dispatch+combine on R={ws.R} E={ws.E} S={ws.S} K={ws.K} "
            f"H={ws.H} ({ws.N} token-slots" + (f"; S reduced from {w.S}" if ws.S < w.S else "; the whole workload") + "); "
            + " ".join(f"{k} {v:.3f}s" for k, v in parts.items()))
    return ws.N / dt, desc, dt


def cpu_sample_S(w, div: int) -> int:
    """Tokens per rank of the CPU sample: S/div, and small enough that the host copy of
    the receive rows stays under 2^31 elements."""
    fit = ((1 << 31) - 1) // (w.R * w.K * w.H)
    return max(1, min(w.S // max(div, 1), fit))


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    S_sample = cpu_sample_S(w, args.ref_div)
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
        "scaling": "weak", "vs_baseline": None, "dtype": "int8" if w.quant else "bf16", "data": "synthetic",
        "config": {"workload": w.name, "R": w.R, "E": w.E, "S": w.S, "K": w.K, "H": w.H,
                   "sample_S": S_sample, "seed": w.seed},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": desc, **host_info()},
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

class Route:
    """Device buffers and the launch sequence of one routing step for one workload.

    Balanced workloads: plan (mep_plan) -> dispatch (bf16, or int8 for the int8
    workload) -> combine. The identity expert returns the dispatched rows; on the int8
    workload they stay int8 and the combine reads the codes and scales
    (mep_combine_int8, the same result as dequantising first).
    Mapping workload: mep_update_expert_ranks (every rank, one launch) -> grouped plan over the physical
    instances -> dispatch -> combine.
    With dedup, the plan is followed by the deduplicated encoding (mep_dedup_plan), the
    dispatch sends one row per (token, destination rank) along its send list, and an
    expand phase (mep_expand) rebuilds the expert-grouped rows on the receiving side.
    """

    def __init__(self, mep, w, dev, epilogue: str = "none", dedup: bool = False, smooth: bool = False):
        self.mep, self.w, self.dev = mep, w, dev
        self.epilogue = epilogue
        self.dedup = dedup
        self.smooth = smooth
        self.n_sent = None
        ids, gates = synth.router(w)
        x = synth.hidden(w)
        self.host = dict(ids=torch.from_numpy(ids).view(-1), gates=torch.from_numpy(gates).view(-1), x=x)
        self.ids = self.host["ids"].to(dev)
        self.gates = self.host["gates"].to(dev)
        self.x = x.to(dev)
        self.out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
        self.launches = 0
        if epilogue == "add_rmsnorm":
            # combine fused with residual add + RMSNorm: residual rows and gamma as inputs
            self.residual = synth.expert_outputs(w, w.T).to(dev)
            self.gamma = torch.ones(w.H, dtype=torch.bfloat16, device=dev)
            self.y_norm = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
            self.rstd = torch.empty(w.T, dtype=torch.float32, device=dev)
        if w.mapping:
            table, thr, active = synth.mapping_inputs(w)
            self.table = torch.from_numpy(table).to(dev)
            self.thr = torch.from_numpy(thr).to(dev)
            self.active = torch.from_numpy(active.astype(np.uint8)).to(dev)
            self.bids = torch.empty((w.T, w.K), dtype=torch.int32, device=dev)
            self.bmask = torch.empty((w.T, w.K), dtype=torch.uint8, device=dev)
            self.n_keys = w.R * w.place_per_rank
            self.pb = mep.PlanBuffers.allocate(w.R, self.n_keys, w.S, w.K, dev)
            self.recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
            self.y = self.recv
        else:
            self.pb = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev)
            if w.quant:
                self.recv = torch.empty((w.N, w.H), dtype=torch.int8, device=dev)
                self.scale = torch.empty(w.N, dtype=torch.float32, device=dev)
                if smooth:
                    # per-expert smoothing scales, one per channel: exp(N(0, 0.25^2)), seeded
                    g = torch.Generator().manual_seed(w.seed * 1000 + 7)
                    self.smooth_scales = torch.exp(0.25 * torch.randn((w.E, w.H), generator=g)).to(dev)
                    # scratch of the sorted slot list
                    self.smooth_ws = torch.empty(max(1, mep.mep_dispatch_int8_smooth_workspace_size(w.T, w.K)),
                                                 dtype=torch.uint8, device=dev)
            else:
                self.recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
                self.y = self.recv
        if dedup:
            # the send buffer holds at most one row per slot; the plan decides how many
            self.db = mep.DedupBuffers.allocate(w.R, w.S, w.K, dev)
            self.sent = torch.empty((w.N, w.H), dtype=self.recv.dtype, device=dev)
            self.sent_scale = torch.empty(w.N, dtype=torch.float32, device=dev) if w.quant else None
        torch.cuda.synchronize()

    def phases(self):
        """The step's phases in launch order (each timed with its own CUDA events)."""
        ph = [("plan", self.plan), ("dispatch", self.dispatch)]
        if self.dedup:
            ph.append(("expand", self.expand))
        return ph + [("combine", self.combine)]

    def plan(self, s):
        w, mep = self.w, self.mep
        if w.mapping:
            mep.mep_update_expert_ranks(self.ids.view(w.T, w.K), self.table, self.gates.view(w.T, w.K),
                                        self.thr, self.active, w.R, 0, self.bids, self.bmask, stream=s)
            mep.mep_plan(self.bids.view(-1), w.R, self.n_keys, w.S, w.K, self.pb,
                         mode=mep.MEP_PLAN_GROUPED, keys_per_rank=w.place_per_rank,
                         keep=self.bmask.view(-1), stream=s)
            n = 1 + mep.mep_plan_launches(w.R, self.n_keys, w.S, w.K)
        else:
            mep.mep_plan(self.ids, w.R, w.E, w.S, w.K, self.pb, stream=s)
            n = mep.mep_plan_launches(w.R, w.E, w.S, w.K)
        if self.dedup:
            mep.mep_dedup_plan(self.pb.pos, self.pb.rank_off, w.R, w.S, w.K, self.db, stream=s)
            n += 6
        return n

    def dispatch(self, s):
        w = self.w
        pos, recv, scale = self.pb.pos, self.recv, (self.scale if w.quant else None)
        if self.dedup:
            pos, recv, scale = self.db.dsend, self.sent, self.sent_scale
        if w.quant and self.smooth:
            # the slots sorted by expert within chunks of tokens, then quantised along that list
            self.mep.mep_dispatch_int8_smooth_grouped(self.x, self.ids, pos, w.K, self.smooth_scales, recv, scale,
                                                      workspace=self.smooth_ws, stream=s)
            return 2 if self.smooth_grouped() else 1
        elif w.quant:
            self.mep.mep_dispatch(self.x, pos, w.K, recv, scale, quant=1, stream=s)
        else:
            self.mep.mep_dispatch(self.x, pos, w.K, recv, stream=s)
        return 1

    def expand(self, s):
        """Receiving side of the deduplicated dispatch: sent rows -> expert-grouped rows."""
        self.mep.mep_expand(self.sent, self.db.gidx, self.recv, src_scale=self.sent_scale,
                            dst_scale=self.scale if self.w.quant else None, stream=s)
        return 1

    def combine(self, s):
        if self.epilogue == "add_rmsnorm":
            self.mep.mep_combine_add_rmsnorm(self.y, self.pb.pos, self.gates, self.w.K, self.residual,
                                             self.gamma, 1e-6, self.out, self.y_norm, self.rstd,
                                             stream=s)
            return 1
        if self.w.quant:
            # the identity expert on int8 rows: the combine reads the codes and scales
            self.mep.mep_combine_int8(self.recv, self.scale, self.pb.pos, self.gates, self.w.K,
                                      self.out, stream=s)
        else:
            self.mep.mep_combine(self.y, self.pb.pos, self.gates, self.w.K, self.out, stream=s)
        return 1

    def step(self, s, ev=None):
        """One step; ev (len(phases()) + 1 events) brackets the phases."""
        n = 0
        for i, (_, run) in enumerate(self.phases()):
            if ev is not None:
                ev[i].record(s)
            n += run(s)
        if ev is not None:
            ev[-1].record(s)
        return n

    def result_ok(self) -> bool:
        """Closed form of the identity expert with gates summing to 1: every token whose
        K slots are all kept comes back as its expert row (compared as values)."""
        w = self.w
        if self.epilogue == "add_rmsnorm":
            ref = (self.x.float() + self.residual.float()).to(torch.bfloat16).float()
            return torch.equal(self.out.float(), ref) and bool(torch.isfinite(self.y_norm.float()).all())
        if w.mapping:
            return bool(torch.isfinite(self.out.float()).all())
        if w.quant and self.smooth:
            # codes and scale per slot: every kept slot's row reaches +-127 (or is all zero),
            # checked on 256 sampled rows; the combine output is finite
            rows = torch.randint(0, w.N, (256,), generator=torch.Generator().manual_seed(3)).to(self.dev)
            amax = self.recv[rows].abs().amax(dim=1)
            return bool(((amax == 127) | (amax == 0)).all()) and bool(torch.isfinite(self.out.float()).all())
        if w.quant:
            first = self.pb.pos.view(w.T, w.K)[:, 0].long()
            y_first = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=self.dev)
            self.mep.mep_dequantize(self.recv[first], self.scale[first], y_first)
            return torch.equal(self.out.float(), y_first.float())
        return torch.equal(self.out.float(), self.x.float())

    def smooth_grouped(self) -> bool:
        """Whether mep_dispatch_int8_smooth_grouped sorts the slots on this workload's
        shapes (two launches) rather than running the per-token kernel."""
        w = self.w
        return w.H % 4 == 0 and w.H <= 8192 and w.E <= 6000

    def kernel_name(self, step: str) -> str:
        """The library kernel that runs a step on this workload's shapes."""
        w = self.w
        if step == "combine":
            if self.epilogue == "add_rmsnorm":
                return "k_combine_add_rmsnorm_v8" if w.H % 8 == 0 else "k_combine_add_rmsnorm_scalar"
            if w.quant:
                if w.H % 16 == 0:
                    return "k_combine_int8_warp"
                return "k_combine_int8_v8" if w.H % 8 == 0 else "k_combine_int8_scalar"
            return "k_combine_v8" if w.H % 8 == 0 else "k_combine_scalar"
        if step == "expand":
            return "k_expand_warp" if w.H % 16 == 0 or (not w.quant and w.H % 8 == 0) else "k_expand_bytes"
        if w.quant and self.smooth:
            if self.smooth_grouped():
                return "k_dispatch_int8_smooth_grouped"
            if w.H % 4 == 0 and w.H // 4 <= 16 * 256:
                return "k_dispatch_int8_smooth_k"
            return "k_dispatch_int8_smooth_scalar"
        if w.quant:
            return "k_dispatch_int8_staged" if w.H % 16 == 0 else "k_dispatch_int8"
        return "k_dispatch_warp" if w.H % 8 == 0 else "k_dispatch_elem"

    def working_set_bytes(self) -> int:
        b = (self.x.numel() * 2 + self.recv.numel() * self.recv.element_size() +
             self.out.numel() * 2 + self.ids.numel() * 8)
        if self.dedup:
            b += self.sent.numel() * self.sent.element_size()
        return b

    def sent_rows(self) -> int:
        """Rows the deduplicated dispatch sends (read once, after the first plan)."""
        if self.n_sent is None:
            self.n_sent = int(self.db.drank_off[-1].item())
        return self.n_sent

    def bytes(self):
        """Algorithmic bytes per launch of dispatch and combine, and of the plan."""
        w = self.w
        row = 2 * w.H
        n_rows = int(self.pb.stats_dict()["n_kept"])
        if w.quant:
            disp = w.T * row + n_rows * w.H + 4 * n_rows + 4 * w.N
            if self.smooth:
                disp += 4 * w.N + 4 * w.E * w.H              # expert ids, smoothing scales
            comb = n_rows * w.H + 4 * n_rows + w.T * row + 8 * w.N
        else:
            disp = w.T * row + n_rows * row + 4 * w.N
            comb = n_rows * row + w.T * row + 8 * w.N
        if self.epilogue == "add_rmsnorm":
            comb += 2 * w.T * row + 4 * w.T + row   # residual in, normalised rows out, rstd, gamma
        plan = 16 * w.N
        out = {"plan": plan, "dispatch": disp, "combine": comb}
        if self.dedup:
            # send: x in, one row (and scale) per (token, rank) out; expand: every
            # expert-grouped row gathered from its sent row (read and write), gidx
            qrow = w.H if w.quant else row
            u = self.sent_rows()
            out["dispatch"] = w.T * row + u * qrow + (4 * u if w.quant else 0) + 4 * w.N
            out["expand"] = 2 * n_rows * qrow + (8 * n_rows if w.quant else 0) + 4 * n_rows
            out["plan"] += 24 * w.N
        return out


def dedup_summary(rt):
    """Rows the deduplicated dispatch sends against the slots it serves: the bytes that
    would cross to other ranks with and without the dedup encoding."""
    w = rt.w
    u = rt.sent_rows()
    kept = int(rt.pb.stats_dict()["n_kept"])
    qrow = w.H if w.quant else 2 * w.H
    return {"rows_sent": u, "slots": kept, "ratio": u / kept if kept else None,
            "transport_bytes": u * qrow, "transport_bytes_without_dedup": kept * qrow}


def maxvio(rt):
    """maxvio = max load / mean load - 1: over ranks before the plan (experts on their
    home ranks) and after it (the rows each rank receives), and over experts, from the
    plan summary through the library's mep_maxvio."""
    w = rt.w
    out = rt.mep.mep_maxvio(rt.pb.stats, w.S, w.K, rt.pb.hist.numel())
    return {k: (None if v != v else v) for k, v in out.items()}     # NaN (no slot kept) -> null


def weight_side(mep, rt, args, dev, stream):
    """The replica weight prefetch and the replica gradient reduce of the step's plan,
    with B = E/R slots per rank (MoonEP's training setting) and experts of H x ffn_dim.
    Timed separately from the routing step, with CUDA events over `steps` repetitions."""
    w = rt.w
    B = w.E // w.R
    D = w.H * args.ffn_dim
    cap = rt.pb.rep_key.shape[1]
    g = torch.Generator(device=dev).manual_seed(1)
    se = torch.empty((w.R, B), dtype=torch.int32, device=dev)
    rw = torch.empty((w.R, cap), dtype=torch.int32, device=dev)
    w_home = torch.randn((w.E, D), generator=g, device=dev).to(torch.bfloat16)
    w_slots = torch.empty((w.R * B, D), dtype=torch.bfloat16, device=dev)
    grad_home = torch.randn((w.E, D), generator=g, device=dev)
    grad_slots = torch.randn((w.R * B, D), generator=g, device=dev)
    reps = max(3, min(args.steps, 20))

    def prefetch():
        mep.mep_prefetch_plan(rt.pb, w.R, w.E, B, se, rw, stream=stream)
        mep.mep_prefetch_weights(w_home, se, w.R, B, w_slots, stream=stream)

    def reduce():
        mep.mep_grad_reduce(grad_home, grad_slots, se, w.R, B, stream=stream)

    out = {"B": B, "ffn_dim": args.ffn_dim, "bytes_per_expert_bf16": 2 * D}
    with torch.cuda.stream(stream):
        prefetch()
    stream.synchronize()
    used = int((se >= 0).sum().item())
    for name, fn, nbytes in [("prefetch", prefetch, 2 * 2 * D * used),
                             ("grad_reduce", reduce, None)]:
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
        stream.synchronize()
        t = e0.elapsed_time(e1) / reps
        if nbytes is None:
            experts = int(torch.unique(se[se >= 0]).numel())
            nbytes = 4 * D * (2 * experts + 2 * used)     # read+write home rows and slots
        out[name] = {"ms": t, "gbs": nbytes / (t * 1e-3) / 1e9, "bytes": nbytes}
    out["slots_used"] = used
    del w_home, w_slots, grad_home, grad_slots
    torch.cuda.empty_cache()
    return out


def e2e_route_host(mep, rt, w, dev, steps, pg):
    """End to end through the C ABI with host buffers: each step is one mep_route_host
    call (upload from pinned host memory, plan, dispatch, combine, download to pinned
    host memory, all on one stream). Three device buffer sets on three streams take the
    steps in turn, so one step's upload, another's kernels and a third's download overlap
    on the full-duplex link."""
    h = {k: v.contiguous().pin_memory() for k, v in rt.host.items()}
    quant = 1 if w.quant else 0
    sets = [mep.RouteBuffers.allocate(w.R, w.E, w.S, w.K, w.H, quant, dev) for _ in range(3)]
    structs = [b.c_struct() for b in sets]
    outs = [torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    streams = [torch.cuda.Stream(dev) for _ in range(3)]
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def run(n):
        torch.cuda.synchronize()
        first, last = ev(), ev()
        first.record(streams[0])
        for j in (1, 2):
            streams[j].wait_event(first)
        for i in range(n):
            j = i % 3
            mep.mep_route_host(sets[j], h["ids"], h["gates"], h["x"], outs[j], stream=streams[j],
                               c_struct=structs[j])
        for j in (1, 2):
            done = ev()
            done.record(streams[j])
            streams[0].wait_event(done)
        last.record(streams[0])
        torch.cuda.synchronize()
        return first.elapsed_time(last)

    run(3)
    if pg:
        pg.barrier()
    ms = max_over_ranks(run(steps) / steps, pg, dev)
    ok = torch.equal(outs[(steps - 1) % 3].view(torch.int16), rt.out.cpu().view(torch.int16))
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = outs[0].numel() * 2
    del sets
    return ms, ok, h2d, d2h, ("one mep_route_host call per step (C ABI, pinned host buffers): upload, "
                              "plan, dispatch, combine, download on one stream; three device buffer sets "
                              "on three streams in turn")


def link_rates(dev, nbytes: int = 1 << 30, reps: int = 5) -> dict:
    """This box's pinned host<->device copy rates in GB/s: upload alone, download alone,
    and each direction while both run on two streams (the end-to-end leg's bound)."""
    h_in = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    h_out = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d_a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_b = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)

    def up():
        s_up.wait_stream(cur)
        with torch.cuda.stream(s_up):
            d_a.copy_(h_in, non_blocking=True)
        cur.wait_stream(s_up)

    def down():
        s_down.wait_stream(cur)
        with torch.cuda.stream(s_down):
            h_out.copy_(d_b, non_blocking=True)
        cur.wait_stream(s_down)

    def both():
        s_up.wait_stream(cur)
        s_down.wait_stream(cur)
        with torch.cuda.stream(s_up):
            d_a.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(s_down):
            h_out.copy_(d_b, non_blocking=True)
        cur.wait_stream(s_up)
        cur.wait_stream(s_down)

    def gbs(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for _ in range(reps):
            fn()
        e1.record(cur)
        torch.cuda.synchronize(dev)
        return nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9

    out = {"h2d_gbs": gbs(up), "d2h_gbs": gbs(down), "duplex_gbs_each": gbs(both), "bytes": nbytes}
    del h_in, h_out, d_a, d_b
    torch.cuda.empty_cache()
    return out


def e2e_pipeline(rt, w, dev, stream, steps, pg):
    """End to end through the binding's calls for the steps mep_route_host does not cover
    (the mapping workload, the fused epilogue, the deduplicated dispatch): every step
    copies its inputs from pinned host memory to the device, routes them, and copies its
    result back to pinned host memory. Double-buffered device inputs/outputs on three
    streams (host-to-device, compute, device-to-host), so that step i+1's upload, step
    i's routing and step i-1's download overlap on the full-duplex link."""
    h = {k: v.pin_memory() for k, v in rt.host.items()}
    out_h = [torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = [dict(ids=rt.ids, gates=rt.gates, x=rt.x, out=rt.out)]
    slots.append({k: torch.empty_like(v) for k, v in slots[0].items()})
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def e2e_run(n):
        in_done, comp_done, out_done = [], [], []
        first, last = ev(), ev()
        first.record(s_in)
        for i in range(n):
            b = slots[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])      # slot i%2 inputs consumed
                b["ids"].copy_(h["ids"], non_blocking=True)
                b["gates"].copy_(h["gates"], non_blocking=True)
                b["x"].copy_(h["x"], non_blocking=True)
                in_done.append(ev())
                in_done[-1].record(s_in)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])         # slot i%2 output downloaded
            rt.ids, rt.gates, rt.x, rt.out = b["ids"], b["gates"], b["x"], b["out"]
            with torch.cuda.stream(stream):
                rt.step(stream)
            comp_done.append(ev())
            comp_done[-1].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                out_h[i % 2].copy_(b["out"], non_blocking=True)
                out_done.append(ev())
                out_done[-1].record(s_out)
        last.record(s_out)
        torch.cuda.synchronize()
        return first.elapsed_time(last)

    e2e_run(3)
    if pg:
        pg.barrier()
    ms = max_over_ranks(e2e_run(steps) / steps, pg, dev)
    ok = rt.result_ok() and torch.equal(out_h[(steps - 1) % 2].float(), rt.out.cpu().float())
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = out_h[0].numel() * 2
    return ms, ok, h2d, d2h, ("binding calls with copies from and to pinned host memory: uploads, "
                              "routing and downloads of consecutive steps overlap (two device buffer "
                              "sets, three streams)")


def time_route(mep, rt, args, dev, stream, pg, steps):
    """Warm-up, eager timed steps (per-phase CUDA events) and, with --graph, timed replays
    of the step captured as a CUDA graph (one event between replays). Returns a dict of
    per-step device times (max over ranks for the job time) and per-phase means."""
    names = [n for n, _ in rt.phases()]
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            rt.step(stream)
    stream.synchronize()
    mep.mep_get_error(clear=True, stream=stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # A working set that fits in L2 is flushed between steps (a 256 MB write, outside
    # the step's events); larger ones are not.
    flush = None
    if rt.working_set_bytes() < 2 * L2_BYTES:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    launches = 0
    local = dev.index or 0
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(steps):
                if flush is not None:
                    flush.fill_(i & 0xff)
                launches += rt.step(stream, evs[i])
            end.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        eager_steps = [e[0].elapsed_time(e[-1]) for e in evs]
        ms = start.elapsed_time(end) if flush is None else float(sum(eager_steps))
        err = mep.mep_get_error(clear=True, stream=stream)
        if err:
            raise RuntimeError(f"device error word {err:#x} after the timed steps")
        t_phase = {n: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs])) for i, n in enumerate(names)}
        ms_eager = max_over_ranks(ms, pg, dev) / steps

        # The same step captured once into a CUDA graph and replayed: the launches of a
        # step go to the GPU as one unit (this matters most for small, launch-bound
        # workloads).
        graph_ms, graph_steps = None, None
        if args.graph:
            g = torch.cuda.CUDAGraph()
            # thread-local capture: other threads (NCCL's watchdog, the clock sampler)
            # may make CUDA calls while this thread captures
            with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                rt.step(stream)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    g.replay()
            stream.synchronize()
            if pg:
                pg.barrier()
            torch.cuda.synchronize()
            gev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
            with torch.cuda.stream(stream):
                if flush is None:
                    for i in range(steps):
                        gev[i].record(stream)
                        g.replay()
                    gev[steps].record(stream)
                    stream.synchronize()
                    graph_steps = [gev[i].elapsed_time(gev[i + 1]) for i in range(steps)]
                    gms = gev[0].elapsed_time(gev[steps])
                else:
                    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    graph_steps = []
                    for i in range(steps):
                        flush.fill_(i & 0xff)
                        g0.record(stream)
                        g.replay()
                        g1.record(stream)
                        stream.synchronize()
                        graph_steps.append(g0.elapsed_time(g1))
                    gms = float(sum(graph_steps))
            torch.cuda.synchronize()
            if pg:
                pg.barrier()
            graph_ms = max_over_ranks(gms, pg, dev) / steps
            err = mep.mep_get_error(clear=True, stream=stream)
            if err:
                raise RuntimeError(f"device error word {err:#x} after the graph replays")
            del g
    per_step = graph_steps if graph_steps is not None else eager_steps
    return {
        "names": names, "t_phase": t_phase, "launches": launches, "ms_eager": ms_eager, "graph_ms": graph_ms,
        "ms_step": graph_ms if graph_ms is not None else ms_eager,
        "step_ms": {"median": float(statistics.median(per_step)), "min": float(min(per_step)),
                    "max": float(max(per_step)), "mean": float(np.mean(per_step)), "n": len(per_step),
                    "of": "cuda_graph_replay" if graph_steps is not None else "eager"},
        "flush": flush is not None, "clocks": clk.summary(),
    }


class EPRoute:
    """A balanced workload (bf16, or int8 rows with scales) routed as R expert-parallel ranks, each with its own
    tokens and its own receive buffer (a separate allocation on this GPU, reached through
    a device table of the R buffers' addresses, as peer mappings would be across GPUs).
    Plan: per source rank its histogram, then (the all-gather: every rank's row is
    already on this GPU) its share of the plan (mep_plan_rank). Dispatch: every source
    rank stores its rows into the ranks' buffers (mep_dispatch_ranks). Combine: every
    rank sums its tokens from the buffers they went to (mep_combine_ranks). The identity
    expert. The R ranks' calls of a phase run on R streams of their own, as R GPUs
    would run them side by side, and the phase ends when all have."""

    def __init__(self, mep, w, dev):
        if w.mapping:
            raise ValueError("the expert-parallel layout is measured on the balanced workloads")
        self.mep, self.w, self.dev = mep, w, dev
        ids, gates = synth.router(w)
        SK = w.S * w.K
        self.ids = torch.from_numpy(ids).to(dev).view(w.R, SK)
        self.gates = torch.from_numpy(gates).to(dev).view(w.R, SK)
        self.x = synth.hidden(w).to(dev)
        dt = torch.int8 if w.quant else torch.bfloat16
        self.bufs = [torch.empty((SK, w.H), dtype=dt, device=dev) for _ in range(w.R)]
        self.table = mep.rank_pointer_table(self.bufs, dev)
        self.quant = 1 if w.quant else 0
        self.scales = [torch.empty(SK, dtype=torch.float32, device=dev) for _ in range(w.R)] if w.quant else None
        self.scale_table = mep.rank_pointer_table(self.scales, dev) if w.quant else None
        self.hist = torch.empty((w.R, w.E), dtype=torch.int32, device=dev)
        self.rps = [mep.RankPlanBuffers.allocate(w.R, w.E, w.S, w.K, dev) for _ in range(w.R)]
        self.out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
        self.streams = [torch.cuda.Stream(dev) for _ in range(w.R)]

    def _side_by_side(self, s, call):
        """call(r, stream) for every rank on its own stream, after the work already on s;
        s then waits for all of them."""
        start = torch.cuda.Event()
        start.record(s)
        done = []
        for r, st in enumerate(self.streams):
            st.wait_event(start)
            call(r, st)
            e = torch.cuda.Event()
            e.record(st)
            done.append(e)
        for e in done:
            s.wait_event(e)

    def phases(self):
        return [("plan", self.plan), ("dispatch", self.dispatch), ("combine", self.combine)]

    def plan(self, s):
        w, mep = self.w, self.mep
        self._side_by_side(s, lambda r, st: mep.mep_histogram(self.ids[r], w.E, self.hist[r], stream=st))
        self._side_by_side(s, lambda r, st: mep.mep_plan_rank(self.ids[r], self.hist, w.R, w.E, w.S, w.K, r,
                                                              self.rps[r], stream=st))
        return w.R * 5           # a histogram, then k_tile_count, k_scan_cols, k_source_meta, k_rank

    def dispatch(self, s):
        w = self.w
        self._side_by_side(s, lambda r, st: self.mep.mep_dispatch_ranks(
            self.x[r * w.S:(r + 1) * w.S], self.rps[r].pos, w.K, self.table, w.S * w.K, quant=self.quant,
            scale_table=self.scale_table, stream=st))
        return w.R

    def combine(self, s):
        w = self.w
        self._side_by_side(s, lambda r, st: self.mep.mep_combine_ranks(
            self.table, self.rps[r].pos, self.gates[r], w.K, w.S * w.K, self.out[r * w.S:(r + 1) * w.S],
            quant=self.quant, scale_table=self.scale_table, stream=st))
        return w.R

    def step(self, s, ev=None):
        n = 0
        for i, (_, run) in enumerate(self.phases()):
            if ev is not None:
                ev[i].record(s)
            n += run(s)
        if ev is not None:
            ev[-1].record(s)
        return n

    def result_ok(self) -> bool:
        """The identity expert with gates summing to 1 returns every token's row (bf16);
        on int8 rows, every token whose slots carry the same codes returns their
        dequantised row (checked on the first slot's buffer row)."""
        if not self.quant:
            return torch.equal(self.out.float(), self.x.float())
        w = self.w
        pos0 = torch.stack([rp.pos.view(w.S, w.K)[:, 0] for rp in self.rps]).view(-1).long()
        SK = w.S * w.K
        rank, local = pos0 // SK, pos0 % SK
        codes = torch.stack([self.bufs[int(r)][int(l)] for r, l in zip(rank[:64].tolist(), local[:64].tolist())])
        scale = torch.stack([self.scales[int(r)][int(l)] for r, l in zip(rank[:64].tolist(), local[:64].tolist())])
        ref = torch.empty((64, w.H), dtype=torch.bfloat16, device=self.dev)
        self.mep.mep_dequantize(codes, scale, ref)
        return torch.equal(self.out[:64].float(), ref.float())

    def kernel_name(self, step: str) -> str:
        if self.quant:
            return {"plan": "k_rank", "dispatch": "k_dispatch_ranks_int8", "combine": "k_combine_ranks_int8"}[step]
        return {"plan": "k_rank", "dispatch": "k_dispatch_ranks_warp", "combine": "k_combine_ranks_v8"}[step]

    def working_set_bytes(self) -> int:
        return (self.x.numel() * 2 * 2 + sum(b.numel() * b.element_size() for b in self.bufs) +
                self.ids.numel() * 8)

    def bytes(self):
        """Algorithmic bytes of the phases: the same rows move as on one buffer."""
        w = self.w
        row = 2 * w.H
        if self.quant:
            return {"plan": 16 * w.N, "dispatch": w.T * row + w.N * w.H + 8 * w.N,
                    "combine": w.N * w.H + 4 * w.N + w.T * row + 8 * w.N}
        return {"plan": 16 * w.N, "dispatch": w.T * row + w.N * row + 4 * w.N,
                "combine": w.N * row + w.T * row + 8 * w.N}


def per_workload_ep_entry(mep, name, args, dev, stream, pg, peak, peak_kind):
    """The per_workload entry of a balanced workload in the expert-parallel layout
    (EPRoute): R receive buffers of their own, reached through a table of addresses."""
    w = synth.get(name)
    rt = EPRoute(mep, w, dev)
    steps = max(5, min(args.steps, 20))
    tm = time_route(mep, rt, args, dev, stream, pg, steps)
    roof, dc = roofline_of(rt, tm, peak, peak_kind)
    entry = {
        "workload": w.name + "_ep", "layout": "R receive buffers of their own through a device address table "
        "(mep_plan_rank, mep_dispatch_ranks, mep_combine_ranks); the all-gather of the histograms is a no-op on "
        "one GPU", "token_slots": w.N, "ms_per_step": tm["ms_step"],
        "token_slots_per_s": w.N / (tm["ms_step"] * 1e-3), "step_ms": tm["step_ms"],
        "breakdown_ms": tm["t_phase"], "dispatch_combine": dc,
        "roofline": {k: roof[k] for k in ("kernel", "phase", "achieved", "frac", "algorithmic_bytes", "traffic")},
        "launches_per_step": tm["launches"] // steps, "result_check": rt.result_ok(), "flush": tm["flush"],
        "clocks": tm["clocks"],
    }
    del rt
    torch.cuda.empty_cache()
    return entry


def roofline_of(rt, tm, peak, peak_kind):
    """The dominant HBM-bound phase (the slower of the moving phases) against the peak,
    with its algorithmic bytes; and the dispatch+combine rate over all moving phases."""
    w = rt.w
    ab = rt.bytes()
    t_phase = tm["t_phase"]
    moving = [n for n in tm["names"] if n != "plan"]
    dom = max(moving, key=lambda n: t_phase[n])
    achieved = ab[dom] / (t_phase[dom] * 1e-3) / 1e9
    kname = rt.kernel_name(dom)
    traffic, capture = captured_traffic(kname, w.name)
    t_move = sum(t_phase[n] for n in moving)
    dc_gbs = sum(ab[n] for n in moving) / (t_move * 1e-3) / 1e9
    roof = {"kernel": kname, "phase": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "algorithmic_bytes": ab[dom],
            "traffic": traffic, "traffic_capture": capture}
    dc = {"token_slots_per_s": w.N / (t_move * 1e-3), "hbm_gbs": dc_gbs, "frac_of_peak": dc_gbs / peak,
          "frac_of_8tbs_nominal": dc_gbs / 8000.0, "algorithmic_bytes": sum(ab[n] for n in moving)}
    return roof, dc


def per_workload_entry(mep, name, args, dev, stream, pg, peak, peak_kind, smooth: bool = False):
    """A shorter measurement of another workload for the `per_workload` block: the same
    timing method (graph replays, per-phase eager events), no end-to-end leg. With
    `smooth` (the int8 workload), the dispatch applies per-expert smoothing scales."""
    w = synth.get(name)
    rt = Route(mep, w, dev, smooth=smooth)
    steps = max(5, min(args.steps, 20))
    tm = time_route(mep, rt, args, dev, stream, pg, steps)
    roof, dc = roofline_of(rt, tm, peak, peak_kind)
    entry = {
        "workload": w.name + ("_smooth" if smooth else ""), "token_slots": w.N, "ms_per_step": tm["ms_step"],
        "token_slots_per_s": w.N / (tm["ms_step"] * 1e-3), "step_ms": tm["step_ms"],
        "breakdown_ms": tm["t_phase"], "dispatch_combine": dc,
        "roofline": {k: roof[k] for k in ("kernel", "phase", "achieved", "frac", "algorithmic_bytes", "traffic")},
        "launches_per_step": tm["launches"] // steps, "result_check": rt.result_ok(), "flush": tm["flush"],
        "clocks": tm["clocks"], "plan_stats": rt.pb.stats_dict(), "maxvio": maxvio(rt),
    }
    del rt
    torch.cuda.empty_cache()
    return entry


def run_gpu(args, w):
    import dispatch_combine_topk_b200 as mep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1 or ("MASTER_ADDR" in os.environ and "RANK" in os.environ):   # under torchrun
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    # every rank routes its own independent batch (different seed)
    if args.epilogue != "none" and (w.quant or w.mapping):
        raise SystemExit("--epilogue applies to the balanced bf16 workloads")
    if args.dedup and w.mapping:
        raise SystemExit("--dedup applies to the balanced workloads")
    if args.smooth and not w.quant:
        raise SystemExit("--smooth applies to the int8 workload")
    if args.smooth and args.dedup:
        # smoothed codes belong to a slot's expert, so one row per (token, rank) cannot
        # carry them for the other slots of that pair
        raise SystemExit("--smooth and --dedup do not combine: smoothed codes are per slot")
    rt = Route(mep, rank_workload(w, rank), dev, args.epilogue, dedup=bool(args.dedup),
               smooth=bool(args.smooth))
    stream = torch.cuda.Stream(dev)
    tm = time_route(mep, rt, args, dev, stream, pg, args.steps)
    weights = weight_side(mep, rt, args, dev, stream) if args.ffn_dim > 0 else None
    ok_device = rt.result_ok()

    e2e_steps = max(4, min(args.steps, 20))
    if args.no_e2e:
        e2e_ms, ok_e2e, h2d, d2h, how = None, None, None, None, "skipped (--no-e2e)"
    elif not w.mapping and args.epilogue == "none" and not args.dedup and not args.smooth:
        e2e_ms, ok_e2e, h2d, d2h, how = e2e_route_host(mep, rt, w, dev, e2e_steps, pg)
    else:
        e2e_ms, ok_e2e, h2d, d2h, how = e2e_pipeline(rt, w, dev, stream, e2e_steps, pg)
    torch.cuda.empty_cache()
    link = None
    if e2e_ms is not None:
        # the copies alone bound the end-to-end step: the larger direction at the duplex rate
        link = link_rates(dev)
        link["bound_ms"] = max(h2d, d2h) / (link["duplex_gbs_each"] * 1e9) * 1e3
        link["frac"] = link["bound_ms"] / e2e_ms

    line = None
    peak, peak_kind = load_peaks()
    if rank == 0:
        roof, dc = roofline_of(rt, tm, peak, peak_kind)
        ms_step = tm["ms_step"]
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, desc, _ = oracle_sample(w, cpu_sample_S(w, args.cpu_div))
            cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc, **host_info()}
        line = {
            "metric": METRIC,
            "value": world * w.N / (ms_step * 1e-3),
            "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "step_ms": tm["step_ms"],
            "timing": {"mode": "cuda_graph_replay" if tm["graph_ms"] is not None else "eager",
                       "graph_ms_per_step": tm["graph_ms"], "eager_ms_per_step": tm["ms_eager"]},
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8" if w.quant else "bf16", "data": "synthetic",
            "config": {"workload": w.name, "R": w.R, "E": w.E, "S": w.S, "K": w.K, "H": w.H,
                       "quant": "per-token dynamic int8 dispatch, combine of the int8 rows" if w.quant else "none",
                       "epilogue": args.epilogue, "dedup": bool(args.dedup), "smooth": bool(args.smooth),
                       "token_slots_per_gpu": w.N, "seed": w.seed, "parallelism": f"replicas{world}",
                       "l2": (f"working set {rt.working_set_bytes() / 1e6:.0f} MB "
                              + ("< 2x L2 (126 MB): L2 flushed between steps (256 MB write, "
                                 "not timed)" if tm["flush"] else
                                 "> 2x L2 (126 MB): inputs larger than L2, no flush"))},
            "breakdown_ms": tm["t_phase"],
            "dispatch_combine": dc,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": None if e2e_ms is None else {
                "value": world * w.N / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "path": how, "link": link},
            "result_check": {"device": ok_device, "e2e": ok_e2e},
            "gpu_launches": tm["launches"],
            "clocks": tm["clocks"],
            "plan_stats": rt.pb.stats_dict(),
            "maxvio": maxvio(rt),
            "replica_weights": weights,
            "dedup": dedup_summary(rt) if args.dedup else None,
        }
    del rt
    torch.cuda.empty_cache()
    # the other workloads, on every rank (each rank its own GPU), reported by rank 0
    others = [n for n in args.per_workload.split(",") if n] if args.per_workload != "none" else []
    per = {}
    for name in others:
        if name.endswith("_ep"):
            e = per_workload_ep_entry(mep, name[:-3], args, dev, stream, pg, peak, peak_kind)
            per[e["workload"]] = e
            continue
        if name.endswith("_smooth"):
            e = per_workload_entry(mep, name[:-7], args, dev, stream, pg, peak, peak_kind, smooth=True)
            e["variant"] = ("per-expert smoothing scales before the int8 quantisation, codes and scale per slot "
                            "(mep_dispatch_int8_smooth_grouped)")
            per[e["workload"]] = e
            continue
        if synth.get(name).name == w.name:
            continue
        e = per_workload_entry(mep, name, args, dev, stream, pg, peak, peak_kind)
        per[e["workload"]] = e
    if line is not None:
        line["per_workload"] = per or None
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
    ap.add_argument("--workload", default="int8")
    ap.add_argument("--per-workload", default="tiny,r8,map,skew,r8_ep,int8_ep,int8_smooth",
                    help="comma-separated workloads measured after the main one and reported under "
                         "per_workload (graph replays, no end-to-end leg); a name ending in _ep routes that "
                         "balanced workload in the expert-parallel layout, int8_smooth the int8 workload "
                         "with per-expert smoothing scales; 'none' to skip")
    ap.add_argument("--ref-div", type=int, default=16,
                    help="--impl reference: the oracle routes S/ref_div tokens per rank per step")
    ap.add_argument("--cpu-div", type=int, default=1,
                    help="cpu_baseline: the oracle routes S/cpu_div tokens per rank once")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (for profiling runs; the line then has no e2e)")
    ap.add_argument("--graph", type=int, default=1,
                    help="1: time the step as a replayed CUDA graph (per-kernel breakdown "
                         "still comes from the eager steps); 0: eager only")
    ap.add_argument("--dedup", type=int, default=0,
                    help="1: send one row per (token, destination rank) and expand on the "
                         "receiving side (mep_dedup_plan, mep_expand)")
    ap.add_argument("--smooth", type=int, default=0,
                    help="1 (int8 workload): per-expert smoothing scales before the int8 "
                         "quantisation, codes and scale per slot (mep_dispatch_int8_smooth_grouped)")
    ap.add_argument("--epilogue", default="none", choices=["none", "add_rmsnorm"],
                    help="add_rmsnorm: combine fused with residual add + RMSNorm")
    ap.add_argument("--ffn-dim", type=int, default=0,
                    help="> 0: also time the replica weight prefetch and gradient reduce with "
                         "experts of H x ffn_dim (MoonEP's benchmark uses 2048), B = E/R")
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
