"""Benchmark: draft+verify positions/s of spec_cycle on the B=64, K=16,
V=129280, r=256 bf16 workload (one fused launch per cycle).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Every rank runs its own batch of
B = 64 independent rows (weak scaling: batch rows are independent, so the
path needs no collective); `value` is the positions all ranks processed over
the slowest rank's device time.  Rank 0 prints one JSON line.

Timing: W >= 3 untimed cycles, then K timed cycles between a barrier and a
device synchronise on both sides, CUDA events on the launching stream; the
Philox cycle counter advances every cycle.  The logit inputs (546 MB) are
larger than L2; the Markov factor W is kept L2-resident by design.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft+verify positions/sec and HBM GB/s vs B200 peak at B=64 K=16 V=129280"
WORKLOAD = "c3"


def csrc_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "draft_sampling_verification_head_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def full_stream_bytes(w) -> int:
    """Logit bytes of a full read (K draft + K+1 target rows per batch row),
    W once, the gathered U rows: s*B*(2K+1)*V + s*r*V + s*B*K*r."""
    s = 2 if w.dtype == "bf16" else 4
    return s * w.B * (2 * w.K + 1) * w.V + s * w.r * w.V + s * w.B * w.K * w.r


def early_exit_bytes(w, tau) -> float:
    """Bytes the method must read when verification stops at the first
    rejection: all K draft rows, target rows 0..tau-1 (plus row K when every
    draft is accepted, already counted by tau = K+1), W once, U rows."""
    s = 2 if w.dtype == "bf16" else 4
    rows_t = float(sum(min(int(t), w.K + 1) for t in tau))
    return s * (w.B * w.K + rows_t) * w.V + s * w.r * w.V + s * w.B * w.K * w.r


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.samples = []
        self.proc = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-i",
                 str(self.idx), "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append([x.strip() for x in line.split(",")])

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[1]) for s in self.samples if len(s) > 8 and s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if len(s) > 8 and s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for s in self.samples if len(s) > 8
                          for j in range(4) if s[5 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(h):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source."""
    p = os.path.join(ROOT, "profiles", "k_cycle_c3_ncu.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    return d.get("dram_bytes_per_launch") if d.get("csrc_hash") == h else None


def cpu_baseline(w, d, max_seconds=20.0):
    """The oracle, as it stands, on a bounded sample of the workload's rows
    (host cores, OpenMP over rows); positions/s scaled to the sample."""
    import oracle
    oracle.build()
    P = oracle.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                      seed=w.seed, cycle=0)
    raw = [oracle_raw(d[k]) for k in ("base", "target", "U", "W")]
    lt = d["last_token"].numpy()
    cores = os.cpu_count() or 1
    rows, t_used, done = 0, 0.0, 0
    chunk = max(1, min(cores, w.B))
    while done < w.B and t_used < max_seconds:
        n = min(chunk, w.B - done)
        t0 = time.perf_counter()
        o = oracle.cycle(P, *raw, lt, b_begin=done, b_end=done + n)
        t_used += time.perf_counter() - t0
        done += n
        threads = o["threads"]
    return {"value": done * w.K / t_used, "unit": "positions/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{done} of {w.B} batch rows of one cycle (K={w.K}, V={w.V}, r={w.r}), "
                      f"{t_used:.1f} s of fp64 C oracle, OpenMP over rows"}


def oracle_raw(t):
    import synth
    return synth.to_numpy_raw(t)


def run_reference(args, rank, world):
    """The reference arm: the oracle (the only implementation of the method the
    pages have behind them) timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    import synth
    w = synth.WORKLOADS[WORKLOAD]
    d = synth.make(w)
    import oracle
    oracle.build()
    P = oracle.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                      seed=w.seed)
    raw = [oracle_raw(d[k]) for k in ("base", "target", "U", "W")]
    lt = d["last_token"].numpy()
    cores = os.cpu_count() or 1
    rows = max(1, min(cores, w.B))
    for c in range(args.warmup):
        P.cycle = c
        oracle.cycle(P, *raw, lt, b_begin=0, b_end=rows)
    t0 = time.perf_counter()
    threads = 1
    for c in range(args.steps):
        P.cycle = args.warmup + c
        o = oracle.cycle(P, *raw, lt, b_begin=0, b_end=rows)
        threads = o["threads"]
    dt = time.perf_counter() - t0
    value = rows * w.K * args.steps / dt
    line = {"metric": METRIC, "value": value, "unit": "positions/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "B=64 K=16 V=129280 r=256 bf16 logits, T=1.0, target noise sigma=0.5",
                       "sample_rows_per_step": rows, "parallelism": "host cores"},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "positions/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"{rows} of {w.B} batch rows per step, fp64 C oracle"},
            "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import synth
    import draft_sampling_verification_head_b200 as sd

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        import datetime
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    w = synth.WORKLOADS[WORKLOAD]
    d = synth.make(w, seed=w.seed + 1000 * rank)  # each rank its own batch of B rows
    dev = torch.device("cuda", local_rank)
    dd = {k: v.to(dev) for k, v in d.items()}
    p = sd.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                  seed=w.seed + rank, cycle=0)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p)
    stream = torch.cuda.current_stream()

    def step(c):
        p.cycle = c
        sd.cycle(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                 o["out"], o["tau"], o["p_draft"], o["q_draft"], ws)

    def barrier():
        if dist is not None:
            dist.barrier()

    for c in range(args.warmup):
        step(c)
    st = sd.sync_status(ws)
    if st != sd.SPEC_OK:
        raise RuntimeError(f"device status {sd.status_string(st)}")
    taus = []
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for c in range(args.steps):
            step(args.warmup + c)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    launches = args.steps  # one fused kernel per cycle
    st = sd.sync_status(ws)
    if st != sd.SPEC_OK:
        raise RuntimeError(f"device status {sd.status_string(st)}")
    tau = o["tau"].cpu().numpy()
    ms_t = torch.tensor([ms], device=dev)
    if dist is not None:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    per_step_ms = ms_max / args.steps
    positions = w.B * w.K * world * args.steps
    value = positions / (ms_max / 1e3)

    # end to end through the C-ABI with host buffers: pinned H2D of the step's
    # logits and last token, the fused call, D2H of the emitted tokens and tau
    hbase = d["base"].pin_memory()
    htarget = d["target"].pin_memory()
    hlast = d["last_token"].pin_memory()
    hout = torch.empty_like(o["out"], device="cpu").pin_memory()
    htau = torch.empty_like(o["tau"], device="cpu").pin_memory()
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step(c):
        dd["base"].copy_(hbase, non_blocking=True)
        dd["target"].copy_(htarget, non_blocking=True)
        dd["last_token"].copy_(hlast, non_blocking=True)
        step(c)
        hout.copy_(o["out"], non_blocking=True)
        htau.copy_(o["tau"], non_blocking=True)

    e2e_step(0)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for c in range(e2e_steps):
        e2e_step(10_000 + c)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([f0.elapsed_time(f1)], device=dev)
    if dist is not None:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = w.B * w.K * world * e2e_steps / (float(e2e_ms.item()) / 1e3)
    h2d = hbase.numel() * hbase.element_size() + htarget.numel() * htarget.element_size() + \
        hlast.numel() * hlast.element_size()
    d2h = hout.numel() * hout.element_size() + htau.numel() * htau.element_size()

    if rank == 0:
        peak, peak_kind = measured_peak()
        fb = full_stream_bytes(w)
        eb = early_exit_bytes(w, tau)
        h = csrc_hash()
        achieved = fb / (per_step_ms / 1e3) / 1e9  # GB/s, one launch per step
        line = {
            "metric": METRIC, "value": value, "unit": "positions/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded generator: N(0,2) + Zipf(1.1) prior, target = draft + N(0,0.5), U,W ~ N(0,0.02))",
            "config": {"workload": "B=64 K=16 V=129280 r=256 bf16 logits, T=1.0, target noise sigma=0.5",
                       "global_batch": w.B * world, "K": w.K, "V": w.V, "r": w.r,
                       "parallelism": f"batch-sharded x{world} (independent rows, no collective)",
                       "l2": "logit inputs 546 MB > L2; W L2-resident by design",
                       "mean_tau": float(tau.mean())},
            "gpu_launches": launches * world,
            "hbm_gbs_full_stream": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic(h),
                         "peak_kind": peak_kind,
                         "bytes_per_launch": fb, "early_exit_bytes_per_launch": eb,
                         "early_exit_achieved": eb / (per_step_ms / 1e3) / 1e9,
                         "kernel": "k_cycle (fused persistent draft+verify)"},
            "clocks": clk.summary(),
            "e2e": {"value": e2e_value, "unit": "positions/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
        }
        if world == 1:
            line["cpu_baseline"] = cpu_baseline(w, d)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
