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


def _strip_comments(src: str) -> str:
    """C/C++ source without comments or blank lines (string literals in the
    kernels hold no comment markers)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(l.rstrip() for l in src.splitlines() if l.strip())


# the sources each profiled kernel is built from (besides the shared headers)
PROFILED_SOURCES = {"k_cycle_tc_c3": ("cycle_tc.cu",), "k_verify_ee_c3": ("verify_ee.cu",)}
SHARED_HEADERS = ("common.cuh", "kernels.cuh")


def csrc_hash(files=None, root: str = ROOT) -> str:
    """Fingerprint of CUDA sources, comments excluded: the given kernel files
    and the shared headers, or every .cu / .cuh file.  A recorded ncu traffic
    figure stays valid while the code it measured is unchanged.  Host-only C++
    (.cpp) launches nothing and is left out."""
    h = hashlib.sha256()
    csrc = os.path.join(root, "draft_sampling_verification_head_b200", "csrc")
    if files is None:
        paths = glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))
    else:
        paths = [os.path.join(csrc, f) for f in (*files, *SHARED_HEADERS)]
    for f in sorted(paths):
        h.update(os.path.basename(f).encode())
        h.update(_strip_comments(open(f, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def kernel_hash(name: str, root: str = ROOT) -> str:
    """csrc_hash of the sources of one profiled kernel."""
    return csrc_hash(PROFILED_SOURCES[name], root)


def full_stream_bytes(w) -> int:
    """Logit bytes of a full read (K draft + K+1 target rows per batch row),
    W once, the gathered U rows: s*B*(2K+1)*V + s*r*V + s*B*K*r."""
    s = 2 if w.dtype == "bf16" else 4
    return s * w.B * (2 * w.K + 1) * w.V + s * w.r * w.V + s * w.B * w.K * w.r


def w_l2_bytes(w, num_sms: int, greedy: bool = False) -> int:
    """W bytes the fused cycle streams from L2 per launch on the tensor-core
    path: each CTA owns ceil(ceil(V/128)/SMs) 128-token chunks, keeps the
    first three chunks' W^T in tensor memory, and streams the rest once per
    MMA round (K draft steps, plus the final step when stochastic)."""
    s = 2 if w.dtype == "bf16" else 4
    nchunks = -(-w.V // 128)
    nc = -(-nchunks // num_sms)
    G = -(-nchunks // nc)
    streamed = sum(max(0, min(nc, nchunks - c * nc) - min(3, nc)) for c in range(G))
    rounds = w.K + (0 if greedy else 1)
    return streamed * 128 * w.r * s * rounds


def early_exit_bytes(w, tau) -> float:
    """Bytes the method must read when verification stops at the first
    rejection: all K draft rows, target rows 0..tau-1 (plus row K when every
    draft is accepted, already counted by tau = K+1), W once, U rows."""
    s = 2 if w.dtype == "bf16" else 4
    rows_t = float(sum(min(int(t), w.K + 1) for t in tau))
    return s * (w.B * w.K + rows_t) * w.V + s * w.r * w.V + s * w.B * w.K * w.r


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms from before
    the warm-up to after the timed region; the summary keeps the samples read
    between mark_start() and mark_end() (host clock), and when that window
    holds fewer than two (a timed region shorter than the sampling period) the
    nearest sample on each side of it."""

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.samples = []  # (host time, fields)
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-i",
                 str(self.idx), "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t_end = time.time() + 5.0  # the first sample before anything is timed
            while not self.samples and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.02)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        ok = [(t, f) for t, f in self.samples if len(f) > 8]
        if self.t0 is None or self.t1 is None:
            ok = []
        rows = [f for t, f in ok if self.t0 <= t <= self.t1]
        window = "timed region"
        if len(rows) < 2 and ok:
            before = [(t, f) for t, f in ok if t < self.t0]
            after = [(t, f) for t, f in ok if t > self.t1]
            rows = ([before[-1][1]] if before else []) + rows + ([after[0][1]] if after else [])
            window = "timed region and the nearest sample on each side"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        num = lambda x: x.replace(".", "", 1).isdigit()
        sm = [float(f[1]) for f in rows if num(f[1])]
        mx = [float(f[2]) for f in rows if num(f[2])]
        pw = [float(f[3]) for f in rows if num(f[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for f in rows for j in range(4) if f[5 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w": statistics.median(pw) if pw else None, "samples": len(rows),
                "window": window}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(h, name="k_cycle_tc_c3"):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel source with hash h (kernel_hash(name) for the current one)."""
    p = os.path.join(ROOT, "profiles", f"{name}_ncu.json")
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
    outs = []
    while done < w.B and t_used < max_seconds:
        n = min(chunk, w.B - done)
        t0 = time.perf_counter()
        o = oracle.cycle(P, *raw, lt, b_begin=done, b_end=done + n)
        t_used += time.perf_counter() - t0
        done += n
        threads = o["threads"]
        outs.append(o)
    ref = {k: __import__("numpy").concatenate([o[k] for o in outs])
           for k in ("out", "tau", "flag_draft", "flag_accept", "flag_final")}
    return {"value": done * w.K / t_used, "unit": "positions/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{done} of {w.B} batch rows of one cycle (K={w.K}, V={w.V}, r={w.r}), "
                      f"{t_used:.1f} s of fp64 C oracle, OpenMP over rows"}, ref


def near_threshold(ref, out, tau, K):
    """Rows of the oracle sample whose outcome depends on a near-threshold
    decision (a draft or accept decision flagged at or before the stop row, or
    a flagged final draw: counted, not compared), and unflagged rows whose
    emitted tokens or tau differ from the oracle's (expected 0)."""
    flagged = mism = 0
    for b in range(len(ref["tau"])):
        stop = int(ref["tau"][b]) - 1
        limit = min(int(ref["flag_draft"][b]), int(ref["flag_accept"][b]))
        if limit <= min(stop, K - 1) or ref["flag_final"][b]:
            flagged += 1
        elif int(tau[b]) != int(ref["tau"][b]) or list(out[b]) != list(ref["out"][b]):
            mism += 1
    return {"rows_checked": int(len(ref["tau"])), "flagged": flagged, "mismatched_unflagged": mism}


def oracle_raw(t):
    import synth
    return synth.to_numpy_raw(t)


def run_reference(args, rank, world):
    """The reference arm: the oracle (the only implementation of the method the
    pages have behind them) timed on the host cores, rank 0 only.

    A step is one batch row's whole cycle (K draft positions and their
    verification), the smallest unit the oracle works in; the oracle runs
    rows in parallel over the host cores, so consecutive steps are handed to it
    in chunks of as many rows as there are cores.  That keeps a run of
    thousands of steps within a few minutes."""
    if rank != 0:
        return
    import synth
    w = synth.WORKLOADS[args.workload]
    d = synth.make(w)
    import oracle
    oracle.build()
    P = oracle.Params(B=w.B, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                      seed=w.seed)
    raw = [oracle_raw(d[k]) for k in ("base", "target", "U", "W")]
    lt = d["last_token"].numpy()
    cores = os.cpu_count() or 1
    chunk = max(1, min(cores, w.B))

    def rows(total, first_cycle):
        done, threads = 0, 1
        while done < total:
            b0 = done % w.B
            n = min(chunk, w.B - b0, total - done)
            P.cycle = first_cycle + done // w.B
            threads = oracle.cycle(P, *raw, lt, b_begin=b0, b_end=b0 + n)["threads"]
            done += n
        return threads

    rows(args.warmup, 0)
    t0 = time.perf_counter()
    threads = rows(args.steps, 1000)
    dt = time.perf_counter() - t0
    value = w.K * args.steps / dt
    line = {"metric": metric_name(args.workload, "cycle", 1), "value": value,
            "unit": "positions/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[args.workload], "call": CALL_TEXT["cycle"],
                       "sample_rows_per_step": 1, "rows_per_oracle_call": chunk,
                       "parallelism": "host cores"},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "positions/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"one batch row of {w.B} per step (its K={w.K} positions), "
                                       f"{chunk} rows per fp64 C oracle call over the host cores"},
            "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


WORKLOAD_TEXT = {
    "c3": "B=64 K=16 V=129280 r=256 bf16 logits, T=1.0, target noise sigma=0.5",
    "c4": "B=256 K=8 V=151936 r=256 bf16 logits, T=1.0, target noise sigma=0.5",
    "c5": "B=128 K=32 V=129280 r=256 bf16 logits, T=1.0, target noise sigma 0.2..1.5 over rows",
}

CALL_TEXT = {
    "cycle": "spec_cycle: drafting and verification fused in one persistent launch per cycle",
    "loop": "spec_decode_loop: C chained cycles per persistent launch",
    "verify": "spec_verify_block: verification of given drafts (draft logits and tokens as inputs)",
    "draft": "spec_markov_bias_sample: sequential Markov-biased drafting only",
    "rnn": "spec_cycle_rnn: the fused cycle with the RNN sequential head (Wh ~ N(0, 1/r))",
}


def metric_name(workload, call, cycles):
    if workload == WORKLOAD and call == "cycle":
        return METRIC
    w = {"c3": "B=64 K=16 V=129280", "c4": "B=256 K=8 V=151936",
         "c5": "B=128 K=32 V=129280"}[workload]
    what = {"cycle": "draft+verify positions/sec", "loop": f"draft+verify positions/sec ({cycles} chained cycles per launch)",
            "rnn": "draft+verify positions/sec (RNN sequential head)",
            "verify": "verified positions/sec", "draft": "drafted positions/sec"}[call]
    return f"{what} and HBM GB/s vs B200 peak at {w}"


def draft_only_bytes(w) -> int:
    """Bytes of the draft-only call: every base logit row, W once, the U rows."""
    s = 2 if w.dtype == "bf16" else 4
    return s * w.B * w.K * w.V + s * w.r * w.V + s * w.B * w.K * w.r


def verify_bytes(w, tau) -> float:
    """Bytes the verification of one batch must read with the early exit: a row
    stopping at position j (tau = j + 1) needs draft and target rows 0..j (the
    stop row twice: statistics, then the residual draw); a row accepting all K
    needs draft rows 0..K-1 and target rows 0..K."""
    s = 2 if w.dtype == "bf16" else 4
    rows = 0.0
    for t in tau:
        t = int(t)
        rows += (2 * w.K + 1) if t == w.K + 1 else (2 * t + 2)
    return s * rows * w.V


def run_ours(args, rank, world, local_rank):
    import torch
    import synth
    import draft_sampling_verification_head_b200 as sd

    from draft_sampling_verification_head_b200 import shard

    torch.cuda.set_device(local_rank)
    multi = shard.init("nccl", timeout_s=120)
    w = synth.WORKLOADS[args.workload]
    call, C = args.call, (args.cycles if args.call == "loop" else 1)
    # Weak scaling: the job's batch is world x B rows; rank r holds rows
    # [r*B, (r+1)*B) (its own seeded logits) and draws with row_offset r*B.
    row0, row1 = shard.shard_range(w.B * world, world, rank)
    if call == "loop":
        d = synth.make_loop(w, C, seed=w.seed + 1000 * rank)
    else:
        d = synth.make(w, seed=w.seed + 1000 * rank)
    dev = torch.device("cuda", local_rank)
    dd = {k: v.to(dev) for k, v in d.items()}
    p = sd.Params(B=row1 - row0, K=w.K, V=w.V, r=w.r, dtype=w.dtype, temperature=w.temperature,
                  seed=w.seed, cycle=0, row_offset=row0)
    ws = sd.make_workspace(p)
    o = sd.alloc_outputs(p, n_cycles=C if call == "loop" else None)
    stream = torch.cuda.current_stream()
    nt = torch.empty(p.B, dtype=torch.int32, device=dev)
    if call == "verify":
        # inputs of the verification: draft tokens and their (biased) draft
        # logits, made once by the library's drafting call (untimed setup)
        biased = torch.empty((p.B, w.K, w.V), dtype=torch.float32, device=dev)
        sd.markov_bias_sample(p, dd["base"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                              None, biased, ws)
        dd["draft_logits"] = biased.to(torch.bfloat16)
        dd["draft"] = o["draft"].clone()
        del biased
        if sd.sync_status(ws) != sd.SPEC_OK:
            raise RuntimeError("drafting for the verify inputs failed")
    if call == "rnn":
        dd["Wh"] = synth.rnn_weights(w).to(dev)
    if call == "loop" and args.schedule:
        # verify lengths from the host scheduler (untimed setup): the stand-in
        # confidence scores and a stand-in steps-per-second table of a target
        # pass over m rows -- flat up to half of the full B (K+1) rows, then
        # falling as 1 / m (a serving engine would profile it once at start-up)
        import numpy as np
        full = p.B * (w.K + 1)
        m = np.arange(full + 1, dtype=np.float64)
        sps = 1.0 / np.maximum(m, full / 2)
        conf = d["conf"].numpy()
        dd["vlen"] = torch.as_tensor(
            np.stack([sd.schedule_verify_len(conf[c], sps)[0] for c in range(C)])).to(dev)
    tau_shape = (C, p.B) if call == "loop" else (p.B,)
    tau_all = torch.zeros((max(1, args.steps),) + tau_shape, dtype=torch.int32, device=dev)

    def step(c, tau=None):
        tau = o["tau"] if tau is None else tau
        if call == "cycle":
            p.cycle = c
            sd.cycle(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                     o["out"], tau, o["p_draft"], o["q_draft"], ws)
        elif call == "loop":
            p.cycle = c * C
            if args.schedule:
                sd.decode_loop(p, C, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"],
                               o["draft"], o["out"], tau, o["p_draft"], o["q_draft"], nt, ws,
                               verify_len=dd["vlen"])
            else:
                sd.decode_loop(p, C, dd["base"], dd["target"], dd["U"], dd["W"], dd["last_token"],
                               o["draft"], o["out"], tau, o["p_draft"], o["q_draft"], nt, ws,
                               conf=dd["conf"], conf_threshold=args.conf_threshold)
        elif call == "rnn":
            p.cycle = c
            sd.cycle_rnn(p, dd["base"], dd["target"], dd["U"], dd["W"], dd["Wh"], dd["last_token"],
                         o["draft"], o["out"], tau, o["p_draft"], o["q_draft"], ws)
        elif call == "verify":
            p.cycle = c
            sd.verify_block(p, dd["target"], dd["draft_logits"], dd["draft"], o["out"], tau,
                            o["p_draft"], o["q_draft"], ws)
        else:
            p.cycle = c
            sd.markov_bias_sample(p, dd["base"], dd["U"], dd["W"], dd["last_token"], o["draft"],
                                  o["q_draft"], None, ws)

    barrier = shard.barrier

    with ClockSampler(local_rank) as clk:
        step(0)  # the first cycle: its outputs are compared with the oracle's sample below
        out0, tau0 = o["out"].cpu().numpy(), o["tau"].cpu().numpy()
        for c in range(1, args.warmup):
            step(c)
        st = sd.sync_status(ws)
        if st != sd.SPEC_OK:
            raise RuntimeError(f"device status {sd.status_string(st)}")
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clk.mark_start()
        e0.record(stream)
        for c in range(args.steps):
            step(args.warmup + c, tau_all[c])
        e1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
        barrier()
    ms = e0.elapsed_time(e1)
    launches = args.steps * sd.last_launch_count()
    st = sd.sync_status(ws)
    if st != sd.SPEC_OK:
        raise RuntimeError(f"device status {sd.status_string(st)}")
    tau = tau_all.cpu().numpy().reshape(-1, p.B)  # every timed cycle
    ms_max = shard.max_over_ranks(ms)
    per_step_ms = ms_max / args.steps
    per_step = p.B * w.K * C
    positions = shard.sum_over_ranks(per_step * args.steps)
    value = positions / (ms_max / 1e3)

    # end to end through the C-ABI with host buffers: pinned H2D of the step's
    # inputs, the call, D2H of the emitted tokens and tau
    ins = {"cycle": ("base", "target", "last_token"), "rnn": ("base", "target", "last_token"),
           "loop": ("base", "target", "last_token", "conf"),
           "verify": ("target", "draft_logits", "draft"), "draft": ("base", "last_token")}[call]
    if call == "loop" and args.schedule:
        ins = ("base", "target", "last_token", "vlen")  # the host scheduler's lengths go in
    outs = ("draft",) if call == "draft" else ("out", "tau")
    hin = {k: dd[k].cpu().pin_memory() for k in ins}
    hout = {k: torch.empty_like(o[k], device="cpu").pin_memory() for k in outs}
    e2e_steps = 20

    def e2e_step(c):
        for k in ins:
            dd[k].copy_(hin[k], non_blocking=True)
        step(c)
        for k in outs:
            hout[k].copy_(o[k], non_blocking=True)

    e2e_step(0)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for c in range(e2e_steps):
        e2e_step(10_000 + c)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = shard.max_over_ranks(f0.elapsed_time(f1))
    e2e_value = shard.sum_over_ranks(per_step * e2e_steps) / (e2e_ms / 1e3)
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = sum(t.numel() * t.element_size() for t in hout.values())

    if rank == 0:
        peak, peak_kind = measured_peak()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        if call in ("cycle", "loop", "rnn"):
            fb = full_stream_bytes(w) * C
            eb = sum(early_exit_bytes(w, t) for t in tau) / len(tau) * C
            wl2 = w_l2_bytes(w, sms) * C
            kernel = "k_cycle_tc (fused persistent draft+verify, tensor-core path)"
        elif call == "verify":
            fb = 2 * w.B * (2 * w.K + 1) * w.V  # every draft and target row
            eb = sum(verify_bytes(w, t) for t in tau) / len(tau)
            wl2 = 0
            kernel = "verify kernels (spec_verify_block)"
        else:
            fb = eb = draft_only_bytes(w)
            wl2 = w_l2_bytes(w, sms, greedy=True)
            kernel = "draft kernel (spec_markov_bias_sample)"
        prof = {"cycle": "k_cycle_tc_c3", "verify": "k_verify_ee_c3"}.get(call)
        achieved = fb / (per_step_ms / 1e3) / 1e9  # GB/s over the step
        cfg = {"workload": WORKLOAD_TEXT[args.workload], "call": CALL_TEXT[call],
               "global_batch": w.B * world, "K": w.K, "V": w.V, "r": w.r,
               "parallelism": f"batch-sharded x{world} (independent rows, no collective)",
               "l2": "logit inputs > L2 (no flush between steps); W^T of 3 of each CTA's "
                     "128-token chunks held in tensor memory, the rest streamed from L2"}
        if call == "loop":
            cfg.update({"cycles_per_launch": C, "conf_threshold": args.conf_threshold,
                        "conf": "uniform(0.5, 1.0) per position (stand-in scores)"})
            if args.schedule:
                cfg.update({"conf_threshold": None,
                            "verify_len": "spec_schedule_verify_len per cycle from the scores and a "
                                          "stand-in steps-per-second table (flat to half of B (K+1) "
                                          "rows, then 1/m)",
                            "mean_verify_len": float(dd["vlen"].float().mean())})
        if call != "draft":
            cfg.update({"mean_tau": float(tau.mean()), "tau_cycles": int(tau.shape[0]),
                        "emitted_tokens_per_s": float(tau.sum()) / args.steps / (per_step_ms / 1e3)})
        line = {
            "metric": metric_name(args.workload, call, C), "value": value, "unit": "positions/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded generator: N(0,2) + Zipf(1.1) prior, target = draft + N(0,sigma), U,W ~ N(0,0.02))",
            "config": cfg,
            "gpu_launches": launches * world,
            "rows_per_rank": p.B,
            "hbm_gbs_full_stream": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "traffic": (recorded_traffic(kernel_hash(prof), prof)
                                     if (call in ("cycle", "verify") and args.workload == WORKLOAD) else None),
                         "peak_kind": peak_kind,
                         "bytes_per_launch": fb, "early_exit_bytes_per_launch": eb,
                         "early_exit_achieved": eb / (per_step_ms / 1e3) / 1e9,
                         "frac_vs_nominal_8000": achieved / 8000.0,
                         "w_from_l2_bytes_per_launch": wl2,
                         "w_from_l2_achieved_gbs": wl2 / (per_step_ms / 1e3) / 1e9,
                         "kernel": kernel},
            "clocks": clk.summary(),
            "e2e": {"value": e2e_value, "unit": "positions/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
        }
        if world == 1 and call == "cycle":
            if args.no_cpu_baseline:
                line["cpu_baseline"] = None
            else:
                cb, ref = cpu_baseline(w, d)
                line["cpu_baseline"] = cb
                line["near_threshold"] = near_threshold(ref, out0, tau0, w.K)
        print(json.dumps(line), flush=True)
    if multi:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the timed oracle sample (profiling runs)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(WORKLOAD_TEXT),
                    help="c3 is the headline configuration")
    ap.add_argument("--call", default="cycle", choices=sorted(CALL_TEXT),
                    help="which entry point one step runs (cycle: the headline)")
    ap.add_argument("--cycles", type=int, default=4, help="cycles per launch for --call loop")
    ap.add_argument("--schedule", action="store_true",
                    help="--call loop: verify lengths chosen by spec_schedule_verify_len")
    ap.add_argument("--conf-threshold", type=float, default=0.0,
                    help="prefix-survival threshold for --call loop (0: every K_b = K)")
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
