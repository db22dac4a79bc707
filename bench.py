"""Benchmark of the GDN mixer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extra]

Headline (``value``): prefill token-heads/s (B x T x H per second) of gdn_chunk_fwd on the
prefill workload B=2, H=16, T=4096, dk=dv=128, bf16 q/k/v, fp32 g/beta/state, S0 = 0,
chunk 64 -- one launch of the tensor-core chunked kernel per step, inputs resident in HBM,
three input sets rotated so that every step reads from DRAM (3 x 137 MB > 126 MB L2).
Secondary workloads measured in the same run (``other_workloads``): decode (256 x 32
heads, 100 in-place steps), long prefill (T=32768, H=32, S0 != 0), full mixer (4 packed
sequences, prep -> chunk -> out gate), full-mixer decode step, backward, and the input
projections fused with prep (gdn_inproj_prep, D = 2048).

N > 1: one process per GPU (torchrun), every rank runs its own batch (independent
sequences, no data-path collective: weak scaling); time = max over ranks.
``--impl reference``: the fp64 CPU oracle on the host cores, same metric and workload,
each step a bounded sample; rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (B×T×H, dk=dv=128) + decode state-updates/s; % roofline"
UNIT = "token-heads/s"


from linear_attention_token_gdn_b200.dist import aggregate, env_rank, rank_seed  # noqa: E402
from linear_attention_token_gdn_b200 import dist as gdist  # noqa: E402


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d.get("bf16_tflops"), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        # raw samples: $GDN_CLOCKS_DIR/clocks_rank<i>.csv when that directory is set, else /tmp
        out_dir = os.environ.get("GDN_CLOCKS_DIR")
        self.path = (os.path.join(out_dir, f"clocks_rank{gpu_index}.csv") if out_dir and os.path.isdir(out_dir)
                     else f"/tmp/gdn_clocks_{os.getpid()}_{gpu_index}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.idx), "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        sm = [float(r[1]) for r in rows]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ----------------------------------------------------------------------------- helpers

def prefill_bytes(N, H, nseq, dk=128, dv=128, in_bytes=2, y_bytes=2, S0=False, S_T=True):
    """Algorithmic HBM bytes of one gdn_chunk_fwd launch: read q, k, v, g, beta (+S0),
    write y (+S_T), each exactly once."""
    b = N * H * ((2 * dk + dv) * in_bytes + 8 + dv * y_bytes)
    state = nseq * H * dk * dv * 4
    return b + (state if S0 else 0) + (state if S_T else 0)


def timed(torch, fn, steps, warmup, stream, on_start=None):
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    if on_start is not None:
        on_start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3  # seconds


def kernel_split(torch, gdn, fn, steps, stream, max_launches=64):
    """Per-kernel device times from a separate pass with the library's launch timing on.  Its
    events bracket every launch, which cancels the programmatic dependent launch between the
    chunked pass's two kernels, so the reported times come from un-instrumented passes and this
    table only splits a call into its kernels."""
    timed(torch, fn, steps, 0, stream, on_start=lambda: gdn.timing_start(max_launches))
    return kernel_table(gdn.timing_stop(), steps)


def kernel_table(per_kernel, steps):
    """{name: (launches, total ms)} from gdn.timing_stop -> per-kernel averages and shares."""
    tot = sum(ms for _, ms in per_kernel.values()) or 1.0
    return [{"name": n, "launches": c, "avg_us": ms * 1e3 / max(c, 1), "share": ms / tot}
            for n, (c, ms) in per_kernel.items()]


def traffic_per_call():
    """DRAM bytes (read + write) of one gdn_chunk_fwd call on the headline workload, from the
    ncu capture summarised in profiles/ -- or None when the kernel source has changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "chunk_fwd_prefill_B2_H16_T4096.md")
    if not os.path.exists(path):
        return None
    src = b"".join(open(os.path.join(ROOT, "linear_attention_token_gdn_b200", "csrc", f), "rb").read()
                   for f in ("chunk_tc.cuh", "tc_ptx.cuh", "common.cuh", "warp_mma.cuh"))
    digest = hashlib.sha256(src).hexdigest()[:16]
    fields = {}
    for line in open(path):
        if line.startswith("traffic:"):
            for kv in line.split()[1:]:
                k, _, v = kv.partition("=")
                fields[k] = v
    if fields.get("source_sha256") != digest:
        return None
    try:
        return int(fields["bytes_per_call"])
    except (KeyError, ValueError):
        return None


def max_over_ranks(torch, dist, x, world):
    return gdist.max_over_ranks(x, world, device="cuda")


def barrier(torch, dist, world):
    gdist.barrier(world, cuda=True)


# ----------------------------------------------------------------------------- CPU baseline

def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


_CPU_INPUTS = {}


def cpu_baseline(workload=None, target_s=12.0):
    """The fp64 oracle (unmodified) on the host cores, on a bounded sample of the prefill
    workload: the first `nh` heads of every sequence (all of them, repeated, when the whole
    workload takes less than target_s), sized to ~target_s of wall time.  Also reports the
    single-threaded rate of the calibration run."""
    import oracle
    from linear_attention_token_gdn_b200 import inputs

    workload = inputs.PREFILL if workload is None else workload
    c = inputs.WORKLOAD_SPECS[workload]
    if workload not in _CPU_INPUTS:  # generated once per process (the reference arm calls this per step)
        _CPU_INPUTS[workload] = inputs.make_prefill(workload, "cpu")
    x = _CPU_INPUTS[workload]
    ncores = os.cpu_count() or 1
    # calibrate: one (sequence, head) unit single-threaded on a 512-token slice
    T = c["T"]
    sl = slice(0, 512)
    t0 = time.perf_counter()
    oracle.recurrence(x["q"][sl, :1], x["k"][sl, :1], x["v"][sl, :1], x["g"][sl, :1], x["beta"][sl, :1], nthreads=1)
    per_tok = (time.perf_counter() - t0) / 512
    units_budget = max(1, int(target_s * ncores / (per_tok * T)))
    nh = max(1, min(c["H"], units_budget // c["B"]))
    reps = max(1, units_budget // (c["B"] * c["H"])) if nh == c["H"] else 1
    hs = slice(0, nh)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.recurrence(x["q"][:, hs], x["k"][:, hs], x["v"][:, hs], x["g"][:, hs], x["beta"][:, hs], None,
                          x["cu_seqlens"], nthreads=0)
    dt = time.perf_counter() - t0
    used = oracle.threads_used(0, c["B"] * nh)
    work = c["B"] * T * nh * reps
    return {"value": work / dt, "unit": UNIT, "cores": used, "kind": "oracle", "cpu_model": cpu_model(),
            "single_thread_value": 1.0 / per_tok,
            "sample": f"prefill B={c['B']} T={T} heads 0..{nh - 1} of {c['H']}, {reps} pass(es) (dk=dv=128, "
                      f"fp64 C oracle, {dt:.1f} s wall on {used} threads); single-threaded rate from one "
                      f"head's first 512 tokens"}


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    cb = None
    times = []
    # each step a bounded sample: the whole run stays near 2.5 minutes of host time
    step_s = min(args.ref_step_s, max(0.5, 150.0 / (args.warmup + args.steps)))
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(target_s=step_s)
        if i >= args.warmup:
            times.append(1.0 / r["value"])
            cb = r
    value = cb["value"] if len(times) == 1 else len(times) / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "prefill_B2_H16_T4096_d128", "global_batch": 2, "seq_len": 4096, "heads": 16,
                       "dk": 128, "dv": 128, "parallelism": "host threads"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    from linear_attention_token_gdn_b200 import build as gbuild
    from linear_attention_token_gdn_b200 import gdn, inputs

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    if rank == 0:
        gbuild.build()
    if world > 1:
        dist.barrier()
    gdn.lib()
    stream = torch.cuda.current_stream()
    hbm_peak, tf_peak, peak_src = peaks()
    if args.only:  # one secondary workload alone (for profiling), its own JSON line
        line = WORKLOADS[args.only](torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    # ---- headline: prefill workload, three rotating input sets --------------------------
    c = inputs.WORKLOAD_SPECS[inputs.PREFILL]
    sets = [inputs.make_prefill(inputs.PREFILL, "cuda", seed=rank_seed(inputs.SEED_BASE + inputs.PREFILL, rank) + s) for s in range(3)]
    N, H = sets[0]["N"], sets[0]["H"]
    nseq = sets[0]["num_seqs"]
    outs = [(torch.empty(N, H, 128, device="cuda", dtype=torch.bfloat16),
             torch.empty(nseq, H, 128, 128, device="cuda")) for _ in range(3)]
    ws_bytes = gdn.workspace_size(N, nseq, H, 128, 128, 64)
    ws = torch.empty(max(ws_bytes, 16), device="cuda", dtype=torch.uint8)

    def step(i):
        x = sets[i % 3]
        y, S_T = outs[i % 3]
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"], chunk=64, y=y, S_T=S_T,
                      workspace=ws)

    barrier(torch, dist, world)
    with ClockSampler(torch.cuda.current_device()) as clk:
        # the timed region runs the calls back to back, as a caller would (no launch events)
        dt = timed(torch, step, args.steps, args.warmup, stream)
        barrier(torch, dist, world)
        if dt < 0.5:  # keep the GPU busy long enough for the clock sampler to see it
            soak = timed(torch, step, max(1, int(args.steps * 0.6 / max(dt, 1e-6))), 0, stream)
    dt = max_over_ranks(torch, dist, dt, world)
    gdn.check_device_error()
    per_step = dt / args.steps
    work = N * H  # token-heads per rank per step
    value = aggregate(work, world, per_step)
    alg_bytes = prefill_bytes(N, H, nseq)
    # the per-kernel split (and the launch count per call) from a separate instrumented pass
    n_split = min(args.steps, 20)
    kern = kernel_split(torch, gdn, step, n_split, stream, 4 * n_split + 8)
    launches_per_call = sum(k["launches"] for k in kern) / n_split
    achieved = alg_bytes / per_step / 1e9  # one gdn_chunk_fwd call per step, timed over the region
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "prefill_B2_H16_T4096_d128", "global_batch": 2 * world, "seq_len": 4096,
                       "heads": 16, "dk": 128, "dv": 128, "chunk": 64, "state": "fp32, S0=0",
                       "parallelism": f"dp{world}",
                       "l2": "3 rotating input sets (3 x 137 MB > 126 MB L2)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": traffic_per_call(), "kernel":
                         "gdn_chunk_fwd = chunk_ut_kernel + chunk_chain_kernel (per call)",
                         "peak_source": f"{peak_src} hbm_gbs", "alg_bytes_per_launch": alg_bytes,
                         "achieved_from": "the call's device time over the timed region (CUDA events, no "
                                          "launch instrumentation)",
                         "kernels": kern,
                         "kernels_note": "per-kernel split from a separate pass with launch events, which "
                                         "serialise the two kernels (no programmatic overlap there)"},
            "gpu_launches": int(round(launches_per_call * args.steps)), "clocks": clk.summary()}

    # ---- end to end through the public API with pinned host buffers ----------------------
    # Each sequence is split into P segments of T/P tokens chained through S_T -> S0 (identical to
    # one call at chunk boundaries), so that the host->device copy of segment p+1, the chunked pass
    # over segment p and the device->host copy of segment p-1 run at once, on three streams.
    hx = {k: sets[0][k].cpu().pin_memory() for k in ("q", "k", "v", "g", "beta")}
    hy = torch.empty(N, H, 128, dtype=torch.bfloat16).pin_memory()
    hS = torch.empty(nseq, H, 128, 128).pin_memory()
    T = N // nseq
    P = 4 if T % (4 * 64) == 0 else 1
    Ts = T // P
    seg_in = [{k: torch.empty((nseq * Ts,) + tuple(hx[k].shape[1:]), device="cuda", dtype=hx[k].dtype) for k in hx}
              for _ in range(2)]
    seg_y = [torch.empty(nseq * Ts, H, 128, device="cuda", dtype=torch.bfloat16) for _ in range(2)]
    seg_S = [torch.empty(nseq, H, 128, 128, device="cuda") for _ in range(2)]
    seg_cu = (torch.arange(nseq + 1, dtype=torch.int32) * Ts).cuda()
    seg_ws = torch.empty(max(gdn.workspace_size(nseq * Ts, nseq, H, 128, 128, 64), 16), device="cuda",
                         dtype=torch.uint8)
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {n: [torch.cuda.Event() for _ in range(P)] for n in ("h2d", "cmp", "d2h")}

    def e2e_step(i):
        start = torch.cuda.Event()
        start.record(stream)
        s_h2d.wait_event(start)
        s_d2h.wait_event(start)
        for p in range(P):
            b = p % 2
            with torch.cuda.stream(s_h2d):
                if p >= 2:
                    s_h2d.wait_event(ev["cmp"][p - 2])  # segment p - 2 has read input buffer b
                for k in hx:
                    for sq in range(nseq):
                        seg_in[b][k][sq * Ts:(sq + 1) * Ts].copy_(hx[k][sq * T + p * Ts:sq * T + (p + 1) * Ts],
                                                                  non_blocking=True)
                ev["h2d"][p].record(s_h2d)
            stream.wait_event(ev["h2d"][p])
            if p >= 2:
                stream.wait_event(ev["d2h"][p - 2])  # y buffer b has been copied out
            x = seg_in[b]
            gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], seg_S[(p - 1) % 2] if p > 0 else None, seg_cu,
                          chunk=64, y=seg_y[b], S_T=seg_S[p % 2], workspace=seg_ws, stream=stream)
            ev["cmp"][p].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev["cmp"][p])
                for sq in range(nseq):
                    hy[sq * T + p * Ts:sq * T + (p + 1) * Ts].copy_(seg_y[b][sq * Ts:(sq + 1) * Ts], non_blocking=True)
                if p == P - 1:
                    hS.copy_(seg_S[p % 2], non_blocking=True)
                ev["d2h"][p].record(s_d2h)
        stream.wait_event(ev["d2h"][P - 1])

    barrier(torch, dist, world)
    e2e_steps = max(3, min(args.steps, 20))
    dte = timed(torch, e2e_step, e2e_steps, 2, stream)
    dte = max_over_ranks(torch, dist, dte, world)
    # the pipelined result against one call on the same inputs (outside the timed region)
    y1, S1 = gdn.chunk_fwd(sets[0]["q"], sets[0]["k"], sets[0]["v"], sets[0]["g"], sets[0]["beta"], None,
                           sets[0]["cu_seqlens"], chunk=64, y=outs[0][0], S_T=outs[0][1], workspace=ws)
    torch.cuda.synchronize()
    same = bool(torch.equal(hy, y1.cpu()) and torch.equal(hS, S1.cpu()))
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = hy.numel() * 2 + hS.numel() * 4
    line["e2e"] = {"value": work * world * e2e_steps / dte, "unit": UNIT, "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "steps": e2e_steps, "segments_per_sequence": P,
                   "pipelined": "H2D of segment p+1, gdn_chunk_fwd of segment p, D2H of segment p-1 on three "
                                "streams; segments chained through S_T -> S0",
                   "equal_to_one_call": same}

    if not args.no_extra:
        line["other_workloads"] = extra_workloads(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak)
    if rank == 0:
        if args.impl_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(target_s=args.cpu_s)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def wl_decode(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    """decode: 256 x 32 heads, 100 in-place steps per "step"."""
    c = inputs.WORKLOAD_SPECS[inputs.DECODE]
    state = inputs.make_decode_state(inputs.DECODE, "cuda", seed=rank_seed(inputs.SEED_BASE + inputs.DECODE, rank))
    steps_in = [inputs.make_decode_step(inputs.DECODE, "cuda", step=s, seed=rank_seed(inputs.SEED_BASE + inputs.DECODE, rank))
                for s in range(c["steps"])]
    y = torch.empty(c["B"], c["H"], 128, device="cuda", dtype=torch.bfloat16)

    def dec(i):
        for x in steps_in:
            gdn.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state, y=y)

    barrier(torch, dist, world)
    # eager launches with per-launch events (the kernel's own device time) ...
    dt_eager = max_over_ranks(torch, dist, timed(torch, dec, 3, 1, stream, on_start=lambda: gdn.timing_start(4096)),
                              world)
    kd = kernel_table(gdn.timing_stop(), 3)
    # ... and the measured number: the 100 steps replayed from one CUDA graph (no launch gaps)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        dec(0)  # warm the capture stream
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        dec(0)
    barrier(torch, dist, world)
    dt = max_over_ranks(torch, dist, timed(torch, lambda i: graph.replay(), 3, 1, stream), world)
    del graph
    per_launch = dt / (3 * c["steps"])
    upd = c["B"] * c["H"]
    bytes_l = upd * (2 * 128 * 128 * 4 + 3 * 128 * 2 + 8 + 128 * 2)
    return {"workload": c["name"], "value": upd * world / per_launch, "unit": "state-updates/s",
            "us_per_step": per_launch * 1e6, "launch": "CUDA graph of the 100 steps",
            "eager_us_per_step": dt_eager / (3 * c["steps"]) * 1e6,
            "roofline": {"bound": "hbm", "achieved": bytes_l / per_launch / 1e9, "peak": hbm_peak,
                         "unit": "GB/s", "frac": bytes_l / per_launch / 1e9 / hbm_peak,
                         "kernel": "decode_step_kernel", "alg_bytes_per_launch": bytes_l,
                         "kernel_avg_us": kd[0]["avg_us"] if kd else None},
            "gpu_launches": 3 * c["steps"]}


def wl_long(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    """long prefill: B=1, H=32, T=32768, S0 != 0."""
    x = inputs.make_prefill(inputs.LONG_PREFILL, "cuda", seed=rank_seed(inputs.SEED_BASE + inputs.LONG_PREFILL, rank))
    N, H, nseq = x["N"], x["H"], x["num_seqs"]
    yb = torch.empty(N, H, 128, device="cuda", dtype=torch.bfloat16)
    ST = torch.empty(nseq, H, 128, 128, device="cuda")
    ws = torch.empty(max(gdn.workspace_size(N, nseq, H, 128, 128, 64), 16), device="cuda", dtype=torch.uint8)

    def lp(i):
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], chunk=64, y=yb, S_T=ST,
                      workspace=ws)

    barrier(torch, dist, world)
    n_lp = 5
    dt = max_over_ranks(torch, dist, timed(torch, lp, n_lp, 2, stream), world) / n_lp
    kl = kernel_split(torch, gdn, lp, n_lp, stream)
    bl = prefill_bytes(N, H, nseq, S0=True)
    return {"workload": inputs.WORKLOAD_SPECS[inputs.LONG_PREFILL]["name"], "value": N * H * world / dt, "unit": UNIT,
                "ms_per_step": dt * 1e3,
                "roofline": {"bound": "hbm", "achieved": bl / dt / 1e9, "peak": hbm_peak, "unit": "GB/s",
                             "frac": bl / dt / 1e9 / hbm_peak,
                             "kernel": "gdn_chunk_fwd = chunk_ut_kernel + chunk_chain_kernel (per call)",
                             "alg_bytes_per_launch": bl, "kernels": kl,
                             "kernels_note": "per-kernel split from a separate instrumented pass"},
                "gpu_launches": sum(k["launches"] for k in kl), "l2": "1.1 GB working set > L2"}


def wl_mixer(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    """full mixer on 4 packed sequences: prep -> chunk -> out gate (the variant with the gate
    fused into the chunked pass is timed beside it)."""
    m = inputs.make_mixer(inputs.MIXER, "cuda", seed=rank_seed(inputs.SEED_BASE + inputs.MIXER, rank))
    N, H = m["N"], m["H"]
    # q, k, v between prep and the chunked pass in fp16 (11 significant bits; the storage the
    # mixer parity test checks on every head)
    bufs = [torch.empty(N, H, 128, device="cuda", dtype=torch.float16) for _ in range(3)]
    gbuf = torch.empty(N, H, device="cuda")
    bbuf = torch.empty(N, H, device="cuda")
    ym = torch.empty(N, H, 128, device="cuda", dtype=torch.bfloat16)  # y between the chunked pass and the gate
    out = torch.empty(N, H, 128, device="cuda", dtype=torch.bfloat16)
    nsq = m["num_seqs"]
    wsm = torch.empty(max(gdn.workspace_size(N, nsq, H, 128, 128, 64), 16), device="cuda", dtype=torch.uint8)

    def mix(i):  # prep -> chunk -> out gate: three launches
        gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"], m["alpha_logit"],
                 m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"], out=(*bufs, gbuf, bbuf))
        gdn.chunk_fwd(bufs[0], bufs[1], bufs[2], gbuf, bbuf, None, m["cu_seqlens"], chunk=64, y=ym,
                      final_state=False, workspace=wsm)
        gdn.out_gate(ym, m["z"], m["norm_w"], m["eps"], out=out)

    def mix_fused(i):  # the gate fused into the chunked pass (gdn_chunk_fwd_gated)
        gdn.prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"], m["alpha_logit"],
                 m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"], out=(*bufs, gbuf, bbuf))
        gdn.chunk_fwd_gated(bufs[0], bufs[1], bufs[2], gbuf, bbuf, m["z"], m["norm_w"], m["eps"], None,
                            m["cu_seqlens"], final_state=False, out=out, workspace=wsm)

    wsp = torch.empty(max(gdn.lib().gdn_chunk_fwd_prep_workspace_size(N, nsq, H, 128, 128, 64), 16), device="cuda",
                      dtype=torch.uint8)

    def mix_prep_fused(i):  # prep fused into the chunked pass (gdn_chunk_fwd_prep), then the out gate
        gdn.chunk_fwd_prep(m["x_q"], m["x_k"], m["x_v"], m["w_q"], m["w_k"], m["w_v"], m["beta_logit"],
                           m["alpha_logit"], m["A_log"], m["alpha_bias"], cu_seqlens=m["cu_seqlens"], l2_eps=m["eps"],
                           qkv_dtype=torch.float16, y=ym, final_state=False, workspace=wsp)
        gdn.out_gate(ym, m["z"], m["norm_w"], m["eps"], out=out)

    barrier(torch, dist, world)
    n_m = 5
    dt_fused = max_over_ranks(torch, dist, timed(torch, mix_fused, n_m, 1, stream), world) / n_m
    dt_prep = max_over_ranks(torch, dist, timed(torch, mix_prep_fused, n_m, 1, stream), world) / n_m
    kp = kernel_split(torch, gdn, mix_prep_fused, n_m, stream)
    dt = max_over_ranks(torch, dist, timed(torch, mix, n_m, 1, stream), world) / n_m
    km = kernel_split(torch, gdn, mix, n_m, stream)
    fused_min = N * (H * 3 * 128 * 2 + H * 2 * 2 + H * 128 * 2 + H * 128 * 2)
    return {"workload": inputs.WORKLOAD_SPECS[inputs.MIXER]["name"], "lengths": m["lengths"], "value": N * H * world / dt,
                "unit": UNIT, "tokens_per_s": N * world / dt, "ms_per_step": dt * 1e3,
                "ms_per_step_gate_fused_into_chunk": dt_fused * 1e3,
                "ms_per_step_prep_fused_into_chunk": dt_prep * 1e3, "kernels_prep_fused": kp,
                "roofline": {"bound": "hbm", "achieved": fused_min / dt / 1e9, "peak": hbm_peak, "unit": "GB/s",
                             "frac": fused_min / dt / 1e9 / hbm_peak, "kernel": "prep+chunk+out_gate",
                             "alg_bytes_per_step": fused_min,
                             "note": "bytes = fused minimum (read projections, logits, z; write out); per-kernel "
                                     "split from a separate instrumented pass",
                             "kernels": km},
                "gpu_launches": sum(k["launches"] for k in km)}


def wl_mixer_decode(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    """full-mixer decode: 256 sequences x H=32, d=128, conv width 4, 100 steps of
    gdn_mixer_decode_step (conv history, prep, recurrence and out gate in one kernel), the fp32
    state and the conv history updated in place."""
    c = inputs.WORKLOAD_SPECS[inputs.DECODE]
    B, H, d, W = c["B"], c["H"], 128, 4
    seed = rank_seed(inputs.SEED_BASE + inputs.DECODE, rank)
    state = inputs.make_decode_state(inputs.DECODE, "cuda", seed=seed)
    m = inputs.make_mixer(inputs.MIXER, "cuda", seed=seed, lengths=[B], H=H)  # weights and one token of inputs
    gen = torch.Generator(device="cuda").manual_seed(seed + 5)
    conv = (torch.randn(B, W - 1, H, 3 * d, device="cuda", generator=gen)).to(torch.bfloat16)
    steps_in = []
    for s in range(c["steps"]):
        x = inputs.make_mixer(inputs.MIXER, "cuda", seed=seed * 1000 + s, lengths=[B], H=H)
        steps_in.append({k: x[k] for k in ("x_q", "x_k", "x_v", "beta_logit", "alpha_logit", "z")})
    out = torch.empty(B, H, d, device="cuda", dtype=torch.bfloat16)

    def dec(i):
        for x in steps_in:
            gdn.mixer_decode_step(x["x_q"], x["x_k"], x["x_v"], m["w_q"], m["w_k"], m["w_v"], x["beta_logit"],
                                  x["alpha_logit"], m["A_log"], m["alpha_bias"], x["z"], m["norm_w"], conv, state,
                                  l2_eps=m["eps"], rms_eps=m["eps"], out=out)

    barrier(torch, dist, world)
    dt_eager = max_over_ranks(torch, dist, timed(torch, dec, 3, 1, stream, on_start=lambda: gdn.timing_start(4096)),
                              world)
    kd = kernel_table(gdn.timing_stop(), 3)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        dec(0)
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        dec(0)
    barrier(torch, dist, world)
    dt = max_over_ranks(torch, dist, timed(torch, lambda i: graph.replay(), 3, 1, stream), world)
    del graph
    per_launch = dt / (3 * c["steps"])
    upd = B * H
    # per (row, head): fp32 state read + write, conv history read + write, the token's q/k/v
    # projections, two logits, z, out (all bf16)
    bytes_l = upd * (2 * d * d * 4 + 2 * (W - 1) * 3 * d * 2 + 3 * d * 2 + 2 * 2 + d * 2 + d * 2)
    return {"workload": f"mixer_decode_B{B}_H{H}_d{d}_W{W}_x100", "value": upd * world / per_launch,
            "unit": "state-updates/s", "us_per_step": per_launch * 1e6, "launch": "CUDA graph of the 100 steps",
            "eager_us_per_step": dt_eager / (3 * c["steps"]) * 1e6,
            "roofline": {"bound": "hbm", "achieved": bytes_l / per_launch / 1e9, "peak": hbm_peak,
                         "unit": "GB/s", "frac": bytes_l / per_launch / 1e9 / hbm_peak,
                         "kernel": "mixer_decode_kernel", "alg_bytes_per_launch": bytes_l,
                         "kernel_avg_us": kd[0]["avg_us"] if kd else None},
            "gpu_launches": 3 * c["steps"]}


def wl_backward(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    """backward of the prefill workload (B=2, H=16, T=4096, bf16 q/k/v and dy): gdn_chunk_bwd,
    the token-sequential reverse pass with its checkpointing forward pass."""
    x = inputs.make_prefill(inputs.PREFILL, "cuda", seed=rank_seed(inputs.SEED_BASE + inputs.PREFILL + 50, rank))
    N, H, nseq = x["N"], x["H"], x["num_seqs"]
    gen = torch.Generator(device="cuda").manual_seed(rank_seed(7, rank))
    dy = torch.randn(N, H, 128, device="cuda", generator=gen).to(torch.bfloat16)
    dS_T = torch.randn(nseq, H, 128, 128, device="cuda", generator=gen) * 0.01
    ws = torch.empty(gdn.lib().gdn_chunk_bwd_workspace_size(N, nseq, H, 128, 128), device="cuda", dtype=torch.uint8)
    out = dict(dq=torch.empty(N, H, 128, device="cuda"), dk=torch.empty(N, H, 128, device="cuda"),
               dv=torch.empty(N, H, 128, device="cuda"), dg=torch.empty(N, H, device="cuda"),
               dbeta=torch.empty(N, H, device="cuda"), dS0=torch.empty(nseq, H, 128, 128, device="cuda"))

    def bwd(i):
        gdn.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dy, None, dS_T, x["cu_seqlens"], out=out, workspace=ws)

    barrier(torch, dist, world)
    n_b = 3
    dt = max_over_ranks(torch, dist, timed(torch, bwd, n_b, 1, stream), world) / n_b
    kb = kernel_split(torch, gdn, bwd, n_b, stream)
    # read q, k, v, dy (bf16), g, beta; write dq, dk, dv (fp32), dg, dbeta; dS_T in, dS0 out
    alg = N * H * (3 * 128 * 2 + 128 * 2 + 8 + 3 * 128 * 4 + 8) + 2 * nseq * H * 128 * 128 * 4
    return {"workload": "backward_prefill_B2_H16_T4096_d128", "value": N * H * world / dt, "unit": UNIT,
            "ms_per_step": dt * 1e3,
            "roofline": {"bound": "latency (token-sequential)", "achieved": alg / dt / 1e9, "peak": hbm_peak,
                         "unit": "GB/s", "frac": alg / dt / 1e9 / hbm_peak, "alg_bytes_per_step": alg,
                         "kernels": kb},
            "gpu_launches": sum(k["launches"] for k in kb)}


def wl_inproj(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    """input projections + prep on the mixer's 4 packed sequences from a D = 2048 residual
    stream: gdn_inproj_prep (one tcgen05 GEMM, eqs. (6)-(10) in its epilogue).  Beside it, as
    context only: the same FLOPs as one cuBLAS GEMM (x @ w^T, bf16 out), and the unfused path
    of six cuBLAS GEMMs (one per projection) followed by gdn_prep."""
    m = inputs.make_inproj(inputs.INPROJ, "cuda", seed=rank_seed(inputs.SEED_BASE + inputs.INPROJ, rank))
    N, H, D, d = m["N"], m["H"], m["D"], m["d"]
    x, w = m["x"], m["w"]
    R = w.shape[0]
    hd = H * d
    out = tuple(torch.empty(N, H, d, device="cuda", dtype=torch.bfloat16) for _ in range(3)) + (
        torch.empty(N, H, device="cuda"), torch.empty(N, H, device="cuda"),
        torch.empty(N, H, d, device="cuda", dtype=torch.bfloat16))
    args_ip = (x, w, H, m["conv_q"], m["conv_k"], m["conv_v"], m["A_log"], m["alpha_bias"], m["cu_seqlens"])

    def fused(i):
        gdn.inproj_prep(*args_ip, eps=m["eps"], out=out)

    pw = torch.empty(N, R, device="cuda", dtype=torch.bfloat16)

    def gemm_only(i):
        torch.matmul(x, w.t(), out=pw)

    blocks = [w[j * hd:(j + 1) * hd] for j in range(4)] + [w[4 * hd:4 * hd + H], w[4 * hd + H:]]
    raw = [torch.empty(N, hd, device="cuda", dtype=torch.bfloat16) for _ in range(4)] + [
        torch.empty(N, H, device="cuda", dtype=torch.bfloat16) for _ in range(2)]
    pbuf = tuple(torch.empty(N, H, d, device="cuda", dtype=torch.bfloat16) for _ in range(3)) + (
        torch.empty(N, H, device="cuda"), torch.empty(N, H, device="cuda"))

    def unfused(i):
        for b, o in zip(blocks, raw):
            torch.matmul(x, b.t(), out=o)
        gdn.prep(raw[0].view(N, H, d), raw[1].view(N, H, d), raw[2].view(N, H, d), m["conv_q"], m["conv_k"],
                 m["conv_v"], raw[4], raw[5], m["A_log"], m["alpha_bias"], m["cu_seqlens"], eps=m["eps"], out=pbuf)

    barrier(torch, dist, world)
    n_i = 10
    dt = max_over_ranks(torch, dist, timed(torch, fused, n_i, 3, stream), world) / n_i
    ki = kernel_split(torch, gdn, fused, n_i, stream)
    dt_gemm = max_over_ranks(torch, dist, timed(torch, gemm_only, n_i, 3, stream), world) / n_i
    dt_unf = max_over_ranks(torch, dist, timed(torch, unfused, n_i, 3, stream), world) / n_i
    flops = 2.0 * N * D * R
    _, tf_peak, src = peaks()
    ach = flops / dt / 1e12  # one launch per step, timed over the region
    return {"workload": inputs.WORKLOAD_SPECS[inputs.INPROJ]["name"], "lengths": m["lengths"],
            "value": N * H * world / dt, "unit": UNIT, "tokens_per_s": N * world / dt, "ms_per_step": dt * 1e3,
            "context_ms_cublas_gemm_same_flops": dt_gemm * 1e3,
            "context_ms_six_cublas_gemms_then_gdn_prep": dt_unf * 1e3,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": tf_peak, "unit": "TFLOP/s", "frac": ach / tf_peak,
                         "peak_source": f"{src} bf16_tflops (burst)", "kernel": "inproj_prep_kernel",
                         "alg_flops_per_launch": flops,
                         "note": "flops = 2 N D (4 H d + 2 H); the conv halo rows recomputed per tile are not counted",
                         "kernels": ki},
            "gpu_launches": sum(k["launches"] for k in ki)}


WORKLOADS = {"decode": wl_decode, "long": wl_long, "mixer": wl_mixer, "mixer_decode": wl_mixer_decode,
             "backward": wl_backward, "inproj": wl_inproj}


def extra_workloads(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak):
    res = []
    for fn in WORKLOADS.values():
        res.append(fn(torch, dist, gdn, inputs, args, rank, world, stream, hbm_peak))
        torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--only", choices=["decode", "long", "mixer", "mixer_decode", "backward", "inproj"], default=None,
                    help="run one secondary workload alone and print its line (profiling aid)")
    ap.add_argument("--cpu-s", type=float, default=12.0, help="target seconds of the CPU-baseline sample")
    ap.add_argument("--ref-step-s", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", dest="impl_cpu_baseline", action="store_false")
    ap.add_argument("--launch-check", action="store_true",
                    help="rendezvous, barrier and max-over-ranks only (gloo, no GPU work); rank 0 prints n_gpus")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus)
    _, world, _ = env_rank()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2
    if args.launch_check:
        return launch_check(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


def launch_ranks(n):
    """`bench.py --gpus N` started as one process: start N ranks of this same command line
    under torch.distributed.run (one node, rendezvous on 127.0.0.1) and return its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def launch_check(args):
    """The launch plumbing alone: every rank joins a gloo group, passes the barrier and takes
    part in the max-over-ranks reduction; rank 0 prints the world size it saw."""
    from datetime import timedelta

    import torch.distributed as dist
    rank, world, local = env_rank()
    if world > 1:
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        gdist.barrier(world, cuda=False)
        slowest = gdist.max_over_ranks(float(rank + 1), world, device="cpu")
        if rank == 0:
            print(json.dumps({"launch_check": True, "n_gpus": world, "max_over_ranks": slowest}), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
