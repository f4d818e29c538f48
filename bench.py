"""Benchmark of one DSpark-style speculative round on B200.

A step is one pass of the whole hot path (draft_sample -> prefix_schedule ->
verify) over one batch of the serving-shape workload: B=256 requests, K=5
drafted positions, V=129280, Markov rank 256, bf16 logits, per-request
temperatures {0.6, 0.8, 1.0}, a cost table with a step at 512 verified tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun every rank runs its own batch (different seed) with no
collective on the data path (weak scaling; with --global-schedule one prefix
cut spans every rank's requests, after an all-gather of their confidence
logits); timing is bracketed by a barrier
and synchronisation, taken with CUDA events, and reduced with MAX over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speculative_decoding_draft_sample_b200 import binding as bn  # noqa: E402
from speculative_decoding_draft_sample_b200 import replicas  # noqa: E402
from speculative_decoding_draft_sample_b200 import workloads as wl  # noqa: E402
from speculative_decoding_draft_sample_b200.spec_round import (DEVICE_KEYS, GlobalSchedule,  # noqa: E402
                                                                SpecRound, run_host, to_device)

METRIC = "spec rounds/s & accepted tok/s at B=256,K=5,V=129280; verify HBM GB/s vs peak"
UNIT = "rounds/s"
L2_BYTES = 126 * 1024 * 1024


CUT_MODES = {"cost": bn.CUT_COST, "threshold": bn.CUT_THRESHOLD, "none": bn.CUT_NONE}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """SM clocks and clock-event reasons sampled through NVML (read-only
    queries) on a background thread during the timed region."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        import threading
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.stop_ev = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            u = str(torch.cuda.get_device_properties(device_index).uuid)
            u = u if u.startswith("GPU-") else "GPU-" + u
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(u)
            self.nv = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._run, daemon=True)
        except Exception:
            self.thread = None

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
            except Exception:
                pass
            self.stop_ev.wait(self.period)

    def start(self):
        if self.thread:
            self.thread.start()

    def stop(self):
        if not self.thread:
            return None
        self.stop_ev.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for bit, n in self.REASONS.items() if self.reasons & bit),
                "samples": len(self.samples), "source": "NVML every 2 ms over the timed region"}


# sources the draft kernel compiles from (its counters are valid while they hash the same)
DRAFT_KERNEL_SOURCES = ("draft_tc.cu", "draft_tc.cuh", "draft.cuh", "sample_warp.cuh", "common.cuh")


def sources_sha256(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "speculative_decoding_draft_sample_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kernel_files, summary: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel's sources changed after the counters were taken."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None, "no ncu summary committed"
    sha = sources_sha256(kernel_files)
    fields = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("source_sha256") != sha:
        return None, "kernel sources changed since the ncu capture"
    try:
        return float(fields["dram_bytes_per_launch"]), "profiles/" + summary
    except (KeyError, ValueError):
        return None, "no dram_bytes_per_launch line"


def time_region(fn, stream, iters: int) -> float:
    """Average ms of fn() over iters runs, CUDA events on ``stream``."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(iters):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / iters


ORACLE_SAMPLE = 64  # requests per oracle step (cpu_baseline and the reference arm)


def oracle_sample_inputs(w: wl.Workload, small, n_req: int):
    """fp64 oracle inputs for the first n_req requests of the round (the
    schedule's inputs cover the whole batch: the cut is batch-wide)."""
    reqs = list(range(n_req))
    part = wl.generate(w, reqs)
    rid = np.asarray(reqs)
    return dict(target=part["target"].double().numpy(), base=part["base"].double().numpy(),
                U=small["U"].double().numpy(), W=small["W"].double().numpy(),
                last_tok=np.asarray(small["last_tok"])[rid],
                bias_scale=np.asarray(small["bias_scale"], np.float64)[rid],
                temp=np.asarray(small["temp"], np.float64)[rid],
                conf_logit=np.asarray(small["conf_logit"], np.float64),
                pos_temp=np.asarray(small["pos_temp"], np.float64),
                step_cost=np.asarray(small["step_cost"], np.float64),
                fixed_cost=float(small["fixed_cost"]), dtype=w.dtype, request_ids=rid)


def host_cores():
    """(logical cores of this host, BLAS threads numpy uses)."""
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        blas = 1
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return int(cores), int(blas)


def oracle_step(o, oi, round_id: int, mode: int, threshold: float):
    """One step of the oracle module ``o`` on prepared inputs: (seconds, accepted drafts)."""
    t0 = time.perf_counter()
    r = o.run_round(oi, wl.PHILOX_SEED, round_id, mode, threshold)
    return time.perf_counter() - t0, int(r["verify"]["a"].sum())


def sample_text(w: wl.Workload, n_req: int) -> str:
    return (f"{n_req} of {w.B} requests of one round per step (draft with the rank-{w.r} bias, "
            f"the batch-wide cut, verify), fp64 numpy; rounds/s = ({n_req}/{w.B}) / step seconds")


def cpu_baseline(w: wl.Workload, small, n_req: int, round_id: int, mode: int = bn.CUT_COST,
                 threshold: float = 0.0):
    """The fp64 oracle on a bounded sample of the round (n_req requests)."""
    from oracle import dspark as o
    oi = oracle_sample_inputs(w, small, n_req)
    dt, acc = oracle_step(o, oi, round_id, mode, threshold)
    cores, blas = host_cores()
    return dict(value=(n_req / w.B) / dt, unit=UNIT, cores=cores, blas_threads=blas, kind="oracle",
                sample=sample_text(w, n_req), seconds=dt, accepted=acc)


def reference_arm(args, w: wl.Workload):
    """The oracle timed on the host cores: every step runs it on the same
    ORACLE_SAMPLE-request sample of the round, so ms_per_step is the time one
    step really took and steps x ms_per_step is the time spent."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    small = wl.small_inputs(w)
    n_req = min(ORACLE_SAMPLE, w.B)
    mode = CUT_MODES[args.cut]
    threshold = args.threshold if mode == bn.CUT_THRESHOLD else 0.0
    from oracle import dspark as o
    oi = oracle_sample_inputs(w, small, n_req)
    for i in range(args.warmup):
        oracle_step(o, oi, 0, mode, threshold)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_step(o, oi, 0, mode, threshold)
    secs = time.perf_counter() - t0
    value = args.steps * (n_req / w.B) / secs
    cores, blas = host_cores()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "K": w.K, "V": w.V, "r": w.r,
                       "cut": args.cut + (f" {threshold}" if mode == bn.CUT_THRESHOLD else ""),
                       "step": f"{n_req} of {w.B} requests"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "blas_threads": blas,
                             "kind": "oracle", "sample": sample_text(w, n_req)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def load_sweep():
    """NEXT-3 of the scheduler: how the early-stopping cut trims the verified
    block as the batch grows, against the DSpark-5 cost table (a step in the
    per-token cost at 512 verified tokens). Prefix schedule only; one JSON line
    per batch size."""
    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    for B in (32, 64, 128, 256, 512, 1024):
        w = wl.scaled(wl.DSPARK5, name=f"load_b{B}", B=B)
        small = wl.small_inputs(w)
        dev = {k: torch.as_tensor(small[k]).cuda() for k in ("conf_logit", "pos_temp", "step_cost")}
        cut = torch.empty(B, dtype=torch.int32, device="cuda")
        surv = torch.empty((B, w.K), dtype=torch.float32, device="cuda")
        ws = torch.zeros(bn.workspace_bytes(bn.OP_SCHEDULE, B, w.K, 8, 1, bn.F32), dtype=torch.uint8,
                         device="cuda")
        def call():
            bn.prefix_schedule(dev["conf_logit"], dev["pos_temp"], dev["step_cost"],
                               small["fixed_cost"], bn.CUT_COST, 0.0, cut, surv, ws, stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                call()
            ms = time_region(call, stream, 20)
        c = cut.cpu().numpy()
        print(json.dumps({"B": B, "K": w.K, "mean_cut": float(c.mean()),
                          "verified_tokens": int(c.sum() + B), "schedule_us": ms * 1e3,
                          "cut_hist": np.bincount(c, minlength=w.K + 1).tolist()}), flush=True)


def calib_bench(N: int):
    """Sequential Temperature Scaling (dspark_sts_fit) on N synthetic samples of
    an over-confident head: CUDA-event time and the ECE before / after."""
    torch.cuda.set_device(0)
    K = 5
    z, y = wl.calib_inputs(N, K=K)
    zt, yt = torch.from_numpy(z).cuda(), torch.from_numpy(y).cuda()
    T = torch.zeros(K, device="cuda")
    idx = torch.zeros(K, dtype=torch.int32, device="cuda")
    eb, ea = torch.zeros(K, device="cuda"), torch.zeros(K, device="cuda")
    ws = torch.zeros(bn.workspace_bytes(bn.OP_CALIB, N, K, 0, 0, 0), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(3):
            bn.sts_fit(zt, yt, T, idx, eb, ea, ws, stream)
        ms = time_region(lambda: bn.sts_fit(zt, yt, T, idx, eb, ea, ws, stream), stream, 10)
    print(json.dumps({"N": N, "K": K, "ms": ms, "samples_x_grid_per_s": 256 * N * K / (ms * 1e-3),
                      "T": T.cpu().tolist(), "ece_before": eb.cpu().tolist(),
                      "ece_after": ea.cpu().tolist(), "launches": 2 * K + 4,
                      "loss_evaluations": 256 * N * K}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=wl.DSPARK5.name, choices=sorted(wl.ALL),
                    help="measure another configuration (the default is the headline one)")
    ap.add_argument("--load-sweep", action="store_true",
                    help="prefix schedule only: mean cut and time as the batch grows")
    ap.add_argument("--calib", type=int, default=0, metavar="N",
                    help="Sequential Temperature Scaling of N synthetic samples (K = 5): time and ECE")
    ap.add_argument("--cut", default="cost", choices=sorted(CUT_MODES),
                    help="prefix schedule: early-stopping cost rule (default), static survival "
                         "threshold, or none (every request verifies all K drafts)")
    ap.add_argument("--threshold", type=float, default=0.5,
                    help="survival threshold of --cut threshold")
    ap.add_argument("--head", default="markov", choices=["markov", "recurrent"],
                    help="sequential draft head: the Markov head (default) or the recurrent one")
    ap.add_argument("--global-schedule", action="store_true",
                    help="one prefix schedule over every rank's requests (an all-gather of the "
                         "confidence logits) instead of one per engine")
    args = ap.parse_args()
    if args.load_sweep:
        load_sweep()
        return
    if args.calib:
        calib_bench(args.calib)
        return
    w = wl.ALL[args.workload]
    if args.impl == "reference":
        reference_arm(args, w)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    world, rank, local = replicas.init("nccl")
    hbm, tflops, tflops_sus, peak_kind = peaks()

    # each rank: its own batch (weak scaling), no collective on the data path
    inp = wl.generate(replicas.rank_workload(w, rank))
    if args.head == "recurrent":
        inp["R"] = wl.recurrent_factor(w)
    dev = to_device(inp)
    tdt = torch.float32 if w.dtype == wl.F32 else torch.bfloat16
    rnd = SpecRound(w.B, w.K, w.V, w.r, tdt)
    stream = torch.cuda.Stream()
    side = torch.cuda.Stream()  # the prefix schedule runs here, beside the draft
    round_id = 0

    mode = CUT_MODES[args.cut]
    threshold = args.threshold if mode == bn.CUT_THRESHOLD else 0.0

    # optionally one cut over every rank's requests, against the combined batch's cost table
    gsched = None
    if args.global_schedule:
        step_cost_g, fixed_g = wl.cost_table(w, w.B * world)
        gsched = GlobalSchedule(w.B, w.K, step_cost_g, fixed_g, rank, world)

    def step():
        rnd.run(dev, wl.PHILOX_SEED, round_id, mode, threshold, stream=stream, side_stream=side,
                global_schedule=gsched)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    code, first = rnd.status(stream)
    if code:
        raise RuntimeError(f"device status {code} at request {first}")

    # CUDA graph of the whole round (2K + 2 launches)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
        stream.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            step()
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):  # replay() launches on the current stream
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    clocks = Clocks(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    replicas.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    replicas.barrier()
    ms = replicas.max_over_ranks(e0.elapsed_time(e1) / args.steps, "cuda")
    clk = clocks.stop() if clocks else None

    accepted = int(rnd.accepted.sum().item())
    emitted = int(rnd.n_emit.sum().item())
    cut = rnd.cut.cpu().numpy()
    acc_np = rnd.accepted.cpu().numpy()
    acc_all = replicas.sum_over_ranks(float(accepted), "cuda")
    emit_all = replicas.sum_over_ranks(float(emitted), "cuda")
    rounds_per_s = world * 1000.0 / ms

    # per-stage times (same stream, CUDA events), each stage alone; the NVTX
    # range lets a profiler select these launches (ncu --nvtx --nvtx-include
    # stage_timing/), e.g. the full-width draft kernel the roofline times
    s_bytes = w.nbytes_per_logit
    torch.cuda.nvtx.range_push("stage_timing")
    with torch.cuda.stream(stream):
        if args.head == "recurrent":
            ms_draft = time_region(lambda: bn.draft_sample_recurrent(
                dev["base"], dev["U"], dev["W"], dev["R"], dev["bias_scale"], dev["last_tok"],
                dev["temp"], wl.PHILOX_SEED, round_id, rnd.x, rnd.d, rnd.q_lse, rnd.q_tok, rnd.h,
                rnd.ws, stream, q_norm=rnd.q_norm), stream, 10)
        else:
            ms_draft = time_region(lambda: bn.draft_sample(
                dev["base"], dev["U"], dev["W"], dev["bias_scale"], dev["last_tok"], dev["temp"],
                wl.PHILOX_SEED, round_id, rnd.x, rnd.d, rnd.q_lse, rnd.q_tok, rnd.ws, stream,
                q_norm=rnd.q_norm), stream, 10)
        ms_sched = time_region(lambda: bn.prefix_schedule(
            dev["conf_logit"], dev["pos_temp"], dev["step_cost"], dev["fixed_cost"], mode,
            threshold, rnd.cut, rnd.survival, rnd.ws, stream), stream, 20)
        ms_verify = time_region(lambda: bn.verify(
            dev["target"], rnd.d, rnd.x, rnd.q_tok, rnd.cut, dev["temp"], wl.PHILOX_SEED,
            round_id, rnd.accepted, rnd.out, rnd.n_emit, rnd.ws, stream, q_norm=rnd.q_norm),
            stream, 20)
        ms_stats = time_region(lambda: bn.verify_target_stats(
            dev["target"], rnd.cut, dev["temp"], rnd.ws, stream), stream, 20)
        ms_final = time_region(lambda: bn.verify_from_stats(
            dev["target"], rnd.d, rnd.x, rnd.q_tok, rnd.cut, dev["temp"], wl.PHILOX_SEED,
            round_id, rnd.accepted, rnd.out, rnd.n_emit, rnd.ws, stream, q_norm=rnd.q_norm),
            stream, 20)

    torch.cuda.nvtx.range_pop()

    # verification's algorithmic bytes (the survey's count): target rows 0..cut[b]
    # of every request, plus draft row a_b of every request rejected before its
    # cut. The statistics pass reads the former, the final kernel the draft rows
    # and (again) the target row of the residual.
    rej = int((acc_np < cut).sum())
    stats_bytes = int((cut + 1).sum()) * w.V * s_bytes
    final_bytes = 2 * rej * w.V * s_bytes
    verify_bytes = stats_bytes + rej * w.V * s_bytes
    verify_gbs = verify_bytes / (ms_verify * 1e-3) / 1e9
    # the draft kernel (one cooperative launch per round): per position the
    # base block in, d out, W once, the chunk partials out and back in, the
    # sampled chunk of d and the gathered U rows
    nchunk = (w.V + 255) // 256
    draft_bytes = w.K * (2 * w.B * w.V * s_bytes + w.r * w.V * s_bytes + 2 * w.B * nchunk * 8
                         + w.B * 256 * s_bytes + w.B * w.r * s_bytes)
    draft_gbs = draft_bytes / (ms_draft * 1e-3) / 1e9
    gemm_tflops = 2.0 * w.B * w.r * w.V * w.K / (ms_draft * 1e-3) / 1e12

    # end to end through the public API from pinned host buffers
    host = to_device(inp, pin=True)
    out_h = torch.empty_like(rnd.out, device="cpu").pin_memory()
    n_h = torch.empty_like(rnd.n_emit, device="cpu").pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in DEVICE_KEYS)
    d2h = out_h.numel() * 4 + n_h.numel() * 4
    with torch.cuda.stream(stream):
        for _ in range(2):
            run_host(rnd, host, dev, wl.PHILOX_SEED, round_id, out_h, n_h, mode, stream=stream,
                     side_stream=side, threshold=threshold, global_schedule=gsched)
        replicas.barrier()
        e2e_steps = max(3, args.steps // 5)
        ms_e2e = time_region(lambda: run_host(rnd, host, dev, wl.PHILOX_SEED, round_id, out_h, n_h,
                                              mode, stream=stream, side_stream=side,
                                              threshold=threshold, global_schedule=gsched),
                                     stream, e2e_steps)
    ms_e2e = replicas.max_over_ranks(ms_e2e, "cuda")

    in_bytes = (w.B * (w.K + 1) * w.V + w.B * w.K * w.V + 2 * w.V * w.r) * s_bytes
    traffic, traffic_src = profiled_traffic(DRAFT_KERNEL_SOURCES, "draft_logits_tc_dspark5.txt")
    if w.name != wl.DSPARK5.name or mode != bn.CUT_COST or args.head != "markov":
        traffic, traffic_src = None, "ncu summary covers the DSpark-5 workload (cost cut, Markov head) only"
    roof = {"kernel": "draft_logits_tc (dspark_draft_sample: all K positions in one launch)",
            "bound": "hbm", "achieved": draft_gbs, "peak": hbm, "unit": "GB/s",
            "frac": draft_gbs / hbm, "traffic": traffic, "traffic_source": traffic_src,
            "peak_source": f"hbm_gbs of {peak_kind} peaks",
            "bytes_per_launch": draft_bytes, "launch_ms": ms_draft,
            "share_of_step": ms_draft / ms}
    line = {
        "metric": METRIC, "value": rounds_per_s, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if w.dtype == wl.F32 else "bf16",
        "data": "synthetic (seeded Zipf+noise logits, random Markov factors)",
        "config": {"workload": w.name, "B": w.B, "K": w.K, "V": w.V, "r": w.r,
                   "global_batch": w.B * world, "parallelism": f"replicas{world}",
                   "schedule": "global" if gsched is not None else "per-engine",
                   "cut": args.cut + (f" {threshold}" if mode == bn.CUT_THRESHOLD else ""),
                   "head": args.head,
                   "l2": (f"inputs ({in_bytes / 1e6:.0f} MB) larger than L2 (126 MB); not flushed"
                          if in_bytes > L2_BYTES else
                          f"inputs ({in_bytes / 1e6:.0f} MB) fit in L2 (126 MB); not flushed"),
                   "timing": "CUDA graph of the round, CUDA events, max over ranks"},
        "accepted_tok_per_s": acc_all * 1000.0 / ms,
        "emitted_tok_per_s": emit_all * 1000.0 / ms,
        "accepted_per_round": accepted, "emitted_per_round": emitted,
        "mean_cut": float(cut.mean()), "mean_accepted": float(acc_np.mean()),
        "stages_ms": {"draft": ms_draft, "schedule": ms_sched, "verify": ms_verify,
                      "verify_target_stats": ms_stats, "verify_from_stats": ms_final,
                      "round_minus_draft": ms - ms_draft},
        # each stage above alone; in the round the draft leaves this many SMs to
        # the schedule and the target statistics on the side stream
        "round_draft_free_sms": rnd.free_sms,
        "verify": {"gbs": verify_gbs, "frac_of_hbm_peak": verify_gbs / hbm,
                   "bytes_per_call": verify_bytes, "call_ms": ms_verify,
                   "target_stats": {"bytes": stats_bytes, "ms": ms_stats,
                                    "gbs": stats_bytes / (ms_stats * 1e-3) / 1e9,
                                    "frac_of_hbm_peak": stats_bytes / (ms_stats * 1e-3) / 1e9 / hbm},
                   "from_stats": {"bytes": final_bytes, "ms": ms_final,
                                  "gbs": final_bytes / (ms_final * 1e-3) / 1e9,
                                  "frac_of_hbm_peak": final_bytes / (ms_final * 1e-3) / 1e9 / hbm},
                   "bytes_rule": "target rows 0..cut[b] + draft row a_b of each rejected request"},
        "draft_stage": {"gbs": draft_gbs, "bias_gemm_tflops": gemm_tflops,
                        "bias_gemm_frac_of_bf16_peak": gemm_tflops / tflops},
        "roofline": roof,
        "e2e": {"value": world * 1000.0 / ms_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and w.name == wl.DSPARK5.name
            and mode == bn.CUT_COST and args.head == "markov"):
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(w, wl.small_inputs(w), ORACLE_SAMPLE,
                                                              0).items()
                                if k in ("value", "unit", "cores", "blas_threads", "kind", "sample")}
    del graph  # released before the process group goes away
    replicas.finish()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
