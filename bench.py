#!/usr/bin/env python
"""Throughput of the residual-compression hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cogvideox]
                    [--impl ours|reference] [--no-cpu-baseline] [--no-e2e]
                    [--no-lowrank-leg]

A "step" is one denoising step of the workload: every exchanged buffer is
encoded by the sender (residual + error feedback + per-token scale +
quantise + pack + error/mirror update) and decoded by the receiver (unpack
+ dequantise + accumulate), each as ONE batched launch over all buffers.

Metric: GB/s of bf16 activation processed = 2 bytes * T * C * buffers *
steps / (encode + decode time), whole job (all ranks).  Inputs are the
seeded synthetic drift trajectories, pre-generated in HBM before timing; one
step of the default workload (CogVideoX-like, 60 buffers of 17550 x 1920)
touches ~45 GB, far more than the 126 MB L2, so no L2 flush is needed
between steps.  The same line also reports, under "lowrank", the low-rank
mode on its own workload (114 x 4096 x 3072, rank 32, 2 iterations).

Multi-GPU: by default sender and receiver share a device, so N ranks run N
independent replicas of the workload ("weak" scaling).  The timed region is
bracketed by barriers and the max over ranks is reported.  --exchange runs
the sequence-parallel exchange instead: each step encodes into one payload,
all-gathers the payloads over NCCL and decodes every peer's shard.

--workload lowrank times the low-rank mode (rank 32, INT4 factors).
--impl reference times the CPU oracle on a bounded sample of the same
workload, with the same metric and unit: the plain C oracle on one core for
the quantize workloads, the numpy fp64 oracle for the low-rank one.
"""
from __future__ import annotations

import argparse
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

import torch  # noqa: E402

from activation_residual_compression_cf_b200 import replicas as R  # noqa: E402
from activation_residual_compression_cf_b200 import workloads as W  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
METRIC = "encode+decode GB/s of bf16 activation processed; % of B200 HBM roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="cogvideox", choices=list(W.WORKLOADS),
                    help="default: cogvideox (60 x 17550 x 1920, 2-bit), the largest workload")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--iters", type=int, default=0,
                    help="low-rank: subspace iterations (default: the workload's)")
    ap.add_argument("--rank", type=int, default=0, help="low-rank: rank (default: the workload's)")
    ap.add_argument("--e2e-chunks", type=int, default=6,
                    help="end-to-end leg: buffers of a step split into this many chunks whose "
                         "copies overlap the kernels of their neighbours")
    ap.add_argument("--emit", action="store_true",
                    help="quantize: the receiver also writes the bf16 reconstruction")
    ap.add_argument("--delta", action="store_true",
                    help="quantize: delta-state sender (previous activation + error buffer)")
    ap.add_argument("--exchange", action="store_true",
                    help="quantize mode: the sequence-parallel exchange (encode into one payload, "
                         "all-gather over the process group, decode every peer's shard; one GPU "
                         "alone decodes its own payload)")
    ap.add_argument("--lowrank-group", type=int, default=-1,
                    help="low-rank: buffers per pass of the batched encode (0 = all; -1 = the "
                         "library default)")
    ap.add_argument("--fused", action="store_true",
                    help="with --exchange: the fused exchange (publishing encode into the receivers' "
                         "slots, waiting decode; no collective)")
    ap.add_argument("--warm", action="store_true",
                    help="low-rank: warm start every encode after the first from the previous Q")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="budget of the oracle timing sample")
    ap.add_argument("--buffers", type=int, default=0,
                    help="override the buffer count (smaller cases for profiling)")
    ap.add_argument("--pipeline", type=int, default=-1,
                    help="quantize kernels: 0 register-resident rows, 1 TMA row staging, "
                         "-1 the library default")
    ap.add_argument("--gen-steps", type=int, default=0,
                    help="distinct pre-generated steps to cycle through (0 = all that fit)")
    ap.add_argument("--e2e-steps", type=int, default=40,
                    help="steps of the end-to-end leg (each moves a whole step's activations "
                         "over PCIe, ~70 ms for cogvideox)")
    ap.add_argument("--no-lowrank-leg", action="store_true",
                    help="quantize workloads: skip the low-rank leg (114 x 4096 x 3072, rank 32) "
                         "that the line also reports under 'lowrank'")
    ap.add_argument("--lowrank-steps", type=int, default=60)
    return ap.parse_args()


# ------------------------------------------------------------ environment

def dist_setup(args):
    info = R.rank_info_from_env()
    if info.distributed:
        torch.cuda.set_device(info.local)
        R.init(info, timeout_s=120.0)
    return info.world, info.rank, info.local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples while the GPU is under load.

    Queries every GPU and keeps the rows of the one torch is using (matched
    by UUID, else by the CUDA_VISIBLE_DEVICES ordinal, else index 0)."""

    FIELDS = ("uuid,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(dev).uuid).lower()
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        k = dev.index or 0
        self.fallback_index = ids[k] if k < len(ids) and ids[k].isdigit() else str(k)
        self.rows, self.proc, self.note = [], None, None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError) as e:
            self.proc, self.note = None, f"nvidia-smi unavailable: {e}"

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def _mine(self, r):
        if self.uuid and self.uuid in r[0].lower():
            return True
        return False

    def stop(self, t0, t1):
        if self.proc is None:
            return {"note": self.note}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        allrows = [(ts, r) for ts, r in self.rows if len(r) >= 10]
        mine = [(ts, r) for ts, r in allrows if self._mine(r)]
        if not mine:
            mine = [(ts, r) for ts, r in allrows if r[1] == self.fallback_index]
        if not mine:
            return {"note": "no nvidia-smi samples", "raw_rows": len(self.rows)}
        win = [r for ts, r in mine if t0 - 0.15 <= ts <= t1 + 0.15]
        rows = win or [r for _, r in mine]

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [x for x in (num(r[2]) for r in rows) if x is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][3]),
                "reasons": reasons, "samples": len(rows),
                "window": "timed region" if win else "whole run (timed region shorter than one sample)"}


QUANT_SOURCES = ("quant_tma.cuh", "quant_kernels.cuh", "cf_common.cuh", "mbar.cuh", "cf_api.cu")
LOWRANK_APPLY_SOURCES = ("lowrank_apply_tc.cuh", "lowrank_umma.cuh", "lowrank_kernels.cuh",
                         "lowrank_api.cuh", "lowrank.cu", "cf_common.cuh", "mbar.cuh")


def kernel_source_hash(files=QUANT_SOURCES):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "activation_residual_compression_cf_b200", "csrc")
    for fn in files:
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, files=QUANT_SOURCES):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}:{workload}")
    if not d or d.get("source_hash") != kernel_source_hash(files):
        return None
    return d.get("dram_bytes_per_launch")


def recorded_tensor_pipe():
    """Tensor-pipe activity of the low-rank kernels from the committed ncu
    summary (profiles/tensor_pipe.json), if it was taken on the current
    low-rank sources; else None."""
    p = os.path.join(ROOT, "profiles", "tensor_pipe.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != kernel_source_hash(LOWRANK_APPLY_SOURCES):
        return None
    return {"kernels": d["kernels"], "metric": d["metric"], "capture": d["capture"]}


# ------------------------------------------------------------ CPU oracle leg

def oracle_sample(wl, seconds, max_buffer_steps=10**9):
    """Times the oracle's encode+decode on host copies of buffer 0's
    trajectory (cycled) until `seconds` of work; returns (GB/s, detail)."""
    import oracle
    xs = W.trajectory(wl, 0, steps=min(wl.steps, 4), device="cpu")
    xb = [W.bf16_bits(x) for x in xs]
    recon_s, _ = oracle.state_init(xb[0])
    recon_r = recon_s.copy()
    done, t_work, i = 0, 0.0, 0
    while t_work < seconds and done < max_buffer_steps:
        x = xb[1 + i % (len(xb) - 1)]
        t0 = time.perf_counter()
        codes, scales, _ = oracle.encode(x, recon_s, wl.bits)
        oracle.decode(codes, scales, recon_r, wl.bits)
        t_work += time.perf_counter() - t0
        done += 1
        i += 1
    gbs = 2 * wl.elems * done / t_work / 1e9
    return gbs, done, t_work


def blas_threads():
    """Threads the host BLAS that numpy calls into actually uses."""
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


class LowrankOracleStepper:
    """The oracle's low-rank sender + receiver on host copies of buffer 0's
    trajectory (cycled), one buffer-step per call."""

    def __init__(self, wl):
        from oracle import lowrank as OL
        self.OL, self.wl = OL, wl
        xs = W.trajectory(wl, 0, steps=min(wl.steps, 4), device="cpu")
        self.xb = [W.bf16_bits(x) for x in xs]
        self.om = [W.omega(wl, 0, s, device="cpu").numpy() for s in range(len(xs))]
        self.recon_s = OL.bf16_bits_to_f32(self.xb[0]).copy()
        self.recon_r = self.recon_s.copy()
        self.i = 0

    def __call__(self):
        k = 1 + self.i % (len(self.xb) - 1)
        o = self.OL.lowrank_encode(self.xb[k], self.recon_s, self.om[k], self.wl.iters)
        self.OL.lowrank_decode(o["p_codes"], o["p_scales"], o["q_codes"], o["q_scales"],
                               self.recon_r, self.wl.rank)
        self.i += 1


def lowrank_oracle_sample(wl, seconds):
    step = LowrankOracleStepper(wl)
    done, t_work = 0, 0.0
    while t_work < seconds:
        t0 = time.perf_counter()
        step()
        t_work += time.perf_counter() - t0
        done += 1
    return 2 * wl.elems * done / t_work / 1e9, done, t_work


def _oracle_worker(job):
    """One host core's share of the all-cores oracle sample (a spawned
    process): buffer `b`'s trajectory, encode+decode for `seconds`."""
    wl, b, seconds = job
    import oracle
    xs = W.trajectory(wl, b, steps=min(wl.steps, 4), device="cpu")
    xb = [W.bf16_bits(x) for x in xs]
    recon_s, _ = oracle.state_init(xb[0])
    recon_r = recon_s.copy()
    done, t_work, i = 0, 0.0, 0
    while t_work < seconds:
        x = xb[1 + i % (len(xb) - 1)]
        t0 = time.perf_counter()
        codes, scales, _ = oracle.encode(x, recon_s, wl.bits)
        oracle.decode(codes, scales, recon_r, wl.bits)
        t_work += time.perf_counter() - t0
        done += 1
        i += 1
    return 2 * wl.elems * done / t_work


def oracle_sample_all_cores(wl, seconds):
    """The same oracle on every host core at once, one spawned process per
    core, each on its own buffer; returns (aggregate GB/s, cores, model)."""
    import multiprocessing as mp
    cores = len(os.sched_getaffinity(0))
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    with mp.get_context("spawn").Pool(cores) as pool:
        rates = pool.map(_oracle_worker, [(wl, b % wl.buffers, seconds) for b in range(cores)])
    return sum(rates) / 1e9, cores, model


# ------------------------------------------------------------ config

def quant_config(args, wl, world):
    """The `config` of a quantize-mode line; both arms print this same dict."""
    n, T, C, bits = wl.buffers, wl.tokens, wl.channels, wl.bits
    return {"workload": args.workload, "tokens": T, "channels": C, "buffers": n,
            "bits": bits, "mode": f"{bits}-bit {'mean-abs' if bits == 1 else 'absmax'} + EF"
            + (", delta-state sender" if args.delta else "")
            + (", emitting decode" if args.emit else ""),
            "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2 ({n * T * C * 14 / 1e9:.1f} GB touched per step)",
            "launches_per_step": 2}


def lowrank_config(args, wl, world):
    """The `config` of a low-rank line; both arms print this same dict."""
    it = wl.iters
    return {"workload": "lowrank", "tokens": wl.tokens, "channels": wl.channels,
            "buffers": wl.buffers, "rank": wl.rank, "iters": it,
            "mode": "low-rank INT4 + EF" + (", warm start" if args.warm else ""),
            "parallelism": f"replicas x{world}", "l2": "inputs larger than L2",
            "launches_per_step": 4 + 3 * it + 1}


def lowrank_workload(args):
    wl = W.WORKLOADS["lowrank"]
    if args.workload == "lowrank" and args.buffers:
        wl = W.replace(wl, buffers=args.buffers)
    if args.iters:
        wl = W.replace(wl, iters=args.iters)
    if args.rank:
        wl = W.replace(wl, rank=args.rank)
    return wl


# ------------------------------------------------------------ GPU leg

def run_ours(args, world, rank, local):
    from activation_residual_compression_cf_b200 import build, cf
    build.build()
    cf.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = W.WORKLOADS[args.workload]
    if args.buffers:
        wl = W.replace(wl, buffers=args.buffers)
    if args.pipeline >= 0:
        cf.cf_set_quant_pipeline(0, args.pipeline, 0)
        cf.cf_set_quant_pipeline(1, args.pipeline, 0)
    n, T, C, bits = wl.buffers, wl.tokens, wl.channels, wl.bits
    d = cf.desc(T, C, bits)
    Wd = cf.cf_codes_words_per_row(d)

    # Pre-generate the trajectory (as many steps as fit a 40 GB budget).
    step_bytes = n * T * C * 2
    S = max(2, min(wl.steps, int(40e9 // step_bytes)))
    if args.gen_steps:
        S = max(2, min(S, args.gen_steps))
    X = torch.empty((S, n, T, C), dtype=torch.bfloat16, device=dev)
    for b in range(n):
        tr = W.Trajectory(wl, b, device=dev, seed=rank)
        for s in range(S):
            X[s, b] = tr.next()
    del tr
    f32 = dict(dtype=torch.float32, device=dev)
    recon_s = torch.empty((n, T, C), **f32)
    recon_r = torch.empty((n, T, C), **f32)
    err = torch.empty((n, T, C), **f32)
    codes = torch.empty((n, T, Wd), dtype=torch.int32, device=dev)
    scales = torch.empty((n, T), **f32)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    X16 = X.view(torch.int16)
    for b in range(n):
        cf.cf_state_init(d, X16[0, b], recon_s[b], err[b])
        cf.cf_state_init(d, X16[0, b], recon_r[b], None)
    if args.delta:
        # delta-state sender: x_prev = the previous generated step; err = 0
        for b in range(n):
            cf.cf_state_init(d, X16[0, b], None, err[b])
        enc = [cf.enc_delta_buffer_array([(X16[s, b], X16[s - 1, b], err[b], codes[b], scales[b])
                                          for b in range(n)], dev) if s > 0 else None
               for s in range(S)]
        encode_batched = cf.cf_encode_delta_batched
    else:
        enc = [cf.enc_buffer_array([(X16[s, b], recon_s[b], err[b], codes[b], scales[b])
                                    for b in range(n)], dev) for s in range(S)]
        encode_batched = cf.cf_encode_batched
    if args.emit:
        # the receiver also writes the bf16 reconstruction its attention reads
        out_bf16 = torch.empty((n, T, C), dtype=torch.bfloat16, device=dev)
        dec = cf.dec_emit_buffer_array([(codes[b], scales[b], recon_r[b], out_bf16[b].view(torch.int16))
                                        for b in range(n)], dev)
        decode_batched = cf.cf_decode_emit_batched
    else:
        dec = cf.dec_buffer_array([(codes[b], scales[b], recon_r[b]) for b in range(n)], dev)
        decode_batched = cf.cf_decode_batched
    stream = torch.cuda.current_stream(dev)

    def step(i):
        encode_batched(d, n, enc[1 + i % (S - 1)], status, stream)
        decode_batched(d, n, dec, status, stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with R.bracket():
        wall0 = time.time()
        t_start.record(stream)
        for i in range(args.steps):
            e0, e1, e2 = ev[i]
            e0.record(stream)
            encode_batched(d, n, enc[1 + (args.warmup + i) % (S - 1)], status, stream)
            e1.record(stream)
            decode_batched(d, n, dec, status, stream)
            e2.record(stream)
        t_end.record(stream)
    wall1 = time.time()
    clocks = sampler.stop(wall0, wall1)
    assert int(status.item()) == 0, cf.cf_status_string(int(status.item()))
    ms = t_start.elapsed_time(t_end)
    enc_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1, _ in ev)
    dec_ms = statistics.mean(e1.elapsed_time(e2) for _, e1, e2 in ev)
    ms = R.reduce_scalar(ms, "max")

    bytes_processed = 2 * T * C * n * args.steps * world
    value = bytes_processed / (ms / 1e3) / 1e9
    if args.delta:
        enc_bytes = n * T * (C * 2 * 2 + C * 4 * 2 + Wd * 4 + 4)  # x, x_prev, err r/w, codes, scale
    else:
        enc_bytes = n * T * (C * 2 + C * 4 * 3 + Wd * 4 + 4)     # x, recon r/w, err w, codes, scale
    dec_bytes = n * T * (Wd * 4 + 4 + C * 4 * 2)             # codes, scale, recon r/w
    if args.emit:
        dec_bytes += n * T * C * 2                           # bf16 copy out
    peak, peak_kind = peaks()
    enc_gbs = enc_bytes / (enc_ms / 1e3) / 1e9
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9

    # Invariants of the state after the run (no oracle): the receiver equals
    # the sender's mirror bit for bit, and recon_s + err == x of the last
    # step within the three fp32 roundings of a step (residual v, error,
    # mirror update: u (|v| + |err| + |recon|), with |v| <= |err| + the
    # row's scale since |deq| <= scale), for every buffer.
    invariants = None
    if not args.delta:
        last = X[1 + (args.warmup + args.steps - 1) % (S - 1)]
        gap_ok = True
        for b in range(n):
            xb = last[b].double()
            rs, er = recon_s[b].double(), err[b].double()
            sc = scales[b].double()[:, None]
            bound = (2 * er.abs() + sc + rs.abs()) * 2.0 ** -24 * (1 + 1e-6) + 3 * 2.0 ** -149
            gap_ok &= bool(((rs + er - xb).abs() <= bound).all())
            del xb, rs, er, sc, bound
        invariants = {"receiver_equals_sender": bool(torch.equal(recon_r.view(torch.int32),
                                                                 recon_s.view(torch.int32))),
                      "ef_identity_within_roundings": gap_ok, "buffers_checked": n}

    # End to end through the public API: pinned host x in, payload out.
    e2e = None
    if not args.no_e2e and not args.delta and not args.emit:
        e2e = run_e2e(cf, d, wl, args, dev, stream, recon_s, recon_r, err, codes, scales, status)
        e2e["ms"] = R.reduce_scalar(e2e["ms"], "max")
        e_steps = e2e["steps"]
        e2e = {"value": round(2 * T * C * n * e_steps * world / (e2e["ms"] / 1e3) / 1e9, 3),
               "unit": "GB/s", "steps": e_steps,
               "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
               "ms_per_step": round(e2e["ms"] / e_steps, 4),
               "overlap": f"{e2e['chunks']} chunks on copy-in / compute / copy-out streams"}

    # A reference for the encode's byte mix: a plain streaming pass over the
    # same slab (x in, recon in/out, err out: 6 B read, 8 B written per
    # element) with none of the per-row work, timed the same way.  Writes
    # dominate the mix, and HBM serves it slower than a copy's even split;
    # the encode is compared with this pass as well as with the copy peak.
    # It overwrites the states, which nothing reads after this point.
    mix = None
    if not args.delta and not args.emit:
        xs1 = X16[1].reshape(-1)
        for _ in range(3):
            cf.cf_diag_stream_mix(xs1, recon_s.view(-1), err.view(-1), stream)
        mev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(20)]
        for m0, m1 in mev:
            m0.record(stream)
            cf.cf_diag_stream_mix(xs1, recon_s.view(-1), err.view(-1), stream)
            m1.record(stream)
        torch.cuda.synchronize()
        mix_ms = statistics.mean(m0.elapsed_time(m1) for m0, m1 in mev)
        mix_gbs = n * T * C * 14 / (mix_ms / 1e3) / 1e9
        mix = {"kernel": "cf_diag_stream_mix (6 B read, 8 B written per element, no per-row work)",
               "achieved": round(mix_gbs, 1), "frac_of_peak": round(mix_gbs / peaks()[0], 4),
               "encode_over_reference": round(enc_gbs / mix_gbs, 4)}
        # the same mix through the encode's own row pipeline (TMA-staged rows)
        # and each of its two store paths, still without the per-row work:
        # the encode's time over that of its store path is what the scale
        # reduction, quantisation and codes cost.  bulk = per-thread stores
        # (the encode's path for long rows) or bulk stores from shared-memory
        # output rows (its path where four CTAs fit on an SM, C <= 2046)
        if C % 8 == 0 and C <= 15360:
            rows_all = n * T
            xs2 = xs1.view(rows_all, C)
            for key, bulk in (("staged", False), ("staged_bulk", True)):
                if bulk and 28 * C + 32 > 227 * 1024:
                    continue
                for _ in range(3):
                    cf.cf_diag_stream_mix_tma(xs2, recon_s.view(rows_all, C), err.view(rows_all, C), rows_all, C,
                                              status, stream, bulk=bulk)
                for m0, m1 in mev:
                    m0.record(stream)
                    cf.cf_diag_stream_mix_tma(xs2, recon_s.view(rows_all, C), err.view(rows_all, C), rows_all, C,
                                              status, stream, bulk=bulk)
                    m1.record(stream)
                torch.cuda.synchronize()
                st_ms = statistics.mean(m0.elapsed_time(m1) for m0, m1 in mev)
                st_gbs = n * T * C * 14 / (st_ms / 1e3) / 1e9
                what = ("bulk stores from two shared-memory output rows, 4 groups per thread, 2 slots" if bulk
                        else "per-thread streaming stores, 2 groups per thread")
                mix[key] = {"kernel": f"cf_diag_stream_mix_tma (the same bytes through the encode's TMA row "
                                      f"pipeline, {what}; no per-row work)",
                            "achieved": round(st_gbs, 1), "frac_of_peak": round(st_gbs / peaks()[0], 4),
                            "encode_over_reference": round(enc_gbs / st_gbs, 4),
                            "status": int(status.item())}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, done, tw = oracle_sample(wl, args.cpu_seconds)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{done} buffer-steps of {args.workload} buffer 0 ({T}x{C}, "
                         f"{bits}-bit encode+decode), {tw:.1f} s single-threaded C"}
        try:
            agg, cores, model = oracle_sample_all_cores(wl, min(5.0, args.cpu_seconds))
            cpu["all_cores"] = {"value": round(agg, 4), "unit": "GB/s", "cores": cores,
                                "cpu_model": model,
                                "sample": "the same C oracle in one process per host core, "
                                          "each on its own buffer, rates summed"}
        except Exception as exc:  # a host without spawn support still reports one core
            cpu["all_cores"] = {"unavailable": str(exc)[:200]}

    traffic = recorded_traffic("encode_delta" if args.delta else "encode", args.workload)
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "dtype_note": "bf16 activations in; fp32 state and arithmetic (fp64 1-bit sums)",
        "data": "synthetic",
        "config": quant_config(args, wl, world),
        "roofline": {"bound": "hbm", "achieved": round(enc_gbs, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(enc_gbs / peak, 4), "traffic": traffic,
                     "kernel": ("encode_tma_kernel (batched, TMA row staging)" if args.pipeline != 0
                                else "encode_rows_kernel (batched, register rows)")
                     + (", delta-state sender" if args.delta else "")
                   + (", emitting decode" if args.emit else ""),
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": enc_bytes, "avg_launch_ms": round(enc_ms, 4),
                     "mix_reference": mix},
        "decode": {"achieved": round(dec_gbs, 1), "frac": round(dec_gbs / peak, 4),
                   "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_ms": round(dec_ms, 4)},
        # the whole timed step against the same roofline: both launches'
        # algorithmic bytes over the step time (the slowest rank's)
        "step_roofline": {"algorithmic_bytes_per_step": enc_bytes + dec_bytes,
                          "achieved": round((enc_bytes + dec_bytes) * args.steps / (ms / 1e3) / 1e9, 1),
                          "frac": round((enc_bytes + dec_bytes) * args.steps / (ms / 1e3) / 1e9 / peak, 4)},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "invariants": invariants,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    return out


def run_exchange(args, world, rank, local):
    """The sequence-parallel exchange: per step one batched encode into the
    payload, one all-gather of the payloads, one batched decode of every
    peer's shard (of its own too when alone)."""
    from activation_residual_compression_cf_b200 import build, cf
    from activation_residual_compression_cf_b200.exchange import FusedShardExchange, ShardExchange
    build.build()
    cf.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = W.WORKLOADS[args.workload]
    if args.buffers:
        wl = W.replace(wl, buffers=args.buffers)
    n, T, C, bits = wl.buffers, wl.tokens, wl.channels, wl.bits
    S = max(2, min(wl.steps, int(40e9 // (n * T * C * 2))))
    if args.gen_steps:
        S = max(2, min(S, args.gen_steps))
    X = torch.empty((S, n, T, C), dtype=torch.bfloat16, device=dev)
    for b in range(n):
        tr = W.Trajectory(wl, b, device=dev, seed=rank)
        for s in range(S):
            X[s, b] = tr.next()
    kind = FusedShardExchange if args.fused else ShardExchange
    ex = kind(T, C, bits, n, device=dev, loopback=(world == 1))
    ex.warmup([X[0, b] for b in range(n)])
    stream = torch.cuda.current_stream(dev)

    def xs(i):
        return [X[1 + i % (S - 1), b] for b in range(n)]

    for i in range(S - 1):
        ex.prepare(xs(i))

    sampler = ClockSampler(dev)
    sampler.start()
    for i in range(args.warmup):
        ex.step(xs(i))
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with R.bracket():
        wall0 = time.time()
        t_start.record(stream)
        for i in range(args.steps):
            ex.step(xs(args.warmup + i), events=ev[i])
        t_end.record(stream)
    wall1 = time.time()
    clocks = sampler.stop(wall0, wall1)
    st = ex.codec.status_value()
    assert st == 0, cf.cf_status_string(st)
    ms = R.reduce_scalar(t_start.elapsed_time(t_end), "max")
    phase = [statistics.mean(e[k].elapsed_time(e[k + 1]) for e in ev) for k in range(3)]
    Wd = ex.layout.words_per_row
    enc_bytes = n * T * (C * 2 + C * 4 * 3 + Wd * 4 + 4)
    dec_bytes = len(ex.peers) * n * T * (Wd * 4 + 4 + C * 4 * 2)
    peak, peak_kind = peaks()
    enc_gbs = enc_bytes / (phase[0] / 1e3) / 1e9
    value = 2 * T * C * n * args.steps * world / (ms / 1e3) / 1e9
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "dtype_note": "bf16 activations in; fp32 state and arithmetic (fp64 1-bit sums)",
        "data": "synthetic",
        "config": {"workload": args.workload, "tokens": T, "channels": C, "buffers": n,
                   "bits": bits, "mode": f"{bits}-bit + EF, sequence-parallel exchange"
                   + (", fused" if args.fused else ""),
                   "parallelism": f"sp{world} (all-gather of payloads)",
                   "l2": "inputs larger than L2", "launches_per_step": 2},
        "roofline": {"bound": "hbm", "achieved": round(enc_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(enc_gbs / peak, 4),
                     "traffic": recorded_traffic("encode", args.workload),
                     "kernel": ("encode_tma_unit_kernel (publishing: codes and scales stored into "
                                "the receivers' slots)" if args.fused
                                else "encode_tma_kernel (batched, codes written into the payload)"),
                     "peak_kind": peak_kind, "algorithmic_bytes_per_launch": enc_bytes,
                     "avg_launch_ms": round(phase[0], 4)},
        "exchange": {"encode_ms": round(phase[0], 4), "all_gather_ms": round(phase[1], 4),
                     "decode_ms": round(phase[2], 4), "payload_bytes_per_rank": ex.payload_bytes_per_step(),
                     "decoded_shards": len(ex.peers) * n,
                     "decode_frac": round(dec_bytes / (phase[2] / 1e3) / 1e9 / peak, 4),
                     "collective": ("none: the encode stores into the receivers' slots, the decode "
                                    "waits on their counters" if args.fused
                                    else ex.backend or "local copy (one rank)")},
        "cpu_baseline": None, "e2e": None,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }


def run_lowrank(args, world, rank, local):
    """Low-rank mode: per step, cf_lowrank_encode then cf_lowrank_decode for
    every buffer (one workspace, reused in stream order)."""
    from activation_residual_compression_cf_b200 import build, cf
    build.build()
    cf.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = lowrank_workload(args)
    n, T, C, r, it = wl.buffers, wl.tokens, wl.channels, wl.rank, wl.iters
    d = cf.desc(T, C, 0, r, it)
    if args.lowrank_group >= 0:
        cf.cf_set_lowrank_group(args.lowrank_group)
    step_bytes = n * T * C * 2
    S = max(2, min(wl.steps, int(30e9 // step_bytes)))
    if args.gen_steps:
        S = max(2, min(S, args.gen_steps))
    X = torch.empty((S, n, T, C), dtype=torch.bfloat16, device=dev)
    OM = torch.empty((S, n, C, r), dtype=torch.float32, device=dev)
    for b in range(n):
        tr = W.Trajectory(wl, b, device=dev, seed=rank)
        for s in range(S):
            X[s, b] = tr.next()
            OM[s, b] = W.omega(wl, b, s, device=dev, seed=rank)
    f32 = dict(dtype=torch.float32, device=dev)
    recon_s = torch.empty((n, T, C), **f32)
    recon_r = torch.empty((n, T, C), **f32)
    err = torch.empty((n, T, C), **f32)
    nb = (r + 1) // 2
    pc = torch.empty((n, T * nb + 16), dtype=torch.uint8, device=dev)
    qc = torch.empty((n, C * nb + 16), dtype=torch.uint8, device=dev)
    ps = torch.empty((n, max(r, 4)), **f32)
    qs = torch.empty((n, max(r, 4)), **f32)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    ws = torch.empty(n * wsb, dtype=torch.uint8, device=dev)
    X16 = X.view(torch.int16)
    for b in range(n):
        cf.cf_state_init(d, X16[0, b], recon_s[b], err[b])
        cf.cf_state_init(d, X16[0, b], recon_r[b], None)
    stream = torch.cuda.current_stream(dev)
    # one batched call per step for all buffers (encode) and one for decode
    encs = [cf.lowrank_buffer_array([(X16[s, b], recon_s[b], err[b], OM[s, b], pc[b], ps[b],
                                      qc[b], qs[b]) for b in range(n)], dev) for s in range(S)]
    # warm start: omega NULL, the iteration starts from the previous Q
    warms = [cf.lowrank_buffer_array([(X16[s, b], recon_s[b], err[b], None, pc[b], ps[b],
                                       qc[b], qs[b]) for b in range(n)], dev) for s in range(S)]
    decs = cf.lowrank_dec_buffer_array([(pc[b], ps[b], qc[b], qs[b], recon_r[b]) for b in range(n)],
                                       dev)

    def enc(i):
        src = warms if (args.warm and i > 0) else encs
        cf.cf_lowrank_encode_batched(d, n, src[1 + i % (S - 1)], ws, stream=stream)

    def dec():
        cf.cf_lowrank_decode_batched(d, n, decs, stream=stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for i in range(args.warmup):
        enc(i)
        dec()
    torch.cuda.synchronize()

    def events(k):
        return [torch.cuda.Event(enable_timing=True) for _ in range(k)]

    ev = [events(3) for _ in range(args.steps)]
    # events the library records around the sender's and the receiver's
    # apply kernel (recorded once here so that they exist)
    aev = [events(4) for _ in range(args.steps)]
    for e in aev:
        for x_ in e:
            x_.record(stream)
    torch.cuda.synchronize()
    with R.bracket():
        wall0 = time.time()
        for i in range(args.steps):
            e0, e1, e2 = ev[i]
            cf.cf_lowrank_set_apply_events(*aev[i])
            e0.record(stream)
            enc(args.warmup + i)
            e1.record(stream)
            dec()
            e2.record(stream)
    cf.cf_lowrank_set_apply_events()
    clocks = sampler.stop(wall0, time.time())
    ms = ev[0][0].elapsed_time(ev[-1][2])
    enc_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    dec_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    app_enc_ms = statistics.mean(a[0].elapsed_time(a[1]) for a in aev)
    app_dec_ms = statistics.mean(a[2].elapsed_time(a[3]) for a in aev)
    ms = R.reduce_scalar(ms, "max")
    peak, peak_kind = peaks()
    value = 2 * T * C * n * args.steps * world / (ms / 1e3) / 1e9
    enc_bytes = n * T * C * 14
    dec_bytes = n * T * C * 8
    # apply kernels: x, recon r/w, err (sender) or recon r/w (receiver), plus
    # the packed factors and their scales
    fac_bytes = n * ((T + C) * nb + 2 * 4 * r)
    app_enc_bytes = enc_bytes + fac_bytes
    app_dec_bytes = dec_bytes + fac_bytes
    status = max(cf.cf_lowrank_status(ws[b * wsb:]) for b in range(n))
    # Launches per step: the sender runs prep, omega, three kernels per
    # subspace iteration (project with its Gram/Cholesky tail -- the first
    # one also forms the bf16 residual --, orthogonalise, back-project with
    # its Q-reduction tail), one INT4 pack of both factors and the apply; the
    # receiver one.
    launches_per_step = 4 + 3 * it + 1

    e2e = None
    if not args.no_e2e:
        e2e = run_lowrank_e2e(cf, d, wl, args, dev, stream, recon_s, recon_r, err, OM, pc, ps,
                              qc, qs, ws)
        e2e["ms"] = R.reduce_scalar(e2e["ms"], "max")
        e_steps = e2e["steps"]
        e2e = {"value": round(2 * T * C * n * e_steps * world / (e2e["ms"] / 1e3) / 1e9, 3),
               "unit": "GB/s", "steps": e_steps, "h2d_bytes_per_step": e2e["h2d"],
               "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(e2e["ms"] / e_steps, 4),
               "overlap": f"{e2e['chunks']} chunks on copy-in / compute / copy-out streams"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, done, tw = lowrank_oracle_sample(wl, args.cpu_seconds)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{done} buffer-steps of {args.workload} buffer 0 ({T}x{C}, rank {r}, "
                         f"{it} iterations, encode+decode), {tw:.1f} s of numpy fp64"}
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "dtype_note": "bf16 activations in; fp32 state; bf16 and tf32 tensor products "
                                      "with fp32 accumulation",
        "data": "synthetic",
        "config": lowrank_config(args, wl, world),
        "roofline": {"bound": "hbm",
                     "achieved": round(app_enc_bytes / (app_enc_ms / 1e3) / 1e9, 1),
                     "peak": peak, "unit": "GB/s",
                     "frac": round(app_enc_bytes / (app_enc_ms / 1e3) / 1e9 / peak, 4),
                     "traffic": recorded_traffic("apply_sender", args.workload,
                                                 LOWRANK_APPLY_SOURCES),
                     "kernel": "lr_apply_tc_kernel<sender> (batched; D, EF update)",
                     "peak_kind": peak_kind, "algorithmic_bytes_per_launch": app_enc_bytes,
                     "avg_launch_ms": round(app_enc_ms, 4)},
        "decode": {"kernel": "lr_apply_tc_kernel<receiver> (batched)",
                   "achieved": round(app_dec_bytes / (app_dec_ms / 1e3) / 1e9, 1),
                   "frac": round(app_dec_bytes / (app_dec_ms / 1e3) / 1e9 / peak, 4),
                   "algorithmic_bytes_per_launch": app_dec_bytes,
                   "avg_launch_ms": round(app_dec_ms, 4)},
        "whole_call": {"encode_ms_per_step": round(enc_ms, 4),
                       "decode_ms_per_step": round(dec_ms, 4),
                       "encode_frac_of_14B_per_elem": round(
                           enc_bytes / (enc_ms / 1e3) / 1e9 / peak, 4)},
        "lowrank_status": status,
        "tensor_pipe": recorded_tensor_pipe(),
        "payload_ratio": round(2 * T * C / cf.cf_payload_bytes(d), 2),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    return out


def lowrank_leg(args, world, rank, local):
    """The low-rank mode on its own workload (114 x 4096 x 3072, rank 32, 2
    iterations), timed like run_lowrank after the quantize line has freed its
    memory: the part of its line that the quantize line does not carry."""
    torch.cuda.empty_cache()
    la = argparse.Namespace(**vars(args))
    la.workload, la.buffers, la.warm = "lowrank", 0, False
    la.steps = max(1, min(args.steps, args.lowrank_steps))
    la.warmup = max(3, min(args.warmup, 5))
    la.gen_steps, la.no_e2e, la.no_cpu_baseline = 3, True, True
    o = run_lowrank(la, world, rank, local)
    keys = ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "config", "roofline",
            "decode", "whole_call", "tensor_pipe", "lowrank_status", "payload_ratio",
            "gpu_launches", "clocks")
    return {k: o[k] for k in keys if k in o}


def run_lowrank_e2e(cf, d, wl, args, dev, stream, recon_s, recon_r, err, OM, pc, ps, qc, qs, ws):
    """Low-rank end to end: every step copies the pinned host activations of
    all buffers in, runs the batched sender and receiver, and reads the INT4
    payload (factor codes and scales) back to the host.  Chunks of buffers on
    three streams overlap the copies with the kernels, as in run_e2e."""
    n, T, C = wl.buffers, wl.tokens, wl.channels
    nch = max(1, min(args.e2e_chunks, n))
    bounds = [round(k * n / nch) for k in range(nch + 1)]
    tr = W.Trajectory(wl, 0, device=dev)
    tr.next()
    x_host = []
    for _ in range(2):
        xk = tr.next().unsqueeze(0).expand(n, T, C).contiguous().cpu()
        x_host.append(xk.pin_memory())
        del xk
    x_dev = [torch.empty((n, T, C), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    wsb = cf.cf_lowrank_workspace_bytes(d)
    enc = [[cf.lowrank_buffer_array([(x_dev[slot].view(torch.int16)[b], recon_s[b], err[b], OM[1, b],
                                      pc[b], ps[b], qc[b], qs[b])
                                     for b in range(bounds[k], bounds[k + 1])], dev)
            for k in range(nch)] for slot in range(2)]
    dec = [cf.lowrank_dec_buffer_array([(pc[b], ps[b], qc[b], qs[b], recon_r[b])
                                        for b in range(bounds[k], bounds[k + 1])], dev)
           for k in range(nch)]
    outs = [pc, ps, qc, qs]
    host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    d2h_done = [None] * nch
    enc_done = [[None] * nch for _ in range(2)]

    def step(i):
        slot = i % 2
        for k in range(nch):
            lo, hi = bounds[k], bounds[k + 1]
            e_in, e_done, e_out = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if enc_done[slot][k] is not None:
                    s_in.wait_event(enc_done[slot][k])
                x_dev[slot][lo:hi].copy_(x_host[slot][lo:hi], non_blocking=True)
                e_in.record(s_in)
            stream.wait_event(e_in)
            if d2h_done[k] is not None:
                stream.wait_event(d2h_done[k])
            cf.cf_lowrank_encode_batched(d, hi - lo, enc[slot][k], ws[lo * wsb:], stream=stream)
            cf.cf_lowrank_decode_batched(d, hi - lo, dec[k], stream=stream)
            e_done.record(stream)
            enc_done[slot][k] = e_done
            s_out.wait_event(e_done)
            with torch.cuda.stream(s_out):
                for h, t in zip(host, outs):
                    h[lo:hi].copy_(t[lo:hi], non_blocking=True)
                e_out.record(s_out)
            d2h_done[k] = e_out

    def settle():
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    for i in range(max(3, args.warmup)):
        step(i)
    settle()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, args.e2e_steps))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    for i in range(steps):
        step(i)
    settle()
    b.record(stream)
    torch.cuda.synchronize()
    st = max(cf.cf_lowrank_status(ws[k * wsb:]) for k in range(n))
    assert st in (0, 6), cf.cf_status_string(st)
    return {"ms": a.elapsed_time(b), "h2d": n * T * C * 2,
            "d2h": sum(t.numel() * t.element_size() for t in outs), "chunks": nch, "steps": steps}


def run_e2e(cf, d, wl, args, dev, stream, recon_s, recon_r, err, codes, scales, status):
    """End to end through the C ABI with host buffers: every step copies the
    pinned host activations of all buffers in, encodes and decodes them, and
    reads the payload (codes, scales) back.  The step is split into chunks of
    buffers on three streams -- host-to-device copies, the library calls,
    device-to-host copies -- ordered by events, so the copies of one chunk
    overlap the kernels of its neighbours (what a serving loop does with the
    same calls).  The activations land in two alternating device slots, so a
    step's copies never wait on the previous step's kernels."""
    n, T, C = wl.buffers, wl.tokens, wl.channels
    nch = max(1, min(args.e2e_chunks, n))
    bounds = [round(k * n / nch) for k in range(nch + 1)]
    # Two host steps of pinned input (buffer 0's trajectory replicated over
    # the buffers), alternated so consecutive steps see a real residual.
    tr = W.Trajectory(wl, 0, device=dev)
    tr.next()
    x_host = []
    for _ in range(2):
        xk = tr.next().unsqueeze(0).expand(n, T, C).contiguous().cpu()
        x_host.append(xk.pin_memory())
        del xk
    x_dev = [torch.empty((n, T, C), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    enc = [[cf.enc_buffer_array([(x_dev[slot].view(torch.int16)[b], recon_s[b], err[b], codes[b],
                                  scales[b]) for b in range(bounds[k], bounds[k + 1])], dev)
            for k in range(nch)] for slot in range(2)]
    dec = [cf.dec_buffer_array([(codes[b], scales[b], recon_r[b])
                                for b in range(bounds[k], bounds[k + 1])], dev) for k in range(nch)]
    codes_h = torch.empty(codes.shape, dtype=codes.dtype).pin_memory()
    scales_h = torch.empty(scales.shape, dtype=scales.dtype).pin_memory()
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    d2h_done = [None] * nch      # last device-to-host copy of each chunk's payload
    enc_done = [[None] * nch for _ in range(2)]   # last kernels reading a slot's chunk

    def step(i):
        slot = i % 2
        for k in range(nch):
            lo, hi = bounds[k], bounds[k + 1]
            e_in, e_done, e_out = ev(), ev(), ev()
            with torch.cuda.stream(s_in):
                if enc_done[slot][k] is not None:
                    s_in.wait_event(enc_done[slot][k])   # slot's chunk no longer read
                x_dev[slot][lo:hi].copy_(x_host[slot][lo:hi], non_blocking=True)
                e_in.record(s_in)
            stream.wait_event(e_in)
            if d2h_done[k] is not None:
                stream.wait_event(d2h_done[k])   # payload of the last step read out
            cf.cf_encode_batched(d, hi - lo, enc[slot][k], status, stream)
            cf.cf_decode_batched(d, hi - lo, dec[k], status, stream)
            e_done.record(stream)
            enc_done[slot][k] = e_done
            s_out.wait_event(e_done)
            with torch.cuda.stream(s_out):
                codes_h[lo:hi].copy_(codes[lo:hi], non_blocking=True)
                scales_h[lo:hi].copy_(scales[lo:hi], non_blocking=True)
                e_out.record(s_out)
            d2h_done[k] = e_out

    def settle():
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    for i in range(max(3, args.warmup // 4)):
        step(i)
    settle()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, args.e2e_steps))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    for i in range(steps):
        step(i)
    settle()
    b.record(stream)
    torch.cuda.synchronize()
    return {"ms": a.elapsed_time(b), "h2d": n * T * C * 2,
            "d2h": codes.numel() * 4 + scales.numel() * 4, "chunks": nch, "steps": steps}


def run_reference(args, world, rank):
    """CPU oracle on the host cores, same metric/unit/config; rank 0 only."""
    if rank != 0:
        return None
    wl = W.WORKLOADS[args.workload]
    if wl.mode == "lowrank":
        wl = lowrank_workload(args)
        config = lowrank_config(args, wl, world)
    else:
        if args.buffers:
            wl = W.replace(wl, buffers=args.buffers)
        config = quant_config(args, wl, world)
    per_step = 1
    cores, kind = 1, "single-threaded C oracle"
    if wl.mode == "lowrank":
        lr_step = LowrankOracleStepper(wl)
        cores, kind = blas_threads(), "numpy fp64 oracle"

        def one(i):
            lr_step()
    else:
        import oracle
        xs = W.trajectory(wl, 0, steps=min(wl.steps, 4), device="cpu")
        xb = [W.bf16_bits(x) for x in xs]
        recon_s, _ = oracle.state_init(xb[0])
        recon_r = recon_s.copy()

        def one(i):
            for _ in range(per_step):
                x = xb[1 + i % (len(xb) - 1)]
                c, s, _ = oracle.encode(x, recon_s, wl.bits)
                oracle.decode(c, s, recon_r, wl.bits)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    sec = time.perf_counter() - t0
    value = 2 * wl.elems * per_step * args.steps / sec / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "dtype_note": "bf16 activations in; fp32 state and arithmetic (the oracle's fp64 sums and products)",
        "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step is {per_step} of the {wl.buffers} buffers "
                                   f"({wl.tokens}x{wl.channels}), {args.steps} steps, {kind}"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.impl == "reference":
        world, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        if W.WORKLOADS[args.workload].mode == "lowrank":
            out = run_lowrank(args, world, rank, local)
        elif args.exchange:
            out = run_exchange(args, world, rank, local)
        else:
            out = run_ours(args, world, rank, local)
            if not args.no_lowrank_leg:
                out["lowrank"] = lowrank_leg(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        R.finish()


if __name__ == "__main__":
    main()
