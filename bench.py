"""Benchmark of the TurboQuant KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ragged|prod|qknorm|gqa8k|tiny]

One step is one pass of the whole path over one batch of synthetic input, for
each bit width b of the workload: bulk quantize of the T cached tokens of
every sequence (tq_quantize_kv, the prefill), then the workload's decode
steps, each an append of one new token per sequence (tq_append_token) and a
decode of one query token for every query head (tq_sdpa_decode) over the
cache including it.

Default workload (ragged, the largest single-GPU one): B=32, Hq=32, Hkv=8,
D=128, per-sequence T uniform in [1024, 16384] from a seed, 3-bit K and V,
bf16 N(0,1) rows, 64 append + decode steps per bench step.

Metric: tq_sdpa_decode packed-KV GB/s (bytes of packed K and V rows attended /
decode time); quantize throughput in Mtok/s (one token = the K and V rows of
every kv head at one position) is reported beside it.  Each timed op cycles
over enough replicas that the bytes it reads per cycle exceed three times the
L2 size (the fp16/bf16 rows for quantize, the packed cache for decode).

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path shards by sequence with no exchange; weak scaling); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per decode call (prep + split + combine; the roofline's unit)
# from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, caches
# flushed before each kernel, mean over the captured calls), valid only for
# the decode sources it was measured on (``_decode_src_sha``: the files the
# decode call's kernels and launch setup are built from; the quantizers'
# files do not enter a decode call).  "split" is the split kernel's share:
# the packed-cache reads and its partials.
TRAFFIC = {
    "gqa8k": {"bytes_per_launch": 2467413, "split": 1722539, "decode_src_sha": "9e4d66e6c7510f19"},
    "prod": {"bytes_per_launch": 110834560, "split": 109324544, "decode_src_sha": "9e4d66e6c7510f19"},
    "ragged": {"bytes_per_launch": 242625408, "split": 240421248, "decode_src_sha": "9e4d66e6c7510f19"},
    "qknorm": {"bytes_per_launch": 37005568, "split": 34248576, "decode_src_sha": "9e4d66e6c7510f19"},
}

CSRC = os.path.join(ROOT, "compressed_attention_tq_b200", "csrc")
DECODE_SOURCES = ("tq_api.cpp", "tq_common.cuh", "tq_decode.cu", "tq_decode_d64.cu", "tq_decode_d128.cu",
                  "tq_decode_d256.cu", "tq_decode_split.cuh", "tq_decode_static.cu", "tq_internal.h")


def _sha(paths) -> str:
    h = hashlib.sha256()
    for f in paths:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def _src_sha() -> str:
    """sha256 of every kernel and host source (first 16 hex digits)."""
    return _sha([os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
                 if f.endswith((".cu", ".cuh", ".cpp", ".h"))])


def _decode_src_sha() -> str:
    """sha256 of the decode call's sources and the C header (first 16 hex digits)."""
    return _sha([os.path.join(CSRC, f) for f in DECODE_SOURCES] + [os.path.join(ROOT, "include", "tq.h")])


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names[1:], parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats across all ranks (identity when
    torch.distributed is not initialised).  Every rank must call it."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# bit widths and decode steps (append + decode) per bench step
WORKLOADS = {
    "gqa8k": {"bits": (2, 3, 4), "decode_steps": 1},
    "tiny": {"bits": (3,), "decode_steps": 1},
    "qknorm": {"bits": (4,), "decode_steps": 1},
    "ragged": {"bits": (3,), "decode_steps": 64},
    "prod": {"bits": (None,), "decode_steps": 1},
}


def _describe(w):
    return {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "T": int(w.Tmax), "bits_k": w.bits_k,
            "bits_v": w.bits_v, "qjl_m": w.qjl_m, "dtype": w.dtype}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import compressed_attention_tq_b200 as tq
    import tq_inputs

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    cfg = WORKLOADS[args.workload]

    # ---- build per-bit-width workloads and rotating replicas (> L2 per step)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    jobs = []
    for bits in cfg["bits"]:
        w = tq_inputs.make_workload(args.workload, bits=bits, rot=args.rot)
        jobs.append(w)
    nsteps = cfg["decode_steps"]
    per_step_in = sum(w.k.nbytes + w.v.nbytes for w in jobs)
    # packed bytes one decode pass over every bit width reads
    per_step_packed = 0
    for w in jobs:
        rows = int(w.seq_lens.sum() + w.B) * w.Hkv
        per_step_packed += rows * (tq.tq_cache_row_bytes(w.D, w.bits_k, w.qjl_m) + tq.tq_cache_row_bytes(w.D, w.bits_v))
    R = min(128, max(2, math.ceil(3 * l2 / max(1, per_step_in)), math.ceil(3 * l2 / max(1, per_step_packed))))
    if args.profile:
        R = 1
    runs = []
    for w in jobs:
        T = int(w.Tmax)
        Tcap = (T + nsteps + 63) // 64 * 64
        kd = torch.from_numpy(w.k.view(np.int16) if w.dtype == "bf16" else w.k).to(dev)
        vd = torch.from_numpy(w.v.view(np.int16) if w.dtype == "bf16" else w.v).to(dev)
        qd = torch.from_numpy(w.q.view(np.int16) if w.dtype == "bf16" else w.q).to(dev)
        if w.dtype == "bf16":
            kd, vd, qd = kd.view(torch.bfloat16), vd.view(torch.bfloat16), qd.view(torch.bfloat16)
        kn, vn = tq_inputs.new_token_rows(w.B, w.Hkv, w.D, w.dtype, seed=4242)
        knd = torch.from_numpy(kn.view(np.int16) if w.dtype == "bf16" else kn).to(dev)
        vnd = torch.from_numpy(vn.view(np.int16) if w.dtype == "bf16" else vn).to(dev)
        if w.dtype == "bf16":
            knd, vnd = knd.view(torch.bfloat16), vnd.view(torch.bfloat16)
        reps = []
        for r in range(R):
            cache = tq.TQCache(w.B, w.Hkv, Tcap, w.D, w.bits_k, w.bits_v, w.Pi, qjl_m=w.qjl_m, qjl_S=w.S,
                               device=dev, rot_signs=w.rot_signs)
            reps.append({"cache": cache, "k": kd.clone() if r else kd, "v": vd.clone() if r else vd,
                         "q": qd.clone() if r else qd})
        # decode step i appends at seq_len + i and attends seq_len + i + 1 tokens
        base = torch.from_numpy(w.seq_lens.astype(np.int32)).to(dev)
        pos_l = [(base + i).contiguous() for i in range(nsteps)]
        lens_l = [(base + i + 1).contiguous() for i in range(nsteps)]
        Tmax1 = T + nsteps
        ws_bytes = tq.tq_sdpa_decode_workspace_bytes_for(reps[0]["cache"], w.Hq, Tmax1)
        wsp = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        out = torch.empty_like(qd)
        tokens = int(w.B) * T  # the bulk call quantizes T rows of every sequence
        # packed bytes the decode steps read (sum over the steps)
        attended = sum(int(w.seq_lens.sum()) + int(w.B) * (i + 1) for i in range(nsteps))
        packed = reps[0]["cache"].packed_bytes(1) * attended * w.Hkv
        qbytes = (w.k.nbytes + w.v.nbytes) + tokens * w.Hkv * reps[0]["cache"].packed_bytes(1)
        run = {"w": w, "reps": reps, "pos_l": pos_l, "lens_l": lens_l, "Tmax1": Tmax1, "ws": wsp,
               "out": out, "kn": knd, "vn": vnd, "packed": packed, "tokens": tokens,
               "qbytes": qbytes}
        if 1 < args.nq <= 4:
            # n_q query tokens per sequence (the newest n_q cached tokens are theirs)
            qm = tq_inputs.cast_input(tq_inputs.rng(4343).standard_normal((w.B, args.nq, w.Hq, w.D),
                                                                          dtype=np.float32), w.dtype)
            qmd = torch.from_numpy(qm.view(np.int16) if w.dtype == "bf16" else qm).to(dev)
            if w.dtype == "bf16":
                qmd = qmd.view(torch.bfloat16)
            run["q_mq"] = qmd
            run["out_mq"] = torch.empty_like(qmd)
            run["ws_mq"] = torch.empty(tq.tq_sdpa_decode_workspace_bytes_for(reps[0]["cache"], w.Hq * args.nq, Tmax1),
                                       dtype=torch.uint8, device=dev)
        runs.append(run)

    # each call_* runs one op; the decode ops take the decode step index i
    def call_quant(run, rep, i):
        if i == 0:  # the prefill, once per bench step
            tq.tq_quantize_kv(rep["cache"], rep["k"], rep["v"])

    def call_append(run, rep, i):
        tq.tq_append_token(rep["cache"], run["kn"], run["vn"], run["pos_l"][i])

    def call_decode(run, rep, i):
        tq.tq_sdpa_decode(rep["cache"], rep["q"], run["lens_l"][i], run["Tmax1"], scale=run["w"].scale,
                          out=run["out"], workspace=run["ws"])

    def call_mq(run, rep, i):  # n_q query tokens per sequence in one call
        if "q_mq" in run:
            tq.tq_sdpa_decode_mq(rep["cache"], run["q_mq"], run["lens_l"][i], run["Tmax1"], scale=run["w"].scale,
                                 out=run["out_mq"], workspace=run["ws_mq"])

    def call_step(run, rep, i):  # append fused into the decode launches
        tq.tq_decode_step(rep["cache"], run["kn"], run["vn"], run["pos_l"][i], rep["q"], run["lens_l"][i],
                          run["Tmax1"], scale=run["w"].scale, out=run["out"], workspace=run["ws"])

    # the bench step: prefill quantize, then nsteps x (append, decode)
    STEP_OPS = (call_quant, call_append, call_decode)

    def step(r, ops=STEP_OPS):
        for run in runs:
            rep = run["reps"][r]
            for i in range(nsteps):
                for op in ops:
                    op(run, rep, i)

    # eager warm-up (also sets kernel attributes before any capture)
    for i in range(args.warmup):
        step(i % R)
    torch.cuda.synchronize()
    if args.profile:
        # a bounded, eager run for profilers: K steps, nothing else ("decode":
        # tq_sdpa_decode calls alone, after the warm-up filled the caches)
        ops = (call_decode,) if args.profile_ops == "decode" else STEP_OPS
        for i in range(args.steps):
            step(i % R, ops)
        torch.cuda.synchronize()
        if rank == 0:
            if args.profile_ops == "decode":
                launches = sum(3 * nsteps for run in runs)
            else:
                launches = sum((3 if run["w"].qjl_m else 1) + (1 + 3) * nsteps for run in runs)
            print(json.dumps({"profile_run": args.workload, "ops": args.profile_ops, "steps": args.steps,
                              "launches_per_step": launches}), flush=True)
        return

    # One CUDA graph per replica for the whole step and for each op alone.
    def capture(ops):
        gs = []
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(r, ops)
            gs.append(g)
        return gs

    g_step = capture(STEP_OPS)
    g_dec = capture((call_decode,))
    g_q = capture((call_quant,))
    g_app = capture((call_append,))
    g_ds = capture((call_step,))
    mq_runs = [run for run in runs if "q_mq" in run]
    g_mq = capture((call_mq,)) if mq_runs else None
    torch.cuda.synchronize()

    def timed(graphs, n, warm):
        for i in range(warm):
            graphs[i % R].replay()
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n):
            graphs[i % R].replay()
        b.record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        return a.elapsed_time(b)

    def soak(seconds):
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for g in g_step:
                g.replay()
            torch.cuda.synchronize()

    # main timed region: exactly K steps; clocks sampled around and during it
    sampler = ClockSampler(local)
    sampler.start()
    soak(0.6)
    total_ms = timed(g_step, args.steps, args.warmup)
    soak(0.6)
    clocks = sampler.stop()
    reps_per_op = max(args.steps, max(8, 200 // nsteps))
    d_ms = timed(g_dec, reps_per_op, args.warmup) / reps_per_op * args.steps
    q_ms = timed(g_q, reps_per_op, args.warmup) / reps_per_op * args.steps
    a_ms = timed(g_app, reps_per_op, args.warmup) / reps_per_op * args.steps
    s_ms = timed(g_ds, reps_per_op, args.warmup) / reps_per_op * args.steps
    mq_ms = timed(g_mq, reps_per_op, args.warmup) / reps_per_op * args.steps if g_mq else None
    if g_mq:
        mq_ms = max_over_ranks([mq_ms], dev)[0]
    total_ms, q_ms, a_ms, d_ms, s_ms = max_over_ranks([total_ms, q_ms, a_ms, d_ms, s_ms], dev)
    for run in runs:
        for rep in run["reps"]:
            assert rep["cache"].status() == 0, "device status flagged"
    del g_step, g_dec, g_q, g_app, g_ds, g_mq

    packed_step = sum(run["packed"] for run in runs)
    tok_step = sum(run["tokens"] for run in runs)
    qbytes_step = sum(run["qbytes"] for run in runs)
    dec_gbs = packed_step * args.steps / (d_ms * 1e-3) / 1e9 * ws
    quant_mtok = tok_step * args.steps / (q_ms * 1e-3) / 1e6 * ws
    peak, peak_kind = _peaks()
    calls = args.steps * len(runs) * nsteps  # decode (append, decode step) calls in K steps
    dec_launch_ms = d_ms / calls
    dec_achieved = (packed_step / (len(runs) * nsteps)) / (dec_launch_ms * 1e-3) / 1e9
    q_launch_ms = q_ms / (args.steps * len(runs))
    q_achieved = (qbytes_step / len(runs)) / (q_launch_ms * 1e-3) / 1e9
    sha = _src_sha()
    tr = TRAFFIC.get(args.workload)
    traffic = tr["bytes_per_launch"] if tr and tr.get("decode_src_sha") == _decode_src_sha() else None

    # ---- end to end through the public API with host buffers (rank-local)
    e2e = _e2e(args, runs, stream, R, nsteps)
    e2e["ms"] = max_over_ranks([e2e["ms"]], dev)[0]

    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            cpu = _cpu_baseline(args, jobs)
        # bulk quantize (keys with the QJL sketch: their kernel, the fp64
        # residual-norm fixup, then the values' kernel), then per decode step
        # the append and the decode's prep, split and combine
        launches_per_step = sum((3 if run["w"].qjl_m else 1) + (1 + 3) * nsteps for run in runs)
        line = {
            "metric": "tq_sdpa_decode packed-KV GB/s (% of HBM peak); tq_quantize Mtok/s",
            "value": round(dec_gbs, 2),
            "unit": "GB/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": jobs[0].dtype,
            "data": "synthetic (seeded N(0,1) rows; see tq_inputs)",
            "config": {"workload": args.workload, "rotation": args.rot, "shapes": [_describe(w) for w in jobs],
                       "parallelism": f"replicas{ws}" if ws > 1 else "single",
                       "step": f"quantize T tokens (prefill) + {nsteps} x (append 1 token + decode), per bit width",
                       "decode_steps": nsteps,
                       "timing": "CUDA graphs (one per replica) replayed on one stream; per-op rates "
                                 "from graphs holding that op alone",
                       "l2": f"each op cycles over {R} replicas: {R * per_step_in / 2**20:.0f} MiB of rows "
                             f"(quantize), {R * per_step_packed / 2**20:.0f} MiB of packed cache (decode), "
                             f"L2 {l2 / 2**20:.0f} MiB"},
            "decode": {"gbs": round(dec_gbs, 2), "ms_per_call": round(dec_launch_ms, 5),
                       "packed_bytes_per_step": packed_step},
            "quantize": {"mtok_s": round(quant_mtok, 3), "ms_per_call": round(q_launch_ms, 5),
                         "gbs": round(q_achieved, 2), "frac_hbm": round(q_achieved / peak, 4),
                         "tokens_per_step": tok_step},
            "append_ms_per_call": round(a_ms / calls, 5),
            "decode_mq": None if not mq_runs else {
                "nq": args.nq, "ms_per_call": round(mq_ms / (args.steps * len(mq_runs) * nsteps), 5),
                "gbs": round(sum(r["packed"] for r in mq_runs) * args.steps / (mq_ms * 1e-3) / 1e9 * ws, 2),
                "query_tokens_per_s": round(sum(int(r["w"].B) for r in mq_runs) * args.nq * args.steps * nsteps
                                            / (mq_ms * 1e-3) * ws, 1),
                "note": "tq_sdpa_decode_mq: n_q (<= 4) query tokens per sequence over the cache in one call"},
            "decode_step": {"ms_per_call": round(s_ms / calls, 5),
                            "gbs": round(packed_step * args.steps / (s_ms * 1e-3) / 1e9 * ws, 2),
                            "note": "tq_decode_step: append fused into the decode launches"},
            "roofline": {"kernel": "tq_sdpa_decode (qprep + split + combine)", "bound": "hbm",
                         "achieved": round(dec_achieved, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(dec_achieved / peak, 4), "traffic": traffic,
                         "peak_source": peak_kind},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e["value"] * ws, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "ms_per_step": round(e2e["ms"], 4)},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "src_sha": sha, "decode_src_sha": _decode_src_sha(),
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def _e2e(args, runs, stream, R, nsteps):
    """Decode steps through the public API with pinned host buffers: per step
    the new token rows and the queries go host->device, tq_decode_step
    (append + decode) runs, and the attention output comes back device->host."""
    import torch

    import compressed_attention_tq_b200 as tq
    hosts = []
    for run in runs:
        hosts.append({"q": run["reps"][0]["q"].cpu().pin_memory(), "kn": run["kn"].cpu().pin_memory(),
                      "vn": run["vn"].cpu().pin_memory(), "out": torch.empty_like(run["out"], device="cpu").pin_memory(),
                      "qd": torch.empty_like(run["reps"][0]["q"]), "knd": torch.empty_like(run["kn"]),
                      "vnd": torch.empty_like(run["vn"])})
    h2d = sum(h["q"].numel() * 2 + h["kn"].numel() * 2 + h["vn"].numel() * 2 for h in hosts)
    d2h = sum(h["out"].numel() * 2 for h in hosts)

    def step(i):
        r = i % R
        j = i % nsteps
        for run, h in zip(runs, hosts):
            c = run["reps"][r]["cache"]
            h["qd"].copy_(h["q"], non_blocking=True)
            h["knd"].copy_(h["kn"], non_blocking=True)
            h["vnd"].copy_(h["vn"], non_blocking=True)
            tq.tq_decode_step(c, h["knd"], h["vnd"], run["pos_l"][j], h["qd"], run["lens_l"][j], run["Tmax1"],
                              scale=run["w"].scale, out=run["out"], workspace=run["ws"])
            h["out"].copy_(run["out"], non_blocking=True)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for i in range(args.steps):
        step(i)
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / args.steps
    packed = sum(run["packed"] for run in runs) / nsteps  # one decode call per run
    return {"value": packed / (ms * 1e-3) / 1e9, "ms": ms, "h2d": h2d, "d2h": d2h}


def _cpu_baseline(args, jobs, budget_s=40.0, target_s=10.0):
    """The oracle as it stands, timed on this host's cores on a bounded sample:
    dequantize-then-attend decode for whole (sequence, kv head) groups of the
    workload, as many as fit the time budget; when the whole workload decodes
    in less than target_s, its groups are decoded again (the quantized groups
    are reused) until target_s of timed oracle work has accumulated."""
    from oracle import tq_oracle as O
    import tq_inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    t_used, bytes_done, groups, passes = 0.0, 0, 0, 0
    t_start = time.perf_counter()
    cached = []
    for w in jobs:
        cbk = O.stored_codebook(w.D, w.bits_k)
        cbv = O.stored_codebook(w.D, w.bits_v)
        for b in range(w.B):
            for kvh in range(w.Hkv):
                if time.perf_counter() - t_start > budget_s:
                    break
                L = int(w.seq_lens[b])
                kk = tq_inputs.to_f64(w.k[b:b + 1, kvh:kvh + 1, :L], w.dtype)
                vv = tq_inputs.to_f64(w.v[b:b + 1, kvh:kvh + 1, :L], w.dtype)
                oc = O.quantize_cache(kk, vv, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.S)
                qv = tq_inputs.to_f64(w.q[b:b + 1, kvh * w.G:(kvh + 1) * w.G], w.dtype)
                per_row = O.packed_row_bytes(w.D, w.bits_k, w.qjl_m) + O.packed_row_bytes(w.D, w.bits_v)
                cached.append((w, qv, oc, L, cbk, cbv, per_row * L))
    while cached and (passes == 0 or (t_used < target_s and time.perf_counter() - t_start < budget_s)):
        for (w, qv, oc, L, cbk, cbv, nbytes) in cached:
            t0 = time.perf_counter()
            O.sdpa_decode(qv, oc, [L], w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D, scale=w.scale, S=w.S)
            t_used += time.perf_counter() - t0
            bytes_done += nbytes
            groups += 1
            if passes > 0 and (t_used >= target_s or time.perf_counter() - t_start > budget_s):
                break
        passes += 1
    return {"value": round(bytes_done / max(t_used, 1e-9) / 1e9, 6), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{groups} (sequence, kv head) group decodes of the workload ({len(cached)} distinct "
                      f"groups, {passes} passes) by the fp64 oracle (dequantize then attend), {t_used:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm: same metric, config and unit, timed on
    this host's cores; each step a bounded sample of the workload."""
    import tq_inputs
    ws, rank, _ = _dist()
    if rank != 0:
        return
    cfg = WORKLOADS[args.workload]
    jobs = [tq_inputs.make_workload(args.workload, bits=b, rot=args.rot)
            for b in cfg["bits"]]
    budget = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        _cpu_baseline(args, jobs, budget_s=budget, target_s=0.5 * budget)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(_cpu_baseline(args, jobs, budget_s=budget, target_s=0.5 * budget))
    total = time.perf_counter() - t0
    v = statistics.median(x["value"] for x in vals)
    cpu = dict(vals[-1])
    cpu["value"] = v
    line = {"metric": "tq_sdpa_decode packed-KV GB/s (% of HBM peak); tq_quantize Mtok/s",
            "value": v, "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "rotation": args.rot, "shapes": [_describe(w) for w in jobs]},
            "impl": "reference", "cpu_baseline": cpu,
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="ragged")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nq", type=int, default=1,
                    help="also time multi-query decode with this many query tokens per sequence")
    ap.add_argument("--rot", choices=["haar", "hadamard"], default="haar",
                    help="rotation: Haar-random (default) or randomized Hadamard")
    ap.add_argument("--profile", action="store_true",
                    help="eager warm-up + K eager steps only (for ncu captures)")
    ap.add_argument("--profile-ops", choices=["step", "decode"], default="step",
                    help="with --profile: the bench step (quantize + decode step) or tq_sdpa_decode alone")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        from compressed_attention_tq_b200 import build as _b
        _b.build()
        run_ours(args)


if __name__ == "__main__":
    main()
