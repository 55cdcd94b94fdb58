#!/usr/bin/env python
"""Benchmark of the rolling-KV-cache attention hot path on B200.

One step = one whole stream of the 512p-shaped workload (B=1, H=24, D=128,
32x32-token frames, chunk 2 frames, sink 1 frame, window 4 frames, 64 chunks,
RoPE refresh every 32 chunks) from an empty cache: per chunk the fused
RoPE + append kernel and the tcgen05 attention kernel, plus the refresh.
Inputs for every chunk of the step are resident in HBM before timing (2.4 GB
per step, larger than the 126 MB L2, so every step starts cold).

Prints one JSON line (rank 0). Under torchrun each rank streams its own
independent streams (weak scaling, no collective on the data path); the
timed region is bracketed by a barrier and synchronisation and the time is
the max over ranks.

--impl reference times the fp64 CPU oracle (the reference implementation of
this repository) on the host cores, on a bounded sample of the same workload.

--path gdn measures the Gated DeltaNet block (sa_gdn_chunk) on the same
stream shape instead: one step = 64 calls of 2,048 tokens from a zero state;
its roofline is the fp32 FMA peak of the CUDA cores it runs on.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "streamed chunks/s and attention TFLOP/s (% of B200 BF16 peak) per config"

# DRAM bytes (read + write) per launch of the attention kernel, from the ncu
# capture summarised in profiles/ (512p, steady chunk with 7168 keys), keyed by
# a hash of the kernel sources it was taken on: a changed kernel reports null.
PROFILED_TRAFFIC = {"c8df9477bcca4326": 173.17e6, "c8df9477bcca4326/e4m3": 61.97e6}


def attend_source_hash() -> str:
    import hashlib
    h = hashlib.sha1()
    for f in ("attend_tc.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "rolling_kv_cache_sa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="512p_32x32_h24",
                    help="workload name, or C1..C5 for the five configurations in order")
    ap.add_argument("--cache", default="", choices=["", "e4m3"],
                    help="e4m3: bf16 in/out with an e4m3 K'/V cache and fp8 attention MMAs")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--eager", action="store_true", help="time eager launches, no CUDA graph")
    ap.add_argument("--chunks", type=int, default=0,
                    help="stream only this many chunks per stream (small profiling cases)")
    ap.add_argument("--path", default="attention", choices=["attention", "gdn"],
                    help="gdn: the Gated DeltaNet block (sa_gdn_chunk) on the same streams")
    ap.add_argument("--gdn-g-scale", type=float, default=0.002,
                    help="gdn: per-token log decay drawn in (-g_scale, 0)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(m["bf16_tflops_sustained"]), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"sa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        loaded = [r[0] for r in rows if r[2] > 300.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


def gpu_id_for(dev: int) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev] if vis else str(dev)


# ------------------------------------------------------------------ oracle timing
def oracle_sample(w, rank_stream: int = 0, budget_rows: int = 4096):
    """Times the fp64 oracle on one steady-state chunk: key build plus
    `budget_rows` output rows, extrapolated linearly to a whole chunk."""
    import numpy as np

    import oracle as O
    from inputgen import spec_for
    cfg = O.cfg_for(w)
    spec = spec_for(w)
    c = min(w.n_chunks - 1, max(3, w.refresh_period + 8 if w.refresh_period else 40))
    t0 = time.perf_counter()
    O.attend_rows(cfg, spec, rank_stream, c, np.zeros(0, np.int32), np.zeros(0, np.int32))
    t_fixed = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    n = min(budget_rows, w.Lc * w.H)
    toks = rng.integers(0, w.Lc, n).astype(np.int32)
    heads = rng.integers(0, w.H, n).astype(np.int32)
    t0 = time.perf_counter()
    O.attend_rows(cfg, spec, rank_stream, c, toks, heads)
    t_rows = time.perf_counter() - t0
    per_row = max(t_rows - t_fixed, 1e-9) / n
    per_chunk = t_fixed + per_row * w.Lc * w.H
    return {"value": 1.0 / per_chunk, "unit": "chunks/s", "cores": O.num_threads(),
            "kind": "oracle",
            "sample": f"{w.name} chunk {c}: visible-key build + {n} of {w.Lc * w.H} (token, head) "
                      f"output rows in fp64, extrapolated linearly to the whole chunk "
                      f"({t_fixed + t_rows:.1f} s of CPU time)"}


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    # each step is a bounded sample (fewer rows) so the whole run stays short
    per = []
    for i in range(warm + steps):
        r = oracle_sample(w, budget_rows=512)
        if i >= warm:
            per.append(1.0 / r["value"])
    ms_step = 1000.0 * w.n_chunks * w.B * statistics.mean(per)
    value = w.n_chunks * w.B / (ms_step / 1000.0)
    line = {"metric": METRIC, "value": value, "unit": "chunks/s", "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": config_json(w, world),
            "cpu_baseline": {"value": value, "unit": "chunks/s", "cores": r["cores"],
                             "kind": "oracle", "sample": r["sample"].replace("4096", "512")},
            "e2e": {"value": value, "unit": "chunks/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_json(w, world):
    return {"workload": w.name, "streams_per_gpu": w.B, "heads": w.H, "head_dim": w.D,
            "frame": f"{w.fh}x{w.fw}", "chunk_frames": w.C, "sink_frames": w.S,
            "window_frames": w.W, "chunks_per_stream": w.n_chunks,
            "refresh_every": w.refresh_period, "rope_dims": list(w.dims),
            "cache": "e4m3 (per-head scales 1)" if w.cache == "e4m3" else w.dtype,
            "parallelism": f"independent streams per GPU x{world} (no collective)",
            "l2": "inputs larger than L2 (every chunk of the step resident, "
                  f"{3 * w.n_chunks * w.B * w.Lc * w.H * w.D * (2 if w.dtype == 'bf16' else 4) / 1e9:.1f}"
                  " GB per step)"}


# ------------------------------------------------------------------ GDN block
GDN_METRIC = "GDN block: streamed chunks/s (gated delta rule state update + outputs)"
FP32_LANES_PER_SM, SM_COUNT, SM_MAX_GHZ = 128, 148, 1.965


def gdn_flops_per_token(D: int, ct: int = 64) -> float:
    """Algorithmic FLOPs per token and head of the chunkwise gated delta rule
    on sub-chunks of ct tokens: K S0^T, Q S0^T and the state update (2 D^2
    each), the two lower-triangular Gram matrices and the two triangular
    products with D columns (ct + 1) D each, and the triangular inverse
    (ct^2 / 3). Counted once per head (the kernel's per-slice recomputation
    is not algorithmic work)."""
    return 6.0 * D * D + 4.0 * (ct + 1) * D + ct * ct / 3.0


def gdn_oracle_sample(w, g_scale: float, n_tok: int = 256):
    import numpy as np

    import oracle as O
    q, k, v, g, beta = O.gdn_inputs(w, 0, 0, g_scale)
    st = np.zeros((w.H, w.D, w.D))
    t0 = time.perf_counter()
    O.gdn_chunk(1.0 / np.sqrt(w.D), st, q[:n_tok], k[:n_tok], v[:n_tok], g[:n_tok], beta[:n_tok])
    dt = time.perf_counter() - t0
    per_chunk = dt * w.Lc / n_tok
    return {"value": 1.0 / per_chunk, "unit": "chunks/s", "cores": O.num_threads(),
            "kind": "oracle",
            "sample": f"{w.name}: the first {n_tok} of {w.Lc} tokens of one chunk, all {w.H} heads "
                      f"(fp64 token-by-token recurrence, heads across threads), extrapolated "
                      f"linearly to the chunk ({dt:.2f} s of CPU time)"}


def gdn_config_json(w, world, g_scale):
    return {"workload": w.name + "_gdn", "streams_per_gpu": w.B, "heads": w.H, "head_dim": w.D,
            "tokens_per_chunk": w.Lc, "chunks_per_stream": w.n_chunks,
            "g_scale": g_scale, "dtype_io": w.dtype, "state": "fp32 [B][H][D][D]",
            "parallelism": f"independent streams per GPU x{world} (no collective)",
            "l2": "inputs larger than L2 (every chunk of the step resident, "
                  f"{3 * w.n_chunks * w.B * w.Lc * w.H * w.D * (2 if w.dtype == 'bf16' else 4) / 1e9:.1f}"
                  " GB per step)"}


def run_gdn(args, w, rank, world):
    g_scale = args.gdn_g_scale
    if args.impl == "reference":
        if rank != 0:
            return
        per = []
        for i in range(args.warmup + args.steps):
            r = gdn_oracle_sample(w, g_scale, n_tok=64)
            if i >= args.warmup:
                per.append(1.0 / r["value"])
        ms_step = 1000.0 * w.n_chunks * w.B * statistics.mean(per)
        value = w.n_chunks * w.B / (ms_step / 1000.0)
        print(json.dumps({
            "metric": GDN_METRIC, "value": value, "unit": "chunks/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": gdn_config_json(w, world, g_scale),
            "cpu_baseline": {"value": value, "unit": "chunks/s", "cores": r["cores"],
                             "kind": "oracle", "sample": r["sample"]},
            "e2e": {"value": value, "unit": "chunks/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return

    import numpy as np
    import torch
    import torch.distributed as dist

    import inputgen as IG
    from rolling_kv_cache_sa_b200 import gdn_workspace, sa_gdn_chunk
    from rolling_kv_cache_sa_b200.dist import aggregate_rate, max_over_ranks, rank_stream_ids

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    esz = 2 if w.dtype == "bf16" else 4
    nC, B = w.n_chunks, w.B
    shape = (nC, B, w.Lc, w.H, w.D)
    q_all = torch.empty(shape, dtype=dt, device="cuda")
    k_all, v_all, out_all = torch.empty_like(q_all), torch.empty_like(q_all), torch.empty_like(q_all)
    g_all = torch.empty((nC, B, w.Lc, w.H), dtype=torch.float32, device="cuda")
    b_all = torch.empty_like(g_all)
    st = torch.cuda.current_stream().cuda_stream
    sids = rank_stream_ids(rank, B)
    for c in range(nC):
        for t, buf in ((IG.Q, q_all), (IG.K, k_all), (IG.V, v_all)):
            IG.fill_device(w, sids, [c] * B, t, buf[c].data_ptr(), st)
        for bi, sid in enumerate(sids):
            g, beta = IG.fill_gates_host(w, sid, c, g_scale)
            g_all[c, bi].copy_(torch.from_numpy(g))
            b_all[c, bi].copy_(torch.from_numpy(beta))
    state = torch.zeros(B, w.H, w.D, w.D, dtype=torch.float32, device="cuda")
    wsp = gdn_workspace(B, w.Lc, w.H, w.D)
    torch.cuda.synchronize()

    def run_step():
        state.zero_()
        for c in range(nC):
            sa_gdn_chunk(state, q_all[c], k_all[c], v_all[c], g_all[c], b_all[c], out_all[c],
                         workspace=wsp)

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()

    def timed(fn, steps):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        e1.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), "cuda")

    sampler = ClockSampler(gpu_id_for(local)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    # eager pass: CUDA events around every launch on the launch stream
    eager_steps = max(1, min(args.steps, 10))
    launch_ms = []
    torch.cuda.synchronize()
    for _ in range(eager_steps):
        state.zero_()
        evs = []
        for c in range(nC):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sa_gdn_chunk(state, q_all[c], k_all[c], v_all[c], g_all[c], b_all[c], out_all[c],
                         workspace=wsp)
            e1.record()
            evs.append((e0, e1))
        torch.cuda.synchronize()
        launch_ms += [a.elapsed_time(b) for a, b in evs]
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        run_step()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        graph.replay()
    ms = timed(graph.replay, args.steps)
    clocks = sampler.stop() if sampler else None
    ms_step = ms / args.steps
    chunks_per_step = nC * B
    value = aggregate_rate(chunks_per_step * args.steps, world, ms)

    flops_per_launch = gdn_flops_per_token(w.D) * w.Lc * w.H * B
    avg_launch_s = statistics.mean(launch_ms) / 1000.0
    achieved = flops_per_launch / avg_launch_s / 1e12
    peak = FP32_LANES_PER_SM * SM_COUNT * 2 * SM_MAX_GHZ / 1e3
    bytes_per_launch = B * (w.Lc * w.H * w.D * esz * 4 + w.Lc * w.H * 8 + 2 * w.H * w.D * w.D * 4)
    # (the workspace of T and P, 32 KiB per 64 tokens and head, is written and
    # read back through L2 and is not algorithmic traffic)
    hbm = peaks()[0]

    # end to end through the public call: pinned host inputs copied in and
    # outputs copied out every chunk, inside the timed region
    qh = torch.empty(q_all.shape, dtype=dt, pin_memory=True)
    kh, vh, oh = (torch.empty_like(qh, pin_memory=True) for _ in range(3))
    gh = torch.empty(g_all.shape, dtype=torch.float32, pin_memory=True)
    bh = torch.empty_like(gh, pin_memory=True)
    qh.copy_(q_all), kh.copy_(k_all), vh.copy_(v_all), gh.copy_(g_all), bh.copy_(b_all)
    dq, dk, dv, do = (torch.empty_like(q_all[0]) for _ in range(4))
    dg, db = torch.empty_like(g_all[0]), torch.empty_like(b_all[0])

    def run_step_host():
        state.zero_()
        for c in range(nC):
            dq.copy_(qh[c], non_blocking=True)
            dk.copy_(kh[c], non_blocking=True)
            dv.copy_(vh[c], non_blocking=True)
            dg.copy_(gh[c], non_blocking=True)
            db.copy_(bh[c], non_blocking=True)
            sa_gdn_chunk(state, dq, dk, dv, dg, db, do, workspace=wsp)
            oh[c].copy_(do, non_blocking=True)

    run_step_host()
    e2e_steps = max(1, args.e2e_steps)
    ems = timed(lambda: run_step_host(), e2e_steps)
    e2e = {"value": aggregate_rate(chunks_per_step * e2e_steps, world, ems), "unit": "chunks/s",
           "steps": e2e_steps,
           "h2d_bytes_per_step": chunks_per_step * (3 * w.Lc * w.H * w.D * esz + 2 * w.Lc * w.H * 4),
           "d2h_bytes_per_step": chunks_per_step * w.Lc * w.H * w.D * esz,
           "api": "sa_gdn_chunk with every chunk's inputs copied from pinned host memory and its "
                  "output copied back, in stream order, inside the timed region"}
    cpu = gdn_oracle_sample(w, g_scale) if (rank == 0 and world == 1 and
                                            not args.no_cpu_baseline) else None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": GDN_METRIC, "value": value, "unit": "chunks/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded counter generator; Irwin-Hall N(0,1) q, k, v; uniform gates)",
        "config": gdn_config_json(w, world, g_scale),
        "ms_per_chunk": ms_step / chunks_per_step,
        "launch_mode": "cuda graph of one step, replayed",
        "roofline": {"bound": "alu",
                     "kernel": f"gdn_prep_kernel<{w.D}> + gdn_chunk_kernel<{w.D}> (one call)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP (FMA) x 1.965 GHz",
                     "algorithmic_flops_per_launch": flops_per_launch,
                     "hbm_bytes_per_launch": bytes_per_launch,
                     "hbm_frac": bytes_per_launch / avg_launch_s / 1e9 / hbm,
                     "duration": "mean of CUDA events around each call (its two launches) on "
                                 "the launch stream, eager pass", "traffic": None},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * nC * args.steps, "clocks": clocks,
        "call_ms": {"mean": statistics.mean(launch_ms),
                      "p50": float(np.percentile(launch_ms, 50)),
                      "p99": float(np.percentile(launch_ms, 99))},
    }), flush=True)


# ------------------------------------------------------------------ GPU arm
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from inputgen.workloads import ALL, BY_NAME
    # C1..C5: the five configurations in order (tiny fp32, 512p, 480x832 ragged,
    # 1280x704, long-stream stress)
    aliases = {f"C{i + 1}": wl.name for i, wl in enumerate(ALL)}
    w = BY_NAME[aliases.get(args.workload, args.workload)]
    if args.chunks:
        w = w.with_(n_chunks=args.chunks)
    if args.cache:
        w = w.with_(cache=args.cache)

    if args.path == "gdn":
        run_gdn(args, w, rank, world)
        return
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    import torch
    import torch.distributed as dist

    import inputgen as IG
    from rolling_kv_cache_sa_b200 import SACache, attention_flops, config_for, sa_plan_chunk
    from rolling_kv_cache_sa_b200.dist import aggregate_rate, max_over_ranks, rank_stream_ids
    from rolling_kv_cache_sa_b200.session import StreamSession

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    cfg = config_for(w)
    cache = SACache(cfg)
    sess = StreamSession(cache, w.refresh_period)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    n_steps_g = w.n_steps
    shape = (n_steps_g, w.B, w.Lc, w.H, w.D)
    q_all = torch.empty(shape, dtype=dt, device="cuda")
    k_all = torch.empty_like(q_all)
    v_all = torch.empty_like(q_all)
    out_all = torch.empty_like(q_all)
    st = torch.cuda.current_stream().cuda_stream
    stream_ids = rank_stream_ids(rank, w.B)  # distinct streams per rank
    actives = []
    for g in range(n_steps_g):
        chunks = w.local_chunks(g)
        actives.append([c >= 0 for c in chunks])
        for t, buf in ((IG.Q, q_all), (IG.K, k_all), (IG.V, v_all)):
            IG.fill_device(w, stream_ids, chunks, t, buf[g].data_ptr(), st)
    torch.cuda.synchronize()

    chunks_per_step = sum(sum(a) for a in actives)
    # algorithmic attention FLOPs of one step: 4 * Lc * n_keys * D * H per stream-chunk
    step_flops = 0.0
    for c in range(w.n_chunks):
        step_flops += w.B * attention_flops(cfg, sa_plan_chunk(cfg, c * w.C, 0).n_keys)
    esz = 2 if w.dtype == "bf16" else 4
    cesz = 1 if w.cache == "e4m3" else esz  # cache element bytes
    append_bytes_per_chunk = 3 * w.Lc * w.H * w.D * (esz + cesz)  # read q,k,v; write q',k',v

    def run_step():
        cache.reset()
        for g in range(n_steps_g):
            sess.step(q_all[g], k_all[g], v_all[g], out_all[g], actives[g])

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    def timed(fn, steps):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        e1.synchronize()
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), "cuda")

    # eager: every library call issued from Python, one launch at a time; the
    # library's per-launch CUDA events (on the launch stream) time each kernel
    sampler = ClockSampler(gpu_id_for(local)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    eager_steps = args.steps if args.eager else max(1, min(args.steps, 20))
    cache.profile_begin()
    ms_eager = timed(run_step, eager_steps)
    launches_per_step = cache.profile_launches() / eager_steps
    prof = cache.profile_end()
    prof_steps = eager_steps

    # graph: one whole step captured once (every hot call of the library is
    # capturable: no synchronisation, parameters by value) and replayed with
    # profiling off, so the graph holds kernel nodes only
    graph = None
    if args.eager:
        ms = ms_eager
    else:
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            run_step()
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        ms = timed(graph.replay, args.steps)
    clocks = sampler.stop() if sampler else None
    launches = int(round(launches_per_step * args.steps))

    # per-call latency: two eager steps, CUDA events around each call (device
    # time of the call's kernels on the launch stream, refresh included when due)
    lat = []
    for _ in range(2):
        cache.reset()
        evs = []
        for g in range(n_steps_g):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sess.step(q_all[g], k_all[g], v_all[g], out_all[g], actives[g])
            e1.record()
            evs.append((e0, e1))
        torch.cuda.synchronize()
        lat += [a.elapsed_time(b) for a, b in evs]
    import numpy as np
    call_latency = {"p50_ms": float(np.percentile(lat, 50)), "p99_ms": float(np.percentile(lat, 99)),
                    "calls": len(lat),
                    "what": "device time per step call (append + attention, refresh when due), "
                            "eager, CUDA events on the launch stream"}
    ms_eager /= eager_steps
    cache.reset()
    ms_step = ms / args.steps
    value = aggregate_rate(chunks_per_step * args.steps, world, ms)

    hbm, pk_burst, pk_sust, pk_src = peaks()
    f8 = w.cache == "e4m3"
    if f8:  # fp8 contraction: the measured bf16 peaks x the nominal 2x (4.5 / 2.25 PFLOP/s)
        pk_burst, pk_sust = 2.0 * pk_burst, 2.0 * pk_sust
    att_ms, att_n = prof["attend"]
    app_ms, app_n = prof["append"]
    ref_ms, ref_n = prof["refresh"]
    att_flops_per_launch = step_flops * prof_steps / max(att_n, 1)
    att_avg_s = att_ms / 1000.0 / max(att_n, 1)
    achieved = att_flops_per_launch / att_avg_s / 1e12
    # append bytes: every active (stream, chunk) of the profiled steps
    append_gbs = (append_bytes_per_chunk * chunks_per_step * prof_steps / (app_ms / 1000.0) / 1e9
                  if app_n and app_ms > 0 else None)

    e2e = None
    if not args.no_e2e:
        qh = torch.empty(q_all.shape, dtype=dt, pin_memory=True)
        kh = torch.empty_like(qh, pin_memory=True)
        vh = torch.empty_like(qh, pin_memory=True)
        oh = torch.empty_like(qh, pin_memory=True)
        qh.copy_(q_all)
        kh.copy_(k_all)
        vh.copy_(v_all)

        def run_step_host():
            # every call is queued: copies of one chunk overlap the compute of
            # another in the library's pipeline; waited for at the end
            cache.reset()
            for g in range(n_steps_g):
                sess.step_host_async(qh[g], kh[g], vh[g], oh[g], actives[g])

        run_step_host()
        cache.host_wait()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.e2e_steps):
            run_step_host()
        cache.host_wait()  # the last copy-out has landed before the closing event
        e1.record()
        e1.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), "cuda")
        per_chunk_in = 3 * w.Lc * w.H * w.D * esz
        e2e = {"value": aggregate_rate(chunks_per_step * args.e2e_steps, world, ems),
               "unit": "chunks/s", "steps": args.e2e_steps,
               "h2d_bytes_per_step": per_chunk_in * chunks_per_step,
               "d2h_bytes_per_step": w.Lc * w.H * w.D * esz * chunks_per_step,
               "api": "sa_append_attend_host_async (pinned host buffers; the copy-in, "
                      "compute and copy-out of consecutive chunks overlap; every copy is "
                      "inside the timed region)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(w)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        cache.close()
        return
    att_tflops_step = step_flops / (ms_step / 1000.0) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "chunks/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if f8 else "bf16",
        "data": "synthetic (seeded counter generator; Irwin-Hall N(0,1) inputs)",
        "config": config_json(w, world),
        "ms_per_chunk": ms_step / chunks_per_step,
        "attention_tflops_whole_step": att_tflops_step,
        "attention_frac_of_peak_whole_step": att_tflops_step / pk_sust,
        "append_gbs": append_gbs,
        "append_frac_of_hbm": (append_gbs / hbm) if append_gbs else None,
        "kernel_ms_per_step": {"attend": att_ms / prof_steps, "append": app_ms / prof_steps,
                               "refresh": ref_ms / prof_steps},
        "call_latency": call_latency,
        "launch_mode": "cuda graph of one step, replayed" if graph is not None else "eager",
        "eager_chunks_per_s": chunks_per_step * world / (ms_eager / 1000.0),
        "eager_ms_per_step": ms_eager,
        # the kernel is timed inside long back-to-back stepping (the eager
        # pass and the replays run continuously under the power cap), so the
        # denominator is the sustained bf16 figure; the burst one is kept too
        "roofline": {"bound": "tensor",
                     "kernel": "attend_tc_kernel<128, e4m3>" if f8 else "attend_tc_kernel<128>",
                     "achieved": achieved, "peak": pk_sust, "unit": "TFLOP/s",
                     "frac": achieved / pk_sust,
                     "peak_source": (f"{pk_src} bf16 sustained x 2 (fp8 nominal ratio)" if f8 else
                                     f"{pk_src} bf16 sustained (timed inside long stepping)"),
                     "frac_of_burst": achieved / pk_burst,
                     "duration": "mean of the library's CUDA events around each launch, on "
                                 "its launch stream, over the eager timed pass",
                     "traffic": PROFILED_TRAFFIC.get(attend_source_hash() + ("/e4m3" if f8 else "")),
                     "traffic_note": ("ncu dram read+write bytes of one steady-state launch "
                                      "(7168 keys, cold L2); algorithmic minimum 63 MB (e4m3 "
                                      "Q', K', V in, bf16 O out)") if f8 else
                                     ("ncu dram read+write bytes of one steady-state launch "
                                      "(7168 keys, cold L2); algorithmic minimum 113 MB; the "
                                      "excess is split-unit fp32 partials written and read "
                                      "back and K/V re-reads past L2")},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    cache.close()


if __name__ == "__main__":
    main()
