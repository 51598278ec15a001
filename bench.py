"""Benchmark of the observation-window KV-compression hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole path over one batch of seeded synthetic input
(Llama-3-8B-shaped layer: n_h 32, n_kv 8, d_h 128, bf16, S 32768, window 32,
pool 7, budget 2048, 1% of keys boosted): kvc_compress_window (score, select
and gather of one sequence in one call), then kvc_gqa_decode_attn for a batch
of 16 compact caches (cache 0 is the one the step's gather writes; caches
1..15 are seeded stand-ins of the same shape).

value = K tokens/s of score + select + gather (S / time / 1e3), whole job over
all ranks; decode GB/s and the per-call breakdown (including the three
separate calls kvc_score_window, kvc_select_topk, kvc_gather_kv) are extra
keys.  Each call is captured once in a CUDA graph and replayed, so the timed
region holds device work only; ssg_us_stats adds an uncaptured timing, and
the e2e leg calls the C ABI directly with host buffers.  Timing: CUDA events
around every step on the launching stream, L2 flushed (256 MiB write, then a
256 MiB read sweep so no dirty lines are left) between steps outside the
events, max over ranks.  With N > 1 every rank runs its own sequences (weak
scaling, no collective on the data path).

--impl reference runs the fp64 CPU oracle on the same workload and metric
(rank 0 only; the pages ship no code, so the oracle is the reference arm).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LLAMA3_8B_S32K = dict(name="llama3-8b-layer-S32768-B2048", n_h=32, n_kv=8, d_h=128, S=32768, w=32, pool_k=7, budget=2048,
               decode_batch=16, boost_frac=0.01, boost=3.0, seed=1002, dtype="bf16")
METRIC = "score+select+gather K-tok/s & GB/s at S=32K; decode-attn GB/s vs 8 TB/s HBM"
FALLBACK_HBM_GBS = 6650.0


def env_rank():
    from kv_cache_compression_score_b200.dist import rank_info
    return rank_info()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(cfg):
    """Bytes the path must move: K read once by scoring; retained K/V rows read
    and written by the gather; every retained K/V row read by decode."""
    esz = 2 if cfg["dtype"] == "bf16" else 4
    row = cfg["n_kv"] * cfg["d_h"] * esz
    score = cfg["S"] * row
    gather = 2 * 2 * cfg["budget"] * row
    decode = 2 * cfg["decode_batch"] * cfg["budget"] * row
    return score, gather, decode


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9 and parts[1].isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [int(r[1]) for r in rows]
        mx = int(rows[0][2])
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": int(statistics.median(loaded)), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, local_rank, world = env_rank()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)

    from kv_cache_compression_score_b200 import build as kbuild
    if rank == 0 or world == 1:
        kbuild.build()
    if world > 1:
        dist.barrier()
    from kv_cache_compression_score_b200 import synth
    from kv_cache_compression_score_b200.dist import max_over_ranks, rank_seed
    from kv_cache_compression_score_b200.runner import Compressor, Decoder, to_device

    cfg = dict(LLAMA3_8B_S32K)
    seed = rank_seed(cfg["seed"], rank)
    S, n_h, n_kv, d, w, B, nb = cfg["S"], cfg["n_h"], cfg["n_kv"], cfg["d_h"], cfg["w"], cfg["budget"], \
        cfg["decode_batch"]
    bt = synth.packed_batch(seed, [S], n_h, n_kv, d, w, cfg["dtype"], cfg["boost_frac"], cfg["boost"])
    q_win, k, v = (to_device(bt[x], cfg["dtype"], dev) for x in ("q_win", "k", "v"))
    comp = Compressor(cfg["dtype"], [S], n_h, n_kv, d, w, cfg["pool_k"], B, device=dev, keep_raw=False)
    # 16 compact caches in one buffer; slot 0 is written by the step's gather
    kc_all = torch.empty((nb * B, n_kv, d), dtype=torch.bfloat16, device=dev)
    vc_all = torch.empty_like(kc_all)
    for b in range(1, nb):
        kk, vv = synth.keys_values(seed + 7, b, B, n_kv, d, cfg["dtype"])
        kc_all[b * B:(b + 1) * B].copy_(to_device(kk, cfg["dtype"], dev))
        vc_all[b * B:(b + 1) * B].copy_(to_device(vv, cfg["dtype"], dev))
    comp.buf.k_c = kc_all[:B]
    comp.buf.v_c = vc_all[:B]
    qd = to_device(synth.decode_queries(seed + 8, nb, n_h, d, cfg["dtype"]), cfg["dtype"], dev)
    off = torch.arange(nb, dtype=torch.int64, device=dev) * B
    ln = torch.full((nb,), B, dtype=torch.int32, device=dev)
    dec = Decoder(nb, n_h, n_kv, d, B, device=dev)
    # L2 flush between steps: write 256 MiB (> 2x L2), then read another
    # 256 MiB so the timed step starts from a cache holding none of its data and
    # no dirty lines waiting to be written back
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sweep = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        torch.sum(sweep, dim=0, out=sink)

    stream = torch.cuda.current_stream(dev)
    from kv_cache_compression_score_b200 import kvc
    hbm, peak_kind = measured_peaks()

    # the C-ABI calls of a step: score -> select -> gather captured as one CUDA
    # graph (the headline), decode as a second; each call also gets a graph of
    # its own for the per-call breakdown.  Graphs keep Python/ctypes enqueue
    # time out of the timed region.
    calls = [lambda: comp.score(q_win, k), lambda: comp.select(), lambda: comp.gather(k, v),
             lambda: dec.run(qd, kc_all, vc_all, off, ln), lambda: comp.compress(q_win, k, v)]
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for fn in calls:
            fn()
    stream.wait_stream(side)
    torch.cuda.synchronize()

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        n0 = kvc.kvc_launch_count()
        with torch.cuda.graph(g):
            for fn in fns:
                fn()
        return g, kvc.kvc_launch_count() - n0

    g_ssg, n_ssg = capture(calls[4:5])          # kvc_compress_window: score + select + gather in one call
    g_dec, n_dec = capture(calls[3:4])
    per_call = [capture([fn])[0] for fn in calls]
    torch.cuda.synchronize()
    kernels_per_step = n_ssg + n_dec

    for _ in range(args.warmup):
        flush_l2()
        g_ssg.replay()
        g_dec.replay()
    torch.cuda.synchronize()
    assert comp.device_error_word() == 0, "device error word set"

    sampler = ClockSampler(local_rank)
    sampler.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush_l2()
        evs[i][0].record(stream)
        g_ssg.replay()
        evs[i][1].record(stream)
        g_dec.replay()
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall = time.perf_counter() - t_wall
    clocks = sampler.stop()
    assert comp.device_error_word() == 0, "device error word set"

    ssg_samples = [evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps)]   # ms
    t_ssg = float(np.mean(ssg_samples))
    t_dec = float(np.mean([evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps)]))
    t_step = t_ssg + t_dec

    # the same call without graph capture (a direct C-ABI call, device-resident inputs)
    uevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2()
        uevs[i][0].record(stream)
        calls[4]()
        uevs[i][1].record(stream)
    torch.cuda.synchronize()
    t_ssg_direct = float(np.mean([a.elapsed_time(b) for a, b in uevs]))

    # per-call breakdown (same flush between steps; separate graphs per call)
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2()
        bevs[i][0].record(stream)
        for j, g in enumerate(per_call):
            g.replay()
            bevs[i][j + 1].record(stream)
    torch.cuda.synchronize()
    per = np.array([[bevs[i][j].elapsed_time(bevs[i][j + 1]) for j in range(5)] for i in range(args.steps)])
    mean = per.mean(axis=0)
    t_ssg, t_step, t_dec = max_over_ranks([t_ssg, t_step, t_dec], dev)
    mean = np.array(max_over_ranks(list(mean), dev))

    # ---- FastKV token-selective propagation on the same layer size (timed on
    # its own, not part of the step): head-summed pooled scores of 8 heads,
    # k_tsp = floor(0.2 S) tokens plus the window, bf16 hidden rows [S, 4096]
    from kv_cache_compression_score_b200.runner import TspSelector
    k_tsp, d_hidden = (S * 2) // 10, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 11)
    hidden = torch.randn((S, d_hidden), generator=gen, device=dev).to(torch.bfloat16)
    raw_tsp = torch.from_numpy(synth.random_scores(seed + 12, (n_kv, S))).to(dev)
    tsp = TspSelector(S, w, cfg["pool_k"], k_tsp, d_hidden, "bf16", device=dev)
    tsp.run(raw_tsp, hidden)
    torch.cuda.synchronize()
    g_tsp, _ = capture([lambda: tsp.run(raw_tsp, hidden)])
    tevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2()
        tevs[i][0].record(stream)
        g_tsp.replay()
        tevs[i][1].record(stream)
    torch.cuda.synchronize()
    t_tsp = max_over_ranks([float(np.mean([a.elapsed_time(b) for a, b in tevs]))], dev)[0]
    tsp_bytes = n_kv * S * 4 + 2 * (k_tsp + w) * d_hidden * 2   # raw scores read; hidden rows read and written
    del hidden

    # ---- the other workloads (each timed on its own, same flush discipline)
    workloads = {}
    if not args.headline_only:
        workloads = run_workloads(args, dev, stream, flush_l2, seed, hbm)
        if rank == 0 and world == 1:
            samples = oracle_workload_samples(seed)
            for name, smp in samples.items():
                key = name if name in workloads else next((k for k in workloads if k.startswith(name)), None)
                if key is not None:
                    workloads[key]["oracle"] = smp
                elif name == "unavailable":
                    workloads["oracle_unavailable"] = smp

    # ---- e2e: the same path through the C ABI with pinned host buffers
    e2e = run_e2e(args, cfg, bt, comp, dec, qd, off, ln, kc_all, vc_all, dev, stream, flush_l2)
    e2e["t_ms"] = max_over_ranks([e2e["t_ms"]], dev)[0]

    score_b, gather_b, decode_b = algorithmic_bytes(cfg)
    ssg_gbs = (score_b + gather_b) / (t_ssg * 1e-3) / 1e9
    dec_gbs = decode_b / (t_dec * 1e-3) / 1e9
    # dominant call by time -> roofline object (all HBM-bound)
    calls = {"score": (mean[0], score_b), "select": (mean[1], 0), "gather": (mean[2], gather_b),
             "decode": (mean[3], decode_b), "compress": (mean[4], score_b + gather_b)}
    dom = max(("compress", "decode"), key=lambda c: calls[c][0])   # the kernels of the timed step
    dom_gbs = calls[dom][1] / (calls[dom][0] * 1e-3) / 1e9 if calls[dom][1] else 0.0
    traffic = load_traffic(dom)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(world * S / (t_ssg * 1e-3) / 1e3, 1),
            "unit": "K-tok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": cfg["dtype"],
            "data": "synthetic (seeded N(0,1), 1% keys boosted +3 sigma)",
            "config": {"workload": cfg["name"], "n_h": n_h, "n_kv": n_kv, "d_h": d, "seq_len": S, "window": w,
                       "pool": cfg["pool_k"], "budget": B, "decode_batch": nb,
                       "l2": "flushed between steps (256 MiB write + 256 MiB read sweep, outside the timed events)",
                       "launch": "kvc_compress_window (score+select+gather in one call) as one CUDA graph, timed "
                                 "for value; decode as a second graph; breakdown_us from one graph per call "
                                 "(the three separate calls, decode and the one-call form)",
                       "parallelism": f"replicas x{world}"},
            "gbs": round(ssg_gbs, 1),
            "decode": {"gbs": round(dec_gbs, 1), "us": round(t_dec * 1e3, 2), "frac_of_8000": round(dec_gbs / 8000, 3)},
            "breakdown_us": {c: round(float(calls[c][0]) * 1e3, 2) for c in calls},
            "ssg_us": round(t_ssg * 1e3, 2),
            "ssg_us_stats": {"graph_median": round(float(np.median(ssg_samples)) * 1e3, 2),
                             "graph_min": round(float(np.min(ssg_samples)) * 1e3, 2),
                             "uncaptured_mean": round(t_ssg_direct * 1e3, 2)},
            "ssg_frac_of_8000": round(ssg_gbs / 8000, 3),
            "tsp": {"us": round(t_tsp * 1e3, 2), "k_tsp": k_tsp, "hidden": [S, d_hidden],
                    "gbs": round(tsp_bytes / (t_tsp * 1e-3) / 1e9, 1),
                    "frac_of_measured_peak": round(tsp_bytes / (t_tsp * 1e-3) / 1e9 / hbm, 3)},
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(dom_gbs, 1), "peak": hbm,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom_gbs / hbm, 3),
                         "traffic": traffic},
            "e2e": {"value": round(world * S / (e2e["t_ms"] * 1e-3) / 1e3, 2), "unit": "K-tok/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "copied": "H2D every step from pinned host memory: q_win, K, V and the decode queries; "
                              "D2H: the index lists and the decode output; the 15 stand-in decode caches "
                              "stay resident"},
            "workloads": workloads,
            "gpu_launches": kernels_per_step * args.steps,
            "kernels_per_step": kernels_per_step,
            "clocks": clocks,
            "wall_s_timed_region": round(t_wall, 3),
        }
        line["cpu_baseline"] = cpu_baseline(cfg, bt) if world == 1 else None
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------ other workloads
def device_inputs(seed, lengths, n_h, n_kv, d, w, dtype, boost_frac, boost, dev):
    """Seeded synthetic inputs drawn on the device with the recipe's
    distributions (N(0,1) Q/K/V; per (sequence, KV head) floor(frac * len)
    keys moved by boost along one random unit direction) -- for timing
    workloads whose sizes make host generation slow.  Returns q_win, k, v."""
    import torch
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed))
    T = int(sum(lengths))
    k = torch.randn((T, n_kv, d), generator=gen, device=dev)
    if boost_frac > 0:
        t0 = 0
        for L in lengths:
            m = int(boost_frac * L)
            for h in range(n_kv):
                u = torch.randn(d, generator=gen, device=dev)
                pos = torch.randperm(int(L), generator=gen, device=dev)[:m] + t0
                k[pos, h, :] += boost * (u / u.norm())
            t0 += int(L)
    v = torch.randn((T, n_kv, d), generator=gen, device=dev)
    q = torch.randn((len(lengths) * w, n_h, d), generator=gen, device=dev)
    return q.to(td), k.to(td), v.to(td)


def time_graph(fns, flush_l2, stream, steps, warmup=3):
    """Capture fns as one CUDA graph and replay it `steps` times with the L2
    flushed before each replay (outside the events).  Returns (mean ms, min ms,
    library kernels per replay)."""
    import torch
    from kv_cache_compression_score_b200 import kvc
    for fn in fns:                       # one direct run first (kernel attributes, tensor maps)
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = kvc.kvc_launch_count()
    with torch.cuda.graph(g):
        for fn in fns:
            fn()
    launches = kvc.kvc_launch_count() - n0
    for _ in range(warmup):
        flush_l2()
        g.replay()
    ts = []
    for _ in range(steps):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ts]
    del g
    return float(np.mean(ms)), float(np.min(ms)), launches


def rate(bytes_, ms, hbm):
    gbs = bytes_ / (ms * 1e-3) / 1e9
    return {"gbs": round(gbs, 1), "frac_of_measured_peak": round(gbs / hbm, 3), "frac_of_8000": round(gbs / 8000, 3)}


WORKLOAD_NAMES = ("pr1", "s131072", "fastkv", "ragged", "freekv", "q8", "xkv")


def run_workloads(args, dev, stream, flush_l2, seed, hbm, only=None):
    """Every workload of the benchmark set besides the headline layer (or the
    one named by `only`), each through the C ABI in one CUDA graph, with
    algorithmic bytes and the fraction of the measured HBM peak."""
    import torch
    from kv_cache_compression_score_b200 import kvc, synth
    from kv_cache_compression_score_b200.runner import Compressor, Decoder, FreeKvStep, TspSelector, to_device
    steps = max(3, min(args.steps, 10))
    out = {}
    n_h, n_kv, d, w, pk = 32, 8, 128, 32, 7
    row = n_kv * d * 2                                   # bytes of one bf16 cache row (all KV heads)

    if only in (None, "pr1"):
        # -- PR1: one fp32 layer, n_h 4, n_kv 2, d_h 64, S 2048, B 256, one decode query
        bt = synth.packed_batch(1001, [2048], 4, 2, 64, 32, "f32")
        q1, k1, v1 = (to_device(bt[x], "f32", dev) for x in ("q_win", "k", "v"))
        c1 = Compressor("f32", [2048], 4, 2, 64, 32, pk, 256, device=dev, keep_raw=False)
        d1 = Decoder(1, 4, 2, 64, 256, device=dev)
        qd1 = to_device(synth.decode_queries(1009, 1, 4, 64, "f32"), "f32", dev)
        z1 = torch.zeros(1, dtype=torch.int64, device=dev)
        l1 = torch.full((1,), 256, dtype=torch.int32, device=dev)
        ms, mn, nl = time_graph([lambda: c1.compress(q1, k1, v1), lambda: d1.run(qd1, c1.buf.k_c, c1.buf.v_c, z1, l1)],
                                flush_l2, stream, steps)
        b_ssg, b_dec = 2048 * 2 * 64 * 4 + 2 * 2 * 256 * 2 * 64 * 4, 2 * 256 * 2 * 64 * 4
        out["pr1_f32_S2048_B256"] = {"us": round(ms * 1e3, 2), "min_us": round(mn * 1e3, 2), "kernels": nl,
                                     "ktok_s": round(2048 / (ms * 1e-3) / 1e3, 1), "bytes": b_ssg + b_dec,
                                     **rate(b_ssg + b_dec, ms, hbm), "note": "latency-bound (1.8 MB)"}
        del c1, d1, q1, k1, v1

    if only in (None, "s131072"):
        # -- S = 131072: B = 4096, B = S (identity), decode at batch 8, full-cache decode
        S3 = 131072
        q3, k3, v3 = device_inputs(seed + 3, [S3], n_h, n_kv, d, w, "bf16", 0.01, 3.0, dev)
        for B3, name in ((4096, "llama8b_S131072_B4096"), (S3, "llama8b_S131072_B=S")):
            c3 = Compressor("bf16", [S3], n_h, n_kv, d, w, pk, B3, device=dev, keep_raw=False)
            ms, mn, nl = time_graph([lambda: c3.compress(q3, k3, v3)], flush_l2, stream, steps)
            b = S3 * row + 2 * 2 * B3 * row
            out[name] = {"us": round(ms * 1e3, 2), "min_us": round(mn * 1e3, 2), "kernels": nl,
                         "ktok_s": round(S3 / (ms * 1e-3) / 1e3, 1), "bytes": b, **rate(b, ms, hbm)}
            if B3 == 4096:
                # decode at batch 8 over compact caches of 4096 rows (cache 0 from this step)
                kc8 = torch.randn((8 * B3, n_kv, d), device=dev).to(torch.bfloat16)
                vc8 = torch.randn_like(kc8)
                qd8 = torch.randn((8, n_h, d), device=dev).to(torch.bfloat16)
                off8 = torch.arange(8, dtype=torch.int64, device=dev) * B3
                ln8 = torch.full((8,), B3, dtype=torch.int32, device=dev)
                dd = Decoder(8, n_h, n_kv, d, B3, device=dev)
                ms, mn, nl = time_graph([lambda: dd.run(qd8, kc8, vc8, off8, ln8)], flush_l2, stream, steps)
                b = 8 * B3 * row * 2
                out["decode_b8_B4096"] = {"us": round(ms * 1e3, 2), "min_us": round(mn * 1e3, 2), "kernels": nl,
                                          "bytes": b, **rate(b, ms, hbm)}
                del kc8, vc8, dd
            del c3
        # full-cache decode: 8 independent caches of 131072 rows (4 GiB of K and V)
        kf = torch.empty((8 * S3, n_kv, d), dtype=torch.bfloat16, device=dev)
        vf = torch.empty_like(kf)
        for i in range(8):
            kf[i * S3:(i + 1) * S3].copy_(k3)
            vf[i * S3:(i + 1) * S3].copy_(v3)
        qd8 = torch.randn((8, n_h, d), device=dev).to(torch.bfloat16)
        off8 = torch.arange(8, dtype=torch.int64, device=dev) * S3
        ln8 = torch.full((8,), S3, dtype=torch.int32, device=dev)
        dd = Decoder(8, n_h, n_kv, d, S3, device=dev)
        ms, mn, nl = time_graph([lambda: dd.run(qd8, kf, vf, off8, ln8)], flush_l2, stream, steps)
        b = 8 * S3 * row * 2
        out["full_cache_decode_b8_S131072"] = {"us": round(ms * 1e3, 2), "min_us": round(mn * 1e3, 2), "kernels": nl,
                                               "bytes": b, **rate(b, ms, hbm)}
        del kf, vf, dd, q3, k3, v3

    if only in (None, "fastkv"):
        # -- FastKV: 32 layers, TSP at layer 15 (k_tsp = floor(0.2 S) + w), hidden [S, 4096]
        S4, L4 = 32768, 32
        k_tsp, b_avg = (S4 * 2) // 10, S4 // 10
        S4n = k_tsp + w
        layers = []
        for layer in range(L4):
            length = S4 if layer <= 15 else S4n
            layers.append(device_inputs(seed + 100 + layer, [length], n_h, n_kv, d, w, "bf16", 0.01, 3.0, dev))
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed + 200)
        hidden = torch.randn((S4, 4096), generator=gen, device=dev).to(torch.bfloat16)
        for sched in ("uniform", "pyramid"):
            budgets = [b_avg] * L4 if sched == "uniform" else [int(x) for x in kvc.kvc_pyramid_budgets(L4, b_avg, 1024)]
            comps = [Compressor("bf16", [S4 if l <= 15 else S4n], n_h, n_kv, d, w, pk, budgets[l], device=dev,
                                keep_raw=(l == 15)) for l in range(L4)]
            tsp = TspSelector(S4, w, pk, k_tsp, 4096, "bf16", device=dev)
            fns = [(lambda c=c, x=x: c.compress(*x)) for c, x in zip(comps, layers)]
            fns.insert(16, lambda: tsp.run(comps[15].buf.scores_raw, hidden))
            ms, mn, nl = time_graph(fns, flush_l2, stream, max(3, steps // 2))
            b = sum((S4 if l <= 15 else S4n) * row + 2 * 2 * min(budgets[l], S4 if l <= 15 else S4n) * row
                    for l in range(L4)) + 2 * (k_tsp + w) * 4096 * 2
            out[f"fastkv_32_layer_chain_{sched}"] = {
                "us": round(ms * 1e3, 2), "min_us": round(mn * 1e3, 2), "kernels": nl, "bytes": b, **rate(b, ms, hbm),
                "budgets": [budgets[0], budgets[15], budgets[31]] if sched == "pyramid" else b_avg}
            del comps, tsp
        del layers, hidden

    if only in (None, "ragged"):
        # -- ragged batch: 16 lengths uniform on [4096, 65536], B = min(1024, len), then decode over the 16 caches
        lens5 = [int(x) for x in synth.ragged_lengths(1005, 16, 4096, 65536)]
        q5, k5, v5 = device_inputs(seed + 5, lens5, n_h, n_kv, d, w, "bf16", 0.01, 3.0, dev)
        c5 = Compressor("bf16", lens5, n_h, n_kv, d, w, pk, 1024, device=dev, keep_raw=False)
        cb5 = c5.buf.cu_budget_host
        off5 = torch.tensor(cb5[:-1], dtype=torch.int64, device=dev)
        ln5 = torch.tensor(np.diff(cb5), dtype=torch.int32, device=dev)
        qd5 = torch.randn((16, n_h, d), device=dev).to(torch.bfloat16)
        d5 = Decoder(16, n_h, n_kv, d, 1024, device=dev)
        ms_c, mn_c, nl_c = time_graph([lambda: c5.compress(q5, k5, v5)], flush_l2, stream, steps)
        ms_d, mn_d, nl_d = time_graph([lambda: d5.run(qd5, c5.buf.k_c, c5.buf.v_c, off5, ln5)], flush_l2, stream, steps)
        b_c = sum(lens5) * row + 2 * 2 * 16 * 1024 * row
        b_d = 16 * 1024 * row * 2
        out["ragged_16_B1024"] = {"tokens": sum(lens5), "compress_us": round(ms_c * 1e3, 2), "compress_kernels": nl_c,
                                  "ktok_s": round(sum(lens5) / (ms_c * 1e-3) / 1e3, 1), "compress_bytes": b_c,
                                  "compress": rate(b_c, ms_c, hbm), "decode_us": round(ms_d * 1e3, 2),
                                  "decode_bytes": b_d, "decode": rate(b_d, ms_d, hbm)}
        del c5, d5, q5, k5, v5

    if only in (None, "freekv"):
        # -- FreeKV decode step: batch 16 over full caches of S = 32768, B = 2048, tau = 0.9
        S6, B6, nb6 = 32768, 2048, 16
        _, k6, v6 = device_inputs(seed + 6, [S6] * nb6, n_h, n_kv, d, w, "bf16", 0.01, 3.0, dev)
        fk = FreeKvStep([S6] * nb6, n_h, n_kv, d, w, pk, B6, 0.9, device=dev)
        q_prev = synth.decode_queries(seed + 61, nb6, n_h, d, "bf16")
        q_cur = synth.drifted_queries(seed + 62, q_prev, "bf16", group=n_h // n_kv)
        qp, qc = to_device(q_prev, "bf16", dev), to_device(q_cur, "bf16", dev)
        fk.step(qp, qp, k6, v6, tau=2.0)                     # first step: every head selects
        torch.cuda.synchronize()
        idx0, kc0, vc0 = fk.idx.clone(), fk.k_c.clone(), fk.v_c.clone()

        def fk_step():
            fk.idx.copy_(idx0)                               # every replay starts from the same previous step
            fk.k_c.copy_(kc0)
            fk.v_c.copy_(vc0)
            fk.step(qc, qp, k6, v6)
        ms, mn, nl = time_graph([fk_step], flush_l2, stream, steps)
        # the restore copies are timed too; time them alone and subtract
        ms_r, _, _ = time_graph([lambda: (fk.idx.copy_(idx0), fk.k_c.copy_(kc0), fk.v_c.copy_(vc0))], flush_l2, stream,
                                steps)
        n_flag = int(fk.reselected.sum().item())
        b = n_flag * (S6 * 256 + 2 * 2 * B6 * 256) + nb6 * B6 * row * 2
        ms_step = max(ms - ms_r, 1e-6)
        out["freekv_step_b16_S32768_B2048"] = {"us": round(ms_step * 1e3, 2), "kernels": nl,
                                               "reselected_heads": n_flag, "heads": nb6 * n_kv, "tau": 0.9,
                                               "bytes": b, **rate(b, ms_step, hbm),
                                               "note": "restore copies timed separately and subtracted"}
        del fk, k6, v6

    if only in (None, "q8"):
        # -- int8 compact caches: gather-and-quantise (16 x 2048 rows) and decode over them at batch 16
        nb7, B7 = 16, 2048
        kb = torch.randn((nb7 * B7, n_kv, d), device=dev).to(torch.bfloat16)
        vb = torch.randn_like(kb)
        idx7 = torch.arange(nb7 * B7, dtype=torch.int32, device=dev).repeat(n_kv, 1).contiguous()
        cu7 = torch.tensor([0, nb7 * B7], dtype=torch.int32, device=dev)
        kq = torch.empty((nb7 * B7, n_kv, d), dtype=torch.int8, device=dev)
        vq = torch.empty_like(kq)
        ks = torch.empty((n_kv, nb7 * B7), dtype=torch.float32, device=dev)
        vs = torch.empty_like(ks)
        ms_g, _, nl_g = time_graph([lambda: kvc.kvc_gather_kv_q8([nb7 * B7], cu7, cu7, nb7 * B7, idx7, kb, vb, kq, vq,
                                                                 ks, vs)], flush_l2, stream, steps)
        qd7 = torch.randn((nb7, n_h, d), device=dev).to(torch.bfloat16)
        off7 = torch.arange(nb7, dtype=torch.int64, device=dev) * B7
        ln7 = torch.full((nb7,), B7, dtype=torch.int32, device=dev)
        d7 = Decoder(nb7, n_h, n_kv, d, B7, device=dev)
        ms_d, mn_d, nl_d = time_graph([lambda: kvc.kvc_gqa_decode_attn_q8(qd7, kq, vq, ks, vs, off7, ln7, B7, 0.0, d7.out,
                                                                          d7.ws)], flush_l2, stream, steps)
        rows = nb7 * B7 * n_kv
        b_g = rows * (2 * 256 + 2 * 128 + 8)
        b_d = rows * (2 * 128 + 8)
        out["q8_b16_B2048"] = {"gather_quantise_us": round(ms_g * 1e3, 2), "gather_quantise_bytes": b_g,
                               "gather_quantise": rate(b_g, ms_g, hbm), "decode_us": round(ms_d * 1e3, 2),
                               "decode_bytes": b_d, "decode": rate(b_d, ms_d, hbm)}
        del kb, vb, kq, vq, d7

    if only in (None, "xkv"):
        # -- xKV: factorise the keys of a window of W = 4 layers (S = 32768, r = 64, bf16 basis, 8 iteration steps),
        #    then rebuild 2048 selected rows per head of one layer (selective) and all S rows (dense)
        S8, W8, r8, it8 = 32768, 4, 64, 8
        F8 = W8 * d
        keys8 = [torch.randn((S8, n_kv, d), device=dev).to(torch.bfloat16) for _ in range(W8)]
        gen8 = torch.Generator(device=dev)
        gen8.manual_seed(seed + 8)
        v08 = torch.randn((n_kv, F8, r8), generator=gen8, device=dev)
        basis8 = torch.empty((n_kv, S8, r8), dtype=torch.bfloat16, device=dev)
        blocks8 = torch.empty((n_kv, r8, F8), dtype=torch.float32, device=dev)
        ws8 = torch.empty(kvc.kvc_xkv_workspace_size(S8, n_kv, d, W8, r8), dtype=torch.uint8, device=dev)
        ms_f, _, nl_f = time_graph([lambda: kvc.kvc_xkv_factorize(keys8, r8, it8, v08, basis8, blocks8, ws8)], flush_l2,
                                   stream, steps)
        gram_flops = 2 * S8 * F8 * F8 * n_kv
        b_f = 2 * W8 * S8 * n_kv * d * 2 + n_kv * S8 * r8 * 2         # keys read by the Gram and the projection, A written
        res = {"factorize_us": round(ms_f * 1e3, 2), "factorize_kernels": nl_f, "iters": it8,
               "gram_tflops_equiv": round(gram_flops / (ms_f * 1e-3) / 1e12, 1), "factorize_bytes": b_f,
               "factorize": rate(b_f, ms_f, hbm)}
        for n_sel, tag in ((2048, "selective_2048"), (S8, "dense")):
            idx8 = torch.randint(0, S8, (n_kv, n_sel), dtype=torch.int32, device=dev)
            out8 = torch.empty((n_sel, n_kv, d), dtype=torch.bfloat16, device=dev)
            ms_r, _, nl_r = time_graph([lambda: kvc.kvc_xkv_reconstruct(W8, 1, basis8, blocks8, idx8, out8)], flush_l2,
                                       stream, steps)
            b_r = n_sel * n_kv * (r8 * 2 + d * 2 + 4) + n_kv * r8 * d * 4
            res[f"rebuild_{tag}_us"] = round(ms_r * 1e3, 2)
            res[f"rebuild_{tag}_bytes"] = b_r
            res[f"rebuild_{tag}"] = rate(b_r, ms_r, hbm)
            res[f"rebuild_{tag}_gflops"] = round(2 * n_sel * n_kv * r8 * d / (ms_r * 1e-3) / 1e9, 1)
            del idx8, out8
        out[f"xkv_S{S8}_W{W8}_r{r8}"] = res
        del keys8, v08, basis8, blocks8, ws8

    torch.cuda.empty_cache()
    return out


def run_e2e(args, cfg, bt, comp, dec, qd, off, ln, kc_all, vc_all, dev, stream, flush_l2):
    """Inputs copied host->device from pinned memory and results device->host
    inside the timed region, every step."""
    import torch
    from kv_cache_compression_score_b200.runner import to_device

    h_q = to_device(bt["q_win"], cfg["dtype"], "cpu").pin_memory()
    h_k = to_device(bt["k"], cfg["dtype"], "cpu").pin_memory()
    h_v = to_device(bt["v"], cfg["dtype"], "cpu").pin_memory()
    h_qd = qd.cpu().pin_memory()
    d_q, d_k, d_v = torch.empty_like(h_q, device=dev), torch.empty_like(h_k, device=dev), torch.empty_like(h_v, device=dev)
    h_idx = torch.empty(comp.buf.idx.shape, dtype=torch.int32).pin_memory()
    h_out = torch.empty(dec.out.shape, dtype=torch.float32).pin_memory()
    n = max(3, min(args.steps, 10))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n + 1)]
    for i in range(n + 1):             # first iteration untimed (warm-up)
        flush_l2()
        evs[i][0].record(stream)
        d_q.copy_(h_q, non_blocking=True)
        d_k.copy_(h_k, non_blocking=True)
        d_v.copy_(h_v, non_blocking=True)
        qd.copy_(h_qd, non_blocking=True)
        comp.compress(d_q, d_k, d_v, stream)
        dec.run(qd, kc_all, vc_all, off, ln, stream)
        h_idx.copy_(comp.buf.idx, non_blocking=True)
        h_out.copy_(dec.out, non_blocking=True)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    t = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in range(1, n + 1))
    h2d = sum(x.numel() * x.element_size() for x in (h_q, h_k, h_v, h_qd))
    d2h = h_idx.numel() * 4 + h_out.numel() * 4
    return {"t_ms": t, "h2d": h2d, "d2h": d2h}


def load_traffic(call):
    """DRAM bytes per launch of a call's kernel from the committed ncu summary
    (profiles/traffic.json), or None once the kernel's source has changed
    since the counters were taken (its sha256 no longer matches)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        e = json.load(f).get(call)
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != e["sha256"]:
        return None
    return e["bytes_per_launch"]


# ----------------------------------------------------------- oracle arm
def oracle_step(cfg, bt):
    from oracle import kvc_oracle as O
    cu = bt["cu_seqlens"]
    raw = O.raw_scores(bt["q_win"], bt["k"], cu, cfg["n_h"], cfg["n_kv"], cfg["w"], cfg["dtype"])
    pooled = O.pool_prefix(raw, cu, cfg["w"], cfg["pool_k"])
    idx = O.select_topk(pooled, cu, cfg["w"], cfg["budget"])
    O.gather_kv(bt["k"], bt["v"], idx, cu, cfg["budget"])


def _timed(fn, min_s=0.3):
    """Seconds per call of fn (repeated until min_s of host time has passed)."""
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        t = time.perf_counter() - t0
        if t >= min_s:
            return t / reps


def oracle_workload_samples(seed):
    """The oracle timed beside every workload of the set, each on a bounded
    sample of the workload (one KV head, one sequence or one batch entry, as
    stated), on the host's cores, scaled to the workload's unit.  Context, not
    a target: about 20 s of host time in all."""
    from oracle import kvc_oracle as O
    from kv_cache_compression_score_b200 import synth
    out = {}
    n_h, n_kv, d, w, pk = 32, 8, 128, 32, 7

    def layer_one_head(S, budget, dtype="bf16", nh=4, nkv=1, dd=128, s=seed):
        bt = synth.packed_batch(s, [S], nh, nkv, dd, w, dtype, 0.01, 3.0)
        cu = bt["cu_seqlens"]

        def step():
            raw = O.raw_scores(bt["q_win"], bt["k"], cu, nh, nkv, w, dtype)
            pooled = O.pool_prefix(raw, cu, w, pk)
            idx = O.select_topk(pooled, cu, w, budget)
            O.gather_kv(bt["k"], bt["v"], idx, cu, budget)
        return _timed(step)

    def decode_one(rows, dtype="bf16", dd=128):
        k, v = synth.keys_values(seed + 1, 0, rows, n_kv, dd, dtype)
        q = synth.decode_queries(seed + 2, 1, n_h, dd, dtype)
        return _timed(lambda: O.gqa_decode(q, k, v, [0], [rows], n_kv, dtype))

    try:
        # PR1: the whole fp32 layer (n_h 4, n_kv 2, d 64, S 2048, B 256) and one decode query
        bt = synth.packed_batch(seed + 11, [2048], 4, 2, 64, 32, "f32")
        cu = bt["cu_seqlens"]

        def pr1():
            raw = O.raw_scores(bt["q_win"], bt["k"], cu, 4, 2, 32, "f32")
            idx = O.select_topk(O.pool_prefix(raw, cu, 32, pk), cu, 32, 256)
            kc, vc = O.gather_kv(bt["k"], bt["v"], idx, cu, 256)
            O.gqa_decode(synth.decode_queries(seed + 12, 1, 4, 64, "f32"), kc, vc, [0], [256], 2, "f32")
        t = _timed(pr1)
        out["pr1_f32_S2048_B256"] = {"value": round(2048 / t / 1e3, 2), "unit": "K-tok/s", "sample": "the whole workload"}
        # S = 131072: one KV head (its 4 query heads) of the layer, times 8 heads
        t = layer_one_head(131072, 4096) * n_kv
        out["llama8b_S131072_B4096"] = {"value": round(131072 / t / 1e3, 2), "unit": "K-tok/s",
                                        "sample": "one KV head of the layer, scaled by 8"}
        # decode: one batch entry (4096 rows; 131072 rows), scaled to the workload's bytes
        t = decode_one(4096) * 8
        out["decode_b8_B4096"] = {"value": round(8 * 4096 * n_kv * d * 4 / t / 1e9, 3), "unit": "GB/s",
                                  "sample": "one of 8 caches, scaled by 8"}
        t = decode_one(131072) * 8
        out["full_cache_decode_b8_S131072"] = {"value": round(8 * 131072 * n_kv * d * 4 / t / 1e9, 3),
                                               "unit": "GB/s", "sample": "one of 8 caches, scaled by 8"}
        # FastKV chain: one head of a 32768-token layer and of a 6585-token layer, 16 of each, plus the TSP select
        t_full = layer_one_head(32768, 3276) * n_kv
        t_short = layer_one_head(6585, 3276) * n_kv
        raw_tsp = synth.random_scores(seed + 13, (n_kv, 32768))
        t_tsp = _timed(lambda: O.tsp_select(raw_tsp, 32768, w, pk, 6553))
        t = 16 * t_full + 16 * t_short + t_tsp
        out["fastkv_32_layer_chain"] = {"value": round(t * 1e6, 0), "unit": "us",
                                        "sample": "one KV head of a 32768- and a 6585-token layer (x8 heads, x16 "
                                                  "layers each) plus the TSP select"}
        # ragged: one sequence of the median length, scaled by tokens
        lens = sorted(int(x) for x in synth.ragged_lengths(1005, 16, 4096, 65536))
        L = lens[len(lens) // 2]
        t = layer_one_head(L, 1024) * n_kv
        out["ragged_16_B1024"] = {"value": round(L / t / 1e3, 2), "unit": "K-tok/s",
                                  "sample": f"one KV head of one {L}-token sequence, scaled by 8"}
        # FreeKV: one batch entry of the step (S 32768, B 2048), scaled by 16
        k6, v6 = synth.keys_values(seed + 14, 0, 32768, n_kv, d, "bf16")
        qp = synth.decode_queries(seed + 15, 1, n_h, d, "bf16")
        qc = synth.drifted_queries(seed + 16, qp, "bf16", group=n_h // n_kv)
        idx0 = np.zeros((n_kv, 2048), dtype=np.int64)
        t = _timed(lambda: O.freekv_step(qc, qp, k6, v6, [0, 32768], idx0, n_kv, w, pk, 2048, 0.9, "bf16")) * 16
        out["freekv_step_b16_S32768_B2048"] = {"value": round(t * 1e6, 0), "unit": "us",
                                               "sample": "one of 16 sequences, scaled by 16"}
        # int8: gather-and-quantise and decode for one 2048-row cache, scaled by 16
        kb, vb = synth.keys_values(seed + 17, 0, 2048, n_kv, d, "bf16")
        idx7 = np.broadcast_to(np.arange(2048), (n_kv, 2048))
        kq, vq, ks, vs = O.gather_kv_q8(kb, vb, idx7, [0, 2048], 2048, "bf16")
        t_g = _timed(lambda: O.gather_kv_q8(kb, vb, idx7, [0, 2048], 2048, "bf16")) * 16
        qd = synth.decode_queries(seed + 18, 1, n_h, d, "bf16")
        t_d = _timed(lambda: O.gqa_decode_q8(qd, kq, vq, ks, vs, [0], [2048], n_kv, "bf16")) * 16
        out["q8_b16_B2048"] = {"gather_quantise_us": round(t_g * 1e6, 0), "decode_us": round(t_d * 1e6, 0),
                               "unit": "us", "sample": "one of 16 caches, scaled by 16"}
        # xKV: the factorisation of one KV head (S 32768, W 4, r 64), scaled by 8
        keys = synth.cross_layer_keys(seed + 19, 32768, 1, d, 4, 64)
        t = _timed(lambda: O.xkv_factorize(keys, 64, "bf16"), min_s=0.1) * n_kv
        out["xkv_S32768_W4_r64"] = {"factorize_us": round(t * 1e6, 0), "unit": "us",
                                    "sample": "one KV head (exact SVD), scaled by 8"}
    except Exception as e:   # context only: never a reason to fail the bench
        out["unavailable"] = str(e)[:120]
    for v in out.values():
        if isinstance(v, dict):
            v["kind"] = "oracle"
            v["cores"] = oracle_threads()
    return out


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(cfg, bt, budget_s=10.0):
    """The oracle, as it stands, on one full layer of the same workload
    (score + select + gather over all KV heads), repeated for ~10 s on the
    host's cores (the BLAS thread pool), then once on one thread."""
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_step(cfg, bt)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    t = time.perf_counter() - t0
    one = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t1 = time.perf_counter()
            oracle_step(cfg, bt)
            t1 = time.perf_counter() - t1
        one = {"value": round(cfg["S"] / t1 / 1e3, 3), "unit": "K-tok/s", "threads": 1,
               "sample": f"1 full layer in {t1:.2f} s"}
    except Exception as e:   # the baseline is context, never a reason to fail the bench
        one = {"unavailable": str(e)[:80]}
    return {"value": round(reps * cfg["S"] / t / 1e3, 3), "unit": "K-tok/s", "cores": oracle_threads(),
            "kind": "oracle", "sample": f"{reps} full layers (S={cfg['S']}, all {cfg['n_kv']} KV heads) in {t:.1f} s",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(), "single_thread": one,
            "threads_note": "cores = BLAS threads of the matrix products; the per-(sequence, head) loops are serial"}


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return
    from kv_cache_compression_score_b200 import synth
    cfg = dict(LLAMA3_8B_S32K)
    bt = synth.packed_batch(cfg["seed"], [cfg["S"]], cfg["n_h"], cfg["n_kv"], cfg["d_h"], cfg["w"], cfg["dtype"],
                            cfg["boost_frac"], cfg["boost"])
    for _ in range(args.warmup):
        oracle_step(cfg, bt)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(cfg, bt)
        ts.append(time.perf_counter() - t0)
    t = statistics.mean(ts)
    v = round(world * cfg["S"] / t / 1e3, 3)
    line = {"metric": METRIC, "value": v, "unit": "K-tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), 1% keys boosted +3 sigma)",
            "config": {"workload": cfg["name"], "n_h": cfg["n_h"], "n_kv": cfg["n_kv"], "d_h": cfg["d_h"],
                       "seq_len": cfg["S"], "window": cfg["w"], "pool": cfg["pool_k"], "budget": cfg["budget"]},
            "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "K-tok/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"one full layer per step (S={cfg['S']}, all KV heads), score+select+gather"},
            "e2e": {"value": v, "unit": "K-tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_one_workload(args):
    """One workload of the set on one GPU, alone, printed as one JSON line."""
    import torch
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    from kv_cache_compression_score_b200 import build as kbuild
    kbuild.build()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sweep = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        torch.sum(sweep, dim=0, out=sink)

    hbm, peak_kind = measured_peaks()
    res = run_workloads(args, dev, torch.cuda.current_stream(dev), flush_l2, LLAMA3_8B_S32K["seed"], hbm,
                        only=args.workload)
    print(json.dumps({"workload": args.workload, "peak_gbs": hbm, "peak_kind": peak_kind, "steps": args.steps,
                      "warmup": args.warmup, "results": res}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the Llama-3-8B S=32K layer (skip the other workloads)")
    ap.add_argument("--workload", choices=WORKLOAD_NAMES, default=None,
                    help="time only this one workload of the set (no headline line; for profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload:
        run_one_workload(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
