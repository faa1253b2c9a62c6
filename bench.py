#!/usr/bin/env python
"""Decode-step benchmark of exact top-k retrieval attention on B200.

A step is one pass of the whole hot path for every layer of the workload, one
ra_decode_step_append call per layer: append the new token's K/V row and score all positions
(the append runs inside the scan), then select the top-k per query head and attend over sinks +
window + top-k (the selection launched behind the scan starts on each KV head as the scan
finishes it).  A phase pass after the timed region runs the scan (ra_score_gqa_append) and the
selection (ra_select_attend) as separate calls to time each.  The cache holds N-1 tokens; each
step appends the N-th and decodes over N, then the next step re-appends into the same slot, so
every step has identical work.  Each step uses its own query.  (The threshold mode, --eps,
appends with ra_append_kv and runs ra_decode_step_eps.)

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Rank 0 prints one JSON line.  `value` is whole-job decode steps/s with the caches resident in
HBM; `e2e` is the same metric through the C ABI's host-buffer step (ra_decode_step_append_host)
with the step's inputs (query, new K/V row) copied from pinned host memory and the outputs
(out, idx) copied back and waited for inside the timed region; `roofline` is the score kernel
(the K scan, the dominant kernel) against the measured HBM copy bandwidth; `cpu_baseline` is the
fp64 oracle on a bounded sample timed on the host cores; `configs` holds the 32-layer 1M-token
cache and the batch-16 256K layer, measured the same way in the same run.  `--impl reference`
times only the oracle (the reference arm).
Under torchrun each rank runs an independent replica (the step does not shard across GPUs).
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode steps/s & K-scan HBM GB/s (frac of peak) at 128K–1M ctx, top-k sparse attn"
DEFAULT_WORKLOAD = "l8b_128k_k1pct"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

# dram__bytes_read.sum + dram__bytes_write.sum of one score-kernel launch, from an ncu capture,
# keyed by the hash of the score kernel's own sources (score.cu and its TMA helpers, comments
# removed) it was taken on, so a changed kernel reports null until it is captured again.  Values
# are per launch of the named workload (the score-kernel ncu summary under profiles/).
TRAFFIC = {("3c7ba5e51d427bb6", "l8b_128k_k1pct"): 274.11e6}


def score_source_hash() -> str:
    """sha256 of the score kernel's sources (its own file, the TMA helpers and tensor maps, and
    the shared header with the digit-1 bin and the parameter structs) with // comments and blank
    lines removed, so that a comment edit keeps the key and any code edit changes it."""
    h = hashlib.sha256()
    for f in ("score.cu", "tma.cuh", "tmap.cu", "common.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "top_retrieval_attention_b200", "csrc", f)) as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: ~1 s of work)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the 1M x 32-layer and batch-16 workloads the default line also reports")
    ap.add_argument("--eps", type=float, default=0.0,
                    help="threshold budget: keep candidates whose softmax weight exceeds eps "
                         "(at most k per head; ra_decode_step_eps)")
    ap.add_argument("--pyramid", type=float, default=0.0,
                    help="per-layer budgets falling linearly with depth to this ratio of the "
                         "first layer's, mean k (ra_pyramid_budgets)")
    ap.add_argument("--paged", action="store_true",
                    help="paged cache (128-token pages, shuffled) with ragged lengths falling "
                         "linearly from N to N/2 over the batch (ra_paged_decode_step)")
    ap.add_argument("--sweep", action="store_true",
                    help="every point of the 512K sweep (top-k x group size x head dim), one JSON "
                         "line each, the dense decode beside it (no e2e / CPU legs)")
    ap.add_argument("--ivf", type=int, default=0, metavar="NLIST",
                    help="decode through a device-built IVF index of NLIST clusters per KV head "
                         "(one layer); reports Recall@k against the exact top-k")
    ap.add_argument("--nprobe", type=int, default=32, help="IVF clusters probed per query head")
    ap.add_argument("--ivf-iters", type=int, default=4, help="k-means iterations of the IVF build")
    ap.add_argument("--prefill-queries", type=int, default=0,
                    help="instead of decode steps: exact top-k of this many prefill queries per "
                         "query head (tensor-core scores + cluster selection), one layer")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing


def dist_info():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def dist_init(world, use_cuda):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group("nccl" if use_cuda else "gloo",
                            timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks during timing


class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * max(mx or [1])] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(rows)}


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            v = float(json.load(fh)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ CPU oracle (baseline legs)


def _blas_threads() -> int:
    from threadpoolctl import threadpool_info
    cores = 1
    for info in threadpool_info():
        if info.get("user_api") == "blas":
            cores = max(cores, int(info.get("num_threads", 1)))
    return cores


def _oracle_group_seconds(w, qh, K, V, k_s) -> float:
    """Wall time of the oracle's decode of the G query heads that share KV head 0."""
    import oracle
    t0 = time.perf_counter()
    for h in range(w.G):
        oracle.decode_head(qh[0, h], K, V, k_s, w.n_sink, w.n_window)
    return time.perf_counter() - t0


def oracle_sample(w, seconds: float):
    """The fp64 oracle on one KV head group (G query heads) of layer 0 at full N, repeated for
    about `seconds`; returns (steps/s, cores, description) scaled to one whole step."""
    from synth import gen
    qh = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    K, V = gen.host_head(w, 0, 0, 0, w.N)
    times = []
    t_end = time.perf_counter() + seconds
    while not times or time.perf_counter() < t_end:
        times.append(_oracle_group_seconds(w, qh, K, V, w.k))
    scale = w.Hkv * w.B * w.layers
    step_s = statistics.median(times) * scale
    desc = (f"oracle decode of the {w.G} query heads of KV head 0 (layer 0, b 0) over all "
            f"{w.N} keys, median of {len(times)} runs, x{scale} for the whole step")
    return 1.0 / step_s, _blas_threads(), desc, sum(times)


def run_reference(args, w, rank, world):
    """The reference arm: the oracle as it stands, on the host cores.  Each step times the
    oracle on a bounded sample of the workload (the G query heads of one KV head over a
    contiguous slice of the keys, with k scaled to the slice), sized so the whole run takes
    about 100 s, and scales it to one whole step (the oracle's cost is linear in N apart from
    the sort's log factor, so this slightly flatters the CPU at large N)."""
    if rank != 0:
        return
    from synth import gen
    steps = args.steps if args.steps is not None else 5
    warm = args.warmup
    budget = max(0.005, 100.0 / max(1, steps + warm))
    qh = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    n_cal = min(w.N, 8192)
    K, V = gen.host_head(w, 0, 0, 0, n_cal)
    t_cal = min(_oracle_group_seconds(w, qh, K, V, max(1, w.k * n_cal // w.N)) for _ in range(3))
    n_keys = int(min(w.N, max(1024, n_cal * budget / max(t_cal, 1e-9))))
    K, V = gen.host_head(w, 0, 0, 0, n_keys)
    k_s = w.k if n_keys == w.N else max(1, int(round(w.k * n_keys / w.N)))
    scale = (w.N / n_keys) * w.Hkv * w.B * w.layers
    vals = []
    timed = 0.0
    for i in range(warm + steps):
        t = _oracle_group_seconds(w, qh, K, V, k_s)
        if i >= warm:
            vals.append(1.0 / (t * scale))
            timed += t
    value = statistics.median(vals)
    desc = (f"per step: oracle decode of the {w.G} query heads of KV head 0 (layer 0, b 0) over "
            f"keys [0, {n_keys}) of {w.N} with k={k_s}, scaled x{scale:.1f} to one whole step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": 1000.0 / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "sampled": True,
        "steps_note": (f"each of the {steps} timed steps runs the oracle on one sample of the "
                       f"workload ({desc}); ms_per_step is the scaled whole-step time, not the "
                       f"time the samples took"),
        "timed_seconds": timed,
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": _blas_threads(),
                         "kind": "oracle", "sample": desc, "sampled": True,
                         "timed_seconds": timed},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N,
            "k": w.k, "n_sink": w.n_sink, "n_window": w.n_window, "layers": w.layers,
            "needles_per_kv_head": w.n_needle, "parallelism": "replicas",
            "l2": "inputs larger than L2 (whole K scanned every step); a distinct query per step"}


# ------------------------------------------------------------------ our arm


def run_ours(args, w, rank, local_rank, world, dist):
    import ctypes

    import torch

    import top_retrieval_attention_b200 as ra
    from synth import device as sdev
    from synth import gen

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ra.lib()
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    L, B, Hq, Hkv, d, N, k = w.layers, w.B, w.Hq, w.Hkv, w.d, w.N, w.k

    # caches: rows [0, N) filled by the generator; the last row is the token each step appends
    caches, knew, vnew = [], [], []
    for layer in range(L):
        c = ra.KVCache(B, Hkv, d, N, device=dev)
        sdev.device_layer(w, layer, c.K, c.V)
        knew.append(c.K[:, :, N - 1:N].clone())
        vnew.append(c.V[:, :, N - 1:N].clone())
        c.N = N - 1
        caches.append(c)
    P = 16
    qpool = torch.empty((P, L, B, Hq, d), dtype=torch.bfloat16, device=dev)
    for s in range(P):
        for layer in range(L):
            sdev.fill_q(qpool[s, layer], w.seed + 7919 * s + 104729 * layer)
    ks = ra.pyramid_budgets(L, k, args.pyramid) if args.pyramid > 0 else [k] * L
    ws_bytes = ra.ra_decode_workspace_bytes(B, Hq, N, d, max(ks), w.n_sink, w.n_window)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    outs = [torch.empty((B, Hq, d), dtype=torch.float32, device=dev) for _ in range(L)]
    idxs = [torch.empty((B, Hq, max(kl, 1)), dtype=torch.int32, device=dev) for kl in ks]
    torch.cuda.synchronize()

    def phases(layer, qptr, ev=None):
        c = caches[layer]
        kv = c.kv
        kl = ks[layer]
        if ev is None and args.eps <= 0:
            # the product call: the scan (with the token's append inside it), and the selection
            # + attention launched behind it, starting on each KV head as the scan finishes it
            ra.check(ra.ra_decode_step_append(kv, qptr, knew[layer].data_ptr(), vnew[layer].data_ptr(),
                                              Hq, kl, w.n_sink, w.n_window, outs[layer].data_ptr(),
                                              idxs[layer].data_ptr(), ws.data_ptr(), ws_bytes, sp),
                     "decode_step_append")
            c.N = N - 1
            return
        if ev is not None:
            ev[0].record(stream)
        if args.eps <= 0:   # the phases launched apart: the scan alone, then select + attend
            ra.check(ra.ra_score_gqa_append(kv, qptr, knew[layer].data_ptr(), vnew[layer].data_ptr(),
                                            Hq, kl, w.n_sink, w.n_window, ws.data_ptr(), ws_bytes,
                                            sp), "score_append")
            if ev is not None:
                ev[1].record(stream)
                ev[2].record(stream)
            ra.check(ra.ra_select_attend(kv, Hq, kl, w.n_sink, w.n_window, idxs[layer].data_ptr(),
                                         outs[layer].data_ptr(), ws.data_ptr(), ws_bytes, sp),
                     "select_attend")
            if ev is not None:
                ev[3].record(stream)
            c.N = N - 1
            return
        ra.check(ra.ra_append_kv(kv, knew[layer].data_ptr(), vnew[layer].data_ptr(), 1, sp), "append")
        if ev is not None:
            ev[1].record(stream)
        if args.eps > 0:   # the threshold step as one call (score, then select + attend)
            ra.check(ra.ra_decode_step_eps(kv, qptr, Hq, kl, args.eps, w.n_sink, w.n_window,
                                           outs[layer].data_ptr(), idxs[layer].data_ptr(),
                                           ws.data_ptr(), ws_bytes, sp), "decode_step_eps")
            if ev is not None:
                ev[2].record(stream)
                ev[3].record(stream)
            c.N = N - 1
            return
        ra.check(ra.ra_score_gqa(kv, qptr, Hq, kl, w.n_sink, w.n_window, ws.data_ptr(), ws_bytes, sp), "score")
        if ev is not None:
            ev[2].record(stream)
        ra.check(ra.ra_select_attend(kv, Hq, kl, w.n_sink, w.n_window, idxs[layer].data_ptr(),
                                     outs[layer].data_ptr(), ws.data_ptr(), ws_bytes, sp), "select_attend")
        if ev is not None:
            ev[3].record(stream)
        c.N = N - 1

    def step(s, evs=None):
        for layer in range(L):
            phases(layer, qpool[s % P, layer].data_ptr(), None if evs is None else evs[layer])

    # warm-up, then (for short timed regions) an untimed soak so clocks reach steady state
    for s in range(max(3, args.warmup)):
        step(s)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for s in range(5):
        step(s)
    torch.cuda.synchronize()
    est = max((time.perf_counter() - t0) / 5, 1e-6)
    steps = args.steps if args.steps is not None else max(10, min(20000, int(1.0 / est)))
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    clk = Clocks(uuid)
    clk.start()
    soak_end = time.perf_counter() + 0.4
    s = 0
    while time.perf_counter() < soak_end:
        step(s)
        s += 1
        if s % 64 == 0:
            torch.cuda.synchronize()
    barrier(dist, local_rank)
    torch.cuda.synchronize()
    t_start.record(stream)
    for s in range(steps):
        step(s)
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(dist, local_rank)
    clocks = clk.stop()
    elapsed_ms = t_start.elapsed_time(t_stop)
    elapsed_ms = max_over_ranks(dist, elapsed_ms, dev)
    ms_per_step = elapsed_ms / steps
    value = world * steps / (elapsed_ms / 1000.0)

    # phase pass right after the timed region: the same launches with events between the
    # phases, which also removes the overlap of the selection with the scan.  It gives the score
    # kernel's own duration (the roofline: inside the step the selection runs beside the scan,
    # so events cannot separate the two there) and the phase breakdown.
    psteps = min(steps, 2000)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(L)]
           for _ in range(psteps)]
    for s in range(psteps):
        step(s, evs[s])
    torch.cuda.synchronize()
    fused = args.eps <= 0
    ph = {"score_with_append" if fused else "append": [], "score": [], "select_attend": []}
    if fused:
        del ph["score"]
    for s in range(psteps):
        for layer in range(L):
            e = evs[s][layer]
            if fused:
                ph["score_with_append"].append(e[0].elapsed_time(e[1]))
            else:
                ph["append"].append(e[0].elapsed_time(e[1]))
                ph["score"].append(e[1].elapsed_time(e[2]))
            ph["select_attend"].append(e[2].elapsed_time(e[3]))
    ph_us = {kk: 1000.0 * statistics.mean(v) for kk, v in ph.items()}
    score_ms = ph["score_with_append"] if fused else ph["score"]

    # algorithmic bytes: K once per KV head, plus the V rows of U per query head
    s1 = min(w.n_sink, N)
    w0 = max(s1, N - w.n_window)
    n_w = s1 + (N - w0)
    k_bytes = B * Hkv * N * 2 * d
    if args.eps > 0:   # the keys the threshold kept (the last step's idx; every step alike)
        kept = [int((t >= 0).sum().item()) for t in idxs]
        v_bytes_all = sum(B * Hq * n_w * 2 * d + kl * 2 * d for kl in kept)
    else:
        kept = None
        v_bytes_all = sum(B * Hq * (n_w + min(kl, w0 - s1)) * 2 * d for kl in ks)
    peak, peak_kind = measured_hbm_peak()
    score_s = statistics.mean(score_ms) / 1e3
    kscan_gbs = k_bytes / score_s / 1e9
    step_gbs = (L * k_bytes + v_bytes_all) / (ms_per_step / 1000.0) / 1e9
    src_hash = score_source_hash()
    traffic = TRAFFIC.get((src_hash, w.name))
    if args.eps > 0:   # the score kernel is inside the one timed call: the roofline is the call's
        kscan_gbs = (k_bytes + v_bytes_all / L) / score_s / 1e9
    roofline = {"kernel": ("decode_step_eps (score + select + attend)" if args.eps > 0
                           else "score_gqa_kernel (K scan)"), "bound": "hbm", "achieved": kscan_gbs,
                "peak": peak, "unit": "GB/s", "frac": kscan_gbs / peak,
                "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": k_bytes,
                "frac_of_nominal_8tbs": kscan_gbs / NOMINAL_HBM_GBS,
                "score_kernel_sha": src_hash,
                "duration_from": ("the phase pass after the timed region: CUDA events around "
                                  "each launch, on the launching stream, in the step's own "
                                  "launch configuration (in the timed step the selection runs "
                                  "beside the scan)")}
    # per layer: the scan with the append inside it, then select + attention, and the attention
    # again as a launch of its own when it is split (the library's own plan); the threshold mode
    # appends with a launch of its own
    step_launches = sum(ra.lib().ra_decode_step_launches(B, Hq, Hkv, N, d, kl, w.n_sink, w.n_window)
                        for kl in ks) + (0 if fused else L)
    result = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 / Irwin-Hall normals, Llama-3-8B-shaped caches)",
        "config": dict(workload_config(w), **({"eps": args.eps} if args.eps > 0 else {}),
                       **({"pyramid_ratio": args.pyramid, "k_per_layer": ks} if args.pyramid > 0 else {})),
        "roofline": roofline,
        "kscan_hbm_gbs": kscan_gbs,
        "step_algorithmic_gbs": step_gbs,
        "step_frac_of_peak": step_gbs / peak,
        "step_frac_of_nominal_8tbs": step_gbs / NOMINAL_HBM_GBS,
        "score_kernel_us": 1000.0 * statistics.mean(score_ms),
        "phases_us_breakdown_pass": ph_us,
        "gpu_launches": step_launches * steps,
        "clocks": clocks,
    }
    if kept is not None:
        result["kept_keys_per_head_mean"] = sum(kept) / (L * B * Hq)
        result["roofline"]["traffic"] = None

    # dense flash-decode on the same cache (decode part only is compared)
    if not args.no_dense:
        for c in caches:
            c.N = N
        dws = torch.zeros(max(ra.ra_dense_workspace_bytes(B, Hq, N, d), 256), dtype=torch.uint8, device=dev)
        dsteps = max(5, min(steps, 2000))
        for s in range(5):
            for layer in range(L):
                ra.check(ra.ra_dense_decode(caches[layer].kv, qpool[s % P, layer].data_ptr(), Hq,
                                            outs[layer].data_ptr(), dws.data_ptr(), dws.numel(), sp), "dense")
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for s in range(dsteps):
            for layer in range(L):
                ra.check(ra.ra_dense_decode(caches[layer].kv, qpool[s % P, layer].data_ptr(), Hq,
                                            outs[layer].data_ptr(), dws.data_ptr(), dws.numel(), sp), "dense")
        b.record(stream)
        torch.cuda.synchronize()
        dense_ms = max_over_ranks(dist, a.elapsed_time(b) / dsteps, dev)
        # the sparse step includes its append (inside the scan); dense decode appends nothing
        sparse_decode_ms = ms_per_step - (0.0 if fused else L * ph_us["append"] / 1000.0)
        result["dense"] = {"ms_per_step": dense_ms, "steps": dsteps,
                           "hbm_gbs": L * 2 * k_bytes / (dense_ms / 1000.0) / 1e9,
                           "speedup_of_sparse_decode": dense_ms / sparse_decode_ms}
        for c in caches:
            c.N = N - 1
        del dws

    # end to end through the C ABI's host-buffer step (the threshold mode: the Python API), the
    # step's inputs from pinned host memory and its outputs back there, waited for every step
    if not args.no_e2e:
        esteps = max(5, min(steps, 1000))
        hq = torch.empty((P, L, B, Hq, d), dtype=torch.bfloat16).pin_memory()
        hq.copy_(qpool.cpu())
        hk = [t.cpu().pin_memory() for t in knew]
        hv = [t.cpu().pin_memory() for t in vnew]
        dq = torch.empty((L, B, Hq, d), dtype=torch.bfloat16, device=dev)
        dk = [torch.empty_like(t) for t in knew]
        dv = [torch.empty_like(t) for t in vnew]
        ho = torch.empty((L, B, Hq, d), dtype=torch.float32).pin_memory()
        hi = [torch.empty((B, Hq, max(kl, 1)), dtype=torch.int32).pin_memory() for kl in ks]

        ios = [ra.ra_step_io(dq[layer].data_ptr(), dk[layer].data_ptr(), dv[layer].data_ptr(),
                             outs[layer].data_ptr(), idxs[layer].data_ptr()) for layer in range(L)]

        def e2e_step(s):
            if args.eps <= 0:
                # one C call per layer: the step's query and token rows from pinned host memory,
                # the step, and out / idx back to pinned host memory, all on the stream
                for layer in range(L):
                    ra.check(ra.ra_decode_step_append_host(
                        caches[layer].kv, hq[s % P, layer].data_ptr(), hk[layer].data_ptr(),
                        hv[layer].data_ptr(), Hq, ks[layer], w.n_sink, w.n_window,
                        ho[layer].data_ptr(), hi[layer].data_ptr(), ios[layer], ws.data_ptr(),
                        ws_bytes, sp), "decode_step_append_host")
                    caches[layer].N = N - 1
                stream.synchronize()
                return
            dq.copy_(hq[s % P], non_blocking=True)
            for layer in range(L):
                dk[layer].copy_(hk[layer], non_blocking=True)
                dv[layer].copy_(hv[layer], non_blocking=True)
                ra.append_kv(caches[layer], dk[layer], dv[layer])
                ra.decode_step_eps(caches[layer], dq[layer], ks[layer], args.eps, w.n_sink,
                                   w.n_window, out=outs[layer], idx=idxs[layer], ws=ws)
                caches[layer].N = N - 1
                ho[layer].copy_(outs[layer], non_blocking=True)
                hi[layer].copy_(idxs[layer], non_blocking=True)
            stream.synchronize()

        for s in range(3):
            e2e_step(s)
        barrier(dist, local_rank)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for s in range(esteps):
            e2e_step(s)
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(dist, a.elapsed_time(b) / esteps, dev)
        h2d = L * (B * Hq * d * 2 + 2 * B * Hkv * d * 2)
        d2h = sum(B * Hq * d * 4 + B * Hq * max(kl, 1) * 4 for kl in ks)
        result["e2e"] = {"value": world * 1000.0 / e2e_ms, "unit": "steps/s",
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": esteps,
                         "ms_per_step": e2e_ms,
                         "note": ("C ABI ra_decode_step_append_host with pinned host buffers (copies in, "
                                  "step, copies out on the stream)" if args.eps <= 0 else
                                  "public API (append_kv + decode_step_eps)") +
                                 ", host sync every step"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, spent = oracle_sample(w, args.cpu_seconds)
        result["cpu_baseline"] = {"value": v, "unit": "steps/s", "cores": cores, "kind": "oracle",
                                  "sample": desc, "sampled": True, "timed_seconds": spent}
    return result


def run_paged(args, w, rank, local_rank, world, dist):
    """Decode steps on a paged cache with ragged lengths: sequence b holds
    N - (N / 2) * b / (B - 1) tokens (rounded down to a multiple of 4), pages shuffled over the
    pool; each step appends one token per sequence and decodes (one layer)."""
    import ctypes

    import torch

    import top_retrieval_attention_b200 as ra
    from synth import device as sdev

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    B, Hq, Hkv, d, N, k = w.B, w.Hq, w.Hkv, w.d, w.N, w.k
    PAGE = 128
    lens = [max(1, (N - (N // 2) * b // max(B - 1, 1)) // 4 * 4) for b in range(B)]
    need = [(n + 1 + PAGE - 1) // PAGE for n in lens]            # room for the appended token
    num_pages, max_pages = sum(need), max(need)
    cache = ra.PagedKVCache(B, Hkv, d, num_pages, max_pages, device=dev)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    order = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.zeros((B, max_pages), dtype=torch.int32)
    j = 0
    for b in range(B):
        table[b, :need[b]] = order[j:j + need[b]]
        j += need[b]
    cache.block_table.copy_(table)
    # fill: each sequence's dense rows from the generator, scattered into its pages
    for b in range(B):
        rows = need[b] * PAGE
        Kd = torch.empty((1, Hkv, rows, d), dtype=torch.bfloat16, device=dev)
        Vd = torch.empty_like(Kd)
        sdev.fill_kv(Kd, Vd, 0, rows, w.seed + b, 0, with_offset=True)
        pages = table[b, :need[b]].to(dev).long()
        cache.K[pages] = Kd[0].view(Hkv, need[b], PAGE, d).permute(1, 0, 2, 3)
        cache.V[pages] = Vd[0].view(Hkv, need[b], PAGE, d).permute(1, 0, 2, 3)
        del Kd, Vd
    cache.set_lengths(lens)
    P = 16
    qpool = torch.empty((P, B, Hq, d), dtype=torch.bfloat16, device=dev)
    for s in range(P):
        sdev.fill_q(qpool[s], w.seed + 7919 * s)
    knew = torch.zeros((B, Hkv, 1, d), dtype=torch.bfloat16, device=dev)
    vnew = torch.zeros_like(knew)
    ws_bytes = ra.lib().ra_paged_workspace_bytes(B, Hq, max(lens) + 1, d, k, w.n_sink, w.n_window)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Hq, k), dtype=torch.int32, device=dev)

    def step(s):
        ra.check(ra.lib().ra_paged_append_kv(ctypes.byref(cache.kv), knew.data_ptr(),
                                             vnew.data_ptr(), 1, sp), "paged_append")
        ra.check(ra.lib().ra_paged_decode_step(ctypes.byref(cache.kv), qpool[s % P].data_ptr(), Hq,
                                               k, w.n_sink, w.n_window, out.data_ptr(),
                                               idx.data_ptr(), ws.data_ptr(), ws_bytes, sp),
                 "paged_decode")
        cache.set_lengths(lens)   # the next step re-appends into the same slot

    for s in range(max(3, args.warmup)):
        step(s)
    torch.cuda.synchronize()
    steps = args.steps if args.steps is not None else 200
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    clk = Clocks(uuid)
    clk.start()
    barrier(dist, local_rank)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        step(s)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(dist, local_rank)
    clocks = clk.stop()
    ms = max_over_ranks(dist, t0.elapsed_time(t1), dev) / steps
    n1 = [n + 1 for n in lens]
    k_bytes = sum(Hkv * n * 2 * d for n in n1)
    v_bytes = 0
    for n in n1:
        s1 = min(w.n_sink, n)
        w0 = max(s1, n - w.n_window)
        v_bytes += Hq * (s1 + n - w0 + min(k, w0 - s1)) * 2 * d
    peak, peak_kind = measured_hbm_peak()
    gbs = (k_bytes + v_bytes) / (ms / 1000.0) / 1e9
    return {
        "metric": METRIC + " (paged, ragged lengths)", "value": world * 1000.0 / ms,
        "unit": "steps/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 / Irwin-Hall normals), pages shuffled",
        "config": dict(workload_config(w), paged=True, page_tokens=PAGE, lengths=lens),
        "roofline": {"kernel": "paged decode step (score + select + attend)", "bound": "hbm",
                     "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": None, "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": k_bytes + v_bytes},
        "gpu_launches": 3 * steps, "clocks": clocks,
    }


def run_ivf(args, w, rank, local_rank, world, dist):
    """Decode steps retrieving through an IVF index of the keys built on the device (spherical
    k-means, `--ivf` clusters per KV head, `--nprobe` probed per query head), one layer of the
    workload.  The index covers the N - 1 cached keys; each step appends the N-th token (served by
    the window) and decodes.  Beside the throughput: the build time, the fraction of candidate
    keys scored, and Recall@k of the IVF selection against the exact top-k of the same step."""
    import ctypes

    import torch

    import top_retrieval_attention_b200 as ra
    from synth import device as sdev

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    B, Hq, Hkv, d, N, k, G = w.B, w.Hq, w.Hkv, w.d, w.N, w.k, w.G
    nlist, nprobe = args.ivf, args.nprobe
    c = ra.KVCache(B, Hkv, d, N, device=dev)
    sdev.device_layer(w, 0, c.K, c.V)
    knew = c.K[:, :, N - 1:N].clone()
    vnew = c.V[:, :, N - 1:N].clone()
    c.N = N - 1
    P = 16
    qpool = torch.empty((P, B, Hq, d), dtype=torch.bfloat16, device=dev)
    for s in range(P):
        sdev.fill_q(qpool[s], w.seed + 7919 * s)

    # the build: once untimed (kernel loading), then timed with events
    ix = ra.ivf_build(c, nlist, args.ivf_iters)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    ix = ra.ivf_build(c, nlist, args.ivf_iters)
    b.record(stream)
    torch.cuda.synchronize()
    build_ms = a.elapsed_time(b)

    n = ra.lib().ra_ivf_search_workspace_bytes(B, Hq, N, d, k, nprobe)
    if n == 0:
        raise SystemExit(f"IVF search shape rejected (nprobe {nprobe}, nlist {nlist})")
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Hq, max(k, 1)), dtype=torch.int32, device=dev)

    def step(s):
        ra.check(ra.ra_append_kv(c.kv, knew.data_ptr(), vnew.data_ptr(), 1, sp), "append")
        ra.check(ra.lib().ra_ivf_decode_step(ctypes.byref(c.kv), ctypes.byref(ix.ix),
                                             qpool[s % P].data_ptr(), Hq, k, nprobe, w.n_sink,
                                             w.n_window, out.data_ptr(), idx.data_ptr(),
                                             ws.data_ptr(), n, sp), "ivf_decode")
        c.N = N - 1

    # quality: Recall@k of every query of the pool against the exact step's selection, and the
    # keys each query head scores (its probed clusters' sizes; diagnostic arithmetic in torch)
    ews = torch.zeros(ra.ra_decode_workspace_bytes(B, Hq, N, d, k, w.n_sink, w.n_window),
                      dtype=torch.uint8, device=dev)
    hits = total = 0
    scanned = []
    sizes = (ix.offsets[..., 1:] - ix.offsets[..., :-1]).float()            # [B, Hkv, nlist]
    for s in range(P):
        step(s)
        ra.check(ra.ra_append_kv(c.kv, knew.data_ptr(), vnew.data_ptr(), 1, sp), "append")
        _, ex = ra.decode_step(c, qpool[s], k, w.n_sink, w.n_window, ws=ews)
        c.N = N - 1
        got = idx[..., :k]
        for bb in range(B):
            for h in range(Hq):
                e = ex[bb, h][ex[bb, h] >= 0]
                hits += int(torch.isin(e, got[bb, h]).sum().item())
                total += int(e.numel())
        zc = torch.einsum("bgcd,bghd->bghc", ix.centroids.float(),
                          qpool[s].float().view(B, Hkv, G, d))
        top = zc.topk(nprobe, dim=-1).indices                                # [B, Hkv, G, nprobe]
        sz = torch.gather(sizes.unsqueeze(2).expand(B, Hkv, G, nlist), 3, top).sum(-1)
        scanned.append(sz.mean().item())
    torch.cuda.synchronize()
    recall = hits / max(total, 1)
    cand_per_head = statistics.mean(scanned)

    for s in range(max(3, args.warmup)):
        step(s)
    torch.cuda.synchronize()
    steps = args.steps if args.steps is not None else 1000
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    clk = Clocks(uuid)
    clk.start()
    barrier(dist, local_rank)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")   # lets a profiler keep to the timed steps
    t0.record(stream)
    for s in range(steps):
        step(s)
    t1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(dist, local_rank)
    clocks = clk.stop()
    ms = max_over_ranks(dist, t0.elapsed_time(t1), dev) / steps

    # the exact step on the same cache, for the speedup
    for s in range(5):
        ra.check(ra.ra_append_kv(c.kv, knew.data_ptr(), vnew.data_ptr(), 1, sp), "append")
        ra.decode_step(c, qpool[s % P], k, w.n_sink, w.n_window, ws=ews)
        c.N = N - 1
    a.record(stream)
    for s in range(steps):
        ra.check(ra.ra_append_kv(c.kv, knew.data_ptr(), vnew.data_ptr(), 1, sp), "append")
        ra.decode_step(c, qpool[s % P], k, w.n_sink, w.n_window, ws=ews)
        c.N = N - 1
    b.record(stream)
    torch.cuda.synchronize()
    exact_ms = max_over_ranks(dist, a.elapsed_time(b), dev) / steps

    # algorithmic bytes per step, per query head: the centroids, the probed clusters' keys, the
    # static set's keys, and the V rows of U
    s1 = min(w.n_sink, N)
    w0 = max(s1, N - w.n_window)
    n_w = s1 + (N - w0)
    row = 2 * d
    alg = B * Hq * (nlist * row + cand_per_head * row + n_w * row + (n_w + min(k, w0 - s1)) * row)
    peak, peak_kind = measured_hbm_peak()
    gbs = alg / (ms / 1000.0) / 1e9
    return {
        "metric": "IVF-retrieval decode steps/s (device-built index, probed top-k)",
        "value": world * 1000.0 / ms, "unit": "steps/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 / Irwin-Hall normals, Llama-3-8B-shaped cache)",
        "config": dict(workload_config(w), layers=1, nlist=nlist, nprobe=nprobe,
                       kmeans_iters=args.ivf_iters),
        "roofline": {"kernel": "IVF decode step (probe + candidate scores + select + attend)",
                     "bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "traffic": None, "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": alg},
        "recall_at_k": recall, "scanned_fraction": cand_per_head / N,
        "candidates_per_query_head": cand_per_head, "build_ms": build_ms,
        "exact_step_ms": exact_ms, "speedup_over_exact": exact_ms / ms,
        # append, probe, candidate scores, selection fused with the attention (one more launch
        # only when the attention is split across clusters, which takes far more than k = 100)
        "gpu_launches": 4 * steps, "clocks": clocks,
    }


def run_prefill(args, w, rank, local_rank, world, dist):
    """Exact top-k of M prefill queries per query head against one layer's cache: the
    tcgen05 score GEMM (timed on its own for its roofline) and the cluster selection."""
    import ctypes

    import torch

    import top_retrieval_attention_b200 as ra
    from synth import device as sdev

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    M = args.prefill_queries
    B, Hq, Hkv, d, N, k = w.B, w.Hq, w.Hkv, w.d, w.N, w.k
    c = ra.KVCache(B, Hkv, d, N, device=dev)
    sdev.device_layer(w, 0, c.K, c.V)
    c.N = N
    P = 4
    qpool = torch.empty((P, B, Hq, M, d), dtype=torch.bfloat16, device=dev)
    for s in range(P):
        sdev.fill_q(qpool[s].view(B, Hq * M, d), w.seed + 7919 * s + 31)
    n = ra.ra_prefill_workspace_bytes(B, Hq, M, N, d, k, w.n_sink, w.n_window)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    idx = torch.empty((B, Hq, M, max(k, 1)), dtype=torch.int32, device=dev)

    def step(s, ev=None):
        q = qpool[s % P].data_ptr()
        if ev is not None:
            ev[0].record(stream)
        ra.check(ra.ra_prefill_score(c.kv, q, Hq, M, k, w.n_sink, w.n_window, ws.data_ptr(), n, sp),
                 "prefill_score")
        if ev is not None:
            ev[1].record(stream)
        ra.check(ra.ra_prefill_select(c.kv, Hq, M, k, w.n_sink, w.n_window, idx.data_ptr(),
                                      ws.data_ptr(), n, sp), "prefill_select")
        if ev is not None:
            ev[2].record(stream)

    for s in range(max(3, args.warmup)):
        step(s)
    torch.cuda.synchronize()
    steps = args.steps if args.steps is not None else 20
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    clk = Clocks(uuid)
    clk.start()
    barrier(dist, local_rank)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        step(s, evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(dist, local_rank)
    clocks = clk.stop()
    ms = max_over_ranks(dist, t0.elapsed_time(t1), dev) / steps
    score_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    select_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    R = B * Hq * M
    flops = 2.0 * R * N * d
    s_bytes = 4.0 * R * N
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            peaks = json.load(fh)
    except Exception:
        peaks = {}
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    tflops_peak = float(peaks.get("bf16_tflops", 1590.0))
    return {
        "metric": "prefill exact top-k queries/s (tcgen05 scores + cluster select)",
        "value": world * R / (ms / 1000.0), "unit": "queries/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 / Irwin-Hall normals, Llama-3-8B-shaped cache)",
        "config": dict(workload_config(w), prefill_queries_per_head=M, rows=R),
        "roofline": {"kernel": "prefill_score_kernel (tcgen05)", "bound": "hbm",
                     "achieved": s_bytes / (score_ms / 1000.0) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": s_bytes / (score_ms / 1000.0) / 1e9 / hbm_peak,
                     "traffic": None, "algorithmic_bytes_per_launch": s_bytes,
                     "tensor_tflops": flops / (score_ms / 1000.0) / 1e12,
                     "tensor_frac_of_bf16_peak": flops / (score_ms / 1000.0) / 1e12 / tflops_peak},
        "score_kernel_us": 1000.0 * score_ms, "select_us": 1000.0 * select_ms,
        "gpu_launches": 2 * steps, "clocks": clocks,
    }


# The other workloads of the decode-step suite reported in the default line (the 32-layer 1M
# cache and the batch-16 256K layer), each measured in this same run the way the headline is.
EXTRA_CONFIGS = ("l8b_1m_32layer", "l8b_b16_256k")


def extra_configs(args, rank, local_rank, world, dist):
    import copy
    import gc

    import torch

    from synth import gen
    out = {}
    for name in EXTRA_CONFIGS:
        a = copy.copy(args)
        a.steps, a.warmup, a.no_e2e, a.no_cpu_baseline = None, 3, True, True
        r = run_ours(a, gen.workload(name), rank, local_rank, world, dist)
        out[name] = {k: r[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup",
                                       "step_frac_of_peak", "step_frac_of_nominal_8tbs",
                                       "score_kernel_us", "gpu_launches", "clocks", "config")}
        out[name]["score_kernel_frac_of_peak"] = r["roofline"]["frac"]
        if "dense" in r:
            out[name]["dense_ms_per_step"] = r["dense"]["ms_per_step"]
            out[name]["speedup_over_dense"] = r["dense"]["speedup_of_sparse_decode"]
        gc.collect()
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank, local_rank, world = dist_info()
    from synth import gen
    w = gen.workload(args.workload)
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product has no CPU path)")
    dist = dist_init(world, True)
    try:
        if args.sweep:
            import gc
            args.no_e2e = True
            args.no_cpu_baseline = True
            for name in gen.sweep_names():
                res = run_ours(args, gen.workload(name), rank, local_rank, world, dist)
                if rank == 0:
                    print(json.dumps(res), flush=True)
                gc.collect()
                torch.cuda.empty_cache()
            return
        if args.prefill_queries > 0:
            res = run_prefill(args, w, rank, local_rank, world, dist)
        elif args.ivf > 0:
            res = run_ivf(args, w, rank, local_rank, world, dist)
        elif args.paged:
            res = run_paged(args, w, rank, local_rank, world, dist)
        else:
            res = run_ours(args, w, rank, local_rank, world, dist)
            if (world == 1 and not args.no_configs and args.workload == DEFAULT_WORKLOAD and
                    args.eps <= 0 and args.pyramid <= 0):
                res["configs"] = extra_configs(args, rank, local_rank, world, dist)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
