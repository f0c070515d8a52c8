#!/usr/bin/env python
"""Throughput of the Recurrent Transformer layer forward (prefill) on B200.

One step = one rt_layer_forward of the whole layer (batched projection, N
sequential steps of finalise -> W_o -> MLP -> persistent K/V projection, and
the lowbit block folds) over one batch of synthetic input already resident
in HBM. Metric: tokens/s = B*N / step time, summed over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload headline|small] [--schedule blocked|naive]

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch of
B sequences with replicated weights (sequences are independent: weak scaling,
no collective on the data path). Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # the pages' single-layer setting (batch 512, width 1024, 16 heads) at N = 2048
    "headline": dict(B=512, N=2048, d=1024, H=16, d_ff=4096),
    "small": dict(B=64, N=1024, d=512, H=8, d_ff=2048),
}
METRIC = "RT-layer prefill tokens/s (B=512,N=2048,d=1024 bf16); % of roofline"

# DRAM traffic per launch from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum of one launch), keyed by (kernel class, workload, hash
# of the CUDA sources at capture time); reported as null once the sources
# change.
NCU_TRAFFIC: dict = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one W_2 GEMM launch at the
    # headline shapes (B = 512, d = 1024, d_ff = 4096), valid for these sources
    ("gemm_w2", "headline", "915c9863cec9"): 14723328,
}


def src_hash() -> str:
    h = hashlib.sha1()
    for f in sorted(glob.glob(os.path.join(ROOT, "blocked_attention_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:12]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="headline")
    ap.add_argument("--schedule", choices=["blocked", "naive"], default="blocked")
    ap.add_argument("--driver", choices=["graph", "stream", "persistent"], default="graph")
    ap.add_argument("--no-drivers", action="store_true",
                    help="skip timing the headline with the other step-loop driver")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ablation", action="store_true", help="skip the naive-schedule ablation")
    ap.add_argument("--ablation-steps", type=int, default=1)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--decode", action="store_true",
                    help="time the autoregressive decode step (B sequences, one new position against a cache)")
    ap.add_argument("--decode-t", type=int, default=0, help="decoded position (default: the workload's N)")
    ap.add_argument("--stack", action="store_true",
                    help="6-layer stack with token embedding (B=64 N=2048 d=1280 H=20x64 d_ff=5120)")
    ap.add_argument("--sweep", action="store_true",
                    help="sequence-length sweep, blocked vs naive (B=32 d=1024 H=16x64 d_ff=4096)")
    ap.add_argument("--sweep-n", default="512,1024,2048,4096,8192,16384")
    ap.add_argument("--pages", action="store_true",
                    help="the paper's own parameterisation (rt_layer_forward_pages) at the workload's shape")
    ap.add_argument("--chunked", type=int, default=0, metavar="C",
                    help="the block-wise recurrence with chunks of C positions at the workload's shape")
    ap.add_argument("--recompute", action="store_true",
                    help="activation-checkpoint recompute of K, V from z over all B*N rows")
    ap.add_argument("--backward", action="store_true",
                    help="backward pass (bf16 storage) at B=64 N=1024 d=512 H=8x64 d_ff=2048")
    ap.add_argument("--profile-case", choices=["step", "persistent", "fold", "fwd", "naive"],
                    help="run one small case for an ncu capture and exit: 'step' = one host-loop forward at "
                         "B=512 N=64 d=1024 (the per-step GEMM shapes of the headline); 'persistent' = the same "
                         "forward with the persistent step kernel; 'fold' = one block fold "
                         "of --lb keys into --lb queries at B=--pB H=16 (position-major); 'fwd' = one "
                         "graph-driver forward at the headline widths with N = --lb; 'naive' = one host-loop "
                         "naive-schedule forward at B=--pB, N=--lb, d=1024 H=16x64 d_ff=4096")
    ap.add_argument("--lb", type=int, default=1024)
    ap.add_argument("--pB", type=int, default=64, help="batch of the 'fold' and 'naive' profile cases")
    return ap.parse_args()


# --------------------------------------------------------------------------
# multi-rank helpers (replicas: no collective on the data path)
# --------------------------------------------------------------------------
def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank scalar (the device-timed step time) over all ranks."""
    import torch
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_input_seed(seed: int, rank: int) -> int:
    """Each replica draws its own batch."""
    return 1000 + 1000 * seed + rank


def aggregate_tokens_per_s(world: int, B: int, N: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes B*N tokens per step."""
    return world * B * N / (ms_per_step / 1e3)


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, flag in zip(names, f[5:9]):
                if flag.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(torch, dev: int) -> str | None:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev] if vis else str(dev)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------
# algorithmic work of each kernel class (per forward)
# --------------------------------------------------------------------------
def lowbit(t: int) -> int:
    return t & -t


def algorithmic_work(cfg: dict, schedule: str = "blocked") -> dict:
    """{class: ("tensor", flops) | ("hbm", bytes)} summed over one forward."""
    B, N, d, H, dff = cfg["B"], cfg["N"], cfg["d"], cfg["H"], cfg["d_ff"]
    w = {
        "proj": ("tensor", 2.0 * B * N * d * 3 * d),
        "gemm_wo": ("tensor", 2.0 * B * d * d * N),
        "gemm_w1": ("tensor", 2.0 * B * d * dff * N),
        "gemm_w2": ("tensor", 2.0 * B * dff * d * N),
        "gemm_wkv": ("tensor", 2.0 * B * d * 2 * d * N),
        "inv_rms": ("hbm", 2.0 * B * N * d + 4.0 * B * N),
        # blocked: only position 1 is finalised by this class (every later
        # position by the last fold into it): q, k~, v~ read, a_1 written (bf16)
        "attend": ("hbm", float(B) * (6 * d + 2 * d)),
    }
    # the persistent step kernel: the four per-step GEMMs of every step (its
    # small folds are accounted in fold_level_work)
    w["steps"] = ("tensor", 2.0 * B * N * (d * d + 2 * d * dff + 2 * d * d))
    if schedule == "naive":
        # query t reads the t-1 persistent pairs (k, v bf16) plus its own q, k~, v~; writes a_t
        w["attend"] = ("hbm", float(B) * (4 * d * N * (N - 1) / 2 + N * 8 * d))
        return w
    warp_b, mma_b = 0.0, 0.0
    for lb, (by, fl) in fold_level_work(cfg).items():
        if lb >= 16:
            mma_b += by
        else:
            warp_b += by
    w["fold_warp"] = ("hbm", warp_b)
    w["fold_tensor"] = ("hbm", mma_b)
    return w


def fold_level_work(cfg: dict) -> dict:
    """{block size: (algorithmic bytes, FLOPs)} of the folds of one forward.
    Bytes per fold: every key's k, v (bf16) read once; every query's q (bf16)
    read and its o (fp32), m, l read and written -- written only for the first
    fold into a query (t a power of two). FLOPs: QK^T and PV, 4 d per pair."""
    B, N, d, H = cfg["B"], cfg["N"], cfg["d"], cfg["H"]
    out = {}
    for t in range(1, N):
        lb = lowbit(t)
        nq = min(lb, N - t)
        init = (t == lb)
        per_q = 2 * d + (4 * d if init else 8 * d) + (8 * H if init else 16 * H)
        by = B * (nq * per_q + lb * 4 * d)
        fl = 4.0 * B * d * nq * lb
        b0, f0 = out.get(lb, (0.0, 0.0))
        out[lb] = (b0 + by, f0 + fl)
    return out


# --------------------------------------------------------------------------
# the oracle as the CPU baseline / reference arm
# --------------------------------------------------------------------------
def blas_threads() -> int:
    """Threads of numpy's BLAS pool: the threads the oracle's matrix products use."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# The oracle's timed sample: a subset of the workload's sequences at the full
# sequence length. Sequences are independent, so the whole batch costs the
# sample's time x B / ORACLE_SEQS and tokens/s is the sample's own.
ORACLE_SEQS = 1


def time_oracle(cfg: dict, n_seq: int, seed: int) -> tuple[float, float]:
    """Runs the fp64 oracle (naive definition) on the first n_seq sequences of
    the workload at its full length N; returns (tokens/s, seconds)."""
    import rtinputs
    from oracle import rt_oracle
    W = rtinputs.weights(seed, cfg["d"], cfg["d_ff"], dtype="bf16")
    x = rtinputs.x_batch(seed, range(n_seq), cfg["N"], cfg["d"], dtype="bf16")
    t0 = time.perf_counter()
    rt_oracle.rt_layer(x, W, cfg["H"])
    dt = time.perf_counter() - t0
    return n_seq * cfg["N"] / dt, dt


def oracle_sample_text(cfg: dict, secs: float | None = None) -> str:
    t = f"; {secs:.1f} s" if secs is not None else ""
    return (f"{ORACLE_SEQS} of the {cfg['B']} sequences at the full N={cfg['N']} (fp64 numpy oracle, naive "
            f"schedule{t}); the whole batch takes B/{ORACLE_SEQS} times as long (sequences are independent)")


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    cfg = WORKLOADS[args.workload]
    for _ in range(args.warmup):
        time_oracle(cfg, ORACLE_SEQS, args.seed)
    secs = [time_oracle(cfg, ORACLE_SEQS, args.seed)[1] for _ in range(args.steps)]
    sample_s = sum(secs) / len(secs)
    value = ORACLE_SEQS * cfg["N"] / sample_s
    ms = 1e3 * sample_s * cfg["B"] / ORACLE_SEQS      # one step of the whole workload
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "nproc": os.cpu_count(),
                         "kind": "oracle", "sample": oracle_sample_text(cfg, sample_s)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def workload_config(args, cfg, world) -> dict:
    return {"workload": (f"RT layer prefill forward, B={cfg['B']} N={cfg['N']} d={cfg['d']} "
                         f"H={cfg['H']}x{cfg['d'] // cfg['H']} d_ff={cfg['d_ff']}"),
            **cfg, "schedule": args.schedule, "driver": args.driver,
            "global_batch": cfg["B"] * world, "seq_len": cfg["N"],
            "parallelism": f"replicas x{world} (batch-sharded, no collective)",
            "l2": "inputs larger than L2 (x 2.1 GB, o 4.3 GB, K/V 4.3 GB per step > 126 MB)"}


# --------------------------------------------------------------------------
STACK = dict(B=64, N=2048, d=1280, H=20, d_ff=5120, layers=6, vocab=32000)
SWEEP = dict(B=32, d=1024, H=16, d_ff=4096)


def run_stack(args, R, torch, rtinputs):
    """Tokens/s of the 6-layer stack: embedding gather, then 6 layer forwards,
    each layer's z feeding the next (one step = the whole stack)."""
    c = STACK
    dev = torch.device("cuda", 0)
    Bsz, N, d, H, dff, L = c["B"], c["N"], c["d"], c["H"], c["d_ff"], c["layers"]
    E = torch.randn((c["vocab"], d), device=dev, dtype=torch.bfloat16) * 0.02
    ids = torch.randint(0, c["vocab"], (Bsz, N), device=dev, dtype=torch.int32)
    Ws = [{k: torch.from_numpy(v.astype("float32")).to(dev, torch.bfloat16)
           for k, v in rtinputs.weights(args.seed, d, dff, dtype="bf16", layer=i).items()} for i in range(L)]
    xs = [torch.empty((Bsz, N, d), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    KV = [(torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev),
           torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev)) for _ in range(L)]
    ws = R.alloc_workspace(R.workspace_bytes(Bsz, N, d, H, dff), dev)

    def step():
        x0 = R.embed_forward(ids, E, workspace=ws)
        xs[0].copy_(x0)
        for i in range(L):
            R.layer_forward(xs[i % 2], Ws[i], H, out=(xs[(i + 1) % 2], KV[i][0], KV[i][1]), workspace=ws)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    assert R.sync_status(ws) == 0
    print(json.dumps({"metric": "RT 6-layer stack prefill tokens/s", "value": Bsz * N / (ms / 1e3),
                      "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
                      "dtype": "bf16", "data": "synthetic", "config": {"workload": "6-layer RT stack", **c}}),
          flush=True)


def run_decode(args, R, torch, rtinputs):
    """Tokens/s of the decode step at the workload's widths: B sequences each
    produce one new position t against a cache of t - 1 persistent pairs (one
    step = one rt_layer_decode_step; the same position is re-decoded every
    step, overwriting cache row t - 1)."""
    cfg = WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    Bsz, N, d, H, dff = cfg["B"], cfg["N"], cfg["d"], cfg["H"], cfg["d_ff"]
    t = args.decode_t or N
    W = {k: torch.from_numpy(v.astype("float32")).to(dev, torch.bfloat16)
         for k, v in rtinputs.weights(args.seed, d, dff, dtype="bf16").items()}
    Kc = torch.randn((t, Bsz, d), device=dev, dtype=torch.bfloat16)
    Vc = torch.randn((t, Bsz, d), device=dev, dtype=torch.bfloat16)
    xt = torch.randn((Bsz, d), device=dev, dtype=torch.bfloat16)
    z = torch.empty_like(xt)
    ws = R.alloc_workspace(R.decode_workspace_bytes(Bsz, d, H, dff), dev)

    def step():
        R.layer_decode_step(xt, W, H, t, Kc, Vc, out=z, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    assert R.sync_status(ws) == 0
    kv_bytes = 2 * (t - 1) * Bsz * d * 2          # the cached keys and values read once
    print(json.dumps({"metric": "RT layer decode tokens/s", "value": Bsz / (ms / 1e3), "unit": "tokens/s",
                      "ms_per_step": ms, "steps": args.steps, "warmup": max(args.warmup, 3), "dtype": "bf16",
                      "data": "synthetic", "cache_read_GBps": kv_bytes / (ms / 1e3) / 1e9,
                      "config": {"workload": f"decode position {t}, B={Bsz} d={d} H={H}x{d // H} d_ff={dff}",
                                 "B": Bsz, "t": t, "d": d, "H": H, "d_ff": dff}}), flush=True)


def run_sweep(args, R, torch):
    """Sequence-length sweep, blocked vs naive schedule: latency per forward."""
    c = SWEEP
    dev = torch.device("cuda", 0)
    Bsz, d, H, dff = c["B"], c["d"], c["H"], c["d_ff"]
    W = {k: (torch.randn(v, device=dev) * 0.02).to(torch.bfloat16) for k, v in
         {"W_q": (d, d), "W_k": (d, d), "W_v": (d, d), "W_o": (d, d), "W_1": (dff, d), "W_2": (d, dff)}.items()}
    for N in [int(v) for v in args.sweep_n.split(",")]:
        x = torch.randn((Bsz, N, d), device=dev, dtype=torch.bfloat16)
        out = (torch.empty_like(x), torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev),
               torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev))
        for sched in ("blocked", "naive"):
            ws = R.alloc_workspace(R.workspace_bytes(Bsz, N, d, H, dff, torch.bfloat16, sched), dev)
            steps = 1 if (sched == "naive" and N >= 8192) else 2
            R.layer_forward(x, W, H, schedule=sched, out=out, workspace=ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                R.layer_forward(x, W, H, schedule=sched, out=out, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            assert R.sync_status(ws) == 0
            print(json.dumps({"sweep": True, "N": N, "schedule": sched, "ms_per_forward": ms,
                              "tokens_per_s": Bsz * N / (ms / 1e3), **c}), flush=True)
            del ws
            torch.cuda.empty_cache()


def _timed(torch, fn, steps: int, warmup: int) -> float:
    """ms per call of fn on the current stream (CUDA events), after warm-up."""
    for _ in range(max(warmup, 1)):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_next_rows(args, R, torch, rtinputs):
    """Measurements of the rows beyond the forward: the paper's own
    parameterisation, the block-wise recurrence, the checkpoint recompute
    and the backward pass. One JSON line each."""
    dev = torch.device("cuda", 0)
    peaks = measured_peaks()
    if args.backward:
        Bsz, N, d, H, dff = 64, 1024, 512, 8, 2048
    else:
        c = WORKLOADS[args.workload]
        Bsz, N, d, H, dff = c["B"], c["N"], c["d"], c["H"], c["d_ff"]
    W = {k: torch.from_numpy(v.astype("float32")).to(dev, torch.bfloat16)
         for k, v in rtinputs.weights(args.seed, d, dff, dtype="bf16").items()}
    x = torch.randn((Bsz, N, d), device=dev, dtype=torch.bfloat16)
    shape = {"B": Bsz, "N": N, "d": d, "H": H, "d_ff": dff}
    line = {"dtype": "bf16", "data": "synthetic", "steps": args.steps, "warmup": args.warmup}
    if args.pages or args.chunked:
        out = (torch.empty_like(x), torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev),
               torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev))
        if args.pages:
            ws = R.alloc_workspace(R.workspace_bytes(Bsz, N, d, H, dff), dev)
            fn = lambda: R.layer_forward_pages(x, W, H, 1, out=out, workspace=ws)
            name, extra = "RT-layer prefill tokens/s, the paper's own parameterisation", {}
        else:
            ws = R.alloc_workspace(int(R.lib().rt_layer_chunked_workspace_bytes(Bsz, N, d, H, dff, args.chunked)), dev)
            fn = lambda: R.layer_forward_chunked(x, W, H, args.chunked, out=out, workspace=ws)
            name, extra = "RT-layer prefill tokens/s, block-wise recurrence", {"chunk": args.chunked}
        ms = _timed(torch, fn, args.steps, args.warmup)
        assert R.sync_status(ws) == 0
        flops = 2.0 * Bsz * N * (6 * d * d + 2 * d * dff) + 4.0 * Bsz * d * N * (N + 1) / 2
        line.update({"metric": name, "value": Bsz * N / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
                     "tflops": flops / (ms / 1e3) / 1e12, "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 /
                     peaks["bf16_tflops"], "config": {"workload": "RT layer forward", **shape, **extra}})
    elif args.recompute:
        z = x
        K = torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev)
        V = torch.empty_like(K)
        ws = R.alloc_workspace(int(R.lib().rt_layer_recompute_workspace_bytes(Bsz, N, d)), dev)
        ms = _timed(torch, lambda: R.recompute_kv(z, W["W_k"], W["W_v"], out=(K, V), workspace=ws), args.steps,
                    args.warmup)
        assert R.sync_status(ws) == 0
        flops = 2.0 * Bsz * N * d * 2 * d
        line.update({"metric": "checkpoint recompute of K, V from z, tokens/s", "value": Bsz * N / (ms / 1e3),
                     "unit": "tokens/s", "ms_per_step": ms, "tflops": flops / (ms / 1e3) / 1e12,
                     "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                     "config": {"workload": "recompute", **shape}})
    else:
        z, K, V = R.layer_forward(x, W, H)
        dz, dK, dV = torch.randn_like(z), torch.randn_like(K), torch.randn_like(V)
        ws = R.alloc_workspace(int(R.lib().rt_layer_backward_workspace_bytes(Bsz, N, d, H, dff, R.RT_BF16)), dev)
        ms = _timed(torch, lambda: R.layer_backward(x, W, H, z, K, V, dz, dK, dV, workspace=ws), args.steps,
                    args.warmup)
        line.update({"metric": "RT-layer backward tokens/s (bf16 storage, fp32 arithmetic)",
                     "value": Bsz * N / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
                     "config": {"workload": "backward", **shape}})
    print(json.dumps(line), flush=True)


def run_profile_case(args, R, torch, rtinputs):
    dev = torch.device("cuda", 0)
    if args.profile_case in ("step", "persistent", "fwd"):
        B, N, d, H, dff = 512, (args.lb if args.profile_case == "fwd" else 64), 1024, 16, 4096
        W = {k: torch.from_numpy(v.astype("float32")).to(dev, torch.bfloat16)
             for k, v in rtinputs.weights(args.seed, d, dff, dtype="bf16").items()}
        x = torch.randn((B, N, d), device=dev, dtype=torch.bfloat16)
        drv = {"step": "stream", "persistent": "persistent", "fwd": "graph"}[args.profile_case]
        z, _, _ = R.layer_forward(x, W, H, driver=drv)
    elif args.profile_case == "naive":
        B, N, d, H, dff = args.pB, args.lb, 1024, 16, 4096
        W = {k: torch.from_numpy(v.astype("float32")).to(dev, torch.bfloat16)
             for k, v in rtinputs.weights(args.seed, d, dff, dtype="bf16").items()}
        x = torch.randn((B, N, d), device=dev, dtype=torch.bfloat16)
        z, _, _ = R.layer_forward(x, W, H, schedule="naive", driver="stream")
    else:
        LB, B, H, dh = args.lb, args.pB, 16, 64
        d = H * dh
        Q = torch.randn((2 * LB, B, 3 * d), device=dev, dtype=torch.bfloat16)
        Kc = torch.randn((2 * LB, B, d), device=dev, dtype=torch.bfloat16)
        Vc = torch.randn((2 * LB, B, d), device=dev, dtype=torch.bfloat16)
        m = torch.zeros((2 * LB, B, H), device=dev)
        l = torch.ones((2 * LB, B, H), device=dev)
        z = torch.zeros((2 * LB, B, d), device=dev)
        R.block_fold(Q, Kc, Vc, m, l, z, H, dh, LB, LB, 0, LB)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile_case, "ok": bool(torch.isfinite(z.float()).all())}))


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    from blocked_attention_b200 import build as B
    B.build()
    from blocked_attention_b200 import rtlayer as R
    import rtinputs

    torch.cuda.set_device(local)
    if args.profile_case:
        run_profile_case(args, R, torch, rtinputs)
        return
    if args.decode:
        run_decode(args, R, torch, rtinputs)
        return
    if args.pages or args.chunked or args.recompute or args.backward:
        run_next_rows(args, R, torch, rtinputs)
        return
    if args.stack or args.sweep:
        (run_stack(args, R, torch, rtinputs) if args.stack else run_sweep(args, R, torch))
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    cfg = WORKLOADS[args.workload]
    Bsz, N, d, H, dff = cfg["B"], cfg["N"], cfg["d"], cfg["H"], cfg["d_ff"]
    dev = torch.device("cuda", local)

    Wnp = rtinputs.weights(args.seed, d, dff, dtype="bf16")
    W = {k: torch.from_numpy(v.astype("float32")).to(dev, torch.bfloat16) for k, v in Wnp.items()}
    g = torch.Generator(device=dev)
    g.manual_seed(rank_input_seed(args.seed, rank))
    x = torch.randn((Bsz, N, d), generator=g, device=dev, dtype=torch.bfloat16)
    z = torch.empty_like(x)
    K = torch.empty((N, Bsz, d), dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    ws = R.alloc_workspace(R.workspace_bytes(Bsz, N, d, H, dff, torch.bfloat16, args.schedule), dev)

    def step():
        R.layer_forward(x, W, H, schedule=args.schedule, driver=args.driver, out=(z, K, V), workspace=ws)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    st = R.sync_status(ws)
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {R.status_string(st)}")

    sampler = ClockSampler(gpu_id_for(torch, local))
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms_total = e0.elapsed_time(e1)
    if world > 1:
        ms_total = max_over_ranks(ms_total, dist, dev)
    st = R.sync_status(ws)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {R.status_string(st)}")
    ms_step = ms_total / args.steps
    value = aggregate_tokens_per_s(world, Bsz, N, ms_step)

    # per-kernel device time: one extra forward with CUDA events around every kernel
    classes = R.layer_forward_timed(x, W, H, (z, K, V), ws, schedule=args.schedule)
    work = algorithmic_work(cfg, args.schedule)
    peaks = measured_peaks()
    # a kernel timed at full clocks is compared with the burst GEMM peak; if
    # the power cap throttled the timed region, with the sustained one
    tensor_key = "bf16_tflops_sustained" if "sw_power_cap" in clocks.get("reasons", []) else "bf16_tflops"
    kernels, fold_levels = {}, {}
    lvl_work = fold_level_work(cfg) if args.schedule == "blocked" else {}
    for name, (kms, launches) in classes.items():
        if name.startswith("fold_lb"):
            lb = int(name[7:])
            by, fl = lvl_work.get(lb, (0.0, 0.0))
            fold_levels[lb] = {"ms_total": round(kms, 3), "launches": launches,
                               "GB/s": by / (kms / 1e3) / 1e9, "TFLOP/s": fl / (kms / 1e3) / 1e12}
            continue
        kind, amount = work.get(name, ("hbm", 0.0))
        per_launch_ms = kms / launches
        per_launch = amount / launches
        if kind == "tensor":
            ach = per_launch / (per_launch_ms / 1e3) / 1e12
            peak, unit = peaks[tensor_key], "TFLOP/s"
        else:
            ach = per_launch / (per_launch_ms / 1e3) / 1e9
            peak, unit = peaks["hbm_gbs"], "GB/s"
        kernels[name] = {"ms_total": round(kms, 3), "launches": launches, "ms_per_launch": per_launch_ms,
                         "bound": "tensor" if kind == "tensor" else "hbm", "achieved": ach, "peak": peak,
                         "unit": unit, "frac": ach / peak, "algorithmic_per_launch": per_launch}
    dom = max(kernels, key=lambda k: kernels[k]["ms_total"])
    kd = kernels[dom]
    tr = NCU_TRAFFIC.get((dom, args.workload, src_hash()))
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"], "peak": kd["peak"],
                "unit": kd["unit"], "frac": kd["frac"], "traffic": tr,
                "peak_source": f"{peaks['source']} ({tensor_key if kd['bound'] == 'tensor' else 'hbm_gbs'})"}
    # whole-step roofline: the method's FLOPs against the bf16 tensor peak
    total_flops = sum(a for k, a in work.values() if k == "tensor") + 4.0 * Bsz * d * N * (N + 1) / 2
    step_roof = {"flops_per_step": total_flops,
                 "achieved_tflops": total_flops / (ms_step / 1e3) / 1e12,
                 "frac_of_bf16_peak": total_flops / (ms_step / 1e3) / 1e12 / peaks[tensor_key],
                 "peak_source": f"{peaks['source']} ({tensor_key})"}

    # the naive Theta(N^2)-traffic schedule on the same inputs (the ablation)
    ablation = None
    if args.schedule == "blocked" and not args.no_ablation:
        wsn = R.alloc_workspace(R.workspace_bytes(Bsz, N, d, H, dff, torch.bfloat16, "naive"), dev)
        outn = (torch.empty_like(z), torch.empty_like(K), torch.empty_like(V))
        ndrv = "graph" if args.driver == "persistent" else args.driver   # the naive schedule has no step kernel
        R.layer_forward(x, W, H, schedule="naive", driver=ndrv, out=outn, workspace=wsn)
        torch.cuda.synchronize()
        n0, n1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0.record(stream)
        for _ in range(args.ablation_steps):
            R.layer_forward(x, W, H, schedule="naive", driver=ndrv, out=outn, workspace=wsn)
        n1.record(stream)
        torch.cuda.synchronize()
        if R.sync_status(wsn) != 0:
            raise RuntimeError("device error in the naive-schedule ablation")
        n_ms = n0.elapsed_time(n1) / args.ablation_steps
        kv_bytes = 4.0 * Bsz * d * N * (N - 1) / 2
        ablation = {"schedule": "naive", "ms_per_step": n_ms, "value": Bsz * N / (n_ms / 1e3),
                    "unit": "tokens/s", "steps": args.ablation_steps,
                    "kv_bytes_per_step": kv_bytes, "kv_GBps": kv_bytes / (n_ms / 1e3) / 1e9,
                    "blocked_speedup": n_ms / ms_step}
        del wsn, outn
        torch.cuda.empty_cache()

    # the same forward with the other step-loop driver (one kernel per phase,
    # or the persistent step kernel): 1 warm-up, 2 timed
    drivers = None
    if args.schedule == "blocked" and not args.no_drivers and args.driver in ("graph", "persistent"):
        other = "persistent" if args.driver == "graph" else "graph"
        R.layer_forward(x, W, H, driver=other, out=(z, K, V), workspace=ws)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(2):
            R.layer_forward(x, W, H, driver=other, out=(z, K, V), workspace=ws)
        d1.record(stream)
        torch.cuda.synchronize()
        if R.sync_status(ws) != 0:
            raise RuntimeError(f"device error with the {other} driver")
        o_ms = d0.elapsed_time(d1) / 2
        drivers = {args.driver: {"ms_per_step": ms_step}, other: {"ms_per_step": o_ms, "steps": 2}}

    # end to end through the public C ABI with HOST buffers (copies in the timed region)
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        xh = x.cpu().pin_memory()
        Wh = {k: v.cpu().pin_memory() for k, v in W.items()}
        outh = [torch.empty((Bsz, N, d), dtype=torch.bfloat16).pin_memory(),
                torch.empty((N, Bsz, d), dtype=torch.bfloat16).pin_memory(),
                torch.empty((N, Bsz, d), dtype=torch.bfloat16).pin_memory()]
        del ws
        torch.cuda.empty_cache()
        wsh = R.alloc_workspace(R.host_workspace_bytes(Bsz, N, d, H, dff, torch.bfloat16, args.schedule), dev)
        R.layer_forward_host(xh, Wh, H, outh, wsh, schedule=args.schedule, driver=args.driver)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for _ in range(args.e2e_steps):
            R.layer_forward_host(xh, Wh, H, outh, wsh, schedule=args.schedule, driver=args.driver)
        h1.record(stream)
        torch.cuda.synchronize()
        e_ms = h0.elapsed_time(h1)
        if world > 1:
            e_ms = max_over_ranks(e_ms, dist, dev)
        e_ms /= args.e2e_steps
        h2d = xh.numel() * 2 + sum(v.numel() * 2 for v in Wh.values())
        d2h = sum(t.numel() * 2 for t in outh)
        e2e = {"value": aggregate_tokens_per_s(world, Bsz, N, e_ms), "unit": "tokens/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": "rt_layer_forward_host (pinned host buffers; H2D, forward, D2H in the timed region)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, secs = time_oracle(cfg, ORACLE_SEQS, args.seed)
        cpu = {"value": val, "unit": "tokens/s", "cores": blas_threads(), "nproc": os.cpu_count(),
               "kind": "oracle", "sample": oracle_sample_text(cfg, secs)}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args, cfg, world),
        "roofline": roofline, "step_roofline": step_roof, "kernels": kernels, "fold_levels": fold_levels,
        "ablation": ablation,
        "drivers": drivers,
        "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": R.launch_count(Bsz, N, d, H, dff, torch.bfloat16, args.schedule, args.driver) * args.steps,
        "clocks": clocks,
    }), flush=True)


if __name__ == "__main__":
    main()
