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

# DRAM traffic per launch from an ncu capture, keyed by (kernel class, workload,
# hash of the CUDA sources at capture time). Reported as null once the sources
# change. Filled from the ncu summaries under profiles/.
NCU_TRAFFIC: dict = {}


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
    ap.add_argument("--driver", choices=["graph", "stream"], default="graph")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
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
        # q, k~, v~ of position t (bf16), (m, l, o) of query t read (fp32), a_t written (bf16)
        "attend": ("hbm", float(N) * B * (6 * d + 4 * d + 8 * H + 2 * d)),
    }
    if schedule == "naive":
        # query t reads the t-1 persistent pairs (k, v bf16) plus its own q, k~, v~; writes a_t
        w["attend"] = ("hbm", float(B) * (4 * d * N * (N - 1) / 2 + N * 8 * d))
        return w
    warp_b, mma_b = 0.0, 0.0
    for t in range(1, N):
        lb = lowbit(t)
        nq = min(lb, N - t)
        init = (t == lb)
        per_q = 2 * d + (4 * d if init else 8 * d) + (8 * H if init else 16 * H)   # q read; o, m, l (read+)write
        by = B * (nq * per_q + lb * 4 * d)                                          # + keys' k, v read
        if lb >= 16:
            mma_b += by
        else:
            warp_b += by
    w["fold_warp"] = ("hbm", warp_b)
    w["fold_mma"] = ("hbm", mma_b)
    return w


# --------------------------------------------------------------------------
# the oracle as the CPU baseline / reference arm
# --------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def time_oracle(cfg: dict, n_seq: int, n_pos: int, seed: int) -> tuple[float, float]:
    """Runs the fp64 oracle (naive definition) on n_seq sequences x n_pos
    positions of the workload; returns (tokens/s, seconds)."""
    import rtinputs
    from oracle import rt_oracle
    W = rtinputs.weights(seed, cfg["d"], cfg["d_ff"], dtype="bf16")
    x = rtinputs.x_batch(seed, range(n_seq), n_pos, cfg["d"], dtype="bf16")
    t0 = time.perf_counter()
    rt_oracle.rt_layer(x, W, cfg["H"])
    dt = time.perf_counter() - t0
    return n_seq * n_pos / dt, dt


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    cfg = WORKLOADS[args.workload]
    n_seq, n_pos = 1, 256
    for _ in range(args.warmup):
        time_oracle(cfg, n_seq, n_pos, args.seed)
    secs = [time_oracle(cfg, n_seq, n_pos, args.seed)[1] for _ in range(args.steps)]
    ms = 1e3 * sum(secs) / len(secs)
    value = n_seq * n_pos / (ms / 1e3)
    cores = blas_threads()
    sample = (f"{n_seq} sequence x first {n_pos} positions of the {args.workload} workload per step "
              f"(fp64 numpy oracle, naive schedule)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
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
    kernels = {}
    for name, (kms, launches) in classes.items():
        kind, amount = work.get(name, ("hbm", 0.0))
        per_launch_ms = kms / launches
        per_launch = amount / launches
        if kind == "tensor":
            ach = per_launch / (per_launch_ms / 1e3) / 1e12
            peak, unit = peaks["bf16_tflops_sustained"], "TFLOP/s"
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
                "peak_source": f"{peaks['source']} ({'bf16_tflops_sustained' if kd['bound'] == 'tensor' else 'hbm_gbs'})"}
    # whole-step roofline: the method's FLOPs against the bf16 tensor peak
    total_flops = sum(a for k, a in work.values() if k == "tensor") + 4.0 * Bsz * d * N * (N + 1) / 2
    step_roof = {"flops_per_step": total_flops,
                 "achieved_tflops": total_flops / (ms_step / 1e3) / 1e12,
                 "frac_of_bf16_peak": total_flops / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops_sustained"]}

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
        n_seq, n_pos = 2, N
        val, secs = time_oracle(cfg, n_seq, n_pos, args.seed)
        cpu = {"value": val, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n_seq} sequences x all {n_pos} positions of the workload "
                         f"(fp64 numpy oracle, naive schedule; {secs:.1f} s)"}

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
        "roofline": roofline, "step_roofline": step_roof, "kernels": kernels,
        "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": R.launch_count(Bsz, N, d, H, dff, torch.bfloat16, args.schedule) * args.steps,
        "clocks": clocks,
    }), flush=True)


if __name__ == "__main__":
    main()
