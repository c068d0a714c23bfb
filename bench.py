"""Benchmark: paged-KV decode attention on B200.

One step = one call of ``paged_decode_attn`` (split kernel, plus the merge
kernel when the planner splits) over one batch of synthetic inputs that are
already resident in HBM. Default workload: B=128 sequences, 32 query / 8 KV
heads, head_dim 128, page_size 16, kv_len 8192, bf16 K/V (4.3 GB of K/V, far
larger than L2, so no flush is needed between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed

For N > 1 (launched by torchrun) every rank runs an independent replica on
its own batch (the path has no exchange step), and the time is the max over
ranks. Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_decode_30_b200 import binding as B  # noqa: E402
from paged_kv_decode_30_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attn: tokens/s and achieved HBM GB/s (% of B200 roofline), 1 GPU"
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE.name, choices=sorted(W.ALL))
    ap.add_argument("--splits", type=int, default=0, help="force a split count (0: planner)")
    ap.add_argument("--tensor-cores", action="store_true",
                    help="bf16 K/V: use the tensor-core kernel instead of the FMA kernel")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (profiling a smaller case)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; the only collectives are barrier / max time)

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# measurement helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [l.strip().split(", ") for l in self.file.read().splitlines() if l.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def recorded_traffic(workload_name: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    record (profiles/dram_traffic.json), or None when there is no record for
    the workload or the kernel sources changed since the counters were
    taken (the record stores their sha256)."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)[workload_name]
        h = hashlib.sha256()
        for src in rec["source_files"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return rec.get("dram_bytes_per_launch_full")
    except (OSError, KeyError, ValueError):
        return None


def algorithmic_bytes(wl: W.Workload, kv_lens):
    """K/V bytes of keys some row may see + Q (bf16) + O (fp32) + LSE (fp32)."""
    elt = 2 if wl.kv_dtype == W.KV_BF16 else 1
    vis = W.visible_token_count(wl, kv_lens)
    kv = vis * wl.num_kv_heads * wl.head_dim * elt * 2
    rows = wl.batch * wl.q_len * wl.num_q_heads
    return kv + rows * wl.head_dim * 2 + rows * wl.head_dim * 4 + rows * 4, kv


# ---------------------------------------------------------------------------
# CPU oracle legs (test infrastructure, timed as the baseline)

def oracle_units(inp, units):
    """Run the oracle on (sequence, kv head) units, each as its own
    sub-problem (1 sequence, G query heads, 1 kv head). Returns seconds."""
    from oracle import oracle as orc
    wl = inp["workload"]
    P, G, D = wl.page_size, wl.group, wl.head_dim
    lens = inp["kv_lens"].cpu()
    pt = inp["page_table"].cpu()
    elapsed = 0.0
    for b, g in units:
        n = (int(lens[b]) + P - 1) // P
        idx = pt[b, :n].to(torch.int64).to(inp["k_pages"].device)
        kp = inp["k_pages"][idx, g: g + 1].contiguous()
        vp = inp["v_pages"][idx, g: g + 1].contiguous()
        q = inp["q"][b: b + 1, :, g * G: (g + 1) * G].contiguous()
        args = (W.to_bits(q), W.to_bits(kp), W.to_bits(vp),
                torch.arange(n, dtype=torch.int32).reshape(1, n).numpy(),
                lens[b: b + 1].numpy())
        t0 = time.perf_counter()
        orc.paged_decode_attn(*args, num_kv_heads=1, page_size=P, scale=W.scale_of(wl),
                              causal_offset=wl.causal_offset, window=wl.window,
                              kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"])
        elapsed += time.perf_counter() - t0
    return elapsed


def cpu_baseline(inp, seconds: float):
    wl = inp["workload"]
    units, elapsed = 0, 0.0
    order = [(b, g) for b in range(wl.batch) for g in range(wl.num_kv_heads)]
    while elapsed < seconds and units < len(order):
        elapsed += oracle_units(inp, [order[units]])
        units += 1
    tokens = units / wl.num_kv_heads * wl.q_len
    return {
        "value": tokens / elapsed, "unit": "tokens/s", "cores": 1, "kind": "oracle",
        "sample": (f"{units} (sequence, kv head) units of {wl.name} "
                   f"({units / wl.num_kv_heads:.3f} full sequences, all heads), "
                   f"single-threaded fp64 C oracle, {elapsed:.1f} s"),
    }


# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores, on bounded
    samples of the same workload (rank 0 only)."""
    if rank != 0:
        return
    # Same shapes and distributions, fewer sequences: the steps cycle over
    # (sequence, kv head) units of the first few sequences.
    wl = W.ALL[args.workload]
    inp = W.generate(wl.with_(batch=min(wl.batch, 4)), device="cpu")
    wl = inp["workload"]
    order = [(b, g) for b in range(wl.batch) for g in range(wl.num_kv_heads)]
    for s in range(args.warmup):
        oracle_units(inp, [order[s % len(order)]])
    total = 0.0
    for s in range(args.steps):
        total += oracle_units(inp, [order[(args.warmup + s) % len(order)]])
    tokens = args.steps / wl.num_kv_heads * wl.q_len
    value = tokens / total
    sample = (f"each step: one (sequence, kv head) unit of {wl.name} "
              f"(1/{wl.num_kv_heads} of a sequence's heads), single-threaded fp64 C oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device (the library has no CPU path)")
    B.load()
    wl = W.ALL[args.workload]
    if args.batch:
        wl = wl.with_(batch=args.batch, name=f"{wl.name}_batch{args.batch}")
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = W.generate(wl, device=dev, seed=wl.seed + rank)
    scale = W.scale_of(wl)
    q, kp, vp = inp["q"], inp["k_pages"], inp["v_pages"]
    pt, kl = inp["page_table"], inp["kv_lens"]
    max_len = int(kl.max().item())
    out = torch.empty((wl.batch, wl.q_len, wl.num_q_heads, wl.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((wl.batch, wl.q_len, wl.num_q_heads), dtype=torch.float32, device=dev)
    flags = B.PDA_FLAG_TENSOR_CORES if args.tensor_cores else 0
    kw = dict(num_kv_heads=wl.num_kv_heads, scale=scale, causal_offset=wl.causal_offset,
              window=wl.window, kv_scale=inp["kv_scale"], max_kv_len=max_len,
              num_splits=args.splits, flags=flags)
    params = B.make_params(
        batch=wl.batch, q_len=wl.q_len, num_q_heads=wl.num_q_heads,
        num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, page_size=wl.page_size,
        max_pages_per_seq=pt.shape[1], num_pages=kp.shape[0], scale=scale,
        causal_offset=wl.causal_offset, window=wl.window, kv_dtype=wl.kv_dtype,
        kv_scale=inp["kv_scale"], max_kv_len=max_len, num_splits=args.splits, flags=flags)
    ws_bytes = B.workspace_bytes(params)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        return B.paged_decode_attn(q, kp, vp, pt, kl, out=out, lse=lse, workspace=ws, **kw)[2]

    splits = step()
    torch.cuda.synchronize()
    if B.last_device_error() != 0:
        raise RuntimeError("device error word set after the first call")
    for _ in range(max(args.warmup, 3)):
        step()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)  # let the sampler start before the timed region
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    elapsed_ms = t_begin.elapsed_time(t_end)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    if B.last_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    elapsed_ms = max_over_ranks(elapsed_ms, world)
    tokens_per_step = wl.batch * wl.q_len
    value = tokens_per_step * args.steps * world / (elapsed_ms / 1e3)
    alg_bytes, kv_bytes = algorithmic_bytes(wl, kl.tolist())
    avg_launch_ms = statistics.mean(step_ms)
    achieved = alg_bytes / (avg_launch_ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    launches_per_step = 1 + (1 if splits > 1 else 0)

    # End to end through the public API with host buffers: every step copies
    # the step's inputs (q, page table, kv lengths) from pinned host memory
    # and reads out + lse back. The paged K/V cache stays resident in HBM, as
    # it does across the decode steps of a serving engine.
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hpt = pt.cpu().pin_memory()
        hkl = kl.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        dq, dpt, dkl = torch.empty_like(q), torch.empty_like(pt), torch.empty_like(kl)

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dpt.copy_(hpt, non_blocking=True)
            dkl.copy_(hkl, non_blocking=True)
            B.paged_decode_attn(dq, kp, vp, dpt, dkl, out=out, lse=lse, workspace=ws, **kw)
            hout.copy_(out, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        for _ in range(max(args.warmup, 3)):
            e2e_step()
        n_e2e = max(10, args.steps // 4)
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": tokens_per_step * n_e2e * world / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": hq.numel() * hq.element_size() + hpt.numel() * 4 + hkl.numel() * 4,
               "d2h_bytes_per_step": hout.numel() * 4 + hlse.numel() * 4,
               "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_seconds)

    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.kv_dtype == W.KV_BF16 else "fp8_e4m3 kv, bf16 q, fp32 accumulate",
        "data": "synthetic",
        "config": {
            "workload": wl.name, "batch": wl.batch, "q_len": wl.q_len,
            "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
            "head_dim": wl.head_dim, "page_size": wl.page_size,
            "kv_len": max_len if wl.kv_lens[0] == "const" else str(wl.kv_lens),
            "causal_offset": wl.causal_offset, "window": wl.window,
            "num_splits": splits, "parallelism": f"replicas x{world}",
            "l2": "no flush: K/V read per step "
                  f"({kv_bytes / 1e9:.2f} GB) larger than L2" if kv_bytes > 126e6
                  else "inputs smaller than L2",
            "algorithmic_bytes_per_step": alg_bytes,
        },
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": None if args.batch else recorded_traffic(wl.name),
            "traffic_unit": "bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)",
            "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "frac_of_8tbs_spec": achieved / 8000.0,
            "kernel": "split_fma_kernel" + (" + merge_states_kernel" if splits > 1 else ""),
            "avg_launch_ms": avg_launch_ms,
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
