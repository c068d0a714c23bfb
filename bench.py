"""Benchmark: paged-KV decode attention on B200.

One step = one call of ``paged_decode_attn`` (split kernel, plus the merge
kernel when the planner splits) over one batch of synthetic inputs that are
already resident in HBM. Default workload: B=128 sequences, 32 query / 8 KV
heads, head_dim 128, page_size 16, kv_len 8192, bf16 K/V (4.3 GB of K/V, far
larger than L2, so no flush is needed between steps). After it, every other
workload is timed in the same process at the same --steps / --warmup, each
with its own L2 policy (pools under 1 GiB rotate among copies; tiny ones get
an L2 flush before every step), into the line's ``workloads`` object.

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
L2_BYTES = 126e6  # B200 L2


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE.name, choices=sorted(W.ALL) + sorted(W.EXTRA))
    ap.add_argument("--splits", type=int, default=0, help="force a split count (0: planner)")
    ap.add_argument("--kernel", choices=["auto", "tensor_cores", "cuda_cores"], default="auto",
                    help="split kernel: the planner's choice, or force one")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (profiling a smaller case)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fused-merge", action="store_true",
                    help="tensor-core kernel: merge splits in the kernel (no merge launch)")
    ap.add_argument("--native-fp8-qk", action="store_true",
                    help="FP8 K/V: q enters QK^T as one e4m3 term (changes the result)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the read-only HBM probe and the CUDA-graph replay (profiling runs)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only --workload (not every workload)")
    ap.add_argument("--cpu-seconds-per-workload", type=float, default=3.0,
                    help="bound of each workload entry's CPU oracle sample")
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


def recorded_traffic(workload_name: str, kernel_name: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    record (profiles/dram_traffic.json, keyed "<workload>/<kernel>"), or None
    when there is no record for that workload and kernel or the kernel
    sources changed since the counters were taken (the record stores their
    sha256)."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)[f"{workload_name}/{kernel_name}"]
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
    """K/V bytes of keys some row may see + Q (bf16) + O (fp32) + LSE (fp32).
    A key's K (or V) row is D * 2 bytes in bf16, D in e4m3, and D/2 bytes of
    codes plus D/16 bytes of block scales in NVFP4."""
    vis = W.visible_token_count(wl, kv_lens)
    if wl.kv_dtype == W.KV_NVFP4:
        row = wl.head_dim // 2 + wl.head_dim // 16
    else:
        row = wl.head_dim * (2 if wl.kv_dtype == W.KV_BF16 else 1)
    kv = vis * wl.num_kv_heads * row * 2
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
        sc = {}
        if inp.get("k_scales") is not None:
            sc = dict(k_scales=W.to_bits(inp["k_scales"][idx, g: g + 1].contiguous()),
                      v_scales=W.to_bits(inp["v_scales"][idx, g: g + 1].contiguous()))
        q = inp["q"][b: b + 1, :, g * G: (g + 1) * G].contiguous()
        args = (W.to_bits(q), W.to_bits(kp), W.to_bits(vp),
                torch.arange(n, dtype=torch.int32).reshape(1, n).numpy(),
                lens[b: b + 1].numpy())
        t0 = time.perf_counter()
        orc.paged_decode_attn(*args, num_kv_heads=1, page_size=P, scale=W.scale_of(wl),
                              causal_offset=wl.causal_offset, window=wl.window,
                              kv_dtype=wl.kv_dtype, kv_scale=inp["kv_scale"], **sc)
        elapsed += time.perf_counter() - t0
    return elapsed


def oracle_sequences_mt(inp, first: int, count: int, threads: int) -> float:
    """Whole sequences [first, first + count), all heads, on `threads`
    OpenMP threads of the oracle (one row per task). Returns seconds."""
    from oracle import oracle as orc
    wl = inp["workload"]
    sl = slice(first, first + count)
    args = (W.to_bits(inp["q"][sl].contiguous()), W.to_bits(inp["k_pages"]),
            W.to_bits(inp["v_pages"]), inp["page_table"][sl].contiguous().cpu().numpy(),
            inp["kv_lens"][sl].contiguous().cpu().numpy())
    sc = {}
    if inp.get("k_scales") is not None:
        sc = dict(k_scales=W.to_bits(inp["k_scales"]), v_scales=W.to_bits(inp["v_scales"]))
    t0 = time.perf_counter()
    orc.paged_decode_attn(*args, num_kv_heads=wl.num_kv_heads, page_size=wl.page_size,
                          scale=W.scale_of(wl), causal_offset=wl.causal_offset,
                          window=wl.window, kv_dtype=wl.kv_dtype,
                          kv_scale=inp["kv_scale"], threads=threads, **sc)
    return time.perf_counter() - t0


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_mt(inp, seconds: float):
    """The oracle on every host core (OpenMP, one output row per task) on
    whole sequences of the workload, for about `seconds`."""
    wl = inp["workload"]
    threads = host_threads()
    seqs, mt_elapsed = 0, 0.0
    # the K/V pools go to the host once; each call then takes whole sequences
    host = dict(inp, q=inp["q"].cpu(), k_pages=inp["k_pages"].cpu(),
                v_pages=inp["v_pages"].cpu(), page_table=inp["page_table"].cpu(),
                kv_lens=inp["kv_lens"].cpu())
    if inp.get("k_scales") is not None:
        host.update(k_scales=inp["k_scales"].cpu(), v_scales=inp["v_scales"].cpu())
    while mt_elapsed < seconds and seqs < wl.batch:
        n = min(max(1, threads // max(1, wl.num_q_heads * wl.q_len) + 1), wl.batch - seqs)
        mt_elapsed += oracle_sequences_mt(host, seqs, n, threads)
        seqs += n
    return {
        "value": seqs * wl.q_len / mt_elapsed, "unit": "tokens/s", "cores": threads,
        "kind": "oracle",
        "sample": (f"{seqs} full sequences (all heads) of {wl.name}, fp64 C oracle on "
                   f"{threads} OpenMP threads (one output row per task), {mt_elapsed:.2f} s"),
    }


def cpu_baseline(inp, seconds: float):
    """The oracle timed on the host: single-threaded on (sequence, kv head)
    units, then on every host core (OpenMP) on whole sequences, each leg on
    a bounded sample of about `seconds`. The reported value is the
    all-cores leg; the single-threaded one rides along."""
    wl = inp["workload"]
    units, elapsed = 0, 0.0
    order = [(b, g) for b in range(wl.batch) for g in range(wl.num_kv_heads)]
    while elapsed < seconds and units < len(order):
        elapsed += oracle_units(inp, [order[units]])
        units += 1
    single = {
        "value": units / wl.num_kv_heads * wl.q_len / elapsed, "unit": "tokens/s", "cores": 1,
        "sample": (f"{units} (sequence, kv head) units of {wl.name} "
                   f"({units / wl.num_kv_heads:.3f} full sequences, all heads), "
                   f"single-threaded fp64 C oracle, {elapsed:.1f} s"),
    }
    mt = cpu_baseline_mt(inp, seconds)
    mt["single_thread"] = single
    return mt


# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores, on bounded
    samples of the same workload (rank 0 only)."""
    if rank != 0:
        return
    # Same shapes and distributions, fewer sequences: the steps cycle over
    # (sequence, kv head) units of the first few sequences.
    wl = {**W.ALL, **W.EXTRA}[args.workload]
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


L2_FLUSH_BYTES = 256 * 1024 * 1024
# K/V pools under this size are timed rotating among copies of themselves,
# so consecutive steps never find their K/V in L2.
ROTATE_BELOW_BYTES = 1 << 30
ROTATE_MIN_POOL_BYTES = 16 * 1024 * 1024  # smaller pools: flush L2 instead


def run_flags(args) -> int:
    flags = {"auto": 0, "tensor_cores": B.PDA_FLAG_TENSOR_CORES,
             "cuda_cores": B.PDA_FLAG_CUDA_CORES}[args.kernel]
    if args.fused_merge:
        flags |= B.PDA_FLAG_FUSED_MERGE
    if args.native_fp8_qk:
        flags |= B.PDA_FLAG_NATIVE_FP8_QK
    return flags


def prepare(wl, dev, rank, splits, flags):
    """Inputs of one workload resident in HBM, the call's arguments, and the
    L2 policy of its timed region: pools of 1 GiB or more are read as they
    are; smaller pools (down to 16 MiB) rotate among enough copies that a
    copy comes back only after 1 GiB of other K/V; tiny pools get a 256 MiB
    write before every timed step instead (outside the step's events)."""
    inp = W.generate(wl, device=dev, seed=wl.seed + rank)
    scale = W.scale_of(wl)
    kp, vp, pt, kl = inp["k_pages"], inp["v_pages"], inp["page_table"], inp["kv_lens"]
    max_len = int(kl.max().item())
    out = torch.empty((wl.batch, wl.q_len, wl.num_q_heads, wl.head_dim), dtype=torch.float32,
                      device=dev)
    lse = torch.empty((wl.batch, wl.q_len, wl.num_q_heads), dtype=torch.float32, device=dev)
    kw = dict(num_kv_heads=wl.num_kv_heads, scale=scale, causal_offset=wl.causal_offset,
              window=wl.window, kv_scale=inp["kv_scale"], max_kv_len=max_len,
              num_splits=splits, flags=flags)
    params = B.make_params(
        batch=wl.batch, q_len=wl.q_len, num_q_heads=wl.num_q_heads,
        num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, page_size=wl.page_size,
        max_pages_per_seq=pt.shape[1], num_pages=kp.shape[0], scale=scale,
        causal_offset=wl.causal_offset, window=wl.window, kv_dtype=wl.kv_dtype,
        kv_scale=inp["kv_scale"], max_kv_len=max_len, num_splits=splits, flags=flags)
    kernel_name = B.KERNEL_NAMES.get(B.plan_kernel(params), "unknown")
    ws = torch.empty(max(B.workspace_bytes(params), 1), dtype=torch.uint8, device=dev)
    ks, vs = inp.get("k_scales"), inp.get("v_scales")  # NVFP4 block-scale pools
    pool_bytes = kp.numel() * kp.element_size() * 2 + (0 if ks is None else ks.numel() * 2)
    pools = [(kp, vp, ks, vs)]
    flush = None
    if pool_bytes >= ROTATE_BELOW_BYTES:
        l2 = (f"no flush: the K/V pools ({pool_bytes / 1e9:.2f} GB) are more than 8x the "
              "L2 (126 MB)")
    elif pool_bytes >= ROTATE_MIN_POOL_BYTES:
        n = max(2, -(-ROTATE_BELOW_BYTES // pool_bytes))
        pools += [(kp.clone(), vp.clone(), None if ks is None else ks.clone(),
                   None if vs is None else vs.clone()) for _ in range(n - 1)]
        l2 = (f"rotating {n} copies of the K/V pools ({pool_bytes / 1e9:.3f} GB each): "
              f"step i reads copy i mod {n}, so a copy returns after "
              f"{(n - 1) * pool_bytes / 1e9:.2f} GB of other K/V")
    else:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        l2 = ("flushed before every timed step (256 MiB write, outside the step's events; "
              "the time is the sum of the per-step events)")
    return dict(wl=wl, inp=inp, out=out, lse=lse, kw=kw, ws=ws, pools=pools, flush=flush,
                l2=l2, kernel_name=kernel_name, max_len=max_len)


def call(ctx, i=0):
    kp, vp, ks, vs = ctx["pools"][i % len(ctx["pools"])]
    inp = ctx["inp"]
    return B.paged_decode_attn(inp["q"], kp, vp, inp["page_table"], inp["kv_lens"],
                               out=ctx["out"], lse=ctx["lse"], workspace=ctx["ws"],
                               k_scales=ks, v_scales=vs, **ctx["kw"])[2]


def time_steps(ctx, steps, warmup, world, local):
    """W warm-up steps, then exactly `steps` steps between a barrier and a
    synchronize on both sides, timed with CUDA events on the launching
    stream, twice: launched from the host one call at a time (each step
    bracketed by its own events), and as one CUDA graph holding the same
    `steps` calls (rotating over the same pool copies: no host launch gaps
    and no L2 reuse), the way a serving engine replays its decode step.
    The graph timing is the primary one; a workload that needs an L2 flush
    before every step (the tiny one) keeps the host-launched timing.
    Returns a dict: elapsed ms (max over ranks), mean ms per step, clocks,
    split count, which timing is primary, and the host-launched figures."""
    stream = torch.cuda.current_stream()
    splits = call(ctx)
    torch.cuda.synchronize()
    if B.last_device_error() != 0:
        raise RuntimeError(f"{ctx['wl'].name}: device error word set after the first call")
    for i in range(max(warmup, 3)):
        call(ctx, i + 1)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)  # let the sampler start before the timed region
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    flush = ctx["flush"]
    t_begin.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        starts[i].record(stream)
        call(ctx, i)
        ends[i].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launched_ms = t_begin.elapsed_time(t_end)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    if flush is not None:  # the flushes are not part of the job
        launched_ms = sum(step_ms)
    if B.last_device_error() != 0:
        raise RuntimeError(f"{ctx['wl'].name}: device error word set during the timed region")
    launched = {"ms_per_step": max_over_ranks(launched_ms, world) / steps,
                "avg_launch_ms": statistics.mean(step_ms)}
    res = {"elapsed_ms": max_over_ranks(launched_ms, world),
           "avg_ms": statistics.mean(step_ms), "splits": splits, "timing": "host-launched",
           "launched": launched}
    if flush is None:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                call(ctx, i)
        g.replay()  # untimed: first replay
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        graph_ms = g0.elapsed_time(g1)
        del g
        if B.last_device_error() != 0:
            raise RuntimeError(f"{ctx['wl'].name}: device error word set during the graph replay")
        res.update(elapsed_ms=max_over_ranks(graph_ms, world), avg_ms=graph_ms / steps,
                   timing=f"one CUDA graph of the {steps} calls")
    res["clocks"] = sampler.stop()
    return res


def launches_per_step(kernel_name, splits, fused_merge):
    """Our kernels per call: the tensor-core kernel runs after its prologue
    kernel (counters, queue order, FP8 Q images); the merge kernel follows
    when the splits are merged apart."""
    merge = splits > 1 and not (kernel_name == "split_tma_kernel" and fused_merge)
    return (2 if kernel_name == "split_tma_kernel" else 1) + (1 if merge else 0), merge


def graph_replay(ctx, steps, world):
    """One call captured in a CUDA graph and replayed (no host launch gaps;
    L2 not flushed between replays)."""
    stream = torch.cuda.current_stream()
    wl = ctx["wl"]
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(ctx)
        for _ in range(3):
            g.replay()
        n_g = max(20, min(steps, 500))
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(n_g):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        g_ms = g0.elapsed_time(g1) / n_g
        del g
        return {"ms_per_step": g_ms, "value": wl.batch * wl.q_len * world / (g_ms / 1e3),
                "unit": "tokens/s", "replays": n_g, "l2": "warm (no flush between replays)"}
    except RuntimeError as e:
        return {"error": str(e).splitlines()[0][:200]}


def workload_entry(ctx, args, world, local, peak, probe_gbs, fused_merge, with_cpu):
    """Time one workload; its numbers as one entry of the line's
    `workloads` object."""
    wl = ctx["wl"]
    t = time_steps(ctx, args.steps, args.warmup, world, local)
    elapsed_ms, avg_ms, clocks, splits = t["elapsed_ms"], t["avg_ms"], t["clocks"], t["splits"]
    alg_bytes, kv_bytes = algorithmic_bytes(wl, ctx["inp"]["kv_lens"].tolist())
    gbs = alg_bytes / (avg_ms / 1e3) / 1e9
    per_step, merge = launches_per_step(ctx["kernel_name"], splits, fused_merge)
    entry = {
        "ms_per_step": elapsed_ms / args.steps,
        "tokens_per_s": wl.batch * wl.q_len * args.steps * world / (elapsed_ms / 1e3),
        "algorithmic_bytes_per_step": alg_bytes,
        "avg_launch_ms": avg_ms,
        "gb_s": gbs,
        "frac_of_copy": gbs / peak,
        "frac_of_8tbs_spec": gbs / 8000.0,
        "frac_of_read_probe": gbs / probe_gbs if probe_gbs else None,
        "kernel": ctx["kernel_name"] + (" + merge_states_kernel" if merge else ""),
        "splits": splits,
        "gpu_launches": per_step * args.steps,
        "steps": args.steps, "warmup": args.warmup,
        "batch": wl.batch, "q_len": wl.q_len, "num_q_heads": wl.num_q_heads,
        "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "page_size": wl.page_size,
        "kv_dtype": {W.KV_BF16: "bf16", W.KV_FP8_E4M3: "fp8_e4m3", W.KV_NVFP4: "nvfp4"}.get(
            wl.kv_dtype, wl.kv_dtype),
        "l2": ctx["l2"],
        "timing": t["timing"],
        "launched": t["launched"],
        "clocks": clocks,
        "graph": None if args.no_extras else graph_replay(ctx, args.steps, world),
        "traffic": recorded_traffic(wl.name, ctx["kernel_name"]),
    }
    if with_cpu:
        entry["cpu_baseline"] = cpu_baseline_mt(ctx["inp"], args.cpu_seconds_per_workload)
    return entry


def run_ours(args, rank, world, local):
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device (the library has no CPU path)")
    B.load()
    wl = {**W.ALL, **W.EXTRA}[args.workload]
    if args.batch:
        wl = wl.with_(batch=args.batch, name=f"{wl.name}_batch{args.batch}")
    dev = torch.device("cuda", torch.cuda.current_device())
    flags = run_flags(args)
    ctx = prepare(wl, dev, rank, args.splits, flags)
    inp, out, lse, ws, kw = ctx["inp"], ctx["out"], ctx["lse"], ctx["ws"], ctx["kw"]
    q, kp, vp = inp["q"], inp["k_pages"], inp["v_pages"]
    pt, kl = inp["page_table"], inp["kv_lens"]
    max_len = ctx["max_len"]
    kernel_name = ctx["kernel_name"]
    stream = torch.cuda.current_stream()

    t = time_steps(ctx, args.steps, args.warmup, world, local)
    elapsed_ms, clocks, splits = t["elapsed_ms"], t["clocks"], t["splits"]
    tokens_per_step = wl.batch * wl.q_len
    value = tokens_per_step * args.steps * world / (elapsed_ms / 1e3)
    alg_bytes, kv_bytes = algorithmic_bytes(wl, kl.tolist())
    avg_launch_ms = t["avg_ms"]
    achieved = alg_bytes / (avg_launch_ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    per_step, merge_launched = launches_per_step(kernel_name, splits, args.fused_merge)

    # Read-only HBM probe in the same run (our streaming-load kernel over a
    # 4 GiB buffer, larger than L2): the ceiling for a kernel that only reads.
    probe_gbs = None
    try:
        if args.no_extras:
            raise RuntimeError("skipped (--no-extras)")
        pbuf = torch.zeros(4 * 1024 ** 3, dtype=torch.uint8, device=dev)
        sink = torch.zeros(1, dtype=torch.int64, device=dev)
        for _ in range(3):
            B.hbm_read_probe(pbuf, sink)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        p0.record(stream)
        for _ in range(reps):
            B.hbm_read_probe(pbuf, sink)
        p1.record(stream)
        torch.cuda.synchronize()
        probe_gbs = pbuf.numel() * reps / (p0.elapsed_time(p1) / 1e3) / 1e9
        del pbuf
    except (RuntimeError, B.PdaError) as e:  # out of memory: report none
        print(f"read probe skipped: {e}", file=sys.stderr)

    graph = None if args.no_extras else graph_replay(ctx, args.steps, world)

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
            B.paged_decode_attn(dq, kp, vp, dpt, dkl, out=out, lse=lse, workspace=ws,
                                k_scales=inp.get("k_scales"), v_scales=inp.get("v_scales"), **kw)
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

    # The KV-cache producer on the same cache (measured after the decode
    # timing; it overwrites the last slots of each sequence): one new token
    # per sequence (a decode step's append) and 64 (a chunk's), K and V.
    kv_append = None
    if not args.no_extras:
        kv_append = {}
        # bytes per element written: bf16 2, e4m3 1, NVFP4 1/2 + 1/16 of a scale
        elt = {W.KV_BF16: 2, W.KV_FP8_E4M3: 1, W.KV_NVFP4: 0.5625}[wl.kv_dtype]
        for T in (1, 64):
            if int(kl.min().item()) < T:
                continue
            kn = torch.randn((wl.batch, T, wl.num_kv_heads, wl.head_dim), device=dev).to(torch.bfloat16)
            vn = torch.randn_like(kn)
            base = (kl - T).contiguous()
            sc = dict(k_scales=inp.get("k_scales"), v_scales=inp.get("v_scales"))
            for _ in range(3):
                B.paged_kv_append(kn, vn, pt, base, kp, vp, kv_scale=inp["kv_scale"], **sc)
            # 50 appends in one CUDA graph: device time, not Python call rate
            n_app = 50
            ga = torch.cuda.CUDAGraph()
            with torch.cuda.graph(ga):
                for _ in range(n_app):
                    B.paged_kv_append(kn, vn, pt, base, kp, vp, kv_scale=inp["kv_scale"], **sc)
            ga.replay()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            ga.replay()
            a1.record(stream)
            torch.cuda.synchronize()
            del ga
            ms = a0.elapsed_time(a1) / n_app
            nbytes = 2 * wl.batch * T * wl.num_kv_heads * wl.head_dim * (2 + elt)
            kv_append[f"tokens_{T}"] = {"ms": ms, "bytes": nbytes, "gb_s": nbytes / (ms / 1e3) / 1e9,
                                        "frac_of_copy": nbytes / (ms / 1e3) / 1e9 / peak}
        if B.last_device_error() != 0:
            raise RuntimeError("device error word set by the append measurement")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_seconds)

    # Every workload, each timed in this process at the same --steps and
    # --warmup with its own L2 policy (the line's top level is the one
    # above; its entry repeats those numbers).
    workloads = None
    if not (args.no_workloads or args.batch):
        workloads = {}
        with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
        for name, other in list(W.ALL.items()) + list(W.EXTRA.items()):
            if name == wl.name:
                entry = {
                    "ms_per_step": elapsed_ms / args.steps, "tokens_per_s": value,
                    "algorithmic_bytes_per_step": alg_bytes, "avg_launch_ms": avg_launch_ms,
                    "gb_s": achieved, "frac_of_copy": achieved / peak,
                    "frac_of_8tbs_spec": achieved / 8000.0,
                    "frac_of_read_probe": achieved / probe_gbs if probe_gbs else None,
                    "kernel": kernel_name + (" + merge_states_kernel" if merge_launched else ""),
                    "splits": splits, "gpu_launches": per_step * args.steps,
                    "steps": args.steps, "warmup": args.warmup, "batch": wl.batch,
                    "q_len": wl.q_len, "num_q_heads": wl.num_q_heads,
                    "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                    "page_size": wl.page_size,
                    "kv_dtype": {W.KV_BF16: "bf16", W.KV_FP8_E4M3: "fp8_e4m3"}.get(
                        wl.kv_dtype, wl.kv_dtype),
                    "l2": ctx["l2"], "timing": t["timing"], "launched": t["launched"],
                    "clocks": clocks, "graph": graph,
                    "traffic": recorded_traffic(wl.name, kernel_name),
                    "cpu_baseline": (cpu_baseline_mt(inp, args.cpu_seconds_per_workload)
                                     if with_cpu else None),
                    "top_level": True,
                }
            else:
                octx = prepare(other, dev, rank, args.splits, flags)
                entry = workload_entry(octx, args, world, local, peak, probe_gbs,
                                       args.fused_merge, with_cpu)
                if name in W.EXTRA:
                    entry["extra"] = "a KV dtype beyond the five workloads (the headline's shape)"
                del octx
                torch.cuda.empty_cache()
            workloads[name] = entry

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
        "dtype": {W.KV_BF16: "bf16", W.KV_FP8_E4M3: "fp8_e4m3 kv, bf16 q, fp32 accumulate",
                  W.KV_NVFP4: "nvfp4 kv, bf16 q, fp32 accumulate"}[wl.kv_dtype],
        "data": "synthetic",
        "config": {
            "workload": wl.name, "batch": wl.batch, "q_len": wl.q_len,
            "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
            "head_dim": wl.head_dim, "page_size": wl.page_size,
            "kv_len": max_len if wl.kv_lens[0] == "const" else str(wl.kv_lens),
            "causal_offset": wl.causal_offset, "window": wl.window,
            "num_splits": splits, "parallelism": f"replicas x{world}",
            "l2": ctx["l2"],
            "timing": t["timing"],
            "algorithmic_bytes_per_step": alg_bytes,
        },
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": None if args.batch else recorded_traffic(wl.name, kernel_name),
            "traffic_unit": "bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)",
            "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "frac_of_8tbs_spec": achieved / 8000.0,
            "kernel": kernel_name + (" + merge_states_kernel" if merge_launched else ""),
            "read_probe_gbs": probe_gbs,
            "frac_of_read_probe": achieved / probe_gbs if probe_gbs else None,
            "avg_launch_ms": avg_launch_ms,
        },
        "gpu_launches": per_step * args.steps,
        "launched": t["launched"],
        "clocks": clocks,
        "graph": graph,
        "kv_append": kv_append,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "workloads": workloads,
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
