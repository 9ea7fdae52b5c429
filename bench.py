"""Sol-Attn benchmark: dense-equivalent TFLOP/s of one forward over a workload.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--tau T]
                [--impl reference]

A step is one sol_attn_forward (block pooling + fused routing / attention /
correction) over one batch of synthetic inputs resident in HBM.  The inputs
(1 GB for the default refine workload) are larger than L2, so no flush is
needed between steps.  Under torchrun each rank runs its own independent
problem (weak scaling, no collective on the data path); the reported value is
the dense-equivalent FLOPs of all ranks over the max-over-ranks time.

`--impl reference` times the CPU fp64 oracle on a bounded sample of the same
workload on the host cores (rank 0 only).
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Sol-Attn dense-equiv TFLOP/s & tensor-pipe % at N=16k-128k, τ=1.0-1.5"
DEFAULT_WORKLOAD = "refine_n32768"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")


def kernel_source_hash() -> str:
    """Hash of the attention kernel's code with comments and blank lines
    stripped: it ties a stored ncu traffic figure to the code it was taken
    on, and a comment edit does not invalidate it."""
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "block_sparse_attention_threshold_b200", "csrc")
    for f in ("attn_kernel.cuh", "ptx.cuh"):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        text = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(text.encode())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- oracle timing

def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def oracle_sample_rate(w, tau, budget_s: float, rank_seed: int = 0, dense_budget_s: float = 0.0):
    """Dense-equivalent TFLOP/s of the CPU oracle, from a bounded sample.

    The routing of the first (up to) four heads is timed head by head, then
    seeded query blocks of those heads are evaluated in a thread pool (one
    BLAS thread per worker) until about `budget_s` of wall time is spent.
    The full operator's time on all cores is extrapolated as
    B*H * (route time per head + M * time per query block) / cores, both
    per-core times.  With dense_budget_s > 0 the dense oracle (every key of
    the sequence for the block's rows) is timed the same way.
    Returns a dict: rate, cores, blocks, seconds, full_s, route_s_per_head,
    and dense_rate / dense_blocks / dense_seconds when timed.
    """
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor

    from block_sparse_attention_threshold_b200 import synthetic as syn

    small = w.replace(H=min(w.H, 4))
    qb, kb, vb = syn.generate_bf16(small)
    cores = os.cpu_count() or 1
    import contextlib
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except Exception:  # pragma: no cover
        limit = contextlib.nullcontext()
    with limit:
        return _oracle_rate(w, tau, budget_s, rank_seed, small, qb, kb, vb, cores, dense_budget_s)


def _oracle_rate(w, tau, budget_s, rank_seed, small, qb, kb, vb, cores, dense_budget_s):
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor

    from block_sparse_attention_threshold_b200 import synthetic as syn
    from oracle import sol_attn_oracle as orc

    heads = [tuple(syn.bf16_bits_to_fp64(a[0, h]) for a in (qb, kb, vb)) for h in range(small.H)]

    def route_one(h):
        q64, k64, _ = heads[h]
        t = time.perf_counter()
        r = orc.route(q64, k64, 64, w.prefix_len, tau)
        return r, time.perf_counter() - t

    with ThreadPoolExecutor(max_workers=min(cores, small.H)) as ex:
        routed = list(ex.map(route_one, range(small.H)))
    routes = [r for r, _ in routed]
    route_s = statistics.mean(t for _, t in routed)
    rng = np.random.default_rng(1000 + rank_seed)

    def pool_rate(fn, budget):
        done, t0 = 0, time.perf_counter()
        with ThreadPoolExecutor(max_workers=cores) as ex:
            while time.perf_counter() - t0 < budget:
                jobs = [(int(rng.integers(small.H)), int(rng.integers(w.M))) for _ in range(cores)]
                done += sum(ex.map(fn, jobs))
        return done, time.perf_counter() - t0

    def sol_one(job):
        h, i = job
        q64, k64, v64 = heads[h]
        orc.solattn_blocks(q64, k64, v64, 64, w.prefix_len, tau, qblocks=[i], routing=routes[h])
        return 1

    done, dt = pool_rate(sol_one, budget_s)
    block_core_s = dt * cores / done
    units = w.B * w.H
    full_s = units * (route_s + w.M * block_core_s) / cores
    res = {"rate": w.dense_flops() / full_s / 1e12, "cores": cores, "blocks": done, "seconds": dt,
           "full_s": full_s, "route_s_per_head": route_s}
    if dense_budget_s > 0:
        def dense_one(job):
            h, i = job
            q64, k64, v64 = heads[h]
            orc.dense_rows(q64, k64, v64, rows=np.arange(64 * i, 64 * i + 64))
            return 1

        dd, ddt = pool_rate(dense_one, dense_budget_s)
        dense_full_s = units * w.M * (ddt * cores / dd) / cores
        res.update(dense_rate=w.dense_flops() / dense_full_s / 1e12, dense_blocks=dd, dense_seconds=ddt)
    return res


def workload_config(w, tau, world: int) -> dict:
    """The `config` object both arms print: the workload, its size against the
    GPU's L2 (the reason no flush is needed between steps) and the replicas."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D,
            "prefix_len": w.prefix_len, "tau": tau, "block": 64,
            "l2": f"inputs {3 * w.B * w.H * w.N * w.D * 2 / 1e9:.2f} GB > L2 126 MB, no flush",
            "parallelism": f"replicas x{world}"}


# --------------------------------------------------------------------------- library comparator

LIBRARY_DENSE_IMPL = "torch scaled_dot_product_attention, cuDNN backend"


def library_dense_ms(q, k, v, timed):
    """Dense attention on the same q, k, v through PyTorch's SDPA with its
    cuDNN backend, timed by `timed`: context for the speedup, beside the
    in-repo dense kernel (the pages quote their operator against a dense
    FA-class kernel).  Returns None when that backend cannot run here."""
    import torch
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        import torch.nn.functional as F
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            F.scaled_dot_product_attention(q, k, v)
            torch.cuda.synchronize()
            return timed(lambda: F.scaled_dot_product_attention(q, k, v))
    except (RuntimeError, ImportError):
        return None


# --------------------------------------------------------------------------- allocator

def keep_pool_memory(device_index: int) -> bool:
    """Let the device's default stream-ordered memory pool keep freed memory.

    sol_attn_forward takes its scratch with cudaMallocAsync and returns it with
    cudaFreeAsync.  With the pool's default release threshold (0) the memory
    goes back to the driver at every synchronisation and the next call maps it
    again, which costs milliseconds.  Keeping it is the usual setting for an
    application that allocates every step; it lasts only for this process.
    """
    import ctypes
    try:
        cu = ctypes.CDLL("libcuda.so.1")
        dev = ctypes.c_int()
        pool = ctypes.c_void_p()
        if cu.cuDeviceGet(ctypes.byref(dev), ctypes.c_int(device_index)) != 0:
            return False
        if cu.cuDeviceGetDefaultMemPool(ctypes.byref(pool), dev) != 0:
            return False
        threshold = ctypes.c_uint64(2 ** 64 - 1)
        CU_MEMPOOL_ATTR_RELEASE_THRESHOLD = 4
        return cu.cuMemPoolSetAttribute(pool, CU_MEMPOOL_ATTR_RELEASE_THRESHOLD,
                                        ctypes.byref(threshold)) == 0
    except OSError:
        return False


# --------------------------------------------------------------------------- replicas

def rank_workload(w, rank: int, world: int):
    """Each rank runs its own independent problem: same shapes, its own seed."""
    return w if world == 1 else w.replace(seed=w.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (the job ends with its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """All ranks' dense-equivalent FLOPs over the max-over-ranks step time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


# --------------------------------------------------------------------------- GPU arm

def run_gpu(args, rank, world, local_rank):
    import numpy as np
    import torch

    from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

    if rank == 0:
        build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    abi.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    torch.zeros(1, device=dev)  # context up before touching the pool
    pool_kept = keep_pool_memory(local_rank)
    w = rank_workload(syn.workload(args.workload), rank, world)
    tau = args.tau if args.tau is not None else w.taus[0]
    qb, kb, vb = syn.generate_bf16(w)
    host = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (qb, kb, vb)]
    q, k, v = (h.to(dev) for h in host)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    dense_flops = w.dense_flops()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def step():
        abi.forward(q, k, v, tau, w.prefix_len, out=out, stream=stream)

    # Counters (outside the timed region).
    opts = abi.Opts()
    cnt = torch.zeros(2, dtype=torch.int64, device=dev)
    opts.kept_pairs = cnt.data_ptr()
    opts.exact_pairs = cnt.data_ptr() + 8
    abi.forward(q, k, v, tau, w.prefix_len, out=out, opts=opts, stream=stream)
    torch.cuda.synchronize()
    st = abi.device_status()
    if st != abi.OK:
        raise RuntimeError(abi.status_string(st))
    kept_pairs, exact_pairs = (int(x) for x in cnt.cpu().tolist())
    total_pairs = w.B * w.H * w.M * w.M
    skipped_pairs = total_pairs - kept_pairs
    kept_flops = kept_pairs * 4.0 * 64 * 64 * w.D
    corr_flops = skipped_pairs * 4.0 * 64 * w.D
    exact_flops = exact_pairs * 4.0 * 64 * 64 * w.D

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    value = whole_job_tflops(dense_flops, world, ms)

    # Per-kernel timing for the roofline: pool and attend launched alone on
    # the same stream, CUDA events around each launch.
    nbytes, _ = abi.workspace_layout(w.B, w.H, w.N, w.D)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 5)

    def timed(fn):
        for _ in range(2):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    pool_ms = timed(lambda: abi.pool(q, k, v, ws, stream=stream))
    attend_ms = timed(lambda: abi.attend(q, k, v, ws, tau, w.prefix_len, out=out, stream=stream))
    dense_ms = timed(lambda: abi.dense_forward(q, k, v, out=out, stream=stream))
    lib_ms = library_dense_ms(q, k, v, timed)
    peaks = measured_peaks()
    pool_bytes = 3.0 * w.B * w.H * w.N * w.D * 2 + w.B * w.H * w.M * w.D * 12
    achieved = (kept_flops + corr_flops) / (attend_ms * 1e-3) / 1e12
    traffic = None
    if os.path.exists(PROFILE_TRAFFIC):
        with open(PROFILE_TRAFFIC) as f:
            prof = json.load(f)
        if prof.get("source_hash") == kernel_source_hash() and prof.get("workload") == w.name:
            traffic = prof.get("dram_bytes_per_launch")

    # End to end through the public host-buffer call (sol_attn_forward_host):
    # every step copies q, k, v in from pinned memory and the output back,
    # inside the library's chunked copy/compute pipeline.
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        abi.forward_host(host[0], host[1], host[2], tau, w.prefix_len, out=out_host, stream=stream)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / args.steps, world, dev)
    e2e_value = whole_job_tflops(dense_flops, world, e2e_ms)

    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            o = oracle_sample_rate(w, tau, args.cpu_budget * 2 / 3, dense_budget_s=args.cpu_budget / 3)
            cpu = {"value": o["rate"], "unit": "TFLOP/s", "cores": o["cores"], "kind": "oracle",
                   "cpu_model": cpu_model(),
                   "sample": f"routing of the first 4 heads ({o['route_s_per_head']:.2f} s per head) plus "
                             f"{o['blocks']} seeded query blocks of 64 rows of those heads of {w.name} at "
                             f"tau={tau} in {o['seconds']:.1f} s; full operator extrapolated to "
                             f"{o['full_s']:.0f} s on {o['cores']} threads",
                   "dense_oracle": {"value": o["dense_rate"], "unit": "TFLOP/s",
                                    "sample": f"{o['dense_blocks']} seeded query blocks of 64 rows against "
                                              f"all {w.N} keys in {o['dense_seconds']:.1f} s, extrapolated"}}
        result = {
            "metric": METRIC,
            "value": value,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded video-grid Q/K/V, no model weights)",
            "config": workload_config(w, tau, world),
            "mempool": "freed scratch kept by the pool" if pool_kept else "default pool",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "traffic": traffic, "kernel": "sol_attn_fwd_kernel<128,false>",
                         "peak_source": f"{peaks['source']} bf16 burst"},
            "kernels": {
                "attend_ms": attend_ms,
                "pool_ms": pool_ms,
                "pool_gbs": pool_bytes / (pool_ms * 1e-3) / 1e9,
                "pool_hbm_frac": pool_bytes / (pool_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "dense_ms": dense_ms,
                "dense_tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
                "speedup_vs_dense": dense_ms / ms,
                "library_dense": None if lib_ms is None else {
                    "impl": LIBRARY_DENSE_IMPL, "ms": lib_ms,
                    "tflops": dense_flops / (lib_ms * 1e-3) / 1e12, "speedup": lib_ms / ms},
                "kept_frac": kept_pairs / total_pairs,
                "exact_frac": exact_pairs / total_pairs,
                "actual_tflops_kept": kept_flops / (attend_ms * 1e-3) / 1e12,
                "actual_tflops_kept_plus_corr": achieved,
                "tensor_tflops_exact_union": exact_flops / (attend_ms * 1e-3) / 1e12,
            },
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 3 * w.B * w.H * w.N * w.D * 2,
                    "d2h_bytes_per_step": w.B * w.H * w.N * w.D * 2},
            "gpu_launches": 2 * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
    return result


def run_sweep(args):
    """One JSON line per (workload, tau): kernel times and rates, kept fractions.

    Pool, attend and dense launches are timed alone with CUDA events (median of
    --reps launches; attend gets more launches when needed so that its timed
    region lasts --sweep-min-ms, with SM clocks sampled meanwhile); the
    dense-equivalent rate counts one pool + one attend as a step.
    """
    import numpy as np
    import torch

    from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

    build.build()
    abi.lib()
    dev = torch.device("cuda", 0)
    torch.zeros(1, device=dev)
    keep_pool_memory(0)
    names = [args.workload] if args.workload != "all" else [
        "draft_n16128", "refine_n32768", "long_n65536", "sweep_n131072"]
    peaks = measured_peaks()
    for name in names:
        w = syn.workload(name)
        if args.heads is not None:
            w = w.replace(H=min(w.H, args.heads))
        if args.fp8:
            run_sweep_fp8(args, w, dev, peaks)
            continue
        qb, kb, vb = syn.generate_bf16(w)
        q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for a in (qb, kb, vb))
        del qb, kb, vb
        out = torch.empty_like(q)
        nbytes, _ = abi.workspace_layout(w.B, w.H, w.N, w.D)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

        def timed(fn, reps, min_ms=0.0):
            # One untimed launch also estimates the duration; short kernels get
            # more launches so the timed region spans at least min_ms.
            a0, b0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            fn()
            b0.record()
            torch.cuda.synchronize()
            est = max(a0.elapsed_time(b0), 1e-3)
            reps = max(reps, min(2000, math.ceil(min_ms / est)))
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(reps)]
            for a, b in ev:
                a.record()
                fn()
                b.record()
            torch.cuda.synchronize()
            return statistics.median(a.elapsed_time(b) for a, b in ev)

        pool_ms = timed(lambda: abi.pool(q, k, v, ws), args.reps)
        dense_ms = timed(lambda: abi.dense_forward(q, k, v, out=out), max(1, args.reps // 2))
        lib_ms = library_dense_ms(q, k, v, lambda fn: timed(fn, max(1, args.reps // 2)))
        taus = [args.tau] if args.tau is not None else list(w.taus)
        budget = 0
        if args.budget_sparsity is not None:  # fixed-budget routing, skipped blocks dropped
            budget = max(1, round((1.0 - args.budget_sparsity) * (w.M - w.P)))
            taus = [0.0]
        total = w.B * w.H * w.M * w.M
        for tau in taus:
            opts = abi.Opts()
            opts.budget_blocks = budget
            opts.skip_correction = 1 if budget else 0
            cnt = torch.zeros(2, dtype=torch.int64, device=dev)
            opts.kept_pairs = cnt.data_ptr()
            opts.exact_pairs = cnt.data_ptr() + 8
            abi.attend(q, k, v, ws, tau, w.prefix_len, out=out, opts=opts)
            torch.cuda.synchronize()
            kept, exact = (int(x) for x in cnt.cpu().tolist())
            run_opts = abi.Opts()
            run_opts.budget_blocks = budget
            run_opts.skip_correction = 1 if budget else 0
            with ClockSampler(0) as clk:
                att_ms = timed(lambda: abi.attend(q, k, v, ws, tau, w.prefix_len, out=out, opts=run_opts),
                               args.reps, min_ms=args.sweep_min_ms)
            kept_fl = kept * 4.0 * 64 * 64 * w.D
            corr_fl = 0.0 if budget else (total - kept) * 4.0 * 64 * w.D
            step = pool_ms + att_ms
            row = {
                "workload": name, "tau": None if budget else tau,
                "routing": f"budget {budget} blocks, no correction" if budget else "threshold",
                "kept_frac": kept / total, "exact_frac": exact / total,
                "attend_ms": att_ms, "pool_ms": pool_ms, "dense_ms": dense_ms,
                "dense_equiv_tflops": w.dense_flops() / step / 1e9,
                "actual_tflops_kept": kept_fl / att_ms / 1e9,
                "actual_tflops_kept_plus_corr": (kept_fl + corr_fl) / att_ms / 1e9,
                "frac_of_peak_kept_plus_corr": (kept_fl + corr_fl) / att_ms / 1e9 / peaks["bf16_tflops"],
                "tensor_tflops_exact_union": exact * 4.0 * 64 * 64 * w.D / att_ms / 1e9,
                "dense_tflops": w.dense_flops() / dense_ms / 1e9,
                "speedup_vs_dense": dense_ms / step,
                "library_dense_tflops": None if lib_ms is None else w.dense_flops() / lib_ms / 1e9,
                "speedup_vs_library_dense": None if lib_ms is None else lib_ms / step,
                "pool_gbs": (3.0 * w.B * w.H * w.N * w.D * 2 + w.B * w.H * w.M * w.D * 12) / pool_ms / 1e6,
                "device_status": abi.device_status(),
                "clocks": clk.summary(),
            }
            print(json.dumps(row), flush=True)
        del q, k, v, out, ws
        torch.cuda.empty_cache()


def run_sweep_fp8(args, w, dev, peaks):
    """The 8-bit entry point on workload `w`: E4M3 inputs (scale 1), pooling
    and attention timed alone with CUDA events (medians), one JSON line per tau.
    The roofline denominator is twice the measured bf16 burst peak (the nominal
    E4M3 / bf16 tensor-rate ratio), stated in the line."""
    import numpy as np
    import torch

    from block_sparse_attention_threshold_b200 import abi, synthetic as syn

    bits = syn.generate_e4m3(w)
    q8, k8, v8 = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in bits)
    del bits
    out = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
    nbytes, _ = abi.workspace_layout(w.B, w.H, w.N, w.D)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    pool_ms = timed(lambda: abi.pool_fp8(q8, k8, v8, ws), max(5, args.reps))
    total = w.B * w.H * w.M * w.M
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    taus = [args.tau] if args.tau is not None else list(w.taus)
    for tau in taus:
        opts = abi.Opts()
        cnt = torch.zeros(2, dtype=torch.int64, device=dev)
        opts.kept_pairs = cnt.data_ptr()
        opts.exact_pairs = cnt.data_ptr() + 8
        abi.attend_fp8(q8, k8, v8, ws, tau, w.prefix_len, out=out, opts=opts)
        torch.cuda.synchronize()
        kept, exact = (int(x) for x in cnt.cpu().tolist())
        with ClockSampler(0) as clk:
            att_ms = timed(lambda: abi.attend_fp8(q8, k8, v8, ws, tau, w.prefix_len, out=out), max(5, args.reps))
        kept_fl = kept * 4.0 * 64 * 64 * w.D
        corr_fl = (total - kept) * 4.0 * 64 * w.D
        step = pool_ms + att_ms
        row = {
            "workload": w.name, "tau": tau, "precision": "e4m3 inputs, e4m3 P, fp32 accumulate, bf16 out",
            "kept_frac": kept / total, "exact_frac": exact / total,
            "attend_ms": att_ms, "pool_ms": pool_ms,
            "dense_equiv_tflops": w.dense_flops() / step / 1e9,
            "actual_tflops_kept_plus_corr": (kept_fl + corr_fl) / att_ms / 1e9,
            "fp8_peak_tflops": fp8_peak,
            "frac_of_fp8_peak": (kept_fl + corr_fl) / att_ms / 1e9 / fp8_peak,
            "peak_source": f"{peaks['source']} bf16 burst x 2 (nominal E4M3/bf16 ratio)",
            "pool_gbs": (3.0 * w.B * w.H * w.N * w.D + w.B * w.H * w.M * w.D * 10) / pool_ms / 1e6,
            "device_status": abi.device_status(),
            "clocks": clk.summary(),
        }
        print(json.dumps(row), flush=True)


def run_prep(args):
    """QKNorm + partial RoPE ahead of Sol-Attn: the fused pass that also fills
    the pooled workspace, against the same chain without pooling followed by
    the standalone pooling pass.  One JSON line; CUDA-event medians."""
    import numpy as np
    import torch

    from block_sparse_attention_threshold_b200 import abi, build, synthetic as syn

    build.build()
    abi.lib()
    dev = torch.device("cuda", 0)
    w = syn.workload(args.workload)
    qb, kb, vb = syn.generate_bf16(w)
    q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for a in (qb, kb, vb))
    del qb, kb, vb
    rng = np.random.default_rng(w.seed + 7)
    wq = torch.from_numpy((1.0 + 0.25 * rng.normal(size=w.D)).astype(np.float32)).to(dev)
    wk = torch.from_numpy((1.0 + 0.25 * rng.normal(size=w.D)).astype(np.float32)).to(dev)
    R = args.rope_dims if args.rope_dims is not None else w.D // 2
    q_out, k_out = torch.empty_like(q), torch.empty_like(k)
    nbytes, _ = abi.workspace_layout(w.B, w.H, w.N, w.D)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    fused_ms = timed(lambda: abi.qknorm_rope_pool(q, k, v, wq, wk, R, q_out=q_out, k_out=k_out, workspace=ws),
                     max(10, args.reps))
    chain_ms = timed(lambda: abi.qknorm_rope_pool(q, k, v, wq, wk, R, q_out=q_out, k_out=k_out, pool=False),
                     max(10, args.reps))
    pool_ms = timed(lambda: abi.pool(q_out, k_out, v, ws), max(10, args.reps))
    elems = w.B * w.H * w.N * w.D
    fused_bytes = 3 * elems * 2 + 2 * elems * 2 + w.B * w.H * w.M * w.D * 12
    peaks = measured_peaks()
    gbs = fused_bytes / (fused_ms * 1e-3) / 1e9
    row = {
        "workload": w.name, "rope_dims": R,
        "fused_ms": fused_ms, "chain_only_ms": chain_ms, "pool_ms": pool_ms,
        "separate_ms": chain_ms + pool_ms, "saved_ms": chain_ms + pool_ms - fused_ms,
        "fused_bytes": fused_bytes, "fused_gbs": gbs, "fused_hbm_frac": gbs / peaks["hbm_gbs"],
        "hbm_peak_gbs": peaks["hbm_gbs"], "device_status": abi.device_status(),
    }
    print(json.dumps(row), flush=True)


def run_reference(args, rank):
    """The oracle as the reference arm: each step is a bounded sample of the
    workload on the host cores; ms_per_step is that sample's measured wall
    time and value the extrapolated dense-equivalent rate."""
    from block_sparse_attention_threshold_b200 import synthetic as syn
    if rank != 0:
        return None
    w = syn.workload(args.workload)
    tau = args.tau if args.tau is not None else w.taus[0]
    rates, walls, fulls = [], [], []
    t0 = time.perf_counter()
    for _ in range(args.warmup):
        oracle_sample_rate(w, tau, max(1.0, args.ref_step_budget / 4))
    for _ in range(args.steps):
        ts = time.perf_counter()
        o = oracle_sample_rate(w, tau, args.ref_step_budget)
        walls.append(time.perf_counter() - ts)
        rates.append(o["rate"])
        fulls.append(o["full_s"])
    value = statistics.mean(rates)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": statistics.mean(walls) * 1e3,
        "extrapolated_full_operator_ms": statistics.mean(fulls) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded video-grid Q/K/V, no model weights)",
        "config": workload_config(w, tau, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": o["cores"], "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"per step: routing of the first 4 heads plus ~{args.ref_step_budget:.0f} s of "
                                   f"seeded query blocks of those heads of {w.name}; rate extrapolated to the "
                                   f"full operator"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t0,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-step-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="kernel table: one JSON line per (workload, tau); --workload all for every one")
    ap.add_argument("--reps", type=int, default=5, help="timed launches per kernel in --sweep")
    ap.add_argument("--prep", action="store_true",
                    help="time the fused QKNorm + partial RoPE + pooling pass against the unfused pair")
    ap.add_argument("--rope-dims", type=int, default=None, help="--prep: rotated dimensions (default D/2)")
    ap.add_argument("--sweep-min-ms", type=float, default=500.0,
                    help="--sweep: lower bound on each attend timing region (more launches if needed)")
    ap.add_argument("--heads", type=int, default=None,
                    help="--sweep on the first H heads only (a reduced case for profiling)")
    ap.add_argument("--fp8", action="store_true",
                    help="--sweep with the 8-bit entry point (E4M3 inputs); frac against twice the bf16 peak")
    ap.add_argument("--budget-sparsity", type=float, default=None,
                    help="--sweep with fixed-budget routing keeping (1 - s) of the video blocks, "
                         "skipped blocks dropped (the draft stage's block-sparse attention)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torchrun (one rank per GPU)")
    if args.sweep:
        if rank == 0:
            run_sweep(args)
        return
    if args.prep:
        if rank == 0:
            run_prep(args)
        return
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
