#!/usr/bin/env python
"""Benchmark of one PagedAttention decode step on B200.

A step is the whole hot path over one batch: the cache append
(pa_reshape_and_cache) followed by paged decode attention (pa_decode: the
split-context kernel plus its log-sum-exp merge).  Default workload: the
LLaMA-7B-shaped layer (32 sequences, 32 q / 32 kv heads, head_dim 128,
block_size 16, context lengths uniform in [128, 2048], fp16, a shuffled pool
of 8400 blocks).

Metric: effective HBM bandwidth = logical K+V bytes the step reads
(sum over sequences of ctx * kv_heads * head_dim * 2 * 2 B) / device time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs an independent
replica of the workload (decode shards over sequences with no exchange);
`value` is the bytes of all ranks / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
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

METRIC = "pa_decode effective HBM GB/s (KV bytes read / device time) and % of B200 peak"
UNIT = "GB/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024

# DRAM traffic of one decode-kernel launch (dram__bytes_read.sum +
# dram__bytes_write.sum, ncu --set full, profiles/paged_decode_*.md), keyed by
# workload; reported only while the decode kernel's device sources hash to `src`.
NCU_TRAFFIC = {
    "llama7b-mha": {"bytes": 584_963_840 + 4_026_112, "src": "f65eb04587b47385"},
    "llama3-8b-gqa": {"bytes": 1_148_161_000 + 6_258_176, "src": "f65eb04587b47385"},
    "long-context-shared-prefix": {"bytes": 1_007_600_000 + 3_718_144, "src": "f65eb04587b47385"},
}


def kernel_source_hash() -> str:
    """Hash of the decode kernel's device code (the kernel whose traffic is quoted)."""
    h = hashlib.sha256()
    for f in ("paged_decode_kernel.cuh", "pa_device.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_368_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def describe(wl) -> str:
    ctx = wl.context_lens
    return (f"{wl.name}: {wl.num_seqs} seqs, {wl.num_heads} q / {wl.num_kv_heads} kv heads, head_dim "
            f"{wl.head_dim}, block_size {wl.block_size}, ctx {int(ctx.min())}..{int(ctx.max())} "
            f"(mean {float(ctx.mean()):.0f}), {wl.dtype}, pool {wl.num_blocks} blocks shuffled")


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]), parts[2], parts[3:7]))
            except ValueError:
                continue

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        use = inside if inside else self.samples
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({names[i] for s in use for i, v in enumerate(s[4]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(s[1] for s in use), "sm_max_mhz": max(s[2] for s in use),
                "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(inside)}


# ------------------------------------------------------------------ distributed


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, dist, device) -> float:
    """Max of a per-rank value over all ranks (identity without a process group)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput_gbs(bytes_per_step_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the bytes every rank processed over the slowest rank's time."""
    return bytes_per_step_per_rank * world * steps / (max_ms * 1e-3) / 1e9


def load_workload(args, poison=False):
    from paged_kv_cache_368_b200 import inputs

    return inputs.config(args.config, block_size=args.block_size, poison=poison)


# ------------------------------------------------------------------ oracle timing (CPU)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_pass(wl, units):
    """Prepare the float64 oracle (append + decode) on `units` = [(seq, kv_head)]
    of the workload.  Returns (run, kv_bytes): run() does one pass."""
    import oracle

    G = wl.num_heads // wl.num_kv_heads
    seqs = sorted({s for s, _ in units})
    kc, vc, tc = wl.compact(seqs)
    row = {s: r for r, s in enumerate(seqs)}
    slots = np.array([oracle.slot_of_position(tc[row[s]], int(wl.context_lens[s]) - 1, wl.block_size)
                      for s in seqs], dtype=np.int64)
    by_head = {}
    for s, h in units:
        by_head.setdefault(h, []).append(s)
    nbytes = sum(int(wl.context_lens[s]) for s, _ in units) * wl.head_dim * 2 * wl.elem_bytes

    def run():
        k2, v2 = oracle.reshape_and_cache(wl.k_new[seqs], wl.v_new[seqs], kc, vc, slots)
        for h, ss in by_head.items():
            rows = [row[s] for s in ss]
            oracle.decode(wl.q[ss][:, h * G:(h + 1) * G], k2[:, h:h + 1], v2[:, h:h + 1], tc[rows],
                          wl.context_lens[ss], wl.scale, wl.dtype)

    return run, nbytes


def time_passes(run, budget_s):
    times = []
    t_end = time.perf_counter() + budget_s
    while True:
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > t_end:
            break
    return statistics.median(times), len(times)


def cpu_baseline(wl, budget_s=12.0):
    # bound the sample: time one sequence, then take as many whole sequences as fit
    run1, _ = oracle_pass(wl, [(0, h) for h in range(wl.num_kv_heads)])
    per_seq, _ = time_passes(run1, 0.0)
    nseq = int(max(1, min(wl.num_seqs, budget_s / 3 / max(per_seq, 1e-4))))
    run, nbytes = oracle_pass(wl, [(s, h) for s in range(nseq) for h in range(wl.num_kv_heads)])
    t, reps = time_passes(run, budget_s)
    return {"value": nbytes / t / 1e9, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"float64 NumPy oracle (append + decode) on sequences 0..{nseq - 1} of {wl.num_seqs}, "
                       f"all {wl.num_kv_heads} kv-heads ({nbytes / 1e6:.1f} MB KV), median of {reps} passes"),
            "host_cpus": os.cpu_count(), "affinity": len(os.sched_getaffinity(0))}


def run_reference(args):
    world, rank, _ = dist_init()
    if rank != 0:
        return 0
    wl = load_workload(args)
    K, W = args.steps, args.warmup
    units = [(s, h) for s in range(wl.num_seqs) for h in range(wl.num_kv_heads)]
    run1, _ = oracle_pass(wl, units[:1])
    t1, _ = time_passes(run1, 0.0)
    budget = 120.0  # seconds for the whole warm-up + timed run
    n_units = int(max(1, min(len(units), budget / max(K + W, 1) / max(t1, 1e-5))))
    run, nbytes = oracle_pass(wl, units[:n_units])
    for _ in range(W):
        run()
    t0 = time.perf_counter()
    for _ in range(K):
        run()
    total = time.perf_counter() - t0
    value = nbytes * K / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": total / K * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(wl), "sample_units": n_units, "parallelism": "none (CPU, rank 0)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{n_units} (sequence, kv-head) units per step of {len(units)}, "
                                   f"{nbytes / 1e6:.2f} MB KV per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm


def run_ours(args):
    import ctypes

    import torch

    from paged_kv_cache_368_b200 import build as pbuild
    from paged_kv_cache_368_b200 import libpaged

    world, rank, local = dist_init()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    if rank == 0:
        pbuild.build()
    if dist is not None:
        dist.barrier()
    lib = libpaged.load()

    wl = load_workload(args)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype]
    dev = torch.device("cuda", local)

    def upload(raw):
        return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16).copy()).view(dt).to(dev)

    shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, wl.head_dim)
    k_cache = torch.zeros(shape, dtype=dt, device=dev)
    v_cache = torch.zeros(shape, dtype=dt, device=dev)
    idx = torch.from_numpy(wl.used).to(dev)
    k_cache.index_copy_(0, idx, upload(wl.k_blocks))
    v_cache.index_copy_(0, idx, upload(wl.v_blocks))
    q, k_new, v_new = upload(wl.q), upload(wl.k_new), upload(wl.v_new)
    slots = torch.from_numpy(wl.slot_mapping.astype(np.int64)).to(dev)
    tables = torch.from_numpy(wl.block_tables.astype(np.int32)).to(dev)
    ctx = torch.from_numpy(wl.context_lens.astype(np.int32)).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    max_ctx = wl.max_context_len
    ws = libpaged.alloc_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, max_ctx, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    kvh, D, bs, nb = wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks
    code = libpaged.dtype_code(dt)
    mb = wl.max_blocks_per_seq
    r_args = (k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), slots.data_ptr(),
              wl.num_seqs, kvh, D, bs, nb, code, err.data_ptr(), sp)
    d_args = (out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), tables.data_ptr(), mb,
              ctx.data_ptr(), wl.num_seqs, max_ctx, float(wl.scale), wl.num_heads, kvh, D, bs, nb, code,
              ws.data_ptr(), ws.numel(), 0, err.data_ptr(), sp)

    def step(dec_events=None):
        st = lib.pa_reshape_and_cache(*r_args)
        if dec_events is not None:
            dec_events[0].record(stream)
        st |= lib.pa_decode(*d_args)
        if dec_events is not None:
            dec_events[1].record(stream)
        return st

    K, W = args.steps, args.warmup
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}")
    time.sleep(0.3)
    for _ in range(W):
        if step() != 0:
            raise SystemExit("libpaged call failed in warm-up")
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise SystemExit(f"device error flags {int(err.item())}")

    # ---- timed region 1: K whole steps, bracketed by one event pair (events
    # between the launches would break the programmatic-launch overlap)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    e0.record(stream)
    bad = 0
    for i in range(K):
        bad |= step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if dist is not None:
        dist.barrier()
    if bad:
        raise SystemExit("libpaged call failed in the timed region")
    elapsed_ms = reduce_max(e0.elapsed_time(e1), dist, dev)

    # ---- timed region 2: the same steps with an event pair around every
    # pa_decode call on its stream -> per-launch duration of the dominant kernel
    dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        bad |= step(dec[i])
    torch.cuda.synchronize(dev)
    if bad:
        raise SystemExit("libpaged call failed in the timed region")
    dec_ms = [a.elapsed_time(b) for a, b in dec]

    # ---- end to end through the public API: one packed pinned host buffer of
    # the step's inputs in, the result out (pa_decode_step_host)
    offs, total = libpaged.step_inputs_layout(wl.num_seqs, wl.num_heads, kvh, D, mb)
    h_in = torch.zeros(total, dtype=torch.uint8).pin_memory()
    t_ = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    libpaged.pack_step_inputs(h_in, offs, q=t_(wl.q), key=t_(wl.k_new), value=t_(wl.v_new),
                              slot_mapping=t_(wl.slot_mapping.astype(np.int64)),
                              block_tables=t_(wl.block_tables.astype(np.int32)),
                              context_lens=t_(wl.context_lens.astype(np.int32)))
    d_in = torch.empty(total, dtype=torch.uint8, device=dev)
    h_out = torch.empty(out.shape, dtype=dt).pin_memory()
    h2d = total
    d2h = h_out.numel() * h_out.element_size()
    e_args = (h_in.data_ptr(), d_in.data_ptr(), h_out.data_ptr(), out.data_ptr(), k_cache.data_ptr(),
              v_cache.data_ptr(), wl.num_seqs, mb, max_ctx, float(wl.scale), wl.num_heads, kvh, D, bs, nb, code,
              ws.data_ptr(), ws.numel(), err.data_ptr(), sp)

    def e2e_step():
        if lib.pa_decode_step_host(*e_args) != 0:
            raise SystemExit("pa_decode_step_host failed")

    Ke = min(K, 2000)
    for _ in range(max(3, W)):
        e2e_step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(Ke):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(f0.elapsed_time(f1), dist, dev)
    clocks.stop()

    kvb = wl.kv_bytes()
    value = throughput_gbs(kvb, world, K, elapsed_ms)
    mean_dec = statistics.mean(dec_ms)
    achieved = kvb / (mean_dec * 1e-3) / 1e9
    peak, peak_src = measured_peak()
    src = kernel_source_hash()
    tr = NCU_TRAFFIC.get(wl.name)
    traffic = tr["bytes"] if tr and tr.get("src") == src else None

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(load_workload(args))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": describe(wl), "kv_bytes_per_step": kvb, "unique_kv_bytes_per_step": wl.unique_kv_bytes(),
                   "l2": f"inputs larger than L2 ({kvb / 2**20:.0f} MiB of KV per step vs 126 MiB L2); no flush",
                   "parallelism": f"{world} independent replica(s), one per GPU", "step": "append + decode + merge"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "kernel": "pa_decode (decode + merge launches)",
                     "timing": "CUDA events around each pa_decode call in a second pass over the K steps",
                     "peak_source": peak_src, "frac_of_8tbs_spec": achieved / SPEC_HBM_GBS,
                     "decode_us_mean": mean_dec * 1e3, "decode_us_median": statistics.median(dec_ms) * 1e3,
                     "decode_us_min": min(dec_ms) * 1e3, "kernel_src": src},
        "cpu_baseline": cpu,
        "e2e": {"value": throughput_gbs(kvb, world, Ke, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke, "ms_per_step": e2e_ms / Ke,
                "path": "pa_decode_step_host (C ABI): packed pinned host inputs -> device (1 copy), append, decode, output -> pinned host (1 copy)"},
        "gpu_launches": 3 * K,
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_block_ops(args):
    """Secondary measurement: copy-on-write block copies inside the device pool
    and swapping blocks to / from pinned host memory, on the LLaMA-7B pool
    (8400 blocks x 32 kv heads x 16 tokens x 128 x fp16 = 128 KB per block per pool)."""
    import torch

    from paged_kv_cache_368_b200 import build as pbuild
    from paged_kv_cache_368_b200 import libpaged

    pbuild.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    nb, kvh, bs, d, npairs = 8400, 32, 16, 128, 1024
    k = torch.randn((nb, kvh, bs, d), dtype=torch.float16, device=dev)
    v = torch.randn_like(k)
    rng = np.random.default_rng(368)
    ids = rng.permutation(nb)
    pairs = torch.from_numpy(np.stack([ids[:npairs], ids[npairs:2 * npairs]], 1).astype(np.int64)).to(dev)
    block_bytes = kvh * bs * d * 2
    K, W = args.steps, args.warmup
    stream = torch.cuda.current_stream(dev)
    peak, peak_src = measured_peak()

    def timed(fn, k_steps):
        for _ in range(W):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k_steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / k_steps

    ms = timed(lambda: libpaged.copy_blocks(k, v, pairs), K)
    moved = 2 * npairs * block_bytes  # K and V pools
    copy_gbs = 2 * moved / (ms * 1e-3) / 1e9  # read + write, as the STREAM copy counts
    host = torch.empty((2 * npairs, kvh, bs, d), dtype=torch.float16).pin_memory()
    out_pairs = torch.from_numpy(np.stack([ids[:npairs], np.arange(npairs)], 1).astype(np.int64)).to(dev)
    in_pairs = torch.from_numpy(np.stack([np.arange(npairs), ids[npairs:2 * npairs]], 1).astype(np.int64)).to(dev)
    k_swap = max(3, K // 10)
    ms_out = timed(lambda: libpaged.swap_blocks(k, host, out_pairs), k_swap)
    ms_in = timed(lambda: libpaged.swap_blocks(host, k, in_pairs), k_swap)
    # reference: one contiguous cudaMemcpy of the same bytes in each direction
    flat_dev = torch.empty(npairs * block_bytes // 2, dtype=torch.float16, device=dev)
    flat_host = host.view(-1)[: flat_dev.numel()]
    ms_d2h = timed(lambda: flat_host.copy_(flat_dev, non_blocking=True), k_swap)
    ms_h2d = timed(lambda: flat_dev.copy_(flat_host, non_blocking=True), k_swap)
    sw = npairs * block_bytes
    line = {
        "metric": "block copy / swap GB/s", "op": "block_ops", "n_gpus": 1, "steps": K, "warmup": W,
        "config": {"pool": f"{nb} blocks x {kvh} kv heads x {bs} x {d} fp16 ({block_bytes // 1024} KB per block per pool)",
                   "pairs_per_call": npairs},
        "copy_blocks": {"us_per_call": ms * 1e3, "bytes_copied": moved, "gbs_read_plus_write": copy_gbs,
                        "frac_of_copy_peak": copy_gbs / peak, "peak": peak, "peak_source": peak_src},
        "swap_out_to_pinned_host": {"us_per_call": ms_out * 1e3, "bytes": sw, "gbs": sw / (ms_out * 1e-3) / 1e9,
                                    "contiguous_memcpy_gbs": sw / (ms_d2h * 1e-3) / 1e9},
        "swap_in_from_pinned_host": {"us_per_call": ms_in * 1e3, "bytes": sw, "gbs": sw / (ms_in * 1e-3) / 1e9,
                                     "contiguous_memcpy_gbs": sw / (ms_h2d * 1e-3) / 1e9},
        "roofline": {"bound": "hbm", "achieved": copy_gbs, "peak": peak, "unit": "GB/s", "frac": copy_gbs / peak,
                     "traffic": None, "kernel": "pa_copy_blocks (read + write bytes)"},
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = block_copy_cpu_baseline(kvh, bs, d)
    print(json.dumps(line), flush=True)
    return 0


def block_copy_cpu_baseline(kvh, bs, d, budget_s=4.0):
    """The oracle's copy_blocks (NumPy, as it stands: it copies the pool it is
    given, then the pairs) on a 512-block host pool with 128 pairs, counted like
    the GPU number (read + write bytes of the copied blocks)."""
    from oracle.block_manager import copy_blocks

    rng = np.random.default_rng(368)
    pool = rng.integers(0, 1 << 16, size=(512, kvh, bs, d), dtype=np.uint16)
    ids = rng.permutation(512)
    pairs = list(zip(ids[:128].tolist(), ids[128:256].tolist()))
    t, reps = time_passes(lambda: copy_blocks(pool, pairs), budget_s)
    nbytes = 2 * 128 * kvh * bs * d * 2
    return {"value": nbytes / t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"oracle copy_blocks on a {pool.nbytes >> 20} MiB host pool, 128 pairs, median of {reps} passes",
            "host_cpus": os.cpu_count(), "affinity": len(os.sched_getaffinity(0))}


def prefill_cpu_baseline(wl, q, qlen, ctx, H, KVH, D, dtype, budget_s=4.0):
    """The float64 oracle on a bounded sample of a prefill workload: the first
    new rows of sequence 0 for the q-heads of kv-head 0, sized to a few
    seconds of host time."""
    import torch

    import oracle

    G = H // KVH
    kp, vp = wl.full_pool(poison=False)
    kp, vp = np.ascontiguousarray(kp[:, :1]), np.ascontiguousarray(vp[:, :1])
    n0, c0 = qlen[0], ctx[0]

    def sample(rows):
        qs = q[:rows, :G].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        cu = np.array([0, rows], dtype=np.int32)
        cl = np.array([c0 - n0 + rows], dtype=np.int32)
        pos = np.arange(c0 - n0, c0 - n0 + rows, dtype=np.float64)
        fl = float(4.0 * D * G * (pos + 1).sum())
        return (lambda: oracle.prefill(qs, cu, kp, vp, wl.block_tables[:1], cl, wl.scale, dtype)), fl

    rows = 1  # double the sample until one pass takes about a sixth of the budget
    while True:
        run, fl = sample(rows)
        t1, _ = time_passes(run, 0.0)
        if t1 > budget_s / 6 or rows >= n0:
            break
        rows = min(n0, rows * 2)
    t, reps = time_passes(run, budget_s)
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"float64 NumPy oracle, sequence 0 rows 0..{rows - 1} of {n0}, the {G} q-heads of "
                       f"kv-head 0, median of {reps} passes"),
            "host_cpus": os.cpu_count(), "affinity": len(os.sched_getaffinity(0))}


def run_prefill(args):
    """Secondary measurement: multi-token causal paged attention (pa_prefill).
    Workloads: the ops-transformer page's example shape (1 sequence, 32 heads,
    8192 tokens, head_dim 64, fp16, block_size 16) and a chunked prefill of
    8 sequences x 1024 new tokens after 1024..3072 cached ones (32 q / 8 kv
    heads, head_dim 128, bf16)."""
    import torch

    from paged_kv_cache_368_b200 import build as pbuild
    from paged_kv_cache_368_b200 import inputs, libpaged

    pbuild.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    K, W = args.steps, args.warmup
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    peak = float(peaks.get("bf16_tflops", 1590.0))
    results = []
    for name, S, H, KVH, D, dtype, qlen, prefix in (
            ("ops-transformer example: 1 x 32 heads x 8192 tokens, d 64, fp16", 1, 32, 32, 64, "f16", [8192], [0]),
            ("chunked prefill: 8 seqs x 1024 new after 1024..3072 cached, 32/8 heads, d 128, bf16", 8, 32, 8, 128,
             "bf16", [1024] * 8, [1024, 1536, 2048, 2560, 3072, 1024, 2048, 3072])):
        ctx = [a + b for a, b in zip(qlen, prefix)]
        wl = inputs.build(name, seed=368, num_seqs=S, num_heads=H, num_kv_heads=KVH, head_dim=D, block_size=16,
                          dtype=dtype, context_lens=ctx, pool_factor=1.0, poison=False)
        dt = torch.float16 if dtype == "f16" else torch.bfloat16
        up = lambda raw: torch.from_numpy(np.ascontiguousarray(raw).view(np.int16).copy()).view(dt).to(dev)  # noqa
        shape = (wl.num_blocks, KVH, 16, D)
        kc = torch.zeros(shape, dtype=dt, device=dev)
        vc = torch.zeros(shape, dtype=dt, device=dev)
        idx = torch.from_numpy(wl.used).to(dev)
        kc.index_copy_(0, idx, up(wl.k_blocks))
        vc.index_copy_(0, idx, up(wl.v_blocks))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(qlen)]), dtype=torch.int32, device=dev)
        total = int(sum(qlen))
        q = torch.randn((total, H, D), dtype=dt, device=dev)
        out = torch.empty_like(q)
        tables = torch.from_numpy(wl.block_tables).to(dev)
        ctx_t = torch.from_numpy(wl.context_lens).to(dev)

        def call(legacy=False):
            libpaged.prefill(out, q, cu, kc, vc, tables, ctx_t, float(wl.scale), max_q_len=max(qlen),
                             max_context_len=max(ctx), legacy_mma=legacy)

        def timed(legacy):
            for _ in range(W):
                call(legacy)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(K):
                call(legacy)
            e1.record()
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) / K

        ms = timed(False)
        ms_mma = timed(True)
        # causal FLOPs: row at position p does 2 * 2 * D * (p + 1) per q-head (QK and PV)
        flops = 0
        for n, c in zip(qlen, ctx):
            pos = np.arange(c - n, c, dtype=np.float64)
            flops += float(4.0 * D * H * (pos + 1).sum())
        tf = flops / (ms * 1e-3) / 1e12
        res = {"workload": name, "us": ms * 1e3, "tflops": tf, "frac_of_bf16_peak": tf / peak,
               "kv_bytes_logical": wl.kv_bytes(), "flops": flops, "kernel": "tcgen05",
               "mma_sync_us": ms_mma * 1e3, "mma_sync_tflops": flops / (ms_mma * 1e-3) / 1e12,
               "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                            "traffic": None, "traffic_note": "kernel changed since the committed ncu capture"}}
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = prefill_cpu_baseline(wl, q, qlen, ctx, H, KVH, D, dtype)
        results.append(res)
    line = {"metric": "pa_prefill causal attention TFLOP/s", "op": "prefill", "n_gpus": 1, "steps": K, "warmup": W,
            "peak_tflops": peak, "peak_source": "MEASURED_PEAKS.json bf16_tflops (cuBLAS burst)",
            "results": results}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=1, help="workload index (1 = LLaMA-7B-shaped layer)")
    ap.add_argument("--block-size", type=int, default=None, help="block size for workload 3 (LLaMA-13B)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=("step", "block_ops", "prefill"), default="step",
                    help="step: the decode step (default); block_ops: block copy/swap throughput; "
                         "prefill: multi-token causal paged attention")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "block_ops":
        return run_block_ops(args)
    if args.op == "prefill":
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
