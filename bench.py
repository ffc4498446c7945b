#!/usr/bin/env python
"""Benchmark of one PagedAttention decode step on B200.

A step is the whole hot path over one batch: the cache append
(pa_reshape_and_cache) followed by paged decode attention (pa_decode: one
split-context kernel launch whose log-sum-exp merge runs inside it).  Default workload: the
LLaMA-7B-shaped layer (32 sequences, 32 q / 32 kv heads, head_dim 128,
block_size 16, context lengths uniform in [128, 2048], fp16, a shuffled pool
of 8400 blocks).

Metric: effective HBM bandwidth = logical K+V bytes the step reads
(sum over sequences of ctx * kv_heads * head_dim * 2 * 2 B) / device time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs an independent
replica of the workload (decode shards over sequences with no exchange);
`value` is the bytes of all ranks / the slowest rank's time.

On one GPU the line also carries `per_config`: the same timings for the other
workloads (the GQA LLaMA-3-8B layer, the LLaMA-13B layer at block sizes 8, 16,
32 and 64, the long-context shared-prefix layer and the tiny case).
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
PREFILL_BURST_S = 0.02  # device time of the burst figure (against the burst bf16 peak)
PREFILL_SUSTAINED_S = 1.0  # device time of the sustained figure (against the sustained peak)

# DRAM traffic of one decode-kernel launch (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture: --set full, or those two
# metrics alone), keyed by workload; reported only while the decode kernel's
# device sources hash to `src`.
NCU_TRAFFIC = {
    "llama7b-mha": {"bytes": 584_962_816 + 3_268_096, "src": "0fc3b1941294cf11"},
    "llama3-8b-gqa": {"bytes": 1_148_157_696 + 3_682_304, "src": "0fc3b1941294cf11"},
    "long-context-shared-prefix": {"bytes": 1_006_903_040 + 3_442_176, "src": "0fc3b1941294cf11"},
    "llama13b-mha-bs8": {"bytes": 671_289_088 + 2_937_344, "src": "0fc3b1941294cf11"},
    "llama13b-mha-bs16": {"bytes": 671_280_128 + 3_345_920, "src": "0fc3b1941294cf11"},
    "llama13b-mha-bs32": {"bytes": 671_282_688 + 3_188_480, "src": "0fc3b1941294cf11"},
    "llama13b-mha-bs64": {"bytes": 671_275_264 + 3_356_416, "src": "0fc3b1941294cf11"},
    "tiny-mha": {"bytes": 315_392 + 0, "src": "0fc3b1941294cf11"},
}


# The same for one launch of the tcgen05 prefill kernel (ncu --set full).
PREFILL_NCU_TRAFFIC = {
    "chunked": {"bytes": 167_832_320 + 45_532_928, "src": "ade5ff18156f9ea0"},
    "d64": {"bytes": 100_769_280 + 16_449_280, "src": "ade5ff18156f9ea0"},
}


def _sources_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_cache_368_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# One pa_copy_blocks launch (one pool) of the block_ops workload: reads and
# the writes that reached DRAM before the launch ended (the rest were still
# in L2); keyed by the copy kernel's source hash.
BLOCK_COPY_NCU = {"read": 134_257_664, "write": 86_838_016, "src": "32cbaa28f7b71298"}


def block_copy_source_hash() -> str:
    return _sources_hash(("block_copy.cu", "pa_device.cuh"))


def kernel_source_hash() -> str:
    """Hash of the decode kernel's device code (the kernel whose traffic is quoted)."""
    return _sources_hash(("paged_decode_kernel.cuh", "paged_merge.cuh", "pa_device.cuh"))


def prefill_source_hash() -> str:
    """Hash of the tcgen05 prefill kernel's device code."""
    return _sources_hash(("paged_prefill_tc.cu", "tcgen05.cuh", "exp2_poly.cuh", "pa_device.cuh"))


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


LAUNCHES_PER_STEP = 2  # our kernels per step: reshape_and_cache_kernel + paged_decode_kernel


class DecodeBench:
    """One workload resident on the device, with the calls that time it."""

    def __init__(self, lib, libpaged, wl, dev):
        import torch

        self.lib, self.wl, self.dev = lib, wl, dev
        dt = {"f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype]
        self.dt = dt

        def upload(raw):
            return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16).copy()).view(dt).to(dev)

        shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, wl.head_dim)
        self.k_cache = torch.zeros(shape, dtype=dt, device=dev)
        self.v_cache = torch.zeros(shape, dtype=dt, device=dev)
        idx = torch.from_numpy(wl.used).to(dev)
        self.k_cache.index_copy_(0, idx, upload(wl.k_blocks))
        self.v_cache.index_copy_(0, idx, upload(wl.v_blocks))
        self.q, self.k_new, self.v_new = upload(wl.q), upload(wl.k_new), upload(wl.v_new)
        self.slots = torch.from_numpy(wl.slot_mapping.astype(np.int64)).to(dev)
        self.tables = torch.from_numpy(wl.block_tables.astype(np.int32)).to(dev)
        self.ctx = torch.from_numpy(wl.context_lens.astype(np.int32)).to(dev)
        self.out = torch.empty_like(self.q)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_ctx = wl.max_context_len
        self.ws = libpaged.alloc_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, self.max_ctx,
                                           device=dev)
        self.stream = torch.cuda.current_stream(dev)
        sp = self.stream.cuda_stream
        kvh, D, bs, nb = wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks
        code = libpaged.dtype_code(dt)
        mb = wl.max_blocks_per_seq
        self.r_args = (self.k_new.data_ptr(), self.v_new.data_ptr(), self.k_cache.data_ptr(),
                       self.v_cache.data_ptr(), self.slots.data_ptr(), wl.num_seqs, kvh, D, bs, nb, code,
                       self.err.data_ptr(), sp)
        self.d_args = (self.out.data_ptr(), self.q.data_ptr(), self.k_cache.data_ptr(), self.v_cache.data_ptr(),
                       self.tables.data_ptr(), mb, self.ctx.data_ptr(), wl.num_seqs, self.max_ctx, float(wl.scale),
                       wl.num_heads, kvh, D, bs, nb, code, self.ws.data_ptr(), self.ws.numel(), 0,
                       self.err.data_ptr(), sp)
        # end to end through the public API: one packed pinned host buffer of
        # the step's inputs in, the result out (pa_decode_step_host)
        offs, total = libpaged.step_inputs_layout(wl.num_seqs, wl.num_heads, kvh, D, mb)
        self.h_in = torch.zeros(total, dtype=torch.uint8).pin_memory()
        t_ = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
        libpaged.pack_step_inputs(self.h_in, offs, q=t_(wl.q), key=t_(wl.k_new), value=t_(wl.v_new),
                                  slot_mapping=t_(wl.slot_mapping.astype(np.int64)),
                                  block_tables=t_(wl.block_tables.astype(np.int32)),
                                  context_lens=t_(wl.context_lens.astype(np.int32)))
        self.h_out = torch.empty(self.out.shape, dtype=dt).pin_memory()
        self.h2d = total
        self.d2h = self.h_out.numel() * self.h_out.element_size()
        # pipelined form: the input copy of step i+1 (second stream, two
        # staging buffers in turn) overlaps the kernels of step i, the output
        # copy of step i (third stream, two device output buffers in turn)
        # those of step i+1.  The C-ABI arguments of both sets are built
        # once, so a step is one library call (no per-step Python marshalling
        # that the GPU would wait for).
        self.pipe = libpaged.StepPipeline(total, self.out.shape, dt, device=dev, stream=self.stream)
        self.e_args = [self.pipe.args(b, self.h_in, self.h_out, self.k_cache, self.v_cache, wl.num_heads, mb,
                                      float(wl.scale), self.max_ctx, self.ws, self.err) for b in range(2)]
        self.e_index = 0

    def step(self):
        st = self.lib.pa_reshape_and_cache(*self.r_args)
        st |= self.lib.pa_decode(*self.d_args)
        if st != 0:
            raise SystemExit(f"libpaged call failed on {self.wl.name}")

    def decode(self):
        if self.lib.pa_decode(*self.d_args) != 0:
            raise SystemExit(f"pa_decode failed on {self.wl.name}")

    def e2e_step(self):
        args = self.e_args[self.e_index & 1]
        self.e_index += 1
        if self.lib.pa_decode_step_host_pipelined(*args) != 0:
            raise SystemExit(f"pa_decode_step_host_pipelined failed on {self.wl.name}")

    def check_e2e_output(self):
        """The pipelined host step's last output equals the device step's."""
        import torch

        self.pipe.wait()
        self.step()
        torch.cuda.synchronize(self.dev)
        if not torch.equal(self.h_out, self.out.cpu()):
            raise SystemExit(f"host-step output differs from the device step on {self.wl.name}")

    def check_flags(self):
        import torch

        torch.cuda.synchronize(self.dev)
        if int(self.err.item()) != 0:
            raise SystemExit(f"device error flags {int(self.err.item())} on {self.wl.name}")

    # ---- timing helpers (CUDA events on the launching stream)

    def time_back_to_back(self, fn, n):
        """ms for n calls between one event pair (no events between the
        launches, which would break the programmatic-launch overlap)."""
        import torch

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.dev)
        e0.record(self.stream)
        for _ in range(n):
            fn()
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1)

    def time_e2e(self, n):
        """ms for n pipelined host steps between one event pair on the
        compute stream, which waits for the last output copy before the
        closing event."""
        import torch

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.dev)
        e0.record(self.stream)
        for _ in range(n):
            self.e2e_step()
        self.pipe.join()
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1)

    def time_each_decode(self, n, flush=None):
        """Per-call ms of n pa_decode calls, an event pair around each (after
        the step's append, so the cache is the step's); with `flush` a buffer
        of twice the L2 is read before every call (cold L2: the lines it
        leaves are clean, so the timed call pays no write-backs)."""
        import torch

        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        torch.cuda.synchronize(self.dev)
        for a, b in ev:
            self.lib.pa_reshape_and_cache(*self.r_args)
            if flush is not None:
                flush.max()  # a read of 2x the L2
            a.record(self.stream)
            self.decode()
            b.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return [a.elapsed_time(b) for a, b in ev]

    def calls_for(self, seconds, ms_per_call):
        return int(max(1, seconds * 1e3 / max(ms_per_call, 1e-3)))


def decode_summary(b, kvb, steps_ms, n_steps, per_call, cold, peak, e2e_ms, e2e_steps, unique=None):
    mean = statistics.mean(per_call)
    achieved = kvb / (mean * 1e-3) / 1e9
    d = {"workload": describe(b.wl), "kv_bytes_per_step": kvb,
         "step_us": steps_ms / n_steps * 1e3, "step_gbs": kvb * n_steps / (steps_ms * 1e-3) / 1e9,
         "decode_us_mean": mean * 1e3, "decode_us_median": statistics.median(per_call) * 1e3,
         "decode_us_min": min(per_call) * 1e3, "decode_calls": len(per_call),
         "decode_gbs": achieved, "frac_of_measured_peak": achieved / peak, "frac_of_8tbs_spec": achieved / SPEC_HBM_GBS,
         "decode_us_cold_l2_mean": statistics.mean(cold) * 1e3, "cold_l2_calls": len(cold),
         "decode_gbs_cold_l2": kvb / (statistics.mean(cold) * 1e-3) / 1e9,
         "e2e_gbs": kvb * e2e_steps / (e2e_ms * 1e-3) / 1e9, "e2e_us_per_step": e2e_ms / e2e_steps * 1e3}
    d["frac_cold_l2_of_measured_peak"] = d["decode_gbs_cold_l2"] / peak
    if unique is not None and unique != kvb:
        d["unique_kv_bytes_per_step"] = unique
        d["decode_gbs_unique"] = unique / (mean * 1e-3) / 1e9
        d["frac_unique_of_measured_peak"] = d["decode_gbs_unique"] / peak
        d["decode_gbs_unique_cold_l2"] = unique / (statistics.mean(cold) * 1e-3) / 1e9
    return d


def measure_config(lib, libpaged, wl, dev, peak, flush, seconds=0.5):
    """Timings of one workload for the per-workload table: back-to-back steps
    and per-call decode (each about `seconds` of device time), decode with a
    flushed L2 before every call, and the end-to-end host step."""
    import torch

    b = DecodeBench(lib, libpaged, wl, dev)
    for _ in range(5):
        b.step()
    b.check_flags()
    one = b.time_back_to_back(b.step, 5) / 5
    n = b.calls_for(seconds, one)
    steps_ms = b.time_back_to_back(b.step, n)
    per_call = b.time_each_decode(n)
    cold = b.time_each_decode(min(200, n), flush=flush)
    for _ in range(3):
        b.e2e_step()
    ne = max(20, n // 4)
    e2e_ms = b.time_e2e(ne)
    b.check_flags()
    b.check_e2e_output()
    res = decode_summary(b, wl.kv_bytes(), steps_ms, n, per_call, cold, peak, e2e_ms, ne, wl.unique_kv_bytes())
    del b
    torch.cuda.empty_cache()
    return res


PER_CONFIG = [(2, None), (3, 8), (3, 16), (3, 32), (3, 64), (4, None), (0, None)]


def run_ours(args):
    import torch

    from paged_kv_cache_368_b200 import build as pbuild
    from paged_kv_cache_368_b200 import inputs, libpaged

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
    dev = torch.device("cuda", local)
    peak, peak_src = measured_peak()
    flush = torch.ones(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    wl = load_workload(args)
    b = DecodeBench(lib, libpaged, wl, dev)
    K, W = args.steps, args.warmup
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}")
    time.sleep(0.3)
    for _ in range(W):
        b.step()
    b.check_flags()

    # ---- timed region 1: exactly K whole steps, bracketed by a barrier and
    # a synchronize, one event pair (max over ranks)
    if dist is not None:
        dist.barrier()
    t_wall0 = time.time()
    elapsed_ms = reduce_max(b.time_back_to_back(b.step, K), dist, dev)

    # ---- timed region 2 (roofline of the dominant kernel): an event pair
    # around every pa_decode call, at least K calls and about 1 s of device
    # time, so that the clock samples (every 100 ms) fall inside it
    if dist is not None:
        dist.barrier()
    n_roof = max(K, b.calls_for(args.roofline_seconds, elapsed_ms / K))
    dec_ms = b.time_each_decode(n_roof)
    t_wall1 = time.time()
    cold_ms = b.time_each_decode(min(200, n_roof), flush=flush)

    # ---- end to end through the public API (pa_decode_step_host)
    Ke = min(K, 2000)
    for _ in range(max(3, W)):
        b.e2e_step()
    if dist is not None:
        dist.barrier()
    e2e_ms = reduce_max(b.time_e2e(Ke), dist, dev)
    b.check_flags()
    b.check_e2e_output()
    clocks.stop()

    kvb = wl.kv_bytes()
    value = throughput_gbs(kvb, world, K, elapsed_ms)
    head = decode_summary(b, kvb, elapsed_ms, K, dec_ms, cold_ms, peak, e2e_ms, Ke, wl.unique_kv_bytes())
    src = kernel_source_hash()
    tr = NCU_TRAFFIC.get(wl.name)
    traffic = tr["bytes"] if tr and tr.get("src") == src else None
    h2d, d2h = b.h2d, b.d2h
    del b
    torch.cuda.empty_cache()

    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = {}
        for ci, bs in PER_CONFIG:
            if ci == args.config and bs == args.block_size:
                continue
            w2 = inputs.config(ci, block_size=bs)
            res = measure_config(lib, libpaged, w2, dev, peak, flush)
            tr2 = NCU_TRAFFIC.get(w2.name)
            res["traffic"] = tr2["bytes"] if tr2 and tr2.get("src") == src else None
            per_config[w2.name] = res

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
                   "l2": (f"inputs larger than L2 ({kvb / 2**20:.0f} MiB of KV per step vs 126 MiB L2), no flush "
                          "between timed steps; decode_us_cold_l2 reads a 252 MiB buffer before every call"),
                   "parallelism": f"{world} independent replica(s), one per GPU",
                   "step": "append (pa_reshape_and_cache) + decode with in-launch merge (pa_decode)"},
        "roofline": {"bound": "hbm", "achieved": head["decode_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": head["decode_gbs"] / peak, "traffic": traffic,
                     "kernel": "paged_decode_kernel (pa_decode: one launch, merge included)",
                     "timing": (f"CUDA events around each of {len(dec_ms)} pa_decode calls (>= 1 s of device time) "
                                "on the launching stream, after the step's append"),
                     "peak_source": peak_src, "frac_of_8tbs_spec": head["decode_gbs"] / SPEC_HBM_GBS,
                     "decode_us_mean": head["decode_us_mean"], "decode_us_median": head["decode_us_median"],
                     "decode_us_min": head["decode_us_min"], "decode_us_cold_l2_mean": head["decode_us_cold_l2_mean"],
                     "frac_cold_l2": head["frac_cold_l2_of_measured_peak"], "kernel_src": src},
        "cpu_baseline": cpu,
        "e2e": {"value": throughput_gbs(kvb, world, Ke, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke, "ms_per_step": e2e_ms / Ke,
                "path": ("pa_decode_step_host_pipelined (C ABI): every step copies its packed pinned host inputs "
                         "to the device (1 copy, on a second stream, overlapping the previous step's kernels), "
                         "appends, decodes and copies the output to pinned host memory (1 copy, on a third "
                         "stream, overlapping the next step's kernels); the timed region ends after the last "
                         "output copy")},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "per_config": per_config,
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
    if BLOCK_COPY_NCU["src"] == block_copy_source_hash():
        # two launches per call (K and V pools)
        line["roofline"]["traffic"] = 2 * (BLOCK_COPY_NCU["read"] + BLOCK_COPY_NCU["write"])
        line["roofline"]["traffic_note"] = ("ncu, per launch: reads equal the copied bytes; 65 % of the "
                                            "writes reach DRAM before the launch ends, the rest leave L2 later")
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
    peak_source = ("MEASURED_PEAKS.json bf16_tflops (cuBLAS burst)" if "bf16_tflops" in peaks
                   else "fallback (1.59 PFLOP/s, earlier cuBLAS burst measurement on this pool)")
    peak_sus = float(peaks.get("bf16_tflops_sustained", 1400.0))
    peak_sus_source = ("MEASURED_PEAKS.json bf16_tflops_sustained (cuBLAS, seconds under the power cap)"
                       if "bf16_tflops_sustained" in peaks
                       else "fallback (~1.4 PFLOP/s, cuBLAS sustained under the power cap on this pool)")
    psrc = prefill_source_hash()
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

        def timed(legacy, seconds):
            """ms per call over at most K calls and about `seconds` of device
            time.  Seconds of back-to-back tensor work bring the power cap's
            lower clocks, so a short burst is set against the burst peak and a
            long run against the sustained one."""
            for _ in range(W):
                call(legacy)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call(legacy)
            e1.record()
            torch.cuda.synchronize(dev)
            n = max(1, min(K, int(seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
            e0.record()
            for _ in range(n):
                call(legacy)
            e1.record()
            torch.cuda.synchronize(dev)
            calls[(legacy, seconds)] = n
            return e0.elapsed_time(e1) / n

        calls = {}
        ms = timed(False, PREFILL_BURST_S)
        ms_mma = timed(True, PREFILL_BURST_S)
        ms_sus = timed(False, PREFILL_SUSTAINED_S)
        # causal FLOPs: row at position p does 2 * 2 * D * (p + 1) per q-head (QK and PV)
        flops = 0
        for n, c in zip(qlen, ctx):
            pos = np.arange(c - n, c, dtype=np.float64)
            flops += float(4.0 * D * H * (pos + 1).sum())
        tf = flops / (ms * 1e-3) / 1e12
        res = {"workload": name, "us": ms * 1e3, "tflops": tf, "frac_of_bf16_peak": tf / peak,
               "kv_bytes_logical": wl.kv_bytes(), "flops": flops, "kernel": "tcgen05",
               "mma_sync_us": ms_mma * 1e3, "mma_sync_tflops": flops / (ms_mma * 1e-3) / 1e12,
               "timed_calls": calls[(False, PREFILL_BURST_S)], "mma_sync_timed_calls": calls[(True, PREFILL_BURST_S)],
               "sustained": {"us": ms_sus * 1e3, "tflops": flops / (ms_sus * 1e-3) / 1e12,
                             "calls": calls[(False, PREFILL_SUSTAINED_S)], "peak": peak_sus,
                             "frac": flops / (ms_sus * 1e-3) / 1e12 / peak_sus, "peak_source": peak_sus_source},
               "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                            "traffic": None, "kernel_src": psrc}}
        tr = PREFILL_NCU_TRAFFIC.get("chunked" if name.startswith("chunked") else "d64")
        if tr and tr["src"] == psrc:
            res["roofline"]["traffic"] = tr["bytes"]
        else:
            res["roofline"]["traffic_note"] = "no ncu capture of this kernel version on this workload"
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = prefill_cpu_baseline(wl, q, qlen, ctx, H, KVH, D, dtype)
        results.append(res)
    line = {"metric": "pa_prefill causal attention TFLOP/s", "op": "prefill", "n_gpus": 1, "steps": K, "warmup": W,
            "peak_tflops": peak, "peak_source": peak_source,
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
    ap.add_argument("--roofline-seconds", type=float, default=1.0,
                    help="device time of the per-call roofline pass (at least K calls); 0 for profiler runs")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload table (all five workloads, LLaMA-13B at block sizes 8-64)")
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
