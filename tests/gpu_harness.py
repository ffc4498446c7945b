"""Helpers for the GPU parity tests: upload a seeded workload, run the library
through its C ABI, and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_368_b200 import inputs, libpaged

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16}

# Attention-output tolerance against the float64 oracle: |gpu - ref| <= atol + rtol*|ref|.
TOL = {"f16": (2e-3, 1e-2), "bf16": (1.6e-2, 2e-2)}


def to_dev(raw: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(raw).view(np.int16).copy())
    return t.view(TORCH_DT[dtype]).cuda()


def to_raw(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class DeviceState:
    """One decode step's state on the GPU."""

    def __init__(self, wl: inputs.Workload, poison: bool = True, full_pool: bool = None):
        self.wl = wl
        dt = TORCH_DT[wl.dtype]
        shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, wl.head_dim)
        if full_pool is None:
            full_pool = np.prod(shape) <= (1 << 24)
        self.host_pool = None
        if full_pool:
            k, v = wl.full_pool(poison=poison)
            self.host_pool = (k, v)
            self.k_cache = to_dev(k, wl.dtype)
            self.v_cache = to_dev(v, wl.dtype)
        else:
            fill = float("nan") if poison else 0.0
            self.k_cache = torch.full(shape, fill, dtype=dt, device="cuda")
            self.v_cache = torch.full(shape, fill, dtype=dt, device="cuda")
            idx = torch.from_numpy(wl.used).cuda()
            self.k_cache.index_copy_(0, idx, to_dev(wl.k_blocks, wl.dtype))
            self.v_cache.index_copy_(0, idx, to_dev(wl.v_blocks, wl.dtype))
        self.q = to_dev(wl.q, wl.dtype)
        self.k_new = to_dev(wl.k_new, wl.dtype)
        self.v_new = to_dev(wl.v_new, wl.dtype)
        self.slots = torch.from_numpy(wl.slot_mapping.astype(np.int64)).cuda()
        self.tables = torch.from_numpy(wl.block_tables.astype(np.int32)).cuda()
        self.ctx = torch.from_numpy(wl.context_lens.astype(np.int32)).cuda()
        self.out = torch.full_like(self.q, float("nan"))
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.ws = libpaged.alloc_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                           max(1, wl.max_context_len))

    def append(self):
        libpaged.reshape_and_cache(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slots, err_flags=self.err)

    def decode(self, max_ctas: int = 0, out=None):
        out = self.out if out is None else out
        libpaged.decode(out, self.q, self.k_cache, self.v_cache, self.tables, self.ctx, float(self.wl.scale),
                        max_context_len=max(1, self.wl.max_context_len), workspace=self.ws, max_ctas=max_ctas,
                        err_flags=self.err)
        return out

    def step(self, max_ctas: int = 0):
        self.append()
        self.decode(max_ctas)
        torch.cuda.synchronize()
        return to_raw(self.out)


def reference_full(wl: inputs.Workload, poison: bool = True):
    """Oracle for the whole workload on the full (small) pool: (out64, k_after, v_after)."""
    k, v = wl.full_pool(poison=poison)
    return oracle.decode_step(wl.q, wl.k_new, wl.v_new, k, v, wl.slot_mapping, wl.block_tables, wl.context_lens,
                              wl.scale, wl.dtype)


def reference_sampled(wl: inputs.Workload, seqs, kv_heads=None):
    """Oracle output for selected sequences (and kv-heads), on a small pool of
    only their blocks.  Returns {(seq, q_head): out64[D]}."""
    G = wl.num_heads // wl.num_kv_heads
    kc, vc, tc = wl.compact(seqs)
    slots = np.array([oracle.slot_of_position(tc[r], int(wl.context_lens[s]) - 1, wl.block_size)
                      for r, s in enumerate(seqs)], dtype=np.int64)
    kc2, vc2 = oracle.reshape_and_cache(wl.k_new[seqs], wl.v_new[seqs], kc, vc, slots)
    heads = range(wl.num_kv_heads) if kv_heads is None else kv_heads
    res = {}
    for h in heads:
        out = oracle.decode(wl.q[seqs][:, h * G:(h + 1) * G], kc2[:, h:h + 1], vc2[:, h:h + 1], tc,
                            wl.context_lens[seqs], wl.scale, wl.dtype)
        for r, s in enumerate(seqs):
            for g in range(G):
                res[(s, h * G + g)] = out[r, g]
    return res


def assert_close(gpu_raw: np.ndarray, ref64: np.ndarray, dtype: str, where: str = ""):
    g = oracle.widen(gpu_raw, dtype)
    assert np.isfinite(g).all(), f"{where}: non-finite output"
    atol, rtol = TOL[dtype]
    err = np.abs(g - ref64)
    bad = err > atol + rtol * np.abs(ref64)
    assert not bad.any(), (f"{where}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"max abs err {err.max():.3e}")
    return float(err.max())
