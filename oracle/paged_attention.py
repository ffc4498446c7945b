"""Float64 CPU oracle for paged decode attention and the cache-append step.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of ``bench.py`` may
import it.  It shares no code with the CUDA library and imports nothing from
it.

What it follows (page titles as published):

* "【infra之路】10-PagedAttention 与 KV Cache 管理"
  - section 1.1: decode attention of one new query against all cached keys,
    ``softmax(Q_t [K_1..K_t]^T / sqrt(d)) [V_1..V_t]``;
  - section 1.2: the new token's K/V are appended to the cache before the
    attention of the same step reads it;
  - section 3.2/3.3: a block holds ``block_size`` consecutive tokens; a
    per-sequence block table maps logical block ``i`` to a physical block;
  - section 3.4: attention reads each physical block through the table and
    the result is an ordinary attention over the gathered keys/values.
* "PagedAttention：KV Cache 的分页革命", page-table diagram: logical block ->
  physical page, physically scattered, logically contiguous.

Paging only moves bytes; the method computes exact attention.  So the
oracle is the plain definition: gather the logical sequence through the
table, then textbook softmax attention in float64.

Readings where the pages are silent or garbled (each is pinned by a test):

* ``context_lens[s]`` counts the token appended in this step; that token sits
  at position ``ctx - 1``.
* The last block may be partly filled: only positions ``< ctx`` are read
  (the section 3.4 pseudocode multiplies whole blocks, which would read
  unwritten slots).
* K and V live in two pools ``[num_blocks, num_kv_heads, block_size, d]``.
* One table per sequence, shared by all kv-heads; q-head ``h`` reads kv-head
  ``h // (H / KVH)``.
* A negative slot in ``slot_mapping`` is skipped.  ``ctx == 0`` gives zeros.
"""
from __future__ import annotations

import numpy as np


def widen(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of fp16/bf16 bit patterns (uint16 or int16 arrays)."""
    bits = np.ascontiguousarray(raw).view(np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def slot_of_position(table_row, position: int, block_size: int) -> int:
    """Flat slot of logical token ``position``: physical block
    ``table_row[position // block_size]`` at offset ``position % block_size``
    (block table, section 3.3 of the tutorial; physical address =
    block id x page size on the ops-transformer page)."""
    return int(table_row[position // block_size]) * block_size + position % block_size


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping):
    """Append step: token ``n`` goes to slot ``s = slot_mapping[n]``, i.e. block
    ``s // bs`` at offset ``s % bs``, for every kv-head.  Negative slots are
    skipped.  Works on raw 16-bit patterns and returns new arrays, so the
    comparison with a device pool is bytewise."""
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    bs = k_cache.shape[2]
    for n, s in enumerate(np.asarray(slot_mapping).tolist()):
        if s < 0:
            continue
        k_out[s // bs, :, s % bs, :] = key[n]
        v_out[s // bs, :, s % bs, :] = value[n]
    return k_out, v_out


def gather(cache, table_row, ctx: int, dtype: str) -> np.ndarray:
    """Logical K (or V) of one sequence as float64 ``[kvh, ctx, d]``.

    Token ``i`` is read from physical block ``table_row[i // bs]`` at offset
    ``i % bs``; only the first ``ceil(ctx / bs)`` table entries are touched."""
    bs = cache.shape[2]
    kvh, d = cache.shape[1], cache.shape[3]
    if ctx == 0:
        return np.zeros((kvh, 0, d))
    pos = np.arange(ctx)
    phys = np.asarray(table_row)[pos // bs].astype(np.int64)
    rows = cache[phys, :, pos % bs, :]  # [ctx, kvh, d]
    return widen(rows, dtype).transpose(1, 0, 2)


def attend(q64: np.ndarray, k64: np.ndarray, v64: np.ndarray, scale: float) -> np.ndarray:
    """Decode attention of one sequence (section 1.1 formula, float64).

    ``q64 [H, d]``, ``k64/v64 [kvh, L, d]``; q-head ``h`` uses kv-head
    ``h // (H / kvh)``.  Scores ``s = scale * q . k``; weights
    ``exp(s - max s) / sum exp(s - max s)`` (subtracting the max is an
    identity, not an approximation); output ``weights @ V``."""
    H, d = q64.shape
    kvh, L, _ = k64.shape
    out = np.zeros((H, d))
    if L == 0:
        return out
    G = H // kvh
    for h in range(H):
        kh = h // G
        s = float(scale) * (k64[kh] @ q64[h])  # [L]
        w = np.exp(s - s.max())
        w /= w.sum()
        out[h] = w @ v64[kh]
    return out


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype: str) -> np.ndarray:
    """Paged decode attention for every sequence: float64 ``[S, H, d]``.

    ``q`` holds raw 16-bit patterns ``[S, H, d]``; the pools are raw
    ``[NB, kvh, bs, d]``; ``scale`` is widened exactly from float32."""
    S, H, d = q.shape
    out = np.zeros((S, H, d))
    sc = float(np.float32(scale))
    for s in range(S):
        L = int(context_lens[s])
        if L <= 0:
            continue
        k64 = gather(k_cache, block_tables[s], L, dtype)
        v64 = gather(v_cache, block_tables[s], L, dtype)
        out[s] = attend(widen(q[s], dtype), k64, v64, sc)
    return out


def decode_step(q, key, value, k_cache, v_cache, slot_mapping, block_tables, context_lens, scale, dtype):
    """One decode step as the tutorial's section 1.2 orders it: append the new
    K/V, then attend over the cache that now holds them.  Returns
    ``(out64, k_cache_after, v_cache_after)``."""
    k2, v2 = reshape_and_cache(key, value, k_cache, v_cache, slot_mapping)
    return decode(q, k2, v2, block_tables, context_lens, scale, dtype), k2, v2


def prefill(q, cu_q, k_cache, v_cache, block_tables, context_lens, scale, dtype: str) -> np.ndarray:
    """Multi-token paged attention (a prompt chunk, or several new tokens):
    float64 ``[total_q, H, d]``.

    Sequence s owns query rows ``cu_q[s] .. cu_q[s+1]-1``; its ``n = cu_q[s+1]
    - cu_q[s]`` new tokens are the last n of its ``context_lens[s]`` cached
    positions (their K/V are already appended), so query row i sits at
    position ``p = ctx - n + i`` and attends to cached positions ``0..p``
    (causal).  This is the ops-transformer page's multi-token call (query
    ``[batch, heads, seq_len, head_dim]`` against the paged cache), each row
    computed by the section 1.1 formula of the tutorial."""
    total, H, d = q.shape
    out = np.zeros((total, H, d))
    sc = float(np.float32(scale))
    for s in range(len(context_lens)):
        lo, hi = int(cu_q[s]), int(cu_q[s + 1])
        L = int(context_lens[s])
        n = hi - lo
        if n == 0 or L == 0:
            continue
        k64 = gather(k_cache, block_tables[s], L, dtype)
        v64 = gather(v_cache, block_tables[s], L, dtype)
        for i in range(n):
            p = L - n + i
            out[lo + i] = attend(widen(q[lo + i], dtype), k64[:, : p + 1], v64[:, : p + 1], sc)
    return out
