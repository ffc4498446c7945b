"""Seeded synthetic inputs for paged decode attention.

This module only lays out synthetic state: it draws numbers and places them
in a block pool the way a block manager would.  It holds none of the
attention arithmetic and is shared, unchanged, by the float64 oracle tests,
the GPU parity tests and the benchmark.

State produced for one decode step (shapes follow the kernel boundary):

* ``context_lens`` int32 ``[S]`` -- tokens per sequence, counting the token
  appended in this step (position ``ctx - 1``).
* ``block_tables`` int32 ``[S, MB]`` -- per-sequence list of physical block
  ids, logical block ``i`` first (the block table of "【infra之路】10-PagedAttention
  与 KV Cache 管理", section 3.3).  Entries past ``ceil(ctx / bs)`` are filler.
* ``slot_mapping`` int64 ``[S]`` -- flat slot (``block_id * bs + offset``) of
  each sequence's new token.
* ``q`` ``[S, H, D]``, ``k_new``/``v_new`` ``[S, KVH, D]`` -- raw 16-bit
  patterns (fp16 or bf16) of N(0, 1) draws.
* ``used`` int64 ``[U]`` and ``k_blocks``/``v_blocks`` ``[U, KVH, BS, D]`` --
  the physical blocks that hold history, with their contents.  Slots at
  positions ``>= ctx - 1`` (the slot the append step writes, and the unused
  tail of the last block) hold NaN when ``poison=True``.

Random streams: one ``numpy.random.SeedSequence(seed)`` child per tensor, so
adding a tensor never shifts another tensor's draw.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

F16_NAN = 0x7E00
BF16_NAN = 0x7FC0

DTYPES = ("f16", "bf16")


def _to_raw16(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 samples to the 16-bit storage type; return the bit patterns."""
    if dtype == "f16":
        return x32.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch  # torch's CPU cast rounds to nearest even

        return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(f"unknown dtype {dtype!r}")


def _normal_raw16(rng: np.random.Generator, shape, dtype: str, chunk: int = 1 << 24) -> np.ndarray:
    """N(0, 1) float32 draws cast to fp16/bf16 bits, generated in chunks to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        out[lo:hi] = _to_raw16(rng.standard_normal(hi - lo, dtype=np.float32), dtype)
    return out.reshape(shape)


def nan_bits(dtype: str) -> int:
    return F16_NAN if dtype == "f16" else BF16_NAN


@dataclasses.dataclass
class Workload:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    scale: np.float32
    context_lens: np.ndarray  # int32 [S]
    block_tables: np.ndarray  # int32 [S, MB]
    slot_mapping: np.ndarray  # int64 [S]
    q: np.ndarray  # uint16 [S, H, D]
    k_new: np.ndarray  # uint16 [S, KVH, D]
    v_new: np.ndarray  # uint16 [S, KVH, D]
    used: np.ndarray  # int64 [U] physical ids holding history
    k_blocks: np.ndarray  # uint16 [U, KVH, BS, D]
    v_blocks: np.ndarray  # uint16 [U, KVH, BS, D]
    shared_prefix_blocks: int = 0
    group_size: int = 1

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def elem_bytes(self) -> int:
        return 2

    def kv_bytes(self) -> int:
        """Logical K+V bytes one decode step reads: sum over sequences of
        ctx * kv_heads * head_dim * 2 (K and V) * element size."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * 2 * self.elem_bytes

    def unique_kv_bytes(self) -> int:
        """Physical K+V bytes when shared-prefix blocks are counted once."""
        if not self.shared_prefix_blocks:
            return self.kv_bytes()
        groups = self.num_seqs // self.group_size
        dup_tokens = groups * (self.group_size - 1) * self.shared_prefix_blocks * self.block_size
        return self.kv_bytes() - dup_tokens * self.num_kv_heads * self.head_dim * 2 * self.elem_bytes

    def full_pool(self, poison: bool = True):
        """Materialise the whole pool as numpy ``[NB, KVH, BS, D]`` uint16 arrays.

        Unused blocks hold NaN when ``poison`` (else zero).  Only sensible for
        small pools."""
        shape = (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)
        fill = nan_bits(self.dtype) if poison else 0
        k = np.full(shape, fill, dtype=np.uint16)
        v = np.full(shape, fill, dtype=np.uint16)
        k[self.used] = self.k_blocks
        v[self.used] = self.v_blocks
        return k, v

    def compact(self, seqs: Optional[Sequence[int]] = None):
        """A small pool holding only the blocks of ``seqs`` (default: all).

        Returns ``(k_pool, v_pool, tables)`` with the tables renumbered into the
        small pool.  Renumbering physical blocks does not change what a
        sequence reads, so the oracle may run on this pool."""
        seqs = list(range(self.num_seqs)) if seqs is None else list(seqs)
        pos_of = {int(p): i for i, p in enumerate(self.used)}
        need: List[int] = []
        seen = {}
        tables = np.full((len(seqs), self.max_blocks_per_seq), -1, dtype=np.int32)
        for r, s in enumerate(seqs):
            nb = -(-int(self.context_lens[s]) // self.block_size)
            for i in range(nb):
                p = int(self.block_tables[s, i])
                if p not in seen:
                    seen[p] = len(need)
                    need.append(p)
                tables[r, i] = seen[p]
        idx = np.array([pos_of[p] for p in need], dtype=np.int64)
        return self.k_blocks[idx], self.v_blocks[idx], tables


def _draw_contexts(rng, n, kind, lo, hi):
    if kind == "fixed":
        return np.full(n, lo, dtype=np.int64)
    if kind == "uniform":
        return rng.integers(lo, hi + 1, n).astype(np.int64)
    if kind == "loguniform":
        x = np.exp(rng.uniform(math.log(lo), math.log(hi), n))
        return np.clip(np.floor(x).astype(np.int64), lo, hi)
    raise ValueError(kind)


def build(
    name: str,
    *,
    seed: int,
    num_seqs: int,
    num_heads: int,
    num_kv_heads: int,
    head_dim: int,
    block_size: int,
    dtype: str,
    context_lens: Optional[Sequence[int]] = None,
    ctx_kind: str = "fixed",
    ctx_lo: int = 1,
    ctx_hi: int = 1,
    pool_blocks: Optional[int] = None,
    pool_factor: float = 1.25,
    shared_prefix_blocks: int = 0,
    group_size: int = 1,
    poison: bool = True,
    table_filler: int = -1,
    data: bool = True,
) -> Workload:
    """Lay out one synthetic decode step.

    ``context_lens`` (or a draw of kind ``ctx_kind`` in ``[ctx_lo, ctx_hi]``)
    counts the appended token.  Physical blocks are handed out in the order of
    a seeded permutation of the pool.  With ``shared_prefix_blocks = P`` and
    ``group_size = g``, each run of g consecutive sequences maps logical
    blocks ``0..P-1`` to the same physical blocks (a shared prompt prefix);
    the new token of every sequence must then lie past the prefix.
    ``data=False`` skips the pool contents (metadata only).
    """
    if dtype not in DTYPES:
        raise ValueError(dtype)
    ss = np.random.SeedSequence(seed)
    r_ctx, r_perm, r_q, r_knew, r_vnew, r_k, r_v, r_fill = [np.random.default_rng(c) for c in ss.spawn(8)]

    S, bs = num_seqs, block_size
    if context_lens is not None:
        ctx = np.asarray(context_lens, dtype=np.int64)
        assert ctx.shape == (S,)
    else:
        ctx = _draw_contexts(r_ctx, S, ctx_kind, ctx_lo, ctx_hi)
    nblk = -(-ctx // bs)  # ceil
    if shared_prefix_blocks:
        assert S % group_size == 0
        assert np.all(ctx - 1 >= shared_prefix_blocks * bs), "appended token would land in a shared block"
        assert np.all(nblk >= shared_prefix_blocks)
        groups = S // group_size
        needed = int(nblk.sum()) - groups * (group_size - 1) * shared_prefix_blocks
    else:
        needed = int(nblk.sum())
    if pool_blocks is None:
        pool_blocks = max(1, int(math.ceil(needed * pool_factor)))
    assert pool_blocks >= needed, (pool_blocks, needed)

    perm = r_perm.permutation(pool_blocks).astype(np.int64)
    MB = max(1, int(nblk.max()) if S else 1)
    tables = np.full((S, MB), table_filler, dtype=np.int64)
    if table_filler == -2:  # random junk in unused entries, including ids out of range
        tables = r_fill.integers(-(1 << 30), 1 << 30, (S, MB)).astype(np.int64)
    cursor = 0
    prefix_ids = None
    for s in range(S):
        first = 0
        if shared_prefix_blocks:
            if s % group_size == 0:
                prefix_ids = perm[cursor : cursor + shared_prefix_blocks]
                cursor += shared_prefix_blocks
            tables[s, :shared_prefix_blocks] = prefix_ids
            first = shared_prefix_blocks
        n = int(nblk[s]) - first
        tables[s, first : first + n] = perm[cursor : cursor + n]
        cursor += n
    assert cursor == needed
    used = perm[:needed].copy()

    # The new token of sequence s sits at position ctx-1: the block that holds
    # it is logical block (ctx-1)//bs, at offset (ctx-1)%bs.
    slots = np.full(S, -1, dtype=np.int64)
    for s in range(S):
        if ctx[s] > 0:
            p = int(ctx[s]) - 1
            slots[s] = int(tables[s, p // bs]) * bs + p % bs

    q = _normal_raw16(r_q, (S, num_heads, head_dim), dtype)
    k_new = _normal_raw16(r_knew, (S, num_kv_heads, head_dim), dtype)
    v_new = _normal_raw16(r_vnew, (S, num_kv_heads, head_dim), dtype)
    if data:
        k_blocks = _normal_raw16(r_k, (needed, num_kv_heads, bs, head_dim), dtype)
        v_blocks = _normal_raw16(r_v, (needed, num_kv_heads, bs, head_dim), dtype)
    else:
        k_blocks = np.zeros((0, num_kv_heads, bs, head_dim), dtype=np.uint16)
        v_blocks = np.zeros((0, num_kv_heads, bs, head_dim), dtype=np.uint16)

    if poison and data:
        # Slots at positions >= ctx-1 are not history: NaN them so that a
        # kernel reading past the context (or the slot before the append)
        # shows up as a non-finite output.
        row_of = {int(p): i for i, p in enumerate(used)}
        nanv = nan_bits(dtype)
        for s in range(S):
            if ctx[s] <= 0:
                continue
            p = int(ctx[s]) - 1
            for pos in range(p, int(nblk[s]) * bs):
                i = row_of[int(tables[s, pos // bs])]
                k_blocks[i, :, pos % bs, :] = nanv
                v_blocks[i, :, pos % bs, :] = nanv

    return Workload(
        name=name,
        num_seqs=S,
        num_heads=num_heads,
        num_kv_heads=num_kv_heads,
        head_dim=head_dim,
        block_size=bs,
        dtype=dtype,
        num_blocks=int(pool_blocks),
        scale=np.float32(1.0) / np.sqrt(np.float32(head_dim)),
        context_lens=ctx.astype(np.int32),
        block_tables=tables.astype(np.int32),
        slot_mapping=slots,
        q=q,
        k_new=k_new,
        v_new=v_new,
        used=used,
        k_blocks=k_blocks,
        v_blocks=v_blocks,
        shared_prefix_blocks=shared_prefix_blocks,
        group_size=group_size,
    )


CONFIG_NAMES = (
    "tiny-mha",
    "llama7b-mha",
    "llama3-8b-gqa",
    "llama13b-mha",
    "long-context-shared-prefix",
)

# Seeds are 368 + the config's index.
SEED_BASE = 368


def config(index: int, *, block_size: Optional[int] = None, poison: bool = True, data: bool = True) -> Workload:
    """The five synthetic decode workloads, shaped like the pages' models.

    0 tiny MHA: 4 seqs, 4 heads, d 64, bs 16, ctx {1,17,50,128}, fp16, pool 64.
    1 LLaMA-7B layer: 32 seqs, 32/32 heads, d 128, bs 16, ctx U[128,2048],
      fp16, pool 8400 blocks (the A100 sizing of the tutorial's section 5).
    2 LLaMA-3-8B GQA layer: 64 seqs, 32 q / 8 kv heads, d 128, bs 16,
      ctx U[512,8192], bf16, pool 1.25x needed.
    3 LLaMA-13B layer: 8 seqs, 40/40 heads, d 128, ctx 4096, fp16,
      bs in {8,16,32,64} (default 16), pool 2x needed.
    4 long context + shared prefix: 16 seqs, 64 q / 8 kv heads, d 128, bs 16,
      bf16, ctx log-uniform [1025, 65536], groups of 4 sharing 64 blocks.
    """
    seed = SEED_BASE + index
    if index == 0:
        return build("tiny-mha", seed=seed, num_seqs=4, num_heads=4, num_kv_heads=4, head_dim=64,
                     block_size=16, dtype="f16", context_lens=[1, 17, 50, 128], pool_blocks=64, poison=poison, data=data)
    if index == 1:
        return build("llama7b-mha", seed=seed, num_seqs=32, num_heads=32, num_kv_heads=32, head_dim=128,
                     block_size=16, dtype="f16", ctx_kind="uniform", ctx_lo=128, ctx_hi=2048,
                     pool_blocks=8400, poison=poison, data=data)
    if index == 2:
        return build("llama3-8b-gqa", seed=seed, num_seqs=64, num_heads=32, num_kv_heads=8, head_dim=128,
                     block_size=16, dtype="bf16", ctx_kind="uniform", ctx_lo=512, ctx_hi=8192,
                     pool_factor=1.25, poison=poison, data=data)
    if index == 3:
        bs = 16 if block_size is None else block_size
        return build(f"llama13b-mha-bs{bs}", seed=seed, num_seqs=8, num_heads=40, num_kv_heads=40,
                     head_dim=128, block_size=bs, dtype="f16", ctx_kind="fixed", ctx_lo=4096,
                     pool_factor=2.0, poison=poison, data=data)
    if index == 4:
        return build("long-context-shared-prefix", seed=seed, num_seqs=16, num_heads=64, num_kv_heads=8,
                     head_dim=128, block_size=16, dtype="bf16", ctx_kind="loguniform", ctx_lo=1025,
                     ctx_hi=65536, pool_factor=1.25, shared_prefix_blocks=64, group_size=4, poison=poison, data=data)
    raise ValueError(index)


def random_case(seed: int, *, num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                block_size: int, dtype: str, ctx_lo: int, ctx_hi: int, poison: bool = True,
                table_filler: int = -1, pool_factor: float = 1.5) -> Workload:
    """A small random case (uniform context lengths) for parity sweeps."""
    return build(f"random-{seed}", seed=seed, num_seqs=num_seqs, num_heads=num_heads,
                 num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size, dtype=dtype,
                 ctx_kind="uniform", ctx_lo=ctx_lo, ctx_hi=ctx_hi, pool_factor=pool_factor,
                 poison=poison, table_filler=table_filler)
