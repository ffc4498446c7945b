"""Reference model of the block manager and of whole-block copies.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only ``tests/`` and the CPU-baseline
timing in ``bench.py`` may use it.  It shares no code with the library's C++
block manager or its copy kernels.

Follows:
* "PagedAttention：KV Cache 的分页革命", section Runtime 如何管理 KV Block: a
  pool of fixed-size blocks is created up front; a step that needs space takes
  a free block; the page table gets the new block; a finished request returns
  its blocks.
* "【infra之路】10-PagedAttention 与 KV Cache 管理", section 3.3 (a request's
  block table grows by one physical block when its last block is full),
  section 4.3 (requests sharing a prefix, and beams, point at the same
  physical blocks; a shared block is copied before it is written; preempted
  requests are swapped to CPU memory and back), section 6 (the scheduler
  admits work by the number of free blocks).

Policies the pages leave open, read the plainest way: the free block with the
smallest id is taken first; running out of blocks is an error that changes
nothing; a sequence moved to another pool gets a fresh block there for each
of its blocks, so blocks it shared stay with the other holders and are not
shared in the new pool.

Pinned in ``tests/test_oracle_block_pins.py`` against hand-worked scenarios
(``tests/golden/block_manager_*.json``, ``tests/golden/block_copy_example.json``)
with planted mistakes that the pins must reject.
"""
from __future__ import annotations

import copy

import numpy as np


class OutOfBlocks(Exception):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int):
        self.block_size = block_size
        self.num_blocks = num_blocks
        self.refs = [0] * num_blocks
        self.tables = {}  # seq -> list of physical blocks
        self.lens = {}  # seq -> tokens held

    # -- pool
    def free_blocks(self):
        return [b for b in range(self.num_blocks) if self.refs[b] == 0]

    def _take(self):
        for b in range(self.num_blocks):
            if self.refs[b] == 0:
                self.refs[b] = 1
                return b
        raise OutOfBlocks()

    # -- sequences
    def add(self, seq, num_tokens):
        assert seq not in self.tables
        need = -(-num_tokens // self.block_size)
        if need > len(self.free_blocks()):
            raise OutOfBlocks()
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lens[seq] = num_tokens

    def fork(self, parent, child):
        assert child not in self.tables and parent in self.tables
        self.tables[child] = list(self.tables[parent])
        for b in self.tables[child]:
            self.refs[b] += 1
        self.lens[child] = self.lens[parent]

    def append_slot(self, seq):
        """Returns (slot, (src, dst) or None)."""
        pos = self.lens[seq]
        table = self.tables[seq]
        cow = None
        if pos % self.block_size == 0:  # last block full, or no block yet
            table.append(self._take())
        else:
            last = table[-1]
            if self.refs[last] > 1:  # shared: copy before writing
                new = self._take()
                self.refs[last] -= 1
                table[-1] = new
                cow = (last, new)
        self.lens[seq] = pos + 1
        return table[pos // self.block_size] * self.block_size + pos % self.block_size, cow

    def free(self, seq):
        for b in self.tables.pop(seq):
            self.refs[b] -= 1
        del self.lens[seq]

    def blocks_needed_to_append(self, seqs):
        """Free blocks that appending one token to each of `seqs` takes (the
        admission count of the tutorial's section 6 scheduler).  Defined by
        doing it: the appends run on a copy whose pool can never run out, and
        the blocks they took are counted.  So a shared last block costs one
        copy per sharer in the batch except the one left holding it alone."""
        sim = copy.deepcopy(self)
        sim.num_blocks += len(seqs)
        sim.refs += [0] * len(seqs)
        before = len(sim.free_blocks())
        for s in seqs:
            sim.append_slot(s)
        return before - len(sim.free_blocks())

    def swap_to(self, other: "BlockManagerModel", seq):
        """Move `seq` into `other`'s pool; returns [(block here, block there)]."""
        src = self.tables[seq]
        if len(src) > len(other.free_blocks()):
            raise OutOfBlocks()
        dst = [other._take() for _ in src]
        other.tables[seq] = dst
        other.lens[seq] = self.lens[seq]
        self.free(seq)
        return list(zip(src, dst))


def copy_blocks(cache: np.ndarray, pairs) -> np.ndarray:
    """Copy-on-write copy: block dst becomes block src, for each (src, dst)."""
    out = np.array(cache, copy=True)
    for src, dst in pairs:
        out[dst] = cache[src]
    return out


def swap_blocks(src_pool: np.ndarray, dst_pool: np.ndarray, pairs) -> np.ndarray:
    """dst_pool with block dst replaced by src_pool's block src, for each pair."""
    out = np.array(dst_pool, copy=True)
    for s, d in pairs:
        out[d] = src_pool[s]
    return out
