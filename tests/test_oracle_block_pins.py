"""Pins for the block-manager and block-copy oracle (``oracle/block_manager.py``):
checks against values worked out by hand from the pages' rules, never
against the library they judge.

Each ``check_*`` takes the oracle module, so that ``test_planted_mistakes``
can rerun every check on a copy of the oracle with one plausible mistake
planted (on the CPU) and show that some check rejects it.

Sources of truth:
* ``tests/golden/block_manager_scenario.json``: one pool's lifecycle (add,
  fork, append with copy on write, free);
* ``tests/golden/block_manager_swap_scenario.json``: admission counts (a full
  last block, a shared last block, a partly filled private block, two sharers
  in one batch) and swapping a sequence between two pools and back;
* ``tests/golden/block_copy_example.json``: a 4-block pool after
  ``copy_blocks`` and a 3-block pool after ``swap_blocks``, written out;
* invariants: each table holds ceil(len / block_size) blocks and the
  reference counts equal the number of tables holding each block.
"""
import random
import types

import numpy as np
import pytest

from block_scenarios import ModelAdapter, golden, run_lifecycle_scenario, run_swap_scenario
from oracle import block_manager as obm


# ---------------------------------------------------------------- checks


def check_lifecycle_scenario(mod):
    run_lifecycle_scenario(lambda n, bs: ModelAdapter(mod, n, bs), golden("block_manager_scenario.json"))


def check_swap_scenario(mod):
    run_swap_scenario(lambda n, bs: ModelAdapter(mod, n, bs), golden("block_manager_swap_scenario.json"))


def _pool(rows):
    return np.asarray(rows, dtype=np.float64)


def check_copy_blocks_example(mod):
    g = golden("block_copy_example.json")["copy"]
    pool = _pool(g["pool"])
    before = pool.copy()
    got = mod.copy_blocks(pool, [tuple(p) for p in g["pairs"]])
    np.testing.assert_array_equal(got, _pool(g["expected"]))
    np.testing.assert_array_equal(pool, before)  # the input pool is not modified


def check_swap_blocks_example(mod):
    g = golden("block_copy_example.json")["swap"]
    src, dst = _pool(g["src_pool"]), _pool(g["dst_pool"])
    got = mod.swap_blocks(src, dst, [tuple(p) for p in g["pairs"]])
    np.testing.assert_array_equal(got, _pool(g["expected"]))


def check_model_invariants(mod):
    """Random operations: tables hold exactly the blocks their lengths need,
    every block's count equals the tables holding it, free blocks are those
    with count 0, and the admission count equals the blocks the batch then
    takes (counted by hand from the free list before and after)."""
    rnd = random.Random(5)
    m = mod.BlockManagerModel(48, 4)
    live, nxt = [], 0
    for _ in range(300):
        op = rnd.random()
        try:
            if op < 0.2 or not live:
                m.add(nxt, rnd.randint(0, 12))
                live.append(nxt)
                nxt += 1
            elif op < 0.35:
                p = rnd.choice(live)
                m.fork(p, nxt)
                live.append(nxt)
                nxt += 1
            elif op < 0.45 and len(live) > 1:
                m.free(live.pop(rnd.randrange(len(live))))
            else:
                batch = rnd.sample(live, min(len(live), rnd.randint(1, 4)))
                need = m.blocks_needed_to_append(batch)
                free_before = set(m.free_blocks())
                if need > len(free_before):
                    continue
                for s in batch:
                    m.append_slot(s)
                assert len(free_before - set(m.free_blocks())) == need
        except mod.OutOfBlocks:
            continue
        refs = [0] * m.num_blocks
        for s, t in m.tables.items():
            assert len(t) == -(-m.lens[s] // m.block_size)
            for b in t:
                refs[b] += 1
        assert refs == m.refs
        assert m.free_blocks() == [b for b in range(m.num_blocks) if refs[b] == 0]


CHECKS = [check_lifecycle_scenario, check_swap_scenario, check_copy_blocks_example, check_swap_blocks_example,
          check_model_invariants]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_block_oracle_pin(check):
    check(obm)


# ---------------------------------------------------------------- planted mistakes

_Model = obm.BlockManagerModel


def _mut_copy_swapped(cache, pairs):
    out = np.array(cache, copy=True)
    for src, dst in pairs:
        out[src] = cache[dst]
    return out


def _mut_swap_blocks_swapped(src_pool, dst_pool, pairs):
    out = np.array(dst_pool, copy=True)
    for s, d in pairs:
        out[s % len(out)] = src_pool[d % len(src_pool)]
    return out


def _mut_needed_ignores_sharing(self, seqs):
    return sum(1 for s in seqs if self.lens[s] % self.block_size == 0)


def _mut_needed_counts_every_sharer(self, seqs):
    return sum(1 for s in seqs if self.lens[s] % self.block_size == 0 or self.refs[self.tables[s][-1]] > 1)


def _mut_swap_pairs_reversed(self, other, seq):
    return [(b, a) for a, b in _Model.swap_to(self, other, seq)]


def _mut_swap_keeps_source(self, other, seq):
    src = self.tables[seq]
    if len(src) > len(other.free_blocks()):
        raise obm.OutOfBlocks()
    dst = [other._take() for _ in src]
    other.tables[seq] = dst
    other.lens[seq] = self.lens[seq]
    del self.tables[seq], self.lens[seq]  # blocks never released
    return list(zip(src, dst))


def _mut_swap_frees_shared(self, other, seq):
    src = list(self.tables[seq])
    pairs = _Model.swap_to(self, other, seq)
    for b in src:
        self.refs[b] = 0  # released even while another sequence holds it
    return pairs


def _mut_swap_highest_first(self, other, seq):
    src = self.tables[seq]
    free = other.free_blocks()
    if len(src) > len(free):
        raise obm.OutOfBlocks()
    dst = sorted(free, reverse=True)[: len(src)]
    for b in dst:
        other.refs[b] = 1
    other.tables[seq] = dst
    other.lens[seq] = self.lens[seq]
    self.free(seq)
    return list(zip(src, dst))


def _mut_swap_shares_with_old_holders(self, other, seq):
    """Moving back into a pool where a former sharer lives: point at that
    sharer's blocks again instead of taking fresh ones."""
    for s, t in other.tables.items():
        if len(t) == len(self.tables[seq]) and other.lens[s] == self.lens[seq] and s != seq:
            other.tables[seq] = list(t)
            for b in t:
                other.refs[b] += 1
            other.lens[seq] = self.lens[seq]
            src = self.tables[seq]
            self.free(seq)
            return list(zip(src, t))
    return _Model.swap_to(self, other, seq)


def _mut_append_no_cow(self, seq):
    pos = self.lens[seq]
    table = self.tables[seq]
    if pos % self.block_size == 0:
        table.append(self._take())
    self.lens[seq] = pos + 1
    return table[pos // self.block_size] * self.block_size + pos % self.block_size, None


def _mut_append_cow_leaks(self, seq):
    pos = self.lens[seq]
    table = self.tables[seq]
    cow = None
    if pos % self.block_size == 0:
        table.append(self._take())
    elif self.refs[table[-1]] > 1:
        new = self._take()
        cow = (table[-1], new)
        table[-1] = new  # the shared block's count is not lowered
    self.lens[seq] = pos + 1
    return table[pos // self.block_size] * self.block_size + pos % self.block_size, cow


MUTANTS = {
    "copy_blocks_src_dst_swapped": ("copy_blocks", _mut_copy_swapped),
    "swap_blocks_src_dst_swapped": ("swap_blocks", _mut_swap_blocks_swapped),
    "needed_ignores_shared_last_block": ("BlockManagerModel.blocks_needed_to_append", _mut_needed_ignores_sharing),
    "needed_counts_every_sharer": ("BlockManagerModel.blocks_needed_to_append", _mut_needed_counts_every_sharer),
    "swap_to_pairs_reversed": ("BlockManagerModel.swap_to", _mut_swap_pairs_reversed),
    "swap_to_keeps_source_blocks": ("BlockManagerModel.swap_to", _mut_swap_keeps_source),
    "swap_to_frees_shared_blocks": ("BlockManagerModel.swap_to", _mut_swap_frees_shared),
    "swap_to_highest_id_first": ("BlockManagerModel.swap_to", _mut_swap_highest_first),
    "swap_to_reshares_blocks": ("BlockManagerModel.swap_to", _mut_swap_shares_with_old_holders),
    "append_without_copy_on_write": ("BlockManagerModel.append_slot", _mut_append_no_cow),
    "append_cow_leaks_shared_count": ("BlockManagerModel.append_slot", _mut_append_cow_leaks),
}


def _planted(attr, fn):
    """A copy of the oracle module with one function or method replaced."""
    mod = types.SimpleNamespace(**{k: getattr(obm, k) for k in dir(obm) if not k.startswith("__")})
    if attr.startswith("BlockManagerModel."):
        name = attr.split(".", 1)[1]
        mod.BlockManagerModel = type("BlockManagerModel", (obm.BlockManagerModel,), {name: fn})
    else:
        setattr(mod, attr, fn)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    mod = _planted(*MUTANTS[name])
    failed = []
    for check in CHECKS:
        try:
            check(mod)
        except (AssertionError, IndexError, KeyError, ValueError, obm.OutOfBlocks):
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
