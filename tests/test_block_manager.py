"""The C++ block manager (through the C ABI, no GPU needed) against the
pages' lifecycle: a hand-worked scenario, a reference model on random
operation sequences, and invariants."""
import random

import numpy as np
import pytest

from block_scenarios import LibraryAdapter, ModelAdapter, golden, run_lifecycle_scenario, run_swap_scenario
from oracle import block_manager as obm
from oracle.block_manager import BlockManagerModel, OutOfBlocks
from paged_kv_cache_368_b200 import build as pbuild
from paged_kv_cache_368_b200 import libpaged


@pytest.fixture(scope="module", autouse=True)
def _lib():
    pbuild.build()
    libpaged.load()


def test_worked_scenario_model():
    run_lifecycle_scenario(lambda n, bs: ModelAdapter(obm, n, bs), golden("block_manager_scenario.json"))


def test_worked_scenario_library():
    run_lifecycle_scenario(LibraryAdapter, golden("block_manager_scenario.json"))


def test_swap_and_admission_scenario_library():
    """The hand-worked two-pool scenario (admission counts, swapping out and
    back, no sharing after the round trip) on the C++ manager."""
    run_swap_scenario(LibraryAdapter, golden("block_manager_swap_scenario.json"))


def test_prepare_decode_admits_exactly_what_it_takes():
    """Two sharers of one partly filled block and a sequence with a full
    block need two free blocks, not three: with exactly two free the batch is
    admitted and leaves none."""
    lib = libpaged.BlockManager(6, 4)
    lib.add(0, 6)    # blocks 0, 1 (block 1 partly filled)
    lib.fork(0, 1)   # shares 0, 1
    lib.add(2, 8)    # blocks 2, 3 (full)
    assert lib.num_free == 2
    assert lib.blocks_needed_to_append([0, 1, 2]) == 2
    tables, ctx, slots, cow = lib.prepare_decode([0, 1, 2], 4)
    assert lib.num_free == 0
    assert cow.tolist() == [[1, 4]]          # sequence 0 copies block 1 into block 4
    assert slots.tolist() == [4 * 4 + 2, 1 * 4 + 2, 5 * 4 + 0]
    assert ctx.tolist() == [7, 7, 9]


def _check_invariants(model: BlockManagerModel):
    refs = [0] * model.num_blocks
    for s, t in model.tables.items():
        assert len(t) == -(-model.lens[s] // model.block_size)
        for b in t:
            refs[b] += 1
    assert refs == model.refs


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_the_model(seed):
    rnd = random.Random(seed)
    nb, bs = rnd.choice([(40, 4), (64, 16), (25, 8)])
    model = BlockManagerModel(nb, bs)
    lib = libpaged.BlockManager(nb, bs)
    live = []
    next_id = 0
    for _ in range(400):
        op = rnd.random()
        try:
            if op < 0.15 or not live:
                n = rnd.randint(0, 3 * bs)
                try:
                    model.add(next_id, n)
                except OutOfBlocks:
                    with pytest.raises(libpaged.LibpagedError) as e:
                        lib.add(next_id, n)
                    assert e.value.status == libpaged.PA_ERR_OUT_OF_BLOCKS
                    continue
                lib.add(next_id, n)
                live.append(next_id)
                next_id += 1
            elif op < 0.25:
                p = rnd.choice(live)
                model.fork(p, next_id)
                lib.fork(p, next_id)
                live.append(next_id)
                next_id += 1
            elif op < 0.35:
                s = live.pop(rnd.randrange(len(live)))
                model.free(s)
                lib.free(s)
            elif op < 0.45:
                batch = rnd.sample(live, min(len(live), rnd.randint(1, 4)))
                need = model.blocks_needed_to_append(batch)
                assert lib.blocks_needed_to_append(batch) == need
                mb = max(-(-(model.lens[s] + 1) // bs) for s in batch) + 1
                if need > len(model.free_blocks()):
                    with pytest.raises(libpaged.LibpagedError):
                        lib.prepare_decode(batch, mb)
                    continue
                tables, ctx, slots, cow = lib.prepare_decode(batch, mb)
                want_cow = []
                for i, s in enumerate(batch):
                    slot, c = model.append_slot(s)
                    assert slots[i] == slot and ctx[i] == model.lens[s]
                    assert tables[i, : len(model.tables[s])].tolist() == model.tables[s]
                    assert np.all(tables[i, len(model.tables[s]):] == -1)
                    if c:
                        want_cow.append(list(c))
                assert cow.tolist() == want_cow
            else:
                s = rnd.choice(live)
                try:
                    slot, c = model.append_slot(s)
                except OutOfBlocks:
                    with pytest.raises(libpaged.LibpagedError):
                        lib.append_slot(s)
                    continue
                got = lib.append_slot(s)
                assert got == (slot, c[0] if c else -1, c[1] if c else -1)
        finally:
            _check_invariants(model)
        assert lib.num_free == len(model.free_blocks())
        for s in live:
            assert lib.block_table(s) == model.tables[s]
            assert lib.context_len(s) == model.lens[s]


def test_swap_between_pools_matches_the_model():
    dev_m, host_m = BlockManagerModel(16, 4), BlockManagerModel(20, 4)
    dev, host = libpaged.BlockManager(16, 4), libpaged.BlockManager(20, 4)
    for mgr in (dev_m, dev):
        mgr.add(0, 9)
        mgr.add(1, 5)
        mgr.fork(0, 2)
    pairs_m = dev_m.swap_to(host_m, 2)
    pairs = dev.swap_to(host, 2)
    assert pairs.tolist() == [list(p) for p in pairs_m]
    assert dev.num_free == len(dev_m.free_blocks()) and host.num_free == len(host_m.free_blocks())
    back_m = host_m.swap_to(dev_m, 2)
    back = host.swap_to(dev, 2)
    assert back.tolist() == [list(p) for p in back_m]
    assert dev.block_table(2) == dev_m.tables[2]


def test_errors_change_nothing():
    lib = libpaged.BlockManager(4, 4)
    lib.add(0, 16)  # all four blocks
    with pytest.raises(libpaged.LibpagedError) as e:
        lib.prepare_decode([0], 8)
    assert e.value.status == libpaged.PA_ERR_OUT_OF_BLOCKS
    assert lib.context_len(0) == 16 and lib.block_table(0) == [0, 1, 2, 3]
    with pytest.raises(libpaged.LibpagedError):
        lib.add(0, 1)  # duplicate id
    with pytest.raises(libpaged.LibpagedError):
        lib.fork(7, 8)  # unknown parent
    with pytest.raises(libpaged.LibpagedError):
        lib.prepare_decode([0, 0], 8)  # same sequence twice
    lib.free(0)
    assert lib.num_free == 4
