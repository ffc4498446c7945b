"""The C++ block manager (through the C ABI, no GPU needed) against the
pages' lifecycle: a hand-worked scenario, a reference model on random
operation sequences, and invariants."""
import json
import os
import random

import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, OutOfBlocks
from paged_kv_cache_368_b200 import build as pbuild
from paged_kv_cache_368_b200 import libpaged


@pytest.fixture(scope="module", autouse=True)
def _lib():
    pbuild.build()
    libpaged.load()


def _golden():
    with open(os.path.join(os.path.dirname(__file__), "golden", "block_manager_scenario.json")) as f:
        return json.load(f)


def _run_scenario(mgr, g, is_model):
    for st in g["steps"]:
        if st["op"] == "add":
            mgr.add(st["seq"], st["tokens"])
        elif st["op"] == "fork":
            mgr.fork(st["parent"], st["child"])
        elif st["op"] == "append":
            if is_model:
                slot, cow = mgr.append_slot(st["seq"])
            else:
                slot, src, dst = mgr.append_slot(st["seq"])
                cow = (src, dst) if src >= 0 else None
            assert slot == st["slot"], st
            assert (list(cow) if cow else None) == st["cow"], st
        elif st["op"] == "free":
            mgr.free(st["seq"])
            n = len(mgr.free_blocks()) if is_model else mgr.num_free
            assert n == st["num_free"]
        if "table" in st:
            seq = st.get("seq", st.get("child"))
            t = mgr.tables[seq] if is_model else mgr.block_table(seq)
            assert t == st["table"], st
    n = len(mgr.free_blocks()) if is_model else mgr.num_free
    assert n == g["final_num_free"]


def test_worked_scenario_model():
    g = _golden()
    _run_scenario(BlockManagerModel(g["num_blocks"], g["block_size"]), g, True)


def test_worked_scenario_library():
    g = _golden()
    _run_scenario(libpaged.BlockManager(g["num_blocks"], g["block_size"]), g, False)


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
