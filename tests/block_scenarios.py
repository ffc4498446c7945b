"""Runs the hand-worked block-manager scenarios of ``tests/golden`` against a
block manager: the oracle's Python model or the library's C++ one (through
the C ABI; no GPU needed).  Each adapter maps one implementation onto the
same small interface, so that the same expected values judge both."""
from __future__ import annotations

import json
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


class OutOfBlocksSeen(Exception):
    pass


class ModelAdapter:
    """The oracle's ``BlockManagerModel`` (from the module passed in, so that
    planted mistakes in a patched module are what runs)."""

    def __init__(self, obm, num_blocks, block_size):
        self.obm = obm
        self.m = obm.BlockManagerModel(num_blocks, block_size)

    def add(self, seq, tokens):
        self.m.add(seq, tokens)

    def fork(self, parent, child):
        self.m.fork(parent, child)

    def append(self, seq):
        slot, cow = self.m.append_slot(seq)
        return slot, (list(cow) if cow else None)

    def free(self, seq):
        self.m.free(seq)

    def num_free(self):
        return len(self.m.free_blocks())

    def table(self, seq):
        return list(self.m.tables[seq])

    def length(self, seq):
        return self.m.lens[seq]

    def needed(self, seqs):
        return self.m.blocks_needed_to_append(seqs)

    def swap_to(self, other, seq):
        try:
            pairs = self.m.swap_to(other.m, seq)
        except self.obm.OutOfBlocks:
            raise OutOfBlocksSeen()
        return [list(p) for p in pairs]


class LibraryAdapter:
    """The C++ block manager of libpaged."""

    def __init__(self, num_blocks, block_size):
        from paged_kv_cache_368_b200 import libpaged

        self.lp = libpaged
        self.m = libpaged.BlockManager(num_blocks, block_size)

    def add(self, seq, tokens):
        self.m.add(seq, tokens)

    def fork(self, parent, child):
        self.m.fork(parent, child)

    def append(self, seq):
        slot, src, dst = self.m.append_slot(seq)
        return slot, ([src, dst] if src >= 0 else None)

    def free(self, seq):
        self.m.free(seq)

    def num_free(self):
        return self.m.num_free

    def table(self, seq):
        return self.m.block_table(seq)

    def length(self, seq):
        return self.m.context_len(seq)

    def needed(self, seqs):
        return self.m.blocks_needed_to_append(seqs)

    def swap_to(self, other, seq):
        try:
            pairs = self.m.swap_to(other.m, seq)
        except self.lp.LibpagedError as e:
            if e.status == self.lp.PA_ERR_OUT_OF_BLOCKS:
                raise OutOfBlocksSeen()
            raise
        return pairs.tolist()


def run_lifecycle_scenario(make, g):
    """``block_manager_scenario.json``: add / fork / append / free in one pool."""
    mgr = make(g["num_blocks"], g["block_size"])
    for st in g["steps"]:
        if st["op"] == "add":
            mgr.add(st["seq"], st["tokens"])
        elif st["op"] == "fork":
            mgr.fork(st["parent"], st["child"])
        elif st["op"] == "append":
            slot, cow = mgr.append(st["seq"])
            assert slot == st["slot"], st
            assert cow == st["cow"], st
        elif st["op"] == "free":
            mgr.free(st["seq"])
            assert mgr.num_free() == st["num_free"], st
        if "table" in st:
            assert mgr.table(st.get("seq", st.get("child"))) == st["table"], st
    assert mgr.num_free() == g["final_num_free"]


def run_swap_scenario(make, g):
    """``block_manager_swap_scenario.json``: two pools, admission counts,
    swapping out and back, copy on write afterwards."""
    pools = {name: make(n, g["block_size"]) for name, n in g["pools"].items()}

    def check_free(st):
        if "free" in st:
            got = {name: p.num_free() for name, p in pools.items()}
            assert got == st["free"], (st, got)

    for st in g["steps"]:
        op = st["op"]
        if op == "add":
            pools[st["pool"]].add(st["seq"], st["tokens"])
            assert pools[st["pool"]].table(st["seq"]) == st["table"], st
        elif op == "fork":
            pools[st["pool"]].fork(st["parent"], st["child"])
            assert pools[st["pool"]].table(st["child"]) == st["table"], st
        elif op == "needed":
            assert pools[st["pool"]].needed(st["seqs"]) == st["blocks"], st
        elif op == "swap":
            src, dst = pools[st["from"]], pools[st["to"]]
            if "error" in st:
                try:
                    src.swap_to(dst, st["seq"])
                except OutOfBlocksSeen:
                    pass
                else:
                    raise AssertionError(f"swap should have run out of blocks: {st}")
            else:
                assert src.swap_to(dst, st["seq"]) == st["pairs"], st
                assert dst.table(st["seq"]) == st["table"], st
                assert dst.length(st["seq"]) == st["len"], st
        elif op == "table":
            assert pools[st["pool"]].table(st["seq"]) == st["table"], st
        elif op == "free":
            pools[st["pool"]].free(st["seq"])
        elif op == "append":
            slot, cow = pools[st["pool"]].append(st["seq"])
            assert slot == st["slot"] and cow == st["cow"], st
            assert pools[st["pool"]].table(st["seq"]) == st["table"], st
        else:
            raise ValueError(op)
        check_free(st)
    assert {name: p.num_free() for name, p in pools.items()} == g["final_free"]
