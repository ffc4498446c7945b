"""The seeded input generator: structure of the synthetic state, and the
algorithmic byte counts against the pages' own size arithmetic."""
import json
import os

import numpy as np
import pytest

from oracle import paged_attention as opa
from paged_kv_cache_368_b200 import inputs


def _golden(name):
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        return json.load(f)


@pytest.mark.parametrize("index", range(5))
def test_config_structure(index):
    wl = inputs.config(index, data=False)
    S, bs = wl.num_seqs, wl.block_size
    nblk = -(-wl.context_lens.astype(np.int64) // bs)
    assert wl.block_tables.shape == (S, int(nblk.max()))
    seen = {}
    for s in range(S):
        ids = wl.block_tables[s, : nblk[s]]
        assert np.all((ids >= 0) & (ids < wl.num_blocks))
        for i, p in enumerate(ids.tolist()):
            seen.setdefault(p, []).append((s, i))
        # the new token's slot is the slot of position ctx-1 through the table
        assert wl.slot_mapping[s] == opa.slot_of_position(wl.block_tables[s], int(wl.context_lens[s]) - 1, bs)
    shared = {p: v for p, v in seen.items() if len(v) > 1}
    if wl.shared_prefix_blocks:
        assert len(shared) == (S // wl.group_size) * wl.shared_prefix_blocks
        for p, owners in shared.items():
            seqs = sorted({s for s, _ in owners})
            assert len(seqs) == wl.group_size and seqs[0] % wl.group_size == 0
            assert len({i for _, i in owners}) == 1 and owners[0][1] < wl.shared_prefix_blocks
        # appends never land in a shared block
        assert np.all(wl.context_lens - 1 >= wl.shared_prefix_blocks * bs)
    else:
        assert not shared
    assert len(wl.used) == len(seen)


def test_config_shapes_match_the_workloads():
    c = [inputs.config(i, data=False) for i in range(5)]
    assert (c[0].num_seqs, c[0].num_heads, c[0].head_dim, c[0].block_size) == (4, 4, 64, 16)
    assert c[0].context_lens.tolist() == [1, 17, 50, 128] and c[0].num_blocks == 64
    assert (c[1].num_seqs, c[1].num_heads, c[1].num_kv_heads, c[1].head_dim) == (32, 32, 32, 128)
    assert c[1].num_blocks == 8400 and c[1].context_lens.min() >= 128 and c[1].context_lens.max() <= 2048
    assert (c[2].num_seqs, c[2].num_heads, c[2].num_kv_heads, c[2].dtype) == (64, 32, 8, "bf16")
    assert c[2].context_lens.min() >= 512 and c[2].context_lens.max() <= 8192
    assert (c[3].num_seqs, c[3].num_heads) == (8, 40) and np.all(c[3].context_lens == 4096)
    assert (c[4].num_seqs, c[4].num_heads, c[4].num_kv_heads) == (16, 64, 8)
    assert c[4].context_lens.min() >= 1025 and c[4].context_lens.max() <= 65536
    for bs in (8, 16, 32, 64):
        wl = inputs.config(3, block_size=bs, data=False)
        assert wl.block_size == bs and wl.num_blocks == 2 * 8 * 4096 // bs


def test_kv_bytes_match_the_pages():
    g = _golden("kv_sizes.json")
    a = g["llama13b_layer"]
    wl = inputs.build("p1", seed=0, num_seqs=1, num_heads=40, num_kv_heads=40, head_dim=128, block_size=16,
                      dtype="f16", context_lens=[a["context_len"]], data=False)
    assert wl.kv_bytes() == a["kv_bytes_per_layer"] == 2 * a["k_bytes_per_layer"]
    # LLaMA-13B-shaped config: 8 sequences of 4096 = 8 x 80 MiB
    assert inputs.config(3, data=False).kv_bytes() == a["batch"] * a["kv_bytes_per_layer"]
    b = g["llama7b_token"]
    one = inputs.build("p2", seed=0, num_seqs=1, num_heads=32, num_kv_heads=b["num_kv_heads"], head_dim=128,
                       block_size=16, dtype="f16", context_lens=[1], data=False)
    assert one.kv_bytes() == b["kv_bytes_per_token_layer"]
    seq = inputs.build("p3", seed=0, num_seqs=1, num_heads=32, num_kv_heads=b["num_kv_heads"], head_dim=128,
                       block_size=16, dtype="f16", context_lens=[2048], data=False)
    assert seq.kv_bytes() * b["layers"] == b["kv_bytes_seq2048_model"]
    gqa = inputs.build("p4", seed=0, num_seqs=1, num_heads=32, num_kv_heads=b["gqa_kv_heads"], head_dim=128,
                       block_size=16, dtype="f16", context_lens=[2048], data=False)
    assert gqa.kv_bytes() * b["layers"] == b["kv_bytes_seq2048_model_gqa"]
    c = g["block_bytes"]
    blk = inputs.build("p5", seed=0, num_seqs=1, num_heads=32, num_kv_heads=c["num_kv_heads"], head_dim=128,
                       block_size=16, dtype="f16", context_lens=[c["block_size"]], data=False)
    assert blk.kv_bytes() == c["kv_bytes_per_block_layer"]
    d = g["block_count"]
    for bs, entries in d["entries_by_block_size"].items():
        w = inputs.build("p6", seed=0, num_seqs=1, num_heads=1, num_kv_heads=1, head_dim=64, block_size=int(bs),
                         dtype="f16", context_lens=[d["max_length"]], data=False)
        assert w.max_blocks_per_seq == entries


def test_page_address_layout():
    """With one kv-head, block_size 64 and head_dim 128 a (block, head) slice
    is the 16 KB page of the ops-transformer page; block b starts at b x 16 KB
    in a [NB, KVH, BS, D] fp16 pool."""
    g = _golden("kv_sizes.json")["page_address"]
    pool = np.zeros((31, g["num_kv_heads"], g["block_size"], g["head_dim"]), dtype=np.uint16)
    base = pool.ctypes.data
    for b, off in g["byte_offset_of_block"].items():
        assert pool[int(b)].ctypes.data - base == off
    assert pool[0].nbytes == g["page_bytes"]


def test_poison_and_data():
    wl = inputs.random_case(3, num_seqs=5, num_heads=4, num_kv_heads=2, head_dim=16, block_size=8,
                            dtype="bf16", ctx_lo=1, ctx_hi=40)
    k, v = wl.full_pool()
    nanv = inputs.nan_bits("bf16")
    for s in range(wl.num_seqs):
        L = int(wl.context_lens[s])
        for pos in range(-(-L // 8) * 8):
            blk, off = int(wl.block_tables[s, pos // 8]), pos % 8
            poisoned = np.all(k[blk, :, off] == nanv)
            assert poisoned == (pos >= L - 1), (s, pos)
    # determinism
    wl2 = inputs.random_case(3, num_seqs=5, num_heads=4, num_kv_heads=2, head_dim=16, block_size=8,
                             dtype="bf16", ctx_lo=1, ctx_hi=40)
    assert np.array_equal(wl.k_blocks, wl2.k_blocks) and np.array_equal(wl.q, wl2.q)


def test_compact_pool_is_equivalent():
    wl = inputs.random_case(4, num_seqs=4, num_heads=4, num_kv_heads=4, head_dim=16, block_size=4,
                            dtype="f16", ctx_lo=2, ctx_hi=25, poison=False)
    k, v = wl.full_pool()
    full = opa.decode(wl.q, k, v, wl.block_tables, wl.context_lens, wl.scale, "f16")
    kc, vc, tc = wl.compact([1, 3])
    part = opa.decode(wl.q[[1, 3]], kc, vc, tc, wl.context_lens[[1, 3]], wl.scale, "f16")
    assert np.array_equal(full[[1, 3]], part)
