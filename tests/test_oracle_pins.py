"""Pins for the float64 oracle: checks against things other than itself.

Each ``check_*`` takes the oracle module, so that ``test_planted_mistakes``
can run every check against copies of the oracle with one plausible mistake
planted (on the CPU) and show that some check fails for each.

Sources of truth used here:
* worked examples printed on the pages (``tests/golden/*.json``);
* a library routine: ``torch.nn.functional.scaled_dot_product_attention`` in
  float64 on contiguous (identity-table) K/V, GQA grouping included;
* closed forms: context length 1 returns V, constant V returns V, q = 0
  returns the mean of V, a dominant key returns its value;
* brute force with scalar Python loops on tiny inputs;
* invariants: permuting physical blocks changes nothing.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import paged_attention as opa
from paged_kv_cache_368_b200 import inputs

pytestmark = []


def _f16(x):
    return np.asarray(x, dtype=np.float16).view(np.uint16)


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _raw(x, dtype):
    return _f16(x) if dtype == "f16" else _bf16(x)


def _golden(name):
    here = os.path.dirname(os.path.abspath(__file__))
    with open(os.path.join(here, "golden", name)) as f:
        return json.load(f)


def _contiguous_case(rng, S, H, KVH, d, bs, ctx, dtype="f16"):
    """Pool laid out so that sequence s owns blocks s*MB .. s*MB+MB-1 in order
    (an identity block table): the logical sequence is a plain reshape."""
    MB = max(-(-c // bs) for c in ctx)
    NB = S * MB
    k = _raw(rng.standard_normal((NB, KVH, bs, d)), dtype)
    v = _raw(rng.standard_normal((NB, KVH, bs, d)), dtype)
    q = _raw(rng.standard_normal((S, H, d)), dtype)
    tables = np.arange(NB, dtype=np.int32).reshape(S, MB)
    return q, k, v, tables, np.asarray(ctx, dtype=np.int32), MB


# ---------------------------------------------------------------- checks


def check_worked_example_slots(orc):
    g = _golden("block_table_example.json")
    bs = g["block_size"]
    for pos, slot in g["expected_slots"].items():
        assert orc.slot_of_position(g["table"], int(pos), bs) == slot, pos
    for pos, slot in g["expected_slots_after_extension"].items():
        assert orc.slot_of_position(g["table_after_extension"], int(pos), bs) == slot, pos


def check_append_worked_example(orc):
    """Token at position 49 of the worked example goes to slot 193, which the
    page's table places in physical block 12 at offset 1; position 64 goes to
    slot 80 = physical block 5, offset 0.  Nothing else may change."""
    g = _golden("block_table_example.json")
    NB, KVH, bs, d = 16, 2, 16, 8
    base = (np.arange(NB * KVH * bs * d) % 1000).astype(np.float16).reshape(NB, KVH, bs, d).view(np.uint16)
    key = _f16(np.full((3, KVH, d), 1500.0) + np.arange(3)[:, None, None])
    val = _f16(np.full((3, KVH, d), -1500.0) - np.arange(3)[:, None, None])
    slots = np.array([g["expected_slots"]["49"], -1, g["expected_slots_after_extension"]["64"]], dtype=np.int64)
    k2, v2 = orc.reshape_and_cache(key, val, base, base, slots)
    expect_k = base.copy()
    expect_v = base.copy()
    b, o = g["expected_block_offset"]["49"]
    expect_k[b, :, o, :] = key[0]
    expect_v[b, :, o, :] = val[0]
    b, o = g["expected_block_offset"]["64"]
    expect_k[b, :, o, :] = key[2]
    expect_v[b, :, o, :] = val[2]
    assert np.array_equal(k2, expect_k)
    assert np.array_equal(v2, expect_v)


def check_identity_table_matches_sdpa(orc):
    """Identity block tables make paged attention ordinary attention: compare
    with torch's SDPA (float64, CPU), whose GQA grouping is the library's."""
    rng = np.random.default_rng(11)
    for (S, H, KVH, d, bs, ctx, dtype) in [
        (3, 4, 2, 16, 4, [5, 9, 16], "f16"),
        (2, 8, 1, 8, 8, [1, 23], "bf16"),
        (2, 3, 3, 32, 16, [40, 17], "f16"),
    ]:
        q, k, v, tables, cl, MB = _contiguous_case(rng, S, H, KVH, d, bs, ctx, dtype)
        scale = np.float32(1.0) / np.sqrt(np.float32(d))
        out = orc.decode(q, k, v, tables, cl, scale, dtype)
        for s in range(S):
            L = int(cl[s])
            kk = orc_free_widen(k[s * MB:(s + 1) * MB], dtype).transpose(1, 0, 2, 3).reshape(KVH, MB * bs, d)[:, :L]
            vv = orc_free_widen(v[s * MB:(s + 1) * MB], dtype).transpose(1, 0, 2, 3).reshape(KVH, MB * bs, d)[:, :L]
            qq = orc_free_widen(q[s], dtype)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(qq)[None, :, None, :],
                torch.from_numpy(kk)[None],
                torch.from_numpy(vv)[None],
                scale=float(scale),
                enable_gqa=True,
            )[0, :, 0, :].numpy()
            np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-13)


def orc_free_widen(raw, dtype):
    """Widen 16-bit patterns without the oracle (pins must not lean on it)."""
    bits = np.ascontiguousarray(raw).view(np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()


def _appended_pool(orc, wl):
    """Full pool after this step's append (the slot at ctx-1 is NaN before)."""
    k, v = wl.full_pool()
    return orc.reshape_and_cache(wl.k_new, wl.v_new, k, v, wl.slot_mapping)


def check_permutation_invariance(orc):
    wl = inputs.random_case(5, num_seqs=3, num_heads=4, num_kv_heads=2, head_dim=16, block_size=4,
                            dtype="f16", ctx_lo=1, ctx_hi=30)
    k, v = _appended_pool(orc, wl)
    assert np.isfinite(orc.decode(wl.q, k, v, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)).all()
    out = orc.decode(wl.q, k, v, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)
    perm = np.random.default_rng(3).permutation(wl.num_blocks)
    k2 = np.empty_like(k)
    v2 = np.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    t2 = np.where(wl.block_tables >= 0, perm[np.clip(wl.block_tables, 0, None)], -1).astype(np.int32)
    out2 = orc.decode(wl.q, k2, v2, t2, wl.context_lens, wl.scale, wl.dtype)
    assert np.array_equal(out, out2)
    # and a different permutation must actually move bytes
    assert not np.array_equal(k2, k)


def check_context_one_returns_v(orc):
    rng = np.random.default_rng(2)
    NB, KVH, bs, d, H = 6, 2, 8, 16, 4
    k = _f16(rng.standard_normal((NB, KVH, bs, d)))
    v = _f16(rng.standard_normal((NB, KVH, bs, d)))
    q = _f16(rng.standard_normal((1, H, d)))
    tables = np.array([[4, 0]], dtype=np.int32)
    out = orc.decode(q, k, v, tables, np.array([1], dtype=np.int32), np.float32(0.25), "f16")
    for h in range(H):
        assert np.array_equal(out[0, h], v[4, h // 2, 0].view(np.float16).astype(np.float64))


def check_brute_force_tiny(orc):
    """Scalar Python loops, reading blocks through the table by hand."""
    rng = np.random.default_rng(9)
    NB, KVH, bs, d, H, S = 7, 1, 2, 3, 2, 2
    kf = rng.standard_normal((NB, KVH, bs, d)).astype(np.float16)
    vf = rng.standard_normal((NB, KVH, bs, d)).astype(np.float16)
    qf = rng.standard_normal((S, H, d)).astype(np.float16)
    tables = np.array([[6, 2], [1, 4]], dtype=np.int32)
    ctx = np.array([3, 4], dtype=np.int32)
    scale = np.float32(0.7)
    out = orc.decode(qf.view(np.uint16), kf.view(np.uint16), vf.view(np.uint16), tables, ctx, scale, "f16")
    for s in range(S):
        for h in range(H):
            keys, vals = [], []
            for blk in range(2):
                for off in range(bs):
                    if blk * bs + off < ctx[s]:
                        keys.append([float(x) for x in kf[tables[s][blk], 0, off]])
                        vals.append([float(x) for x in vf[tables[s][blk], 0, off]])
            qs = [float(x) for x in qf[s, h]]
            sc = [float(scale) * sum(a * b for a, b in zip(qs, kk)) for kk in keys]
            mx = max(sc)
            e = [math.exp(x - mx) for x in sc]
            z = sum(e)
            ref = [sum(e[i] / z * vals[i][j] for i in range(len(vals))) for j in range(d)]
            np.testing.assert_allclose(out[s, h], ref, rtol=1e-12, atol=1e-14)


def check_constant_v(orc):
    wl = inputs.random_case(21, num_seqs=3, num_heads=2, num_kv_heads=2, head_dim=8, block_size=4,
                            dtype="f16", ctx_lo=2, ctx_hi=20)
    k, v = _appended_pool(orc, wl)
    c = _f16(np.linspace(-2, 2, 8))
    v[...] = c
    out = orc.decode(wl.q, k, v, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)
    np.testing.assert_allclose(out, np.broadcast_to(c.view(np.float16).astype(np.float64), out.shape), rtol=1e-13, atol=1e-13)


def check_zero_q_gives_mean(orc):
    """q = 0 makes every weight 1/L: the output is the mean of the gathered V,
    which here is computed from the pool through the worked-example table."""
    g = _golden("block_table_example.json")
    rng = np.random.default_rng(4)
    NB, KVH, bs, d = 16, 1, 16, 4
    k = _f16(rng.standard_normal((NB, KVH, bs, d)))
    v = _f16(rng.standard_normal((NB, KVH, bs, d)))
    q = _f16(np.zeros((1, 1, d)))
    L = 51  # positions 0..50: blocks 3, 7, 1 in full, block 12 offsets 0..2
    out = orc.decode(q, k, v, np.array([g["table"]], dtype=np.int32), np.array([L], dtype=np.int32), np.float32(1.0), "f16")
    vf = v.view(np.float16).astype(np.float64)
    rows = [vf[3, 0], vf[7, 0], vf[1, 0], vf[12, 0, :3]]
    mean = np.concatenate(rows, axis=0).mean(axis=0)
    np.testing.assert_allclose(out[0, 0], mean, rtol=1e-12, atol=1e-14)


def check_gqa_equals_repeated_kv(orc):
    wl = inputs.random_case(8, num_seqs=2, num_heads=8, num_kv_heads=2, head_dim=8, block_size=4,
                            dtype="bf16", ctx_lo=3, ctx_hi=17)
    k, v = _appended_pool(orc, wl)
    out = orc.decode(wl.q, k, v, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)
    G = wl.num_heads // wl.num_kv_heads
    k_rep = np.repeat(k, G, axis=1)  # kv-head j -> q-heads jG .. jG+G-1
    v_rep = np.repeat(v, G, axis=1)
    out2 = orc.decode(wl.q, k_rep, v_rep, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)
    assert np.array_equal(out, out2)


def check_dominant_key(orc):
    """Make the key at one target position c*q: its weight is ~1, the output
    is that position's value, wherever the table put it."""
    wl = inputs.random_case(13, num_seqs=2, num_heads=2, num_kv_heads=2, head_dim=16, block_size=4,
                            dtype="f16", ctx_lo=9, ctx_hi=14)
    k, v = _appended_pool(orc, wl)
    for s in range(wl.num_seqs):
        t = int(wl.context_lens[s]) - 3
        blk, off = int(wl.block_tables[s, t // 4]), t % 4
        for h in range(2):
            qv = wl.q[s, h].view(np.float16).astype(np.float32)
            k[blk, h, off] = (qv * 8.0).astype(np.float16).view(np.uint16)
    out = orc.decode(wl.q, k, v, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)
    for s in range(wl.num_seqs):
        t = int(wl.context_lens[s]) - 3
        blk, off = int(wl.block_tables[s, t // 4]), t % 4
        for h in range(2):
            np.testing.assert_allclose(out[s, h], v[blk, h, off].view(np.float16).astype(np.float64), atol=1e-6)


def check_append_then_attend(orc):
    """After the append of section 1.2, context length 1 reads back the new V
    exactly, and a step is append followed by attention."""
    wl = inputs.build("one", seed=1, num_seqs=2, num_heads=2, num_kv_heads=1, head_dim=8, block_size=4,
                      dtype="f16", context_lens=[1, 6], pool_blocks=5)
    k, v = wl.full_pool()
    out, k2, v2 = orc.decode_step(wl.q, wl.k_new, wl.v_new, k, v, wl.slot_mapping, wl.block_tables,
                                  wl.context_lens, wl.scale, wl.dtype)
    assert np.isfinite(out).all()
    for h in range(2):
        assert np.array_equal(out[0, h], wl.v_new[0, 0].view(np.float16).astype(np.float64))


CHECKS = [
    check_worked_example_slots,
    check_append_worked_example,
    check_identity_table_matches_sdpa,
    check_permutation_invariance,
    check_context_one_returns_v,
    check_brute_force_tiny,
    check_constant_v,
    check_zero_q_gives_mean,
    check_gqa_equals_repeated_kv,
    check_dominant_key,
    check_append_then_attend,
]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(opa)


# ------------------------------------------------- planted mistakes


def _mut_attend_no_scale(q64, k64, v64, scale):
    return _ATTEND(q64, k64, v64, 1.0)


def _mut_attend_head_modulo(q64, k64, v64, scale):
    H, d = q64.shape
    kvh = k64.shape[0]
    out = np.zeros((H, d))
    for h in range(H):
        s = scale * (k64[h % kvh] @ q64[h])
        w = np.exp(s - s.max())
        out[h] = (w / w.sum()) @ v64[h % kvh]
    return out


def _mut_attend_unnormalised(q64, k64, v64, scale):
    H, d = q64.shape
    kvh = k64.shape[0]
    G = H // kvh
    out = np.zeros((H, d))
    for h in range(H):
        s = scale * (k64[h // G] @ q64[h])
        out[h] = np.exp(s - s.max()) @ v64[h // G]
    return out


def _mut_attend_k_for_v(q64, k64, v64, scale):
    return _ATTEND(q64, k64, k64, scale)


def _mut_attend_sign(q64, k64, v64, scale):
    return _ATTEND(q64, k64, v64, -scale)


def _mut_gather_swapped(cache, table_row, ctx, dtype):
    bs = cache.shape[2]
    pos = np.arange(ctx)
    idx = np.clip(pos % bs, 0, len(table_row) - 1)
    phys = np.asarray(table_row)[idx].astype(np.int64)
    return opa.widen(cache[phys, :, (pos // bs) % bs, :], dtype).transpose(1, 0, 2)


def _mut_gather_drop_last(cache, table_row, ctx, dtype):
    return _GATHER(cache, table_row, max(ctx - 1, 1), dtype)


def _mut_gather_whole_blocks(cache, table_row, ctx, dtype):
    bs = cache.shape[2]
    return _GATHER(cache, table_row, -(-ctx // bs) * bs, dtype)


def _mut_slot_off_by_one(table_row, position, block_size):
    return _SLOT(table_row, position + 1, block_size)


def _mut_append_transposed(key, value, k_cache, v_cache, slot_mapping):
    k_out, v_out = np.array(k_cache), np.array(v_cache)
    bs = k_cache.shape[2]
    for n, s in enumerate(np.asarray(slot_mapping).tolist()):
        if s < 0:
            continue
        k_out[(s % bs) % k_cache.shape[0], :, (s // bs) % bs, :] = key[n]
        v_out[(s % bs) % k_cache.shape[0], :, (s // bs) % bs, :] = value[n]
    return k_out, v_out


_ATTEND, _GATHER, _SLOT = opa.attend, opa.gather, opa.slot_of_position

MUTANTS = {
    "attend_no_scale": ("attend", _mut_attend_no_scale),
    "attend_head_modulo": ("attend", _mut_attend_head_modulo),
    "attend_unnormalised": ("attend", _mut_attend_unnormalised),
    "attend_k_for_v": ("attend", _mut_attend_k_for_v),
    "attend_sign": ("attend", _mut_attend_sign),
    "gather_swapped_index": ("gather", _mut_gather_swapped),
    "gather_drop_last": ("gather", _mut_gather_drop_last),
    "gather_whole_blocks": ("gather", _mut_gather_whole_blocks),
    "slot_off_by_one": ("slot_of_position", _mut_slot_off_by_one),
    "append_transposed": ("reshape_and_cache", _mut_append_transposed),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(opa, attr, fn)
    failed = []
    for check in CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(opa)
        except (AssertionError, IndexError, ValueError, FloatingPointError):
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
