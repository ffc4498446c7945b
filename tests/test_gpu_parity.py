"""GPU parity: libpaged (through its C ABI) against the float64 oracle.

* append: bit-exact over the whole pool (or, for pools too big to copy
  back, the touched rows bit-exact and every other byte unchanged);
* decode: every output element within |gpu - ref| <= atol + rtol |ref|
  (fp16: 2e-3 + 1e-2, bf16: 1.6e-2 + 2e-2), at small sizes and at the full
  sizes of every workload (all sequences, all q-heads);
* invariants that must hold bit-for-bit on the GPU: permuting physical
  blocks, sharing prefix blocks, context length 1 returning V.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import DeviceState, TOL, assert_close, reference_full, reference_sampled, to_dev, to_raw
from paged_kv_cache_368_b200 import inputs, libpaged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    libpaged.load()
    yield


# ------------------------------------------------------------------ config 0 (tiny MHA), whole thing


def test_tiny_mha_step_matches_oracle():
    wl = inputs.config(0)
    ds = DeviceState(wl, full_pool=True)
    out = ds.step()
    ref, k_ref, v_ref = reference_full(wl)
    assert np.array_equal(to_raw(ds.k_cache), k_ref)
    assert np.array_equal(to_raw(ds.v_cache), v_ref)
    assert_close(out, ref, wl.dtype, "tiny-mha")
    assert int(ds.err.item()) == 0
    # context length 1 (sequence 0) returns its new V exactly
    for h in range(wl.num_heads):
        assert np.array_equal(out[0, h], wl.v_new[0, h])


# ------------------------------------------------------------------ sweep of small random cases

SWEEP = [(dt, d, bs, g) for dt in ("f16", "bf16") for d in (64, 128) for bs in (8, 16, 32, 64) for g in (1, 2, 4, 8)]


@pytest.mark.parametrize("dtype,head_dim,block_size,group", SWEEP,
                         ids=[f"{a}-d{b}-bs{c}-g{d}" for a, b, c, d in SWEEP])
def test_small_random_cases(dtype, head_dim, block_size, group):
    kvh = 2
    seed = 1000 + head_dim + block_size * 3 + group * 7 + (0 if dtype == "f16" else 500)
    wl = inputs.random_case(seed, num_seqs=5, num_heads=kvh * group, num_kv_heads=kvh, head_dim=head_dim,
                            block_size=block_size, dtype=dtype, ctx_lo=1, ctx_hi=300, table_filler=-2)
    ds = DeviceState(wl, full_pool=True)
    out = ds.step()
    ref, k_ref, v_ref = reference_full(wl)
    assert np.array_equal(to_raw(ds.k_cache), k_ref)
    assert np.array_equal(to_raw(ds.v_cache), v_ref)
    assert_close(out, ref, dtype, f"{dtype}-d{head_dim}-bs{block_size}-g{group}")
    assert int(ds.err.item()) == 0


@pytest.mark.parametrize("max_ctas", [1, 2, 3, 7, 0])
def test_split_choice_does_not_change_the_result(max_ctas):
    """Capping the grid changes where units are split (and how many partials
    the merge combines); every choice must stay within tolerance."""
    wl = inputs.random_case(77, num_seqs=6, num_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                            dtype="bf16", ctx_lo=1, ctx_hi=3000)
    ds = DeviceState(wl, full_pool=True)
    out = ds.step(max_ctas=max_ctas)
    ref, _, _ = reference_full(wl)
    assert_close(out, ref, wl.dtype, f"max_ctas={max_ctas}")


@pytest.mark.parametrize("num_seqs,kvh,head_dim",
                         [(2048, 4, 64), (16384, 8, 64), (16384, 8, 128), (16385, 8, 64), (33000, 2, 64)])
def test_many_short_sequences_and_empty_contexts(num_seqs, kvh, head_dim):
    """Many sequences with contexts 0..40; empty ones give zeros.  One
    launch takes at most 16384 sequences: 16385 and 33000 run as two and
    three launches in one call (the last one of 1 and 232 sequences)."""
    wl = inputs.random_case(5, num_seqs=num_seqs, num_heads=kvh, num_kv_heads=kvh, head_dim=head_dim,
                            block_size=16, dtype="f16", ctx_lo=1, ctx_hi=40)
    ctx = wl.context_lens.copy()
    ctx[::7] = 0
    wl.context_lens = ctx
    wl.slot_mapping = np.where(ctx > 0, wl.slot_mapping, -1)
    ds = DeviceState(wl, full_pool=True)
    out = ds.step()
    ref, k_ref, v_ref = reference_full(wl)
    assert np.array_equal(to_raw(ds.k_cache), k_ref)
    assert_close(out, ref, wl.dtype, f"{num_seqs} seqs")
    assert np.all(out[::7] == 0)
    assert int(ds.err.item()) == 0


# ------------------------------------------------------------------ full-size configs

FULL = [1, 2, 4] + [("bs", b) for b in (8, 16, 32, 64)]


def _full_workload(spec):
    if isinstance(spec, tuple):
        return inputs.config(3, block_size=spec[1])
    return inputs.config(spec)


@pytest.mark.parametrize("spec", FULL, ids=lambda s: f"llama13b-bs{s[1]}" if isinstance(s, tuple) else inputs.CONFIG_NAMES[s])
def test_full_size_config(spec):
    wl = _full_workload(spec)
    ds = DeviceState(wl, full_pool=False)
    k_before = ds.k_cache.clone()
    v_before = ds.v_cache.clone()
    out = ds.step()
    assert int(ds.err.item()) == 0
    # append: the new rows bit-exact, nothing else touched
    slots = wl.slot_mapping
    blk = torch.from_numpy(slots // wl.block_size).cuda()
    off = torch.from_numpy(slots % wl.block_size).cuda()
    assert torch.equal(ds.k_cache[blk, :, off, :].view(torch.int16), ds.k_new.view(torch.int16))
    assert torch.equal(ds.v_cache[blk, :, off, :].view(torch.int16), ds.v_new.view(torch.int16))
    k_after = ds.k_cache.clone()
    v_after = ds.v_cache.clone()
    k_after[blk, :, off, :] = 0
    v_after[blk, :, off, :] = 0
    k_before[blk, :, off, :] = 0
    v_before[blk, :, off, :] = 0
    assert torch.equal(k_after.view(torch.int16), k_before.view(torch.int16))
    assert torch.equal(v_after.view(torch.int16), v_before.view(torch.int16))
    del k_before, v_before, k_after, v_after
    # decode: every (sequence, q-head) row against the oracle, one sequence
    # at a time on a pool of only its blocks (bounded host memory)
    assert np.isfinite(oracle.widen(out, wl.dtype)).all()
    worst = 0.0
    for s in range(wl.num_seqs):
        ref = np.stack([r for _, r in sorted(reference_sampled(wl, [s]).items())])
        worst = max(worst, assert_close(out[s], ref, wl.dtype, f"{wl.name} seq {s}"))
    print(f"{wl.name}: {wl.num_seqs * wl.num_heads} rows, max |err| {worst:.3e}")


# ------------------------------------------------------------------ invariants, bit for bit


def test_permuting_physical_blocks_is_bit_identical():
    wl = inputs.random_case(31, num_seqs=7, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                            dtype="f16", ctx_lo=1, ctx_hi=900)
    out1 = DeviceState(wl, full_pool=True).step()
    perm = np.random.default_rng(9).permutation(wl.num_blocks)
    wl2 = inputs.random_case(31, num_seqs=7, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                             dtype="f16", ctx_lo=1, ctx_hi=900)
    wl2.used = perm[wl.used]
    nb = -(-wl.context_lens // 16)
    t2 = wl.block_tables.copy()
    for s in range(wl.num_seqs):
        t2[s, : nb[s]] = perm[wl.block_tables[s, : nb[s]]]
    wl2.block_tables = t2
    wl2.slot_mapping = perm[wl.slot_mapping // 16] * 16 + wl.slot_mapping % 16
    out2 = DeviceState(wl2, full_pool=True).step()
    assert np.array_equal(out1, out2)


def test_shared_prefix_equals_private_copies():
    """Sequences whose tables point at the same prefix blocks give the same
    bits as when each holds its own copy of those blocks."""
    wl = inputs.build("prefix", seed=55, num_seqs=8, num_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
                      dtype="bf16", ctx_kind="uniform", ctx_lo=1100, ctx_hi=3000, shared_prefix_blocks=64,
                      group_size=4, pool_factor=2.0)
    out_shared = DeviceState(wl, full_pool=False).step()
    # private copies: every sequence gets fresh blocks holding the prefix data
    import copy

    wl2 = copy.deepcopy(wl)
    row_of = {int(p): i for i, p in enumerate(wl.used)}
    free = [b for b in range(wl.num_blocks) if b not in row_of]
    extra_k, extra_v, extra_ids = [], [], []
    t2 = wl.block_tables.copy()
    for s in range(wl.num_seqs):
        if s % wl.group_size == 0:
            continue
        for i in range(wl.shared_prefix_blocks):
            b = free.pop()
            src = row_of[int(wl.block_tables[s, i])]
            extra_ids.append(b)
            extra_k.append(wl.k_blocks[src])
            extra_v.append(wl.v_blocks[src])
            t2[s, i] = b
    wl2.block_tables = t2
    wl2.used = np.concatenate([wl.used, np.array(extra_ids, dtype=np.int64)])
    wl2.k_blocks = np.concatenate([wl.k_blocks, np.stack(extra_k)])
    wl2.v_blocks = np.concatenate([wl.v_blocks, np.stack(extra_v)])
    out_private = DeviceState(wl2, full_pool=False).step()
    assert np.array_equal(out_shared, out_private)
    ref = reference_sampled(wl, [0, 1, 5], [0, 7])
    for (s, h), r in ref.items():
        assert_close(out_shared[s, h], r, wl.dtype, f"prefix seq {s} head {h}")


@pytest.mark.parametrize("dtype,group", [("f16", 1), ("bf16", 1), ("f16", 4), ("bf16", 8), ("f16", 2)])
def test_context_one_returns_v_exactly(dtype, group):
    wl = inputs.build("ctx1", seed=3, num_seqs=3, num_heads=2 * group, num_kv_heads=2, head_dim=128,
                      block_size=16, dtype=dtype, context_lens=[1, 1, 1], pool_blocks=9)
    out = DeviceState(wl, full_pool=True).step()
    for s in range(3):
        for h in range(2 * group):
            assert np.array_equal(out[s, h], wl.v_new[s, h // group])


@pytest.mark.parametrize("group", [1, 8])
def test_dominant_key_selects_its_value(group):
    """Key at one target position = 8 * q: its weight is ~1, so the output is
    that position's V -- checks the table indexing of every target."""
    wl = inputs.random_case(41, num_seqs=4, num_heads=2 * group, num_kv_heads=2, head_dim=64, block_size=8,
                            dtype="f16", ctx_lo=40, ctx_hi=200)
    k, v = wl.full_pool()
    targets = []
    for s in range(wl.num_seqs):
        t = (s * 37) % (int(wl.context_lens[s]) - 1)
        blk, off = int(wl.block_tables[s, t // 8]), t % 8
        for h in range(2):
            qv = wl.q[s, h * group].view(np.float16).astype(np.float32)
            k[blk, h, off] = (qv * 8.0).astype(np.float16).view(np.uint16)
        targets.append((s, blk, off))
    ds = DeviceState(wl, full_pool=True)
    ds.k_cache.copy_(to_dev(k, "f16"))
    ds.v_cache.copy_(to_dev(v, "f16"))
    out = ds.step()
    for s, blk, off in targets:
        for h in range(2):
            got = oracle.widen(out[s, h * group], "f16")
            want = v[blk, h, off].view(np.float16).astype(np.float64)
            np.testing.assert_allclose(got, want, atol=2e-3, rtol=1e-2)


# ------------------------------------------------------------------ error reporting without faults


def test_out_of_range_ids_set_flags_and_stay_finite():
    wl = inputs.random_case(8, num_seqs=4, num_heads=4, num_kv_heads=4, head_dim=128, block_size=16,
                            dtype="f16", ctx_lo=20, ctx_hi=100)
    ds = DeviceState(wl, full_pool=True)
    bad_tables = ds.tables.clone()
    bad_tables[2, 0] = wl.num_blocks + 5  # decode: skip that chunk, flag it
    ds.tables = bad_tables
    slots = ds.slots.clone()
    slots[1] = wl.num_blocks * wl.block_size + 3  # append: skip that token, flag it
    ds.slots = slots
    out = ds.step()
    flags = int(ds.err.item())
    assert flags & libpaged.ERRF_BLOCK_RANGE
    assert flags & libpaged.ERRF_SLOT_RANGE
    # sequences 0 and 3 are untouched by the bad entries
    ref, _, _ = reference_full(wl)
    assert_close(out[[0, 3]], ref[[0, 3]], "f16", "good sequences")


def test_context_above_bound_is_clamped_and_flagged():
    wl = inputs.random_case(9, num_seqs=3, num_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                            dtype="f16", ctx_lo=30, ctx_hi=60)
    ds = DeviceState(wl, full_pool=True)
    ds.append()
    ds.err.zero_()
    libpaged.decode(ds.out, ds.q, ds.k_cache, ds.v_cache, ds.tables, ds.ctx, float(wl.scale),
                    max_context_len=int(wl.context_lens.min()) - 1, workspace=ds.ws, err_flags=ds.err)
    torch.cuda.synchronize()
    assert int(ds.err.item()) & libpaged.ERRF_CONTEXT
    assert torch.isfinite(ds.out.float()).all()


def test_status_codes_through_binding():
    wl = inputs.random_case(10, num_seqs=2, num_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
                            dtype="f16", ctx_lo=5, ctx_hi=9)
    ds = DeviceState(wl, full_pool=True)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(libpaged.LibpagedError) as e:
        libpaged.decode(ds.out, ds.q, ds.k_cache, ds.v_cache, ds.tables, ds.ctx, 0.1, workspace=small)
    assert e.value.status == libpaged.PA_ERR_WORKSPACE


def test_decode_step_from_host_buffers():
    """pa_decode_step_host (one packed copy in, append, decode, copy out)
    gives the same bits as the device-resident calls, and matches the oracle."""
    wl = inputs.random_case(71, num_seqs=6, num_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                            dtype="bf16", ctx_lo=1, ctx_hi=1500)
    ds = DeviceState(wl, full_pool=True)
    dev_out = ds.step()
    ds2 = DeviceState(wl, full_pool=True)
    offs, total = libpaged.step_inputs_layout(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                              wl.max_blocks_per_seq)
    assert all(o % 256 == 0 for o in offs.values())
    h_in = torch.zeros(total, dtype=torch.uint8).pin_memory()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    libpaged.pack_step_inputs(h_in, offs, q=t(wl.q), key=t(wl.k_new), value=t(wl.v_new),
                              slot_mapping=t(wl.slot_mapping.astype(np.int64)),
                              block_tables=t(wl.block_tables.astype(np.int32)),
                              context_lens=t(wl.context_lens.astype(np.int32)))
    d_in = torch.empty(total, dtype=torch.uint8, device="cuda")
    h_out = torch.empty(ds2.q.shape, dtype=torch.bfloat16).pin_memory()
    libpaged.decode_step_host(h_in, d_in, h_out, torch.empty_like(ds2.q), ds2.k_cache, ds2.v_cache,
                              wl.num_heads, wl.max_blocks_per_seq, float(wl.scale),
                              max_context_len=wl.max_context_len, workspace=ds2.ws, err_flags=ds2.err)
    torch.cuda.synchronize()
    host_out = h_out.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(host_out, dev_out)
    assert np.array_equal(to_raw(ds2.k_cache), to_raw(ds.k_cache))
    ref, _, _ = reference_full(wl)
    assert_close(host_out, ref, wl.dtype, "host step")
    assert int(ds2.err.item()) == 0


def test_merge_tickets_return_to_zero_and_workspace_reuse_is_exact():
    """The in-launch merge counts each split unit's chunks on ticket counters
    at the front of the workspace (one int32 per warp of the largest grid:
    SMs x 8, the same region for every call) and leaves every counter at
    zero: one zeroed workspace reused across shapes and grid caps (a capped
    grid's partials must not land on a larger grid's counters) gives the same
    bits as a fresh one, and every output row is written by every call."""
    shared = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")
    nbytes = 4 * 8 * torch.cuda.get_device_properties(0).multi_processor_count
    for seed, g, max_ctas in ((201, 4, 0), (202, 1, 3), (203, 8, 7), (204, 2, 0), (201, 4, 2)):
        wl = inputs.random_case(seed, num_seqs=7, num_heads=2 * g, num_kv_heads=2, head_dim=128, block_size=16,
                                dtype="bf16", ctx_lo=1, ctx_hi=5000)
        want = DeviceState(wl, full_pool=True).step(max_ctas=max_ctas)
        ds = DeviceState(wl, full_pool=True)
        ds.ws = shared
        for _ in range(2):
            ds.out.fill_(float("nan"))  # a row the call fails to write stays NaN
            got = ds.step(max_ctas=max_ctas)  # the repeated append rewrites the same rows
            assert np.array_equal(got, want), (seed, max_ctas)
            assert int(shared[:nbytes].count_nonzero().item()) == 0, (seed, max_ctas)
        assert int(ds.err.item()) == 0


def test_pipelined_host_steps_match_single_steps():
    """pa_decode_step_host_pipelined (input copy of step i+1 on a second
    stream, overlapping step i's kernels; output copy of step i on a third,
    overlapping step i+1's; two sets of staging and output buffers in turn,
    so steps 0, 2 and 4 reuse one device output buffer) gives, step after
    step, the same bits as pa_decode_step_host."""
    steps = []
    for seed in (301, 302, 303, 304, 305):
        steps.append(inputs.random_case(seed, num_seqs=6, num_heads=16, num_kv_heads=4, head_dim=128,
                                        block_size=16, dtype="bf16", ctx_lo=1, ctx_hi=1500))
    # one pool for all steps: each step's tables were drawn for its own pool,
    # so use one workload's pool and tables and vary q and the new tokens
    base = steps[0]
    mb = base.max_blocks_per_seq
    offs, total = libpaged.step_inputs_layout(base.num_seqs, base.num_heads, base.num_kv_heads, base.head_dim, mb)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    h_ins = []
    for wl in steps:
        h = torch.zeros(total, dtype=torch.uint8).pin_memory()
        libpaged.pack_step_inputs(h, offs, q=t(wl.q), key=t(wl.k_new), value=t(wl.v_new),
                                  slot_mapping=t(base.slot_mapping.astype(np.int64)),
                                  block_tables=t(base.block_tables.astype(np.int32)),
                                  context_lens=t(base.context_lens.astype(np.int32)))
        h_ins.append(h)
    want_state = DeviceState(base, full_pool=True)
    got_state = DeviceState(base, full_pool=True)
    d_in = torch.empty(total, dtype=torch.uint8, device="cuda")
    pipe = libpaged.StepPipeline(total, got_state.q.shape, torch.bfloat16)
    want, got = [], []
    for h in h_ins:
        ho = torch.empty(want_state.q.shape, dtype=torch.bfloat16).pin_memory()
        libpaged.decode_step_host(h, d_in, ho, torch.empty_like(want_state.q), want_state.k_cache,
                                  want_state.v_cache, base.num_heads, mb, float(base.scale),
                                  max_context_len=base.max_context_len, workspace=want_state.ws,
                                  err_flags=want_state.err)
        torch.cuda.synchronize()
        want.append(ho.clone())
    outs = []
    for h in h_ins:
        ho = torch.empty(got_state.q.shape, dtype=torch.bfloat16).pin_memory()
        pipe.step(h, ho, got_state.k_cache, got_state.v_cache, base.num_heads, mb, float(base.scale),
                  max_context_len=base.max_context_len, workspace=got_state.ws, err_flags=got_state.err)
        outs.append(ho)
    pipe.wait()  # the last output copy; the earlier ones ran before it on the same stream
    for a, b in zip(want, outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(want_state.k_cache.view(torch.int16), got_state.k_cache.view(torch.int16))
    assert int(got_state.err.item()) == 0
