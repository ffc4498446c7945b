"""GPU tests of the block operations: copy-on-write copies, swapping to
pinned host memory, and a multi-step decode loop driven by the block manager
(beams forked from one sequence, shared blocks copied on write, a sequence
swapped out and back), mirrored on the CPU by the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, assert_close, to_dev, to_raw
from oracle import block_manager as obm
from paged_kv_cache_368_b200 import inputs, libpaged

pytestmark = pytest.mark.gpu


def _rand_pool(rng, nb, kvh, bs, d, dtype):
    return inputs._normal_raw16(rng, (nb, kvh, bs, d), dtype)


@pytest.mark.parametrize("dtype,kvh,bs,d", [("f16", 4, 16, 128), ("bf16", 2, 8, 64), ("f16", 1, 64, 128)])
def test_copy_blocks_bit_exact(dtype, kvh, bs, d):
    rng = np.random.default_rng(3)
    nb = 40
    k, v = _rand_pool(rng, nb, kvh, bs, d, dtype), _rand_pool(rng, nb, kvh, bs, d, dtype)
    pairs = [(3, 10), (7, 0), (39, 21), (5, 6)]
    kd, vd = to_dev(k, dtype), to_dev(v, dtype)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    libpaged.copy_blocks(kd, vd, torch.tensor(pairs, dtype=torch.int64, device="cuda"), err_flags=err)
    torch.cuda.synchronize()
    assert np.array_equal(to_raw(kd), obm.copy_blocks(k, pairs))
    assert np.array_equal(to_raw(vd), obm.copy_blocks(v, pairs))
    assert int(err.item()) == 0
    # an out-of-range pair is skipped and flagged, the others still happen
    libpaged.copy_blocks(kd, vd, torch.tensor([(1, nb + 3), (2, 4)], dtype=torch.int64, device="cuda"),
                         err_flags=err)
    torch.cuda.synchronize()
    assert int(err.item()) & libpaged.ERRF_BLOCK_RANGE
    assert np.array_equal(to_raw(kd)[4], to_raw(kd)[2])


def test_copy_blocks_rejects_host_pair_list():
    kd = torch.zeros((4, 1, 16, 64), dtype=torch.float16, device="cuda")
    pairs = np.array([[0, 1]], dtype=np.int64)  # pageable host memory
    lib = libpaged._setup_block_api(libpaged.load())
    st = lib.pa_copy_blocks(kd.data_ptr(), kd.data_ptr(), pairs.ctypes.data, 1, 1, 64, 16, 4, 0, None, None)
    assert st == libpaged.PA_ERR_INVALID


def test_swap_out_and_in_through_pinned_host_memory():
    rng = np.random.default_rng(4)
    nb_dev, nb_host, kvh, bs, d = 32, 20, 2, 16, 128
    pool = _rand_pool(rng, nb_dev, kvh, bs, d, "bf16")
    dev_pool = to_dev(pool, "bf16")
    host_pool = torch.zeros((nb_host, kvh, bs, d), dtype=torch.bfloat16).pin_memory()
    out_pairs = torch.tensor([(5, 0), (9, 1), (31, 19)], dtype=torch.int64).pin_memory()
    libpaged.swap_blocks(dev_pool, host_pool, out_pairs)
    torch.cuda.synchronize()
    host_raw = host_pool.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(host_raw, obm.swap_blocks(pool, np.zeros_like(host_raw), out_pairs.tolist()))
    # back into other device blocks, pair list on the device this time
    in_pairs = torch.tensor([(0, 12), (1, 13), (19, 14)], dtype=torch.int64, device="cuda")
    libpaged.swap_blocks(host_pool, dev_pool, in_pairs)
    torch.cuda.synchronize()
    want = obm.swap_blocks(host_raw, pool, in_pairs.tolist())
    assert np.array_equal(to_raw(dev_pool), want)
    # pageable host memory is refused before any launch
    lib = libpaged._setup_block_api(libpaged.load())
    pageable = np.zeros((nb_host, kvh, bs, d), dtype=np.uint16)
    st = lib.pa_swap_blocks(dev_pool.data_ptr(), nb_dev, pageable.ctypes.data, nb_host, kvh * bs * d * 2,
                            in_pairs.data_ptr(), 3, None, None)
    assert st == libpaged.PA_ERR_INVALID


@pytest.mark.parametrize("dtype,heads,kvh", [("bf16", 8, 2), ("f16", 4, 4)])
def test_decode_loop_with_beams_copy_on_write_and_swap(dtype, heads, kvh):
    rng = np.random.default_rng(11)
    nb, bs, d = 48, 16, 128
    G = heads // kvh
    dt = torch.bfloat16 if dtype == "bf16" else torch.float16
    scale = np.float32(1.0) / np.sqrt(np.float32(d))
    mgr, model = libpaged.BlockManager(nb, bs), obm.BlockManagerModel(nb, bs)
    host_mgr, host_model = libpaged.BlockManager(24, bs), obm.BlockManagerModel(24, bs)
    k_cpu = np.full((nb, kvh, bs, d), inputs.nan_bits(dtype), dtype=np.uint16)
    v_cpu = k_cpu.copy()
    k_dev, v_dev = to_dev(k_cpu, dtype), to_dev(v_cpu, dtype)
    k_host = torch.zeros((24, kvh, bs, d), dtype=dt).pin_memory()
    v_host = torch.zeros((24, kvh, bs, d), dtype=dt).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def write_tokens(slots):
        nonlocal k_cpu, v_cpu
        key = inputs._normal_raw16(rng, (len(slots), kvh, d), dtype)
        val = inputs._normal_raw16(rng, (len(slots), kvh, d), dtype)
        s = np.asarray(slots, dtype=np.int64)
        libpaged.reshape_and_cache(to_dev(key, dtype), to_dev(val, dtype), k_dev, v_dev,
                                   torch.from_numpy(s).cuda(), err_flags=err)
        k_cpu, v_cpu = oracle.reshape_and_cache(key, val, k_cpu, v_cpu, s)

    # prompts: sequence 0 with 40 tokens, sequence 1 with 17
    for seq, n in ((0, 40), (1, 17)):
        mgr.add(seq, n)
        model.add(seq, n)
        write_tokens([oracle.slot_of_position(model.tables[seq], p, bs) for p in range(n)])
    # two beams of sequence 0 share its blocks
    for child in (2, 3):
        mgr.fork(0, child)
        model.fork(0, child)
    live = [0, 1, 2, 3]
    ws = libpaged.alloc_workspace(len(live), heads, kvh, d, 256)
    for step in range(6):
        if step == 3:  # preempt beam 2: swap it out, then back in
            pairs = mgr.swap_to(host_mgr, 2)
            assert pairs.tolist() == [list(p) for p in model.swap_to(host_model, 2)]
            pp = torch.from_numpy(pairs).cuda()
            libpaged.swap_blocks(k_dev, k_host, pp)
            libpaged.swap_blocks(v_dev, v_host, pp)
            back = host_mgr.swap_to(mgr, 2)
            assert back.tolist() == [list(p) for p in host_model.swap_to(model, 2)]
            bp = torch.from_numpy(back).cuda()
            libpaged.swap_blocks(k_host, k_dev, bp)
            libpaged.swap_blocks(v_host, v_dev, bp)
            torch.cuda.synchronize()
            k_cpu = obm.swap_blocks(k_cpu, k_cpu, [(s, dd) for (s, _), (_, dd) in zip(pairs, back)])
            v_cpu = obm.swap_blocks(v_cpu, v_cpu, [(s, dd) for (s, _), (_, dd) in zip(pairs, back)])
        mb = 8
        tables, ctx, slots, cow = mgr.prepare_decode(live, mb)
        want_cow = []
        for i, s in enumerate(live):
            slot, c = model.append_slot(s)
            assert slot == slots[i] and ctx[i] == model.lens[s]
            if c:
                want_cow.append(list(c))
        assert cow.tolist() == want_cow
        if len(cow):
            libpaged.copy_blocks(k_dev, v_dev, torch.from_numpy(cow).cuda(), err_flags=err)
            k_cpu, v_cpu = obm.copy_blocks(k_cpu, cow.tolist()), obm.copy_blocks(v_cpu, cow.tolist())
        write_tokens(slots.tolist())
        q = inputs._normal_raw16(rng, (len(live), heads, d), dtype)
        out = torch.empty((len(live), heads, d), dtype=dt, device="cuda")
        libpaged.decode(out, to_dev(q, dtype), k_dev, v_dev, torch.from_numpy(tables).cuda(),
                        torch.from_numpy(ctx).cuda(), float(scale), max_context_len=mb * bs, workspace=ws,
                        err_flags=err)
        torch.cuda.synchronize()
        assert np.array_equal(to_raw(k_dev), k_cpu) and np.array_equal(to_raw(v_dev), v_cpu), f"pool at step {step}"
        ref = oracle.decode(q, k_cpu, v_cpu, tables, ctx, scale, dtype)
        assert_close(to_raw(out), ref, dtype, f"step {step}")
        assert int(err.item()) == 0
    # beams 0 and 3 still share the full prefix blocks; their last blocks were
    # split by copy on write
    t0, t3 = mgr.block_table(0), mgr.block_table(3)
    assert t0[:2] == t3[:2] and t0[2] != t3[2]
