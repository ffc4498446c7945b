"""GPU parity of multi-token (prefill / chunked-prefill) paged attention
against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TORCH_DT, assert_close, to_dev, to_raw
from paged_kv_cache_368_b200 import inputs, libpaged

pytestmark = pytest.mark.gpu


def _chunk_case(seed, S, H, KVH, d, bs, dtype, qlens, prefixes, pool_factor=1.5):
    """Sequences whose last q_len tokens are new: their K/V are appended into a
    NaN-poisoned pool (positions past the context stay NaN)."""
    qlens = np.asarray(qlens)
    ctx = (np.asarray(prefixes) + qlens).tolist()
    wl = inputs.build("prefill", seed=seed, num_seqs=S, num_heads=H, num_kv_heads=KVH, head_dim=d, block_size=bs,
                      dtype=dtype, context_lens=ctx, pool_factor=pool_factor, poison=True)
    k, v = wl.full_pool(poison=True)
    rng = np.random.default_rng(seed + 7)
    slots = []
    for s in range(S):
        for p in range(ctx[s] - qlens[s], ctx[s]):
            slots.append(oracle.slot_of_position(wl.block_tables[s], p, bs))
    nk = inputs._normal_raw16(rng, (len(slots), KVH, d), dtype)
    nv = inputs._normal_raw16(rng, (len(slots), KVH, d), dtype)
    k, v = oracle.reshape_and_cache(nk, nv, k, v, np.asarray(slots, dtype=np.int64))
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = inputs._normal_raw16(rng, (int(cu[-1]), H, d), dtype)
    return wl, k, v, cu, q


def _run(wl, k, v, cu, q, max_q=None, legacy=False):
    dt = TORCH_DT[wl.dtype]
    out = torch.full((q.shape[0], wl.num_heads, wl.head_dim), float("nan"), dtype=dt, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    libpaged.prefill(out, to_dev(q, wl.dtype), torch.from_numpy(cu).cuda(), to_dev(k, wl.dtype), to_dev(v, wl.dtype),
                     torch.from_numpy(wl.block_tables).cuda(), torch.from_numpy(wl.context_lens).cuda(),
                     float(wl.scale), max_q_len=int(max_q or np.diff(cu).max()), err_flags=err, legacy_mma=legacy)
    torch.cuda.synchronize()
    return to_raw(out), int(err.item())


SWEEP = [(dt, d, bs, g) for dt in ("f16", "bf16") for d in (64, 128) for bs in (8, 16, 64) for g in (1, 4)]


@pytest.mark.parametrize("legacy", [False, True], ids=["tcgen05", "mma"])
@pytest.mark.parametrize("dtype,d,bs,g", SWEEP, ids=[f"{a}-d{b}-bs{c}-g{e}" for a, b, c, e in SWEEP])
def test_chunks_match_oracle(dtype, d, bs, g, legacy):
    rng = np.random.default_rng(d + bs + g)
    S, kvh = 4, 2
    qlens = rng.integers(1, 150, S)
    prefixes = rng.integers(0, 200, S)
    prefixes[0] = 0  # one whole prompt
    wl, k, v, cu, q = _chunk_case(500 + d + bs * 3 + g, S, kvh * g, kvh, d, bs, dtype, qlens, prefixes)
    out, err = _run(wl, k, v, cu, q, legacy=legacy)
    assert err == 0
    ref = oracle.prefill(q, cu, k, v, wl.block_tables, wl.context_lens, wl.scale, dtype)
    assert_close(out, ref, dtype, f"prefill {dtype} d{d} bs{bs} g{g}")


@pytest.mark.parametrize("legacy", [False, True], ids=["tcgen05", "mma"])
@pytest.mark.parametrize("dtype,d,bs", [("f16", 64, 8), ("bf16", 128, 16), ("bf16", 64, 32), ("f16", 128, 64)])
def test_multi_tile_chunks(dtype, d, bs, legacy):
    """Chunks spanning several 128- and 256-row query tiles with ragged tails,
    after prefixes that leave the last key tile shared by two query tiles."""
    qlens = [257, 384, 511, 130, 700, 129]
    prefixes = [0, 10, 77, 1000, 3, 190]
    wl, k, v, cu, q = _chunk_case(900 + d + bs, 6, 8, 2, d, bs, dtype, qlens, prefixes)
    out, err = _run(wl, k, v, cu, q, legacy=legacy)
    assert err == 0
    ref = oracle.prefill(q, cu, k, v, wl.block_tables, wl.context_lens, wl.scale, dtype)
    assert_close(out, ref, dtype, f"prefill multi-tile {dtype} d{d} bs{bs}")


def test_single_token_chunks_equal_decode_kernel():
    """With one new token per sequence, prefill is decode: both kernels agree."""
    wl, k, v, cu, q = _chunk_case(77, 6, 8, 2, 128, 16, "bf16", [1] * 6, [5, 100, 700, 33, 1, 2000])
    out, _ = _run(wl, k, v, cu, q)
    dec = torch.empty((6, 8, 128), dtype=torch.bfloat16, device="cuda")
    libpaged.decode(dec, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"),
                    torch.from_numpy(wl.block_tables).cuda(), torch.from_numpy(wl.context_lens).cuda(),
                    float(wl.scale), max_context_len=wl.max_context_len)
    torch.cuda.synchronize()
    ref = oracle.prefill(q, cu, k, v, wl.block_tables, wl.context_lens, wl.scale, "bf16")
    assert_close(out, ref, "bf16", "prefill n=1")
    assert_close(to_raw(dec), ref, "bf16", "decode")


@pytest.mark.parametrize("legacy", [False, True], ids=["tcgen05", "mma"])
def test_long_prompt_sampled_rows(legacy):
    """The ops-transformer page's example shape: 1 sequence, 32 heads, 8192
    tokens, head_dim 64, fp16, block_size 16 -- rows checked one by one
    against the oracle's decode of the context that ends at that row."""
    L, H = 8192, 32
    wl, k, v, cu, q = _chunk_case(88, 1, H, H, 64, 16, "f16", [L], [0], pool_factor=1.0)
    out, err = _run(wl, k, v, cu, q, legacy=legacy)
    assert err == 0
    assert np.isfinite(oracle.widen(out, "f16")).all()
    kc, vc = k, v
    for row in (0, 1, 15, 16, 63, 64, 1000, 4095, 4096, L - 2, L - 1):
        heads = [0, 13, 31]
        ref = oracle.decode(q[row:row + 1][:, heads], kc[:, heads], vc[:, heads], wl.block_tables,
                            np.array([row + 1], dtype=np.int32), wl.scale, "f16")
        assert_close(out[row, heads], ref[0], "f16", f"row {row}")


def test_bad_lengths_are_clamped_and_flagged():
    wl, k, v, cu, q = _chunk_case(5, 2, 4, 4, 64, 16, "f16", [10, 5], [3, 0])
    bad_cu = cu.copy()
    bad_cu[2] = bad_cu[1] + 9  # 9 rows claimed for a context of 5
    qq = np.concatenate([q, inputs._normal_raw16(np.random.default_rng(1), (4, 4, 64), "f16")])
    out, err = _run(wl, k, v, bad_cu, qq, max_q=10)
    assert err & libpaged.ERRF_CONTEXT
    ref = oracle.prefill(q[:10], cu[:2], k, v, wl.block_tables[:1], wl.context_lens[:1], wl.scale, "f16")
    assert_close(out[:10], ref, "f16", "first sequence unaffected")


def test_malformed_offsets_touch_nothing():
    wl, k, v, cu, q = _chunk_case(6, 2, 4, 4, 128, 16, "bf16", [20, 30], [5, 0])
    bad = cu.copy()
    bad[2] = 10_000  # past total_q
    out, err = _run(wl, k, v, bad, q, max_q=64)
    assert err & libpaged.ERRF_CONTEXT
    ref = oracle.prefill(q[:20], cu[:2], k, v, wl.block_tables[:1], wl.context_lens[:1], wl.scale, "bf16")
    assert_close(out[:20], ref, "bf16", "first sequence")
    assert np.all(out[20:] == to_raw(torch.full((1,), float("nan"), dtype=torch.bfloat16))[0])  # untouched


def test_polynomial_exp2_against_exp2f():
    """The softmax's FMA-pipe 2^x, on the device, against CUDA's exp2f on the
    same inputs: relative error below 1.0e-4 over the range the kernel feeds it
    (scaled scores minus the reference max, up to the 2^8 head room), and the
    clamp to 2^-125 below."""
    x = torch.cat([torch.linspace(-124.9, 8.5, 1 << 20), torch.arange(-124, 9, dtype=torch.float32),
                   torch.rand(1 << 18) - 0.5]).cuda()
    y_poly, y_ref = libpaged.selftest_exp2(x)
    torch.cuda.synchronize()
    rel = ((y_poly.double() - y_ref.double()) / y_ref.double()).abs()
    assert float(rel.max()) < 1.0e-4
    exact = torch.exp2(x.double())
    assert float(((y_ref.double() - exact) / exact).abs().max()) < 1e-6  # exp2f itself: the yardstick
    low, _ = libpaged.selftest_exp2(torch.tensor([float("-inf"), -1e30, -300.0, -125.0], device="cuda"))
    torch.cuda.synchronize()
    assert float(((low.double() / 2.0**-125) - 1).abs().max()) < 1.0e-4
