"""Pins for the multi-token (prefill / chunked-prefill) oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import paged_attention as opa
from paged_kv_cache_368_b200 import inputs


def _case(seed, S, H, KVH, d, bs, ctx, qlens, dtype="f16"):
    wl = inputs.build("pf", seed=seed, num_seqs=S, num_heads=H, num_kv_heads=KVH, head_dim=d, block_size=bs,
                      dtype=dtype, context_lens=ctx, pool_factor=1.5, poison=False)
    k, v = wl.full_pool(poison=True)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = inputs._normal_raw16(np.random.default_rng(seed + 1), (int(cu[-1]), H, d), dtype)
    return wl, k, v, cu, q


def test_single_token_rows_equal_decode():
    """Row i of a chunk equals a decode whose context ends at that row's position."""
    wl, k, v, cu, q = _case(3, 3, 4, 2, 16, 4, [9, 5, 13], [3, 5, 1])
    out = opa.prefill(q, cu, k, v, wl.block_tables, wl.context_lens, wl.scale, "f16")
    for s in range(3):
        n = cu[s + 1] - cu[s]
        for i in range(n):
            p = wl.context_lens[s] - n + i
            ref = opa.decode(q[cu[s] + i][None], k, v, wl.block_tables[s:s + 1], np.array([p + 1]), wl.scale, "f16")
            assert np.array_equal(out[cu[s] + i], ref[0])


def test_full_prompt_equals_causal_sdpa():
    """Identity tables and a whole prompt (n = ctx): torch SDPA with is_causal."""
    S, H, KVH, d, bs, L = 2, 4, 2, 16, 4, 11
    rng = np.random.default_rng(5)
    MB = -(-L // bs)
    k = inputs._normal_raw16(rng, (S * MB, KVH, bs, d), "bf16")
    v = inputs._normal_raw16(rng, (S * MB, KVH, bs, d), "bf16")
    q = inputs._normal_raw16(rng, (S * L, H, d), "bf16")
    tables = np.arange(S * MB, dtype=np.int32).reshape(S, MB)
    cu = np.array([0, L, 2 * L], dtype=np.int32)
    ctx = np.array([L, L], dtype=np.int32)
    scale = np.float32(0.3)
    out = opa.prefill(q, cu, k, v, tables, ctx, scale, "bf16")
    w = lambda a: torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64)  # noqa: E731
    for s in range(S):
        kk = w(k[s * MB:(s + 1) * MB]).permute(1, 0, 2, 3).reshape(KVH, MB * bs, d)[:, :L]
        vv = w(v[s * MB:(s + 1) * MB]).permute(1, 0, 2, 3).reshape(KVH, MB * bs, d)[:, :L]
        qq = w(q[s * L:(s + 1) * L]).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(qq[None], kk[None], vv[None], is_causal=True,
                                                               scale=float(scale), enable_gqa=True)[0]
        np.testing.assert_allclose(out[s * L:(s + 1) * L], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_brute_force_tiny_chunk():
    wl, k, v, cu, q = _case(7, 1, 2, 1, 3, 2, [5], [3])
    out = opa.prefill(q, cu, k, v, wl.block_tables, wl.context_lens, wl.scale, "f16")
    kf, vf, qf = k.view(np.float16), v.view(np.float16), q.view(np.float16)
    t = wl.block_tables[0]
    for i in range(3):
        p = 5 - 3 + i
        for h in range(2):
            sc = [float(wl.scale) * sum(float(qf[i, h, c]) * float(kf[t[j // 2], 0, j % 2, c]) for c in range(3))
                  for j in range(p + 1)]
            m = max(sc)
            e = [math.exp(x - m) for x in sc]
            ref = [sum(e[j] / sum(e) * float(vf[t[j // 2], 0, j % 2, c]) for j in range(p + 1)) for c in range(3)]
            np.testing.assert_allclose(out[i, h], ref, rtol=1e-12, atol=1e-14)


def test_empty_rows_and_sequences():
    wl, k, v, cu, q = _case(9, 3, 2, 2, 8, 4, [6, 7, 3], [0, 2, 0])
    out = opa.prefill(q, cu, k, v, wl.block_tables, wl.context_lens, wl.scale, "f16")
    assert out.shape == (2, 2, 8) and np.isfinite(out).all()


# ------------------------------------------------------------------ planted mistakes
# Each mutant is a plausible slip in the prefill oracle (planted here, on the
# CPU); at least one of the pins above must reject it.

def _mutant(last_offset=1, ignore_prefix=False, no_causal=False):
    def prefill(q, cu_q, k_cache, v_cache, block_tables, context_lens, scale, dtype):
        total, H, d = q.shape
        out = np.zeros((total, H, d))
        sc = float(np.float32(scale))
        for s in range(len(context_lens)):
            lo, hi, L = int(cu_q[s]), int(cu_q[s + 1]), int(context_lens[s])
            n = hi - lo
            if n == 0 or L == 0:
                continue
            k64 = opa.gather(k_cache, block_tables[s], L, dtype)
            v64 = opa.gather(v_cache, block_tables[s], L, dtype)
            for i in range(n):
                p = i if ignore_prefix else L - n + i
                end = L if no_causal else min(L, max(1, p + last_offset))
                out[lo + i] = opa.attend(opa.widen(q[lo + i], dtype), k64[:, :end], v64[:, :end], sc)
        return out
    return prefill


PREFILL_MUTANTS = {
    "excludes own position": _mutant(last_offset=0),
    "sees the next position": _mutant(last_offset=2),
    "ignores the cached prefix": _mutant(ignore_prefix=True),
    "no causal mask": _mutant(no_causal=True),
}
PREFILL_PINS = (test_single_token_rows_equal_decode, test_full_prompt_equals_causal_sdpa, test_brute_force_tiny_chunk)


def test_unmutated_oracle_passes_every_pin():
    for pin in PREFILL_PINS:
        pin()


@pytest.mark.parametrize("name", sorted(PREFILL_MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(opa, "prefill", PREFILL_MUTANTS[name])
    caught = 0
    for pin in PREFILL_PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"mutant '{name}' passed every prefill pin"
