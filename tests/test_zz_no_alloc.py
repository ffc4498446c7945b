"""pa_decode_static: decode for callers that cannot allocate device memory.

Such callers (code where cudaMalloc is not allowed, or a host that gives a
plugin only its input and output buffers) cannot provide pa_decode's
workspace; pa_decode_static uses the library's own fixed scratch array
instead.  This test calls it through the C ABI twice in a row and checks
both results against pa_decode's on the same inputs, within the attention
tolerance the other tests use.  The file is named so that pytest collects it
last; it depends on no other test.
"""
import numpy as np
import pytest
import torch

from gpu_harness import TOL, DeviceState
from paged_kv_cache_368_b200 import inputs, libpaged

pytestmark = pytest.mark.gpu

CASES = [
    dict(seed=600, num_seqs=9, num_heads=8, num_kv_heads=8, head_dim=128, block_size=16, dtype="f16",
         ctx_lo=1, ctx_hi=2500),
    dict(seed=601, num_seqs=6, num_heads=32, num_kv_heads=4, head_dim=128, block_size=32, dtype="bf16",
         ctx_lo=100, ctx_hi=4000),
    dict(seed=602, num_seqs=5, num_heads=8, num_kv_heads=4, head_dim=64, block_size=8, dtype="f16",
         ctx_lo=1, ctx_hi=700),
]


def _static_call(lib, ds, out):
    wl = ds.wl
    st = lib.pa_decode_static(
        out.data_ptr(), ds.q.data_ptr(), ds.k_cache.data_ptr(), ds.v_cache.data_ptr(), ds.tables.data_ptr(),
        wl.max_blocks_per_seq, ds.ctx.data_ptr(), wl.num_seqs, wl.max_context_len, float(wl.scale), wl.num_heads,
        wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks, libpaged.dtype_code(out.dtype), 0,
        ds.err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == libpaged.PA_OK, libpaged.load().pa_last_error().decode()


def _within(a: torch.Tensor, b: torch.Tensor, dtype: str):
    atol, rtol = TOL[dtype]
    x, y = a.double(), b.double()
    assert torch.isfinite(x).all()
    bad = (x - y).abs() > atol + rtol * y.abs()
    assert not bad.any(), f"{int(bad.sum())} elements differ beyond tolerance"


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['dtype']}-h{c['num_heads']}-kv{c['num_kv_heads']}-d{c['head_dim']}")
def test_static_scratch_decode_matches_workspace_decode(case):
    assert torch.cuda.is_available()
    lib = libpaged.load()
    wl = inputs.random_case(**case)
    ds = DeviceState(wl, full_pool=True)
    ds.append()
    ref = ds.decode().clone()
    for _ in range(2):  # two calls in a row share (and reuse) the static array
        out = torch.full_like(ref, float("nan"))
        _static_call(lib, ds, out)
        torch.cuda.synchronize()
        _within(out, ref, wl.dtype)
    assert int(ds.err.item()) == 0
