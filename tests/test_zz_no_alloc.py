"""pa_decode_static: decode for callers that cannot allocate device memory.

Such callers (a plugin whose host application owns every device allocation
and hands it only input and output buffers, or code under a policy that
forbids cudaMalloc on its path) cannot provide pa_decode's workspace;
pa_decode_static uses the library's own fixed scratch array instead.  These
tests call it through the C ABI twice in a row and check each result against
pa_decode's on the same inputs and the same launch grid: the two paths run the
same kernel on the same grid, so the outputs must be bit-identical.  They also
check that the calls allocate no device memory.  The file is named so that
pytest collects it last; it depends on no other test and passes alone in a
fresh process.
"""
import numpy as np
import pytest
import torch

from gpu_harness import DeviceState, assert_close, reference_full
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


def _static_call(lib, ds, out, max_ctas=0):
    wl = ds.wl
    st = lib.pa_decode_static(
        out.data_ptr(), ds.q.data_ptr(), ds.k_cache.data_ptr(), ds.v_cache.data_ptr(), ds.tables.data_ptr(),
        wl.max_blocks_per_seq, ds.ctx.data_ptr(), wl.num_seqs, wl.max_context_len, float(wl.scale), wl.num_heads,
        wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks, libpaged.dtype_code(out.dtype), max_ctas,
        ds.err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == libpaged.PA_OK, lib.pa_last_error().decode()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("max_ctas", [0, 5])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['dtype']}-h{c['num_heads']}-kv{c['num_kv_heads']}-d{c['head_dim']}")
def test_static_scratch_decode_matches_workspace_decode(case, max_ctas):
    assert torch.cuda.is_available()
    lib = libpaged.load()
    wl = inputs.random_case(**case)
    ds = DeviceState(wl, full_pool=True)
    ds.append()
    ref = ds.decode(max_ctas=max_ctas).clone()
    torch.cuda.synchronize()
    ref_oracle, _, _ = reference_full(wl)
    assert_close(_bits(ref).view(np.uint16), ref_oracle, wl.dtype, "pa_decode")
    for _ in range(2):  # two calls in a row share (and reuse) the static array
        out = torch.full_like(ref, float("nan"))
        _static_call(lib, ds, out, max_ctas)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(out), _bits(ref)), "pa_decode_static differs from pa_decode on the same grid"
    assert int(ds.err.item()) == 0


def test_static_calls_allocate_nothing():
    """After one call has set the scratch up, further calls change neither
    torch's allocator nor the device's free memory."""
    lib = libpaged.load()
    wl = inputs.random_case(**CASES[1])
    ds = DeviceState(wl, full_pool=True)
    ds.append()
    out = torch.empty_like(ds.q)
    _static_call(lib, ds, out)
    torch.cuda.synchronize()
    allocated = torch.cuda.memory_allocated()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(4):
        _static_call(lib, ds, out)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == allocated
    assert free_after == free_before
    assert int(ds.err.item()) == 0
