"""The bounded barrier wait behind every kernel gives up, flags the timeout
and returns, and the CUDA context stays usable afterwards.  The failure is
made on purpose without any fault: the waits are on barriers that nothing
ever completes (a flag that nothing sets), with a 2 ms limit."""
import time

import numpy as np
import pytest
import torch

from gpu_harness import DeviceState, assert_close, reference_full, to_raw
from paged_kv_cache_368_b200 import inputs, libpaged

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    err = torch.zeros(2, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    libpaged.selftest_wait_timeout(err, limit_ns=2_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert err.tolist() == [libpaged.ERRF_TIMEOUT, libpaged.ERRF_TIMEOUT]
    assert elapsed < 5.0
    # the same context still runs a decode step correctly
    wl = inputs.config(0)
    ds = DeviceState(wl, full_pool=True)
    out = ds.step()
    ref, k_ref, v_ref = reference_full(wl)
    assert np.array_equal(to_raw(ds.k_cache), k_ref)
    assert_close(out, ref, wl.dtype, "decode after the timeout self-test")
    assert int(ds.err.item()) == 0
