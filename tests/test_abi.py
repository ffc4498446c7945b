"""The C-ABI library loads, exports every symbol ``include/paged.h`` declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_368_b200 import build as pbuild
from paged_kv_cache_368_b200 import libpaged

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return libpaged.load()


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert set(libpaged.SYMBOLS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    assert lib.pa_version() >= 100
    for code in range(5):
        assert libpaged.status_string(code).startswith("PA_")
    assert "unknown" in libpaged.status_string(99)


def _decode(lib, **kw):
    a = dict(out=16, q=16, k=16, v=16, tables=16, mb=4, ctx=16, S=2, maxctx=64, scale=0.1, H=4, KVH=4, D=128,
             BS=16, NB=8, dtype=0, ws=16, wsb=1 << 30, max_ctas=0, err=None, stream=None)
    a.update(kw)
    return lib.pa_decode(a["out"], a["q"], a["k"], a["v"], a["tables"], a["mb"], a["ctx"], a["S"], a["maxctx"],
                         a["scale"], a["H"], a["KVH"], a["D"], a["BS"], a["NB"], a["dtype"], a["ws"], a["wsb"],
                         a["max_ctas"], a["err"], a["stream"])


def test_decode_host_checks(lib):
    I, U = libpaged.PA_ERR_INVALID, libpaged.PA_ERR_UNSUPPORTED
    assert _decode(lib, H=6, KVH=4) == I  # heads not a multiple of kv-heads
    assert _decode(lib, H=0) == I
    assert _decode(lib, S=-1) == I
    assert _decode(lib, mb=0) == I
    assert _decode(lib, NB=0) == I
    assert _decode(lib, dtype=7) == I
    assert _decode(lib, scale=float("inf")) == I
    assert _decode(lib, max_ctas=-1) == I
    assert _decode(lib, H=48, KVH=3) == U  # group of 16 q-heads
    assert _decode(lib, D=96) == U
    assert _decode(lib, BS=24) == U
    # one launch's chunk count: 16384 sequences x 4096 kv-heads x 32 chunks = 2^31
    assert _decode(lib, S=16384, H=4096, KVH=4096, mb=32, maxctx=512) == U
    assert _decode(lib, S=16385, H=4096, KVH=4096, mb=32, maxctx=512) == U  # the same per launch
    assert _decode(lib, KVH=1 << 15, H=1 << 15) == U
    assert _decode(lib, out=None) == I
    assert _decode(lib, q=24) == I  # misaligned
    assert _decode(lib, S=0) == libpaged.PA_OK  # nothing to do, nothing touched


def _decode_static(lib, **kw):
    a = dict(out=16, q=16, k=16, v=16, tables=16, mb=4, ctx=16, S=2, maxctx=64, scale=0.1, H=4, KVH=4, D=128,
             BS=16, NB=8, dtype=0, max_ctas=0, err=None, stream=None)
    a.update(kw)
    return lib.pa_decode_static(a["out"], a["q"], a["k"], a["v"], a["tables"], a["mb"], a["ctx"], a["S"],
                                a["maxctx"], a["scale"], a["H"], a["KVH"], a["D"], a["BS"], a["NB"], a["dtype"],
                                a["max_ctas"], a["err"], a["stream"])


def test_decode_static_host_checks(lib):
    """The no-allocation entry point rejects bad and unsupported arguments
    on the host, before any CUDA call (this runs without a GPU)."""
    I, U = libpaged.PA_ERR_INVALID, libpaged.PA_ERR_UNSUPPORTED
    assert _decode_static(lib, H=6, KVH=4) == I
    assert _decode_static(lib, S=-1) == I
    assert _decode_static(lib, dtype=9) == I
    assert _decode_static(lib, max_ctas=-2) == I
    assert _decode_static(lib, out=None) == I
    assert _decode_static(lib, tables=18) == I  # misaligned int32
    assert _decode_static(lib, D=80) == U
    assert _decode_static(lib, BS=128) == U
    assert _decode_static(lib, H=64, KVH=4) == U  # group of 16
    assert _decode_static(lib, S=20000, H=4096, KVH=4096, mb=32, maxctx=512) == U  # 2^31 chunks in a launch
    assert _decode_static(lib, S=0) == libpaged.PA_OK


def test_pipelined_step_host_checks(lib):
    """The pipelined host step rejects missing buffers and events before any
    CUDA call (this runs without a GPU)."""
    I = libpaged.PA_ERR_INVALID
    f = lib.pa_decode_step_host_pipelined

    def call(**kw):
        a = dict(h_in=16, d_in=256, h_out=16, d_out=16, kc=16, vc=16, S=2, mb=4, maxctx=64, scale=0.1, H=4, KVH=4,
                 D=128, BS=16, NB=8, dt=0, ws=16, wsb=1 << 20, err=None, s=None, ins=None, outs=None, ready=16,
                 free=16, oready=16, ofree=16)
        a.update(kw)
        return f(a["h_in"], a["d_in"], a["h_out"], a["d_out"], a["kc"], a["vc"], a["S"], a["mb"], a["maxctx"],
                 a["scale"], a["H"], a["KVH"], a["D"], a["BS"], a["NB"], a["dt"], a["ws"], a["wsb"], a["err"], a["s"],
                 a["ins"], a["outs"], a["ready"], a["free"], a["oready"], a["ofree"])

    assert call(ready=None) == I
    assert call(free=None) == I
    assert call(oready=None) == I
    assert call(ofree=None) == I
    assert call(h_in=None) == I
    assert call(d_in=264) == I  # staging buffer not 256-byte aligned
    assert call(H=6, KVH=4) == I
    assert call(S=0) == libpaged.PA_OK


def test_reshape_host_checks(lib):
    f = lib.pa_reshape_and_cache
    I, U = libpaged.PA_ERR_INVALID, libpaged.PA_ERR_UNSUPPORTED
    ok = dict(key=16, value=16, kc=16, vc=16, slots=16, T=4, KVH=2, D=64, BS=16, NB=4, dt=0)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["key"], a["value"], a["kc"], a["vc"], a["slots"], a["T"], a["KVH"], a["D"], a["BS"], a["NB"],
                 a["dt"], None, None)

    assert call(T=-1) == I
    assert call(KVH=0) == I
    assert call(NB=0) == I
    assert call(dt=5) == I
    assert call(D=32) == U
    assert call(BS=12) == U
    assert call(key=None) == I
    assert call(kc=8) == I  # misaligned
    assert call(slots=4) == I  # misaligned int64
    assert call(T=0) == libpaged.PA_OK


@pytest.mark.parametrize("entry", ["pa_prefill", "pa_prefill_mma"])
def test_prefill_host_checks(lib, entry):
    f = getattr(lib, entry)
    I, U = libpaged.PA_ERR_INVALID, libpaged.PA_ERR_UNSUPPORTED
    ok = dict(out=16, q=16, cu=16, T=40, maxq=20, k=16, v=16, tables=16, mb=4, ctx=16, S=2, maxctx=64, scale=0.1,
              H=4, KVH=2, D=64, BS=16, NB=8, dt=1)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["out"], a["q"], a["cu"], a["T"], a["maxq"], a["k"], a["v"], a["tables"], a["mb"], a["ctx"],
                 a["S"], a["maxctx"], a["scale"], a["H"], a["KVH"], a["D"], a["BS"], a["NB"], a["dt"], None, None)

    assert call(H=6, KVH=4) == I
    assert call(T=-1) == I
    assert call(mb=0) == I
    assert call(dt=3) == I
    assert call(scale=float("nan")) == I
    assert call(D=256) == U
    assert call(BS=4) == U
    assert call(S=70000) == U
    assert call(out=None) == I
    assert call(cu=2) == I  # misaligned int32
    assert call(S=0) == libpaged.PA_OK
    if entry == "pa_prefill":
        assert call(scale=0.0) == U  # row maxima are taken on unscaled scores
        assert call(scale=-0.1) == U


def test_selftest_host_checks(lib):
    I = libpaged.PA_ERR_INVALID
    assert lib.pa_selftest_exp2(None, None, None, 5, None) == I
    assert lib.pa_selftest_exp2(16, 16, 16, -1, None) == I
    assert lib.pa_selftest_exp2(None, None, None, 0, None) == libpaged.PA_OK
    assert lib.pa_selftest_wait_timeout(1000, None, None) == I  # no flag words
    assert lib.pa_selftest_wait_timeout(0, 16, None) == I  # zero limit
    assert lib.pa_selftest_wait_timeout(200_000_000, 16, None) == I  # above 0.1 s


def test_workspace_size_rejects_bad_shapes(lib):
    assert lib.pa_decode_workspace_size(4, 6, 4, 128, 100) == 0
    assert lib.pa_decode_workspace_size(4, 32, 2, 128, 100) == 0  # group of 16
    assert lib.pa_decode_workspace_size(4, 8, 8, 80, 100) == 0


def test_binding_refuses_cpu_tensors(lib):
    import torch

    q = torch.zeros(1, 1, 64, dtype=torch.float16)
    kc = torch.zeros(2, 1, 16, 64, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        libpaged.decode(q.clone(), q, kc, kc.clone(), torch.zeros(1, 1, dtype=torch.int32),
                        torch.ones(1, dtype=torch.int32), 0.125, workspace=torch.zeros(16, dtype=torch.uint8))
