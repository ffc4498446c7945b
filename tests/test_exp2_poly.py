"""The polynomial 2^x of exp2_poly.cuh (used by the multi-token kernel to move
part of its exponentials off the special-function unit): its constants are
what fit_exp2_poly.py computes, and a float32 emulation of the device
function (same operations, same bit manipulation) is within 1.0e-4 relative
of 2^x over the range softmax uses.  The GPU test against ex2.approx is in
tests/test_gpu_prefill.py."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_368_b200", "csrc")
sys.path.insert(0, CSRC)

import fit_exp2_poly  # noqa: E402


def _header_constants():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return {k: np.float32(float(v)) for k, v in re.findall(r"constexpr float (kExp2\w+) = ([0-9.eE+-]+)f;", text)}


def test_constants_are_the_fit():
    c = _header_constants()
    fit = fit_exp2_poly.coefficients_f32()
    for i, ck in enumerate(fit):
        assert c[f"kExp2C{i}"] == ck, i
    assert c["kExp2Round"] == np.float32(1.5 * 2**23)


def test_fit_error_bound():
    assert fit_exp2_poly.max_relative_error() < 1.0e-4


def _emulate(x):
    """exp2_poly in float32, step for step."""
    c = _header_constants()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + c["kExp2Round"]).astype(f32)
    f = (x - (t - c["kExp2Round"]).astype(f32)).astype(f32)
    p = fit_exp2_poly.horner_f32(np.array([c[f"kExp2C{i}"] for i in range(4)]), f).astype(f32)
    bits = p.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF)
    bits = ((bits + 2**31) % 2**32 - 2**31).astype(np.int32)
    return bits.view(f32)


def test_emulated_device_function():
    x = np.concatenate([np.linspace(-124.9, 9.9, 300001), np.arange(-124, 10, dtype=np.float64)]).astype(np.float32)
    y = _emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.0e-4
    # clamped below: -inf and very negative inputs give 2^-125 (a normal float)
    low = _emulate(np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(low / 2.0**-125 - 1.0) < 1.0e-4)
