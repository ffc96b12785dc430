"""CPU checks of the polynomial 2^x the kernels run on the FMA pipe
(nea_device.cuh, exp2_poly2): its coefficients are the ones the committed
fit produces, and the algorithm, replayed step by step in float32, stays
within its stated relative error over the whole range the softmax uses."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "causal_gqa_attention_sm_b200", "csrc")


def _coefficients_in_source():
    src = open(os.path.join(CSRC, "nea_device.cuh")).read()
    body = src[src.index("uint64_t exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body) if float(v) != 12582912.0]
    # order in the source: c3, c2, c1, c0 (Horner from the top)
    assert len(vals) == 4, vals
    return np.array(vals[::-1], dtype=np.float32)


def test_coefficients_match_the_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c, err = mod.fit()
    np.testing.assert_array_equal(c, _coefficients_in_source())
    assert err < 7.5e-5


def _replay(x):
    """The device steps in float32: clamp, round to the nearest integer with
    the 1.5 * 2^23 trick, polynomial on the remainder, integer add of j << 23
    to the polynomial's bits; then 0 below the clamp and NaN through."""
    c0, c1, c2, c3 = _coefficients_in_source()
    f32 = np.float32
    x_in = x.astype(f32)
    x = np.maximum(x_in, f32(-125.0))
    magic = f32(12582912.0)
    y = (x + magic).astype(f32)
    f = (x - (y - magic).astype(f32)).astype(f32)
    p = (f * c3 + c2).astype(f32)
    p = (p * f + c1).astype(f32)
    p = (p * f + c0).astype(f32)
    bits = (p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    r = bits.astype(np.uint32).view(np.float32)
    with np.errstate(invalid="ignore"):
        return np.where(x_in >= f32(-125.0), r, np.where(x_in < f32(-125.0), f32(0.0), x_in))


def test_replayed_algorithm_relative_error():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9) + 0.5]).astype(np.float32)
    got = _replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 8e-5, rel.max()


def test_below_the_range_gives_zero_and_nan_passes_through():
    """Masked scores (-inf) must contribute exactly nothing, like the
    exponential unit's flush-to-zero 2^x, and a NaN score must stay NaN."""
    x = np.array([-np.inf, -1e30, -200.0, -126.0, np.nan], dtype=np.float32)
    got = _replay(x)
    assert np.all(got[:4] == 0.0)
    assert np.isnan(got[4])
