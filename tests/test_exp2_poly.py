"""The FMA-pipe 2^x of the attention kernel, re-evaluated on the CPU in
float32 exactly as the device code does it (round-to-nearest split with
the 1.5*2^23 constant, polynomial of exp2_poly.h, exponent-field add)."""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_exact_attn_b200", "csrc", "exp2_poly.h")


def coeffs():
    text = open(HDR).read()
    c = {int(k): np.float32(float(v)) for k, v in re.findall(r"RA_EXP2_C(\d) ([-0-9.e+]+)f", text)}
    return c[1], c[2], c[3]


def device_exp2(x):
    c1, c2, c3 = coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1)).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_the_used_range():
    x = np.linspace(-125, 9, 2_000_001, dtype=np.float32)
    got = device_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.5e-4           # far below bf16's 2^-8 rounding of P
    assert np.all(np.isfinite(got)) and np.all(got > 0)


def test_exact_at_zero_and_masked_scores_vanish():
    assert device_exp2(np.float32(0.0)) == np.float32(1.0)
    tiny = device_exp2(np.float32(-np.inf))
    assert 0 < tiny < 1e-37


def test_generated_header_is_current():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gen", os.path.join(os.path.dirname(HDR), "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c = gen.fit()
    for a, b in zip(c, coeffs()):
        assert abs(np.float32(a) - b) <= 1e-7
