"""The FMA-pipe exponential of the forward kernel (exp2_poly2 in
fwd_sm100.cu): its constants are the Remez fit of exp2_poly_remez.py rounded
to fp32, and the evaluation scheme -- round-to-nearest range reduction by the
1.5 * 2^23 trick, degree-3 Horner in fp32, the integer part added into the
exponent field -- keeps the relative error within the fit's bound over the
range the softmax uses (x <= 16 after the lazy running max; inputs below -125
are clamped and give 2^-125)."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attn_fwd_04_b200", "csrc")


def _kernel_constants():
    src = open(os.path.join(CSRC, "fwd_sm100.cu")).read()
    vals = {}
    for k in range(4):
        m = re.search(r"kExp2P%d = ([0-9.eE+-]+)f" % k, src)
        assert m, k
        vals[k] = float(np.float32(float(m.group(1))))
    return [vals[k] for k in range(4)]


def _remez():
    pytest.importorskip("mpmath")
    spec = importlib.util.spec_from_file_location("exp2_poly_remez",
                                                  os.path.join(CSRC, "exp2_poly_remez.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_constants_are_the_remez_fit():
    mod = _remez()
    c, emax = mod.remez(3)
    assert _kernel_constants() == [float(np.float32(x)) for x in c]
    assert emax < 7.6e-5


def _exp2_poly_fp32(x, c):
    """The kernel's steps in numpy fp32 (every operation rounded to fp32)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    big = f32(12582912.0)                     # 1.5 * 2^23
    y = (x + big).astype(f32)                 # round(x) in the low mantissa bits
    j = (y - big).astype(f32)
    fr = (x - j).astype(f32)                  # in [-1/2, 1/2]
    p = f32(c[3])
    for k in (2, 1, 0):
        p = (p * fr + f32(c[k])).astype(f32)  # fp32 Horner (fused or not: within 1 ulp)
    bits = p.view(np.uint32) + (y.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(f32)


def test_fp32_evaluation_within_the_bound():
    c = _kernel_constants()
    x = np.concatenate([np.linspace(-125.0, 16.0, 2_000_001, dtype=np.float64),
                        np.arange(-125, 17, dtype=np.float64),          # integers
                        np.arange(-125, 16, dtype=np.float64) + 0.5])   # rounding ties
    got = _exp2_poly_fp32(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / want - 1)
    assert rel.max() < 7.6e-5 + 2e-7, rel.max()


def test_clamped_inputs_give_a_tiny_normal_number():
    c = _kernel_constants()
    got = _exp2_poly_fp32(np.array([-126.0, -1000.0, -np.inf]), c)
    assert np.all(got > 0) and np.all(got < 2.0 ** -124)
    assert np.all(np.isfinite(got))
