"""The FMA-pipe exp2 used for a quarter of the forward's exponentials
(exp2_poly2 in csrc/sm100.cuh), checked on the CPU by replaying its steps in
float32 with numpy: the coefficients in the source are those the committed
fit script produces, and the result stays within the fit's relative-error
bound of 2^x over the whole argument range the kernel feeds it."""

import os
import re
import subprocess
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "exact_attention_150_b200", "csrc")


def _source_coefficients():
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = text[text.index("exp2_poly2(float2 x)"):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([-+]?\d\.\d+e[-+]\d+)f, \1f\)", body)]
    return vals  # c3, c2, c1 in order of use


def _replay(x: np.ndarray, c3, c2, c1) -> np.ndarray:
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.5))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)
    p = (f32(c3) * f + f32(c2)).astype(f32)
    p = (p * f + f32(c1)).astype(f32)
    p = (p * f + f32(1.0)).astype(f32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_source_coefficients_match_fit_script():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "exp2_fit.py")], capture_output=True, text=True,
                         check=True).stdout
    fit = [float(v) for v in re.findall(r"([-+]?\d\.\d+e[-+]\d+)f", out.splitlines()[0])]
    c0, c1, c2, c3 = fit
    assert c0 == 1.0
    assert _source_coefficients() == [c3, c2, c1]


def test_relative_error_bound():
    c3, c2, c1 = _source_coefficients()
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.arange(-126, 9, dtype=np.float64)])
    got = _replay(x, c3, c2, c1).astype(np.float64)
    rel = np.abs(got / np.exp2(x) - 1.0)
    assert rel.max() < 1.1e-4
    assert _replay(np.array([0.0]), c3, c2, c1)[0] == 1.0


def test_masked_and_tiny_arguments_give_tiny_results():
    c3, c2, c1 = _source_coefficients()
    got = _replay(np.array([-np.inf, -1e30, -200.0, -127.0, -126.6]), c3, c2, c1)
    assert np.all(got >= 0) and np.all(got < 2e-38)
