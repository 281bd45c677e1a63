"""The FMA-pipe 2^t of the attention kernel, emulated bit for bit in float32 on the CPU,
against its stated error bound (Cody-Waite split + minimax polynomial; the coefficients are
read from the kernel source and refitted by the committed fitting script)."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "sequence_partition_attn_b200", "csrc", "attn_tc.cu")


def kernel_coeffs():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"kC{k} = ([0-9.eE+-]+)f;", text).group(1))) for k in range(4)]


def poly_exp2_f32(t, c):
    t = np.maximum(t.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    rnd = (t + magic).astype(np.float32)
    n = (rnd - magic).astype(np.float32)
    f = (t - n).astype(np.float32)
    p = np.float32(c[3])
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)        # the kernel uses fma; error bound holds either way
    bits = p.view(np.int32) + (rnd.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_bound_over_the_kernel_range():
    c = kernel_coeffs()
    t = np.linspace(-120.0, 8.0, 2_000_001).astype(np.float32)
    y = poly_exp2_f32(t, c).astype(np.float64)
    ref = np.exp2(t.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4                # fit bound 7.5e-5 plus float32 rounding
    assert np.all(y > 0)


def test_clamp_keeps_tiny_values_tiny_and_non_negative():
    c = kernel_coeffs()
    t = np.array([-np.inf, -1e30, -200.0, -126.0, -125.7], dtype=np.float32)
    y = poly_exp2_f32(t, c)
    assert np.all(y >= 0) and np.all(y < 2.0 ** -124)


def test_fitting_script_reproduces_the_kernel_coefficients():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "sequence_partition_attn_b200", "csrc",
                                                      "fit_exp2_poly.py")],
                         capture_output=True, text=True, check=True).stdout
    fitted = [float(x) for x in re.findall(r"c\d = +([0-9.eE+-]+)", out)]
    np.testing.assert_allclose(fitted, [float(v) for v in kernel_coeffs()], rtol=1e-6)
