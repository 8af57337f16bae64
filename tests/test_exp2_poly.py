"""The polynomial exp2 of the attention softmax (Cody-Waite range reduction + degree-3 minimax
polynomial): the kernel's coefficients are the ones the committed Remez fit produces, and the
float32 arithmetic the kernel performs stays within its error bound of the exact 2^x."""
import math
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "pose_retrieved_kv_b200"))
import exp2_poly  # noqa: E402

KERNEL = os.path.join(ROOT, "pose_retrieved_kv_b200", "csrc", "attention_sm100.cu")


def _kernel_coefficients():
    src = open(KERNEL).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("__device__ __forceinline__ float fmax3")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    return vals          # c3, c2, c1, c0 in the order Horner uses them


def test_kernel_holds_the_fitted_coefficients():
    c = exp2_poly.coefficients_f32()
    assert _kernel_coefficients() == [float(c[3]), float(c[2]), float(c[1]), float(c[0])]


def test_remez_levels_the_relative_error():
    c, e = exp2_poly.remez()
    f = np.linspace(-0.5, 0.5, 100001)
    err = np.polyval(c[::-1], f) / 2.0 ** f - 1.0
    assert abs(np.abs(err).max() - e) <= 1e-7 and e < 1e-4
    # equioscillation: the extrema alternate in sign, five of them at the levelled size
    assert np.sum(np.abs(err) > 0.999 * e) >= 5


def test_float32_emulation_within_bound():
    x = np.linspace(-125.0, 8.0, 1_000_001).astype(np.float32)
    y = exp2_poly.exp2_emulated(x).astype(np.float64)
    rel = np.abs(y / 2.0 ** x.astype(np.float64) - 1.0)
    assert rel.max() <= 1.5e-4                  # << 2^-9, the bf16 rounding of P that follows
    # integers are near-exact powers of two, and the masked scores map to (almost) zero
    assert np.all(np.abs(exp2_poly.exp2_emulated(np.arange(-20, 8, dtype=np.float32))
                         / 2.0 ** np.arange(-20, 8) - 1) <= 1e-4)
    tiny = exp2_poly.exp2_emulated(np.array([-np.inf, -1e30, -300.0, -126.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -124)
    assert math.isfinite(float(tiny.sum()))
