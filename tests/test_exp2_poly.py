"""The FMA-pipe exponential of the attention softmaxes (prefill and decode), checked on the CPU.

The kernels evaluate 2^x for a quarter of the attention probabilities as round-to-nearest
range reduction (add / subtract 1.5 * 2^23), a cubic in the remainder, and an integer add into
the exponent field.  This test re-derives the cubic with the fitting script that sits beside
the kernel, checks that the kernel source carries exactly those coefficients, and emulates the
float32 bit-level evaluation with numpy against exact 2^x.
"""
import importlib.util
import pathlib
import re

import numpy as np

CSRC = pathlib.Path(__file__).resolve().parents[1] / "differential_latent_attention_fwd_b200" / "csrc"


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", CSRC / "exp2_poly_fit.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients():
    src = (CSRC / "gdla_common.cuh").read_text()
    body = src[src.index("void exp2_poly2("):]
    body = body[: body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"(\d\.\d+)f", body)]
    # c3 appears as the Horner seed (twice), then c2, c1, c0
    return np.array([nums[4], nums[3], nums[2], nums[0]], dtype=np.float32)


def _emulate(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    q = np.full_like(f, c[3])
    for k in (2, 1, 0):
        q = (q * f + c[k]).astype(np.float32)
    bits = (t.view(np.int32).astype(np.int64) * 8388608 + q.view(np.int32).astype(np.int64)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_carries_the_fitted_cubic():
    c = _fit_module().fit()
    np.testing.assert_array_equal(_kernel_coefficients(), c)


def test_cubic_error_below_fp16_half_ulp():
    mod = _fit_module()
    assert mod.max_rel_err_f32(mod.fit()) < 2.0 ** -12


def test_bit_level_exponential_matches_exp2():
    c = _kernel_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 200001), -np.arange(0, 126, dtype=np.float64),
                        np.array([0.5, -0.5, 7.999, -0.25])])
    got = _emulate(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x) - 1.0)
    assert rel.max() < 1e-4, rel.max()
    # below the clamp the result is a tiny value (fp16 P rounds it to 0), never inf or NaN
    low = _emulate(np.array([-200.0, -np.inf], dtype=np.float32), c)
    assert np.all(np.isfinite(low)) and np.all(low < 1e-37)
