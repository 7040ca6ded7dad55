"""The FMA-pipe 2^x of the softmax (sm100.cuh: ex2_poly_pair) checked on the CPU:
its coefficients are the ones the committed fit reproduces, and an fp32 emulation of
the same steps (clamp, 1.5*2^23 shifter, exact x - rint(x), degree-3 Horner, exponent
add) stays within the fitted relative-error bound over the whole argument range the
kernel uses, against 2^x computed in fp64."""
import importlib.util
import re
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent.parent
CSRC = ROOT / "exact_attention_146_b200" / "csrc"


def kernel_coefficients():
    text = (CSRC / "sm100.cuh").read_text()
    return np.array([float(re.search(rf"kExp2C{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for i in range(4)],
                    dtype=np.float32)


def emulate(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)                      # exact, as the device's fma(n, -1, x)
    p = ((c[3] * f + c[2]).astype(f32) * f + c[1]).astype(f32)
    p = (p * f + c[0]).astype(f32)
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_reproduce_from_fit():
    spec = importlib.util.spec_from_file_location("fit", CSRC / "exp2_poly_fit.py")
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c = fit.remez_exp2(3).astype(np.float32)
    assert np.allclose(c, kernel_coefficients(), rtol=0, atol=2e-7)
    assert fit.fp32_horner_rel_error(kernel_coefficients()) < 7.6e-5


def test_relative_error_over_kernel_range():
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-125.9, 8.0, 2_000_001), np.arange(-125, 9, 0.5)]).astype(np.float32)
    y = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 7.6e-5, rel.max()


def test_tiny_and_clamped_arguments_stay_small_and_finite():
    c = kernel_coefficients()
    x = np.array([-126.0, -130.0, -1e4, -3.4e38], dtype=np.float32)
    y = emulate(x, c)
    assert np.isfinite(y).all() and (y >= 0).all() and (y < 1.2e-38 * 1.5).all()


def test_integers_are_nearly_exact_powers_of_two():
    c = kernel_coefficients()
    x = np.arange(-120, 9, dtype=np.float32)
    y = emulate(x, c).astype(np.float64)
    assert np.abs(y / np.exp2(x.astype(np.float64)) - 1).max() < 7.5e-5
