"""Error bound of the FMA-pipe 2^x used for part of the softmax exponentials.

The kernel's exp2_fma (csrc/sm100.cuh) splits x = j + f with j = rint(x)
(add/subtract 1.5 * 2^23), evaluates a degree-3 polynomial p(f) ~ 2^f and adds
j to the exponent field. This test re-evaluates the same float32 steps on the
CPU with the coefficients read from the kernel source and checks the result
against 2^x: relative error <= 1e-4 on [-125, 8] (far below the 2^-9 relative
rounding of the bf16 P values it produces), exact powers of two at integers
within that bound, monotone non-negative output, and tiny non-negative output
at the clamp (x <= -126).
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "audio_diffusion_transformer_h3_b200", "csrc", "sm100.cuh")


def _coeffs():
    text = open(SRC).read()
    body = text[text.index("float exp2_fma(float x)"):]
    body = body[:body.index("\n}\n")]
    vals = dict(re.findall(r"\b(c[0-3]) = ([0-9.eE+-]+)f", body))
    shift = float(re.search(r"kShift = ([0-9.]+)f", body).group(1))
    clamp = float(re.search(r"fmaxf\(x, (-?[0-9.]+)f\)", body).group(1))
    return [np.float32(vals[f"c{i}"]) for i in range(4)], np.float32(shift), np.float32(clamp)


def _f32_fma(a, b, c):
    # fused multiply-add of float32 operands, rounded once to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_emulated(x):
    (c0, c1, c2, c3), shift, clamp = _coeffs()
    x = np.maximum(x.astype(np.float32), clamp)
    t = (x + shift).astype(np.float32)
    r = (t + (-shift)).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = _f32_fma(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _f32_fma(p, f, np.full_like(f, c1))
    p = _f32_fma(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    y = exp2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 1e-4, rel.max()


def test_integers_and_halves():
    x = np.arange(-125, 9, dtype=np.float32)
    y = exp2_fma_emulated(x).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1) <= 1e-4)
    xh = x + np.float32(0.5)
    yh = exp2_fma_emulated(xh).astype(np.float64)
    assert np.all(np.abs(yh / np.exp2(xh.astype(np.float64)) - 1) <= 1e-4)


def test_monotone_and_nonnegative_including_clamp():
    x = np.linspace(-140.0, 8.0, 400_001).astype(np.float32)
    y = exp2_fma_emulated(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert np.all(y[x <= -126] < 2.0 ** -125)
    # non-decreasing up to the polynomial's relative error at the interval joints
    d = np.diff(y.astype(np.float64)) / y[1:].astype(np.float64).clip(1e-300)
    assert d.min() >= -2e-4


def test_packed_form_uses_the_same_method_and_constants():
    # exp2_fma2 (two lanes in f32x2 registers, used by the dense softmax) takes the
    # same steps as exp2_fma: the clamp, the shift pair, f = x - rint(x) (as
    # fma(rint(x), -1, x), exact), the cubic by Horner with the same coefficients,
    # and j added to the exponent field
    text = open(SRC).read()
    body = text[text.index("void exp2_fma2("):]
    body = body[:body.index("\n}\n")]
    (c0, c1, c2, c3), shift, clamp = _coeffs()
    consts = [np.float32(v) for v in re.findall(r'"f"\(([-0-9.eE]+)f\)', body)]
    assert consts == [shift, -shift, np.float32(-1.0), c0, c1, c2, c3], consts
    assert body.count(f"fmaxf(x0, {clamp:.1f}f)") == 1 and body.count(f"fmaxf(x1, {clamp:.1f}f)") == 1
    steps = re.findall(r"(add|fma)\.rn\.f32x2 (\w+), (\w+), (\w+)(?:, (\w+))?;", body)
    assert [s[:3] for s in steps] == [("add", "ta", "xa"), ("add", "ra", "ta"), ("fma", "fa", "ra"),
                                      ("fma", "pa", "c3"), ("fma", "pa", "pa"), ("fma", "pa", "pa")]
    assert body.count("* 8388608u +") == 2
