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


# ---- the degree-2 form used by the FP8 (SAGE-style) softmax, whose P values
# are rounded to e4m3 right after

SAGE_SRC = os.path.join(ROOT, "audio_diffusion_transformer_h3_b200", "csrc", "attn_sage.cuh")


def _deg2_body():
    text = open(SAGE_SRC).read()
    body = text[text.index("void exp2_fma2_deg2("):]
    return body[:body.index("\n}\n")]


def exp2_deg2_emulated(x):
    # the float32 steps of exp2_fma2_deg2, constants read from the kernel source
    consts = [np.float32(v) for v in re.findall(r'"f"\(([-0-9.eE]+)f\)', _deg2_body())]
    shift, nshift, m1, c0, c1, c2 = consts
    clamp = np.float32(re.search(r"fmaxf\(x0, (-?[0-9.]+)f\)", _deg2_body()).group(1))
    x = np.maximum(x.astype(np.float32), clamp)
    t = (x + shift).astype(np.float32)
    r = (t + nshift).astype(np.float32)
    f = _f32_fma(r, np.full_like(r, m1), x)
    p = _f32_fma(np.full_like(f, c2), f, np.full_like(f, c1))
    p = _f32_fma(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_deg2_steps_and_constants():
    body = _deg2_body()
    consts = [np.float32(v) for v in re.findall(r'"f"\(([-0-9.eE]+)f\)', body)]
    assert consts[:3] == [np.float32(12582912.0), np.float32(-12582912.0), np.float32(-1.0)]
    assert len(consts) == 6
    steps = re.findall(r"(add|fma)\.rn\.f32x2 (\w+), (\w+), (\w+)(?:, (\w+))?;", body)
    assert [s[:3] for s in steps] == [("add", "ta", "xa"), ("add", "ra", "ta"), ("fma", "fa", "ra"),
                                      ("fma", "pa", "c2"), ("fma", "pa", "pa")]
    assert body.count("* 8388608u +") == 2


def test_deg2_relative_error_bound():
    # below 1.8e-3 over the whole range the FP8 softmax feeds it: x - m + log2(112)
    # with the lazy maximum at most 2 above m, so x <= log2(448)
    x = np.linspace(-125.0, 9.0, 2_000_001).astype(np.float32)
    y = exp2_deg2_emulated(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1.8e-3, rel.max()
    # and it is the minimax degree-2 fit, not a loose one: the error reaches
    # 1.7e-3 (equioscillation), which a Taylor polynomial at 0 would exceed
    assert rel.max() >= 1.6e-3, rel.max()


def test_deg2_nonnegative_and_clamped():
    x = np.linspace(-140.0, 9.0, 400_001).astype(np.float32)
    y = exp2_deg2_emulated(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert np.all(y[x <= -126] < 2.0 ** -125)


def _e4m3_grid():
    # the 127 finite non-negative e4m3 values (3 mantissa bits, subnormals
    # m/8 * 2^-6, largest 448), ascending
    grid = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # NaN code
            grid.add((m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(sorted(grid))


def _e4m3_index(v):
    # index on the e4m3 grid of round-to-nearest-even(v), saturating at 448,
    # by brute force over the grid (even index = even mantissa code)
    grid = _e4m3_grid()
    v = np.minimum(np.asarray(v, dtype=np.float64), 448.0)
    i = np.clip(np.searchsorted(grid, v), 1, len(grid) - 1)
    lo, hi = grid[i - 1], grid[i]
    pick_hi = (v - lo > hi - v) | ((v - lo == hi - v) & (i % 2 == 0))
    return np.where(pick_hi, i, i - 1)


def test_e4m3_grid_brute_force():
    g = _e4m3_grid()
    assert len(g) == 127 and g[0] == 0.0 and g[1] == 2.0 ** -9 and g[-1] == 448.0
    # rounding: exact grid points map to themselves, midpoints to the even neighbour
    assert np.array_equal(g[_e4m3_index(g)], g)
    mid = 0.5 * (g[1:] + g[:-1])
    idx = _e4m3_index(mid)
    assert np.all(idx % 2 == 0) and np.all(np.abs(g[idx] - mid) == 0.5 * np.diff(g))


def test_deg2_moves_e4m3_codes_by_at_most_one_step():
    # P8 = e4m3(112 * 2^(x - m)): with the approximation the code equals the
    # exactly rounded one, or its neighbour when the exact value lies within
    # the polynomial's error of a rounding boundary
    x = np.linspace(-16.0, 2.0, 400_001)
    log2_112 = np.float32(6.807354922057604)
    xs = (x.astype(np.float32) + log2_112).astype(np.float32)
    exact = _e4m3_index(112.0 * np.exp2(x))
    approx = _e4m3_index(exp2_deg2_emulated(xs).astype(np.float64))
    assert np.abs(exact - approx).max() <= 1
    assert (exact != approx).mean() < 0.02, (exact != approx).mean()
