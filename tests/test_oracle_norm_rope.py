"""Pins for the oracle's per-head RMSNorm and RoPE.

RMSNorm follows the per-head RMS form in soft3/glia/run/arch/decoder/forward.rs
(forward_layer): sumsq, rms = sqrt(sumsq * (1/D) + eps), x * (1/rms), with the
weight applied after the normalisation (makarna/pkg/model/arch/hybrid_decoder.go,
QNorm/KNorm). RoPE is read as rotate-half with angle p * theta^(-2i/D)
(the pages leave the formula to HybridRoPE / Op::Rope, whose bodies are absent).
Every check here is a closed form, an exact invariant or a library routine,
never a re-typing of the oracle's own loops.
"""

import math

import numpy as np
import pytest

f32 = np.float32


def ulp(x):
    return np.spacing(np.abs(np.asarray(x, dtype=np.float32))).astype(np.float64)


# ----------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_row_closed_form(orc):
    rng = np.random.default_rng(1)
    D, eps = 128, 1e-6
    w = (1 + 0.1 * rng.standard_normal(D)).astype(f32)
    for c in (0.37, -2.5, 11.0, 1e-3):
        x = np.full(D, c, dtype=f32)
        y = orc.rmsnorm_row(x, w, eps).astype(np.float64)
        want = w.astype(np.float64) * float(f32(c)) / math.sqrt(float(f32(c)) ** 2 + float(f32(eps)))
        assert np.all(np.abs(y - want) <= 3 * ulp(want)), c


def test_rmsnorm_pythagorean_row(orc):
    # x = (3, 4), eps = 0: mean square 12.5, so y = (3, 4) / sqrt(12.5)
    y = orc.rmsnorm_row(np.array([3, 4], dtype=f32), None, 0.0).astype(np.float64)
    want = np.array([3, 4]) / math.sqrt(12.5)
    assert np.all(np.abs(y - want) <= 2 * ulp(want))


def test_rmsnorm_output_mean_square(orc):
    rng = np.random.default_rng(2)
    D, eps = 128, 1e-6
    for _ in range(50):
        x = rng.standard_normal(D).astype(f32) * f32(rng.uniform(0.01, 10))
        y = orc.rmsnorm_row(x, None, eps).astype(np.float64)
        ms = np.mean(x.astype(np.float64) ** 2)
        assert abs(np.mean(y ** 2) - ms / (ms + eps)) < 2e-6


def test_rmsnorm_power_of_two_scale_invariance(orc):
    # with eps = 0 every step scales exactly by powers of two
    rng = np.random.default_rng(3)
    x = rng.standard_normal(64).astype(f32)
    w = (1 + 0.1 * rng.standard_normal(64)).astype(f32)
    base = orc.rmsnorm_row(x, w, 0.0)
    for k in (-6, -1, 3, 9):
        assert np.array_equal(orc.rmsnorm_row(x * f32(2.0 ** k), w, 0.0), base)


def test_rmsnorm_sums_squares_sequentially(orc):
    # x = (2^12, 1, 1, ..., 1), D = 128, eps = 0. In order d = 0, 1, ... the
    # running sum sits at 2^24 where adding 1 is a tie that rounds back to
    # 2^24, so the fp32 sum of squares is exactly 2^24 (a pairwise or fp64 sum
    # would include the 127 ones). rms = sqrt(2^24 / 128) = sqrt(131072).
    D = 128
    x = np.ones(D, dtype=f32)
    x[0] = f32(4096.0)
    y = orc.rmsnorm_row(x, None, 0.0)
    inv = f32(1.0) / f32(np.sqrt(f32(131072.0)))
    assert y[1] == inv and y[0] == f32(4096.0) * inv


# -------------------------------------------------------------------- RoPE
def test_rope_table_position_zero_is_identity(orc):
    t = orc.rope_table(1e4, 64, 1)
    assert np.all(t[0, :, 0] == 1.0) and np.all(t[0, :, 1] == 0.0)
    x = np.random.default_rng(4).standard_normal(64).astype(f32)
    assert np.array_equal(orc.rope_row(x, t[0]), x)


def test_rope_table_frequencies(orc):
    # i = 0 has frequency 1; i = D/4 has frequency theta^(-1/2) (0.01 at 1e4)
    D, theta = 64, 1e4
    t = orc.rope_table(theta, D, 3000).astype(np.float64)
    p = np.arange(3000, dtype=np.float64)
    for i, fr in ((0, 1.0), (D // 4, theta ** -0.5), (D // 2 - 1, theta ** (-(D - 2) / D))):
        c, s = np.cos(p * fr), np.sin(p * fr)
        tol_c = ulp(c) + 1e-15 * (1 + p)
        tol_s = ulp(s) + 1e-15 * (1 + p)
        assert np.all(np.abs(t[:, i, 0] - c) <= tol_c), i
        assert np.all(np.abs(t[:, i, 1] - s) <= tol_s), i


def test_rope_rotate_half_basis_vectors(orc):
    # e_0 rotates into the plane (0, D/2); e_{D/2} into (-sin, cos)
    D = 8
    t = orc.rope_table(1e4, D, 50)
    for p in (1, 7, 49):
        c, s = t[p, 0]
        e0 = np.zeros(D, f32); e0[0] = 1
        eh = np.zeros(D, f32); eh[D // 2] = 1
        y0, yh = orc.rope_row(e0, t[p]), orc.rope_row(eh, t[p])
        w0 = np.zeros(D, f32); w0[0], w0[D // 2] = c, s
        wh = np.zeros(D, f32); wh[0], wh[D // 2] = -s, c
        assert np.array_equal(y0, w0) and np.array_equal(yh, wh)
    # pair i=1 uses frequency theta^(-2/D)
    e1 = np.zeros(D, f32); e1[1] = 1
    y = orc.rope_row(e1, t[3])
    ang = 3 * 1e4 ** (-2 / D)
    assert abs(y[1] - math.cos(ang)) < 1e-7 and abs(y[1 + D // 2] - math.sin(ang)) < 1e-7


def test_rope_preserves_pair_norms(orc):
    rng = np.random.default_rng(5)
    D = 128
    t = orc.rope_table(5e5, D, 5000)
    for p in rng.integers(0, 5000, size=40):
        x = rng.standard_normal(D).astype(f32)
        y = orc.rope_row(x, t[p]).astype(np.float64)
        xd = x.astype(np.float64)
        h = D // 2
        assert np.allclose(y[:h] ** 2 + y[h:] ** 2, xd[:h] ** 2 + xd[h:] ** 2, rtol=1e-6, atol=1e-6)


def test_rope_relative_position(orc):
    # <rope(q, p), rope(k, p')> depends only on p - p'
    rng = np.random.default_rng(6)
    D = 128
    t = orc.rope_table(1e4, D, 4000)
    q = rng.standard_normal(D).astype(f32)
    k = rng.standard_normal(D).astype(f32)
    for _ in range(30):
        p, pp, sh = (int(v) for v in rng.integers(0, 1300, size=3))
        a = float(np.dot(orc.rope_row(q, t[p]).astype(np.float64), orc.rope_row(k, t[pp]).astype(np.float64)))
        b = float(np.dot(orc.rope_row(q, t[p + sh]).astype(np.float64), orc.rope_row(k, t[pp + sh]).astype(np.float64)))
        assert abs(a - b) < 2e-4 * (1 + abs(a))


def test_softmax_scale_is_float32_of_inverse_sqrt(orc):
    # makarna/pkg/model/arch/hybrid_decoder.go: scale := float32(1.0 / math.Sqrt(float64(cfg.HeadDim)))
    for D in (64, 96, 128, 256):
        assert orc.softmax_scale(D) == float(f32(1.0 / math.sqrt(D)))
