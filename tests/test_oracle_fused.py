"""Pins of the oracle's RMSNorm and SwiGLU, the steps the fused quantizers add in
front of the activation quantizer, against things other than the oracle itself.

  rmsnorm   hand-derived rows (golden/rmsnorm_swiglu_handmade.txt) that fix where eps
            enters, that the mean (not the sum) of squares is taken and that gamma
            multiplies per column; numpy's fp64 mean and sqrt in another arrangement
            of the formula; exact invariance under a power-of-two scale of x (eps = 0);
            unit mean square of the output; the ss_scale bracket scales r exactly
  swiglu    hand-derived textbook logistic values (same fixture); scipy's expit;
            closed forms for large |g| and g = 0; SiLU(g) - SiLU(-g) = g; exact
            linearity in u under a power-of-two scale
  the fused definitions are quantize_act(rmsnorm(x)) and quantize_act(swiglu(g, u));
  quantize_act is pinned in test_oracle.py
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_golden

scipy_special = pytest.importorskip("scipy.special")


def f32_ulp(x):
    return np.spacing(np.abs(np.asarray(x, np.float64)).astype(np.float32)).astype(np.float64)


# ---------------------------------------------------------------- rmsnorm

def test_rmsnorm_handmade():
    g = read_golden("rmsnorm_swiglu_handmade.txt")
    x = np.zeros((1, 256), np.float32)
    x[0, :2] = [3, 4]
    gam = np.ones(256, np.float32)
    gam[1] = 0.5
    y = oracle.rmsnorm(x, gam, 0.0)
    assert list(y[0, :2]) == [np.float32(float(t)) for t in g["A_y"].split()]
    assert np.all(y[0, 2:] == 0)

    xb = np.full((1, 512), float(g["B_x"]), np.float32)
    yb = oracle.rmsnorm(xb, np.ones(512, np.float32), float(g["B_eps"]))
    assert np.all(yb == np.float32(float(g["B_y"])))

    xc = np.full((1, 256), float(g["C_x"]), np.float32)
    yc = oracle.rmsnorm(xc, np.full(256, float(g["C_gamma"]), np.float32), 0.0)
    assert np.all(yc == np.float32(float(g["C_y"])))


@pytest.mark.parametrize("K", [256, 3584, 4096])
def test_rmsnorm_vs_numpy(K):
    rng = np.random.default_rng(K)
    x = (rng.standard_normal((9, K)) * rng.uniform(0.01, 100, (9, 1))).astype(np.float32)
    gam = rng.uniform(0.2, 3.0, K).astype(np.float32)
    eps = 1e-5
    y = oracle.rmsnorm(x, gam, eps)
    x64 = x.astype(np.float64)
    ref = x64 * gam.astype(np.float64) / np.sqrt(np.mean(x64 * x64, axis=1, keepdims=True) + np.float64(np.float32(eps)))
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(err <= f32_ulp(ref) * 0.5 + np.abs(ref) * 1e-13)


def test_rmsnorm_power_of_two_invariance():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 1024)).astype(np.float32)
    gam = rng.uniform(0.5, 2.0, 1024).astype(np.float32)
    y = oracle.rmsnorm(x, gam, 0.0)
    for k in (-20, -3, 5, 30):
        assert np.array_equal(oracle.rmsnorm(x * np.float32(2.0 ** k), gam, 0.0), y)
    # gamma scales the output exactly by a power of two
    assert np.array_equal(oracle.rmsnorm(x, gam * np.float32(4), 0.0), y * np.float32(4))


def test_rmsnorm_unit_mean_square_and_eps():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((6, 2048)).astype(np.float32) * 50
    y = oracle.rmsnorm(x, np.ones(2048, np.float32), 0.0).astype(np.float64)
    assert np.allclose((y * y).mean(1), 1.0, rtol=1e-6)
    # eps shrinks the output of a small row; a zero row stays zero for eps > 0
    x[0] = 1e-3
    x[1] = 0
    y2 = oracle.rmsnorm(x, np.ones(2048, np.float32), 1e-6).astype(np.float64)
    assert np.allclose(y2[0], 1e-3 / np.sqrt(1e-6 + 1e-6), rtol=1e-6)
    assert np.all(y2[1] == 0)


def test_rmsnorm_ss_scale_bracket():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((4, 768)).astype(np.float32)
    gam = np.ones(768, np.float32)
    y = oracle.rmsnorm(x, gam, 0.0)
    # scaling ss by 4 halves r exactly (eps = 0)
    assert np.array_equal(oracle.rmsnorm(x, gam, 0.0, ss_scale=4.0), y / np.float32(2))
    lo = oracle.rmsnorm(x, gam, 0.0, ss_scale=1 + 1e-9)
    hi = oracle.rmsnorm(x, gam, 0.0, ss_scale=1 - 1e-9)
    ay = np.abs(y)
    assert np.all(np.abs(lo) <= ay) and np.all(ay <= np.abs(hi))


def test_rmsnorm_rejects_bad_args():
    with pytest.raises(ValueError):
        oracle.rmsnorm(np.ones((1, 256), np.float32), np.ones(256, np.float32), -1.0)


# ---------------------------------------------------------------- swiglu

def test_swiglu_handmade():
    g = read_golden("rmsnorm_swiglu_handmade.txt")
    gs = np.array([[float(t) for t in g["S_g"].split()]], np.float32)
    hs = [float(t) for t in g["S_h"].split()]
    h = oracle.swiglu(gs, np.ones_like(gs))
    assert list(h[0]) == [np.float32(v) for v in hs]


def test_swiglu_vs_scipy_expit():
    rng = np.random.default_rng(21)
    g = (rng.standard_normal((7, 4096)) * 4).astype(np.float32)
    u = (rng.standard_normal((7, 4096)) * 3).astype(np.float32)
    h = oracle.swiglu(g, u)
    g64, u64 = g.astype(np.float64), u.astype(np.float64)
    ref = g64 * scipy_special.expit(g64) * u64
    err = np.abs(h.astype(np.float64) - ref)
    assert np.all(err <= f32_ulp(ref) * 0.5 + np.abs(ref) * 1e-14 + 1e-300)


def test_swiglu_closed_forms_and_identity():
    rng = np.random.default_rng(22)
    u = rng.standard_normal((1, 512)).astype(np.float32)
    big = np.full((1, 512), 45.0, np.float32)
    assert np.array_equal(oracle.swiglu(big, u), (big.astype(np.float64) * u).astype(np.float32))
    assert np.all(oracle.swiglu(-np.full((1, 512), 800.0, np.float32), u) == 0)
    assert np.all(oracle.swiglu(np.zeros((1, 512), np.float32), u) == 0)
    g = (rng.standard_normal((3, 1024)) * 6).astype(np.float32)
    one = np.ones_like(g)
    d = oracle.swiglu(g, one).astype(np.float64) - oracle.swiglu(-g, one).astype(np.float64)
    assert np.all(np.abs(d - g) <= 2 * f32_ulp(g) + 1e-30)
    # power-of-two scale of u is exact
    assert np.array_equal(oracle.swiglu(g, one * np.float32(8)), oracle.swiglu(g, one) * np.float32(8))


def test_swiglu_h_scale_bracket():
    rng = np.random.default_rng(23)
    g = rng.standard_normal((2, 512)).astype(np.float32)
    u = rng.standard_normal((2, 512)).astype(np.float32)
    h = oracle.swiglu(g, u)
    assert np.array_equal(oracle.swiglu(g, u, h_scale=0.5), h / np.float32(2))
    lo = np.abs(oracle.swiglu(g, u, h_scale=1 - 1e-12))
    hi = np.abs(oracle.swiglu(g, u, h_scale=1 + 1e-12))
    assert np.all(lo <= np.abs(h)) and np.all(np.abs(h) <= hi)


def test_fused_definitions_compose():
    rng = np.random.default_rng(24)
    x = rng.standard_normal((3, 512)).astype(np.float32)
    gam = rng.uniform(0.5, 1.5, 512).astype(np.float32)
    for a, b in zip(oracle.rmsnorm_quantize(x, gam, 1e-6), oracle.quantize_act(oracle.rmsnorm(x, gam, 1e-6))):
        assert np.array_equal(a, b)
    for a, b in zip(oracle.swiglu_quantize(x, x[::-1]), oracle.quantize_act(oracle.swiglu(x, x[::-1]))):
        assert np.array_equal(a, b)
