"""Pins of the oracle's elementary steps: storage rounding, softmax,
LayerNorm, GELU, dropout scaling.  Each check compares with something other
than the oracle's own formula: another library's conversion, a printed
table, a closed form or an invariant."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import (gelu, gelu_grad, gelu_tanh, gelu_tanh_grad, layer_norm_backward, layer_norm_backward_from_output, layer_norm_forward,
                    round_to_storage, softmax_rows)
from oracle.layer import _apply_dropout, dropout_keep

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- rounding
def _samples(rng):
    v = np.concatenate([
        rng.normal(0, 1, 20000), rng.normal(0, 1e3, 5000), rng.normal(0, 1e-6, 5000),
        rng.uniform(-70000, 70000, 2000), np.ldexp(rng.uniform(0.5, 1, 2000), rng.integers(-30, 20, 2000)),
        [0.0, -0.0, 65504.0, 65519.9, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26],
    ])
    # exact ties between neighbouring half values
    h = rng.normal(0, 4, 4000).astype(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(h).astype(np.float16)).astype(np.float64)
    return np.concatenate([v, h + ulp / 2, h - ulp / 2])


def test_round_f16_matches_numpy():
    v = _samples(np.random.default_rng(0))
    ref = v.astype(np.float16).astype(np.float64)
    got = round_to_storage(v, "f16")
    assert np.array_equal(got, ref)


def test_round_f32_matches_numpy():
    v = np.random.default_rng(1).normal(0, 1, 50000) * np.exp(np.random.default_rng(2).normal(0, 20, 50000))
    assert np.array_equal(round_to_storage(v, "f32"), v.astype(np.float32).astype(np.float64))


def test_round_bf16_matches_torch():
    # torch converts float32 -> bfloat16 with round-to-nearest-even; start
    # from float32-representable values so that conversion is a single rounding
    rng = np.random.default_rng(3)
    v32 = np.concatenate([rng.normal(0, 1, 50000), rng.normal(0, 1e30, 1000), rng.normal(0, 1e-38, 1000)]).astype(np.float32)
    bits = v32.view(np.uint32)
    ties = ((bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)  # exact halfway points
    v32 = np.concatenate([v32, ties])
    ref = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    got = round_to_storage(v32.astype(np.float64), "bf16")
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- softmax
def test_softmax_rows_sum_to_one_and_mask():
    rng = np.random.default_rng(4)
    s = rng.normal(0, 3, (64, 50))
    s[:, 40:] = -np.inf
    p = softmax_rows(s)
    assert np.all(np.abs(p.sum(-1) - 1) <= 1e-14)
    assert np.all(p[:, 40:] == 0.0)
    assert np.all(p[:, :40] > 0)


def test_softmax_all_masked_row_is_zero():
    s = np.full((2, 8), -np.inf)
    assert np.all(softmax_rows(s) == 0.0)


def test_softmax_shift_invariance_and_uniform():
    rng = np.random.default_rng(5)
    s = rng.normal(0, 2, (10, 16))
    assert np.allclose(softmax_rows(s), softmax_rows(s + 123.0), atol=1e-15)
    assert np.allclose(softmax_rows(np.zeros((3, 7))), 1 / 7, atol=1e-16)
    # two-way closed form: p = 1 / (1 + e^-(a-b))
    a, b = 0.7, -1.3
    p = softmax_rows(np.array([[a, b]]))[0, 0]
    assert abs(p - 1 / (1 + math.exp(-(a - b)))) < 1e-15


# ---------------------------------------------------------------- LayerNorm
def test_layernorm_normalises_each_token():
    rng = np.random.default_rng(6)
    x = rng.normal(3.0, 2.5, (7, 5, 96))
    y, mean, rstd = layer_norm_forward(x, np.ones(96), np.zeros(96), 1e-12)
    assert np.allclose(y.mean(-1), 0, atol=1e-13)
    var = x.var(-1)
    assert np.allclose((y ** 2).mean(-1), var / (var + 1e-12), atol=1e-12)
    # statistics are per token over the hidden axis, not over the batch
    assert np.allclose(mean, x.mean(-1)) and mean.shape == (7, 5)


def test_layernorm_affine_and_eps():
    x = np.array([[1.0, 3.0]])  # mean 2, biased variance 1
    y, _, rstd = layer_norm_forward(x, np.array([2.0, 3.0]), np.array([0.5, -1.0]), 0.25)
    assert np.allclose(rstd, 1 / math.sqrt(1.25))
    assert np.allclose(y, [[0.5 - 2 / math.sqrt(1.25), -1 + 3 / math.sqrt(1.25)]])


def test_layernorm_backward_finite_differences():
    rng = np.random.default_rng(7)
    x = rng.normal(0, 1, (3, 24))
    g = rng.normal(1, 0.3, 24)
    b = rng.normal(0, 0.3, 24)
    dy = rng.normal(0, 1, (3, 24))
    _, mean, rstd = layer_norm_forward(x, g, b, 1e-5)
    dx, dg, db = layer_norm_backward(dy, x, mean, rstd, g)
    L = lambda x_, g_, b_: float((layer_norm_forward(x_, g_, b_, 1e-5)[0] * dy).sum())
    h = 1e-6
    for idx in [(0, 0), (1, 7), (2, 23)]:
        xp, xm = x.copy(), x.copy(); xp[idx] += h; xm[idx] -= h
        assert abs((L(xp, g, b) - L(xm, g, b)) / (2 * h) - dx[idx]) < 1e-7
    for j in [0, 11, 23]:
        gp, gm = g.copy(), g.copy(); gp[j] += h; gm[j] -= h
        assert abs((L(x, gp, b) - L(x, gm, b)) / (2 * h) - dg[j]) < 1e-7
        bp, bm = b.copy(), b.copy(); bp[j] += h; bm[j] -= h
        assert abs((L(x, g, bp) - L(x, g, bm)) / (2 * h) - db[j]) < 1e-7


def test_layernorm_backward_from_output_finite_differences():
    # the output-based form (input dropped) against central differences of the
    # forward; gamma with mixed signs, away from zero
    rng = np.random.default_rng(8)
    x = rng.normal(0.5, 2.0, (4, 32))
    g = rng.choice([-1.0, 1.0], 32) * rng.uniform(0.3, 1.5, 32)
    b = rng.normal(0, 0.5, 32)
    dy = rng.normal(0, 1, (4, 32))
    y, _, rstd = layer_norm_forward(x, g, b, 1e-5)
    dx, dg, db = layer_norm_backward_from_output(dy, y, rstd, g, b)
    L = lambda x_, g_, b_: float((layer_norm_forward(x_, g_, b_, 1e-5)[0] * dy).sum())
    h = 1e-6
    for idx in [(0, 0), (2, 13), (3, 31)]:
        xp, xm = x.copy(), x.copy(); xp[idx] += h; xm[idx] -= h
        assert abs((L(xp, g, b) - L(xm, g, b)) / (2 * h) - dx[idx]) < 1e-7
    for j in [0, 17, 31]:
        gp, gm = g.copy(), g.copy(); gp[j] += h; gm[j] -= h
        assert abs((L(x, gp, b) - L(x, gm, b)) / (2 * h) - dg[j]) < 1e-7
    assert np.allclose(db, dy.sum(axis=0), atol=1e-13, rtol=0)


# ---------------------------------------------------------------- GELU
def test_gelu_normal_table():
    tab = np.loadtxt(os.path.join(GOLDEN, "normal_cdf.txt"))
    x, phi = tab[:, 0], tab[:, 1]
    for xs in (x, -x):
        want = xs * np.where(xs >= 0, phi, 1 - phi)
        assert np.allclose(gelu(xs), want, atol=5e-15, rtol=0)


def test_gelu_identities():
    x = np.random.default_rng(8).normal(0, 3, 1000)
    assert np.allclose(gelu(x) - gelu(-x), x, atol=1e-14)
    assert gelu(np.array([0.0]))[0] == 0.0
    # the exact form differs from the tanh approximation by ~1.5e-4 at x = 1
    tanh_form = 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * (1 + 0.044715)))
    assert abs(gelu(np.array([1.0]))[0] - tanh_form) > 1e-4


def test_gelu_grad_finite_differences():
    x = np.linspace(-6, 6, 241)
    h = 1e-5
    fd = (gelu(x + h) - gelu(x - h)) / (2 * h)
    assert np.allclose(gelu_grad(x), fd, atol=1e-9)


def test_gelu_tanh_form():
    # the tanh approximation: odd-part identity (tanh is odd), zero at 0,
    # close to the exact erf form everywhere (the largest gap of the
    # approximation is a few 1e-4) but not equal to it, derivative by
    # central differences, and the asymptotes u and 0
    x = np.random.default_rng(10).normal(0, 3, 1000)
    assert np.allclose(gelu_tanh(x) - gelu_tanh(-x), x, atol=1e-14)
    assert gelu_tanh(np.array([0.0]))[0] == 0.0
    g = np.linspace(-10, 10, 20001)
    gap = np.abs(gelu_tanh(g) - gelu(g))
    assert 1e-4 < gap.max() < 1e-3
    h = 1e-5
    xs = np.linspace(-6, 6, 241)
    assert np.allclose(gelu_tanh_grad(xs), (gelu_tanh(xs + h) - gelu_tanh(xs - h)) / (2 * h), atol=1e-9)
    assert gelu_tanh(np.array([30.0]))[0] == 30.0 and gelu_tanh(np.array([-30.0]))[0] == 0.0


# ---------------------------------------------------------------- dropout
def test_dropout_scaling_exact():
    v = np.random.default_rng(9).normal(0, 1, 4096)
    keep = dropout_keep(0, 4096, 1, 0, 1234, 0.1)
    out = _apply_dropout(v, keep, 0.1)
    assert np.array_equal(out[keep], v[keep] * (1 / 0.9))
    assert np.all(out[~keep] == 0.0)
    assert np.array_equal(_apply_dropout(v, dropout_keep(0, 4096, 1, 0, 1234, 0.0), 0.0), v)
