"""Pins of the Progressive Layer Dropping oracle: closed forms of the
schedule, the depth profile, kept-frequency statistics of the draw, and
finite differences through a stack with a skipped layer."""
import math

import numpy as np
import pytest

import oracle
from oracle import LayerConfig, pld_keep, pld_keep_prob, pld_theta, stack_forward_backward


@pytest.mark.parametrize("theta_bar", [0.0, 0.1, 0.5, 0.9, 1.0])
@pytest.mark.parametrize("gamma", [0.001, 0.01])
def test_schedule_endpoints_and_half_life(theta_bar, gamma):
    # starts at 1 (no layer dropped at step 0), ends at theta_bar
    assert pld_theta(theta_bar, gamma, 0) == 1.0
    assert abs(pld_theta(theta_bar, gamma, 10 ** 7) - theta_bar) < 1e-15
    # the distance to the target halves every ln(2)/gamma steps
    t_half = math.log(2.0) / gamma
    mid = (1.0 + theta_bar) / 2
    assert pld_theta(theta_bar, math.log(2.0) / 1000, 1000) == pytest.approx(mid, abs=1e-15)
    assert pld_theta(theta_bar, math.log(2.0) / 1000, 2000) == pytest.approx((3 * theta_bar + 1) / 4, abs=1e-15)
    # integer steps bracket the half-life point: theta is monotone, so the
    # value at t_half lies between its neighbours
    lo, hi = pld_theta(theta_bar, gamma, math.ceil(t_half)), pld_theta(theta_bar, gamma, math.floor(t_half))
    assert lo - 1e-15 <= mid <= hi + 1e-15
    ts = np.arange(0, 5000, 7)
    th = np.array([pld_theta(theta_bar, gamma, int(t)) for t in ts])
    assert np.all(np.diff(th) <= 0.0)
    if theta_bar == 1.0:
        assert np.all(th == 1.0)


def test_schedule_values_at_large_and_small_rates():
    # gamma * t = 1: theta = theta_bar + (1 - theta_bar) / e
    assert pld_theta(0.5, 0.001, 1000) == pytest.approx(0.5 + 0.5 / math.e, abs=1e-15)
    assert pld_theta(0.0, 0.5, 2) == pytest.approx(1.0 / math.e, abs=1e-15)


def test_depth_profile():
    L = 24
    for theta in (1.0, 0.9, 0.5, 0.0):
        p = np.array([pld_keep_prob(l, L, theta) for l in range(L)])
        assert p[-1] == pytest.approx(theta, abs=1e-15)
        assert p[0] == pytest.approx(1.0 - (1.0 - theta) / L, abs=1e-15)
        assert p.mean() == pytest.approx(1.0 - (L + 1) / (2 * L) * (1.0 - theta), abs=1e-14)
        assert np.all(np.diff(p) <= 0.0)
    with pytest.raises(AssertionError):
        pld_keep_prob(24, 24, 0.5)


def test_draws_keep_all_at_theta_one_and_match_probabilities():
    L = 4
    assert all(pld_keep(1234, t, l, L, 1.0) for t in range(200) for l in range(L))
    n = 20000
    for l in range(L):
        p = pld_keep_prob(l, L, 0.5)
        k = sum(pld_keep(1234, t, l, L, 0.5) for t in range(n))
        assert abs(k / n - p) <= 5 * math.sqrt(p * (1 - p) / n)
    # different layers draw independently: joint frequency of two layers
    both = sum(pld_keep(99, t, 2, L, 0.5) and pld_keep(99, t, 3, L, 0.5) for t in range(n))
    pj = pld_keep_prob(2, L, 0.5) * pld_keep_prob(3, L, 0.5)
    assert abs(both / n - pj) <= 5 * math.sqrt(pj * (1 - pj) / n)


def _tiny(pre_ln=True):
    return LayerConfig(batch=1, seq=8, hidden=16, heads=2, ffn=32, attn_dropout=0.1, hidden_dropout=0.1,
                       pre_layer_norm=pre_ln, seed=7)


def _weights(rng, cfg):
    h, f = cfg.hidden, cfg.ffn_dim
    w = {"wqkv": rng.normal(0, 0.3, (3 * h, h)), "bqkv": rng.normal(0, 0.1, 3 * h),
         "wo": rng.normal(0, 0.3, (h, h)), "bo": rng.normal(0, 0.1, h),
         "ln1_g": 1 + rng.normal(0, 0.1, h), "ln1_b": rng.normal(0, 0.1, h),
         "w1": rng.normal(0, 0.3, (f, h)), "b1": rng.normal(0, 0.1, f),
         "w2": rng.normal(0, 0.3, (h, f)), "b2": rng.normal(0, 0.1, h),
         "ln2_g": 1 + rng.normal(0, 0.1, h), "ln2_b": rng.normal(0, 0.1, h)}
    return w


@pytest.mark.parametrize("pre_ln", [True, False])
def test_stack_backward_matches_finite_differences_with_a_skipped_layer(pre_ln):
    cfg = _tiny(pre_ln)
    rng = np.random.default_rng(11)
    ws = [_weights(rng, cfg) for _ in range(3)]
    x = rng.normal(0, 1, (1, cfg.seq, cfg.hidden))
    dy = rng.normal(0, 1, (1, cfg.seq, cfg.hidden))
    keep = [True, False, True]
    out = stack_forward_backward(cfg, x, None, ws, dy, keep)
    assert out["grads"][1] is None and out["grads"][0] is not None

    def loss(x_, ws_):
        return float((stack_forward_backward(cfg, x_, None, ws_, dy, keep)["y"] * dy).sum())

    h = 1e-6
    for idx in [(0, 0, 0), (0, 5, 11)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        assert abs((loss(xp, ws) - loss(xm, ws)) / (2 * h) - out["dx"][idx]) < 1e-6
    for l, name, idx in [(0, "w1", (3, 4)), (0, "ln1_g", (2,)), (2, "wqkv", (20, 1)), (2, "b2", (5,))]:
        wp = [dict(w) for w in ws]
        wm = [dict(w) for w in ws]
        wp[l][name] = ws[l][name].copy()
        wm[l][name] = ws[l][name].copy()
        wp[l][name][idx] += h
        wm[l][name][idx] -= h
        fd = (loss(x, wp) - loss(x, wm)) / (2 * h)
        assert abs(fd - out["grads"][l][name][idx]) < 1e-6, (l, name)


def test_skipped_layers_are_the_identity():
    cfg = _tiny()
    rng = np.random.default_rng(12)
    ws = [_weights(rng, cfg) for _ in range(2)]
    x = rng.normal(0, 1, (1, cfg.seq, cfg.hidden))
    dy = rng.normal(0, 1, (1, cfg.seq, cfg.hidden))
    none = stack_forward_backward(cfg, x, None, ws, dy, [False, False])
    assert np.array_equal(none["y"], x) and np.array_equal(none["dx"], dy)
    assert none["grads"] == [None, None]
    # the dropout stream of a layer depends on its position in the stack
    # (philox_offset = layer id), not on which other layers ran
    only1 = stack_forward_backward(cfg, x, None, ws, dy, [False, True])
    direct = oracle.layer_forward_backward(LayerConfig(**{**cfg.__dict__, "philox_offset": 1}), x, None, ws[1], dy)
    assert np.array_equal(only1["y"], direct["y"]) and np.array_equal(only1["dx"], direct["dx"])
