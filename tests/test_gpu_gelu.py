"""The device GELU (erf form, Phi from Abramowitz & Stegun 26.2.17 with
absolute error below 7.5e-8, evaluated in float32 with the approximate
reciprocal and base-2 exponential) against the oracle's exact GELU and its
derivative."""
import numpy as np
import pytest
import torch

import oracle
import transformer_layer_pre_b200 as tlp

pytestmark = pytest.mark.gpu


def test_device_gelu_matches_exact_erf_form():
    u = np.concatenate([np.linspace(-10, 10, 200001), np.random.default_rng(3).normal(0, 3, 100000),
                        [0.0, -0.0, 1e-30, -1e-30, 1e-6, 40.0, -40.0]]).astype(np.float32)
    g, dg = tlp.gelu_eval(torch.from_numpy(u).cuda())
    u64 = u.astype(np.float64)
    ref_g, ref_dg = oracle.gelu(u64), oracle.gelu_grad(u64)
    # |Phi error| <= 7.5e-8 (the approximation) + a few float32 ulps of 1
    # (rounding of the polynomial, reciprocal, exponential and 1 - Q); GELU
    # error <= |u| * that + float32 rounding of the product
    eps = np.finfo(np.float32).eps
    tol_g = np.abs(u64) * (7.5e-8 + 4 * eps) + 4 * eps * np.abs(ref_g)
    assert np.all(np.abs(g.cpu().double().numpy() - ref_g) <= tol_g + 1e-30)
    assert np.abs(dg.cpu().double().numpy() - ref_dg).max() <= 1e-6


def test_device_tanh_gelu_matches_the_tanh_form():
    u = np.concatenate([np.linspace(-10, 10, 200001), np.random.default_rng(4).normal(0, 3, 100000),
                        [0.0, -0.0, 1e-30, -1e-30, 1e-6, 40.0, -40.0]]).astype(np.float32)
    g, dg = tlp.gelu_eval(torch.from_numpy(u).cuda(), tanh_form=True)
    u64 = u.astype(np.float64)
    ref_g, ref_dg = oracle.gelu_tanh(u64), oracle.gelu_tanh_grad(u64)
    # tanh(|z|) = (1 - e)/(1 + e): a few float32 ulps of 1 in tanh, so the
    # GELU error is at most |u| times that plus the rounding of the product
    eps = np.finfo(np.float32).eps
    tol_g = np.abs(u64) * 4 * eps + 4 * eps * np.abs(ref_g)
    assert np.all(np.abs(g.cpu().double().numpy() - ref_g) <= tol_g + 1e-30)
    # GELU' = (1 + t)/2 + u (1 - t^2) z'(u)/2: an error dt in t moves it by at
    # most dt (1/2 + |u| z'(u)), z'(u) = sqrt(2/pi) (1 + 3 * 0.044715 u^2)
    dz = np.sqrt(2 / np.pi) * (1 + 3 * 0.044715 * u64 ** 2)
    tol_dg = 8 * eps * (1 + np.abs(u64) * dz)
    assert np.all(np.abs(dg.cpu().double().numpy() - ref_dg) <= tol_dg)
