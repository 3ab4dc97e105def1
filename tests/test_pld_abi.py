"""The library's Progressive Layer Dropping entry points (host functions of
the C ABI, no GPU needed) against the oracle: the schedule value, the depth
profile and every keep decision, bit for bit."""
import pytest

import oracle
import transformer_layer_pre_b200 as tlp


def test_theta_and_keep_probability_match_the_oracle():
    for tb in (0.0, 0.25, 0.5, 1.0):
        for gamma in (0.001, 0.01):
            for t in (0, 1, 17, 693, 5000, 10 ** 6):
                a, b = tlp.pld_theta(tb, gamma, t), oracle.pld_theta(tb, gamma, t)
                assert abs(a - b) <= 2e-16 * max(1.0, abs(b)), (tb, gamma, t)
    for L in (1, 3, 24):
        for l in range(L):
            for th in (0.0, 0.3, 0.5, 0.999, 1.0):
                assert tlp.pld_keep_prob(l, L, th) == oracle.pld_keep_prob(l, L, th)


def test_keep_decisions_are_bit_exact():
    L = 24
    n_diff = 0
    for seed in (1234, 2 ** 40 + 7):
        for t in range(0, 3000, 3):
            th = oracle.pld_theta(0.5, 0.001, t)
            for l in range(L):
                n_diff += tlp.pld_keep(seed, t, l, L, th) != oracle.pld_keep(seed, t, l, L, th)
    assert n_diff == 0
    # steps beyond 2^32 use the counter's second word
    for t in (2 ** 32, 2 ** 32 + 5, 2 ** 45):
        for l in range(L):
            assert tlp.pld_keep(9, t, l, L, 0.5) == oracle.pld_keep(9, t, l, L, 0.5)


def test_bad_layer_index_is_rejected():
    with pytest.raises(ValueError):
        tlp.pld_keep(1, 0, 24, 24, 0.5)
    assert tlp.pld_keep_prob(-1, 24, 0.5) == -1.0
