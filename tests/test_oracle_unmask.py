"""Pins of the confidence-unmasking oracle (CPU only)."""
import numpy as np
from scipy.special import softmax

from oracle import confidence_unmask


def test_probability_is_the_softmax_of_the_argmax_token():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 3, 50)) * 3
    _, _, p, arg, _ = confidence_unmask(x, np.zeros((2, 3)), np.ones((2, 3), bool))
    sm = softmax(x, axis=2)
    assert np.array_equal(arg, sm.argmax(axis=2))
    assert np.allclose(p, sm.max(axis=2), rtol=1e-14)


def test_two_level_closed_form():
    V, a, b = 1000, 5.0, 1.0
    x = np.full((1, 1, V), b)
    x[0, 0, 17] = a
    _, _, p, arg, _ = confidence_unmask(x, np.zeros((1, 1)), np.ones((1, 1), bool))
    assert arg[0, 0] == 17
    assert abs(p[0, 0] - 1.0 / (1.0 + (V - 1) * np.exp(b - a))) < 1e-15


def test_commit_rule_threshold_and_untouched_positions():
    V = 10
    x = np.zeros((1, 4, V))
    x[0, 0, 3] = 20.0          # p ~ 1: commits
    x[0, 1, 4] = np.log(0.79 * (V - 1) / 0.21)  # p = 0.79: below the threshold
    x[0, 2, 5] = 20.0          # confident but already committed: untouched
    tokens = np.array([[-1, -1, 42, -1]])
    masked = np.array([[True, True, False, True]])
    t, m, p, arg, n = confidence_unmask(x, tokens, masked, gamma=0.8)
    assert abs(p[0, 1] - 0.79) < 1e-12
    assert t.tolist() == [[3, -1, 42, -1]] and m.tolist() == [[False, True, False, True]] and n.tolist() == [1]


def test_fallback_commits_the_most_confident_masked_position_only_when_none_passes():
    x = np.zeros((2, 3, 8))
    x[:, 1, 2] = 1.0           # position 1 is the most confident but far below 0.8
    tokens = np.full((2, 3), -1)
    masked = np.ones((2, 3), bool)
    t, m, _, _, n = confidence_unmask(x, tokens, masked, gamma=0.8, min_one=True)
    assert t[0].tolist() == [-1, 2, -1] and m[0].tolist() == [True, False, True] and n.tolist() == [1, 1]
    t2, m2, _, _, n2 = confidence_unmask(x, tokens, masked, gamma=0.8, min_one=False)
    assert (t2 == -1).all() and m2.all() and n2.tolist() == [0, 0]


def test_ties_take_the_lowest_index_and_uniform_logits():
    x = np.zeros((1, 2, 6))
    x[0, 0, [1, 4]] = 3.0      # tie between vocabulary entries 1 and 4
    _, _, p, arg, _ = confidence_unmask(x, np.zeros((1, 2)), np.ones((1, 2), bool), min_one=False)
    assert arg[0, 0] == 1 and arg[0, 1] == 0
    assert abs(p[0, 1] - 1 / 6) < 1e-15
