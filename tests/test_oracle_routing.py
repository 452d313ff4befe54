"""Pins for the oracle's router: top-k, tie-break, gates, histogram, bias step.

Each check here is independent of the oracle's own formulation: brute-force rank
counting instead of sorting, hand-worked values from tests/golden, closed forms and
invariants.
"""
import json
import math
import os

import numpy as np
import pytest

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


def brute_topk(logits, bias, k):
    """Expert e is chosen with rank r iff exactly r experts beat it, where e' beats e
    when its float32 score is larger, or equal with a smaller index."""
    T, E = logits.shape
    out = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        s = [float(np.float32(logits[t, e]) + np.float32(bias[e])) for e in range(E)]
        for e in range(E):
            beaten_by = sum(1 for f in range(E) if s[f] > s[e] or (s[f] == s[e] and f < e))
            if beaten_by < k:
                out[t, beaten_by] = e
    return out


def test_worked_example_routing():
    g = _golden("worked_examples.json")["routing"]
    # float64 logits: the selection still takes float32 scores, the gates see the
    # decimal values the example was worked with (2.6 is not a float32)
    logits = np.array(g["logits"], dtype=np.float64)
    bias = np.array(g["bias"], dtype=np.float32)
    idx, gate, hist = O.route(logits, bias, g["k"])
    assert idx.tolist() == g["idx"]
    np.testing.assert_allclose(gate, np.array(g["gate"]), rtol=0, atol=1e-15)
    assert hist.tolist() == g["hist"]


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("k", [1, 2, 5])
def test_topk_matches_brute_force(ties, k):
    logits = synth.make_logits(40, 12, seed=7 + k, ties=ties)
    bias = np.random.default_rng(3).integers(-2, 3, size=12).astype(np.float32) / np.float32(4.0)
    idx, _, hist = O.route(logits, bias, k)
    assert np.array_equal(idx, brute_topk(logits, bias, k))
    assert hist.sum() == 40 * k
    assert np.array_equal(hist, np.bincount(brute_topk(logits, bias, k).ravel(), minlength=12))


def test_signed_zero_ties_go_to_lower_index():
    logits = np.array([[-0.0, 0.0, -0.0, 0.0]], dtype=np.float32)
    idx, gate, _ = O.route(logits, np.zeros(4, np.float32), 3)
    assert idx.tolist() == [[0, 1, 2]]
    np.testing.assert_allclose(gate, [[1 / 3, 1 / 3, 1 / 3]], rtol=1e-15)


def test_score_is_a_float32_add():
    # 1 + 2^-30 rounds to 1 in float32: the two experts tie and the lower index wins,
    # although in float64 expert 1 would score higher.
    logits = np.array([[1.0, 1.0]], dtype=np.float32)
    bias = np.array([0.0, 2.0 ** -30], dtype=np.float32)
    idx, _, _ = O.route(logits, bias, 1)
    assert idx.tolist() == [[0]]


def test_gates_sum_to_one_and_top1_is_one():
    logits = synth.make_logits(64, 16, seed=11)
    bias = np.zeros(16, np.float32)
    _, gate, _ = O.route(logits, bias, 4)
    np.testing.assert_allclose(gate.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert (gate > 0).all()
    _, g1, _ = O.route(logits, bias, 1)
    assert np.all(g1 == 1.0)


def test_gates_use_unbiased_logits():
    # A large bias forces expert 3 in, but its gate is set by its raw logit.
    logits = np.array([[2.0, 1.0, 0.0, -3.0]], dtype=np.float32)
    bias = np.array([0.0, 0.0, 0.0, 10.0], dtype=np.float32)
    idx, gate, _ = O.route(logits, bias, 2)
    assert idx.tolist() == [[3, 0]]
    expect = [math.exp(-3.0) / (math.exp(-3.0) + math.exp(2.0)),
              math.exp(2.0) / (math.exp(-3.0) + math.exp(2.0))]
    np.testing.assert_allclose(gate[0], expect, rtol=1e-14)


def test_gates_are_shift_invariant():
    logits = synth.make_logits(32, 10, seed=5)
    bias = np.zeros(10, np.float32)
    idx0, g0, _ = O.route(logits, bias, 3)
    shift = np.arange(32, dtype=np.float32)[:, None] * np.float32(0.5)
    idx1, g1, _ = O.route(logits + shift, bias, 3)
    assert np.array_equal(idx0, idx1)
    np.testing.assert_allclose(g0, g1, rtol=1e-5)


def test_nan_is_rejected():
    logits = np.zeros((2, 4), np.float32)
    logits[1, 2] = np.nan
    with pytest.raises(ValueError):
        O.route(logits, np.zeros(4, np.float32), 2)


# ------------------------------------------------------------------------- bias step


def test_bias_step_worked_example():
    g = _golden("worked_examples.json")["bias_step"]
    b = O.bias_update(np.array(g["hist"]), np.array(g["bias"], np.float32), g["step"], g["T"], g["k"])
    expect = np.float32(g["step"]) * np.array(g["sign"], dtype=np.float32)
    assert np.array_equal(b, expect)


def test_bias_step_is_zero_mean_and_directional():
    rng = np.random.default_rng(0)
    E, T, k = 384, 16384, 8
    hist = rng.multinomial(T * k, rng.dirichlet(np.ones(E) * 3.0))
    bias = np.zeros(E, np.float32)
    for _ in range(5):                                   # several steps keep the mean at 0
        new = O.bias_update(hist, bias, 1e-3, T, k)
        step = new.astype(np.float64) - bias.astype(np.float64)
        assert abs(step.sum()) <= E * 1e-3 * np.finfo(np.float32).eps * 4
        mean_load = T * k / E
        over, under = hist > mean_load, hist < mean_load
        if over.any() and under.any():
            assert step[over].max() < step[under].min()
        bias = new
    assert abs(bias.astype(np.float64).sum()) <= 5 * E * 1e-3 * np.finfo(np.float32).eps * 8


def test_bias_step_balanced_histogram_is_a_no_op():
    E, T, k = 24, 512, 3
    hist = np.full(E, T * k // E)
    bias = np.linspace(-1, 1, E).astype(np.float32)
    assert np.array_equal(O.bias_update(hist, bias, 1e-3, T, k), bias)
