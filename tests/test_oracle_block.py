"""Pins for the oracle's forward and backward pass of the whole block.

Closed forms with one-hot and identity weights fix the [out][in] layouts and show
that every term is present; the pages' width identity and compute share fix the
shapes; finite differences in float64 fix the backward pass.
"""
import json
import math
import os

import numpy as np
import pytest

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _figures():
    with open(os.path.join(GOLDEN, "pages_figures.json"), encoding="utf-8") as f:
        return json.load(f)


MICRO = synth.MoEShape("micro", T=24, d_model=16, d_latent=8, n_experts=6, top_k=2, n_dest=2,
                       hidden_routed=8, n_shared=1, hidden_shared=8, seed=0)


def _zero_weights(s):
    w = synth.make_weights(s, np.random.default_rng(0))
    return {k: np.zeros_like(v) for k, v in w.items()}


# --------------------------------------------------------------------- pages' figures


def test_routed_width_identity_at_full_shape():
    f = _figures()["routed_width_identity"]
    s = synth.FULL
    assert s.top_k * s.hidden_routed == f["product"] == f["ratio"] * s.d_model


def test_shared_share_of_expert_compute_is_one_third():
    s = synth.FULL
    shared = s.n_shared * 3 * s.d_model * s.hidden_shared            # MACs per token
    routed = s.top_k * 3 * s.d_latent * s.hidden_routed
    assert shared * 3 == shared + routed                             # exactly 1/3
    fig = _figures()
    assert fig["shared_share_of_expert_compute"]["value"] == "1/3"
    w = fig["model_width"]
    assert (s.d_model, s.d_latent, s.n_experts, s.top_k, s.n_shared, s.hidden_shared) == (
        w["d_model"], w["d_latent"], w["n_routed"], w["top_k"], w["n_shared"], w["shared_width"])
    assert s.n_experts // s.n_dest == w["experts_per_gpu"] and s.n_waves == w["waves"]


def test_forward_flop_count_at_full_shape():
    s = synth.FULL
    per_token = O.forward_flops(s) / s.T
    # down 37.7M + router 2.36M + routed 452.98M + up 37.7M + shared 226.5M
    assert per_token == 2 * 6144 * 3072 * 2 + 2 * 3072 * 384 + 8 * 6 * 3072 * 3072 + 2 * 2 * 3 * 6144 * 3072
    assert abs(per_token - 757.3e6) < 0.1e6


# --------------------------------------------------------------------- closed forms


def test_one_hot_latent_weights_fix_layouts():
    """w_lat_down[i, j] = 1 moves input column j to latent column i; w_lat_up[p, q] = 1
    moves latent column q to output column p; shared and routed paths off."""
    s = MICRO
    w = _zero_weights(s)
    w["w_lat_down"][3, 5] = 1.0
    w["w_lat_up"][11, 3] = 1.0
    # one expert that is the identity on the latent: w1 huge on the diagonal makes
    # silu(a) ~ a, w3 = I, w2 = I / c, with a single expert chosen by every token
    c = 32.0
    for e in range(s.n_experts):
        w["w1"][e] = c * np.eye(s.hidden_routed, s.d_latent)
        w["w3"][e] = np.eye(s.hidden_routed, s.d_latent)
        w["w2"][e] = np.eye(s.d_latent, s.hidden_routed) / c
    x = np.abs(synth.make_tokens(s, np.random.default_rng(1))) + 0.5
    y, ctx = O.forward(x, w, np.zeros(s.n_experts, np.float32), s, storage="f64")
    # with zero router weights every score ties: experts 0 and 1, gates 1/2 each
    assert (ctx["idx"] == [0, 1]).all()
    kept = ctx["kept"]
    lat = x[:, 5].astype(np.float64)
    # per kept expert: silu(c*lat)*lat/c ~= lat^2 ... since w3 = I the value path is lat
    per = (c * lat / (1 + np.exp(-c * lat))) * lat / c
    want = 0.5 * per * kept.sum(axis=1)
    expect = np.zeros_like(y)
    expect[:, 11] = want
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-12)


def test_swiglu_closed_form():
    """Expert with w1 = c I, w3 = I, w2 = I: output silu(c z) * z, elementwise."""
    s = MICRO.with_(T=6)
    w = _zero_weights(s)
    w["w_lat_down"][:, : s.d_latent] = np.eye(s.d_latent)
    w["w_lat_up"][: s.d_latent, :] = np.eye(s.d_latent)
    c = 0.75
    for e in range(s.n_experts):
        w["w1"][e] = c * np.eye(s.hidden_routed, s.d_latent)
        w["w3"][e] = np.eye(s.hidden_routed, s.d_latent)
        w["w2"][e] = np.eye(s.d_latent, s.hidden_routed)
    s1 = s.with_(top_k=1, cap_send=(1000, 1), cap_recv=(1000, 1))   # all tokens pick expert 0
    x = synth.make_tokens(s1, np.random.default_rng(2))
    y, ctx = O.forward(x, w, np.zeros(s.n_experts, np.float32), s1, storage="f64")
    for t in range(s.T):
        assert ctx["kept"][t, 0]
        for i in range(s.d_latent):
            zi = float(x[t, i])
            want = (c * zi) / (1.0 + math.exp(-c * zi)) * zi
            assert abs(y[t, i] - want) < 1e-12
    assert np.all(y[:, s.d_latent:] == 0)


def test_shared_path_alone():
    """Routed path zeroed: y is the shared SwiGLU of x, expert s on hidden rows
    [s*h_s, (s+1)*h_s) of ws1/ws3 and the matching columns of ws2."""
    s = MICRO.with_(n_shared=2)
    w = synth.make_weights(s, np.random.default_rng(3))
    w = {k: v.astype(np.float64) for k, v in w.items()}
    w["w_lat_up"][:] = 0
    x = synth.make_tokens(s, np.random.default_rng(4)).astype(np.float64)
    y, _ = O.forward(x, w, np.zeros(s.n_experts, np.float32), s, storage="f64")
    hs = s.hidden_shared
    want = np.zeros_like(y)
    for t in range(s.T):
        for sx in range(2):
            for u in range(hs):
                a = float(np.dot(w["ws1"][sx * hs + u], x[t]))
                b = float(np.dot(w["ws3"][sx * hs + u], x[t]))
                hval = a / (1 + math.exp(-a)) * b
                want[t] += hval * w["ws2"][:, sx * hs + u]
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12)


def test_combine_then_project_equals_projecting_each_expert():
    """The gate-weighted sum is taken in latent space before one up-projection; by
    linearity it equals the sum of the up-projected expert outputs."""
    s = MICRO
    inp = synth.make_inputs(s)
    w = inp["weights"]
    w_no_shared = dict(w, ws2=np.zeros_like(w["ws2"]))
    y, ctx = O.forward(inp["x"], w_no_shared, inp["bias"], s, storage="f64")
    alt = np.zeros_like(y)
    for t in range(s.T):
        for j in range(s.top_k):
            if ctx["kept"][t, j]:
                alt[t] += ctx["gate"][t, j] * (w["w_lat_up"].astype(np.float64) @ ctx["Yrow"][t, j])
    np.testing.assert_allclose(y, alt, rtol=1e-10, atol=1e-12)


def test_dropped_assignments_contribute_nothing():
    s = MICRO.with_(cap_recv=(20, 100))          # tiny receiver capacity: many drops
    inp = synth.make_inputs(s)
    y, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, storage="f64")
    assert ctx["slots"]["dropped_receiver"] > 0
    # rebuild r from kept rows only, by hand
    r = np.zeros((s.T, s.d_latent))
    for t in range(s.T):
        for j in range(s.top_k):
            if ctx["slots"]["rslot"][t, j] >= 0:
                e = ctx["idx"][t, j]
                z = ctx["z"][t]
                W = {k: v.astype(np.float64) for k, v in inp["weights"].items()}
                a = W["w1"][e] @ z
                b = W["w3"][e] @ z
                r[t] += ctx["gate"][t, j] * (W["w2"][e] @ (a / (1 + np.exp(-a)) * b))
    np.testing.assert_allclose(ctx["r"], r, rtol=1e-10, atol=1e-12)


def test_all_experts_chosen_is_a_dense_softmax_mixture():
    """k = E and no caps: every expert sees every token, gates are a full softmax."""
    s = MICRO.with_(top_k=6, cap_send=(1000, 1), cap_recv=(1000, 1))
    inp = synth.make_inputs(s)
    y, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, storage="f64")
    assert ctx["kept"].all()
    lg = ctx["logits"].astype(np.float64)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    g_by_expert = np.zeros_like(p)
    np.put_along_axis(g_by_expert, ctx["idx"].astype(np.int64), ctx["gate"], axis=1)
    np.testing.assert_allclose(g_by_expert, p, rtol=1e-12)


# --------------------------------------------------------------------- backward


def _loss(x, w, bias, dy, s, logits_override=None):
    y, _ = O.forward(x, w, bias, s, storage="f64", logits_override=logits_override)
    return float((y * dy).sum())


FD_SHAPE = synth.MoEShape("fd", T=12, d_model=8, d_latent=6, n_experts=6, top_k=2, n_dest=2,
                          hidden_routed=5, n_shared=1, hidden_shared=4, cap_recv=(60, 100), seed=0)


@pytest.fixture(scope="module")
def fd_case():
    s = FD_SHAPE
    rng = np.random.default_rng(21)
    w = {k: v.astype(np.float64) for k, v in synth.make_weights(s, rng).items()}
    w["w_router"] *= 4.0                                  # well-separated scores
    x = rng.standard_normal((s.T, s.d_model))
    dy = rng.standard_normal((s.T, s.d_model))
    bias = np.zeros(s.n_experts, np.float32)
    y, ctx = O.forward(x, w, bias, s, storage="f64")
    dx, grads, _ = O.backward(dy, w, ctx)
    return s, w, x, dy, bias, ctx, dx, grads


def test_fd_case_has_drops_and_margins(fd_case):
    s, w, x, dy, bias, ctx, dx, grads = fd_case
    sl = ctx["slots"]
    assert sl["dropped_receiver"] + sl["dropped_sender"] > 0
    sc = ctx["logits"].astype(np.float64)
    srt = -np.sort(-sc, axis=1)
    assert (srt[:, s.top_k - 1] - srt[:, s.top_k]).min() > 1e-3   # no near-tie at the cut


@pytest.mark.parametrize("name", ["x", "w_lat_down", "w_router", "w1", "w3", "w2",
                                  "w_lat_up", "ws1", "ws3", "ws2"])
def test_backward_matches_finite_differences(fd_case, name):
    s, w, x, dy, bias, ctx, dx, grads = fd_case
    eps = 1e-6
    base_idx = ctx["idx"]
    target = x if name == "x" else w[name]
    analytic = dx if name == "x" else grads[name]
    rng = np.random.default_rng(hash(name) % 2**32)
    flat = rng.choice(target.size, size=min(25, target.size), replace=False)
    for f in flat:
        pos = np.unravel_index(f, target.shape)
        old = target[pos]
        target[pos] = old + eps
        lp = _loss(x, w, bias, dy, s)
        _, cp = O.forward(x, w, bias, s, storage="f64")
        target[pos] = old - eps
        lm = _loss(x, w, bias, dy, s)
        _, cm = O.forward(x, w, bias, s, storage="f64")
        target[pos] = old
        assert np.array_equal(cp["idx"], base_idx) and np.array_equal(cm["idx"], base_idx)
        num = (lp - lm) / (2 * eps)
        assert abs(num - analytic[pos]) <= 1e-6 * (1 + abs(num)), (name, pos, num, analytic[pos])


def test_bias_gets_no_gradient(fd_case):
    """The bias only moves the selection: a change too small to flip any choice
    leaves the output exactly as it was."""
    s, w, x, dy, bias, ctx, dx, grads = fd_case
    y0, _ = O.forward(x, w, bias, s, storage="f64")
    y1, c1 = O.forward(x, w, bias + np.float32(1e-5), s, storage="f64")
    assert np.array_equal(c1["idx"], ctx["idx"])
    assert np.array_equal(y0, y1)


def test_expert_without_kept_rows_has_zero_weight_grad(fd_case):
    s, w, x, dy, bias, ctx, dx, grads = fd_case
    for e in range(s.n_experts):
        if ctx["slots"]["expert_kept"][e] == 0:
            assert not grads["w1"][e].any() and not grads["w2"][e].any() and not grads["w3"][e].any()
    # and experts with kept rows do get gradient
    assert any(grads["w1"][e].any() for e in range(s.n_experts))
