"""The oracle's sampled evaluation (used at full width) equals its whole-batch one."""
import numpy as np
import pytest

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID.with_(T=1024, cap_recv=(90, 100))],
                         ids=["tiny", "mid1024_drops"])
def test_sampled_equals_whole_batch(shape):
    s = shape.with_(backward=True)
    inp = synth.make_inputs(s)
    y, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s)
    dx, grads, _ = O.backward(inp["dy"], inp["weights"], ctx)
    rb = O.route_batch(inp["x"], inp["weights"], inp["bias"], s)
    assert np.array_equal(rb["idx"], ctx["idx"]) and np.array_equal(rb["kept"], ctx["kept"])
    if "drops" in shape.name or shape.cap_recv[0] < 100:
        assert rb["slots"]["dropped_receiver"] > 0
    toks = np.random.default_rng(0).choice(s.T, size=12, replace=False)
    ys, per = O.forward_tokens(inp["weights"], rb, toks)
    np.testing.assert_allclose(ys, y[toks], rtol=1e-10, atol=1e-10)
    dxs = O.backward_tokens(inp["dy"][toks], inp["weights"], rb, toks, per)
    np.testing.assert_allclose(dxs, dx[toks], rtol=1e-9, atol=1e-9)
    for e in (0, s.n_experts // 2, s.n_experts - 1):
        gw = O.expert_weight_grads(inp["dy"], inp["weights"], rb, e)
        for n in ("w1", "w3", "w2"):
            np.testing.assert_allclose(gw[n], grads[n][e], rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID.with_(T=1024, cap_recv=(90, 100))],
                         ids=["tiny", "mid1024_drops"])
def test_sampled_weight_grads_equal_whole_batch_with_sparse_upstream_grad(shape):
    """Every weight gradient of the sampled evaluation equals the whole-batch backward
    run with the upstream gradient zeroed outside the sampled tokens."""
    s = shape.with_(backward=True)
    inp = synth.make_inputs(s)
    toks = np.sort(np.random.default_rng(1).choice(s.T, size=10, replace=False))
    dy = np.zeros_like(inp["dy"])
    dy[toks] = inp["dy"][toks]
    y, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s)
    dx, grads, _ = O.backward(dy, inp["weights"], ctx)
    rb = O.route_batch(inp["x"], inp["weights"], inp["bias"], s)
    ys, per = O.forward_tokens(inp["weights"], rb, toks)
    dense, routed = O.sampled_weight_grads(dy[toks], inp["weights"], rb, toks, per)
    for n, v in dense.items():
        np.testing.assert_allclose(v, grads[n], rtol=1e-9, atol=1e-9, err_msg=n)
    touched = set(int(e) for e in np.unique(ctx["idx"][toks][ctx["kept"][toks]]))
    assert set(routed) == touched
    for n in ("w1", "w3", "w2"):
        for e in range(s.n_experts):
            want = grads[n][e]
            if e in routed:
                np.testing.assert_allclose(routed[e][n], want, rtol=1e-9, atol=1e-9, err_msg=f"{n}[{e}]")
            else:
                assert not np.any(want), f"{n}[{e}] should be zero"


def test_shared_weight_grad_rows_equal_whole_batch():
    """The shared experts' gradients restricted to a few hidden units equal those rows
    (and columns) of the whole-batch backward."""
    s = synth.TINY.with_(backward=True, n_shared=2)
    inp = synth.make_inputs(s)
    y, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s)
    dx, grads, _ = O.backward(inp["dy"], inp["weights"], ctx)
    units = np.array([0, 5, s.hidden_shared - 1, s.hidden_shared, 2 * s.hidden_shared - 1])
    g1, g3, g2 = O.shared_weight_grad_rows(inp["x"], inp["dy"], inp["weights"], units)
    np.testing.assert_allclose(g1, grads["ws1"][units], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(g3, grads["ws3"][units], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(g2, grads["ws2"][:, units], rtol=1e-9, atol=1e-9)
