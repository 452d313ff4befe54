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
