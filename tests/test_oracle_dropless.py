"""Pins of the oracle's dropless variant: the capacity-limited assignment with no cap
binding ([ZH] §3.3 and §7 of the Marin 535B pages: the run later switched to a dropless
ragged all-to-all)."""
import numpy as np

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

SMALL = synth.MoEShape("small", T=160, d_model=64, d_latent=32, n_experts=12, top_k=3, n_dest=2,
                       hidden_routed=48, n_shared=1, hidden_shared=32, seed=31)


def _skewed(shape):
    """A router skew that overloads the low-index experts, so the capped path drops."""
    off = (-2.0 * np.log1p(np.arange(shape.n_experts))).astype(np.float32)
    return off


def test_dropless_keeps_every_assignment_and_counts_exactly():
    s = SMALL.with_(dropless=True)
    inp = synth.make_inputs(s)
    _, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, logit_offset=_skewed(s))
    sl = ctx["slots"]
    assert sl["kept"] == s.T * s.top_k and sl["dropped_sender"] == 0 and sl["dropped_receiver"] == 0
    # exact per-expert counts: the kept rows of each expert are its whole load
    assert np.array_equal(sl["expert_kept"], np.bincount(ctx["idx"].ravel(), minlength=s.n_experts))
    assert np.array_equal(sl["expert_kept"], ctx["hist"])
    # receiver slots of each expert are 0..n_e-1 in (token, rank) order
    for e in range(s.n_experts):
        t, j = np.nonzero(ctx["idx"] == e)
        assert np.array_equal(sl["rslot"][t, j], np.arange(t.size))


def test_dropless_equals_capped_path_whose_caps_never_bind():
    """With capacity factors so large that no rank reaches them, the capped path is the
    dropless one: same routing, same slots, the same outputs bit for bit."""
    s = SMALL.with_(backward=True)
    inp = synth.make_inputs(s)
    big = s.with_(cap_send=(110 * 50, 100), cap_recv=(115 * 50, 100))
    y_c, ctx_c = O.forward(inp["x"], inp["weights"], inp["bias"], big, logit_offset=_skewed(s))
    y_d, ctx_d = O.forward(inp["x"], inp["weights"], inp["bias"], s.with_(dropless=True),
                           logit_offset=_skewed(s))
    assert ctx_c["slots"]["kept"] == s.T * s.top_k
    assert np.array_equal(ctx_c["slots"]["rslot"], ctx_d["slots"]["rslot"])
    assert np.array_equal(y_c, y_d)
    dx_c, g_c, _ = O.backward(inp["dy"], inp["weights"], ctx_c)
    dx_d, g_d, _ = O.backward(inp["dy"], inp["weights"], ctx_d)
    assert np.array_equal(dx_c, dx_d)
    for n in g_c:
        assert np.array_equal(g_c[n], g_d[n]), n


def test_dropless_changes_only_tokens_the_caps_touched():
    """A token's output depends on its own routing and kept set alone: where the
    capped path kept all of a token's assignments, the two variants agree on it."""
    s = SMALL.with_(backward=True)
    inp = synth.make_inputs(s)
    y_c, ctx_c = O.forward(inp["x"], inp["weights"], inp["bias"], s, logit_offset=_skewed(s))
    y_d, _ = O.forward(inp["x"], inp["weights"], inp["bias"], s.with_(dropless=True), logit_offset=_skewed(s))
    dropped = ctx_c["slots"]["dropped_sender"] + ctx_c["slots"]["dropped_receiver"]
    assert dropped > 0
    full = ctx_c["kept"].all(axis=1)
    assert 0 < full.sum() < s.T
    assert np.array_equal(y_c[full], y_d[full])
    assert not np.allclose(y_c[~full], y_d[~full])
