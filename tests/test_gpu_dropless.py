"""The dropless variant on the GPU (no cap binds; pools and expert buffers packed) against
the oracle's dropless variant: routing and slots bit-exact, every assignment kept,
outputs and gradients within the block's tolerances."""
import numpy as np
import pytest
import torch

from _helpers import (REL_TOL, ROUTED_GRAD_FRO, ROUTED_GRAD_TOL, assert_close_rms, assert_fro_close, bf16_dev,
                      dev, host64)
from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

RAGGED = synth.MoEShape("ragged", T=333, d_model=192, d_latent=128, n_experts=48, top_k=3, n_dest=8,
                        hidden_routed=256, n_shared=2, hidden_shared=128, seed=9)
SHAPES = [synth.TINY.with_(name="tiny_zipf", zipf_s=1.1, dropless=True),
          RAGGED.with_(dropless=True),
          synth.MID.with_(dropless=True)]


def _run(s):
    from capacity_limited_routed_b200.block import MoEBlock
    inp = synth.make_inputs(s)
    blk = MoEBlock(s, training=True)
    blk.load(inp)
    x = bf16_dev(inp["x"])
    y = blk.forward(x)
    dx = blk.backward(x, bf16_dev(inp["dy"]))
    torch.cuda.synchronize()
    return inp, blk, y, dx


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_dropless_block_matches_oracle(shape):
    s = shape.with_(backward=True)
    inp, blk, y, dx = _run(s)
    y_o, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, logit_offset=inp["logit_offset"])
    dx_o, grads_o, _ = O.backward(inp["dy"], inp["weights"], ctx)
    st = blk.stats_dict()
    A = s.T * s.top_k
    assert st["status"] == 0
    assert st["kept"] == A and st["dropped_sender"] == 0 and st["dropped_receiver"] == 0
    v = blk.saved_views()
    idx_g = v["topk_idx"].cpu().numpy()
    rows_g = v["expert_rows"].cpu().numpy()
    assert np.array_equal(rows_g, np.bincount(idx_g.ravel(), minlength=s.n_experts))
    assert np.array_equal(rows_g, st["hist"])
    match = (idx_g == ctx["idx"]).all(axis=1)
    print(f"\n[{s.name}] routing mismatch {1 - match.mean():.5f}; largest expert load {rows_g.max()} "
          f"(capped path would keep {O.geometry(s.with_(dropless=False)).C_r})")
    assert 1 - match.mean() <= 0.01
    if match.all():
        sl = ctx["slots"]
        assert np.array_equal(v["slot"][..., 0].cpu().numpy(), sl["sslot"])
        assert np.array_equal(v["slot"][..., 1].cpu().numpy(), sl["rslot"])
    assert_close_rms(host64(y)[match], y_o[match], what="y")
    assert_close_rms(host64(dx)[match], dx_o[match], what="dx")
    affected = set(np.unique(idx_g[~match]).tolist()) | set(np.unique(ctx["idx"][~match]).tolist())
    keep_e = np.array([e not in affected for e in range(s.n_experts)])
    for name in ("w1", "w3", "w2"):
        got, want = host64(blk.grads[name])[keep_e], grads_o[name][keep_e]
        assert_close_rms(got, want, tol=ROUTED_GRAD_TOL, what=f"d{name}")
        assert_fro_close(got, want, ROUTED_GRAD_FRO, what=f"d{name}")
    if match.all():
        for name in ("w_lat_down", "w_router", "w_lat_up", "ws1", "ws3", "ws2"):
            assert_close_rms(host64(blk.grads[name]), grads_o[name], what=f"d{name}")


@pytest.mark.slow
def test_dropless_skewed_full_size_keeps_everything():
    """T = 65,536 with the Zipf(1.1) skew at full width: the capped path drops most
    assignments; the dropless one keeps all of them, with exact per-expert counts, and
    its outputs agree with the oracle on sampled tokens."""
    from capacity_limited_routed_b200.block import MoEBlock
    s = synth.SKEWED_DROPLESS
    inp = synth.make_inputs_device(s, device=dev())
    blk = MoEBlock(s, device=dev(), training=True)  # keeps the forward context the views read
    blk.load(inp)
    y = blk.forward(inp["x"])
    torch.cuda.synchronize()
    st = blk.stats_dict()
    A = s.T * s.top_k
    assert st["status"] == 0 and st["kept"] == A
    assert st["dropped_sender"] == 0 and st["dropped_receiver"] == 0
    v = blk.saved_views()
    idx_g = v["topk_idx"].cpu().numpy()
    rows_g = v["expert_rows"].cpu().numpy()
    assert np.array_equal(rows_g, np.bincount(idx_g.ravel(), minlength=s.n_experts))
    # receiver slots of each expert are dense and unique
    rs = v["slot"][..., 1].cpu().numpy()
    order = np.argsort(idx_g.ravel(), kind="stable")
    e_sorted = idx_g.ravel()[order]
    r_sorted = rs.ravel()[order]
    starts = np.concatenate([[0], np.cumsum(rows_g)[:-1]])
    assert np.array_equal(r_sorted, np.arange(A) - np.repeat(starts, rows_g))
    print(f"\n[{s.name}] largest expert load {rows_g.max()} of {A} assignments")
    W = {n: inp["weights"][n].float().cpu().numpy() for n in ("w_lat_down", "w_router", "w_lat_up", "ws1", "ws3",
                                                               "ws2")}

    class _Lazy:
        def __init__(self, t):
            self.t = t

        def __getitem__(self, e):
            return self.t[e].float().cpu().numpy()
    for n in ("w1", "w3", "w2"):
        W[n] = _Lazy(inp["weights"][n])
    x_h = inp["x"].float().cpu().numpy()
    rb = O.route_batch(x_h, W, inp["bias"].cpu().numpy(), s, logit_offset=inp["logit_offset"].cpu().numpy())
    match = (idx_g == rb["idx"]).all(axis=1)
    print(f"[{s.name}] routing mismatch {1 - match.mean():.5f}")
    assert 1 - match.mean() <= 0.01
    toks = np.random.default_rng(8).choice(np.nonzero(match)[0], size=32, replace=False)
    ys, _ = O.forward_tokens(W, rb, toks)
    assert_close_rms(host64(y)[toks], ys, what="y (sampled)")
