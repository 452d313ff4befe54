"""Whole forward and backward pass through moe_forward / moe_backward against the oracle.

The GPU computes its own router logits, so a token whose float32 scores nearly tie
can be routed differently from the oracle (float64 accumulation).  Every token routed
differently must be such a near tie, and the rate of routing mismatches is reported;
outputs are compared on the tokens whose chosen experts and drop decisions agree.
For the backward the upstream gradient of the mismatched tokens is set to zero on
both sides: every gradient is then a sum over tokens that both sides route alike,
so dx and every weight gradient (dense and routed, all experts) are compared in full.
"""
import numpy as np
import pytest
import torch

from _helpers import (REL_TOL, ROUTED_GRAD_FRO, ROUTED_GRAD_TOL, assert_bf16_close, assert_close_rms,
                      assert_fro_close, bf16_dev, dev, host64, routing_mismatch_check)
from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

RAGGED = synth.MoEShape("ragged", T=333, d_model=192, d_latent=128, n_experts=48, top_k=3, n_dest=8,
                        hidden_routed=256, n_shared=2, hidden_shared=128, seed=9)
# more choices per token than the combine kernels batch per pass (8), and a single one
WIDE_K = synth.MoEShape("wide_k", T=200, d_model=192, d_latent=128, n_experts=48, top_k=12, n_dest=8,
                        hidden_routed=256, n_shared=1, hidden_shared=128, seed=13)
TOP1 = synth.MoEShape("top1", T=300, d_model=192, d_latent=128, n_experts=24, top_k=1, n_dest=4,
                      hidden_routed=128, n_shared=1, hidden_shared=128, seed=14)


def _run(shape, backward):
    from capacity_limited_routed_b200.block import MoEBlock
    s = shape.with_(backward=backward)
    inp = synth.make_inputs(s)
    blk = MoEBlock(s, training=True)
    blk.load(inp)
    x = bf16_dev(inp["x"])
    y = blk.forward(x)
    out = {"s": s, "inp": inp, "blk": blk, "x": x, "y": y}
    if backward:
        out["dx"] = blk.backward(x, bf16_dev(inp["dy"]))
    torch.cuda.synchronize()
    return out


def _routing_agreement(views, ctx):
    idx_g = views["topk_idx"].cpu().numpy()
    kept_g = views["slot"][..., 1].cpu().numpy() >= 0
    match = (idx_g == ctx["idx"]).all(axis=1) & (kept_g == ctx["kept"]).all(axis=1)
    affected = set(np.unique(idx_g[~match]).tolist()) | set(np.unique(ctx["idx"][~match]).tolist())
    return match, affected


@pytest.mark.parametrize("shape", [synth.TINY, RAGGED, WIDE_K, TOP1, synth.MID], ids=lambda s: s.name)
def test_forward_matches_oracle(shape):
    r = _run(shape, backward=False)
    s, inp, blk = r["s"], r["inp"], r["blk"]
    y_o, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, logit_offset=inp["logit_offset"])
    st = blk.stats_dict()
    assert st["status"] == 0 and st["nan_logits"] == 0
    v = blk.saved_views()
    assert_bf16_close(host64(v["z"]), ctx["z"], what="z")
    assert_close_rms(host64(v["logits"]), ctx["logits"], tol=1e-2, what="logits")
    match, _ = _routing_agreement(v, ctx)
    rate, near = routing_mismatch_check(v["logits"].cpu().numpy(), ctx["logits"], inp["bias"],
                                        v["topk_idx"].cpu().numpy(), ctx["idx"], match, s.top_k, s.name)
    print(f"\n[{s.name}] routing mismatch rate {rate:.5f} ({(~match).sum()} of {s.T} tokens; "
          f"{near} near ties)")
    assert_close_rms(host64(r["y"])[match], y_o[match], what="y")
    if match.all():
        sl = ctx["slots"]
        assert (st["kept"], st["dropped_sender"], st["dropped_receiver"]) == (
            sl["kept"], sl["dropped_sender"], sl["dropped_receiver"])
        assert np.array_equal(st["hist"], ctx["hist"])
        assert np.array_equal(v["slot"][..., 0].cpu().numpy(), sl["sslot"])
        assert np.array_equal(v["slot"][..., 1].cpu().numpy(), sl["rslot"])
        assert np.array_equal(v["expert_rows"].cpu().numpy(), sl["expert_kept"])


@pytest.mark.parametrize("shape", [synth.TINY, RAGGED, WIDE_K, TOP1, synth.MID], ids=lambda s: s.name)
def test_backward_matches_oracle(shape):
    r = _run(shape, backward=True)
    s, inp, blk, x = r["s"], r["inp"], r["blk"], r["x"]
    y_o, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, logit_offset=inp["logit_offset"])
    v = blk.saved_views()
    match, _ = _routing_agreement(v, ctx)
    rate, near = routing_mismatch_check(v["logits"].cpu().numpy(), ctx["logits"], inp["bias"],
                                        v["topk_idx"].cpu().numpy(), ctx["idx"], match, s.top_k, s.name)
    print(f"\n[{s.name}] routing mismatch rate {rate:.5f}; upstream gradient zeroed on {(~match).sum()} tokens")
    # the mismatched tokens contribute nothing on either side
    dy = np.where(match[:, None], inp["dy"], 0.0).astype(np.float32)
    dx = blk.backward(x, bf16_dev(dy))
    torch.cuda.synchronize()
    dx_o, grads_o, _ = O.backward(dy, inp["weights"], ctx)
    e_dx = assert_close_rms(host64(dx), dx_o, what="dx")
    print(f"  dx: max-abs/rms {e_dx:.4f}")
    for name in ("w1", "w3", "w2"):
        got, want = host64(blk.grads[name]), grads_o[name]
        e = assert_close_rms(got, want, tol=ROUTED_GRAD_TOL, what=f"d{name}")
        f = assert_fro_close(got, want, ROUTED_GRAD_FRO, what=f"d{name}")
        print(f"  d{name}: max-abs/rms {e:.4f}, frobenius {f:.2e}")
    for name in ("w_router", "w_lat_down", "w_lat_up", "ws1", "ws3", "ws2"):
        e = assert_close_rms(host64(blk.grads[name]), grads_o[name], what=f"d{name}")
        print(f"  d{name}: max-abs/rms {e:.4f}")
    assert blk.stats_dict()["status"] == 0


def test_bias_step_after_forward_matches_oracle():
    r = _run(synth.TINY, backward=False)
    s, inp, blk = r["s"], r["inp"], r["blk"]
    hist = blk.stats_dict()["hist"]
    want = O.bias_update(hist, inp["bias"], 1e-3, s.T, s.top_k)
    blk.bias_update(1e-3)
    got = blk.bias.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert abs(float(got.astype(np.float64).sum())) < 1e-7


def test_empty_batch_is_a_no_op():
    from capacity_limited_routed_b200.block import MoEBlock
    s = synth.TINY.with_(T=0)
    blk = MoEBlock(s, training=True)
    blk.load(synth.make_inputs(synth.TINY.with_(backward=True)))
    x = torch.empty((0, s.d_model), dtype=torch.bfloat16, device=dev())
    y = blk.forward(x)
    dx = blk.backward(x, x)
    torch.cuda.synchronize()
    assert y.shape == (0, s.d_model) and dx.shape == (0, s.d_model)
    assert all(int(g.abs().max().item()) == 0 for g in blk.grads.values())
    assert blk.stats_dict()["kept"] == 0


def test_backward_idle_experts_get_zero_gradients():
    """A batch too small to reach every expert: the weight gradients of experts that
    received no rows must come out exactly zero (the contraction over their rows is empty),
    whatever the gradient buffers held before."""
    s = RAGGED.with_(T=12, backward=True, seed=21)
    inp = synth.make_inputs(s)
    from capacity_limited_routed_b200.block import MoEBlock
    blk = MoEBlock(s, training=True)
    blk.load(inp)
    x = bf16_dev(inp["x"])
    blk.forward(x)
    for t in blk.grads.values():
        t.fill_(float("nan"))
    blk.backward(x, bf16_dev(inp["dy"]))
    torch.cuda.synchronize()
    rows = blk.saved_views()["expert_rows"].cpu().numpy()
    idle = rows == 0
    assert idle.sum() >= s.n_experts // 2
    y_o, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], s, logit_offset=inp["logit_offset"])
    _, grads_o, _ = O.backward(inp["dy"], inp["weights"], ctx)
    _, affected = _routing_agreement(blk.saved_views(), ctx)
    for name in ("w1", "w3", "w2"):
        got = host64(blk.grads[name])
        assert np.all(got[idle] == 0.0), name
        assert np.isfinite(got).all(), name
        busy = ~idle & np.array([e not in affected for e in range(s.n_experts)])
        assert_close_rms(got[busy], grads_o[name][busy], tol=ROUTED_GRAD_TOL, what=f"d{name}")


def test_side_stream_off_gives_identical_results():
    """moe_set_side_stream(0) runs the shared experts in order on the caller's stream; the
    outputs, dx, every gradient and the statistics must be bit for bit those of the default
    (shared experts on the second stream)."""
    from capacity_limited_routed_b200 import moe as M
    runs = []
    try:
        for on in (True, False):
            M.moe_set_side_stream(on)
            r = _run(synth.MID.with_(T=2048, seed=33), backward=True)
            runs.append((r["y"].clone(), r["dx"].clone(), {n: g.clone() for n, g in r["blk"].grads.items()},
                         r["blk"].stats.clone()))
    finally:
        M.moe_set_side_stream(True)
    (y0, dx0, g0, st0), (y1, dx1, g1, st1) = runs
    assert torch.equal(y0, y1) and torch.equal(dx0, dx1) and torch.equal(st0, st1)
    for n in g0:
        assert torch.equal(g0[n], g1[n]), n
