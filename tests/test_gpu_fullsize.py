"""Parity at full width, in the launch configuration the benchmark times.

Inputs come from the benchmark's own seeded generator (drawn on the device by
PyTorch's RNG).  Checks:
  * routing and slot assignment bit-exact against the oracle on the same float32
    logits, at T = 16,384 and 65,536 with 384 experts (plain and Zipf-skewed);
  * properties that hold at any size on the whole block's own routing: counters add
    up, no pool or expert exceeds its capacity, slots are dense and unique;
  * y (and dx, and the gradients of two experts) on sampled tokens against the
    oracle, whose routing and drops are computed over the whole batch; every token
    routed differently must be a near tie, and the routing mismatch rate is reported;
  * the training step's weight gradients: the shared experts' (which do not depend on
    routing) on sampled hidden units over all 16,384 tokens, and every weight gradient
    in full from a second backward pass whose upstream gradient is zero except on a
    sample of tokens both sides route alike.
"""
import numpy as np
import pytest
import torch

from _helpers import (REL_TOL, ROUTED_GRAD_FRO, ROUTED_GRAD_TOL, assert_close_rms, assert_fro_close, dev,
                      f32_dev, host64, i32_dev, routing_mismatch_check)
from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def M():
    from capacity_limited_routed_b200 import moe
    return moe


# ------------------------------------------------------------------ routing and slots, bit-exact


@pytest.mark.parametrize("shape", [synth.FULL, synth.SKEWED], ids=["full", "skewed"])
def test_route_and_dispatch_bit_exact_full_size(M, shape):
    s = shape
    g = O.geometry(s)
    plan = M.Plan.from_shape(s)
    logits = synth.make_logits(s.T, s.n_experts, seed=s.seed + 100)
    off = synth.make_logit_offset(s)
    if off is not None:
        logits = (logits + off[None, :]).astype(np.float32)
    bias = (np.random.default_rng(5).standard_normal(s.n_experts) * 1e-2).astype(np.float32)
    idx_o, gate_o, hist_o = O.route(logits, bias, s.top_k)
    idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device=dev())
    gate = torch.empty((s.T, s.top_k), dtype=torch.float32, device=dev())
    hist = torch.empty((s.n_experts,), dtype=torch.int32, device=dev())
    M.moe_route(plan, f32_dev(logits), f32_dev(bias), idx, gate, hist)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.array_equal(hist.cpu().numpy(), hist_o)
    np.testing.assert_allclose(gate.cpu().numpy(), gate_o, rtol=2e-6, atol=1e-7)
    slots = O.assign_slots(idx_o, g)
    info = plan.info
    gen = torch.Generator(device=dev()).manual_seed(11)
    z = torch.randn((s.T, s.d_latent), generator=gen, device=dev()).to(torch.bfloat16)
    pools = torch.empty(info.pools_bytes // 2, dtype=torch.int16, device=dev())
    slot = torch.empty((s.T, s.top_k, 2), dtype=torch.int32, device=dev())
    stats = torch.zeros(info.stats_bytes // 4, dtype=torch.int32, device=dev())
    ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=dev())
    M.moe_dispatch(plan, z, i32_dev(idx_o), pools, slot, stats, ws)
    sl = slot.cpu().numpy()
    assert np.array_equal(sl[..., 0], slots["sslot"]) and np.array_equal(sl[..., 1], slots["rslot"])
    st = stats.cpu().numpy()
    assert (st[0], st[1], st[2], st[3]) == (slots["kept"], slots["dropped_sender"], slots["dropped_receiver"], 0)
    E = s.n_experts
    assert np.array_equal(st[8 + E:8 + 4 * E], np.concatenate(
        [slots["expert_kept"], slots["expert_dropped_sender"], slots["expert_dropped_receiver"]]))
    # pool rows of sampled kept assignments hold the token's latent row bit for bit, and
    # their headers the packed expert id
    pl = O.placement(g)
    rows = pools[: g.n_pools * g.C_s * (s.d_latent + 8)].view(g.n_pools, g.C_s, s.d_latent + 8)
    t_all, j_all = np.nonzero(slots["sslot"] >= 0)
    pick = np.random.default_rng(6).choice(t_all.size, size=min(512, t_all.size), replace=False)
    t_s, j_s = t_all[pick], j_all[pick]
    e_s = idx_o[t_s, j_s]
    got = rows[torch.from_numpy(pl["pool"][e_s]).to(dev()), torch.from_numpy(slots["sslot"][t_s, j_s]).to(dev())]
    assert torch.equal(got[:, : s.d_latent], z.view(torch.int16)[torch.from_numpy(t_s).to(dev())])
    hdr = got[:, s.d_latent:].cpu().numpy().copy().view(np.int32)[:, 0]
    assert np.array_equal(hdr, e_s)
    print(f"\n[{s.name}] drops: sender {slots['dropped_sender']}, receiver {slots['dropped_receiver']} "
          f"of {s.T * s.top_k}")


# ------------------------------------------------------------------ whole block on sampled tokens


class _LazyExperts:
    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].cpu().float().numpy()  # bf16 over the bus, widened on the host


def _host_weights(w):
    out = {n: w[n].float().cpu().numpy() for n in ("w_lat_down", "w_router", "w_lat_up", "ws1", "ws3", "ws2")}
    for n in ("w1", "w3", "w2"):
        out[n] = _LazyExperts(w[n])
    return out


def _slot_properties(s, g, idx, slot, st):
    """Whatever the routing, the slot map of the block must be a valid capacity-limited
    assignment of it: dense unique slots, caps respected, counters adding up."""
    E = s.n_experts
    T, k = idx.shape
    assert st["kept"] + st["dropped_sender"] + st["dropped_receiver"] == T * k
    assert int(st["hist"].sum()) == T * k and st["status"] == 0
    assert st["max_pool_fill"] <= g.C_s and st["max_expert_fill"] <= g.C_r
    pool = O.placement(g)["pool"][idx]
    ss, rs = slot[..., 0], slot[..., 1]
    for p in range(g.n_pools):
        v = np.sort(ss[(pool == p) & (ss >= 0)])
        assert np.array_equal(v, np.arange(v.size))
    for e in range(E):
        v = np.sort(rs[(idx == e) & (rs >= 0)])
        assert np.array_equal(v, np.arange(v.size))
        assert v.size == st["expert_kept"][e]
    assert not np.any((rs >= 0) & (ss < 0))


@pytest.mark.parametrize("wid", [3, 4, 5], ids=["full", "skewed", "train"])
def test_block_full_size_sampled(wid):
    from capacity_limited_routed_b200.block import MoEBlock
    s = synth.WORKLOADS[wid]
    g = O.geometry(s)
    inp = synth.make_inputs_device(s, device=dev())
    blk = MoEBlock(s, device=dev(), training=True)
    blk.load(inp)
    y = blk.forward(inp["x"])
    dx = blk.backward(inp["x"], inp["dy"]) if s.backward else None
    torch.cuda.synchronize()
    st = blk.stats_dict()
    v = blk.saved_views()
    idx_g = v["topk_idx"].cpu().numpy()
    slot_g = v["slot"].cpu().numpy()
    _slot_properties(s, g, idx_g, slot_g, st)
    A = s.T * s.top_k
    print(f"\n[{s.name}] drop fraction sender {st['dropped_sender'] / A:.4f} receiver "
          f"{st['dropped_receiver'] / A:.4f}")

    W = _host_weights(inp["weights"])
    x_h = inp["x"].float().cpu().numpy()
    off = None if inp["logit_offset"] is None else inp["logit_offset"].cpu().numpy()
    rb = O.route_batch(x_h, W, inp["bias"].cpu().numpy(), s, logit_offset=off)
    match = (idx_g == rb["idx"]).all(axis=1) & ((slot_g[..., 1] >= 0) == rb["kept"]).all(axis=1)
    rate, near = routing_mismatch_check(v["logits"].cpu().numpy(), rb["logits"], inp["bias"].cpu().numpy(),
                                        idx_g, rb["idx"], match, s.top_k, s.name)
    print(f"[{s.name}] routing mismatch rate {rate:.5f} ({(~match).sum()} of {s.T}; {near} near ties)")
    sl = rb["slots"]
    # drop counts of the two routings differ at most by what the mismatched tokens move
    assert abs(st["dropped_sender"] + st["dropped_receiver"] - sl["dropped_sender"] - sl["dropped_receiver"]) \
        <= s.top_k * (~match).sum() + 1
    rng = np.random.default_rng(wid)
    toks = rng.choice(np.nonzero(match)[0], size=48, replace=False)
    ys, per = O.forward_tokens(W, rb, toks)
    e_y = assert_close_rms(host64(y)[toks], ys, what="y (sampled)")
    print(f"[{s.name}] y: max-abs / rms {e_y:.4f} on {toks.size} tokens")
    if s.backward:
        dy_h = inp["dy"].float().cpu().numpy()
        dxs = O.backward_tokens(dy_h[toks], W, rb, toks, per)
        e_dx = assert_close_rms(host64(dx)[toks], dxs, what="dx (sampled)")
        print(f"[{s.name}] dx: max-abs / rms {e_dx:.4f}")
        touched = set(np.unique(idx_g[~match]).tolist()) | set(np.unique(rb["idx"][~match]).tolist())
        clean = [e for e in range(s.n_experts) if e not in touched]
        for e in (clean[0], clean[len(clean) // 2]):
            gw = O.expert_weight_grads(dy_h, W, rb, e)
            for n in ("w1", "w3", "w2"):
                got = host64(blk.grads[n][e])
                er = assert_close_rms(got, gw[n], tol=ROUTED_GRAD_TOL, what=f"d{n}[{e}]")
                fr = assert_fro_close(got, gw[n], ROUTED_GRAD_FRO, what=f"d{n}[{e}]")
                print(f"[{s.name}] d{n}[{e}]: max-abs / rms {er:.4f}, frobenius {fr:.2e}")
        # shared experts: routing plays no part, so sampled hidden units are checked over
        # every token of the full upstream gradient
        SH = s.n_shared * s.hidden_shared
        units = np.sort(rng.choice(SH, size=6, replace=False))
        g1, g3, g2 = O.shared_weight_grad_rows(x_h, dy_h, W, units)
        for n, got, want in (("ws1", blk.grads["ws1"][units], g1), ("ws3", blk.grads["ws3"][units], g3),
                             ("ws2", blk.grads["ws2"][:, units], g2)):
            er = assert_close_rms(host64(got), want, what=f"d{n} (units {units.tolist()}, all tokens)")
            print(f"[{s.name}] d{n}: max-abs / rms {er:.4f} on {units.size} hidden units")
        _sparse_upstream_backward(s, blk, inp, W, rb, match, dy_h, rng)


def _sparse_upstream_backward(s, blk, inp, W, rb, match, dy_h, rng):
    """Backward again with the upstream gradient zero except on sampled tokens that both
    sides route alike: the weight-gradient GEMMs still contract over all T tokens, and
    every gradient is now a sum the oracle can form from the sampled tokens alone."""
    toks = np.sort(rng.choice(np.nonzero(match)[0], size=32, replace=False))
    dy_s = torch.zeros_like(inp["dy"])
    sel = torch.from_numpy(toks).to(dev())
    dy_s[sel] = inp["dy"][sel]
    blk.backward(inp["x"], dy_s)
    torch.cuda.synchronize()
    assert blk.stats_dict()["status"] == 0
    _, per = O.forward_tokens(W, rb, toks)
    dense, routed = O.sampled_weight_grads(dy_h[toks], W, rb, toks, per)
    # each gradient is now a sum of 32 token terms of bf16-stored factors: held to the
    # bars of few-term sums (tests/test_oracle_precision.py::test_sparse_upstream_spread)
    for n, want in dense.items():
        got = host64(blk.grads[n])
        er = assert_close_rms(got, want, tol=ROUTED_GRAD_TOL, what=f"d{n} (sparse upstream)")
        fr = assert_fro_close(got, want, ROUTED_GRAD_FRO, what=f"d{n} (sparse upstream)")
        print(f"[{s.name}] d{n}: max-abs / rms {er:.4f}, frobenius {fr:.2e} ({toks.size} tokens, K = {s.T})")
    touched = np.zeros(s.n_experts, dtype=bool)
    touched[list(routed)] = True
    mask = torch.from_numpy(~touched).to(dev())
    for n in ("w1", "w3", "w2"):
        assert float(blk.grads[n][mask].abs().max().item()) == 0.0, f"d{n} of untouched experts"
    pick = sorted(rng.choice(sorted(routed), size=min(8, len(routed)), replace=False).tolist())
    for n in ("w1", "w3", "w2"):
        got = np.concatenate([host64(blk.grads[n][e]).ravel() for e in pick])
        want = np.concatenate([routed[e][n].ravel() for e in pick])
        er = assert_close_rms(got, want, tol=0.5, what=f"d{n} (sparse upstream, experts {pick})")
        fr = assert_fro_close(got, want, ROUTED_GRAD_FRO, what=f"d{n} (sparse upstream)")
        print(f"[{s.name}] d{n}: max-abs / rms {er:.4f}, frobenius {fr:.2e} on {len(pick)} of "
              f"{int(touched.sum())} touched experts")
