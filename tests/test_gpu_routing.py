"""Routing, slot assignment, pooled transport, experts and combine through the C ABI,
each against the oracle on the same inputs.  Integer results (top-k indices, slots,
drop decisions, counters, pool headers, copied rows) must match bit for bit."""
import numpy as np
import pytest
import torch

from _helpers import REL_TOL, assert_bf16_close, assert_close_rms, bf16_dev, dev, f32_dev, host64, i32_dev
from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from capacity_limited_routed_b200 import moe
    return moe


def _plan(M, s):
    return M.Plan.from_shape(s)


# ------------------------------------------------------------------ router


@pytest.mark.parametrize("E,k,ties", [(24, 2, False), (96, 8, True), (384, 8, False), (384, 8, True),
                                      (1024, 32, True)])
def test_route_bit_exact(M, E, k, ties):
    T = 1000
    s = synth.TINY.with_(T=T, n_experts=E, top_k=k, n_dest=E // 6 if E % 6 == 0 else 4)
    if E == 1024:
        s = s.with_(n_dest=1024 // 32 // 1, n_waves=1)
    plan = _plan(M, s)
    logits = synth.make_logits(T, E, seed=E + k, ties=ties)
    bias = (np.random.default_rng(E).integers(-4, 5, size=E) / 8.0).astype(np.float32)
    idx_o, gate_o, hist_o = O.route(logits, bias, k)
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev())
    gate = torch.zeros((T, k), dtype=torch.float32, device=dev())
    hist = torch.full((E,), 99, dtype=torch.int32, device=dev())
    M.moe_route(plan, f32_dev(logits), f32_dev(bias), idx, gate, hist)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.array_equal(hist.cpu().numpy(), hist_o)
    np.testing.assert_allclose(gate.cpu().numpy(), gate_o, rtol=2e-6, atol=1e-7)


def test_route_signed_zero_and_empty(M):
    s = synth.TINY
    plan = _plan(M, s)
    logits = np.zeros((s.T, s.n_experts), np.float32)
    logits[::2] = -0.0
    bias = np.zeros(s.n_experts, np.float32)
    idx = torch.zeros((s.T, s.top_k), dtype=torch.int32, device=dev())
    gate = torch.zeros((s.T, s.top_k), dtype=torch.float32, device=dev())
    hist = torch.zeros((s.n_experts,), dtype=torch.int32, device=dev())
    M.moe_route(plan, f32_dev(logits), f32_dev(bias), idx, gate, hist)
    assert (idx.cpu().numpy() == np.arange(s.top_k)[None, :]).all()
    assert np.allclose(gate.cpu().numpy(), 1.0 / s.top_k)


@pytest.mark.parametrize("shape", [
    synth.TINY,
    synth.MoEShape("e48k3", T=333, d_model=192, d_latent=128, n_experts=48, top_k=3, n_dest=8,
                   hidden_routed=128, n_shared=1, hidden_shared=128, seed=41),
    synth.MoEShape("e48k12", T=200, d_model=192, d_latent=128, n_experts=48, top_k=12, n_dest=8,
                   hidden_routed=128, n_shared=1, hidden_shared=128, seed=42),
    synth.MoEShape("e96k20", T=130, d_model=192, d_latent=192, n_experts=96, top_k=20, n_dest=8,
                   hidden_routed=128, n_shared=1, hidden_shared=128, seed=43),
    synth.MoEShape("e384k8", T=300, d_model=256, d_latent=256, n_experts=384, top_k=8, n_dest=64,
                   hidden_routed=128, n_shared=1, hidden_shared=128, seed=44),
], ids=lambda s: s.name)
def test_forward_topk_matches_moe_route(M, shape):
    """The forward's topk_idx and topk_gate must be bit for bit what moe_route makes of the
    logits and bias the forward saved (T not a multiple of 128, k up to 20, E up to 384)."""
    from capacity_limited_routed_b200.block import MoEBlock
    inp = synth.make_inputs(shape)
    blk = MoEBlock(shape, training=True)
    blk.load(inp)
    blk.forward(bf16_dev(inp["x"]))
    torch.cuda.synchronize()
    v = blk.saved_views()
    T, k, E = shape.T, shape.top_k, shape.n_experts
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev())
    gate = torch.zeros((T, k), dtype=torch.float32, device=dev())
    hist = torch.zeros((E,), dtype=torch.int32, device=dev())
    M.moe_route(blk.plan, v["logits"], blk.bias, idx, gate, hist)
    torch.cuda.synchronize()
    assert torch.equal(v["topk_idx"], idx)
    assert torch.equal(v["topk_gate"], gate)
    assert int(blk.stats_dict()["nan_logits"]) == 0


# ------------------------------------------------------------------ dispatch


def _skewed_idx(T, E, k, seed, skew):
    logits = synth.make_logits(T, E, seed)
    logits = logits - np.float32(skew) * np.log1p(np.arange(E, dtype=np.float32))[None, :]
    return O.route(logits, np.zeros(E, np.float32), k)


@pytest.mark.parametrize("shape,skew", [(synth.TINY, 0.0), (synth.TINY, 1.5), (synth.MID, 0.3),
                                        (synth.TINY.with_(T=777, top_k=5), 0.8),
                                        # the largest top-k a plan accepts: 32 pool rows per token
                                        (synth.MoEShape("e96k32", T=333, d_model=192, d_latent=128,
                                                        n_experts=96, top_k=32, n_dest=8, hidden_routed=128,
                                                        n_shared=1, hidden_shared=128, seed=45), 0.5)],
                         ids=["tiny", "tiny_skew", "mid", "ragged_k5", "e96k32"])
def test_dispatch_bit_exact(M, shape, skew):
    s = shape
    g = O.geometry(s)
    plan = _plan(M, s)
    idx_o, _, _ = _skewed_idx(s.T, s.n_experts, s.top_k, 3, skew)
    slots = O.assign_slots(idx_o, g)
    rng = np.random.default_rng(4)
    z = synth._bf16(rng.standard_normal((s.T, s.d_latent), dtype=np.float32))
    payload, header = O.pack_pools(z, idx_o, slots["sslot"], g)
    info = plan.info
    pools = torch.full((info.pools_bytes // 2,), 0x7FC0, dtype=torch.int16, device=dev()).view(torch.bfloat16)
    slot = torch.full((s.T, s.top_k, 2), -5, dtype=torch.int32, device=dev())
    stats = torch.full((info.stats_bytes // 4,), 77, dtype=torch.int32, device=dev())
    stats[3] = 0
    ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=dev())
    M.moe_dispatch(plan, bf16_dev(z), i32_dev(idx_o), pools, slot, stats, ws)
    torch.cuda.synchronize()
    sl = slot.cpu().numpy()
    assert np.array_equal(sl[..., 0], slots["sslot"])
    assert np.array_equal(sl[..., 1], slots["rslot"])
    st = stats.cpu().numpy()
    E, NP = s.n_experts, g.n_pools
    assert (st[0], st[1], st[2], st[3]) == (slots["kept"], slots["dropped_sender"], slots["dropped_receiver"], 0)
    assert st[6] == s.T * s.top_k
    assert np.array_equal(st[8 + E:8 + 2 * E], slots["expert_kept"])
    assert np.array_equal(st[8 + 2 * E:8 + 3 * E], slots["expert_dropped_sender"])
    assert np.array_equal(st[8 + 3 * E:8 + 4 * E], slots["expert_dropped_receiver"])
    assert np.array_equal(st[8 + 4 * E:8 + 4 * E + NP], slots["pool_fill"])
    assert st[4] == slots["pool_fill"].max() and st[5] == slots["expert_kept"].max()
    # pools: packed ids in the header, rows copied bit for bit
    rows = pools.view(torch.int16).cpu().numpy().reshape(NP, g.C_s, s.d_latent + 8)
    hdr = rows[:, :, s.d_latent:].copy().view(np.int32)[:, :, 0]
    assert np.array_equal(hdr, header)
    got = rows[:, :, : s.d_latent].view(np.uint16)
    want = synth.to_bf16_bits(payload.astype(np.float32))
    filled = header >= 0
    assert np.array_equal(got[filled], want[filled])
    if skew:
        assert slots["dropped_sender"] + slots["dropped_receiver"] > 0


# ------------------------------------------------------------------ experts and combine


def _pools_device(plan, s, g, payload, header):
    """The oracle's pools in the device layout."""
    rows = np.zeros((g.n_pools, g.C_s, s.d_latent + 8), dtype=np.uint16)
    rows[:, :, : s.d_latent] = synth.to_bf16_bits(payload.astype(np.float32))
    hdr = np.zeros((g.n_pools, g.C_s, 4), dtype=np.int32)
    hdr[:, :, 0] = header
    rows[:, :, s.d_latent:] = hdr.view(np.uint16)
    assert rows.nbytes == plan.info.pools_bytes
    return torch.from_numpy(rows.view(np.int16)).to(dev()).view(torch.bfloat16)


@pytest.mark.parametrize("shape,skew", [(synth.TINY, 1.0), (synth.MID, 0.5)])
def test_expert_ffn_and_combine(M, shape, skew):
    s = shape
    g = O.geometry(s)
    plan = _plan(M, s)
    inp = synth.make_inputs(s, seed=11)
    w = inp["weights"]
    idx_o, gate_o, _ = _skewed_idx(s.T, s.n_experts, s.top_k, 5, skew)
    slots = O.assign_slots(idx_o, g)
    rng = np.random.default_rng(6)
    z = synth._bf16(rng.standard_normal((s.T, s.d_latent), dtype=np.float32))
    payload, header = O.pack_pools(z, idx_o, slots["sslot"], g)
    rows_o, counts_o = O.receive(payload, header, g)
    info = plan.info
    pools = _pools_device(plan, s, g, payload, header)
    out = torch.full((s.n_experts, g.C_r, s.d_latent), float("nan"), dtype=torch.bfloat16, device=dev())
    erows = torch.full((s.n_experts,), -1, dtype=torch.int32, device=dev())
    ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=dev())
    M.moe_expert_ffn(plan, bf16_dev(w["w1"]), bf16_dev(w["w3"]), bf16_dev(w["w2"]), pools, out, erows, ws)
    torch.cuda.synchronize()
    assert np.array_equal(erows.cpu().numpy(), counts_o)
    Y = host64(out)
    W1, W3, W2 = (w[n].astype(np.float64) for n in ("w1", "w3", "w2"))
    want_all, got_all = [], []
    Yo = np.zeros((s.n_experts, g.C_r, s.d_latent), dtype=np.float32)
    for e in range(s.n_experts):
        n = counts_o[e]
        if n == 0:
            continue
        # the oracle's SwiGLU of the rows the receiver kept (bf16 hidden); the device's
        # bf16 output is held against the unrounded product, its bf16 value feeds combine
        _, _, H = O.swiglu_hidden(rows_o[e].astype(np.float64), W1[e], W3[e], O.round_bf16)
        want_all.append(H @ W2[e].T)
        Yo[e, :n] = O.round_bf16(want_all[-1])
        got_all.append(Y[e, :n])
    assert_close_rms(np.concatenate(got_all), np.concatenate(want_all), what="expert_out")
    # combine, fed the oracle's own expert outputs (uploaded as bf16)
    slot = np.stack([slots["sslot"], slots["rslot"]], axis=-1).astype(np.int32)
    r = torch.empty((s.T, s.d_latent), dtype=torch.bfloat16, device=dev())
    M.moe_combine(plan, bf16_dev(Yo), f32_dev(gate_o), i32_dev(idx_o), i32_dev(slot), r)
    kept = slots["rslot"] >= 0
    want_r = np.zeros((s.T, s.d_latent))
    for t in range(s.T):
        for j in range(s.top_k):
            if kept[t, j]:
                want_r[t] += gate_o[t, j] * Yo[idx_o[t, j], slots["rslot"][t, j]]
    # one rounding of a float32 sum of bf16 terms
    assert_bf16_close(host64(r), want_r, what="combine")


# ------------------------------------------------------------------ bias step


@pytest.mark.parametrize("E,T,k", [(24, 512, 2), (384, 16384, 8)])
def test_bias_update_bit_exact(M, E, T, k):
    s = synth.FULL.with_(T=T, n_experts=E, top_k=k, n_dest=E // 6)
    plan = _plan(M, s)
    rng = np.random.default_rng(E)
    hist = rng.multinomial(T * k, rng.dirichlet(np.ones(E) * 2.0)).astype(np.int32)
    bias = (rng.standard_normal(E) * 1e-3).astype(np.float32)
    want = O.bias_update(hist, bias, 1e-3, T, k)
    b = f32_dev(bias)
    M.moe_bias_update(plan, i32_dev(hist), b, 1e-3)
    assert np.array_equal(b.cpu().numpy().view(np.uint32), want.view(np.uint32))
