"""Pins of the oracle's multiple virtual sources: T splits into S equal token ranges,
each sending its own (destination, wave) pools with its own sender caps, as each GPU of
the expert-parallel layout does ([RU] §2 caps per source-destination pool; [ZH] §3.1
topology); the receiver takes a destination's pools source by source."""
import numpy as np

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

SHAPE = synth.MoEShape("src", T=192, d_model=64, d_latent=32, n_experts=12, top_k=3, n_dest=2,
                       hidden_routed=48, n_shared=1, hidden_shared=32, seed=41)


def _idx(T, E, k, seed, skew=1.0):
    logits = synth.make_logits(T, E, seed)
    logits = (logits - np.float32(skew) * np.log1p(np.arange(E, dtype=np.float32))[None, :]).astype(np.float32)
    return O.route(logits, np.zeros(E, np.float32), k)[0]


def test_capacity_per_source():
    # C_s scales with the source's T/S tokens; C_r with all T tokens
    for S in (1, 2, 4, 8):
        g = O.geometry(SHAPE.with_(n_sources=S))
        assert g.C_s == -(-SHAPE.T * SHAPE.top_k * 110 // (100 * 2 * 3 * S))
        assert g.C_r == -(-SHAPE.T * SHAPE.top_k * 115 // (100 * 12))


def test_each_source_sends_as_a_single_source_of_its_own_tokens():
    S = 4
    s = SHAPE.with_(n_sources=S)
    g = O.geometry(s)
    idx = _idx(s.T, s.n_experts, s.top_k, seed=3)
    sl = O.assign_slots(idx, g)
    Ts = s.T // S
    g1 = O.geometry(s.with_(T=Ts, n_sources=1))
    assert g1.C_s == g.C_s
    for src in range(S):
        part = idx[src * Ts:(src + 1) * Ts]
        one = O.assign_slots(part, g1)
        assert np.array_equal(sl["sslot"][src * Ts:(src + 1) * Ts], one["sslot"])
        assert np.array_equal(sl["pool_fill"][src * g.n_pools:(src + 1) * g.n_pools], one["pool_fill"])


def test_receiver_ranks_in_token_order_by_brute_force():
    S = 3
    s = SHAPE.with_(n_sources=S, T=198)
    g = O.geometry(s)
    idx = _idx(s.T, s.n_experts, s.top_k, seed=5, skew=1.5)
    sl = O.assign_slots(idx, g)
    count = [0] * s.n_experts
    for t in range(s.T):
        for j in range(s.top_k):
            e = idx[t, j]
            if sl["sslot"][t, j] < 0:
                assert sl["rslot"][t, j] == -1
                continue
            want = count[e] if count[e] < g.C_r else -1
            assert sl["rslot"][t, j] == want
            count[e] += 1
    assert sl["dropped_sender"] > 0


def test_pools_and_receiver_agree_with_the_slots():
    S = 4
    s = SHAPE.with_(n_sources=S)
    g = O.geometry(s)
    idx = _idx(s.T, s.n_experts, s.top_k, seed=7, skew=1.2)
    sl = O.assign_slots(idx, g)
    z = np.random.default_rng(1).standard_normal((s.T, s.d_latent))
    payload, header = O.pack_pools(z, idx, sl["sslot"], g)
    assert payload.shape[0] == S * g.n_pools
    assert np.array_equal((header >= 0).sum(axis=1), sl["pool_fill"])
    rows, counts = O.receive(payload, header, g)
    assert np.array_equal(counts, sl["expert_kept"])
    for e in range(s.n_experts):
        t, j = np.nonzero((idx == e) & (sl["rslot"] >= 0))
        order = np.argsort(sl["rslot"][t, j])
        assert np.array_equal(rows[e], z[t[order]])
