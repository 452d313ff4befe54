"""Expert parallelism, on the oracle: G sources of T tokens each pack their own pools; the
blocks of every pool go to the rank that owns its destination, source-major; every
receiver then keeps exactly the rows, in exactly the order, that the receiver of a
single run with n_sources = G over all G*T tokens keeps for the same experts.  Sender
caps are each source's, receiver caps come from all G*T tokens ("Marin начинает открытое
обучение MoE-модели с 535 млрд параметров", §2: per-pool sender cap, per-expert receiver
cap, ids in the payload and no count exchange)."""
import numpy as np
import pytest

from capacity_limited_routed_b200 import synth
from capacity_limited_routed_b200.parallel import BlockSchedule
from oracle import moe_oracle as O


@pytest.mark.parametrize("G", [2, 4])
def test_ep_receivers_keep_the_rows_of_the_multi_source_run(G):
    T, E, k, D, W, dl = 256, 48, 4, 8, 3, 16
    s_all = synth.MoEShape("ep", T=G * T, d_model=64, d_latent=dl, n_experts=E, top_k=k, n_dest=D,
                           hidden_routed=128, n_shared=1, hidden_shared=128, n_sources=G)
    g_all = O.geometry(s_all)
    logits = synth.make_logits(G * T, E, seed=7) - 0.8 * np.log1p(np.arange(E, dtype=np.float32))[None, :]
    idx, _, _ = O.route(logits.astype(np.float32), np.zeros(E, np.float32), k)
    z = np.random.default_rng(8).standard_normal((G * T, dl)).astype(np.float32)
    # the single run with G virtual sources: its pools and what its receiver keeps
    sl_all = O.assign_slots(idx, g_all)
    pay_all, hdr_all = O.pack_pools(z, idx, sl_all["sslot"], g_all)
    rows_all, counts_all = O.receive(pay_all, hdr_all, g_all)
    assert sl_all["dropped_receiver"] > 0 and sl_all["dropped_sender"] > 0
    # G ranks: each packs its own tokens as one source with its own sender caps
    g_src = O.geometry(s_all.with_(T=T, n_sources=1))
    assert g_src.C_s == g_all.C_s
    packed = []
    for r in range(G):
        ir = idx[r * T:(r + 1) * T]
        sl = O.assign_slots(ir, g_src)
        assert np.array_equal(sl["sslot"], sl_all["sslot"][r * T:(r + 1) * T])
        packed.append(O.pack_pools(z[r * T:(r + 1) * T], ir, sl["sslot"], g_src))
    El, Dl = E // G, D // G
    for q in range(G):
        sched = BlockSchedule(G, q, Dl, W, g_src.C_s)
        # receiver q's buffer: block (a * Dl + d) * W + w holds source a's pool of destination q * Dl + d
        pay = np.zeros((sched.n_blocks, g_src.C_s, dl), np.float32)
        hdr = np.full((sched.n_blocks, g_src.C_s), -1, np.int32)
        for a in range(G):
            for d in range(Dl):
                for w in range(W):
                    b = sched.block(a, d, w)
                    p_src = (q * Dl + d) * W + w       # the source's pool of that destination and wave
                    pay[b], hdr[b] = packed[a][0][p_src], packed[a][1][p_src]
        g_rcv = O.Geometry(T=T, E=El, k=k, D=Dl, W=W, L=g_all.L, P=g_all.P, C_s=g_src.C_s, C_r=g_all.C_r, S=G)
        local_hdr = np.where(hdr >= 0, hdr - q * El, -1)
        rows, counts = O.receive(pay, local_hdr, g_rcv)
        for e in range(El):
            assert counts[e] == counts_all[q * El + e]
            assert np.array_equal(rows[e], rows_all[q * El + e])
