"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device memory.

Some callers have no allocator of their own (a plugin inside a host program that owns
the whole device-memory budget, for instance), so they cannot hand moe_dispatch a
workspace.  moe_dispatch_noalloc keeps the scan's scratch in a static array inside the
library.  Its results must be those of moe_dispatch, bit for bit, call after call:
the array is shared by every call and keeps the previous call's contents.  Both are
also held against the oracle's slot assignment and pool packing.
"""
import ctypes

import numpy as np
import pytest
import torch

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O


def _idx(T, E, k, seed, skew):
    """k distinct experts per token, skewed towards low ids (input generation only)."""
    rng = np.random.default_rng(seed)
    scores = rng.standard_normal((T, E)) - skew * np.log1p(np.arange(E))[None, :]
    return np.argsort(-scores, axis=1, kind="stable")[:, :k].astype(np.int32)


def _run_both(M, shape, seed, skew):
    dev = torch.device("cuda:0")
    plan = M.Plan.from_shape(shape)
    info = plan.info
    T, k, dl = shape.T, shape.top_k, shape.d_latent
    z = torch.from_numpy(np.random.default_rng(seed + 1).standard_normal((T, dl), dtype=np.float32)).to(dev)
    z = z.to(torch.bfloat16)
    idx_np = _idx(T, shape.n_experts, k, seed, skew)
    idx = torch.from_numpy(idx_np).to(dev)
    outs = []
    for use_static in (False, True):
        pools = torch.zeros(info.pools_bytes // 2, dtype=torch.int16, device=dev)
        slot = torch.full((T, k, 2), -9, dtype=torch.int32, device=dev)
        stats = torch.zeros(info.stats_bytes // 4, dtype=torch.int32, device=dev)
        if use_static:
            M.moe_dispatch_noalloc(plan, z, idx, pools, slot, stats)
        else:
            ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=dev)
            M.moe_dispatch(plan, z, idx, pools, slot, stats, ws)
        torch.cuda.synchronize()
        outs.append((pools.cpu().numpy(), slot.cpu().numpy(), stats.cpu().numpy()))
    return plan, idx_np, z.view(torch.int16).cpu().numpy(), outs


def _check_against_oracle(shape, plan, idx_np, z_bits, pools, slot, stats):
    """Slots, counters, headers and payload rows as the oracle assigns and packs them."""
    g = O.geometry(shape)
    sl = O.assign_slots(idx_np, g)
    payload, header = O.pack_pools(z_bits, idx_np, sl["sslot"], g)
    E, dl = shape.n_experts, shape.d_latent
    assert np.array_equal(slot[..., 0], sl["sslot"]) and np.array_equal(slot[..., 1], sl["rslot"])
    assert (stats[0], stats[1], stats[2], stats[3]) == (sl["kept"], sl["dropped_sender"], sl["dropped_receiver"], 0)
    assert np.array_equal(stats[8 + E:8 + 4 * E], np.concatenate(
        [sl["expert_kept"], sl["expert_dropped_sender"], sl["expert_dropped_receiver"]]))
    assert np.array_equal(stats[8 + 4 * E:8 + 4 * E + plan.info.n_pools], sl["pool_fill"])
    rows = pools.reshape(plan.info.n_pools, plan.info.cap_send, dl + 8)
    hdr = rows[:, :, dl:dl + 2].copy().view(np.int32)[:, :, 0]
    assert np.array_equal(hdr, header)
    used = header >= 0
    assert np.array_equal(rows[:, :, :dl][used], payload[used])
    return sl


@pytest.mark.gpu
def test_noalloc_dispatch_matches_dispatch_on_consecutive_calls():
    from capacity_limited_routed_b200 import moe as M
    small = synth.TINY.with_(T=777, top_k=5)
    cases = [(small, 3, 1.2),                              # drops at both caps
             (synth.MID, 4, 0.3),                          # a larger scan next
             (synth.MID.with_(n_sources=2), 6, 0.8),       # two sources: per-source pool scan
             (small, 3, 1.2)]                              # the first plan again, over stale words
    for shape, seed, skew in cases:
        plan, idx_np, z_bits, ((p_ref, s_ref, st_ref), (p_new, s_new, st_new)) = _run_both(M, shape, seed, skew)
        assert np.array_equal(s_new, s_ref)
        assert np.array_equal(st_new, st_ref)
        assert np.array_equal(p_new[:p_ref.size].reshape(-1, shape.d_latent + 8)[:, shape.d_latent:],
                              p_ref.reshape(-1, shape.d_latent + 8)[:, shape.d_latent:])
        sl = _check_against_oracle(shape, plan, idx_np, z_bits, p_new, s_new, st_new)
        _check_against_oracle(shape, plan, idx_np, z_bits, p_ref, s_ref, st_ref)
        assert sl["dropped_sender"] + sl["dropped_receiver"] > 0 or skew < 1.0


def test_noalloc_dispatch_rejects_plans_beyond_its_static_scratch():
    """A plan whose scan needs more than the static array holds is refused, with a
    message that names both sizes, before anything touches a device."""
    from capacity_limited_routed_b200 import moe as M
    plan = M.Plan(T=1 << 20, d_model=64, d_latent=64, n_experts=1024, top_k=2, n_dest=32,
                  hidden_routed=128, n_shared=1, hidden_shared=128, n_waves=1)
    fake = ctypes.c_void_p(0x1000)
    code = M.lib().moe_dispatch_noalloc(plan.handle, fake, fake, fake, fake, fake, None)
    assert code == 2
    msg = M.moe_last_error()
    assert "static array holds 2097152" in msg and "moe_dispatch" in msg
