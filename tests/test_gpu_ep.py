"""Expert parallelism through the moe_ep_* calls, G ranks emulated on one GPU.

Each rank has its own plan and buffers; the four exchanges are device copies of the
fixed-shape blocks that torch.distributed would move between GPUs, done between the
phases (every rank's phase has finished before its blocks move, so no kernel ever waits
on another rank).  The G ranks together must reproduce the one-GPU run with
n_sources = G over all their tokens: the same sender slots, the same rows at every
expert, the same outputs, dx and expert gradients, and dense gradients whose per-rank
parts add up to the one-GPU ones.  The one-GPU run itself is held against the oracle by
the n_sources tests.
"""
import numpy as np
import pytest
import torch

from _helpers import REL_TOL, assert_close_rms, bf16_dev, dev, f32_dev, host64
from capacity_limited_routed_b200 import synth

pytestmark = pytest.mark.gpu


def _exchange(blocks, send_key, recv_key):
    """Rank r receives into block (a * Dl + d) * W + w what rank a sent from its block
    (r * Dl + d) * W + w (the pairing of parallel.exchange)."""
    for r, br in enumerate(blocks):
        sc = br.sched
        for a, ba in enumerate(blocks):
            for d in range(sc.Dl):
                for w in range(sc.W):
                    br.buf[recv_key][sc.rows(sc.block(a, d, w))].copy_(ba.buf[send_key][sc.rows(sc.block(r, d, w))])


def _run_ep(shape_rank, G, weights, bias, x, dy):
    from capacity_limited_routed_b200.parallel import EPBlock
    T = shape_rank.T
    blocks = [EPBlock(shape_rank, G, r, device=dev()) for r in range(G)]
    for b in blocks:
        b.load(weights, bias)
    xs = [x[r * T:(r + 1) * T].contiguous() for r in range(G)]
    dys = [dy[r * T:(r + 1) * T].contiguous() for r in range(G)]
    ys = [torch.empty((T, shape_rank.d_model), dtype=torch.float32, device=dev()) for _ in range(G)]
    dxs = [torch.empty_like(y) for y in ys]
    for b, xr in zip(blocks, xs):
        b.fwd_send(xr)
    _exchange(blocks, "send_pools", "recv_pools")
    for b in blocks:
        b.fwd_experts()
    _exchange(blocks, "y_send", "y_recv")
    for b, y in zip(blocks, ys):
        b.fwd_combine(y)
    for b, xr, d in zip(blocks, xs, dys):
        b.bwd_send(xr, d)
    _exchange(blocks, "dy_send", "dy_recv")
    for b in blocks:
        b.bwd_experts()
    _exchange(blocks, "dx_send", "dx_recv")
    for b, xr, dxr in zip(blocks, xs, dxs):
        b.bwd_finish(xr, dxr)
    torch.cuda.synchronize()
    return blocks, torch.cat(ys), torch.cat(dxs)


@pytest.mark.parametrize("base,G", [(synth.TINY, 2), (synth.TINY, 4), (synth.MID.with_(T=4096), 2)],
                         ids=["tiny-2", "tiny-4", "mid-2"])
def test_ep_ranks_reproduce_the_multi_source_run(base, G):
    from capacity_limited_routed_b200.block import MoEBlock
    T = base.T
    s_all = base.with_(T=G * T, n_sources=G, backward=True, seed=base.seed + 40)
    inp = synth.make_inputs(s_all)
    W = {n: bf16_dev(w) for n, w in inp["weights"].items()}
    bias = f32_dev(inp["bias"])
    x, dy = bf16_dev(inp["x"]), bf16_dev(inp["dy"])
    ref = MoEBlock(s_all, device=dev(), training=True)
    ref.load({"weights": W, "bias": bias, "logit_offset": None})
    y_ref = ref.forward(x)
    dx_ref = ref.backward(x, dy)
    torch.cuda.synchronize()
    v = ref.saved_views()
    st = ref.stats_dict()
    assert st["status"] == 0 and st["dropped_sender"] + st["dropped_receiver"] > 0

    blocks, y, dx = _run_ep(base.with_(T=T, n_sources=1, backward=True), G, W, bias, x, dy)
    for b in blocks:
        assert int(b.stats[3].item()) == 0
    # routing and the sender side: bit for bit
    slot_ref = v["slot"].cpu().numpy()
    idx_ref = v["topk_idx"].cpu().numpy()
    for r, b in enumerate(blocks):
        rs = slice(r * T, (r + 1) * T)
        assert np.array_equal(b.topk_idx.cpu().numpy(), idx_ref[rs])
        assert np.array_equal(b.slot[..., 0].cpu().numpy(), slot_ref[rs, :, 0])   # sender slots
    rows = torch.cat([b.expert_rows for b in blocks]).cpu().numpy()
    assert np.array_equal(rows, v["expert_rows"].cpu().numpy())
    # outputs and gradients: the same kernels on the same rows in the same order
    e_y = assert_close_rms(host64(y), host64(y_ref), tol=1e-5, what="y (EP vs one GPU)")
    e_dx = assert_close_rms(host64(dx), host64(dx_ref), tol=1e-5, what="dx (EP vs one GPU)")
    print(f"\n[{base.name} G={G}] y {e_y:.2e}, dx {e_dx:.2e} (max-abs / rms against the one-GPU run)")
    for n in ("w1", "w3", "w2"):
        got = torch.cat([b.grads[n] for b in blocks])
        assert_close_rms(host64(got), host64(ref.grads[n]), tol=1e-5, what=f"d{n} (EP)")
    # dense weights are replicated: their gradient is the sum of the ranks' parts
    for n in ("w_lat_down", "w_router", "w_lat_up", "ws1", "ws3", "ws2"):
        got = sum(b.grads[n].double() for b in blocks)
        e = assert_close_rms(got.cpu().numpy(), host64(ref.grads[n]), tol=REL_TOL / 10, what=f"d{n} (EP, summed)")
        print(f"  d{n}: {e:.2e}")
