"""How far two correct bf16-storage implementations of the block drift apart.

The device stores every tensor passed between steps in bf16 and accumulates in
float32; the oracle mirrors the bf16 storage but accumulates in float64.  Where a
float32 and a float64 sum fall on opposite sides of a bf16 rounding point the stored
values differ by one bf16 ulp.  For the routed expert weight gradients, sums over
the few rows an expert keeps of heavy-tailed products (dA, dB are products of
Gaussians), one such flip moves a gradient element by several percent of the
tensor's RMS.  This test runs the oracle with float32 accumulation against itself
with float64 accumulation (same steps, same bf16 storage points) and pins the size
of that spread: it is the floor below which no bf16-storage implementation can be
held, and the GPU parity tests take their tolerances from it.
"""
import numpy as np
import pytest
import torch

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

from _helpers import REL_TOL as BAR, ROUTED_GRAD_FRO, ROUTED_GRAD_TOL as ROUTED_GRAD_BAR


def _rel_max(a, b):
    return float(np.max(np.abs(a - b)) / np.sqrt(np.mean(np.asarray(b, np.float64) ** 2)))


def _rel_fro(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID.with_(T=2048)], ids=["tiny", "mid2048"])
def test_float32_accumulation_spread(shape):
    s = shape.with_(backward=True)
    inp = synth.make_inputs(s)
    y64, c64 = O.forward(inp["x"], inp["weights"], inp["bias"], s)
    dx64, g64, _ = O.backward(inp["dy"], inp["weights"], c64)
    y32, c32 = O.forward(inp["x"], inp["weights"], inp["bias"], s, acc="f32")
    dx32, g32, _ = O.backward(inp["dy"], inp["weights"], c32)
    assert np.array_equal(c32["idx"], c64["idx"])          # same routing: a pure precision spread
    spread = {"y": _rel_max(y32, y64), "dx": _rel_max(dx32, dx64)}
    spread.update({n: _rel_max(g32[n], g64[n]) for n in g64})
    print("\nmax-abs spread / rms:", {k: f"{v:.4f}" for k, v in spread.items()})
    routed = ("w1", "w3", "w2")
    for n, v in spread.items():
        if n in routed:
            assert v < ROUTED_GRAD_BAR
            assert _rel_fro(g32[n], g64[n]) < ROUTED_GRAD_FRO / 5
        else:
            assert v < BAR / 1.5, n
    # the stated 2e-2 bar is below this floor for the routed weight gradients
    assert max(spread[n] for n in routed) > BAR


def test_round_bf16_matches_the_library_conversion():
    """The oracle's own bf16 rounding equals torch's float32 -> bfloat16 conversion
    (round to nearest even), including signed zeros, infinities and exact ties."""
    rng = np.random.default_rng(0)
    a = rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000)
    a = np.concatenate([a, [0.0, -0.0, np.inf, -np.inf, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)]])
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(a)
    assert np.array_equal(got, ref)
    assert np.signbit(got[-6]) and O.round_bf16(np.array([1.0 + 2 ** -8]))[0] == 1.0


def test_sparse_upstream_spread():
    """With the upstream gradient non-zero on a few tokens only, every weight gradient is
    a sum of a few outer products of bf16-stored factors, and one flip of one stored
    element moves a sizeable share of the sum's RMS.  The float32-vs-float64 spread of
    two correct implementations then exceeds the 2e-2 bar for the routed gradients by
    far (one or two rows per expert), while the relative Frobenius error stays small.
    The full-width sparse-upstream parity check therefore holds every gradient to the
    routed bars (max-abs 6e-2 * RMS, Frobenius 1e-2), routed ones to the Frobenius bar
    and a loose max-abs sanity bound."""
    s = synth.MID.with_(T=2048, backward=True)
    inp = synth.make_inputs(s)
    toks = np.sort(np.random.default_rng(1).choice(s.T, size=32, replace=False))
    dy = np.zeros_like(inp["dy"])
    dy[toks] = inp["dy"][toks]
    y64, c64 = O.forward(inp["x"], inp["weights"], inp["bias"], s)
    _, g64, _ = O.backward(dy, inp["weights"], c64)
    y32, c32 = O.forward(inp["x"], inp["weights"], inp["bias"], s, acc="f32")
    _, g32, _ = O.backward(dy, inp["weights"], c32)
    assert np.array_equal(c32["idx"], c64["idx"])
    spread = {n: _rel_max(g32[n], g64[n]) for n in g64}
    fro = {n: _rel_fro(g32[n], g64[n]) for n in g64}
    print("\nsparse upstream, 32 tokens: max-abs spread / rms", {k: f"{v:.4f}" for k, v in spread.items()})
    routed = ("w1", "w3", "w2")
    assert max(spread[n] for n in routed) > 2 * ROUTED_GRAD_BAR     # no max-abs bar holds there
    for n in g64:
        assert fro[n] < ROUTED_GRAD_FRO / 5, n
        if n not in routed:
            assert spread[n] < ROUTED_GRAD_BAR / 2, n
        else:
            assert spread[n] < 0.5, n
