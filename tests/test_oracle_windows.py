"""Correlated token windows and drops, on the oracle.

Tokens of one sequence share a component (x_t = sqrt(rho) g_seq + sqrt(1 - rho) eps_t),
so they pick similar experts and fill the same pools: with the caps fixed, drops rise
as more of a source's tokens share one component.  This is the mechanism the pages
give for drops growing with context length ("Marin начинает открытое обучение MoE-модели
с 535 млрд параметров", §4; "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §3.3).
The pages' own figures come from a trained router on real text and are not expected
here; only the direction is pinned.
"""
import numpy as np
import pytest

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

BASE = synth.MoEShape("windows", T=4096, d_model=256, d_latent=128, n_experts=48, top_k=4, n_dest=8,
                      hidden_routed=128, n_shared=1, hidden_shared=128, seed=17)


def _drops(shape):
    inp = synth.make_inputs(shape)
    rb = O.route_batch(inp["x"], inp["weights"], inp["bias"], shape)
    sl = rb["slots"]
    return (sl["dropped_sender"] + sl["dropped_receiver"]) / (shape.T * shape.top_k)


def test_correlated_windows_drop_more_than_independent_tokens():
    iid = _drops(BASE)
    win = _drops(BASE.with_(window=512, rho=0.6))
    print(f"\ndrop fraction: independent tokens {iid:.4f}, rho=0.6 windows of 512 {win:.4f}")
    assert win > iid + 0.02


def test_drops_grow_with_the_length_of_the_shared_sequence():
    fr = [_drops(BASE.with_(window=L, rho=0.6)) for L in (256, 1024, 4096)]
    print("\ndrop fraction for shared sequences of 256, 1024, 4096 tokens:", [f"{f:.4f}" for f in fr])
    assert fr[0] < fr[1] < fr[2]


def test_higher_capacity_factors_drop_less():
    s = BASE.with_(window=1024, rho=0.6)
    lo = _drops(s)
    hi = _drops(s.with_(cap_send=(125, 100), cap_recv=(130, 100)))
    assert hi < lo
