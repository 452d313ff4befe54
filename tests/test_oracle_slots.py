"""Pins for the oracle's capacity-limited slot assignment and pooled transport.

The brute force below simulates the pools and the experts one assignment at a time
with plain dictionaries; the oracle ranks with a stable sort.  Invariants and
special cases (no caps: dropless; no sender cap: textbook per-expert capacity)
cover the rest.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from capacity_limited_routed_b200 import synth
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


def simulate(idx, E, D, W, C_s, C_r):
    """One assignment at a time: a counter per pool and one per expert."""
    L = E // D
    P = L // W
    pool_cnt, exp_cnt = {}, {}
    T, k = idx.shape
    sslot = np.full((T, k), -1, dtype=np.int64)
    rslot = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            p = (e // L) * W + (e % L) // P
            s = pool_cnt.get(p, 0)
            pool_cnt[p] = s + 1
            if s >= C_s:
                continue
            sslot[t, j] = s
            r = exp_cnt.get(e, 0)
            exp_cnt[e] = r + 1
            if r < C_r:
                rslot[t, j] = r
    return sslot, rslot


def _geom(T, E, k, D, W, C_s, C_r):
    L = E // D
    return O.Geometry(T=T, E=E, k=k, D=D, W=W, L=L, P=L // W, C_s=C_s, C_r=C_r)


def _random_idx(T, E, k, seed, skew=0.0):
    logits = synth.make_logits(T, E, seed)
    if skew:
        logits = logits - np.float32(skew) * np.log1p(np.arange(E, dtype=np.float32))[None, :]
    idx, _, _ = O.route(logits, np.zeros(E, np.float32), k)
    return idx


def test_worked_example_slots():
    g = _golden("worked_examples.json")["slots"]
    geo = _geom(len(g["idx"]), g["E"], g["k"], g["D"], g["W"], g["C_s"], g["C_r"])
    assert O.placement(geo)["pool"].tolist() == g["pool_of_expert"]
    s = O.assign_slots(np.array(g["idx"], dtype=np.int32), geo)
    assert s["sslot"].tolist() == g["sslot"]
    assert s["rslot"].tolist() == g["rslot"]
    assert (s["kept"], s["dropped_sender"], s["dropped_receiver"]) == (
        g["kept"], g["dropped_sender"], g["dropped_receiver"])
    assert s["pool_fill"].tolist() == g["pool_fill"]


def test_capacity_table_matches_exact_rationals():
    tab = _golden("capacities.json")
    for name in ("tiny", "mid", "full", "skewed"):
        c = tab[name]
        exp_rows_s = Fraction(c["T"] * c["k"], c["D"] * c["W"])
        exp_rows_r = Fraction(c["T"] * c["k"], c["E"])
        want_s = -(-(exp_rows_s * Fraction(110, 100)).numerator // (exp_rows_s * Fraction(110, 100)).denominator)
        want_r = -(-(exp_rows_r * Fraction(115, 100)).numerator // (exp_rows_r * Fraction(115, 100)).denominator)
        assert (want_s, want_r) == (c["C_s"], c["C_r"])
        assert O.capacities(c["T"], c["k"], c["E"], c["D"], c["W"]) == (c["C_s"], c["C_r"])
    assert (tab["full"]["C_s"], tab["full"]["C_r"]) == (751, 393)


@pytest.mark.parametrize("seed,skew", [(0, 0.0), (1, 0.8), (2, 2.0)])
def test_slots_match_simulation(seed, skew):
    T, E, k, D, W = 300, 24, 3, 4, 3
    C_s, C_r = O.capacities(T, k, E, D, W)
    idx = _random_idx(T, E, k, seed, skew)
    geo = _geom(T, E, k, D, W, C_s, C_r)
    s = O.assign_slots(idx, geo)
    ss, rr = simulate(idx, E, D, W, C_s, C_r)
    assert np.array_equal(s["sslot"], ss)
    assert np.array_equal(s["rslot"], rr)


@pytest.mark.parametrize("seed,skew", [(3, 0.0), (4, 1.5)])
def test_slot_invariants(seed, skew):
    T, E, k, D, W = 512, 24, 2, 4, 3
    C_s, C_r = O.capacities(T, k, E, D, W)
    idx = _random_idx(T, E, k, seed, skew)
    geo = _geom(T, E, k, D, W, C_s, C_r)
    s = O.assign_slots(idx, geo)
    assert s["kept"] + s["dropped_sender"] + s["dropped_receiver"] == T * k
    pl = O.placement(geo)
    pool = pl["pool"][idx]
    # sender slots are dense 0..fill-1 and unique per pool; fill <= C_s
    for p in range(geo.n_pools):
        sl = np.sort(s["sslot"][(pool == p) & (s["sslot"] >= 0)])
        assert np.array_equal(sl, np.arange(sl.size))
        assert sl.size <= C_s and sl.size == s["pool_fill"][p]
    for e in range(E):
        sl = np.sort(s["rslot"][(idx == e) & (s["rslot"] >= 0)])
        assert np.array_equal(sl, np.arange(sl.size))
        assert sl.size <= C_r and sl.size == s["expert_kept"][e]
    # a receiver drop is always a sender-kept row
    assert not np.any((s["rslot"] >= 0) & (s["sslot"] < 0))
    assert (s["expert_kept"] + s["expert_dropped_sender"] + s["expert_dropped_receiver"]
            == np.bincount(idx.ravel(), minlength=E)).all()
    if skew:
        assert s["dropped_sender"] + s["dropped_receiver"] > 0


def test_no_caps_means_no_drops():
    T, E, k, D, W = 256, 24, 4, 4, 3
    idx = _random_idx(T, E, k, 9, skew=3.0)
    s = O.assign_slots(idx, _geom(T, E, k, D, W, C_s=T * k, C_r=T * k))
    assert s["kept"] == T * k and s["dropped_sender"] == 0 and s["dropped_receiver"] == 0


def test_no_sender_cap_is_textbook_expert_capacity():
    """With the sender cap out of reach only the per-expert capacity acts: each
    expert keeps its first C_r assignments in token order."""
    T, E, k, D, W = 256, 24, 2, 4, 3
    C_r = 17
    idx = _random_idx(T, E, k, 10, skew=1.0)
    s = O.assign_slots(idx, _geom(T, E, k, D, W, C_s=T * k, C_r=C_r))
    for e in range(E):
        pos = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e]
        for n, (t, j) in enumerate(pos):
            assert s["rslot"][t, j] == (n if n < C_r else -1)


def test_pack_and_receive_use_the_packed_ids():
    """The receiver, seeing only the pools (payload + packed expert id), recovers the
    same rows in the same receiver-slot order as the sender's scan."""
    T, E, k, D, W = 200, 24, 3, 4, 3
    C_s, C_r = O.capacities(T, k, E, D, W)
    idx = _random_idx(T, E, k, 12, skew=1.2)
    geo = _geom(T, E, k, D, W, C_s, C_r)
    s = O.assign_slots(idx, geo)
    z = np.random.default_rng(0).standard_normal((T, 8))
    payload, header = O.pack_pools(z, idx, s["sslot"], geo)
    assert np.array_equal((header >= 0).sum(axis=1), s["pool_fill"])
    rows, counts = O.receive(payload, header, geo)
    assert np.array_equal(counts, s["expert_kept"])
    for e in range(E):
        tj = sorted(((s["rslot"][t, j], t) for t in range(T) for j in range(k)
                     if idx[t, j] == e and s["rslot"][t, j] >= 0))
        want = np.array([z[t] for _, t in tj]).reshape(-1, 8)
        assert np.array_equal(rows[e], want)
