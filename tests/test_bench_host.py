"""The benchmark's algorithmic work per step, pinned to figures derived by hand from the
block's definition (full width: T=16384, d_model 6144, latent 3072, 384 experts top-8,
hidden 3072, two shared experts of 3072)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from capacity_limited_routed_b200 import synth  # noqa: E402


@pytest.fixture(scope="module")
def full():
    s = synth.TRAIN
    kept = s.T * s.top_k                     # no drops
    return s, bench.step_work(s, kept)


def test_forward_flops_per_token(full):
    s, (f, _) = full
    fwd = sum(v for k, v in f.items() if k.startswith("fwd.") or k.startswith("experts."))
    # per token: down 2*6144*3072, router 2*3072*384, routed 8 experts x 3 matrices of
    # 3072 x 3072 x 2, up 2*3072*6144, shared 2 experts x 3 matrices of 6144 x 3072 x 2
    per_token = (2 * 6144 * 3072 + 2 * 3072 * 384 + 8 * 3 * 3072 * 3072 * 2 + 2 * 3072 * 6144
                 + 2 * 3 * 6144 * 3072 * 2)
    assert fwd == per_token * s.T
    assert round(per_token / 1e6, 1) == 757.3


def test_backward_is_twice_the_forward_gemm_work(full):
    s, (f, _) = full
    fwd = sum(v for k, v in f.items() if k.startswith("fwd.") or k.startswith("experts."))
    bwd = sum(v for k, v in f.items() if k.startswith("bwd."))
    assert bwd == 2 * fwd


def test_mover_bytes(full):
    s, (_, b) = full
    # dispatch: z read once (6 KB) and 8 rows of 6 KB + a 16-byte header written
    assert b["fwd.dispatch_pack"] == s.T * (3072 * 2 + 8 * (3072 * 2 + 16))
    assert b["fwd.dispatch_pack"] // s.T == 55424
    # combine: 8 expert rows read, gate and slot pair read, r written
    assert b["fwd.combine"] == s.T * (8 * 3072 * 2 + 8 * 12 + 3072 * 2)
    # routed weight gradients of w1 and w3: float32 writes dominate
    assert b["bwd.experts_wgrad_gate_up"] >= 2 * 384 * 3072 * 3072 * 4


def test_measured_traffic_only_for_the_captured_shape():
    assert bench.measured_traffic("no such step", synth.TRAIN) is None
    assert bench.measured_traffic("bwd.experts_wgrad_gate_up", synth.MID) is None
