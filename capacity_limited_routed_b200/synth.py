"""Seeded synthetic workloads for the capacity-limited, pooled-wave MoE block.

This module only draws random numbers and names workload shapes.  It holds none
of the block's arithmetic (no routing, no capacities, no GEMMs), so that both the
CUDA path and the CPU oracle can be fed the very same buffers from here without
sharing any of the method's code.

Shapes follow the five workloads the block is measured on:
  1. tiny     T=512,   d_model 256,  latent 128,  E=24,  top-2, D=4,  h=128,  1 shared (128)
  2. mid      T=8192,  d_model 2048, latent 1024, E=96,  top-8, D=16, h=1024, 2 shared (1024)
  3. full     T=16384, d_model 6144, latent 3072, E=384, top-8, D=64, h=3072, 2 shared (3072)
  4. skewed   as 3 with T=65536, Zipf(1.1) per-expert logit skew, rho=0.6 windows of 512
  5. train    as 3, forward + backward, upstream grad ~ N(0,1)
The full width (6144 model, 3072 latent, 384 routed experts, top-8, 2 shared
experts of width 3072, 64-GPU expert-parallel domain with six experts per GPU)
is the one the Marin 535B-A23B pages describe ("Marin 535B-A23B：一场完全公开的前沿
MoE 训练直播", §2.1 spec table and §2.2 MoE diagram; "Marin начинает открытое обучение
MoE-модели с 535 млрд параметров", §2).

Recipe (same for every workload): ``numpy.random.default_rng(seed)`` (PCG64),
values drawn in float32, rounded to bfloat16 with round-to-nearest-even.
Weights ~ N(0, 1/fan_in).  Router bias starts at 0.  Seeds: workload i uses
seed i-1 unless a test overrides it.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
import math

import numpy as np


@dataclass(frozen=True)
class MoEShape:
    """Sizes of one MoE block workload (all counts in elements)."""

    name: str
    T: int
    d_model: int
    d_latent: int
    n_experts: int
    top_k: int
    n_dest: int
    hidden_routed: int
    n_shared: int
    hidden_shared: int
    n_waves: int = 3
    cap_send: tuple = (110, 100)
    cap_recv: tuple = (115, 100)
    dropless: bool = False       # no cap binds: every assignment kept (ragged buffers)
    n_sources: int = 1           # T splits into this many sources with their own sender pools
    # workload-only knobs (input recipe, not part of the block)
    zipf_s: float = 0.0          # >0: per-expert logit skew with Zipf(s) expected load
    window: int = 0              # >0: tokens in windows of this size share a component
    rho: float = 0.0             # share of variance carried by the window component
    backward: bool = False
    seed: int = 0

    def with_(self, **kw) -> "MoEShape":
        return replace(self, **kw)


TINY = MoEShape("tiny", T=512, d_model=256, d_latent=128, n_experts=24, top_k=2,
                n_dest=4, hidden_routed=128, n_shared=1, hidden_shared=128, seed=0)
MID = MoEShape("mid", T=8192, d_model=2048, d_latent=1024, n_experts=96, top_k=8,
               n_dest=16, hidden_routed=1024, n_shared=2, hidden_shared=1024, seed=1)
FULL = MoEShape("full", T=16384, d_model=6144, d_latent=3072, n_experts=384, top_k=8,
                n_dest=64, hidden_routed=3072, n_shared=2, hidden_shared=3072, seed=2)
SKEWED = FULL.with_(name="skewed", T=65536, zipf_s=1.1, window=512, rho=0.6, seed=3)
TRAIN = FULL.with_(name="train", backward=True, seed=4)

WORKLOADS = {1: TINY, 2: MID, 3: FULL, 4: SKEWED, 5: TRAIN}

# A small case of the full-width kernels for profiler captures: full widths, 24 experts
# over 4 destinations and T=1024, so each expert still receives ~341 of C_r=393 rows
# as in the full layer, with ~4.5 GB on the device instead of ~50 GB.
PROFILE = TRAIN.with_(name="profile", T=1024, n_experts=24, n_dest=4, seed=5)
# The forward with the same 24 experts and T=8192: the routing and movement kernels move
# 50 MB to 400 MB per launch (their traffic does not depend on the expert count), beyond
# L2, with ~4 GB on the device.
PROFILE_MOVERS = FULL.with_(name="profile_movers", T=8192, n_experts=24, n_dest=4, seed=6)
# The routing kernels at the full layer's size (T=16384, 384 experts top-8, 64 x 3 pools,
# latent 3072) with the routed hidden width cut to 256, so ~5 GB sit on the device: the
# router, top-k and slot scan see exactly the full layer's inputs.
PROFILE_ROUTER = FULL.with_(name="profile_router", hidden_routed=256, seed=8)
# the same with the backward and the bias step: the router's gradient GEMMs at full size
PROFILE_ROUTER_TRAIN = PROFILE_ROUTER.with_(name="profile_router_train", backward=True)
# the dropless variant of the full-width training step and of the skewed stress
TRAIN_DROPLESS = TRAIN.with_(name="train_dropless", dropless=True)
SKEWED_DROPLESS = SKEWED.with_(name="skewed_dropless", dropless=True)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16, returned as float32."""
    return bf16_bits_to_f32(to_bf16_bits(a))


def _normal(rng, shape, std):
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def make_weights(shape: MoEShape, rng: np.random.Generator) -> dict:
    """Random-init weights of the block, [out][in] row-major, bf16-valued float32.

    Names: w_lat_down [d_l][d_m], w_router [E][d_l], w1/w3 (routed gate/value)
    [E][h][d_l], w2 (routed down) [E][d_l][h], w_lat_up [d_m][d_l], ws1/ws3 (shared
    gate/value, experts stacked on rows) [S*h_s][d_m], ws2 (shared down, experts
    side by side on columns) [d_m][S*h_s].
    """
    s = shape
    dm, dl, E, h, S, hs = s.d_model, s.d_latent, s.n_experts, s.hidden_routed, s.n_shared, s.hidden_shared
    w = {
        "w_lat_down": _normal(rng, (dl, dm), 1.0 / math.sqrt(dm)),
        "w_router": _normal(rng, (E, dl), 1.0 / math.sqrt(dl)),
        "w1": _normal(rng, (E, h, dl), 1.0 / math.sqrt(dl)),
        "w3": _normal(rng, (E, h, dl), 1.0 / math.sqrt(dl)),
        "w2": _normal(rng, (E, dl, h), 1.0 / math.sqrt(h)),
        "w_lat_up": _normal(rng, (dm, dl), 1.0 / math.sqrt(dl)),
        "ws1": _normal(rng, (S * hs, dm), 1.0 / math.sqrt(dm)),
        "ws3": _normal(rng, (S * hs, dm), 1.0 / math.sqrt(dm)),
        "ws2": _normal(rng, (dm, S * hs), 1.0 / math.sqrt(hs)),
    }
    return {k: _bf16(v) for k, v in w.items()}


def make_tokens(shape: MoEShape, rng: np.random.Generator) -> np.ndarray:
    """Input activations x [T][d_model], bf16-valued float32.

    With ``window``/``rho`` set, x_t = sqrt(rho)*g_{t // window} + sqrt(1-rho)*eps_t
    (g, eps i.i.d. N(0, I)): tokens inside one window are correlated, the way the
    tokens of one long sequence are.
    """
    s = shape
    if s.window and s.rho > 0.0:
        n_win = (s.T + s.window - 1) // s.window
        g = _normal(rng, (n_win, s.d_model), 1.0)
        x = np.empty((s.T, s.d_model), dtype=np.float32)
        a, b = np.float32(math.sqrt(s.rho)), np.float32(math.sqrt(1.0 - s.rho))
        for wi in range(n_win):
            lo, hi = wi * s.window, min(s.T, (wi + 1) * s.window)
            x[lo:hi] = a * g[wi] + b * _normal(rng, (hi - lo, s.d_model), 1.0)
    else:
        x = _normal(rng, (s.T, s.d_model), 1.0)
    return _bf16(x)


def make_logit_offset(shape: MoEShape) -> np.ndarray | None:
    """Per-expert additive logit skew so that expected load follows Zipf(s).

    offset_e = ln p_e - mean(ln p), p_e proportional to (e+1)^-s.  ``None`` when the
    workload has no skew.  float32.
    """
    if not shape.zipf_s:
        return None
    e = np.arange(shape.n_experts, dtype=np.float64)
    lp = -shape.zipf_s * np.log(e + 1.0)
    lp -= np.log(np.exp(lp).sum())
    return (lp - lp.mean()).astype(np.float32)


def make_upstream_grad(shape: MoEShape, rng: np.random.Generator) -> np.ndarray:
    """dy [T][d_model] ~ N(0, 1), bf16-valued float32."""
    return _bf16(_normal(rng, (shape.T, shape.d_model), 1.0))


def make_inputs(shape: MoEShape, seed: int | None = None) -> dict:
    """Everything one step of the block consumes, as host float32 arrays.

    Keys: x, weights (dict), bias (zeros, float32 [E]), logit_offset (or None),
    dy (only when ``shape.backward``).
    """
    rng = np.random.default_rng(shape.seed if seed is None else seed)
    weights = make_weights(shape, rng)
    x = make_tokens(shape, rng)
    out = {
        "x": x,
        "weights": weights,
        "bias": np.zeros(shape.n_experts, dtype=np.float32),
        "logit_offset": make_logit_offset(shape),
    }
    if shape.backward:
        out["dy"] = make_upstream_grad(shape, rng)
    return out


def make_logits(T: int, E: int, seed: int, ties: bool = False) -> np.ndarray:
    """Stand-alone router logits [T][E] float32 for routing-only tests.

    With ``ties`` the values are drawn from a coarse grid (multiples of 1/4 in
    [-2, 2]) so that equal scores, and +0.0 / -0.0 pairs, occur often.
    """
    rng = np.random.default_rng(seed)
    if ties:
        v = rng.integers(-8, 9, size=(T, E)).astype(np.float32) / np.float32(4.0)
        neg_zero = (v == 0) & (rng.random(size=(T, E)) < 0.5)
        v[neg_zero] = np.float32(-0.0)
        return v
    return rng.standard_normal(size=(T, E), dtype=np.float32)


# ------------------------------------------------------------------ device-side generation
#
# Full-width workloads carry 22 GB of expert weights; drawing them with numpy on the
# host takes minutes.  For those the same recipe (N(0, 1/fan_in) weights, N(0, 1)
# tokens, windowed correlation, Zipf logit skew) is drawn with PyTorch's seeded CUDA
# generator instead.  Tensor i of a workload uses seed (1000003 * seed + i), so any
# one tensor can be regenerated on its own.


def _dev_normal(shape, std, seed, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # draw in slabs to bound the float32 temporary
    flat = out.view(-1)
    step = 1 << 28
    for lo in range(0, flat.numel(), step):
        hi = min(flat.numel(), lo + step)
        flat[lo:hi] = (torch.randn(hi - lo, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)
    return out


def make_inputs_device(shape: MoEShape, device="cuda", seed: int | None = None) -> dict:
    """Same keys as ``make_inputs`` but bf16 / float32 tensors on ``device``."""
    import torch
    s = shape
    base = (shape.seed if seed is None else seed) * 1000003
    dm, dl, E, h, S, hs = s.d_model, s.d_latent, s.n_experts, s.hidden_routed, s.n_shared, s.hidden_shared
    spec = [("w_lat_down", (dl, dm), dm), ("w_router", (E, dl), dl), ("w1", (E, h, dl), dl),
            ("w3", (E, h, dl), dl), ("w2", (E, dl, h), h), ("w_lat_up", (dm, dl), dl),
            ("ws1", (S * hs, dm), dm), ("ws3", (S * hs, dm), dm), ("ws2", (dm, S * hs), hs)]
    weights = {n: _dev_normal(shp, 1.0 / math.sqrt(fan), base + i, device) for i, (n, shp, fan) in enumerate(spec)}
    out = make_tokens_device(s, device=device, seed=seed)
    out["weights"] = weights
    return out


def make_tokens_device(shape: MoEShape, device="cuda", seed: int | None = None) -> dict:
    """The per-batch inputs of ``make_inputs_device`` alone (x, bias, logit_offset and,
    for a backward workload, dy), drawn exactly as there: a workload of the same widths
    can then run on weights that already sit on the device."""
    import torch
    s = shape
    base = (shape.seed if seed is None else seed) * 1000003
    dm, E = s.d_model, s.n_experts
    if s.window and s.rho > 0.0:
        n_win = (s.T + s.window - 1) // s.window
        gwin = _dev_normal((n_win, dm), 1.0, base + 20, device).float()
        eps = _dev_normal((s.T, dm), 1.0, base + 21, device)
        x = torch.empty((s.T, dm), dtype=torch.bfloat16, device=device)
        a, b = math.sqrt(s.rho), math.sqrt(1.0 - s.rho)
        for wi in range(n_win):
            lo, hi = wi * s.window, min(s.T, (wi + 1) * s.window)
            x[lo:hi] = (a * gwin[wi][None, :] + b * eps[lo:hi].float()).to(torch.bfloat16)
    else:
        x = _dev_normal((s.T, dm), 1.0, base + 21, device)
    lo_ = make_logit_offset(s)
    out = {
        "x": x,
        "bias": torch.zeros(E, dtype=torch.float32, device=device),
        "logit_offset": None if lo_ is None else torch.from_numpy(lo_).to(device),
    }
    if s.backward:
        out["dy"] = _dev_normal((s.T, dm), 1.0, base + 22, device)
    return out
