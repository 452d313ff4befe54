"""Shared helpers of the GPU tests: device upload, tolerances, bf16 bit handling."""
import numpy as np
import torch

# Floating-point bar of the block: max |gpu - oracle| <= 2e-2 * RMS(oracle) per tensor
# (bf16 storage, float32 accumulation).
REL_TOL = 2e-2
# Routed expert weight gradients: the float32-vs-float64 spread of bf16-stored
# intermediates alone reaches ~4% of RMS there (tests/test_oracle_precision.py), so
# they are held to max-abs <= 6e-2 * RMS and relative Frobenius error <= 1e-2.
ROUTED_GRAD_TOL = 6e-2
ROUTED_GRAD_FRO = 1e-2


def dev():
    return torch.device("cuda:0")


def bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev()).to(torch.bfloat16)


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def i32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())


def host64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rms(a):
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def assert_close_rms(got, want, tol=REL_TOL, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if want.size == 0:
        return 0.0
    err = float(np.max(np.abs(got - want)))
    scale = rms(want)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert err <= tol * scale + 1e-30, f"{what}: max|err| {err:.3e} > {tol} * rms {scale:.3e}"
    return err / scale if scale else 0.0


def assert_bf16_close(got, want, what=""):
    """Both sides rounded the same float32/float64 value to bf16: allow one bf16 ulp
    (2^-7 relative) where the two sums fall on different sides of a rounding point."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    # the absolute term covers float32-vs-float64 accumulation where a sum cancels
    bound = 2.0 ** -7 * np.abs(want) + 1e-4 * rms(want)
    bad = np.abs(got - want) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond one bf16 ulp, e.g. {got[bad][:4]} vs {want[bad][:4]}"


def assert_fro_close(got, want, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))
    assert err <= tol, f"{what}: relative Frobenius error {err:.3e} > {tol}"
    return err


def routing_mismatch_check(logits_gpu, logits_oracle, bias, idx_gpu, idx_oracle, match, k, what=""):
    """Bound the routing mismatches by near ties instead of a flat rate.

    The device computes its own float32 router logits, which differ from the oracle's
    by a small accumulation error.  A token's selection (its k experts and their rank
    order) can differ only if two of its top k+1 oracle scores lie closer than twice
    that token's largest score error, delta_t = max_e |s_gpu - s_oracle|: every token
    whose expert list differs must be such a near tie.  Tokens that kept their experts
    but saw a drop decision move were pushed across a cap by an earlier differing token;
    each differing token moves at most k assignments out of pools and k into others (at
    most 2k sender-cap crossings) and, with those, at most 4k receiver-cap crossings, so
    at most (6k + 1) tokens mismatch per differing token.  Returns (rate, near ties)."""
    lg = np.asarray(logits_gpu, np.float64)
    lo = np.asarray(logits_oracle, np.float32).astype(np.float64)
    b = np.asarray(bias, np.float32).astype(np.float64)
    s_g = (lg.astype(np.float32) + b.astype(np.float32)[None, :]).astype(np.float64)
    s_o = (lo.astype(np.float32) + b.astype(np.float32)[None, :]).astype(np.float64)
    delta = np.max(np.abs(s_g - s_o), axis=1)
    top = -np.sort(-s_o, axis=1)[:, :k + 1]
    gap = np.min(top[:, :-1] - top[:, 1:], axis=1) if top.shape[1] > 1 else np.full(top.shape[0], np.inf)
    near = gap <= 2.0 * delta
    differs = ~(np.asarray(idx_gpu) == np.asarray(idx_oracle)).all(axis=1)
    n_mis = int((~match).sum())
    bad = differs & ~near
    assert not bad.any(), (f"{what}: {int(bad.sum())} tokens routed differently without a near tie, "
                           f"e.g. token {int(np.nonzero(bad)[0][0])}")
    assert n_mis <= (6 * k + 1) * int(differs.sum()), (
        f"{what}: {n_mis} mismatched tokens from {int(differs.sum())} differing selections")
    return n_mis / match.size, int(near.sum())
