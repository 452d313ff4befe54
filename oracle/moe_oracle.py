"""CPU oracle of the capacity-limited, pooled-wave MoE block (forward, backward, bias step).

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU-baseline leg
of the benchmark may import this module.  It shares no code with the CUDA library:
it is a plain, slow, float64 restatement of what the block computes, written so a
reader can hold it against the pages.

Sources (web pages on the Marin 535B-A23B training run):
  [RU]  "Marin начинает открытое обучение MoE-модели с 535 млрд параметров"
        (lamjinlab.com), §2 "Как организована разреженная модель"
  [KO]  "Marin, 5,350억 파라미터 MoE 모델의 공개 학습 시작" (lamjinlab.com), §2
        (the same article as [RU], in Korean)
  [ZH]  "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播" (ranhao.site), §2.2 MoE
        diagram and bullets, §3.2 three-wave buffers, §3.3 token dropping
  [PT]  "Treinamento aberto do Marin 535B: um modelo de fronteira, ao vivo e em
        público" (aoyii.com), section "A matemática do MoE"

What the pages fix, and the readings taken where they are silent:
  * Per token: latent down-projection d_model -> d_latent before the routed path,
    projection back to d_model after it, and two always-on shared experts added on
    top ([RU] §2, [ZH] §2.2).  No residual and no norm inside the block.
  * Router on the latent z, top-k of (logits + bias); the bias is a zero-mean,
    next-step, non-gradient balancing term ([ZH] §2.2).  Gates: softmax of the
    *unbiased* logits over the k chosen experts (reading; the pages name no gate).
    Ties between equal scores go to the lower expert index (reading).
  * One fixed pool per destination per wave; experts are placed in contiguous
    blocks of L = E/D per destination, split into W = 3 waves of P = L/W experts
    ([RU] §2: six experts per GPU, three waves).
  * Sender cap 1.10 per (source, destination) pool and receiver cap 1.15 per local
    expert; overflow assignments are dropped and counted separately ([RU] §2).
    Capacities are the expected row counts times the factor, rounded up in exact
    integer arithmetic (reading): C_s = ceil(1.10 * T*k / (D*W)),
    C_r = ceil(1.15 * T*k / E).  The dropless variant ([ZH] §3.3, §7) is the same
    assignment with no cap binding (``dropless_geometry``).
  * Sender slots are given in (token, rank) order; receiver slots are given among
    the sender-kept rows in the same order (reading).  One GPU is one source.
  * Combine: gate-weighted sum in latent space of the kept expert outputs, then
    one up-projection (linear, so equal to up-projecting each term).  Dropped
    assignments contribute zero; gates are not renormalised after drops.
  * Bias step: sign step of size eta towards the mean load c_bar = T*k/E, made
    exactly zero-mean across experts, from the pre-drop selection histogram
    (reading of "histogram-based quantile router, next-step zero-mean bias").
  * Precision: the block stores every tensor that passes between two of its steps
    in bfloat16 and accumulates in float32.  With ``storage="bf16"`` the oracle
    rounds at those same points (arithmetic stays float64); with
    ``storage="f64"`` nothing is rounded.  The block's own outputs (y, dx and the
    weight gradients) are returned unrounded in both modes: they are the values
    the device's results are measured against.  The two places where floating point
    decides an integer, the score ``logits + bias`` and its comparison, are taken
    in float32, the precision of the logits and of the bias.  The bias step is
    float32 arithmetic on the float32 bias.

Every function here is pinned by tests that do not reuse its formulas: brute-force
enumeration on tiny inputs, closed forms, invariants and finite differences.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------------------
# precision helpers
# --------------------------------------------------------------------------------------


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value of each element, as float64.

    The value is first taken to float32 (round to nearest), then to the 8-bit
    significand of bfloat16 by round-to-nearest-even on the float32 bit pattern: add
    0x7FFF plus the lowest kept bit, clear the 16 dropped bits.  NaN stays NaN."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).astype(np.float64)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = np.nan
    return out


def _storage(mode: str, dt=np.float64):
    if mode == "bf16":
        return lambda a: round_bf16(a).astype(dt)
    if mode == "f64":
        return lambda a: np.asarray(a, dtype=dt)
    raise ValueError(f"unknown storage mode {mode!r}")


def _acc_dtype(acc: str):
    """Accumulation precision.  "f64" is the oracle.  "f32" runs the same steps with
    float32 arithmetic; it exists only to measure how far two correct implementations
    with bf16 storage drift apart when nothing but the accumulation precision differs."""
    return {"f64": np.float64, "f32": np.float32}[acc]


def silu(a: np.ndarray) -> np.ndarray:
    """SiLU (swish with beta = 1): a * sigmoid(a)."""
    return a / (1.0 + np.exp(-a))


def silu_grad(a: np.ndarray) -> np.ndarray:
    """d silu(a) / da = sigmoid(a) * (1 + a * (1 - sigmoid(a)))."""
    s = 1.0 / (1.0 + np.exp(-a))
    return s * (1.0 + a * (1.0 - s))


# --------------------------------------------------------------------------------------
# geometry: capacities and expert placement ([RU] §2; [ZH] §3.2)
# --------------------------------------------------------------------------------------


@dataclass(frozen=True)
class Geometry:
    T: int
    E: int
    k: int
    D: int
    W: int
    L: int        # local experts per destination
    P: int        # experts per wave
    C_s: int      # sender capacity of one (destination, wave) pool of one source
    C_r: int      # receiver capacity of one expert
    S: int = 1    # sources: T splits into S equal contiguous token ranges, each sending
                  # its own pools with its own sender caps (as each GPU does under EP)

    @property
    def n_pools(self) -> int:
        """(destination, wave) pools of one source."""
        return self.D * self.W


def ceil_ratio(a: int, b: int) -> int:
    """ceil(a / b) for positive integers, exact."""
    return (a + b - 1) // b


def capacities(T: int, k: int, E: int, D: int, W: int,
               cap_send=(110, 100), cap_recv=(115, 100), S: int = 1) -> tuple[int, int]:
    """Sender and receiver capacities ([RU] §2: factors 1.10 and 1.15).

    Expected rows per (destination, wave) pool from one source of T/S tokens are
    (T/S)*k/(D*W); per expert (all sources together) T*k/E.  Each is scaled by its
    factor num/den and rounded up exactly.
    """
    ns, ds = cap_send
    nr, dr = cap_recv
    C_s = ceil_ratio(T * k * ns, ds * D * W * S)
    C_r = ceil_ratio(T * k * nr, dr * E)
    return C_s, C_r


def geometry(shape) -> Geometry:
    """Geometry of a workload object with the attributes of ``synth.MoEShape``."""
    E, D, W = shape.n_experts, shape.n_dest, shape.n_waves
    if E % D or (E // D) % W:
        raise ValueError("E must split into D destinations of W equal waves")
    L = E // D
    S = getattr(shape, "n_sources", 1)
    if S < 1 or shape.T % S:
        raise ValueError("T must split into S equal sources")
    C_s, C_r = capacities(shape.T, shape.top_k, E, D, W, shape.cap_send, shape.cap_recv, S)
    return Geometry(T=shape.T, E=E, k=shape.top_k, D=D, W=W, L=L, P=L // W, C_s=C_s, C_r=C_r, S=S)


def source_pool(g: Geometry, idx: np.ndarray) -> np.ndarray:
    """Pool of every assignment of idx [T][k] across sources: source * (D*W) + pool, where
    the source of token t is t // (T/S)."""
    idx = np.asarray(idx)
    src = np.arange(idx.shape[0]) // (idx.shape[0] // g.S) if g.S > 1 else np.zeros(idx.shape[0], np.int64)
    return src[:, None] * g.n_pools + placement(g)["pool"][idx]


def dropless_geometry(g: Geometry, idx: np.ndarray) -> Geometry:
    """Capacities of the dropless variant for one routing ([ZH] §3.3 and §7: the run
    later switched to a dropless ragged all-to-all).

    Reading: the same slot assignment with no cap binding (C = infinity).  A rank can
    never reach past the largest pool load or the largest expert load of the routing
    itself, so those two numbers serve as the capacities: every assignment is kept,
    every pool and expert holds exactly its load.
    """
    pool = source_pool(g, idx)
    C_s = int(np.bincount(pool.ravel(), minlength=g.S * g.n_pools).max()) if pool.size else 0
    C_r = int(np.bincount(np.asarray(idx).ravel(), minlength=g.E).max()) if pool.size else 0
    return Geometry(T=g.T, E=g.E, k=g.k, D=g.D, W=g.W, L=g.L, P=g.P, C_s=max(C_s, 1), C_r=max(C_r, 1), S=g.S)


def placement(g: Geometry) -> dict:
    """Expert e -> destination e // L, local index e % L, wave (e % L) // P, pool dest*W + wave."""
    e = np.arange(g.E)
    dest = e // g.L
    loc = e % g.L
    wave = loc // g.P
    return {"dest": dest, "loc": loc, "wave": wave, "pool": dest * g.W + wave}


# --------------------------------------------------------------------------------------
# router: top-k, gates, load histogram ([ZH] §2.2)
# --------------------------------------------------------------------------------------


def route(logits: np.ndarray, bias: np.ndarray, k: int):
    """Top-k selection on float32 scores, softmax gates on the unbiased logits.

    The selection always uses float32(logits) + float32(bias).  The gates use the
    logits at the precision they are given in (float32 from the device's router,
    float64 when the oracle runs with nothing rounded).

    Returns (idx [T][k] int32 in selection order, gate [T][k] float64,
    hist [E] int64 = pre-drop selections per expert).
    """
    logits = np.asarray(logits)
    bias = np.asarray(bias, dtype=np.float32)
    if np.isnan(logits).any() or np.isnan(bias).any():
        raise ValueError("router logits and bias must not contain NaN")
    T, E = logits.shape
    scores = logits.astype(np.float32) + bias[None, :]  # one float32 add, as on the device
    # order: larger score first; equal scores -> lower expert index first.
    # np.lexsort sorts by the last key first; +0.0 and -0.0 compare equal as floats,
    # so map -0.0 to +0.0 before using the values as a sort key.
    key = np.where(scores == 0, np.float32(0.0), scores).astype(np.float64)
    cols = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((cols, -key), axis=1)
    idx = order[:, :k].astype(np.int32)
    chosen = np.take_along_axis(logits.astype(np.float64), idx, axis=1)
    m = chosen.max(axis=1, keepdims=True)
    ex = np.exp(chosen - m)
    gate = ex / ex.sum(axis=1, keepdims=True)
    hist = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    return idx, gate, hist


# --------------------------------------------------------------------------------------
# capacity-limited slot assignment ([RU] §2; [ZH] §3.2, §3.3)
# --------------------------------------------------------------------------------------


def _running_rank(keys: np.ndarray, valid: np.ndarray) -> np.ndarray:
    """For each valid position i: number of earlier valid positions with the same key."""
    rank = np.full(keys.shape, -1, dtype=np.int64)
    pos = np.nonzero(valid)[0]
    if pos.size == 0:
        return rank
    kv = keys[pos]
    order = np.argsort(kv, kind="stable")              # groups by key, keeps visiting order
    sk = kv[order]
    starts = np.r_[0, np.nonzero(np.diff(sk))[0] + 1]
    first = np.repeat(starts, np.diff(np.r_[starts, sk.size]))
    r = np.arange(sk.size) - first
    out = np.empty(pos.size, dtype=np.int64)
    out[order] = r
    rank[pos] = out
    return rank


def assign_slots(idx: np.ndarray, g: Geometry) -> dict:
    """Sender and receiver slots of every assignment, visited in (token, rank) order.

    sslot[t][j]: position in pool(e) among the assignments of t's source to that
                 pool, or -1 when it is at or past C_s (sender drop).
    rslot[t][j]: position among the sender-kept assignments of expert e, or -1 when
                 it was sender-dropped or is at or past C_r (receiver drop).
    Also returns the counters: kept, dropped_sender, dropped_receiver, per-expert
    kept / sender-dropped / receiver-dropped, and the fill of every pool (source-major,
    S * D * W pools).  The receiver sees a pool group's sources in order, so its
    (token, rank) visiting order is the global one.
    """
    e = np.asarray(idx, dtype=np.int64).ravel()
    pool = source_pool(g, idx).ravel()                  # one set of pools per source
    srank = _running_rank(pool, np.ones(e.size, dtype=bool))
    skept = srank < g.C_s
    rrank = _running_rank(e, skept)
    rkept = skept & (rrank < g.C_r)
    sslot = np.where(skept, srank, -1)
    rslot = np.where(rkept, rrank, -1)
    drop_s = ~skept
    drop_r = skept & ~rkept
    per_kept = np.bincount(e[rkept], minlength=g.E)
    per_ds = np.bincount(e[drop_s], minlength=g.E)
    per_dr = np.bincount(e[drop_r], minlength=g.E)
    fill = np.bincount(pool[skept], minlength=g.S * g.n_pools)
    return {
        "sslot": sslot.reshape(idx.shape).astype(np.int32),
        "rslot": rslot.reshape(idx.shape).astype(np.int32),
        "kept": int(rkept.sum()),
        "dropped_sender": int(drop_s.sum()),
        "dropped_receiver": int(drop_r.sum()),
        "expert_kept": per_kept.astype(np.int64),
        "expert_dropped_sender": per_ds.astype(np.int64),
        "expert_dropped_receiver": per_dr.astype(np.int64),
        "pool_fill": fill.astype(np.int64),
    }


def pack_pools(z: np.ndarray, idx: np.ndarray, sslot: np.ndarray, g: Geometry):
    """Sender side: one fixed pool per (destination, wave), expert id in each row.

    Returns (payload [D*W][C_s][d_l], header [D*W][C_s] int32): the header of a row
    holds the global expert id of the assignment stored there, -1 for an empty row.
    """
    d_l = z.shape[1]
    payload = np.zeros((g.S * g.n_pools, g.C_s, d_l), dtype=z.dtype)
    header = np.full((g.S * g.n_pools, g.C_s), -1, dtype=np.int32)
    spool = source_pool(g, idx)
    T, k = idx.shape
    for t in range(T):
        for j in range(k):
            s = sslot[t, j]
            if s >= 0:
                p = spool[t, j]
                payload[p, s] = z[t]
                header[p, s] = idx[t, j]
    return payload, header


def receive(payload: np.ndarray, header: np.ndarray, g: Geometry):
    """Receiver side: unpack each pool by the expert id in its rows.

    The receiver of a (destination, wave) takes the pools that every source sent it,
    sources in order, rows of each pool in pool order; each local expert keeps its
    first C_r rows.  Returns (rows [E] list of [n_e][d_l] arrays, counts [E]), the rows
    in receiver-slot order.  Uses nothing but the pools themselves.
    """
    d_l = payload.shape[2]
    buckets = [[] for _ in range(g.E)]
    for p in range(g.n_pools):
        for src in range(g.S):
            q = src * g.n_pools + p
            for s in range(g.C_s):
                e = int(header[q, s])
                if e >= 0 and len(buckets[e]) < g.C_r:
                    buckets[e].append(payload[q, s])
    rows = [np.array(b, dtype=payload.dtype).reshape(len(b), d_l) for b in buckets]
    return rows, np.array([r.shape[0] for r in rows], dtype=np.int64)


# --------------------------------------------------------------------------------------
# forward ([RU] §2; [ZH] §2.2; [PT] "A matemática do MoE")
# --------------------------------------------------------------------------------------


def swiglu_hidden(X, w_gate, w_value, st):
    """Pre-activations a = X w_gate^T, b = X w_value^T and hidden H = silu(a) * b.

    H is formed from the unrounded a and b; the a and b returned are the values kept
    for the backward pass, which pass between steps and so are stored (rounded)."""
    a = X @ w_gate.T
    b = X @ w_value.T
    return st(a), st(b), st(silu(a) * b)


def forward(x, weights: dict, bias, shape, logit_offset=None, storage: str = "bf16",
            logits_override=None, acc: str = "f64"):
    """One forward pass of the block.  Returns (y [T][d_model], ctx) where ctx holds
    every intermediate the backward pass and the tests need.

    ``logits_override`` replaces the computed router logits (float32 [T][E]); tests
    use it to study routing separately from the GEMMs.
    """
    dt = _acc_dtype(acc)
    st = _storage(storage, dt)
    g = geometry(shape)
    W = {k: np.asarray(v, dtype=dt) for k, v in weights.items()}
    x = np.asarray(x, dtype=dt)
    # latent down-projection
    z = st(x @ W["w_lat_down"].T)
    # router logits (float32, as the router hands them to top-k)
    if logits_override is None:
        lg = z @ W["w_router"].T
        if logit_offset is not None:
            lg = lg + np.asarray(logit_offset, dtype=dt)[None, :]
        logits = lg.astype(np.float32) if storage == "bf16" else lg
    else:
        logits = np.asarray(logits_override, dtype=np.float32)
    idx, gate, hist = route(logits, bias, g.k)
    if getattr(shape, "dropless", False):
        g = dropless_geometry(g, idx)
    slots = assign_slots(idx, g)
    # routed experts on their kept rows, receiver-slot order
    T, k = idx.shape
    d_l = z.shape[1]
    rows_of = [[] for _ in range(g.E)]                  # (t, j) of each kept row, by rslot
    for t in range(T):
        for j in range(k):
            if slots["rslot"][t, j] >= 0:
                rows_of[idx[t, j]].append((t, j))
    expert = []
    Yrow = np.zeros((T, k, d_l), dtype=dt)
    for e in range(g.E):
        tj = rows_of[e]
        ts = np.array([a for a, _ in tj], dtype=np.int64)
        X = z[ts] if ts.size else np.zeros((0, d_l), dtype=dt)
        a, b, H = swiglu_hidden(X, W["w1"][e], W["w3"][e], st)
        Y = st(H @ W["w2"][e].T)
        expert.append({"tj": tj, "X": X, "a": a, "b": b, "H": H, "Y": Y})
        for n, (t, j) in enumerate(tj):
            Yrow[t, j] = Y[n]
    kept = slots["rslot"] >= 0
    # gate-weighted combine in latent space, in rank order
    r = np.zeros((T, d_l), dtype=dt)
    gate = gate.astype(dt)
    for j in range(k):
        r += np.where(kept[:, j:j + 1], gate[:, j:j + 1] * Yrow[:, j, :], 0.0)
    r = st(r)
    # always-on shared experts on x, experts stacked on the hidden axis
    a_s, b_s, H_s = swiglu_hidden(x, W["ws1"], W["ws3"], st)
    y = r @ W["w_lat_up"].T + H_s @ W["ws2"].T
    ctx = {
        "geometry": g, "storage": storage, "acc": acc, "x": x, "z": z, "logits": logits,
        "idx": idx, "gate": gate, "hist": hist, "slots": slots, "kept": kept,
        "expert": expert, "Yrow": Yrow, "r": r, "a_s": a_s, "b_s": b_s, "H_s": H_s,
    }
    return y, ctx


# --------------------------------------------------------------------------------------
# backward: analytic, dropped assignments get zero gradient, the bias gets none
# --------------------------------------------------------------------------------------


def backward(dy, weights: dict, ctx: dict):
    """Gradients of sum(y * dy) w.r.t. x and every weight.  Returns (dx, grads)."""
    dt = _acc_dtype(ctx.get("acc", "f64"))
    st = _storage(ctx["storage"], dt)
    g: Geometry = ctx["geometry"]
    W = {k: np.asarray(v, dtype=dt) for k, v in weights.items()}
    dy = np.asarray(dy, dtype=dt)
    x, z, idx, gate, kept = ctx["x"], ctx["z"], ctx["idx"], ctx["gate"], ctx["kept"]
    T, k = idx.shape
    d_l = z.shape[1]
    grads = {}
    # y = r w_lat_up^T + H_s ws2^T
    dr = st(dy @ W["w_lat_up"])
    grads["w_lat_up"] = dy.T @ ctx["r"]
    grads["ws2"] = dy.T @ ctx["H_s"]
    dH_s = dy @ W["ws2"]
    da_s = st(dH_s * ctx["b_s"] * silu_grad(ctx["a_s"]))
    db_s = st(dH_s * silu(ctx["a_s"]))
    # r = sum_j kept g_j Y_j
    dg = np.where(kept, np.einsum("td,tjd->tj", dr, ctx["Yrow"]), 0.0)
    dXrow = np.zeros((T, k, d_l), dtype=dt)
    for n in ("w1", "w3", "w2"):
        grads[n] = np.zeros_like(W[n])
    for e, ex in enumerate(ctx["expert"]):
        tj = ex["tj"]
        if not tj:
            continue
        ts = np.array([a for a, _ in tj])
        js = np.array([b for _, b in tj])
        dY = st(gate[ts, js][:, None] * dr[ts])
        dH = dY @ W["w2"][e]
        dA = st(dH * ex["b"] * silu_grad(ex["a"]))
        dB = st(dH * silu(ex["a"]))
        dX = st(dA @ W["w1"][e] + dB @ W["w3"][e])
        grads["w1"][e] = dA.T @ ex["X"]
        grads["w3"][e] = dB.T @ ex["X"]
        grads["w2"][e] = dY.T @ ex["H"]
        dXrow[ts, js] = dX
    # softmax over the chosen logits: dl_j = g_j (dg_j - sum_i g_i dg_i)
    dl_chosen = gate * (dg - (gate * dg).sum(axis=1, keepdims=True))
    dlogits = np.zeros((T, g.E), dtype=dt)
    np.put_along_axis(dlogits, idx.astype(np.int64), dl_chosen, axis=1)
    dlogits = st(dlogits)
    grads["w_router"] = dlogits.T @ z
    dz = st(dlogits @ W["w_router"] + np.where(kept[:, :, None], dXrow, 0.0).sum(axis=1))
    grads["w_lat_down"] = dz.T @ x
    grads["ws1"] = da_s.T @ x
    grads["ws3"] = db_s.T @ x
    dx = dz @ W["w_lat_down"] + da_s @ W["ws1"] + db_s @ W["ws3"]
    inter = {"dr": dr, "dg": dg, "dlogits": dlogits, "dz": dz, "da_s": da_s, "db_s": db_s}
    return dx, grads, inter


# --------------------------------------------------------------------------------------
# bias step ([ZH] §2.2: next-step, zero-mean, outside backprop)
# --------------------------------------------------------------------------------------


def bias_update(hist, bias, step: float, T: int, k: int) -> np.ndarray:
    """b_e <- b_e + step * (sgn_e - sum(sgn)/E), sgn_e = sign(T*k/E - c_e).

    The sign is decided exactly on integers (T*k versus E*c_e).  The update is
    float32 arithmetic on the float32 bias, in this order: mean = float(sum)/float(E),
    delta = float(sgn) - mean, b + float32(step) * delta.
    """
    hist = np.asarray(hist, dtype=np.int64)
    E = hist.size
    sgn = np.sign(T * k - E * hist).astype(np.int64)
    mean = np.float32(np.float32(sgn.sum()) / np.float32(E))
    delta = sgn.astype(np.float32) - mean
    return (np.asarray(bias, dtype=np.float32) + np.float32(step) * delta).astype(np.float32)


# --------------------------------------------------------------------------------------
# work counts (used by the benchmark's roofline arithmetic)
# --------------------------------------------------------------------------------------


def forward_flops(shape, kept_rows: int | None = None) -> int:
    """Algorithmic forward FLOPs: 2 per multiply-add; routed part on kept rows only."""
    s = shape
    T = s.T
    rows = T * s.top_k if kept_rows is None else kept_rows
    down = 2 * T * s.d_model * s.d_latent
    router = 2 * T * s.d_latent * s.n_experts
    routed = rows * 2 * (3 * s.d_latent * s.hidden_routed)
    up = 2 * T * s.d_latent * s.d_model
    shared = T * 2 * (3 * s.d_model * s.hidden_shared) * s.n_shared
    return down + router + routed + up + shared


# --------------------------------------------------------------------------------------
# the same definition evaluated on a sample (for full-size workloads)
# --------------------------------------------------------------------------------------
#
# At full width one forward is ~1e13 FLOPs: too much for float64 on the host.  The
# functions below take the same steps as forward()/backward() above, but evaluate the
# routed experts only for the sampled tokens (or experts).  Routing and drop
# decisions are still computed over the whole batch, since every token's drops
# depend on the tokens before it.  Routed weights are read one expert at a time
# (``weights["w1"][e]``), so they may be a lazy view of device memory.


def route_batch(x, weights, bias, shape, logit_offset=None, storage="bf16"):
    """Latent projection, logits, top-k, gates and slots for every token."""
    st = _storage(storage)
    g = geometry(shape)
    x = np.asarray(x, dtype=np.float64)
    z = st(x @ np.asarray(weights["w_lat_down"], np.float64).T)
    lg = z @ np.asarray(weights["w_router"], np.float64).T
    if logit_offset is not None:
        lg = lg + np.asarray(logit_offset, dtype=np.float64)[None, :]
    logits = lg.astype(np.float32) if storage == "bf16" else lg
    idx, gate, hist = route(logits, bias, g.k)
    if getattr(shape, "dropless", False):
        g = dropless_geometry(g, idx)
    slots = assign_slots(idx, g)
    return {"geometry": g, "storage": storage, "x": x, "z": z, "logits": logits, "idx": idx, "gate": gate,
            "hist": hist, "slots": slots, "kept": slots["rslot"] >= 0}


def _expert_rows(X, weights, e, st):
    W1 = np.asarray(weights["w1"][e], np.float64)
    W3 = np.asarray(weights["w3"][e], np.float64)
    W2 = np.asarray(weights["w2"][e], np.float64)
    a, b, H = swiglu_hidden(X, W1, W3, st)
    return a, b, H, st(H @ W2.T), (W1, W3, W2)


def forward_tokens(weights, rb: dict, tokens):
    """y for the given tokens of a batch routed by ``route_batch``; also the per-token
    pieces the sampled backward needs."""
    st = _storage(rb["storage"])
    idx, gate, kept, z, x = rb["idx"], rb["gate"], rb["kept"], rb["z"], rb["x"]
    W_up = np.asarray(weights["w_lat_up"], np.float64)
    ws1 = np.asarray(weights["ws1"], np.float64)
    ws3 = np.asarray(weights["ws3"], np.float64)
    ws2 = np.asarray(weights["ws2"], np.float64)
    out, per = [], []
    for t in tokens:
        r = np.zeros(z.shape[1])
        rows = []
        for j in range(idx.shape[1]):
            if kept[t, j]:
                a, b, H, Y, Ws = _expert_rows(z[t:t + 1], weights, int(idx[t, j]), st)
                r = r + gate[t, j] * Y[0]
                rows.append((j, a[0], b[0], H[0], Y[0], Ws))
        r = st(r)
        a_s, b_s, H_s = swiglu_hidden(x[t:t + 1], ws1, ws3, st)
        out.append(r @ W_up.T + H_s[0] @ ws2.T)
        per.append({"r": r, "rows": rows, "a_s": a_s[0], "b_s": b_s[0], "H_s": H_s[0]})
    return np.array(out), per


def _backward_token(dy, weights, rb: dict, t, p, dense):
    """The backward pass of one token t of a batch routed by ``route_batch``, for the
    loss y_t . dy: every intermediate of the token and its kept rows."""
    st = _storage(rb["storage"])
    idx, gate = rb["idx"], rb["gate"]
    dy = np.asarray(dy, np.float64)
    dr = st(dy @ dense["w_lat_up"])
    dH_s = dy @ dense["ws2"]
    da_s = st(dH_s * p["b_s"] * silu_grad(p["a_s"]))
    db_s = st(dH_s * silu(p["a_s"]))
    k = idx.shape[1]
    dg = np.zeros(k)
    dXsum = np.zeros(dr.shape[0])
    rows = []
    for (j, a, b, H, Y, (W1, W3, W2)) in p["rows"]:
        dg[j] = float(dr @ Y)
        dY = st(gate[t, j] * dr)
        dH = dY @ W2
        dA = st(dH * b * silu_grad(a))
        dB = st(dH * silu(a))
        dXsum = dXsum + st(dA @ W1 + dB @ W3)
        rows.append((j, dY, dA, dB, H))
    dl_chosen = gate[t] * (dg - (gate[t] * dg).sum())
    dlog = np.zeros(dense["w_router"].shape[0])
    dlog[idx[t].astype(np.int64)] = dl_chosen
    dlog = st(dlog)
    dz = st(dlog @ dense["w_router"] + dXsum)
    dx = dz @ dense["w_lat_down"] + da_s @ dense["ws1"] + db_s @ dense["ws3"]
    return {"dx": dx, "dr": dr, "da_s": da_s, "db_s": db_s, "dlogits": dlog, "dz": dz, "rows": rows}


def _dense_weights(weights):
    return {n: np.asarray(weights[n], np.float64)
            for n in ("w_lat_up", "w_router", "w_lat_down", "ws1", "ws3", "ws2")}


def backward_tokens(dy_rows, weights, rb: dict, tokens, per):
    """dx for the given tokens (rows of dy given for those tokens, in order)."""
    dense = _dense_weights(weights)
    return np.array([_backward_token(dy_rows[n], weights, rb, t, per[n], dense)["dx"]
                     for n, t in enumerate(tokens)])


def sampled_weight_grads(dy_rows, weights, rb: dict, tokens, per):
    """Every weight gradient of the loss sum over the given tokens of y_t . dy_t (the
    upstream gradient is zero on every other token): each gradient is the sum over
    those tokens of its per-token outer products, formed as one matrix product of the
    stacked per-token factors.  Returns the dense gradients as arrays and the routed
    ones as {expert: {"w1", "w3", "w2"}} for the experts those tokens' kept rows reach
    (every other expert's gradient is zero)."""
    dense = _dense_weights(weights)
    x, z, idx = rb["x"], rb["z"], rb["idx"]
    cols = {n: [] for n in ("dy", "r", "H_s", "dlogits", "z", "dz", "x", "da_s", "db_s")}
    rows_of = {}
    for n, t in enumerate(tokens):
        dy = np.asarray(dy_rows[n], np.float64)
        p = per[n]
        b = _backward_token(dy, weights, rb, t, p, dense)
        for key, val in (("dy", dy), ("r", p["r"]), ("H_s", p["H_s"]), ("dlogits", b["dlogits"]), ("z", z[t]),
                         ("dz", b["dz"]), ("x", x[t]), ("da_s", b["da_s"]), ("db_s", b["db_s"])):
            cols[key].append(val)
        for (j, dY, dA, dB, H) in b["rows"]:
            rows_of.setdefault(int(idx[t, j]), []).append((dA, dB, dY, z[t], H))
    m = {key: np.array(v) for key, v in cols.items()}
    g = {"w_lat_up": m["dy"].T @ m["r"], "ws2": m["dy"].T @ m["H_s"], "w_router": m["dlogits"].T @ m["z"],
         "w_lat_down": m["dz"].T @ m["x"], "ws1": m["da_s"].T @ m["x"], "ws3": m["db_s"].T @ m["x"]}
    routed = {}
    for e, rows in rows_of.items():
        dA, dB, dY, X, H = (np.array(c) for c in zip(*rows))
        routed[e] = {"w1": dA.T @ X, "w3": dB.T @ X, "w2": dY.T @ H}
    return g, routed


def shared_weight_grad_rows(x, dy, weights, units, storage="bf16"):
    """Gradients of the shared experts' weights for the hidden units ``units`` (rows of
    ws1 and ws3, columns of ws2) over every token, for the loss sum(y * dy).  The shared
    path does not depend on routing, so this is the whole-batch gradient restricted to
    those units: a_u = x ws1[u]^T, b_u = x ws3[u]^T, H_u = silu(a_u) b_u, dH_u = dy ws2[:, u],
    dws1[u] = (dH_u b_u silu'(a_u))^T x, dws3[u] = (dH_u silu(a_u))^T x, dws2[:, u] = dy^T H_u.
    Returns (dws1 rows [n][d_model], dws3 rows [n][d_model], dws2 columns [d_model][n])."""
    st = _storage(storage)
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    units = np.asarray(units, np.int64)
    ws1 = np.asarray(weights["ws1"][units], np.float64)
    ws3 = np.asarray(weights["ws3"][units], np.float64)
    ws2 = np.asarray(weights["ws2"][:, units], np.float64)
    a, b, H = swiglu_hidden(x, ws1, ws3, st)
    dH = dy @ ws2
    da = st(dH * b * silu_grad(a))
    db = st(dH * silu(a))
    return da.T @ x, db.T @ x, dy.T @ H


def expert_weight_grads(dy, weights, rb: dict, e: int):
    """Gradients of w1[e], w3[e], w2[e] over every row expert e kept."""
    st = _storage(rb["storage"])
    idx, gate, kept, z = rb["idx"], rb["gate"], rb["kept"], rb["z"]
    W_up = np.asarray(weights["w_lat_up"], np.float64)
    tj = [(t, j) for t, j in zip(*np.nonzero((idx == e) & kept))]
    tj.sort(key=lambda p: rb["slots"]["rslot"][p])
    ts = np.array([t for t, _ in tj], dtype=np.int64)
    js = np.array([j for _, j in tj], dtype=np.int64)
    X = z[ts]
    a, b, H, Y, (W1, W3, W2) = _expert_rows(X, weights, e, st)
    dr = st(np.asarray(dy, np.float64)[ts] @ W_up)
    dY = st(gate[ts, js][:, None] * dr)
    dH = dY @ W2
    dA = st(dH * b * silu_grad(a))
    dB = st(dH * silu(a))
    return {"w1": dA.T @ X, "w3": dB.T @ X, "w2": dY.T @ H}
