"""Benchmark of the capacity-limited, pooled-wave MoE block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload train|full|mid|skewed|train_dropless|skewed_dropless]
                    [--impl ours|reference]

A step is one pass of the whole hot path on one batch: forward (latent down-projection,
router, top-k, slot assignment, pack, unpack, grouped SwiGLU experts, combine, shared
experts, up-projection), backward (every dgrad and wgrad, combine backward,
un-dispatch, router backward) and the bias step.  The default workload is the
full-width training layer (T=16384, d_model 6144, latent 3072, 384 experts, top-8,
64 destinations x 3 waves, 2 shared experts of 3072).

Prints one JSON line on rank 0.  For N > 1 (torchrun) every rank runs its own
source of T tokens (data-parallel replicas, weak scaling); the only exchange is the
all-reduce of the load histogram before the bias step, which keeps the bias the
same on every replica.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-block tokens/s fwd & fwd+bwd on 1 B200; GEMM % BF16 peak; dispatch % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "_source": "fallback"}


# DRAM bytes (read + write) of the dominant step, from one ncu capture (--set full,
# --clock-control none) of its kernels on the small profiling workload (24 experts,
# T = 1024, same widths and rows per expert), summed over the step's launches.  The
# step's traffic scales with the expert count, so a workload with the same shape per
# expert reports it scaled; it is reported only while the kernel sources hash to the
# captured ones, and as null once they change.
NCU_TRAFFIC = {
    "bwd.experts_wgrad_gate_up": {
        "sources_sha256": "4591362332d8b9b20415fee24dce1562ba2fc3cae0b03bb95434ff18b3dd29df",
        "dram_bytes": 1915889152, "experts": 24, "tokens": 1024, "d_latent": 3072, "hidden_routed": 3072,
    },
}
KERNEL_SOURCES = ("gemm_sm100.cu", "ptx.cuh")  # the GEMM kernels and the PTX they use


def measured_traffic(name, s):
    rec = NCU_TRAFFIC.get(name)
    if rec is None:
        return None
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "capacity_limited_routed_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    if (s.d_latent, s.hidden_routed) != (rec["d_latent"], rec["hidden_routed"]) or \
            s.T * rec["experts"] != rec["tokens"] * s.n_experts:
        return None
    return int(rec["dram_bytes"] * s.n_experts / rec["experts"])


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def workload_shape(name):
    from capacity_limited_routed_b200 import synth
    return {"train": synth.TRAIN, "full": synth.FULL, "mid": synth.MID, "skewed": synth.SKEWED,
            "tiny": synth.TINY.with_(backward=True), "profile": synth.PROFILE,
            "profile_movers": synth.PROFILE_MOVERS,
            "profile_router": synth.PROFILE_ROUTER,
            "profile_router_train": synth.PROFILE_ROUTER_TRAIN,
            "train_dropless": synth.TRAIN_DROPLESS, "skewed_dropless": synth.SKEWED_DROPLESS}[name]


def describe(s):
    return (f"{s.name}: MoE block {'fwd+bwd+bias step' if s.backward else 'forward'}, T={s.T}, "
            f"d_model {s.d_model}, latent {s.d_latent}, E={s.n_experts} top-{s.top_k}, "
            f"D={s.n_dest} x {s.n_waves} waves, "
            + ("dropless (no caps)" if s.dropless else
               f"caps {s.cap_send[0]/s.cap_send[1]:.2f}/{s.cap_recv[0]/s.cap_recv[1]:.2f}")
            + f", {s.n_shared} shared x {s.hidden_shared}"
            + (f", Zipf({s.zipf_s}) logit skew, rho={s.rho} windows of {s.window}" if s.zipf_s else ""))


# ------------------------------------------------------------------ algorithmic work per step


def step_work(s, kept):
    """Algorithmic FLOPs (2 per multiply-add) and HBM bytes of each named step.

    Routed GEMMs count kept rows only."""
    T, dm, dl, E, k, h, SH = s.T, s.d_model, s.d_latent, s.n_experts, s.top_k, s.hidden_routed, s.n_shared * s.hidden_shared
    f = {
        "fwd.lat_down": 2 * T * dm * dl,
        "fwd.router": 2 * T * dl * E,
        "experts.gate_up": 2 * kept * dl * 2 * h,
        "experts.down": 2 * kept * h * dl,
        "fwd.shared_gate_up": 2 * T * dm * 2 * SH,
        "fwd.lat_up_shared_down": 2 * T * dm * (dl + SH),
        "bwd.dr": 2 * T * dm * dl,
        "bwd.shared_dgrad_swiglu": 2 * T * dm * SH,
        "bwd.wgrad_lat_up": 2 * T * dm * dl,
        "bwd.wgrad_shared": 2 * T * dm * 3 * SH,
        "bwd.experts_dgrad_down": 2 * kept * dl * h,
        "bwd.experts_wgrad_down": 2 * kept * dl * h,
        "bwd.experts_dgrad_gate_up": 2 * kept * 2 * h * dl,
        "bwd.experts_wgrad_gate_up": 2 * kept * 2 * h * dl,
        "bwd.router_dgrad": 2 * T * E * dl,
        "bwd.router_wgrad": 2 * T * E * dl,
        "bwd.dx": 2 * T * dm * (dl + 2 * SH),
        "bwd.wgrad_lat_down": 2 * T * dm * dl,
    }
    A = T * k
    w_routed = E * h * dl * 2           # one routed weight tensor, bf16
    b = {
        # GEMMs: operands read once, results written once (bf16 unless noted)
        "fwd.lat_down": T * dm * 2 + dl * dm * 2 + T * dl * 2,
        "fwd.router": T * dl * 2 + E * dl * 2 + T * E * 4,
        "experts.gate_up": 2 * w_routed + kept * dl * 2 + 3 * kept * h * 2,
        "experts.down": w_routed + kept * h * 2 + kept * dl * 2,
        "fwd.shared_gate_up": T * dm * 2 + 2 * SH * dm * 2 + 3 * T * SH * 2,
        "fwd.lat_up_shared_down": T * (dl + SH) * 2 + dm * (dl + SH) * 2 + T * dm * 4,
        "bwd.dr": T * dm * 2 + dm * dl * 2 + T * dl * 2,
        "bwd.shared_dgrad_swiglu": T * dm * 2 + dm * SH * 2 + 4 * T * SH * 2,
        "bwd.wgrad_lat_up": T * dm * 2 + T * dl * 2 + dm * dl * 4,
        "bwd.wgrad_shared": T * dm * 2 + T * SH * 2 + dm * SH * 4 + 2 * T * SH * 2 + T * dm * 2 + 2 * SH * dm * 4,
        "bwd.experts_dgrad_down": kept * dl * 2 + w_routed + 4 * kept * h * 2,
        "bwd.experts_wgrad_down": kept * dl * 2 + kept * h * 2 + E * dl * h * 4,
        "bwd.experts_dgrad_gate_up": 2 * kept * h * 2 + 2 * w_routed + kept * dl * 2,
        "bwd.experts_wgrad_gate_up": 2 * kept * h * 2 + kept * dl * 2 + 2 * E * h * dl * 4,
        "bwd.router_dgrad": T * E * 2 + E * dl * 2 + T * dl * 4 + T * dl * 2,
        "bwd.router_wgrad": T * E * 2 + T * dl * 2 + E * dl * 4,
        "bwd.dx": T * (dl + 2 * SH) * 2 + dm * (dl + 2 * SH) * 2 + T * dm * 4,
        "bwd.wgrad_lat_down": T * dl * 2 + T * dm * 2 + dm * dl * 4,
        # logits read, idx + gate written
        "fwd.route_topk": T * E * 4 + A * 8 + E * 4,
        # z read once, every sender-kept row written with its 16-byte header
        "fwd.dispatch_pack": T * dl * 2 + kept * (dl * 2 + 16),
        # pools read (kept rows + headers), expert rows written
        "experts.unpack": kept * (dl * 2 + 16) + kept * dl * 2,
        # expert rows read, gate + slot read, r written
        "fwd.combine": kept * dl * 2 + A * 12 + T * dl * 2,
        # dr read, Y read, dY written, gate/slot read
        "bwd.combine": T * dl * 2 + 2 * kept * dl * 2 + A * 16,
        # dX read, dz (fp32) and dlogits written
        "bwd.undispatch": kept * dl * 2 + T * dl * 4 + T * E * 2 + A * 16,
        "fwd.slot_scan": A * 4 * 3 + A * 8,
    }
    return f, b


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    def __init__(self, gpu_index, path):
        self.path = path
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(path, "w")
            self.p = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle baseline


def oracle_sample_shape(s, T=256):
    """A bounded sample of the workload for the CPU oracle: T tokens at the full widths
    (every token still runs top-k full-width experts, the shared experts and both latent
    projections), with 24 routed experts (4 destinations x 6) instead of 384 so the
    weights fit the host; per-token work is the same."""
    return s.with_(T=T, n_experts=24, n_dest=4)


def oracle_inputs(s, T=256):
    """The sample's synthetic inputs (drawn once; drawing is not part of a step)."""
    from capacity_limited_routed_b200 import synth
    ss = oracle_sample_shape(s, T).with_(backward=True)
    return ss, synth.make_inputs(ss, seed=123)


def run_oracle_sample(s, ss, inp):
    """One step of the oracle on the sample: forward, and for a training workload the
    backward and the bias step.  Returns (tokens/s, threads used)."""
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    y, ctx = O.forward(inp["x"], inp["weights"], inp["bias"], ss, logit_offset=inp["logit_offset"])
    if s.backward:
        O.backward(inp["dy"], inp["weights"], ctx)
        O.bias_update(ctx["hist"], inp["bias"], 1e-3, ss.T, ss.top_k)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return ss.T / dt, cores


def reference_arm(args, s):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # every step is a bounded sample (64 tokens, a few seconds of host work), so that the
    # whole run of exactly --warmup + --steps steps ends within a few minutes
    steps, warm = max(1, args.steps), max(0, args.warmup)
    ss, inp = oracle_inputs(s, T=64)
    for _ in range(warm):
        run_oracle_sample(s, ss, inp)
    rates = []
    for _ in range(steps):
        r, cores = run_oracle_sample(s, ss, inp)
        rates.append(r)
    v = statistics.median(rates)
    sample = (f"per step {ss.T} tokens at full widths ({ss.d_model}/{ss.d_latent}/{ss.hidden_routed}, "
              f"top-{ss.top_k}, {ss.n_shared} shared), {ss.n_experts} routed experts instead of "
              f"{s.n_experts}; forward{' + backward + bias step' if s.backward else ''}")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": 1000.0 * ss.T / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(s)},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm


def end_to_end(args, s, blk, x, dy, hist_plan, world, dev, barrier):
    """The same steps through the public API with host buffers: every step copies its
    inputs (x, and dy for training) in from pinned host memory and its results (y, and
    dx for training) out to pinned host memory.  The copies run on two copy streams and
    overlap the neighbouring steps' kernels (inputs one step ahead, outputs one step
    behind, double-buffered on the device); the timed region ends when the last step's
    results are on the host."""
    import torch
    from capacity_limited_routed_b200 import moe as M
    from capacity_limited_routed_b200.parallel import global_histogram
    cs = torch.cuda.current_stream(dev)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    x_h = x.cpu().pin_memory()
    dy_h = dy.cpu().pin_memory() if s.backward else None
    y_h = torch.empty((s.T, s.d_model), dtype=torch.float32).pin_memory()
    dx_h = torch.empty((s.T, s.d_model), dtype=torch.float32).pin_memory() if s.backward else None
    xs = [torch.empty_like(x) for _ in range(2)]
    dys = [torch.empty_like(dy) for _ in range(2)] if s.backward else None
    ys = [torch.empty((s.T, s.d_model), dtype=torch.float32, device=dev) for _ in range(2)]
    dxs = [torch.empty((s.T, s.d_model), dtype=torch.float32, device=dev) for _ in range(2)] if s.backward else None
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready = [ev(), ev()]      # inputs of buffer b are on the device
    in_free = [ev(), ev()]       # the step that used buffer b no longer reads its inputs
    out_ready = [ev(), ev()]     # results of buffer b are written
    out_free = [ev(), ev()]      # results of buffer b are on the host
    # one GPU: each buffer's step (forward, backward, bias step) is captured once into a
    # CUDA graph and replayed between the copy events, as in the device-resident timing
    graphs = None
    if world == 1 and not args.no_graph:
        graphs = []
        for b in range(2):
            xs[b].copy_(x)
            if s.backward:
                dys[b].copy_(dy)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                blk.forward(xs[b], y=ys[b])
                if s.backward:
                    blk.backward(xs[b], dys[b], dx=dxs[b])
                    M.moe_bias_update(hist_plan, blk.hist(), blk.bias, 1e-3)
            g.replay()
            graphs.append(g)
        torch.cuda.synchronize()
    for b in range(2):
        in_free[b].record(cs)
        out_free[b].record(cs)

    def load(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            h2d.wait_event(in_free[b])
            xs[b].copy_(x_h, non_blocking=True)
            if s.backward:
                dys[b].copy_(dy_h, non_blocking=True)
            in_ready[b].record(h2d)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(cs)
    h2d.wait_event(e0)
    d2h.wait_event(e0)
    load(0)
    for i in range(args.steps):
        b = i % 2
        if i + 1 < args.steps:
            load(i + 1)
        cs.wait_event(in_ready[b])
        cs.wait_event(out_free[b])
        if graphs is not None:
            graphs[b].replay()
        else:
            blk.forward(xs[b], y=ys[b])
            if s.backward:
                blk.backward(xs[b], dys[b], dx=dxs[b])
                global_histogram(blk.hist())
                M.moe_bias_update(hist_plan, blk.hist(), blk.bias, 1e-3)
        in_free[b].record(cs)
        out_ready[b].record(cs)
        with torch.cuda.stream(d2h):
            d2h.wait_event(out_ready[b])
            y_h.copy_(ys[b], non_blocking=True)
            if s.backward:
                dx_h.copy_(dxs[b], non_blocking=True)
            out_free[b].record(d2h)
    cs.wait_stream(d2h)
    e1.record(cs)
    torch.cuda.synchronize()
    barrier()
    e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
    e_step = float(e_ms.item()) / args.steps
    if not bool(torch.isfinite(y_h[:: max(1, s.T // 64)]).all()):
        raise RuntimeError("end-to-end: non-finite y on the host")
    h2d_b = x.numel() * 2 + (dy.numel() * 2 if s.backward else 0)
    d2h_b = y_h.numel() * 4 + (dx_h.numel() * 4 if s.backward else 0)
    return {"value": world * s.T / (e_step * 1e-3), "unit": "tokens/s", "ms_per_step": e_step,
            "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
            "copies": "x, dy in from pinned host; y, dx out to pinned host, every step "
                      "(two copy streams, overlapping the neighbouring steps)",
            "cuda_graph": graphs is not None}


def drop_sweep(weights, dev):
    """Drop fraction against context length and capacity factor, on the device: router
    path only (latent projection, router, top-k, slot assignment, pack) for one source of
    T = 65,536 tokens at full width, uniform router, bias 0.  The tokens of one sequence of
    L tokens share a component (x_t = sqrt(0.6) g_seq + sqrt(0.4) eps_t): L = 512 is the
    skewed workload's windows, L = T one sequence per source; "independent" has none.
    Capacity factors 1.10/1.15 (the pages'), 1.25/1.30, and dropless (no cap: its largest
    expert load is reported instead)."""
    import torch
    from capacity_limited_routed_b200 import moe as M
    from capacity_limited_routed_b200 import synth
    T, s0 = 65536, synth.FULL
    out = {"tokens_per_source": T, "rho": 0.6, "rows": []}
    dl, E, k = s0.d_latent, s0.n_experts, s0.top_k
    z = torch.empty((T, dl), dtype=torch.bfloat16, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    bias = torch.zeros(E, dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    hist = torch.empty(E, dtype=torch.int32, device=dev)
    for L in (0, 512, 4096, 16384, 65536):
        shape = s0.with_(T=T, window=L, rho=0.6 if L else 0.0, seed=31)
        x = synth.make_tokens_device(shape, device=dev)["x"]
        M.moe_gemm_bf16(T, dl, s0.d_model, x, 0, weights["w_lat_down"], 0, z)
        M.moe_gemm_bf16(T, E, dl, z, 0, weights["w_router"], 0, logits)
        del x
        row = {"sequence_tokens": L or "independent"}
        for name, cs, cr in (("caps_1.10_1.15", (110, 100), (115, 100)), ("caps_1.25_1.30", (125, 100), (130, 100))):
            plan = M.Plan(T, s0.d_model, dl, E, k, s0.n_dest, s0.hidden_routed, s0.n_shared, s0.hidden_shared,
                          cap_send=cs, cap_recv=cr)
            info = plan.info
            M.moe_route(plan, logits, bias, idx, gate, hist)
            pools = torch.empty(info.pools_bytes // 2, dtype=torch.int16, device=dev)
            slot = torch.empty((T, k, 2), dtype=torch.int32, device=dev)
            stats = torch.zeros(info.stats_bytes // 4, dtype=torch.int32, device=dev)
            ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=dev)
            M.moe_dispatch(plan, z, idx, pools, slot, stats, ws)
            st = stats[:4].cpu().tolist()
            if st[3] != 0:
                raise RuntimeError(f"kernel status {st[3]} in the drop sweep")
            row[name] = {"sender": st[1] / (T * k), "receiver": st[2] / (T * k)}
            del pools, slot, stats, ws
        h = hist.cpu().numpy()
        row["dropless_largest_expert_load"] = int(h.max())
        row["mean_expert_load"] = T * k / E
        out["rows"].append(row)
    out["note"] = ("synthetic latent correlations with an untrained router; the pages' 7% (4K) -> 40% (65K) "
                   "comes from a trained router on real text and is not reproduced, only the direction")
    return out


def forward_pass(shape, weights, dev, steps, warmup):
    """Forward-only throughput of a full-width workload on weights already on the device
    (same widths): CUDA events around `steps` forward passes after `warmup` of them."""
    import torch
    from capacity_limited_routed_b200 import synth
    from capacity_limited_routed_b200.block import MoEBlock
    inp = synth.make_tokens_device(shape, device=dev)
    inp["weights"] = weights
    blk = MoEBlock(shape, device=dev, training=False)
    blk.load(inp)
    x = inp["x"]
    y = torch.empty((shape.T, shape.d_model), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        blk.forward(x, y=y)
    st = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(steps):
        blk.forward(x, y=y)
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    sd = blk.stats_dict()
    if sd["status"] != 0:
        raise RuntimeError(f"kernel status {sd['status']} in the {shape.name} forward pass")
    A = shape.T * shape.top_k
    out = {"tokens_per_s": shape.T / (ms * 1e-3), "ms_per_step": ms, "steps": steps, "warmup": warmup,
           "workload": describe(shape), "kept": sd["kept"],
           "drop_fraction": {"sender": sd["dropped_sender"] / A, "receiver": sd["dropped_receiver"] / A}}
    del blk, inp, x, y
    return out



def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="train")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-only", action="store_true", help="a few steps, no baseline, no e2e (for ncu)")
    ap.add_argument("--parallelism", default="auto", choices=["auto", "ep", "replicas"],
                    help="N > 1: expert parallelism (each rank one source and the receiver of D/N destinations, "
                         "blocks exchanged over NCCL) or data-parallel replicas; auto = ep when D divides by N")
    ap.add_argument("--no-forward-passes", action="store_true",
                    help="skip the forward-only passes of the full and skewed workloads")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying a CUDA graph of one step")
    args = ap.parse_args()
    s = workload_shape(args.workload)
    if args.impl == "reference":
        reference_arm(args, s)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    from capacity_limited_routed_b200 import moe as M
    from capacity_limited_routed_b200 import synth
    from capacity_limited_routed_b200.block import MoEBlock
    from capacity_limited_routed_b200.parallel import global_histogram, global_tokens

    peaks = load_peaks()
    mode = args.parallelism
    if mode == "auto":
        mode = "ep" if world > 1 and s.n_dest % world == 0 and not s.dropless else "replicas"
    if mode == "ep" and world < 2:
        mode = "replicas"
    if mode == "ep":
        # the same weights on every rank (one seed), each rank its own tokens
        from capacity_limited_routed_b200.parallel import EPBlock
        inp = synth.make_inputs_device(s, device=dev, seed=s.seed)
        tok = synth.make_tokens_device(s, device=dev, seed=s.seed + 7919 * rank)
        inp.update({k_: v_ for k_, v_ in tok.items() if k_ in ("x", "dy")})
        blk = EPBlock(s, world, rank, device=dev)
        blk.load(inp["weights"], inp["bias"], inp["logit_offset"], training=s.backward)
        del inp["weights"]
    else:
        inp = synth.make_inputs_device(s, device=dev, seed=s.seed + 7919 * rank)
        blk = MoEBlock(s, device=dev, training=s.backward)
        blk.load(inp)
    x, dy = inp["x"], inp.get("dy")
    hist_plan = M.Plan.from_shape(s.with_(T=global_tokens(s.T))) if world > 1 else blk.plan
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)

    def step():
        blk.forward(x)
        if s.backward:
            blk.backward(x, dy)
            global_histogram(blk.hist())
            M.moe_bias_update(hist_plan, blk.hist(), blk.bias, 1e-3)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    st0 = blk.stats_dict()
    if st0["status"] != 0:
        raise RuntimeError(f"kernel status {st0['status']} after warm-up")

    # One GPU: the step (its launches, side-stream fork and join, the bias step) is captured
    # once into a CUDA graph and replayed; the library allocates nothing and never syncs
    # inside a step, so the graph holds exactly the eager launches.  The launch count is
    # taken at capture, per step.
    graph, graph_launches = None, 0
    if world == 1 and not args.no_graph:
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        l0 = M.moe_kernel_launches()
        with torch.cuda.graph(graph):
            step()
        graph_launches = M.moe_kernel_launches() - l0
        graph.replay()  # one untimed replay
        torch.cuda.synchronize()
        st0 = blk.stats_dict()
        if st0["status"] != 0:
            raise RuntimeError(f"kernel status {st0['status']} after the graph's first replay")

    # ---------------- timed region: K steps, device-resident inputs
    # the raw clock samples go to MOE_BENCH_CLOCKS_DIR (default: the system temp directory)
    clocks_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
    clocks = ClockSampler(local, os.path.join(clocks_dir, f"clocks_rank{rank}.csv"))
    launches0 = M.moe_kernel_launches()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = (M.moe_kernel_launches() - launches0) if graph is None else graph_launches * args.steps
    ms = ev0.elapsed_time(ev1)
    # the same K steps again, launched one by one with the library's per-step CUDA events on
    # (two events around each named step cost ~1.3% of the step, so they stay out of the
    # region above) and every step in order on one stream (so no step's event time includes
    # another's): the per-kernel table and the roofline come from this second timed region
    M.moe_set_side_stream(False)  # each step's event time its own: the shared experts in order
    M.moe_profile_start()
    ev2 = torch.cuda.Event(enable_timing=True)
    ev3 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev2.record(stream)
    for _ in range(args.steps):
        step()
    ev3.record(stream)
    torch.cuda.synchronize()
    barrier()
    prof = M.moe_profile_stop()
    M.moe_set_side_stream(True)
    ms_prof = ev2.elapsed_time(ev3)
    clk = clocks.stop()
    ms_t = torch.tensor([ms, ms_prof], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max, ms_prof_max = float(ms_t[0].item()), float(ms_t[1].item())
    st = blk.stats_dict()
    if st["status"] != 0:
        raise RuntimeError(f"kernel status {st['status']} in the timed region")

    # per-step timing from the library's events (same stream, same timed region)
    per = {}
    for name, t, n in prof:
        d = per.setdefault(name, [0.0, 0, 0])
        d[0] += t
        d[1] += 1
        d[2] += n
    if mode == "ep":
        # rows kept by this rank's experts, and the step's drops summed over ranks
        agg = torch.tensor([st["kept_here"], st["dropped_sender"]], dtype=torch.int64, device=dev)
        dist.all_reduce(agg)
        kept_all, ds_all = int(agg[0].item()), int(agg[1].item())
        st = dict(st, kept=kept_all // world, dropped_sender=ds_all / world,
                  dropped_receiver=(world * s.T * s.top_k - kept_all - ds_all) / world)
    kept = st["kept"]
    flops, bytes_ = step_work(s, kept)
    tc_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    # each step against the roofline that binds it: the larger of its tensor time at
    # the sustained bf16 peak and its HBM time at the copy bandwidth
    hbm = peaks["hbm_gbs"]
    kernels = {}
    for name, (tot, cnt, nl) in per.items():
        avg = tot / args.steps  # per step (a step may launch a name more than once, e.g. per wave)
        e = {"ms": round(avg, 4), "share": round(tot / sum(v[0] for v in per.values()), 4)}
        t_tc = flops[name] / (tc_peak * 1e12) if name in flops else 0.0
        t_mem = bytes_[name] / (hbm * 1e9) if name in bytes_ else 0.0
        if name in flops:
            e["tflops"] = round(flops[name] / (avg * 1e-3) / 1e12, 1)
        if name in bytes_:
            e["gbs"] = round(bytes_[name] / (avg * 1e-3) / 1e9, 1)
        if t_tc or t_mem:
            e["bound"] = "tensor" if t_tc >= t_mem else "hbm"
            e["frac"] = round(max(t_tc, t_mem) / (avg * 1e-3), 3)
        kernels[name] = e
    top = max(per.items(), key=lambda kv: kv[1][0])[0]
    kt = kernels[top]
    per_step = per[top][1] / args.steps  # records of the top step per training step (waves: 3)
    traffic = measured_traffic(top, s)
    if kt.get("bound") == "tensor":
        roof = {"kernel": top, "bound": "tensor", "achieved": kt["tflops"], "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(kt["tflops"] / tc_peak, 3), "traffic": traffic,
                "peak_kind": f"bf16_tflops_sustained ({peaks['_source']}): kernel timed inside a long step",
                "flops_per_launch": flops[top] / per_step, "launches_per_step": per_step}
    else:
        roof = {"kernel": top, "bound": "hbm", "achieved": kt.get("gbs"), "peak": hbm,
                "unit": "GB/s", "frac": round((kt.get("gbs") or 0) / hbm, 3), "traffic": traffic,
                "peak_kind": f"hbm_gbs ({peaks['_source']})", "bytes_per_launch": bytes_.get(top, 0) / per_step,
                "launches_per_step": per_step}
    fwd_ms = sum(v[0] for k_, v in per.items() if k_.startswith("fwd.") or k_.startswith("experts.")) / args.steps
    step_ms = ms_max / args.steps
    value = world * s.T / (step_ms * 1e-3)

    # ---------------- end to end through the public API, host buffers
    e2e = None
    if not args.profile_only:
        e2e = end_to_end(args, s, blk, x, dy, hist_plan, world, dev, barrier)

    # ---------------- forward-only passes of the full-width layer and the skewed stress
    fwd_extra = {}
    if not args.profile_only and not args.no_forward_passes and world == 1 and \
            (s.d_model, s.d_latent, s.n_experts, s.hidden_routed) == (6144, 3072, 384, 3072):
        for name, shape in (("fwd_full", synth.FULL), ("fwd_skewed", synth.SKEWED)):
            fwd_extra[name] = forward_pass(shape, blk.weights, dev, args.steps, max(args.warmup, 3))
        fwd_extra["drop_sweep"] = drop_sweep(blk.weights, dev)
        torch.cuda.synchronize()

    # ---------------- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile_only:
        ss, oinp = oracle_inputs(s, T=256)
        r, cores = run_oracle_sample(s, ss, oinp)
        del oinp
        cpu = {"value": r, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{ss.T} tokens of this workload at full widths with {ss.n_experts} routed experts "
                         f"instead of {s.n_experts} (same per-token work), one pass, float64 numpy"}

    if rank == 0:
        A = s.T * s.top_k
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": describe(s),
                       "parallelism": (f"expert parallelism x{world} (each GPU one source of T tokens and the "
                                       f"receiver of {s.n_dest // world} destinations; fixed-shape blocks per wave "
                                       f"over NCCL)" if mode == "ep" else
                                       f"replicas x{world} (one source per GPU)"),
                       "l2": "inputs larger than L2 (22 GB of expert weights streamed every step)"},
            "fwd_tokens_per_s": world * s.T / (fwd_ms * 1e-3) if fwd_ms > 0 else None,
            "fwd_tokens_per_s_kind": "sum of the forward steps' CUDA-event times inside the profiled timed steps",
            **fwd_extra,
            "drop_fraction": {"sender": st["dropped_sender"] / A, "receiver": st["dropped_receiver"] / A},
            "roofline": roof,
            "dispatch_hbm_frac": kernels.get("fwd.dispatch_pack", {}).get("frac"),
            "kernels": kernels,
            "kernels_note": ("per training step, from a second timed region of the same K steps launched one "
                             "by one with the library's per-step CUDA events on and every step in order on one "
                             "stream (ms_per_step_profiled); the region that gives value replays a CUDA graph "
                             "with the shared experts on a second stream beside the routing and movement "
                             "kernels and no per-step events"),
            "ms_per_step_profiled": ms_prof_max / args.steps,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "cuda_graph": (f"timed steps replay one CUDA graph of the step ({graph_launches} kernel launches "
                           f"captured); the profiled region runs the steps eagerly") if graph is not None else None,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
