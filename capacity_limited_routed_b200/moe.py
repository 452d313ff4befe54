"""Python binding of libmoe: the C ABI in include/moe.h, one function per entry point.

Argument marshalling only.  Tensors are PyTorch CUDA tensors (device memory and
streams come from PyTorch); every step of the block runs in libmoe's kernels.  If
the library is missing the import fails loudly: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

# the symbols include/moe.h declares
EXPORTS = (
    "moe_plan_create", "moe_plan_destroy", "moe_plan_info", "moe_route", "moe_dispatch", "moe_dispatch_noalloc",
    "moe_expert_ffn", "moe_combine", "moe_forward", "moe_backward", "moe_bias_update",
    "moe_saved_view", "moe_gemm_bf16", "moe_profile_start", "moe_profile_stop", "moe_kernel_launches",
    "moe_set_side_stream",
    "moe_last_error", "moe_ep_view", "moe_ep_forward_send", "moe_ep_forward_experts", "moe_ep_forward_combine",
    "moe_ep_backward_send", "moe_ep_backward_experts", "moe_ep_backward_finish",
)

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}: {msg}")
        self.code = code


class moe_config_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "T", "d_model", "d_latent", "n_experts", "top_k", "n_dest", "n_waves", "hidden_routed",
        "n_shared", "hidden_shared", "cap_send_num", "cap_send_den", "cap_recv_num", "cap_recv_den",
        "n_sources", "ep_ranks", "ep_rank")]


class moe_plan_info_t(ctypes.Structure):
    _fields_ = [("local_experts", ctypes.c_int32), ("experts_per_wave", ctypes.c_int32),
                ("n_pools", ctypes.c_int32), ("cap_send", ctypes.c_int32), ("cap_recv", ctypes.c_int32),
                ("pool_row_elems", ctypes.c_int32), ("pools_bytes", ctypes.c_uint64),
                ("expert_out_bytes", ctypes.c_uint64), ("slot_bytes", ctypes.c_uint64),
                ("stats_bytes", ctypes.c_uint64), ("saved_bytes", ctypes.c_uint64),
                ("workspace_bytes", ctypes.c_uint64)]


_W = ("w_lat_down", "w_router", "w1", "w3", "w2", "w_lat_up", "ws1", "ws3", "ws2")


class moe_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _W]


class moe_grads_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _W]


class moe_expert_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w1", "w3", "w2")]


class moe_profile_record_t(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("ms", ctypes.c_float), ("launches", ctypes.c_int32)]


class moe_saved_view_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "z", "logits", "topk_idx", "topk_gate", "slot", "expert_rows", "expert_in", "expert_out", "r")]


class moe_ep_view_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("ranks", "rank", "dest_per_rank", "n_waves", "cap_send",
                                                "pool_row_elems", "row_elems")] + \
               [(n, ctypes.c_void_p) for n in ("send_pools", "recv_pools", "y_send", "y_recv", "dy_send", "dy_recv",
                                                "dx_send", "dx_recv", "expert_rows", "topk_idx", "slot")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run "
                          "`python -m capacity_limited_routed_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, U, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t
    sig = {
        "moe_plan_create": [ctypes.POINTER(moe_config_t), ctypes.POINTER(P)],
        "moe_plan_destroy": [P],
        "moe_plan_info": [P, ctypes.POINTER(moe_plan_info_t)],
        "moe_route": [P, P, P, P, P, P, P],
        "moe_dispatch": [P, P, P, P, P, P, P, S, P],
        "moe_dispatch_noalloc": [P, P, P, P, P, P, P],
        "moe_expert_ffn": [P, ctypes.POINTER(moe_expert_weights_t), P, P, P, P, S, P],
        "moe_combine": [P, P, P, P, P, P, P],
        "moe_forward": [P, ctypes.POINTER(moe_weights_t), P, P, P, P, P, P, P, S, P],
        "moe_backward": [P, ctypes.POINTER(moe_weights_t), P, P, P, P, ctypes.POINTER(moe_grads_t), P, S, P],
        "moe_bias_update": [P, P, P, ctypes.c_float, P],
        "moe_saved_view": [P, P, ctypes.POINTER(moe_saved_view_t)],
        "moe_gemm_bf16": [I, I, I, P, I, P, I, P, I, P, P],
        "moe_profile_start": [],
        "moe_set_side_stream": [I],
        "moe_profile_stop": [ctypes.POINTER(moe_profile_record_t), I, ctypes.POINTER(I)],
        "moe_ep_view": [P, P, P, ctypes.POINTER(moe_ep_view_t)],
        "moe_ep_forward_send": [P, ctypes.POINTER(moe_weights_t), P, P, P, P, P, P, S, P],
        "moe_ep_forward_experts": [P, ctypes.POINTER(moe_expert_weights_t), P, P, P, S, P],
        "moe_ep_forward_combine": [P, ctypes.POINTER(moe_weights_t), P, P, P, S, P],
        "moe_ep_backward_send": [P, ctypes.POINTER(moe_weights_t), P, P, P, ctypes.POINTER(moe_grads_t), P, S, P],
        "moe_ep_backward_experts": [P, ctypes.POINTER(moe_expert_weights_t), P, ctypes.POINTER(moe_grads_t), P, S,
                                    P],
        "moe_ep_backward_finish": [P, ctypes.POINTER(moe_weights_t), P, P, P, ctypes.POINTER(moe_grads_t), P, S, P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.moe_kernel_launches.argtypes = []
    lib.moe_kernel_launches.restype = ctypes.c_int64
    lib.moe_last_error.argtypes = []
    lib.moe_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise MoEError(code, where, _lib.moe_last_error().decode(errors="replace"))


def _ptr(t):
    """Device pointer of a tensor (or None)."""
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class PlanInfo:
    local_experts: int
    experts_per_wave: int
    n_pools: int
    cap_send: int
    cap_recv: int
    pool_row_elems: int
    pools_bytes: int
    expert_out_bytes: int
    slot_bytes: int
    stats_bytes: int
    saved_bytes: int
    workspace_bytes: int


class Plan:
    """Owns a moe_plan_t for one block shape."""

    def __init__(self, T, d_model, d_latent, n_experts, top_k, n_dest, hidden_routed, n_shared, hidden_shared,
                 n_waves=3, cap_send=(110, 100), cap_recv=(115, 100), n_sources=1, ep_ranks=0, ep_rank=0):
        self.cfg = moe_config_t(T, d_model, d_latent, n_experts, top_k, n_dest, n_waves, hidden_routed,
                                n_shared, hidden_shared, cap_send[0], cap_send[1], cap_recv[0], cap_recv[1],
                                n_sources, ep_ranks, ep_rank)
        h = ctypes.c_void_p()
        _check(_lib.moe_plan_create(ctypes.byref(self.cfg), ctypes.byref(h)), "moe_plan_create")
        self.handle = h
        info = moe_plan_info_t()
        _check(_lib.moe_plan_info(self.handle, ctypes.byref(info)), "moe_plan_info")
        self.info = PlanInfo(**{f: getattr(info, f) for f, _ in moe_plan_info_t._fields_})

    @classmethod
    def from_shape(cls, s, ep_ranks=0, ep_rank=0):
        # both capacity numerators 0 select the dropless variant
        cap_send, cap_recv = ((0, 1), (0, 1)) if getattr(s, "dropless", False) else (s.cap_send, s.cap_recv)
        return cls(s.T, s.d_model, s.d_latent, s.n_experts, s.top_k, s.n_dest, s.hidden_routed, s.n_shared,
                   s.hidden_shared, s.n_waves, cap_send, cap_recv, getattr(s, "n_sources", 1), ep_ranks, ep_rank)

    def __del__(self):
        # at interpreter shutdown the module globals may already be gone
        h = getattr(self, "handle", None)
        lib_ = globals().get("_lib")
        if h is not None and h.value and lib_ is not None:
            lib_.moe_plan_destroy(h)
            self.handle = None


def weights_struct(w: dict) -> moe_weights_t:
    return moe_weights_t(*[_ptr(w[n]) for n in _W])


def grads_struct(g: dict) -> moe_grads_t:
    return moe_grads_t(*[_ptr(g[n]) for n in _W])


# ------------------------------------------------------------------ entry points


def moe_route(plan: Plan, logits, bias, topk_idx, topk_gate, hist, stream=None):
    _check(_lib.moe_route(plan.handle, _ptr(logits), _ptr(bias), _ptr(topk_idx), _ptr(topk_gate), _ptr(hist),
                          _stream(stream)), "moe_route")


def moe_dispatch(plan: Plan, z, topk_idx, pools, slot, stats, ws, stream=None):
    _check(_lib.moe_dispatch(plan.handle, _ptr(z), _ptr(topk_idx), _ptr(pools), _ptr(slot), _ptr(stats), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "moe_dispatch")


def moe_dispatch_noalloc(plan: Plan, z, topk_idx, pools, slot, stats, stream=None):
    """moe_dispatch without a workspace (scan scratch in the library's static array)."""
    _check(_lib.moe_dispatch_noalloc(plan.handle, _ptr(z), _ptr(topk_idx), _ptr(pools), _ptr(slot), _ptr(stats),
                                     _stream(stream)), "moe_dispatch_noalloc")


def moe_expert_ffn(plan: Plan, w1, w3, w2, pools, expert_out, expert_rows, ws, stream=None):
    ew = moe_expert_weights_t(_ptr(w1), _ptr(w3), _ptr(w2))
    _check(_lib.moe_expert_ffn(plan.handle, ctypes.byref(ew), _ptr(pools), _ptr(expert_out), _ptr(expert_rows),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_expert_ffn")


def moe_combine(plan: Plan, expert_out, topk_gate, topk_idx, slot, r, stream=None):
    _check(_lib.moe_combine(plan.handle, _ptr(expert_out), _ptr(topk_gate), _ptr(topk_idx), _ptr(slot), _ptr(r),
                            _stream(stream)), "moe_combine")


def moe_forward(plan: Plan, weights: dict, x, bias, logit_offset, y, stats, saved, ws, stream=None):
    ws_ = weights_struct(weights)
    _check(_lib.moe_forward(plan.handle, ctypes.byref(ws_), _ptr(x), _ptr(bias), _ptr(logit_offset), _ptr(y),
                            _ptr(stats), _ptr(saved), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_forward")


def moe_backward(plan: Plan, weights: dict, saved, x, dy, dx, grads: dict, ws, stream=None):
    w_ = weights_struct(weights)
    g_ = grads_struct(grads)
    _check(_lib.moe_backward(plan.handle, ctypes.byref(w_), _ptr(saved), _ptr(x), _ptr(dy), _ptr(dx),
                             ctypes.byref(g_), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_backward")


def moe_bias_update(plan: Plan, hist, bias, step: float, stream=None):
    _check(_lib.moe_bias_update(plan.handle, _ptr(hist), _ptr(bias), ctypes.c_float(step), _stream(stream)),
           "moe_bias_update")


def moe_saved_view(plan: Plan, saved) -> dict:
    v = moe_saved_view_t()
    _check(_lib.moe_saved_view(plan.handle, _ptr(saved), ctypes.byref(v)), "moe_saved_view")
    return {f: getattr(v, f) for f, _ in moe_saved_view_t._fields_}


def moe_gemm_bf16(M, N, K, A, a_mn_major, B, b_mn_major, D, status=None, stream=None):
    import torch
    d_f32 = 1 if D.dtype == torch.float32 else 0
    _check(_lib.moe_gemm_bf16(M, N, K, _ptr(A), int(a_mn_major), _ptr(B), int(b_mn_major), _ptr(D), d_f32,
                              _ptr(status), _stream(stream)), "moe_gemm_bf16")


def moe_profile_start():
    _check(_lib.moe_profile_start(), "moe_profile_start")


def moe_profile_stop(cap: int = 65536) -> list[tuple[str, float, int]]:
    """Per-step (name, milliseconds, kernel launches) since moe_profile_start."""
    buf = (moe_profile_record_t * cap)()
    n = ctypes.c_int32(0)
    _check(_lib.moe_profile_stop(buf, cap, ctypes.byref(n)), "moe_profile_stop")
    return [(buf[i].name.decode(), float(buf[i].ms), int(buf[i].launches)) for i in range(min(n.value, cap))]


def moe_set_side_stream(enable: bool) -> None:
    """Shared experts on the library's second stream (True, the default) or in order on
    the caller's stream (False)."""
    _check(_lib.moe_set_side_stream(1 if enable else 0), "moe_set_side_stream")


def moe_kernel_launches() -> int:
    return int(_lib.moe_kernel_launches())


def moe_last_error() -> str:
    return _lib.moe_last_error().decode(errors="replace")


# ------------------------------------------------------------------ expert parallelism


def _nbytes(t):
    return t.numel() * t.element_size()


def _grads_or_null(g: dict) -> moe_grads_t:
    return moe_grads_t(*[_ptr(g.get(n)) for n in _W])


def moe_ep_view(plan: Plan, saved, ws) -> moe_ep_view_t:
    v = moe_ep_view_t()
    _check(_lib.moe_ep_view(plan.handle, _ptr(saved), _ptr(ws), ctypes.byref(v)), "moe_ep_view")
    return v


def moe_ep_forward_send(plan: Plan, weights: dict, x, bias, logit_offset, stats, saved, ws, stream=None):
    w_ = weights_struct(weights)
    _check(_lib.moe_ep_forward_send(plan.handle, ctypes.byref(w_), _ptr(x), _ptr(bias), _ptr(logit_offset),
                                    _ptr(stats), _ptr(saved), _ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_ep_forward_send")


def moe_ep_forward_experts(plan: Plan, w1, w3, w2, stats, saved, ws, stream=None):
    ew = moe_expert_weights_t(_ptr(w1), _ptr(w3), _ptr(w2))
    _check(_lib.moe_ep_forward_experts(plan.handle, ctypes.byref(ew), _ptr(stats), _ptr(saved), _ptr(ws),
                                       _nbytes(ws), _stream(stream)), "moe_ep_forward_experts")


def moe_ep_forward_combine(plan: Plan, weights: dict, y, saved, ws, stream=None):
    w_ = weights_struct(weights)
    _check(_lib.moe_ep_forward_combine(plan.handle, ctypes.byref(w_), _ptr(y), _ptr(saved), _ptr(ws), _nbytes(ws),
                                       _stream(stream)), "moe_ep_forward_combine")


def moe_ep_backward_send(plan: Plan, weights: dict, saved, x, dy, grads: dict, ws, stream=None):
    w_ = weights_struct(weights)
    g_ = _grads_or_null(grads)
    _check(_lib.moe_ep_backward_send(plan.handle, ctypes.byref(w_), _ptr(saved), _ptr(x), _ptr(dy), ctypes.byref(g_),
                                     _ptr(ws), _nbytes(ws), _stream(stream)), "moe_ep_backward_send")


def moe_ep_backward_experts(plan: Plan, w1, w3, w2, saved, grads: dict, ws, stream=None):
    ew = moe_expert_weights_t(_ptr(w1), _ptr(w3), _ptr(w2))
    g_ = _grads_or_null(grads)
    _check(_lib.moe_ep_backward_experts(plan.handle, ctypes.byref(ew), _ptr(saved), ctypes.byref(g_), _ptr(ws),
                                        _nbytes(ws), _stream(stream)), "moe_ep_backward_experts")


def moe_ep_backward_finish(plan: Plan, weights: dict, saved, x, dx, grads: dict, ws, stream=None):
    w_ = weights_struct(weights)
    g_ = _grads_or_null(grads)
    _check(_lib.moe_ep_backward_finish(plan.handle, ctypes.byref(w_), _ptr(saved), _ptr(x), _ptr(dx),
                                       ctypes.byref(g_), _ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_ep_backward_finish")
