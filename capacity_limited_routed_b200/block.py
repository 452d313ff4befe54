"""MoEBlock: device buffers of one MoE block around the libmoe C ABI.

PyTorch provides device memory and streams; every step runs in libmoe's kernels.
This class only allocates (weights, forward context, scratch, stats) and calls the
entry points of include/moe.h in order.
"""
from __future__ import annotations

import numpy as np
import torch

from . import moe as M

WEIGHT_NAMES = ("w_lat_down", "w_router", "w1", "w3", "w2", "w_lat_up", "ws1", "ws3", "ws2")


def to_device_bf16(a: np.ndarray, device) -> torch.Tensor:
    """bf16-valued float32 host array -> bf16 device tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device).to(torch.bfloat16)


class MoEBlock:
    def __init__(self, shape, device="cuda", training: bool = False):
        self.shape = shape
        self.device = torch.device(device)
        self.plan = M.Plan.from_shape(shape)
        info = self.plan.info
        self.training = training
        self.ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.saved = (torch.empty(info.saved_bytes, dtype=torch.uint8, device=self.device)
                      if training else None)
        self.stats = torch.zeros(info.stats_bytes // 4, dtype=torch.int32, device=self.device)
        self.weights: dict[str, torch.Tensor] = {}
        self.grads: dict[str, torch.Tensor] = {}
        self.bias = torch.zeros(shape.n_experts, dtype=torch.float32, device=self.device)
        self.logit_offset = None

    # ------------------------------------------------------------------ setup

    def load(self, inputs: dict) -> None:
        """Weights, bias and logit offset from ``synth.make_inputs`` (host arrays, uploaded)
        or ``synth.make_inputs_device`` (device tensors, used as they are)."""
        for n in WEIGHT_NAMES:
            w = inputs["weights"][n]
            self.weights[n] = w if isinstance(w, torch.Tensor) else to_device_bf16(w, self.device)
        b = inputs["bias"]
        self.bias = (b.clone() if isinstance(b, torch.Tensor)
                     else torch.from_numpy(np.asarray(b, np.float32)).to(self.device))
        lo = inputs.get("logit_offset")
        if lo is None:
            self.logit_offset = None
        elif isinstance(lo, torch.Tensor):
            self.logit_offset = lo
        else:
            self.logit_offset = torch.from_numpy(np.asarray(lo, np.float32)).to(self.device)
        if self.training:
            self.grads = {n: torch.empty(self.weights[n].shape, dtype=torch.float32, device=self.device)
                          for n in WEIGHT_NAMES}

    # ------------------------------------------------------------------ steps

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        s = self.shape
        if y is None:
            y = torch.empty((s.T, s.d_model), dtype=torch.float32, device=self.device)
        M.moe_forward(self.plan, self.weights, x, self.bias, self.logit_offset, y, self.stats, self.saved, self.ws,
                      stream)
        return y

    def backward(self, x: torch.Tensor, dy: torch.Tensor, dx: torch.Tensor | None = None, stream=None):
        if not self.training:
            raise RuntimeError("backward needs a block built with training=True")
        s = self.shape
        if dx is None:
            dx = torch.empty((s.T, s.d_model), dtype=torch.float32, device=self.device)
        M.moe_backward(self.plan, self.weights, self.saved, x, dy, dx, self.grads, self.ws, stream)
        return dx

    def bias_update(self, step: float, stream=None) -> None:
        M.moe_bias_update(self.plan, self.hist(), self.bias, step, stream)

    # ------------------------------------------------------------------ views

    def hist(self) -> torch.Tensor:
        return self.stats[8:8 + self.shape.n_experts]

    def stats_dict(self) -> dict:
        s = self.stats.cpu().numpy()
        E = self.shape.n_experts
        NP = self.plan.info.n_pools
        return {
            "kept": int(s[0]), "dropped_sender": int(s[1]), "dropped_receiver": int(s[2]), "status": int(s[3]),
            "max_pool_fill": int(s[4]), "max_expert_fill": int(s[5]), "assignments": int(s[6]),
            "nan_logits": int(s[7]),
            "hist": s[8:8 + E].copy(), "expert_kept": s[8 + E:8 + 2 * E].copy(),
            "expert_dropped_sender": s[8 + 2 * E:8 + 3 * E].copy(),
            "expert_dropped_receiver": s[8 + 3 * E:8 + 4 * E].copy(),
            "pool_fill": s[8 + 4 * E:8 + 4 * E + NP].copy(),
        }

    def saved_views(self) -> dict:
        """Tensors viewing the forward context (needs training=True)."""
        s = self.shape
        v = M.moe_saved_view(self.plan, self.saved)
        base = self.saved.data_ptr()
        Cr = self.plan.info.cap_recv

        def view(ptr, shape, dtype):
            off = ptr - base
            n = int(np.prod(shape))
            return self.saved[off:off + n * torch.tensor([], dtype=dtype).element_size()].view(dtype).view(*shape)

        T, k, E = s.T, s.top_k, s.n_experts
        return {
            "z": view(v["z"], (T, s.d_latent), torch.bfloat16),
            "logits": view(v["logits"], (T, E), torch.float32),
            "topk_idx": view(v["topk_idx"], (T, k), torch.int32),
            "topk_gate": view(v["topk_gate"], (T, k), torch.float32),
            "slot": view(v["slot"], (T, k, 2), torch.int32),
            "expert_rows": view(v["expert_rows"], (E,), torch.int32),
            "expert_in": view(v["expert_in"], (E, Cr, s.d_latent), torch.bfloat16),
            "expert_out": view(v["expert_out"], (E, Cr, s.d_latent), torch.bfloat16),
            "r": view(v["r"], (T, s.d_latent), torch.bfloat16),
        }
