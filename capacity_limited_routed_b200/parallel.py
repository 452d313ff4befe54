"""Multi-GPU forms of the MoE block: data-parallel replicas and expert parallelism.

Replicas.  Each GPU is one source with its own T tokens (its own slots, caps and drops).
The bias step must see the load of the whole step so that every replica keeps the same
bias: the per-expert selection histograms are summed over ranks (int32, exact) and the
step uses the total token count.  Nothing else crosses ranks on the block's data path.

Expert parallelism (the pages' transport: "Marin начинает открытое обучение MoE-модели с
535 млрд параметров", §2; "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §3.1-3.2).
Every rank is one source of T tokens and the receiver of D/G destinations.  The pools
travel as fixed-shape blocks, one exchange per wave, with no count or metadata exchange;
expert outputs and gradients travel back the same way.  The block layout and the order
of the six library calls are those of include/moe.h; this module only moves blocks
(torch.distributed point-to-point, NCCL on GPUs) and sequences the calls.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe as M


def global_histogram(hist: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the int32 [E] selection histogram over the ranks of ``group`` (in place)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(hist, op=dist.ReduceOp.SUM, group=group)
    return hist


def global_tokens(T_local: int, group=None) -> int:
    """Tokens of the whole step (every replica holds the same T)."""
    if dist.is_available() and dist.is_initialized():
        return T_local * dist.get_world_size(group)
    return T_local


# ------------------------------------------------------------------ expert parallelism


class BlockSchedule:
    """Where the blocks of an expert-parallel exchange go.

    Every exchange buffer holds D*W blocks of C_s rows; block b = (a * Dl + d) * W + w
    for peer a, local destination d < Dl = D/G and wave w.  In every exchange a rank
    sends block b of its send buffer to peer a and receives block b of its receive
    buffer from peer a."""

    def __init__(self, ranks: int, rank: int, dest_per_rank: int, n_waves: int, cap_send: int):
        self.G, self.rank, self.Dl, self.W, self.Cs = ranks, rank, dest_per_rank, n_waves, cap_send

    @property
    def n_blocks(self) -> int:
        return self.G * self.Dl * self.W

    def block(self, peer: int, d: int, w: int) -> int:
        return (peer * self.Dl + d) * self.W + w

    def rows(self, b: int) -> slice:
        return slice(b * self.Cs, (b + 1) * self.Cs)

    def wave_blocks(self, w: int):
        """(peer, block) pairs of wave w, peers in rank order, local destinations in order."""
        return [(a, self.block(a, d, w)) for a in range(self.G) for d in range(self.Dl)]


def exchange(sched: BlockSchedule, send: torch.Tensor, recv: torch.Tensor, group=None) -> None:
    """One exchange, wave by wave: block b of ``send`` to peer a, block b of ``recv`` from
    peer a (a rank's own blocks are copied locally).  ``send`` and ``recv`` are 2-D
    [D*W*C_s][row] tensors.  Sends and receives between a pair of ranks are posted in the
    same order on both sides, so they match one to one."""
    for w in range(sched.W):
        ops = []
        for a, b in sched.wave_blocks(w):
            rs = sched.rows(b)
            if a == sched.rank:
                recv[rs].copy_(send[rs])
            else:
                ops.append(dist.P2POp(dist.isend, send[rs], a, group))
                ops.append(dist.P2POp(dist.irecv, recv[rs], a, group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()


def _view(base: torch.Tensor, ptr: int, rows: int, row_elems: int) -> torch.Tensor:
    """[rows][row_elems] bf16 view of the byte buffer ``base`` at device address ``ptr``."""
    off = ptr - base.data_ptr()
    n = rows * row_elems * 2
    return base[off:off + n].view(torch.bfloat16).view(rows, row_elems)


class EPBlock:
    """The MoE block as rank ``rank`` of ``ranks`` under expert parallelism, on one GPU.

    Weights: the dense ones whole, the routed ones this rank's E/G experts.  The six
    phases are separate methods so that a driver can exchange blocks between them;
    ``forward`` and ``backward`` run them with torch.distributed exchanges."""

    def __init__(self, shape, ranks: int, rank: int, device="cuda", group=None):
        self.shape, self.G, self.rank, self.group = shape, ranks, rank, group
        self.device = torch.device(device)
        self.plan = M.Plan.from_shape(shape, ep_ranks=ranks, ep_rank=rank)
        info = self.plan.info
        self.saved = torch.empty(info.saved_bytes, dtype=torch.uint8, device=self.device)
        self.ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.stats = torch.zeros(info.stats_bytes // 4, dtype=torch.int32, device=self.device)
        v = M.moe_ep_view(self.plan, self.saved, self.ws)
        self.sched = BlockSchedule(v.ranks, v.rank, v.dest_per_rank, v.n_waves, v.cap_send)
        n = self.sched.n_blocks * v.cap_send
        self.buf = {
            "send_pools": _view(self.ws, v.send_pools, n, v.pool_row_elems),
            "recv_pools": _view(self.saved, v.recv_pools, n, v.pool_row_elems),
            "y_send": _view(self.ws, v.y_send, n, v.row_elems), "y_recv": _view(self.saved, v.y_recv, n, v.row_elems),
            "dy_send": _view(self.ws, v.dy_send, n, v.row_elems), "dy_recv": _view(self.ws, v.dy_recv, n, v.row_elems),
            "dx_send": _view(self.ws, v.dx_send, n, v.row_elems), "dx_recv": _view(self.ws, v.dx_recv, n, v.row_elems),
        }
        off = v.expert_rows - self.saved.data_ptr()
        self.expert_rows = self.saved[off:off + 4 * (shape.n_experts // ranks)].view(torch.int32)
        T, k = shape.T, shape.top_k
        off = v.topk_idx - self.saved.data_ptr()
        self.topk_idx = self.saved[off:off + 4 * T * k].view(torch.int32).view(T, k)
        off = v.slot - self.saved.data_ptr()
        self.slot = self.saved[off:off + 8 * T * k].view(torch.int32).view(T, k, 2)
        self.weights, self.grads = {}, {}

    def load(self, weights: dict, bias: torch.Tensor, logit_offset=None, training=True) -> None:
        """Dense weights whole; routed weights of this rank's experts (slices of the full ones)."""
        El = self.shape.n_experts // self.G
        lo = self.rank * El
        self.weights = {n: (w[lo:lo + El].contiguous() if n in ("w1", "w3", "w2") else w) for n, w in weights.items()}
        self.bias = bias
        self.logit_offset = logit_offset
        if training:
            self.grads = {n: torch.empty(self.weights[n].shape, dtype=torch.float32, device=self.device)
                          for n in self.weights}

    def hist(self) -> torch.Tensor:
        """This source's selection histogram [E] (pre-drop)."""
        return self.stats[8:8 + self.shape.n_experts]

    def stats_dict(self) -> dict:
        s = self.stats.cpu().numpy()
        return {"kept_here": int(self.expert_rows.sum().item()), "dropped_sender": int(s[1]), "status": int(s[3]),
                "nan_logits": int(s[7]), "hist": s[8:8 + self.shape.n_experts].copy()}

    # phases (each one library call)
    def fwd_send(self, x, stream=None):
        M.moe_ep_forward_send(self.plan, self.weights, x, self.bias, self.logit_offset, self.stats, self.saved,
                              self.ws, stream)

    def fwd_experts(self, stream=None):
        w = self.weights
        M.moe_ep_forward_experts(self.plan, w["w1"], w["w3"], w["w2"], self.stats, self.saved, self.ws, stream)

    def fwd_combine(self, y, stream=None):
        M.moe_ep_forward_combine(self.plan, self.weights, y, self.saved, self.ws, stream)

    def bwd_send(self, x, dy, stream=None):
        M.moe_ep_backward_send(self.plan, self.weights, self.saved, x, dy, self.grads, self.ws, stream)

    def bwd_experts(self, stream=None):
        w = self.weights
        M.moe_ep_backward_experts(self.plan, w["w1"], w["w3"], w["w2"], self.saved, self.grads, self.ws, stream)

    def bwd_finish(self, x, dx, stream=None):
        M.moe_ep_backward_finish(self.plan, self.weights, self.saved, x, dx, self.grads, self.ws, stream)

    # whole passes with the exchanges between ranks (one process per GPU)
    def forward(self, x, y=None):
        s = self.shape
        y = torch.empty((s.T, s.d_model), dtype=torch.float32, device=self.device) if y is None else y
        self.fwd_send(x)
        exchange(self.sched, self.buf["send_pools"], self.buf["recv_pools"], self.group)
        self.fwd_experts()
        exchange(self.sched, self.buf["y_send"], self.buf["y_recv"], self.group)
        self.fwd_combine(y)
        return y

    def backward(self, x, dy, dx=None):
        s = self.shape
        dx = torch.empty((s.T, s.d_model), dtype=torch.float32, device=self.device) if dx is None else dx
        self.bwd_send(x, dy)
        exchange(self.sched, self.buf["dy_send"], self.buf["dy_recv"], self.group)
        self.bwd_experts()
        exchange(self.sched, self.buf["dx_send"], self.buf["dx_recv"], self.group)
        self.bwd_finish(x, dx)
        return dx
