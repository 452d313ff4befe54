"""Two data-parallel replicas on CPU (gloo): the histogram exchange before the bias step
keeps the bias identical on both ranks and equal to a single process's bias step over
the concatenated batch."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from capacity_limited_routed_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, T, E, k, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from capacity_limited_routed_b200.parallel import global_histogram, global_tokens
    from oracle import moe_oracle as O
    logits = synth.make_logits(T, E, seed=100 + rank)
    _, _, hist = O.route(logits, np.zeros(E, np.float32), k)
    h = torch.from_numpy(hist.astype(np.int32))
    global_histogram(h)
    bias = O.bias_update(h.numpy(), np.zeros(E, np.float32), 1e-3, global_tokens(T), k)
    np.save(os.path.join(out_dir, f"bias{rank}.npy"), bias)
    np.save(os.path.join(out_dir, f"hist{rank}.npy"), h.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_histogram_exchange_two_ranks(tmp_path):
    T, E, k, world = 256, 24, 2, 2
    mp.spawn(_rank_main, args=(world, _free_port(), T, E, k, str(tmp_path)), nprocs=world, join=True)
    b0, b1 = (np.load(tmp_path / f"bias{r}.npy") for r in range(world))
    h0, h1 = (np.load(tmp_path / f"hist{r}.npy") for r in range(world))
    assert np.array_equal(h0, h1) and np.array_equal(b0.view(np.uint32), b1.view(np.uint32))
    from oracle import moe_oracle as O
    both = np.concatenate([synth.make_logits(T, E, seed=100 + r) for r in range(world)])
    _, _, hist_all = O.route(both, np.zeros(E, np.float32), k)
    assert np.array_equal(h0, hist_all)
    ref = O.bias_update(hist_all, np.zeros(E, np.float32), 1e-3, world * T, k)
    assert np.array_equal(b0.view(np.uint32), ref.view(np.uint32))


def _ep_rank_main(rank, world, port, Dl, W, Cs, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from capacity_limited_routed_b200.parallel import BlockSchedule, exchange
    sched = BlockSchedule(world, rank, Dl, W, Cs)
    n = sched.n_blocks * Cs
    # every row of the send buffer names its sender, block and row
    send = torch.zeros((n, 4), dtype=torch.int32)
    for b in range(sched.n_blocks):
        send[b * Cs:(b + 1) * Cs, 0] = rank
        send[b * Cs:(b + 1) * Cs, 1] = b
        send[b * Cs:(b + 1) * Cs, 2] = torch.arange(Cs)
    recv = torch.full((n, 4), -1, dtype=torch.int32)
    exchange(sched, send, recv)
    np.save(os.path.join(out_dir, f"recv{rank}.npy"), recv.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_expert_parallel_block_exchange(tmp_path):
    """The fixed-shape exchange of expert parallelism on CPU ranks (gloo): rank r receives
    into block (a * Dl + d) * W + w what peer a sent from its block (r * Dl + d) * W + w, for
    every peer (itself included), local destination and wave, rows in order."""
    Dl, W, Cs = 3, 3, 5
    for world in (2, 3):
        mp.spawn(_ep_rank_main, args=(world, _free_port(), Dl, W, Cs, str(tmp_path)), nprocs=world, join=True)
        for r in range(world):
            recv = np.load(tmp_path / f"recv{r}.npy")
            for a in range(world):
                for d in range(Dl):
                    for w in range(W):
                        b = (a * Dl + d) * W + w
                        rows = recv[b * Cs:(b + 1) * Cs]
                        assert (rows[:, 0] == a).all() and (rows[:, 1] == (r * Dl + d) * W + w).all()
                        assert np.array_equal(rows[:, 2], np.arange(Cs))
