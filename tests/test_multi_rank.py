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
