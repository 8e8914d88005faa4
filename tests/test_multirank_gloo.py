"""The N>1 path on CPU: world size 2 over gloo.

The mixer shards by batch: sequences are independent, so each rank runs its
own sequences and no collective touches the data; only the step time is
reduced (max over ranks) as bench.py does.  Here each rank runs the oracle on
its half of a batch and the concatenation must equal the single-process
result exactly, and the max-reduce of per-rank times must give the max."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    from oracle import bitssm_oracle as O
    from ternary_weight_selective_b200 import synthetic as S

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = S.WORKLOADS["tiny"]
    x, layers = S.make_inputs(wl, seed=0, batch=4, seqlen=24)
    P = O.TernaryLayer(layers[0], "A8")
    per = x.shape[0] // world
    out, _ = O.bitssm_layer(x[rank * per:(rank + 1) * per], P)
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), out)
    t = torch.tensor([float(10 + rank)], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    assert t.item() == 10.0 + world - 1
    dist.barrier()
    dist.destroy_process_group()


def test_batch_sharding_world2(tmp_path):
    from oracle import bitssm_oracle as O
    from ternary_weight_selective_b200 import synthetic as S

    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    parts = [np.load(tmp_path / f"rank{r}.npy") for r in range(2)]
    wl = S.WORKLOADS["tiny"]
    x, layers = S.make_inputs(wl, seed=0, batch=4, seqlen=24)
    full, _ = O.bitssm_layer(x, O.TernaryLayer(layers[0], "A8"))
    assert np.array_equal(np.concatenate(parts, axis=0), full)
