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


def _worker_forms(rank, world, port, out_dir):
    """Each rank runs its half of the batch through the block form and the
    SSD scan (both are independent per sequence)."""
    import torch.distributed as dist

    from oracle import bitssm_oracle as O
    from oracle import ssd_oracle as SSD
    from ternary_weight_selective_b200 import synthetic as S

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = S.Workload("blk_gloo", 4, 10, 64, 128, 16, 4, "f32", "A8", block=True)
    x, layers = S.make_inputs(wl, seed=1)
    per = x.shape[0] // world
    out, _ = O.bitssm_block_a8(x[rank * per:(rank + 1) * per], O.TernaryLayer(layers[0], "A8"))
    np.save(os.path.join(out_dir, f"blk{rank}.npy"), out)
    xs, dt, A, Bm, Cm, D = S.random_ssd_inputs(2, 4, 12, 4, 8, 2, 16)
    sl = slice(rank * per, (rank + 1) * per)
    y, _ = SSD.ssd_chunked(xs[sl], dt[sl], A, Bm[sl], Cm[sl], D, Q=4)
    np.save(os.path.join(out_dir, f"ssd{rank}.npy"), y)
    dist.barrier()
    dist.destroy_process_group()


def test_block_and_ssd_sharding_world2(tmp_path):
    from oracle import bitssm_oracle as O
    from oracle import ssd_oracle as SSD
    from ternary_weight_selective_b200 import synthetic as S

    port = _free_port()
    mp.start_processes(_worker_forms, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    wl = S.Workload("blk_gloo", 4, 10, 64, 128, 16, 4, "f32", "A8", block=True)
    x, layers = S.make_inputs(wl, seed=1)
    full, _ = O.bitssm_block_a8(x, O.TernaryLayer(layers[0], "A8"))
    parts = [np.load(tmp_path / f"blk{r}.npy") for r in range(2)]
    assert np.array_equal(np.concatenate(parts, axis=0), full)
    y_full, _ = SSD.ssd_chunked(*S.random_ssd_inputs(2, 4, 12, 4, 8, 2, 16), Q=4)
    parts = [np.load(tmp_path / f"ssd{r}.npy") for r in range(2)]
    np.testing.assert_allclose(np.concatenate(parts, axis=0), y_full, rtol=1e-13, atol=1e-14)


def _worker_fail(rank, world, port, out_dir):
    """Rank 1 fails before the timing reduce; rank 0's reduce must end with
    an error within the process group's short timeout instead of hanging."""
    import datetime

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        raise SystemExit(3)          # leaves between steps, nothing in flight
    t = torch.tensor([1.0], dtype=torch.float64)
    try:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        outcome = "completed"
    except Exception as e:  # the collective reports the missing peer
        outcome = "error: " + type(e).__name__
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(outcome)


def test_a_failed_rank_is_reported_not_hung(tmp_path):
    port = _free_port()
    ctx = mp.start_processes(_worker_fail, args=(2, port, str(tmp_path)), nprocs=2, join=False,
                             start_method="spawn")
    import time
    deadline = time.time() + 60
    while time.time() < deadline:
        try:
            if ctx.join(timeout=1):
                break
        except Exception:
            # rank 1's exit is reported here; keep waiting for rank 0
            pass
        if (tmp_path / "rank0.txt").exists():
            break
    for p in ctx.processes:
        p.join(timeout=20)
        if p.is_alive():
            p.kill()
    outcome = (tmp_path / "rank0.txt").read_text()
    assert outcome.startswith("error"), outcome

