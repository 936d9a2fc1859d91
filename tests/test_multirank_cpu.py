"""The N > 1 host logic on CPU: world_size-2 gloo ranks (no GPU).

Each rank takes its shard of a global batch (no data-path collective); timing is the max over
ranks.  Checked here: the shards cover the batch disjointly, every rank regenerates exactly its
sequences of the global batch, the max-over-ranks reduction, and that the oracle run per shard
equals the oracle run on the whole batch.
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
TOK = ("q", "k", "v", "alpha", "b", "w")


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    import gdn2_workloads as W
    import oracle
    # loopback for the rendezvous and for gloo's own connections (the host name may not resolve)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      GLOO_SOCKET_IFNAME="lo")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = W.Workload("mr", B=2, T=70, H=2, dk=16, dv=8, dtype="f32")
    n_global = wl.B * world
    mine = W.shard(n_global, world, rank)
    d = W.chunk_inputs(wl, device="cpu", seed=3, indices=mine)
    o, S = oracle.recurrent(*[d[n].double().numpy() for n in TOK], S0=d["S0"].double().numpy())
    t_max = bench.max_over_ranks(float(rank + 1), world, torch.device("cpu"))
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), o=o, S=S, mine=np.array(mine), t_max=t_max)
    dist.barrier()
    dist.destroy_process_group()


def test_shards_cover_the_batch_disjointly():
    sys.path.insert(0, ROOT)
    import gdn2_workloads as W
    for n in (1, 7, 8, 130):
        for world in (1, 2, 3, 8):
            parts = [W.shard(n, world, r) for r in range(world)]
            flat = [i for p in parts for i in p]
            assert flat == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1


def test_two_gloo_ranks_match_the_unsharded_oracle(tmp_path):
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    world = 2
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    sys.path.insert(0, ROOT)
    import gdn2_workloads as W
    import oracle
    wl = W.Workload("mr", B=2, T=70, H=2, dk=16, dv=8, dtype="f32")
    full = W.chunk_inputs(wl, device="cpu", seed=3, indices=list(range(wl.B * world)))
    o_ref, S_ref = oracle.recurrent(*[full[n].double().numpy() for n in TOK], S0=full["S0"].double().numpy())
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        mine = list(z["mine"])
        assert float(z["t_max"]) == pytest.approx(float(world))
        assert np.array_equal(z["o"], o_ref[mine])
        assert np.array_equal(z["S"], S_ref[mine])
