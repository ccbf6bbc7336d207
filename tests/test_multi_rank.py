"""The multi-GPU path's host logic on two gloo ranks (CPU).

Each rank owns a full batch of its own tokens (weak scaling).  The forward
and dX need no exchange; the layer's weight gradient is the sum of the
ranks' gradients, which bench.py forms with one all-reduce.  Here each rank
computes its dW/db with the float64 oracle, the same all-reduce helper sums
them over gloo, and the result must equal the oracle's gradient over the
concatenated tokens of both ranks.  The max-over-ranks timing helper is
checked alongside.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

N, C, D, WID = 96, 6, 10, 5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from group_dft_structured_b200.workloads import make_inputs
    from oracle import feql_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = make_inputs(bench.rank_seed_id(WID, rank), N, C, D, "fp32")
        dW, db = O.backward_dw(inp["x"].astype(np.float64), inp["dy"].astype(np.float64))
        tdW, tdb = torch.from_numpy(dW), torch.from_numpy(db)
        bench.dp_allreduce_grads(tdW, tdb)
        slowest = bench.max_over_ranks(10.0 * (rank + 1), "cpu")
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), dW=tdW.numpy(), db=tdb.numpy(),
                 slowest=slowest)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_weight_gradient_all_reduce(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from group_dft_structured_b200.workloads import make_inputs
    from oracle import feql_oracle as O

    xs, dys = [], []
    for r in range(world):
        inp = make_inputs(bench.rank_seed_id(WID, r), N, C, D, "fp32")
        xs.append(inp["x"].astype(np.float64))
        dys.append(inp["dy"].astype(np.float64))
    ref_dW, ref_db = O.backward_dw(np.concatenate(xs), np.concatenate(dys))
    for r in range(world):
        got = np.load(os.path.join(tmp_path, f"r{r}.npz"))
        assert np.allclose(got["dW"], ref_dW, rtol=0, atol=1e-10)
        assert np.allclose(got["db"], ref_db, rtol=0, atol=1e-10)
        assert float(got["slowest"]) == 20.0


def test_rank_seeds_differ():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.rank_seed_id(5, 0) == 5
    assert len({bench.rank_seed_id(5, r) for r in range(8)}) == 8
