"""The N > 1 data-parallel path on CPU: two gloo ranks, each holding a shard of
the batch rows, compute their parameter gradients with the oracle and sum them
with the library's GradReducer; the sum must equal the full-batch gradients.

(The CUDA path needs one GPU per rank; what can run without a GPU -- the
sharding and the packed all-reduce -- runs here.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from parallelizable_recurrence_b200.dist import GradReducer, batch_shard
from synthetic import SRUConfig, generate


def test_batch_shard_covers_every_row_once():
    for total in (0, 1, 7, 16, 64, 65):
        for world in (1, 2, 3, 8):
            rows = []
            for r in range(world):
                a, b = batch_shard(total, world, r)
                assert 0 <= a <= b <= total
                rows.extend(range(a, b))
            assert rows == list(range(total))
            sizes = [batch_shard(total, world, r)[1] - batch_shard(total, world, r)[0] for r in range(world)]
            assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CFG = SRUConfig(name="dp", L=12, B=5, d=8, n_dir=2, seed=77, proj_dtype="fp32", bias="normal0.1", c0="normal",
                masked=True)


def _shard_grads(rows):
    """Oracle parameter gradients (dW_cat, dv, db) of the given batch rows."""
    inp = generate(CFG)
    L, B, d = CFG.L, CFG.B, CFG.d
    X = inp["X"].reshape(L, B, d)[:, rows].reshape(-1, d).astype(np.float64)
    W = inp["W"].astype(np.float64)
    U = oracle.project(X, W).reshape(L, len(rows), 2, 3, d)
    g = oracle.backward(U, inp["x"][:, rows], inp["v"], inp["bias"], inp["dh"][:, rows],
                        c0=inp["c0"][rows], mask=inp["mask"][:, rows])
    dW = oracle.project_dW(g["dU"].reshape(L * len(rows), -1), X)
    return dW, g["dv"], g["dbias"]


def _rank_main(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, b = batch_shard(CFG.B, world, rank)
        dW, dv, db = (torch.from_numpy(np.ascontiguousarray(t)) for t in _shard_grads(list(range(a, b))))
        GradReducer([dW, dv, db])()
        if rank == 0:
            np.savez(out_path, dW=dW.numpy(), dv=dv.numpy(), db=db.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_gradient_allreduce_equals_full_batch(tmp_path):
    out = str(tmp_path / "reduced.npz")
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    got = np.load(out)
    dW, dv, db = _shard_grads(list(range(CFG.B)))
    np.testing.assert_allclose(got["dW"], dW, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dv"], dv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["db"], db, rtol=1e-12, atol=1e-12)
