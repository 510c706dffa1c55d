"""Multi-rank host logic on CPU: two gloo ranks, no GPU.

Checks the replica decomposition the bench uses on N GPUs: every rank's
batch rows are independent problems, so the ranks' outputs (CPU oracle here)
equal the single-process result on the global batch; the max-over-ranks time
and whole-job throughput are formed as documented.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as orc
from long_context_symmetric_b200 import dist as lhdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, k, v, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    assert lhdist.init("gloo", timeout_s=60)
    info = lhdist.rank_info()
    rows = lhdist.batch_rows(q.shape[0], info.rank, info.world)
    O, _ = orc.forward(q[rows.start:rows.stop], k[rows.start:rows.stop], v[rows.start:rows.stop],
                       p=4, L=3, K=4, dtype="bf16")
    np.save(os.path.join(out_dir, f"o{rank}.npy"), O)
    lhdist.barrier()
    ms = 10.0 + 5.0 * rank                 # a per-rank "device time"
    mx = lhdist.max_over_ranks(ms)
    rate = lhdist.job_throughput(1000.0, info.world, mx / 1e3)
    np.save(os.path.join(out_dir, f"m{rank}.npy"), np.array([mx, rate, lhdist.replica_seed(3, rank)]))
    lhdist.shutdown()


def test_replicas_equal_global_batch(tmp_path):
    world = 2
    rng = np.random.default_rng(0)
    B, N, H, D = 4, 64, 2, 16
    q, k, v = (orc.round_to_dtype(rng.standard_normal((B, N, H, D)), "bf16") for _ in range(3))
    mp.start_processes(_worker, args=(world, _free_port(), q, k, v, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)], axis=0)
    want, _ = orc.forward(q, k, v, p=4, L=3, K=4, dtype="bf16")
    assert np.array_equal(got, want)
    m = [np.load(tmp_path / f"m{r}.npy") for r in range(world)]
    for r in range(world):
        assert m[r][0] == 15.0                           # max over ranks
        assert m[r][1] == pytest.approx(1000.0 * 2 / 0.015)
    assert m[0][2] != m[1][2]                            # distinct replica seeds


@pytest.mark.parametrize("gb,world", [(4, 2), (5, 2), (7, 3), (1, 1)])
def test_batch_rows_partition(gb, world):
    rows = [lhdist.batch_rows(gb, r, world) for r in range(world)]
    flat = [i for rr in rows for i in rr]
    assert flat == list(range(gb))
    assert max(len(r) for r in rows) - min(len(r) for r in rows) <= 1
