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


# ---------------------------------------------------------------------------
# sequence-sharded (context-parallel) oracle: distributed top-K descent
# ---------------------------------------------------------------------------

from oracle import sharded  # noqa: E402


class _GlooComm:
    """all_gather of Python objects over the default torch.distributed group."""

    def __init__(self):
        import torch.distributed as dist
        self._dist = dist
        self.rank, self.world = dist.get_rank(), dist.get_world_size()

    def all_gather(self, obj):
        out = [None] * self.world
        self._dist.all_gather_object(out, obj)
        return out


def _cp_inputs(N=512, D=16, seed=3):
    rng = np.random.default_rng(seed)
    return [orc.round_to_dtype(rng.standard_normal((N, D)), "bf16") for _ in range(4)]


def _cp_worker(rank, world, port, args, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    assert lhdist.init("gloo", timeout_s=60)
    q, k, v, do, p, L, K = args
    comm = _GlooComm()
    n = q.shape[0] // world
    sl = slice(rank * n, (rank + 1) * n)
    fw = sharded.forward_shard(comm, q[sl], k[sl], v[sl], p, L, K, "bf16")
    bw = sharded.backward_shard(comm, fw, do[sl], p)
    np.savez(os.path.join(out_dir, f"cp{rank}.npz"), lvl=fw["lvl"], idx=fw["idx"], o=fw["o"],
             seg=np.array(fw["seg"]), dq=bw["dq"], dk=bw["dk"], dv=bw["dv"],
             **{f"sel{l}": fw["sel"][l] for l in range(1, L)})
    lhdist.shutdown()


def test_sequence_sharded_oracle_over_gloo_equals_single_process(tmp_path):
    """Two gloo ranks, each holding half of one head's tokens, run the sharded
    forward and backward (local pool and scores, per-level all-gather of local
    top-k candidates, all-gather of the sub-sequence K and V, reduce of the
    key gradients). The selection, the gather map (the ranks' segments in rank
    order) and the output equal the single-process oracle bit for bit; the
    gradients, whose key-side sums are grouped by rank, agree to 1e-12."""
    world, p, L, K = 2, 4, 3, 6
    q, k, v, do = _cp_inputs()
    mp.start_processes(_cp_worker, args=(world, _free_port(), (q, k, v, do, p, L, K), str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    parts = [np.load(tmp_path / f"cp{r}.npz") for r in range(world)]
    ref = orc.forward_head(q, k, v, p, L, K, "bf16")
    rb = orc.backward_head(ref, do, p)
    for l in range(1, L):
        for part in parts:
            assert np.array_equal(part[f"sel{l}"], ref["sel"][l])
    assert np.array_equal(np.concatenate([x["lvl"] for x in parts]), ref["lvl"])
    assert np.array_equal(np.concatenate([x["idx"] for x in parts]), ref["idx"])
    assert parts[0]["seg"][0] == 0 and parts[1]["seg"][0] == parts[0]["seg"][1]
    assert np.array_equal(np.concatenate([x["o"] for x in parts]), ref["o"])
    for name in ("dq", "dk", "dv"):
        assert np.max(np.abs(np.concatenate([x[name] for x in parts]) - rb[name])) < 1e-12


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("readings", [
    {}, {"ties": "high"}, {"score": "maxpool"}, {"inclusion": "partition"},
    {"score": "sum", "order": "pre", "weight": "mean"},
])
def test_sequence_sharded_oracle_ranks_in_one_process(world, readings):
    """The same decomposition with the ranks as threads of one process, for
    every reading switch and up to 8 ranks (a shard down to one coarsest
    block), including exactly tied scores (codebook rows)."""
    p, L, K = 2, 4, 3
    rng = np.random.default_rng(world)
    N, D = 128, 8
    book = orc.round_to_dtype(rng.standard_normal((4, D)), "bf16")
    q = book[rng.integers(0, 4, N)]                     # many exactly tied scores
    k = book[rng.integers(0, 4, N)]
    v, do = (orc.round_to_dtype(rng.standard_normal((N, D)), "bf16") for _ in range(2))
    n = N // world

    def fn(comm):
        sl = slice(comm.rank * n, (comm.rank + 1) * n)
        fw = sharded.forward_shard(comm, q[sl], k[sl], v[sl], p, L, K, "bf16", **readings)
        return fw, sharded.backward_shard(comm, fw, do[sl], p)

    res = sharded.run_local(world, fn)
    ref = orc.forward_head(q, k, v, p, L, K, "bf16", **readings)
    rb = orc.backward_head(ref, do, p)
    for l in range(1, L):
        assert all(np.array_equal(f["sel"][l], ref["sel"][l]) for f, _ in res)
    assert np.array_equal(np.concatenate([f["lvl"] for f, _ in res]), ref["lvl"])
    assert np.array_equal(np.concatenate([f["idx"] for f, _ in res]), ref["idx"])
    assert np.array_equal(np.concatenate([f["o"] for f, _ in res]), ref["o"])
    for name in ("dq", "dk", "dv"):
        assert np.max(np.abs(np.concatenate([b[name] for _, b in res]) - rb[name])) < 1e-12


def test_sequence_sharded_oracle_rejects_unaligned_shards():
    with pytest.raises(ValueError):
        sharded.shard_sizes(96, 4, 3, 4)                # 24 tokens per rank, not a multiple of 16


# ---------------------------------------------------------------------------
# the sharded driver's collectives (cp.run_distributed) over gloo, on CPU
# ---------------------------------------------------------------------------

class _RecordingRank:
    """Stands in for cp.ShardRank on the CPU: each step fills its buffers with
    rank-tagged values and checks what the collectives delivered, so the
    driver's order of steps and collectives is exercised without a GPU."""

    def __init__(self, rank, world):
        self.rank, self.world, self.device = rank, world, torch.device("cpu")
        self.sq_loc = torch.empty(2, 1, 2, 5, dtype=torch.float64)
        self.scale = torch.zeros(4, 1, 2, dtype=torch.int32)
        S = 4 * world
        self.ks, self.vs = torch.zeros(1, 2, S, 3), torch.zeros(1, 2, S, 3)
        self.dks, self.dvs = torch.zeros(1, 2, S, 3), torch.zeros(1, 2, S, 3)
        self.log = []

    def gathered_shape(self):
        return (self.world,) + tuple(self.sq_loc.shape)

    def pool(self, q, k, v):
        self.sq_loc.fill_(self.rank + 1)
        self.scale[:3] = torch.tensor([10, 20, 30]).view(3, 1, 1) * (self.rank + 1) % 7   # per-rank maxima
        self.scale[3] = -1
        self.log.append("pool")

    def select_gather(self, gathered, q, k, v):
        for r in range(self.world):                      # every rank's norms, in rank order
            assert torch.all(gathered[r] == r + 1)
        want = torch.stack([torch.tensor([10, 20, 30])[i] * torch.arange(1, self.world + 1) % 7 for i in range(3)])
        assert torch.equal(self.scale[:3, 0, 0], want.max(dim=1).values.int())   # max over the ranks
        assert torch.all(self.scale[3] == -1)            # the dO row stays the rank's own
        rows = slice(4 * self.rank, 4 * self.rank + 4)   # this rank's segment, zero elsewhere
        self.ks.zero_()
        self.vs.zero_()
        self.ks[:, :, rows] = self.rank + 1
        self.vs[:, :, rows] = -(self.rank + 1)
        self.log.append("select_gather")

    def attend_scatter(self, o):
        for r in range(self.world):                      # the all-reduce assembled every segment
            assert torch.all(self.ks[:, :, 4 * r:4 * r + 4] == r + 1)
            assert torch.all(self.vs[:, :, 4 * r:4 * r + 4] == -(r + 1))
        o.fill_(self.rank)
        self.log.append("attend_scatter")

    def attend_bwd(self, do):
        self.dks.fill_(self.rank + 1)                    # this rank's queries' part of every key gradient
        self.dvs.fill_(2 * (self.rank + 1))
        self.log.append("attend_bwd")

    def spread(self, dq, dk, dv):
        tot = self.world * (self.world + 1) // 2
        assert torch.all(self.dks == tot) and torch.all(self.dvs == 2 * tot)
        self.log.append("spread")


def _cp_driver_worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    assert lhdist.init("gloo", timeout_s=60)
    from long_context_symmetric_b200 import cp
    st = _RecordingRank(rank, world)
    o = torch.empty(3)
    cp.run_distributed(st, None, None, None, o, do=torch.empty(1), dq=None, dk=None, dv=None)
    assert torch.all(o == rank)
    np.save(os.path.join(out_dir, f"log{rank}.npy"), np.array(st.log))
    lhdist.shutdown()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_driver_collectives_over_gloo(tmp_path, world):
    mp.start_processes(_cp_driver_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert list(np.load(tmp_path / f"log{r}.npy")) == ["pool", "select_gather", "attend_scatter",
                                                            "attend_bwd", "spread"]
