"""Host logic of the multi-process path on CPU (gloo, world size 2): each rank
scores its own seeded batch (rows shard across ranks with no data-path
collective), the step time is the maximum over ranks, and the whole-job value
counts every rank's rows.  The scoring itself is the oracle here (CPU)."""

import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    import oracle
    import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.fullvocab(rows=4, vocab=2048, seed=bench.rank_seed(rank))
        r = oracle.score(w["logits"], w["targets"], temperature=w["temperature"].astype(np.float64),
                         top_p=float(np.float32(w["top_p"])))
        fake_ms = 1.0 + rank  # per-rank step time
        t = bench.max_over_ranks(fake_ms, world)
        out[rank] = (float(r["lp_full"].sum()), t, bench.weak_value(4, world, t),
                     int(w["logits"][0, :8].astype(np.int64).sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_host_logic():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert set(out.keys()) == {0, 1}
    # every rank sees the slowest rank's time
    assert out[0][1] == out[1][1] == 2.0
    # value = all ranks' rows over that time
    assert out[0][2] == pytest.approx(4 * 2 / 2e-3)
    # ranks score different batches
    assert out[0][3] != out[1][3] and out[0][0] != out[1][0]


class _OracleOps:
    """The per-rank steps of sampling_support_b200.dist run by the oracle on
    the CPU (the library needs a GPU; this checks the cross-rank protocol:
    which scalars are reduced, and that the gradient takes the global
    denominator)."""

    @staticmethod
    def weight_sum(rows, row_weight, device):
        import torch

        w = np.ones(rows) if row_weight is None else row_weight.numpy().astype(np.float64)
        return torch.tensor([float(np.sum(w))], dtype=torch.float64)

    @staticmethod
    def l1_distance(draft, target, row_weight, global_weight_sum, want_grad, grad_dtype):
        import torch

        import oracle

        w = None if row_weight is None else row_weight.numpy().astype(np.float64)
        r = oracle.l1(draft.numpy(), target.numpy(), w, want_grad=want_grad,
                      global_wsum=float(global_weight_sum.item()))
        out = {"l1": torch.from_numpy(r["l1"]),
               "loss": torch.tensor([r["loss_num"], r["loss_den"], r["loss"]], dtype=torch.float64)}
        if want_grad:
            out["grad"] = torch.from_numpy(r["grad"])
        return out


def _sharded_worker(rank, world, port, out):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch

    import workloads
    from sampling_support_b200 import dist as vdist

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        d = workloads.random_logits(10, 700, 2.0, seed=41)
        t = workloads.random_logits(10, 700, 2.0, seed=42)
        w = workloads.uniform(10, 0.0, 1.0, 41, 3).astype(np.float32)
        cut = [0, 3, 10]  # uneven shards
        s = slice(cut[rank], cut[rank + 1])
        r = vdist.sharded_l1_distance(torch.from_numpy(d[s].copy()), torch.from_numpy(t[s].copy()),
                                      torch.from_numpy(w[s].copy()), want_grad=True,
                                      ops=_OracleOps)
        ent = vdist.sharded_entropy_mean(torch.tensor([1.5 + rank], dtype=torch.float64),
                                         torch.tensor([2 + rank], dtype=torch.int32))
        out[rank] = (r["grad"].numpy(), float(r["loss_global"].item()),
                     float(r["num_global"].item()), float(r["den_global"].item()),
                     float(ent.item()))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_distance_loss_and_gradient():
    """A distance batch split unevenly over two gloo ranks: the concatenated
    gradients and the reduced loss equal the single-process oracle's on the
    whole batch (gradient normalised by the global weight sum)."""
    sys.path.insert(0, str(ROOT))
    import oracle
    import workloads

    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_sharded_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    d = workloads.random_logits(10, 700, 2.0, seed=41)
    t = workloads.random_logits(10, 700, 2.0, seed=42)
    w = workloads.uniform(10, 0.0, 1.0, 41, 3).astype(np.float32)
    ref = oracle.l1(d, t, w.astype(np.float64), want_grad=True)
    g = np.concatenate([out[0][0], out[1][0]])
    assert np.abs(g - ref["grad"]).max() <= 1e-12 * np.abs(ref["grad"]).max()
    for r in (0, 1):
        assert out[r][1] == pytest.approx(ref["loss"], rel=1e-12)
        assert out[r][2] == pytest.approx(ref["loss_num"], rel=1e-12)
        assert out[r][3] == pytest.approx(ref["loss_den"], rel=1e-12)
        assert out[r][4] == pytest.approx((1.5 + 2.5) / (2 + 3))


class _RecordOps:
    """Stand-ins for the two library steps of the vocabulary-parallel head
    (they need a GPU): the partial step writes a block naming its rank and
    shard, the merge step returns what it was given, so the test sees the
    exchange itself."""

    @staticmethod
    def lmhead_partial(hidden, weight_shard, vocab_begin, vocab_total, targets, temperature,
                       top_k):
        import torch

        blk = torch.zeros(64, dtype=torch.uint8)
        blk[0] = dist.get_rank()
        blk[1] = vocab_begin // 100
        blk[2] = weight_shard.shape[0] // 100
        return blk

    @staticmethod
    def lmhead_merge(partials, rows, vocab_total, targets, temperature, top_k, top_p, min_p):
        return partials


def _tp_worker(rank, world, port, out):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch

    from sampling_support_b200 import dist as vdist

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        begin = [0, 700][rank]
        shard = torch.zeros((700 if rank == 0 else 300, 4))
        g = vdist.tp_fused_lmhead_score(torch.zeros((5, 4)), shard, begin, 1000,
                                        torch.zeros(5, dtype=torch.int32), 1.0, 8, 0.9, 0.0,
                                        ops=_RecordOps)
        out[rank] = g.numpy().copy()
    finally:
        dist.destroy_process_group()


def test_two_rank_vocabulary_parallel_exchange():
    """Every rank ends with every rank's partial block, in rank (= shard)
    order, which is what the merge step reads."""
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_tp_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in (0, 1):
        g = out[r]
        assert g.shape == (2, 64)
        assert g[0, :3].tolist() == [0, 0, 7] and g[1, :3].tolist() == [1, 7, 3]
