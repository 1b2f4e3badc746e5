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
