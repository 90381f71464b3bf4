"""Multi-GPU host logic on the CPU: two gloo ranks run bench.py's replica
aggregation (no GPU, no data exchange besides the timing reductions)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    from paged_kv_cache_322_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.replica_workload(wl.WORKLOADS["llama2_7b"], rank)
        ms_local = 10.0 + rank * 5.0                 # rank 1 is the slow one
        bytes_local = 1e9 * (rank + 1)
        ms, gbs, tok = bench.aggregate(ms_local, bytes_local, 64.0 * 100, ws)
        out[rank] = (w.seed, ms, gbs, tok, float(wl.context_lens(w).sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_replica_aggregation():
    ws = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(ws, port, out), nprocs=ws, start_method="spawn", join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] != r1[0]                                  # each replica its own seed ...
    assert r0[4] != r1[4]                                  # ... hence its own batch
    for r in (r0, r1):
        assert r[1] == pytest.approx(15.0)                 # max over ranks
        assert r[2] == pytest.approx(3e9 / 15e-3 / 1e9)    # all ranks' bytes over that time
        assert r[3] == pytest.approx(2 * 6400 / 15e-3)
