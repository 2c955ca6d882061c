"""Multi-process host logic of bench.py with two gloo ranks on CPU: rank
discovery from the torchrun environment, the max-over-ranks timing reduction,
the barrier, and the per-rank layer seeds (weak scaling, no data-path
collective)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _worker(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import bench
    from decode_gemm_e8_b200 import synth
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench._dist()
        t = bench._max_over_ranks(10.0 + 3.0 * rank, w, torch.device("cpu"))
        bench._barrier(w)
        lay = synth.workloads()[bench.WORKLOAD].layers[0]
        w_seed, rs = bench._rank_layer_seeds(lay, r)
        # a small slice of this rank's weights, to compare layers across ranks
        Wr = synth.gaussian_weights(4, 64, lay.std, w_seed)
        q.put((r, w, local, t, rs, Wr))
    finally:
        dist.destroy_process_group()


def test_two_rank_host_logic():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(ws):
        r, w, local, t, rs, Wr = q.get(timeout=120)
        got[r] = (w, local, t, rs, Wr)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(got) == [0, 1]
    for r, (w, local, t, rs, Wr) in got.items():
        assert w == ws and local == r
        assert t == 13.0                     # max over ranks of 10 + 3 rank
    # rank 0 is the seeded workload; the other rank has its own layer and seed
    sys.path.insert(0, ROOT)
    import bench
    from decode_gemm_e8_b200 import synth
    lay = synth.workloads()[bench.WORKLOAD].layers[0]
    assert got[0][3] == lay.rht_seed
    assert got[1][3] != got[0][3]
    assert np.array_equal(got[0][4], synth.gaussian_weights(4, 64, lay.std, lay.w_seed))
    assert not np.array_equal(got[0][4], got[1][4])
