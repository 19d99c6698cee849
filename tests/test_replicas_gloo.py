"""The multi-process plumbing of bench.py on CPU: two gloo ranks launched the way torchrun
launches them (RANK / WORLD_SIZE / LOCAL_RANK / MASTER_* in the environment).  PBSA shards
as replicas (every (batch, head) pair is independent; no collective in the data path), so
the only cross-rank steps are the barrier, the max of the ranks' times and the sum of
their FLOPs, and the reference arm runs on rank 0 alone."""
import os
import socket
import time

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(ws)
    assert (w, r, local) == (ws, rank, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    ms = bench.all_max(w, 10.0 + rank)              # device time of this rank's steps
    flops = bench.all_sum(w, 1e12 * (rank + 1))     # FLOPs this rank processed
    # whole-job throughput: all ranks' work over the slowest rank's time
    value = flops / (ms * 1e-3) / 1e12
    t0 = time.time()
    class A:  # the reference arm's arguments
        warmup, steps, gpus = 1, 1, ws
    ref = bench.run_reference(A, w, r) if r != 0 else "rank0"
    out[rank] = (ms, flops, value, ref, time.time() - t0)
    dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_bench():
    ws, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(ws, port, out), nprocs=ws, join=True,
                           start_method="spawn")
        res = dict(out)
    for rank in range(ws):
        ms, flops, value, ref, dt = res[rank]
        assert ms == 11.0 and flops == 3e12
        assert abs(value - 3e12 / 11e-3 / 1e12) < 1e-9
    # the reference arm does no work on ranks other than 0
    assert res[1][3] is None and res[1][4] < 1.0
