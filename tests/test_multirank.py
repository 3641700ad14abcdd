"""The benchmark's multi-rank host logic on CPU: two `gloo` ranks (world size 2, spawned
processes, rendezvous on 127.0.0.1).  Every rank gets the slowest rank's time back, the job
value counts every rank's work in that time (weak scaling), and each rank draws its own input
batch.  The data path itself has no collective, so nothing else crosses ranks."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from nvfp4_quantized_b200 import synth
        ms = [3.0, 5.5][rank]                                   # rank 1 is the slow one
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        x0, _, _ = synth.linear_inputs("tiny", seed=bench.rank_input_seed(rank, 0))
        # gather every rank's first input row sum to compare batches across ranks
        s = torch.tensor([float(x0.float().sum())], dtype=torch.float64)
        all_s = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_s, s)
        out[rank] = (got, [float(v) for v in all_s])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.5                        # both ranks see the max
    sums = res[0][1]
    assert sums[0] != sums[1]                                   # each rank has its own batch


def test_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_tflops(1, 1e12, 10, 5.0)
    two = bench.job_tflops(2, 1e12, 10, 5.0)
    assert abs(one - 2000.0) < 1e-9 and abs(two - 2 * one) < 1e-9
    # a slower rank lowers the job value: time is the max over ranks
    assert bench.job_tflops(2, 1e12, 10, 10.0) == one
    assert bench.max_over_ranks(4.25, 1, torch.device("cpu")) == 4.25
