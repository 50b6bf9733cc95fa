"""Two-rank (gloo, CPU) check of the benchmark's multi-GPU aggregation: the
job time is the max over ranks and the rate counts every rank's work."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from nvfp4_block_scaled_gemm_b200.dist_timing import max_over_ranks, whole_job_rate
    my_ms = [2.0, 5.0][rank]
    ms = max_over_ranks(my_ms)
    out[rank] = (ms, whole_job_rate(1000.0, world, ms))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_rate():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (5.0, 1000.0 * 2 / 5e-3)


def test_single_process_is_identity():
    from nvfp4_block_scaled_gemm_b200.dist_timing import max_over_ranks, whole_job_rate
    assert max_over_ranks(3.5) == 3.5
    assert whole_job_rate(10.0, 1, 1.0) == 10000.0
