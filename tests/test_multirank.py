"""Host-side logic of the multi-GPU benchmark path on CPU: two gloo ranks.

The prefill linear layer is token-parallel, so the N-GPU benchmark runs one
independent batch per rank with no data-path collective; the only
cross-rank steps are the barrier around the timed region and the max over
ranks of the step time.  These run here with the gloo backend.
"""
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


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    try:
        dist.barrier()
        ms = bench.max_over_ranks(1.0 + 0.5 * rank)          # rank 1 is the slow one
        v = bench.whole_job_tflops(2.0e12, world, ms)
        q.put((rank, ms, v))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, v in res:
        assert ms == 1.5                                       # max over ranks
        assert v == pytest.approx(2.0e12 * 2 / 1.5e-3 / 1e12)  # whole-job work / slowest rank


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_nonzero_rank_does_no_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0
