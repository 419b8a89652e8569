"""The multi-replica path of bench.py on CPU: two gloo ranks on 127.0.0.1.

`bench.py --gpus N` runs N independent replicas (the layer shards over
tokens; no exchange on the data path). What the ranks share is the timing:
the job's step time is the slowest replica's, and the whole-job rate counts
every replica's work. The reference arm runs on rank 0 only."""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        step_ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        rate = bench.job_tflops(2.0e12, world, step_ms)
        printed = io.StringIO()
        args = types.SimpleNamespace(steps=1, warmup=1)
        with contextlib.redirect_stdout(printed):
            if rank != 0:
                bench.run_reference(args, rank, world)  # must return at once, printing nothing
        dist.barrier()
        out.put((rank, step_ms, rate, printed.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_and_count_both():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, step_ms, rate, printed in got:
        assert step_ms == 15.0          # max over ranks: rank 1's 15 ms
        assert abs(rate - 2 * 2.0e12 / 15e-3 / 1e12) < 1e-9  # both replicas' work
        assert printed == ""
