"""The N > 1 replica path of bench.py on CPU: two gloo ranks (127.0.0.1).  The job's time is
the slowest rank's, every rank sees it, the whole-job rate counts every rank's work, and the
reference arm prints only on rank 0."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from srnl_inputs import CONFIGS
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 is slower on the first value
        got = bench.max_over_ranks(local, world)
        rate = bench.whole_job_rate(world, 1000.0, 4, got[0])
        buf = io.StringIO()

        class A:
            steps, warmup = 1, 1
        with redirect_stdout(buf):
            bench.run_reference(A, CONFIGS["pr1_8x8"], rank, world)
        dist.barrier()
        out.put((rank, got, rate, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate, printed in res:
        assert got == [15.0, 3.0]
        assert rate == pytest.approx(2 * 1000.0 * 4 / 15e-3)
        if rank == 0:
            line = json.loads(printed)
            assert line["impl"] == "reference" and line["n_gpus"] == 2
        else:
            assert printed == ""
