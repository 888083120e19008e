"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

N > 1 runs independent replicas (decode sweeps share nothing), so the only
cross-rank steps are the timing reduction (max over ranks) and the whole-job
aggregate; the reference arm runs on rank 0 alone.
"""
import datetime
import io
import os
import socket
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    elapsed_ms = 100.0 * (rank + 1)              # rank 1 is the slower one
    m = bench.max_over_ranks(elapsed_ms, world)
    value = bench.aggregate(1.5, m / 1e3, world)  # 1.5 GB per rank
    dist.barrier()
    # the reference arm prints on rank 0 only; other ranks exit 0 silently
    buf = io.StringIO()
    if rank != 0:
        with redirect_stdout(buf):
            rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", "2",
                                                        "--steps", "1", "--warmup", "3"]))
    else:
        rc = 0
    q.put((rank, m, value, rc, buf.getvalue()))
    dist.destroy_process_group()


def test_two_rank_timing_reduction_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, m, value, rc, printed in out:
        assert m == 200.0                          # the max over ranks
        assert value == pytest.approx(1.5 * 2 / 0.2)
        assert rc == 0
        if rank == 1:
            assert printed == ""


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.aggregate(3.0, 0.5, 1) == 6.0
