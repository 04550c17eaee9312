"""Multi-rank host logic of bench.py with world_size 2 on the gloo backend (CPU):
device times are reduced with MAX over ranks, the job throughput counts every rank's
units over the slowest rank's time, and the reference arm prints from rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    import bench
    ms = 2.0 + 3.0 * rank                       # rank 1 is the slow one
    mx = bench.max_over_ranks(ms, ws)
    val, ms_max = bench.job_throughput(1000, ms, ws)
    bench.barrier(ws)

    class A:
        steps, warmup, ref_tokens = 1, 0, 8
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference(A)
    out[rank] = (mx, val, ms_max, buf.getvalue())
    dist.destroy_process_group()


def test_two_rank_reduction_and_reference_arm():
    ws = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(ws, port, out), nprocs=ws, start_method="spawn")
    for r in range(ws):
        mx, val, ms_max, printed = out[r]
        assert mx == 5.0 and ms_max == 5.0
        assert abs(val - 2 * 1000 / 5e-3) < 1e-6
    line = json.loads(out[0][3].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == ws and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert out[1][3] == ""
