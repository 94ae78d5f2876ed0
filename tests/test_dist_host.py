"""The multi-process plumbing of bench.py on the host (world size 2, gloo):
process-group set-up, the barrier, the max over ranks of the timed region,
and the reference arm's rule that only rank 0 works and prints."""
import io
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


def _rank_main(rank, ws, port, results):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(ws),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    got_ws, got_rank, _ = bench.init_dist()
    out = {"ws": got_ws, "rank": got_rank, "backend": dist.get_backend()}
    bench.barrier(ws)
    out["max"] = bench.max_over_ranks(1.5 + rank, ws)          # per-rank times -> the slowest
    # reference arm: a fast stand-in for the oracle sample; rank 0 prints one line, the others nothing
    bench.cpu_baseline = lambda workload, budget_s=0: {"value": 1.0, "unit": "TFLOPS", "cores": 1,
                                                       "kind": "oracle", "sample": "stub", "seconds": 0.01}

    class A:
        warmup, steps, gpus, workload = 1, 2, ws, "w4a16_asym_sweep"
    buf = io.StringIO()
    with redirect_stdout(buf):
        out["ref_rc"] = bench.run_reference(A, ws, rank)
    out["ref_lines"] = [l for l in buf.getvalue().splitlines() if l.strip()]
    bench.barrier(ws)
    dist.destroy_process_group()
    results[rank] = out


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="host-only check; with GPUs the ranks would take NCCL and one GPU each")
def test_two_ranks_on_gloo():
    ws = 2
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(ws, _free_port(), results), nprocs=ws, join=True)
        res = dict(results)
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        assert res[r]["ws"] == 2 and res[r]["rank"] == r and res[r]["backend"] == "gloo"
        assert res[r]["max"] == 2.5
        assert res[r]["ref_rc"] == 0
    assert len(res[0]["ref_lines"]) == 1 and '"impl": "reference"' in res[0]["ref_lines"][0]
    assert res[1]["ref_lines"] == []
