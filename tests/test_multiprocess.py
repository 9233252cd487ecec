"""The multi-rank paths of bench.py on CPU (gloo, world size 2).

Every (batch, KV head) unit is independent, so N processes decode N batches
with no collective on the data path; the only cross-rank steps are the
barrier and the reduction of the timed result: the work summed over ranks,
the time as the maximum over ranks.  These tests run that reduction on two
gloo ranks, and the reference arm under torchrun with two ranks (rank 0
alone measures and prints).
"""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import torch.distributed as dist
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _aggregate_worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    import bench
    work, t = bench.aggregate(1000 * (rank + 1), 0.25 * (rank + 1), dist)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"work": work, "time": t}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_work_is_summed_and_time_is_the_max_over_two_ranks(tmp_path):
    tmp.spawn(_aggregate_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    for rank in range(2):
        got = json.load(open(tmp_path / f"rank{rank}.json"))
        assert got == {"work": 3000.0, "time": 0.5}


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny_f32", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--ref-seconds-per-step", "0.05"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
