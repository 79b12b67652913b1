"""The bench's N > 1 path on CPU. Two ranks on gloo (127.0.0.1) drive the same
cross-rank helpers that the GPU run drives on NCCL: the maximum over ranks of
the timed region, the unanimous host-memory decision, and the whole-job
tokens/s. The reference arm launched by torchrun on two ranks prints one line,
from rank 0, while rank 1 exits 0 without work."""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    r = bench.Ranks(torch, dist, torch.device("cpu"))
    res = {"max": r.allmax(rank + 1.5), "all_true": r.all_ok(True), "one_false": r.all_ok(rank == 0)}
    # rank 1's host has less memory: both ranks must take the abort branch together
    avail = (100 << 30) if rank == 0 else (15 << 30)
    res["ram"] = r.all_ok(bench.host_ram_fits(5 << 30, world, avail))
    r.barrier()
    # the slower rank's time decides the whole-job value
    t = r.allmax(1.0 + rank)
    res["value"] = bench.weak_value(1000, world, 5, t)
    dist.destroy_process_group()
    q.put((rank, res))


def test_cross_rank_helpers_on_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        assert out[rank]["max"] == 2.5
        assert out[rank]["all_true"] is True
        assert out[rank]["one_false"] is False
        assert out[rank]["ram"] is False
        assert out[rank]["value"] == 1000 * 2 * 5 / 2.0


def test_host_ram_rule():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.host_ram_fits(20 << 30, 8, 196 << 30)         # eight 1.3B replicas with the gradient ring
    assert not bench.host_ram_fits(25 << 30, 8, 196 << 30)     # not with a full gradient arena
    assert bench.host_ram_fits(1, 1, None)                    # unknown host memory: no refusal


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "tiny", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "OMP_NUM_THREADS": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # every key the bench line carries, with the reference arm's own values
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 0
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"] and cb["cpu_model"]
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["unit"] == line["unit"]
    assert line["e2e"]["d2h_bytes_per_step"] == 0
