"""Host logic of the N>1 benchmark path on CPU: world-size-2 gloo process
groups check the max-over-ranks timing and the whole-job throughput the
benchmark reports (each rank is an independent replica; there is no
data-path collective), and the reference arm prints its JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, local_ms, q):
    import datetime

    import torch.distributed as dist
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world)})
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    mx = bench.max_over_ranks(local_ms[rank], world)
    gbs = bench.job_throughput(1e9, 10, world, mx)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, gbs))


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    local_ms = [12.5, 20.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, mx, gbs in res:
        assert mx == 20.0  # the slowest rank sets the time
        # 2 ranks x 10 steps x 1 GB in 20 ms
        assert abs(gbs - 2 * 10 * 1e9 / 0.020 / 1e9) < 1e-6


def test_single_rank_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_throughput(2e9, 4, 1, 8.0) == pytest.approx(1000.0)


def test_step_accounting():
    # the headline step: both 70B-shaped layers at M = 1, 16 and 64
    case, probs = bench.case_problems(bench.HEADLINE, bench.HEADLINE_MS)
    assert len(probs) == 6
    assert sum(p[3] for p in probs) == 2 * (1 + 16 + 64)
    # packed weights dominate: 3 x 2 x 8192*28672/4 bytes per step
    w = 3 * 2 * 8192 * 28672 // 4
    step = sum(bench.forward_bytes(M, N, K) for _, K, N, M in probs)
    assert w < step < 1.06 * w   # + activations, x_q round trip and outputs


def test_reference_arm_prints_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                         env=env, timeout=600, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True,
                       env=env, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
