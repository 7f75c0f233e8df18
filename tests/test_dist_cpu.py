"""Multi-rank host logic on CPU (gloo, world size 2): the timing collectives
that turn per-rank times and unit counts into the whole-job throughput, and
the reference arm's rank handling under torchrun."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from video_diffusion_transformer_rms_b200 import dist
    r, lr, w = dist.init("gloo", timeout_s=60)
    # rank 0 processed 100 units in 2 s, rank 1 processed 300 units in 4 s
    units = 100.0 if r == 0 else 300.0
    secs = 2.0 if r == 0 else 4.0
    thr, total, slowest = dist.job_throughput(units, secs)
    mx = dist.max_over_ranks(float(r))
    dist.barrier()
    dist.shutdown()
    q.put((r, w, thr, total, slowest, mx))


def test_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, thr, total, slowest, mx in res:
        assert w == 2
        assert total == 400.0 and slowest == 4.0 and mx == 1.0
        assert thr == 100.0  # 400 units / 4 s: the slowest rank sets the time


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    from video_diffusion_transformer_rms_b200 import dist
    assert not dist.active()
    assert dist.job_throughput(50.0, 2.0) == (25.0, 50.0, 2.0)


def _run_bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_other_ranks_exit_without_work():
    p = _run_bench({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference",
                   "--gpus", "2", "--steps", "1", "--warmup", "0")
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_json_line():
    p = _run_bench({"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "2"}, "--impl", "reference",
                   "--gpus", "2", "--steps", "1", "--warmup", "0")
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] == max(1, min(os.cpu_count() or 1, 32))
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["higher_is_better"] is True
