"""The multi-process plumbing of bench.py on CPU: two gloo ranks, the
max-over-ranks timing, the replica throughput, and the reference arm's
rank handling under a launcher (rank 0 alone prints its line)."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_init()
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    bench.barrier(w)
    secs = 1.0 + rank            # rank 1 is the slow one
    m = bench.max_over_ranks(secs, w)
    out.put((rank, m, bench.replica_throughput(1_000_000, 100, m, w)))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [2.0, 2.0]
    # 2 ranks x 1 MB x 100 launches in 2 s
    assert all(abs(g[2] - 0.1) < 1e-12 for g in got)


def _run_bench(env, *args):
    e = dict(os.environ, **env)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=e, timeout=300)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench({"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}, "--impl", "reference", "--gpus", "2")
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _run_bench({"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"}, "--impl", "reference", "--gpus", "2",
                   "--steps", "5", "--warmup", "3", "--cpu-budget", "0.5")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["steps"] == 5 and d["warmup"] == 3 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["sample"].startswith("5 timed + 3 untimed steps")
