"""Multi-rank host logic of the benchmark with the gloo backend (CPU only):
the timed value is the max over ranks, ranks get independent batches, and
the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.max_over_ranks(10.0 * (rank + 1), "cpu", world)
        q.put((rank, m, bench.rank_seed(1002, rank)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [20.0, 20.0]
    assert got[0][2] != got[1][2]


def test_reference_arm_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "1", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    # a launch whose world size is not --gpus is refused
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "1", "--gpus", "4"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode != 0 and "rank" in r.stderr
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "1", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_bench_spawns_its_own_ranks():
    """`--gpus 2` without a launcher starts two ranks itself; the reference
    arm then prints one line from rank 0 with n_gpus = 2."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "1", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["impl"] == "reference"


def test_bench_config_names():
    """Named workloads, sweep points and the flat 192-codeword VQ resolve to
    the generator's configs; unknown or malformed names stop the bench."""
    import pytest

    import bench
    from adaptive_vector_quantized_b200 import synth

    assert bench.resolve_config("long") == synth.get_config("long")
    c = bench.resolve_config("sweep:64:4096:random")
    assert (c["P"], c["N"], c["order"], c["H"], c["M0"], c["C"]) == (64, 4096, "random", 8, 64, 8)
    assert bench.resolve_config("sweep:4:16384")["order"] == "hilbert"
    f = bench.resolve_config("flat192:65536")
    assert (f["M0"], f["C"], f["P"]) == (192, 0, 0)
    assert bench.config_seed("sweep:4:16384", synth) == synth.CONFIG_SEEDS["sweep"]
    assert bench.config_seed("vit28", synth) == synth.CONFIG_SEEDS["vit28"]
    for bad in ("nope", "sweep:4", "sweep:x:4096", "sweep:4:1000"):
        with pytest.raises(SystemExit):
            bench.resolve_config(bad)
