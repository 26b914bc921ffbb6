"""Sharding one head's tokens over ranks (CPU): block-aligned slices, and the
statistics all-reduce of the sharded path, checked with two gloo ranks that
use the float64 oracle for the per-rank compute.  The sum over ranks of the
local Eq. 3 statistics equals the statistics of all keys, and every rank's
output rows equal the unsharded output's rows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from adaptive_vector_quantized_b200.sharding import shard_rows

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N,block,world", [(1000, 128, 2), (4096, 128, 3), (65, 64, 4), (129, 128, 2)])
def test_shard_rows_cover_and_align(N, block, world):
    spans = [shard_rows(N, block, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    for a0, a1 in spans:
        assert (a0 % block == 0 or a0 == N) and a0 <= a1
    sizes = [(a1 - a0 + block - 1) // block for a0, a1 in spans]
    assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(N, block, world, world)


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
    import oracle
    from adaptive_vector_quantized_b200 import synth
    from adaptive_vector_quantized_b200.sharding import allreduce_stats, shard_rows

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = dict(dtype="f32", B=1, H=2, N=1000, d=64, M0=16, C=4, P=4, block=128, keys="tree",
                   key_sigma=0.1, sigma_c=0.3, two_pass=False)
        inp = synth.make_inputs(cfg, 31)  # every rank draws the same full inputs
        orc = oracle.default()
        n0, n1 = shard_rows(cfg["N"], cfg["block"], rank, world)
        sl = lambda t: t[:, :, n0:n1]  # noqa: E731
        _, vs, ns, _ = orc.quantize(sl(inp["K"]), sl(inp["V"]), inp["parents"], inp["children"])
        vs_t, ns_t = torch.from_numpy(vs.copy()), torch.from_numpy(ns.copy())
        allreduce_stats(vs_t, ns_t)
        _, vs_full, ns_full, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
        ok_counts = bool(np.array_equal(ns_t.numpy(), ns_full))
        err_vs = float(np.abs(vs_t.numpy() - vs_full).max() / np.abs(vs_full).max())
        O_loc, _, _ = orc.attention(sl(inp["Q"]), inp["parents"], inp["children"], vs_t.numpy(), ns_t.numpy(),
                                    cfg["P"], cfg["block"], inp["scale"])
        O_full, _, _ = orc.attention(inp["Q"], inp["parents"], inp["children"], vs_full, ns_full,
                                     cfg["P"], cfg["block"], inp["scale"])
        err_o = float(np.abs(O_loc - O_full[:, :, n0:n1]).max())
        q.put((rank, ok_counts, err_vs, err_o, n1 - n0))
    finally:
        dist.destroy_process_group()


def test_sharded_statistics_and_output_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sum(r[4] for r in res) == 1000
    for rank, ok_counts, err_vs, err_o, _ in res:
        assert ok_counts, f"rank {rank}: counts differ"
        assert err_vs < 1e-12 and err_o < 1e-12, (rank, err_vs, err_o)


def _failing_worker(rank, world, port, q):
    """Rank 1 leaves between steps (an exception before the statistics
    exchange); rank 0 must learn of it from its collective, within the
    process group's short timeout, instead of waiting for ever."""
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from adaptive_vector_quantized_b200.sharding import allreduce_stats

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        q.put((1, "left"))
        raise SystemExit(3)  # no destroy_process_group: the rank is simply gone
    vs = torch.ones(1, 2, 80, 64, dtype=torch.float64)
    ns = torch.ones(1, 2, 80, dtype=torch.int64)
    try:
        allreduce_stats(vs, ns)
        q.put((0, "no error"))
    except Exception as e:  # the failure surfaces as an error of the collective
        q.put((0, "error: " + type(e).__name__))


def test_a_lost_rank_surfaces_as_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
            p.join(timeout=10)
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]
    assert procs[1].exitcode == 3
