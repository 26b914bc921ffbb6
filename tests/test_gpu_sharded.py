"""The token-sharded forward on the GPU (needs a B200): two ranks, each a
process on cuda:0 joined by a gloo group (gloo sums CUDA tensors through the
host), run `sharded_forward` on their block-aligned slices of one batch.  The
ranks' codes, outputs, selections and importances put back together, and
the summed statistics, are compared with the float64 oracle on the full
inputs, element by element (the same checks as the unsharded parity tests).
One case leaves the second rank without tokens: it still joins the exchange.
No kernel waits on another rank; the only exchange is the host-side
all-reduce between the two stages."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from adaptive_vector_quantized_b200 import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _cfg(N):
    return dict(dtype="bf16", B=1, H=2, N=N, d=64, M0=64, C=8, P=16, block=128, keys="tree",
                key_sigma=0.1, sigma_c=0.3, two_pass=False)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, N, seed, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import adaptive_vector_quantized_b200 as avq
    from adaptive_vector_quantized_b200 import synth as sy
    from adaptive_vector_quantized_b200.sharding import shard_rows, sharded_forward

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = _cfg(N)
        inp = sy.make_inputs(cfg, seed)  # every rank draws the same full inputs
        n0, n1 = shard_rows(N, cfg["block"], rank, world)
        dev = torch.device("cuda", 0)
        sl = lambda t: t[:, :, n0:n1].contiguous().to(dev)  # noqa: E731
        out = sharded_forward(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), inp["parents"].to(dev),
                              inp["children"].to(dev), cfg["P"], cfg["block"], scale=inp["scale"],
                              importance=True)
        avq.avq_check_device()
        torch.cuda.synchronize()
        assign, vsum, counts, O, sel, imp = out
        q.put((rank, n0, n1, assign.cpu().numpy(), vsum.cpu().numpy(), counts.cpu().numpy(),
               O.cpu().view(torch.int16).numpy(), sel.cpu().numpy(), imp.cpu().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N,seed", [(1000, 41), (100, 42)])
def test_sharded_forward_two_ranks_on_one_gpu(N, seed):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, WORLD, port, N, seed, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(WORLD)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spans = [(r[1], r[2]) for r in res]
    assert spans[0][0] == 0 and spans[-1][1] == N
    if N <= 128:
        assert spans[1][0] == spans[1][1], "the second rank should hold no tokens"
    # the exchanged statistics are the same on every rank
    for r in res[1:]:
        assert np.array_equal(r[5], res[0][5])
        assert np.array_equal(r[4], res[0][4])
    inp = synth.make_inputs(_cfg(N), seed)
    full = dict(assign=np.concatenate([r[3] for r in res], axis=2), vsum=res[0][4], counts=res[0][5],
                O=torch.from_numpy(np.concatenate([r[6] for r in res], axis=2)).view(torch.bfloat16),
                sel=np.concatenate([r[7] for r in res], axis=2),
                imp=np.concatenate([r[8] for r in res], axis=2))
    assert full["assign"].shape == (1, 2, N)
    diag = gh.check_forward(inp, full)
    print("sharded", N, spans, diag)
