"""The bench runs its avq arm end to end on the GPU for workloads whose
shapes differ from the headline one: no child refinement (P = 0, an empty
selection output), the flat 192-codeword VQ, and a ragged token count, each
printing one JSON line with the contract's keys; and the CUDA-graph replay
of each stage's call (two-level and depth-3), whose output must equal the
eager calls'."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("config", ["sweep:0:4096", "flat192:4096", "vit28"])
def test_bench_line(config):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", config, "--steps", "2",
                        "--warmup", "3", "--no-cpu-baseline", "--profile"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("{")][-1]
    d = json.loads(line)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "config", "roofline",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 2 and d["config"]["workload"] == config


@pytest.mark.parametrize("config", ["vit28", "deep3"])
def test_bench_graph_replay(config):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", config, "--steps", "2",
                        "--warmup", "3", "--no-cpu-baseline", "--profile", "--graph"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([x for x in r.stdout.splitlines() if x.startswith("{")][-1])
    assert d["value"] > 0 and "launch" in d["config"]


def test_graph_replay_equals_eager():
    """Both stages captured as CUDA graphs through the public calls and
    replayed give bit-identical codes, counts, selections and outputs to the
    eager calls (same kernels, same order)."""
    import torch

    import adaptive_vector_quantized_b200 as avq
    from adaptive_vector_quantized_b200 import synth

    cfg = synth.get_config("vit28")
    inp = synth.make_inputs(cfg, synth.CONFIG_SEEDS["vit28"])
    dev = torch.device("cuda", 0)
    Q, K, V, par, ch = (inp[k].to(dev) for k in ("Q", "K", "V", "parents", "children"))
    P, block = cfg["P"], cfg["block"]
    a, vs, n = avq.avq_quantize(K, V, par, ch)
    O, sel, _ = avq.avq_attention(Q, par, ch, vs, n, P, block, inp["scale"])
    torch.cuda.synchronize()
    ref = [t.clone() for t in (a, vs, n, O, sel)]
    for t in (a, vs, n, O, sel):
        t.zero_()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    gq, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gq, stream=cap, capture_error_mode="relaxed"):
        avq.avq_quantize(K, V, par, ch, assign=a, vsum=vs, counts=n, stream=cap)
    with torch.cuda.graph(ga, stream=cap, capture_error_mode="relaxed"):
        avq.avq_attention(Q, par, ch, vs, n, P, block, inp["scale"], O=O, sel=sel, stream=cap)
    torch.cuda.current_stream(dev).wait_stream(cap)
    for _ in range(2):
        gq.replay()
        ga.replay()
    torch.cuda.synchronize()
    avq.avq_check_device()
    for name, got, want in zip(("assign", "counts", "sel"), (a, n, sel), (ref[0], ref[2], ref[4])):
        assert torch.equal(got, want), name
    # value sums come from red.global.add (order not fixed): within fp32 reordering
    assert torch.allclose(vs, ref[1], rtol=1e-5, atol=1e-4)
    assert (O.float() - ref[3].float()).abs().max().item() <= 2e-2 * V.float().abs().max().item()
