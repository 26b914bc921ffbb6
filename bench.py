#!/usr/bin/env python3
"""Throughput of the AVQ-Attention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config long] [--impl avq|reference]
    (--config: a named workload, "sweep:P:N[:order]" or "flat192:N")

One step = stage 1 (avq_quantize: full-tree key quantisation + aggregation)
and stage 2 (avq_attention: parent attention, top-P per query block, child
refinement) over one batch of the workload, inputs already resident in HBM.
Metric: queries/s = B*H*N per step / step time, whole job over all ranks
(weak scaling: every rank runs its own independent batch; there is no
collective on the data path).  Rank 0 prints one JSON line.

`--impl reference` times the float64 CPU oracle instead, on a bounded sample
of the same workload (rank 0 only): min(H, host cores) heads of one batch.

`--gpus N` with N > 1, run without a distributed launcher, starts N ranks
itself (torch.distributed.run on 127.0.0.1); under a launcher the world size
must equal N.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import re
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "AVQ fwd queries/s at N=64K,M0=64,C=8,P=16,d=64; % of HBM/TC roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="long")
    ap.add_argument("--impl", default="avq", choices=["avq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--shard", default="batch", choices=["batch", "tokens"],
                    help="batch: every rank runs its own batch (weak scaling); tokens: the ranks "
                         "split one batch's tokens and sum the statistics (strong scaling)")
    ap.add_argument("--denominator", default=None, choices=["auto", "two_pass", "extrapolated"],
                    help="importance denominator for parent codebooks over several tiles "
                         "(default: the workload's own setting)")
    ap.add_argument("--profile", action="store_true",
                    help="for profiler runs: no clock soak, no end-to-end leg, no CPU baseline")
    ap.add_argument("--graph", action="store_true",
                    help="capture each stage's library call once as a CUDA graph and replay the graphs "
                         "in the timed steps (the same kernels without the host's per-call launch work)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def algorithmic3(cfg):
    """Bytes and tensor-free FLOPs of a depth-3 step (parents, M0*C children,
    M0*C*C grandchildren; P parents and P2 children refined per block)."""
    B, H, N, d, M0, C, P, blk = (cfg[k] for k in ("B", "H", "N", "d", "M0", "C", "P", "block"))
    P2 = cfg.get("P2", P)
    s = 2 if cfg["dtype"] == "bf16" else 4
    BH = B * H
    Mt = M0 + M0 * C + M0 * C * C
    nblk = -(-N // blk)
    stats = BH * Mt * (4 * d + 4)
    code = H * Mt * d * s
    s1_bytes = 2 * BH * N * d * s + code + stats + 4 * BH * N
    s1_flops = 2 * BH * N * (M0 + 2 * C) * d
    s2_bytes = BH * N * d * 2 * s + stats + code + 4 * BH * nblk * (P + P2)
    s2_flops = 4 * BH * N * (M0 + P * C + P2 * C) * d + 2 * BH * N * P * C * d
    return dict(s1_bytes=s1_bytes, s1_flops=s1_flops, s2_bytes=s2_bytes, s2_flops=s2_flops)


def algorithmic(cfg):
    """Bytes and tensor FLOPs the method must move/compute per step, per stage.

    Stage 1 reads K and V once, the codebook once per head and writes the
    assignments and the statistics; stage 2 reads Q, the codebook and the
    statistics and writes O and the selections.  FLOPs count the score
    contractions and the value products (2 per multiply-add)."""
    B, H, N, d, M0, C, P, blk = (cfg[k] for k in ("B", "H", "N", "d", "M0", "C", "P", "block"))
    s = 2 if cfg["dtype"] == "bf16" else 4
    BH = B * H
    Mt = M0 * (1 + C)
    nblk = -(-N // blk)
    stats = BH * Mt * (4 * d + 4)
    code = H * Mt * d * s
    s1_bytes = 2 * BH * N * d * s + code + stats + 4 * BH * N
    s1_flops = 2 * BH * N * (M0 + C) * d
    s2_bytes = BH * N * d * (s + s) + stats + code + 4 * BH * nblk * P
    s2_flops = 4 * BH * N * (M0 + P * C) * d
    return dict(s1_bytes=s1_bytes, s1_flops=s1_flops, s2_bytes=s2_bytes, s2_flops=s2_flops)


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(self.out or "")) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for k, nm in enumerate(names):
                if r[5 + k].strip().lower() == "active":
                    reasons.add(nm)
        sm.sort()
        return dict(sm_mhz=sm[len(sm) // 2] if sm else None, sm_max_mhz=max(smax) if smax else None,
                    reasons=sorted(reasons), samples=len(rows))


def src_sha(path):
    """Hash of a kernel source with comments and blank space removed, so that a
    comment edit keeps the recorded counters while any code change drops them."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", " ", text).strip()
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def traffic_for(kernel_file, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rows = json.load(open(p))
    except ValueError:
        return None
    src = os.path.join(ROOT, "adaptive_vector_quantized_b200", "csrc", kernel_file)
    for r in rows:
        if r.get("file") == kernel_file and r.get("workload") == workload and \
                os.path.exists(src) and r.get("source_sha") == src_sha(src):
            return r.get("bytes_per_launch")
    return None


def max_over_ranks(ms, device, world):
    """The slowest rank's time: every rank contributes, every rank gets the max."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base, rank):
    """Each rank runs its own independent batch (weak scaling)."""
    return base + 17 * rank


# ---------------------------------------------------------------------------
def cpu_oracle_sample(inp, heads, steps=1):
    """Time the float64 oracle (Alg. 1 + Alg. 2) on `heads` heads of the
    workload: every key and every query of those heads."""
    import oracle

    orc = oracle.default()
    # every host core (a distributed launcher sets OMP_NUM_THREADS=1 per rank;
    # the oracle runs on rank 0 alone)
    orc.set_threads(max(1, os.cpu_count() or 1))
    Kh = inp["K"][:1, :heads]
    Vh = inp["V"][:1, :heads]
    Qh = inp["Q"][:1, :heads]
    par = inp["parents"][:heads]
    ch = inp["children"][:heads]
    K64, V64, Q64 = (oracle._f64(t) for t in (Kh, Vh, Qh))
    p64, c64 = oracle._f64(par), oracle._f64(ch)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        a, vs, n, _ = orc.quantize(K64, V64, p64, c64)
        orc.attention(Q64, p64, c64, vs, n, inp["P"], inp["block"], inp["scale"])
        times.append(time.perf_counter() - t0)
    return heads * inp["N"], times, orc.num_threads()


def run_reference(args, cfg, inp):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle  # noqa: F401  (the reference arm is the oracle)

    heads = inp["H"]  # min(H, host cores): the oracle's stage 1 parallelises over heads
    queries, times, cores = cpu_oracle_sample(inp, heads, steps=args.warmup + args.steps)
    timed = times[args.warmup:]
    t = sum(timed)
    value = queries * len(timed) / t
    sample = (f"{heads} of the workload's {cfg['H']} heads x N={inp['N']} (b=0): all keys quantised "
              f"and all queries attended per step, float64, OpenMP")
    rcfg = dict(workload_config(args.config, cfg), B=1, H=heads, heads_of_workload=cfg["H"],
                batches_of_workload=cfg["B"])
    line = dict(metric=METRIC, value=value, unit="queries/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * t / len(timed), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=rcfg,
                cpu_baseline=dict(value=value, unit="queries/s", cores=cores, kind="oracle",
                                  sample=sample),
                e2e=dict(value=value, unit="queries/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def workload_config(name, cfg):
    keys = ("B", "H", "N", "d", "M0", "C", "P", "block")
    out = {"workload": name}
    out.update({k: cfg[k] for k in keys})
    if cfg.get("depth", 2) == 3:
        out.update(depth=3, P2=cfg.get("P2", cfg["P"]))
    out["order"] = cfg.get("order", "natural")
    out["two_pass"] = int(cfg.get("two_pass", False))
    return out


# ---------------------------------------------------------------------------
def run_avq(args, cfg, inp, n_global=None):
    """n_global: with --shard tokens, the tokens of all ranks (cfg and inp
    then hold this rank's slice)."""
    import torch
    import torch.distributed as dist

    import adaptive_vector_quantized_b200 as avq
    from adaptive_vector_quantized_b200.sharding import allreduce_stats

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    B, H, N, d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
    P, block = cfg["P"], cfg["block"]
    two_pass = int(cfg.get("two_pass", False))
    Q, K, V = (inp[k].to(dev) for k in ("Q", "K", "V"))
    par = inp["parents"].to(dev)
    ch = inp["children"].to(dev) if cfg["C"] > 0 else None
    stream = torch.cuda.current_stream(dev)
    dims = avq.avq_dims(B, H, N, d, cfg["M0"], cfg["C"])
    dt = avq.AVQ_BF16 if cfg["dtype"] == "bf16" else avq.AVQ_F32
    depth3 = cfg.get("depth", 2) == 3
    ws = None if depth3 else avq.workspace(dims, dt, dev, two_pass=two_pass, P=P, block=block)
    Mt = avq.m_total3(cfg["M0"], cfg["C"]) if depth3 else cfg["M0"] * (1 + cfg["C"])
    nblk = -(-N // block)
    assign = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    vsum = torch.empty((B, H, Mt, d), dtype=torch.float32, device=dev)
    counts = torch.empty((B, H, Mt), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    sel = torch.empty((B, H, nblk, P), dtype=torch.int32, device=dev)
    gch = inp["grandchildren"].to(dev) if depth3 else None

    exchange = n_global is not None and world > 1

    def quantize(Kb, Vb, st=stream):
        if depth3:
            avq.avq_quantize3(Kb, Vb, par, ch, gch, assign, vsum, counts, stream=st)
        else:
            avq.avq_quantize(Kb, Vb, par, ch, assign, vsum, counts, ws=ws, stream=st)

    def attend(Qb, Ob, selb, st=stream):
        """Stage 2; returns the parent selection it wrote."""
        if depth3:
            return avq.avq_attention3(Qb, par, ch, gch, vsum, counts, P, cfg.get("P2", P), block, inp["scale"],
                                      O=Ob, stream=st)[1]
        avq.avq_attention(Qb, par, ch, vsum, counts, P, block, inp["scale"], two_pass, Ob, selb,
                          ws=ws, stream=st)
        return selb

    last_sel = [sel]

    def step(bufs=None):
        Qb, Kb, Vb, Ob, selb = bufs if bufs is not None else (Q, K, V, O, sel)
        quantize(Kb, Vb)
        k1 = avq.last_kernels()
        if exchange:
            allreduce_stats(vsum, counts)
        last_sel[0] = attend(Qb, Ob, selb)
        return k1, avq.last_kernels()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    # inputs that fit in L2 (126 MB on B200) would be timed warm: write a
    # buffer of twice the L2 size between timed steps
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    in_bytes = 3 * B * H * N * d * Q.element_size()
    fbuf = torch.empty(2 * l2_bytes // 4 + 1, dtype=torch.float32, device=dev) if in_bytes < 2 * l2_bytes else None
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        wall0 = time.time()
        for _ in range(args.warmup):
            k1, k2 = step()
        avq.avq_check_device(stream)
        kernels_per_step = len(k1.split()) + len(k2.split())
        # untimed soak so that the clock sampler sees the GPU under this load
        soak = 0
        while not args.profile and time.time() - wall0 < 1.0:
            step()
            soak += 1
            if soak % 32 == 0:
                torch.cuda.synchronize(dev)
        # --graph: each stage's call captured once (on a side stream, as graph
        # capture requires) and replayed on the timing stream
        gq = ga = None
        if args.graph:
            if exchange:
                raise SystemExit("--graph is not offered with the token-sharded statistics exchange")
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            gq, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(gq, stream=cap, capture_error_mode="relaxed"):
                quantize(K, V, st=cap)
            with torch.cuda.graph(ga, stream=cap, capture_error_mode="relaxed"):
                attend(Q, O, sel, st=cap)
            stream.wait_stream(cap)
            for _ in range(3):
                gq.replay()
                ga.replay()
            avq.avq_check_device(stream)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for s in range(args.steps):
            if fbuf is not None:  # inputs fit in L2: evict them before every timed step
                fbuf.zero_()
            ev[s][0].record(stream)
            if gq is not None:
                gq.replay()
            else:
                quantize(K, V)
            if exchange:
                allreduce_stats(vsum, counts)
            ev[s][1].record(stream)
            if ga is not None:
                ga.replay()
            else:
                attend(Q, O, sel)
            ev[s][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    avq.avq_check_device(stream)
    t_s1 = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    t_s2 = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    if fbuf is None:
        ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    else:  # the flushes are outside the steps' own events
        ms = max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in ev), dev, world)
    ms_step = ms / args.steps
    queries = B * H * N * world if n_global is None else B * H * n_global
    value = queries / (ms_step * 1e-3)

    # end to end through the public API with host buffers: every step copies
    # its Q, K, V in from pinned host memory and its O and selections out.
    # The steps are pipelined as a streaming caller would run them: inputs on
    # a copy-in stream, outputs on a copy-out stream, two device buffer sets,
    # so step i+1's inputs cross the link while step i computes and step i's
    # outputs go back while step i+1's inputs come in (the link is full duplex).
    e2e = None
    if not args.no_e2e and not args.profile:
        hQ, hK, hV = (inp[k].pin_memory() for k in ("Q", "K", "V"))
        hO = [torch.empty(O.shape, dtype=O.dtype).pin_memory() for _ in range(2)]
        hsel = [torch.empty(sel.shape, dtype=sel.dtype).pin_memory() for _ in range(2)]
        bufs = [(Q, K, V, O, sel), tuple(torch.empty_like(t) for t in (Q, K, V, O, sel))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(n):
            s_in.wait_stream(stream)
            read = [None, None]  # per buffer set: its last step has read its inputs
            sent = [None, None]  # per buffer set: its last outputs are on the host
            for i in range(n):
                b = i % 2
                Qb, Kb, Vb, Ob, selb = bufs[b]
                with torch.cuda.stream(s_in):
                    if read[b] is not None:
                        s_in.wait_event(read[b])
                    Qb.copy_(hQ, non_blocking=True)
                    Kb.copy_(hK, non_blocking=True)
                    Vb.copy_(hV, non_blocking=True)
                    arrived = torch.cuda.Event()
                    arrived.record(s_in)
                stream.wait_event(arrived)
                if sent[b] is not None:
                    stream.wait_event(sent[b])
                step(bufs[b])
                read[b] = torch.cuda.Event()
                read[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(read[b])
                    hO[b].copy_(Ob, non_blocking=True)
                    last_sel[0].record_stream(s_out)  # a selection the binding allocated
                    hsel[b].copy_(last_sel[0], non_blocking=True)
                    sent[b] = torch.cuda.Event()
                    sent[b].record(s_out)
            stream.wait_stream(s_out)
            stream.wait_stream(s_in)

        e2e_run(2)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 10))
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        a0.record(stream)
        e2e_run(n_e2e)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(a0.elapsed_time(a1), dev, world)
        h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV))
        d2h = hO[0].numel() * hO[0].element_size() + hsel[0].numel() * hsel[0].element_size()
        e2e = dict(value=queries / (ems / n_e2e * 1e-3), unit="queries/s", h2d_bytes_per_step=h2d,
                   d2h_bytes_per_step=d2h, steps=n_e2e)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = load_peaks()
    alg = algorithmic3(cfg) if depth3 else algorithmic(cfg)
    s1_gbs = alg["s1_bytes"] / (t_s1 * 1e-3) / 1e9
    s2_gbs = alg["s2_bytes"] / (t_s2 * 1e-3) / 1e9
    s2_tfs = alg["s2_flops"] / (t_s2 * 1e-3) / 1e12
    t_roof = (max(alg["s1_bytes"] / (peaks["hbm"] * 1e9), alg["s1_flops"] / (peaks["bf16"] * 1e12))
              + max(alg["s2_bytes"] / (peaks["hbm"] * 1e9), alg["s2_flops"] / (peaks["bf16"] * 1e12)))
    # The roofline object describes the attention kernel, the largest single
    # kernel of the step in the ncu launch list (the stage-2 time also holds its
    # 1% image-preparation kernel).  Stage 1 is reported under "stages".
    achieved = alg["s2_bytes"] / (t_s2 * 1e-3) / 1e9
    att = "attention3_tc" if depth3 else "attention_tc"
    roofline = dict(bound="hbm", achieved=achieved, peak=peaks["hbm"], unit="GB/s",
                    frac=achieved / peaks["hbm"], traffic=traffic_for(att + ".cu", args.config),
                    kernel=att, peak_source=peaks["source"],
                    step_roofline_us=t_roof * 1e6, step_frac=t_roof * 1e3 / ms_step)
    cpu = None
    if not args.no_cpu_baseline and not args.profile and world == 1 and not depth3:  # rank 0 at N=1 only
        heads = min(cfg["H"], max(1, os.cpu_count() or 1))
        q, times, cores = cpu_oracle_sample(inp, heads, steps=1)
        cpu = dict(value=q / times[0], unit="queries/s", cores=cores, kind="oracle",
                   sample=f"{heads} head(s) x N={N} of the same workload, b=0: all keys quantised "
                          f"and all queries attended, float64, OpenMP")
    l2_note = ("inputs larger than L2 (Q, K, V %.0f MB each per step); no flush" % (in_bytes / 3e6)
               if fbuf is None else
               "inputs smaller than 2x L2: a %.0f MB buffer written before every timed step, "
               "outside the step's events" % (fbuf.numel() * 4 / 1e6))
    line = dict(metric=METRIC, value=value, unit="queries/s", n_gpus=world, steps=args.steps,
                warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
                scaling="weak" if n_global is None else "strong",
                vs_baseline=None, dtype=cfg["dtype"], data="synthetic",
                config=dict(workload_config(args.config, cfg),
                            l2=l2_note, **({"launch": "CUDA graph replay of each stage's call"}
                                           if args.graph else {})),
                roofline=roofline, cpu_baseline=cpu, e2e=e2e,
                gpu_launches=kernels_per_step * args.steps,
                clocks=dict(clk.summary() or {}, window=f"sampled every 200 ms over warmup, "
                            f"{soak} untimed soak steps and the timed steps"),
                stages=dict(quantize_us=t_s1 * 1e3, attention_us=t_s2 * 1e3,
                            quantize_gbs=s1_gbs, attention_gbs=s2_gbs, attention_tflops=s2_tfs,
                            quantize_kernels=k1, attention_kernels=k2))
    print(json.dumps(line), flush=True)


def resolve_config(name):
    """A named workload, or one point of the P x N sweep: "sweep:P:N[:order]"
    (H=8, d=64, 64/P/8, order hilbert, raster or random) or the flat
    192-codeword VQ "flat192:N"."""
    from adaptive_vector_quantized_b200 import synth

    if name in synth.CONFIGS:
        return synth.get_config(name)
    parts = name.split(":")
    try:
        if parts[0] == "sweep" and len(parts) in (3, 4):
            return synth.sweep_config(int(parts[1]), int(parts[2]), parts[3] if len(parts) == 4 else "hilbert")
        if parts[0] == "flat192" and len(parts) == 2:
            return synth.sweep_config(0, int(parts[1]), flat192=True)
    except ValueError as e:
        raise SystemExit(f"bad config {name}: {e}")
    raise SystemExit(f"unknown config {name}")


def config_seed(name, synth):
    base = name.split(":")[0]
    return synth.CONFIG_SEEDS.get(name, synth.CONFIG_SEEDS.get("sweep" if base in ("sweep", "flat192") else base, 1000))


def launch_ranks(args):
    """`--gpus N` with N > 1 outside a distributed launch: start N ranks (one
    per GPU) with torch.distributed.run on this node and return its exit code."""
    import socket

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__)] + sys.argv[1:]
    try:
        return subprocess.run(cmd, timeout=1800).returncode
    except subprocess.TimeoutExpired:
        print("bench: the ranks did not finish within 30 minutes", file=sys.stderr)
        return 124


def main():
    args = parse()
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        raise SystemExit(launch_ranks(args))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        print(f"bench: --gpus {args.gpus} but the launch has {world} rank(s)", file=sys.stderr)
        raise SystemExit(2)
    from adaptive_vector_quantized_b200 import synth

    cfg = resolve_config(args.config)
    if args.denominator is not None:
        cfg["two_pass"] = {"auto": 0, "two_pass": 1, "extrapolated": 2}[args.denominator]
    rank = int(os.environ.get("RANK", "0"))
    seed = rank_seed(args.seed if args.seed is not None else config_seed(args.config, synth), rank)
    if args.impl == "reference":
        if rank != 0:
            return
        heads = min(cfg["H"], max(1, os.cpu_count() or 1))
        inp = synth.make_inputs(dict(cfg, B=1, H=heads), seed)
        run_reference(args, cfg, inp)
        return
    if args.shard == "tokens":  # same inputs on every rank, each takes its slice of the tokens
        from adaptive_vector_quantized_b200.sharding import shard_rows

        world = int(os.environ.get("WORLD_SIZE", "1"))
        base = args.seed if args.seed is not None else config_seed(args.config, synth)
        inp = synth.make_inputs(cfg, base)
        n0, n1 = shard_rows(cfg["N"], cfg["block"], rank, world)
        if n1 <= n0:
            raise SystemExit("more ranks than query blocks")
        for k in ("Q", "K", "V"):
            inp[k] = inp[k][:, :, n0:n1].contiguous()
        run_avq(args, dict(cfg, N=n1 - n0), inp, n_global=cfg["N"])
        return
    inp = synth.make_inputs3(cfg, seed) if cfg.get("depth", 2) == 3 else synth.make_inputs(cfg, seed)
    run_avq(args, cfg, inp)


if __name__ == "__main__":
    main()
