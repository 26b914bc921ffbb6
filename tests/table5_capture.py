"""Top-P capture of three selections at the large-codebook workload, the
synthetic counterpart of the pages' Table 5 ("AVQ-Attention: Adaptive
Vector-Quantized Attention", Sec. B: tiled importance with the
count-extrapolated denominator, Eqs. 13-14; non-tiled importance with the
exact denominator, Eq. 7; exact selection from the full attention matrix).

Capture = fraction of the true attention mass (exact softmax over all keys)
that falls on keys assigned to a block's selected parents, averaged over
query blocks.  Everything here is the float64 oracle and brute force; no GPU.

    python -m tests.table5_capture [--seeds 1003,1004] [--heads 8] [--coherent 0,1]
"""
from __future__ import annotations

import argparse
import json
import time

import numpy as np

import oracle
from adaptive_vector_quantized_b200 import synth
from oracle import brute


def capture_row(inp, tiles=(128, 64)):
    orc = oracle.default()
    assign, vsum, counts, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
    args = (inp["parents"], inp["children"], vsum, counts, inp["P"], inp["block"], inp["scale"])
    mass = brute.parent_attention_mass(inp["Q"], inp["K"], assign, inp["M0"], inp["C"],
                                       inp["block"], inp["scale"])
    N, block, P = inp["N"], inp["block"], inp["P"]
    exact_sel = np.argsort(-mass, axis=-1, kind="stable")[..., :P]
    out = {"exact": brute.top_p_capture(mass, exact_sel, N, block)}
    _, sel_x, _ = orc.attention(inp["Q"], *args)
    out["non_tiled"] = brute.top_p_capture(mass, sel_x, N, block)
    for t in tiles:
        _, sel_t, _ = orc.attention(inp["Q"], *args, tile=t)
        out[f"tiled_{t}"] = brute.top_p_capture(mass, sel_t, N, block)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--seeds", default="1003,1004,1005")
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--coherent", default="0,1")
    ap.add_argument("--P", default="24,32")
    a = ap.parse_args()
    for g in (float(x) for x in a.coherent.split(",")):
        for P in (int(x) for x in a.P.split(",")):
            rows = []
            for seed in (int(s) for s in a.seeds.split(",")):
                cfg = synth.get_config("largecb", H=a.heads, P=P, q_coherent=g)
                t0 = time.time()
                r = capture_row(synth.make_inputs(cfg, seed))
                r.update(seed=seed, seconds=round(time.time() - t0, 1))
                rows.append(r)
            keys = [k for k in rows[0] if k not in ("seed", "seconds")]
            mean = {k: float(np.mean([r[k] for r in rows])) for k in keys}
            print(json.dumps(dict(q_coherent=g, P=P, heads=a.heads, mean=mean, rows=rows)), flush=True)


if __name__ == "__main__":
    main()
