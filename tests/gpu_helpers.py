"""Running the CUDA path through the Python binding of the C ABI (GPU tests)."""
from __future__ import annotations

import numpy as np
import torch

import adaptive_vector_quantized_b200 as avq
import oracle
from tests import parity


def to_dev(inp):
    out = dict(inp)
    for k in ("Q", "K", "V", "parents", "children"):
        out[k] = inp[k].cuda().contiguous()
    return out


def gpu_forward(inp, P=None, block=None, two_pass=None, path=avq.AVQ_PATH_AUTO,
                deterministic=False, dev=None, apath=None, scale=None):
    """Both stages on the GPU; returns CPU copies and the kernels launched.
    `path` selects the kernel family of both stages, `apath` overrides it for
    the attention stage."""
    P = inp["P"] if P is None else P
    block = inp["block"] if block is None else block
    two_pass = inp.get("two_pass", False) if two_pass is None else two_pass
    d = dev or to_dev(inp)
    ch = d["children"] if inp["C"] > 0 else None
    old = avq.avq_set_path(path)
    try:
        assign, vsum, counts = avq.avq_quantize(d["K"], d["V"], d["parents"], ch,
                                                deterministic=deterministic)
        k1 = avq.last_kernels()
        avq.avq_set_path(path if apath is None else apath)
        O, sel, imp = avq.avq_attention(d["Q"], d["parents"], ch, vsum, counts, P, block,
                                        scale=inp["scale"] if scale is None else scale,
                                        two_pass=two_pass, importance=True)
        k2 = avq.last_kernels()
        avq.avq_check_device()
    finally:
        avq.avq_set_path(old)
    torch.cuda.synchronize()
    return dict(assign=assign.cpu().numpy(), vsum=vsum.cpu().numpy(), counts=counts.cpu().numpy(),
                O=O.cpu(), sel=sel.cpu().numpy(), imp=imp.cpu().numpy(), kernels=(k1 + " " + k2))


def check_forward(inp, res, P=None, block=None, blocks=None, tile=0):
    """Full parity of one forward against the oracle; `blocks` limits the
    attention check to a list of (bh, block) pairs; `tile` > 0 compares the
    importance and selection with the oracle's tiled, count-extrapolated
    importance over parent tiles of that size.  Returns diagnostics."""
    orc = oracle.default()
    P = inp["P"] if P is None else P
    block = inp["block"] if block is None else block
    M0, C = inp["M0"], inp["C"]
    o_assign, _, _, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
    n_ties = parity.check_assign(res["assign"], o_assign, inp["K"], inp["parents"], inp["children"])
    ref_vs, ref_n = orc.aggregate(res["assign"], inp["V"], M0, C)
    abs_vs, _ = orc.aggregate(res["assign"], inp["V"].abs() if hasattr(inp["V"], "abs") else np.abs(inp["V"]), M0, C)
    parity.check_stats(res["vsum"], res["counts"], ref_vs, ref_n, abs_vs)
    # importance and selection against the oracle on the same statistics
    _, o_sel, o_imp = orc.attention(inp["Q"], inp["parents"], inp["children"], ref_vs, ref_n, P,
                                    block, inp["scale"], blocks=blocks, tile=tile)
    B, H = inp["B"], inp["H"]
    nblk = res["sel"].shape[2]
    mask_blk = np.ones((B, H, nblk), dtype=bool)
    if blocks is not None:
        mask_blk[:] = False
        for bh, b in blocks:
            mask_blk[bh // H, bh % H, b] = True
    # importance: fp32 block sums of A n / z against float64, relative to each
    # entry (1e-4), with a 1e-6 floor for entries that underflow in fp32
    # (a block's importances sum to its row count, up to 128)
    g_imp, r_imp = res["imp"][mask_blk], o_imp[mask_blk]
    imp_err = float(np.max(np.abs(g_imp - r_imp) / (np.abs(r_imp) + 1e-6)))
    assert imp_err <= 1e-4, f"importance off by {imp_err} (relative)"
    gsel = res["sel"][mask_blk]
    differ = parity.check_sel(gsel, o_imp[mask_blk], P) if P > 0 else 0
    if P > 0:
        parity.check_order(gsel, res["imp"][mask_blk])
    # output against the oracle rerun on the GPU's own selection
    O_ref, _, _ = orc.attention(inp["Q"], inp["parents"], inp["children"], ref_vs, ref_n, P,
                                block, inp["scale"], sel=res["sel"] if P > 0 else None,
                                blocks=blocks)
    rows = None
    if blocks is not None:
        rows = np.zeros((B, H, inp["N"]), dtype=bool)
        for bh, b in blocks:
            rows[bh // H, bh % H, b * block:(b + 1) * block] = True
    rel = parity.check_output(res["O"], O_ref, inp["V"], inp["dtype"], rows=rows)
    return dict(near_tie_keys=n_ties, sel_blocks_differ=differ, O_rel_err=rel, imp_err=imp_err)
