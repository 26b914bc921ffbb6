"""One head's tokens sharded over ranks, with one exchange step.

Every rank holds a contiguous slice of the same heads' keys, values and
queries.  Stage 1 runs on the local keys; the statistics of Eq. 3 are sums
over keys, so the global statistics are the sum over ranks of the local ones:
one all-reduce (sum) of the value sums and counts, BH * Mt * (d + 1) * 4
bytes.  Stage 2 then runs on the local queries against the global
statistics.  The slices are cut at query-block boundaries, so every block of
`block` queries (which selects its own top-P parents) lives on one rank and
the result equals the unsharded one up to the order of the float sums.

The compute stays in the CUDA kernels (`avq_quantize`, `avq_attention`); the
exchange is a `torch.distributed` all-reduce (NCCL over NVLink on GPUs).
"""
from __future__ import annotations


def shard_rows(N: int, block: int, rank: int, world: int) -> tuple[int, int]:
    """[start, end) of this rank's tokens: whole blocks of `block`, spread as
    evenly as possible, earlier ranks taking the extra blocks; the last rank's
    slice ends at N (its last block may be partial)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    nblk = -(-N // block)
    base, extra = divmod(nblk, world)
    b0 = rank * base + min(rank, extra)
    b1 = b0 + base + (1 if rank < extra else 0)
    return min(N, b0 * block), min(N, b1 * block)


def allreduce_stats(vsum, counts, group=None):
    """Sum the local Eq. 3 statistics over the ranks of `group`, in place."""
    import torch.distributed as dist

    dist.all_reduce(vsum, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return vsum, counts


def sharded_forward(Q, K, V, parents, children, P: int, block: int = 128, scale=None,
                    two_pass=0, group=None, stream=None, importance=False):
    """Both stages on this rank's slices Q, K, V [B,H,n_local,d] (cut by
    `shard_rows`), with the statistics summed over `group` in between.
    Returns (assign, vsum, counts, O, sel): local codes, global statistics,
    local output and selections; with `importance` also the local blocks'
    importances [B,H,nblk_local,M0] as a sixth item."""
    import torch

    import adaptive_vector_quantized_b200 as avq

    B, H, n, d = K.shape
    if n == 0:  # a rank without tokens still takes part in the exchange
        M0 = parents.shape[1]
        C = 0 if children is None else children.shape[2]
        Mt = M0 * (1 + C)
        vsum = torch.zeros((B, H, Mt, d), dtype=torch.float32, device=K.device)
        counts = torch.zeros((B, H, Mt), dtype=torch.int32, device=K.device)
        allreduce_stats(vsum, counts, group)
        empty = torch.empty((B, H, 0), dtype=torch.int32, device=K.device)
        out = (empty, vsum, counts, Q, torch.empty((B, H, 0, P), dtype=torch.int32, device=K.device))
        if importance:
            out += (torch.empty((B, H, 0, M0), dtype=torch.float32, device=K.device),)
        return out
    assign, vsum, counts = avq.avq_quantize(K, V, parents, children, stream=stream)
    allreduce_stats(vsum, counts, group)
    O, sel, imp = avq.avq_attention(Q, parents, children, vsum, counts, P, block, scale=scale,
                                    two_pass=two_pass, stream=stream, importance=importance)
    if importance:
        return assign, vsum, counts, O, sel, imp
    return assign, vsum, counts, O, sel
