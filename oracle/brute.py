"""Independent closed forms that pin the oracle (test infrastructure only).

Written separately from `avq_oracle.c` and vectorised with numpy, so that a
mistake in the step-by-step oracle shows up as a disagreement here.

- `assign_brute`: nearest parent, then nearest child of that parent, moved
  only when strictly closer (Sec. 4.2; Alg. 1), by full distance tables.
- `aggregate_brute`: value sums and counts of Eq. 3 for a two-level tree.
- `representative_attention`: the identity behind the correcting attention
  (Sec. C, Eqs. 15-17): AVQ output equals exact softmax attention over keys
  that are each replaced by a representative -- the child when the key moved
  to a child whose parent is selected for the query's block, else the parent.
- `flat_vq_attention`: VQ attention over a fixed codebook (Eq. 4).
- `exact_attention`: softmax attention (Eq. 1), logits scaled by `scale`.
- `importance_brute`: Eq. 7 written as a block sum of the flat-VQ softmax
  mass of each parent, n_j exp(s_ij) / sum_l n_l exp(s_il).
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    if hasattr(a, "detach"):
        import torch

        a = a.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def assign_brute(K, parents, children):
    """Final codes [B,H,N] from full distance tables."""
    K, parents, children = _f64(K), _f64(parents), _f64(children)
    B, H, N, d = K.shape
    M0 = parents.shape[1]
    C = children.shape[2]
    codes = np.empty((B, H, N), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            k = K[b, h]
            dp = ((k[:, None, :] - parents[h][None, :, :]) ** 2).sum(-1)  # [N, M0]
            a = dp.argmin(axis=1)  # first minimum
            best = dp[np.arange(N), a]
            if C == 0:
                codes[b, h] = a
                continue
            ch = children[h][a]  # [N, C, d]
            dc = ((k[:, None, :] - ch) ** 2).sum(-1)  # [N, C]
            c = dc.argmin(axis=1)
            move = dc[np.arange(N), c] < best
            codes[b, h] = np.where(move, M0 + a * C + c, a)
    return codes


def aggregate_brute(codes, V, M0, C):
    """V-bar [B,H,Mt,d] and n [B,H,Mt]: every key counts for its parent, and
    for its child when it moved to one."""
    V = _f64(V)
    codes = np.asarray(codes)
    B, H, N, d = V.shape
    Mt = M0 * (1 + C)
    vs = np.zeros((B, H, Mt, d))
    ns = np.zeros((B, H, Mt), dtype=np.int64)
    parent = np.where(codes < M0, codes, (codes - M0) // max(C, 1))
    for b in range(B):
        for h in range(H):
            np.add.at(vs[b, h], parent[b, h], V[b, h])
            np.add.at(ns[b, h], parent[b, h], 1)
            mv = codes[b, h] >= M0
            np.add.at(vs[b, h], codes[b, h][mv], V[b, h][mv])
            np.add.at(ns[b, h], codes[b, h][mv], 1)
    return vs, ns


def _softmax_rows(logits):
    mx = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - mx)
    return e / e.sum(axis=-1, keepdims=True)


def representative_attention(Q, K_codes, V, parents, children, sel, block, scale):
    """Exact softmax attention over representative keys (Sec. C identity)."""
    Q, V, parents, children = _f64(Q), _f64(V), _f64(parents), _f64(children)
    codes = np.asarray(K_codes)
    B, H, N, d = Q.shape
    M0 = parents.shape[1]
    C = children.shape[2]
    sel = np.asarray(sel)
    Y = np.empty_like(Q)
    nblk = (N + block - 1) // block
    for b in range(B):
        for h in range(H):
            c = codes[b, h]
            par = np.where(c < M0, c, (c - M0) // max(C, 1))
            parent_vec = parents[h][par]  # [N, d]
            if C > 0:
                flat_children = children[h].reshape(M0 * C, d)
                child_vec = flat_children[np.clip(c - M0, 0, M0 * C - 1)]
            for blk in range(nblk):
                i0, i1 = blk * block, min(N, (blk + 1) * block)
                rep = parent_vec.copy()
                if C > 0 and sel.shape[-1] > 0:
                    chosen = np.zeros(M0, dtype=bool)
                    chosen[sel[b, h, blk]] = True
                    use_child = (c >= M0) & chosen[par]
                    rep[use_child] = child_vec[use_child]
                logits = scale * Q[b, h, i0:i1] @ rep.T  # [nI, N]
                Y[b, h, i0:i1] = _softmax_rows(logits) @ V[b, h]
    return Y


def flat_vq_attention(Q, codebook, vsum, counts, scale):
    """Eq. 4: sum_a exp(q c_a) V-bar_a / sum_a exp(q c_a) n_a over one codebook
    per head (codebook [H,M,d], vsum [B,H,M,d], counts [B,H,M])."""
    Q, codebook, vsum, counts = _f64(Q), _f64(codebook), _f64(vsum), _f64(counts)
    B, H, N, d = Q.shape
    Y = np.empty_like(Q)
    for b in range(B):
        for h in range(H):
            s = scale * Q[b, h] @ codebook[h].T  # [N, M]
            live = counts[b, h] > 0
            s = np.where(live[None, :], s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            e = np.where(live[None, :], np.exp(s - mx), 0.0)
            Y[b, h] = (e @ vsum[b, h]) / (e @ counts[b, h])[:, None]
    return Y


def exact_attention(Q, K, V, scale):
    """Eq. 1 with scaled logits."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, N, d = Q.shape
    Y = np.empty_like(Q)
    for b in range(B):
        for h in range(H):
            Y[b, h] = _softmax_rows(scale * Q[b, h] @ K[b, h].T) @ V[b, h]
    return Y


def importance_brute(Q, parents, counts, block, scale):
    """w_j(I) = sum_{i in I} n_j exp(s_ij) / sum_l n_l exp(s_il)  [B,H,nblk,M0]."""
    Q, parents, counts = _f64(Q), _f64(parents), _f64(counts)
    B, H, N, d = Q.shape
    M0 = parents.shape[1]
    nblk = (N + block - 1) // block
    W = np.zeros((B, H, nblk, M0))
    for b in range(B):
        for h in range(H):
            n = counts[b, h][:M0]
            with np.errstate(divide="ignore"):
                logn = np.where(n > 0, np.log(np.where(n > 0, n, 1.0)), -np.inf)
            mass = _softmax_rows(scale * Q[b, h] @ parents[h].T + logn[None, :])  # [N, M0]
            for blk in range(nblk):
                W[b, h, blk] = mass[blk * block:(blk + 1) * block].sum(axis=0)
    return W


def parent_attention_mass(Q, K, codes, M0, C, block, scale):
    """True attention mass per parent and query block [B,H,nblk,M0]: the sum
    over the block's queries i of the exact softmax weights (Eq. 1, scaled
    logits, all N keys) of the keys whose parent is j.  Dividing the mass of
    a set of parents by the block's row count gives the "capture" of the
    pages' Table 5 (Sec. B) and Table 6: the fraction of true attention
    weight that falls on keys assigned to the selected parents."""
    Q, K = _f64(Q), _f64(K)
    codes = np.asarray(codes)
    B, H, N, d = Q.shape
    nblk = (N + block - 1) // block
    W = np.zeros((B, H, nblk, M0))
    for b in range(B):
        for h in range(H):
            c = codes[b, h]
            par = np.where(c < M0, c, (c - M0) // max(C, 1))
            onehot = np.zeros((N, M0))
            onehot[np.arange(N), par] = 1.0
            for blk in range(nblk):
                q = Q[b, h, blk * block:(blk + 1) * block]
                p = _softmax_rows(scale * q @ K[b, h].T)  # [nI, N]
                W[b, h, blk] = p.sum(axis=0) @ onehot
    return W


def top_p_capture(mass, sel, N, block):
    """Mean over blocks of (sum of the selected parents' true mass) / |I|."""
    mass = np.asarray(mass)
    sel = np.asarray(sel)
    nblk = mass.shape[-2]
    sizes = np.array([min(block, N - k * block) for k in range(nblk)], dtype=np.float64)
    got = np.take_along_axis(mass, sel.astype(np.int64), axis=-1).sum(-1)  # [B,H,nblk]
    return float(np.mean(got / sizes))


# ---- depth-3 tree --------------------------------------------------------
def assign_brute3(K, parents, children, grandchildren):
    """Final codes [B,H,N] of the depth-3 descent by full distance tables:
    nearest parent; nearest child of it, taken when strictly closer; then
    nearest grandchild of that child, taken when strictly closer than it."""
    K, parents, children, grandchildren = map(_f64, (K, parents, children, grandchildren))
    codes2 = assign_brute(K, parents, children)
    B, H, N, d = K.shape
    M0, C = parents.shape[1], children.shape[2]
    M1 = M0 * C
    codes = codes2.copy()
    for b in range(B):
        for h in range(H):
            k = K[b, h]
            c2 = codes2[b, h]
            moved = np.nonzero(c2 >= M0)[0]
            if moved.size == 0:
                continue
            cidx = c2[moved] - M0
            ch = children[h].reshape(M1, d)[cidx]                      # [n, d]
            gc = grandchildren[h].reshape(M1, C, d)[cidx]              # [n, C, d]
            dch = ((k[moved] - ch) ** 2).sum(-1)
            dg = ((k[moved][:, None, :] - gc) ** 2).sum(-1)            # [n, C]
            g = dg.argmin(axis=1)
            go = dg[np.arange(moved.size), g] < dch
            codes[b, h, moved[go]] = M0 + M1 + cidx[go] * C + g[go]
    return codes


def _lineage3(codes, M0, C):
    """(parent, child or -1, grandchild or -1) code arrays of depth-3 codes."""
    codes = np.asarray(codes)
    M1 = M0 * C
    is_g = codes >= M0 + M1
    is_c = (codes >= M0) & ~is_g
    child = np.where(is_c, codes, np.where(is_g, M0 + (codes - M0 - M1) // C, -1))
    parent = np.where(codes < M0, codes, (child - M0) // C)
    grand = np.where(is_g, codes, -1)
    return parent, child, grand


def aggregate_brute3(codes, V, M0, C):
    """Eq. 3 statistics of the depth-3 tree: a key counts at its parent, its
    child (if it moved) and its grandchild (if it moved twice)."""
    V = _f64(V)
    B, H, N, d = V.shape
    Mt = M0 + M0 * C + M0 * C * C
    vs = np.zeros((B, H, Mt, d))
    ns = np.zeros((B, H, Mt), dtype=np.int64)
    parent, child, grand = _lineage3(codes, M0, C)
    for b in range(B):
        for h in range(H):
            for lvl in (parent[b, h], child[b, h], grand[b, h]):
                ok = lvl >= 0
                np.add.at(vs[b, h], lvl[ok], V[b, h][ok])
                np.add.at(ns[b, h], lvl[ok], 1)
    return vs, ns


def representative_attention3(Q, codes, V, parents, children, grandchildren, sel, sel2, block,
                              scale, depth2_only=False):
    """Exact softmax attention over representative keys of the depth-3 tree:
    a key is represented by its grandchild if its child is among the block's
    selected children, else by its child if its parent is among the block's
    selected parents, else by its parent.  With `depth2_only` the grandchild
    level is ignored (the representatives after the child refinement)."""
    Q, V, parents, children, grandchildren = map(_f64, (Q, V, parents, children, grandchildren))
    B, H, N, d = Q.shape
    M0, C = parents.shape[1], children.shape[2]
    M1 = M0 * C
    parent, child, grand = _lineage3(codes, M0, C)
    sel, sel2 = np.asarray(sel), np.asarray(sel2)
    nblk = (N + block - 1) // block
    Y = np.empty_like(Q)
    for b in range(B):
        for h in range(H):
            pv = parents[h][parent[b, h]]
            cv = children[h].reshape(M1, d)[np.clip(child[b, h] - M0, 0, M1 - 1)]
            gv = grandchildren[h].reshape(M1 * C, d)[np.clip(grand[b, h] - M0 - M1, 0, M1 * C - 1)]
            for blk in range(nblk):
                i0, i1 = blk * block, min(N, (blk + 1) * block)
                rep = pv.copy()
                if sel.shape[-1] > 0:
                    use_c = (child[b, h] >= 0) & np.isin(parent[b, h], sel[b, h, blk])
                    rep[use_c] = cv[use_c]
                    if not depth2_only and sel2.shape[-1] > 0:
                        use_g = (grand[b, h] >= 0) & use_c & np.isin(child[b, h], sel2[b, h, blk])
                        rep[use_g] = gv[use_g]
                Y[b, h, i0:i1] = _softmax_rows(scale * Q[b, h, i0:i1] @ rep.T) @ V[b, h]
    return Y


def child_mass3(Q, codes, parents, children, grandchildren, sel, block, scale):
    """Importance of the refined children written as a block sum of softmax
    mass: for each block and each child of its selected parents (in the order
    of sel, C each), the mass that exact softmax attention over the depth-2
    representatives (after the child refinement) puts on the keys counted at
    that child.  [B,H,nblk,P*C]"""
    Q = _f64(Q)
    B, H, N, d = Q.shape
    M0, C = parents.shape[1], children.shape[2]
    parent, child, _ = _lineage3(codes, M0, C)
    parents_f, children_f = _f64(parents), _f64(children)
    sel = np.asarray(sel)
    P = sel.shape[-1]
    nblk = (N + block - 1) // block
    W = np.zeros((B, H, nblk, P * C))
    for b in range(B):
        for h in range(H):
            for blk in range(nblk):
                i0, i1 = blk * block, min(N, (blk + 1) * block)
                use_c = (child[b, h] >= 0) & np.isin(parent[b, h], sel[b, h, blk])
                rep = parents_f[h][parent[b, h]].copy()
                rep[use_c] = children_f[h].reshape(M0 * C, d)[child[b, h][use_c] - M0]
                mass = _softmax_rows(scale * Q[b, h, i0:i1] @ rep.T).sum(axis=0)  # [N]
                for k, p in enumerate(sel[b, h, blk]):
                    for c in range(C):
                        W[b, h, blk, k * C + c] = mass[child[b, h] == M0 + p * C + c].sum()
    return W
