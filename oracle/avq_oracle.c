/*
 * AVQ-Attention oracle: a plain, slow float64 CPU implementation of the
 * forward pass of "AVQ-Attention: Adaptive Vector-Quantized Attention".
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code with the CUDA path.
 *
 * Stage 1 follows Algorithm 1 (VQ Precompute kernel, Sec. 4.2) and Stage 2
 * follows Algorithm 2 (Flash AVQ-Attention kernel, Sec. 4.3), step by step,
 * in the order and notation of the paper, with no blocking or reordering
 * beyond the per-query-block structure the algorithm itself defines.
 *
 * Readings taken where the paper leaves a step open:
 *   - Logits are scaled by `scale` (1/sqrt(d) in every workload); the paper's
 *     Eq. 1 omits the factor "for clarity" (Sec. 3.1).  Distances use raw keys.
 *   - Parent ties go to the lowest index (argmin in Algorithm 1).  A child is
 *     taken only if strictly closer than the running best child and the key
 *     moves only if that child is strictly closer than the parent (the two
 *     strict comparisons of Algorithm 1).
 *   - Top-P ties go to the lower parent index; the selection is listed in
 *     descending importance (the top-P of Algorithm 2).
 *   - Importance uses the parents-only denominator (Algorithm 2 computes it
 *     before the selection and the refinement; Eq. 7).
 *   - A partial last query block (N not a multiple of the block) is a block
 *     with fewer rows that selects independently.
 *
 * Layouts (all row-major, contiguous):
 *   K, V, Q, O   [BH][N][d]            BH = B*H, head h = bh % H
 *   parents      [H][M0][d]
 *   children     [H][M0][C][d]         child (m,c) is codeword M0 + m*C + c
 *   assign       [BH][N]               final code in [0, M0*(1+C))
 *   vsum         [BH][Mt][d]           Mt = M0*(1+C)  (value sums, Eq. 3)
 *   counts       [BH][Mt]              key counts n_a (Eq. 3)
 *   sel          [BH][nblk][P]         nblk = ceil(N/block)
 *   importance   [BH][nblk][M0]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double sqdist(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int t = 0; t < d; ++t) {
    double diff = a[t] - b[t];
    s += diff * diff;
  }
  return s;
}

static double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int t = 0; t < d; ++t) s += a[t] * b[t];
  return s;
}

/*
 * Algorithm 1 for one key: nearest parent, then the nearest of that parent's
 * C children, reassigned only if the child is strictly closer than the cached
 * parent distance.
 * Returns the final code.  The decision distances are written for the
 * near-tie rule used by the tests:
 *   dec[0] = best parent distance, dec[1] = second-best parent distance,
 *   dec[2] = best child distance (INFINITY if C == 0),
 *   dec[3] = second-best child distance (INFINITY if C < 2).
 */
static int32_t assign_one(const double* k, const double* par_h, const double* ch_h,
                          int d, int M0, int C, double* dec) {
  /* d = ||k - c_p||^2 over the M0 parents, a = argmin, d_best = min */
  int a = 0;
  double d_best = INFINITY, d_second = INFINITY;
  for (int m = 0; m < M0; ++m) {
    double dm = sqdist(k, par_h + (size_t)m * d, d);
    if (dm < d_best) {
      d_second = d_best;
      d_best = dm;
      a = m;
    } else if (dm < d_second) {
      d_second = dm;
    }
  }
  /* c0 = M0 + a*C, d_child = inf, c* = c0, scan the C children of a */
  int32_t c0 = M0 + a * C;
  double d_child = INFINITY, d_child2 = INFINITY;
  int32_t c_star = c0;
  for (int c = 0; c < C; ++c) {
    const double* cc = ch_h + ((size_t)a * C + c) * d;
    double dc = sqdist(k, cc, d);
    if (dc < d_child) { /* where d_c < d_child: strict */
      d_child2 = d_child;
      d_child = dc;
      c_star = c0 + c;
    } else if (dc < d_child2) {
      d_child2 = dc;
    }
  }
  if (dec) {
    dec[0] = d_best;
    dec[1] = d_second;
    dec[2] = d_child;
    dec[3] = d_child2;
  }
  /* where d_child < d_best (strict) the key moves to child c* */
  if (C > 0 && d_child < d_best) return c_star;
  return a;
}

/*
 * Algorithm 1 (VQ Precompute).  The statistics start at zero; every key then
 * adds its value and a count of one to its parent and, if it moved, also to
 * its child (the masked add).  Parents thus hold their whole cluster and
 * children only the keys that are closer to them than to the parent.
 * `dec` (nullable) receives 4 decision distances per key, see assign_one.
 */
void avq_oracle_quantize(int BH, int H, int N, int d, int M0, int C,
                         const double* K, const double* V,
                         const double* parents, const double* children,
                         int32_t* assign, double* vsum, int64_t* counts,
                         double* dec) {
  const int Mt = M0 * (1 + C);
#pragma omp parallel for schedule(dynamic)
  for (int bh = 0; bh < BH; ++bh) {
    const int h = bh % H;
    const double* par_h = parents + (size_t)h * M0 * d;
    const double* ch_h = children + (size_t)h * M0 * C * d;
    double* vs = vsum + (size_t)bh * Mt * d;
    int64_t* ns = counts + (size_t)bh * Mt;
    /* initialise V-bar = 0, n = 0 */
    memset(vs, 0, sizeof(double) * (size_t)Mt * d);
    memset(ns, 0, sizeof(int64_t) * (size_t)Mt);
    for (int j = 0; j < N; ++j) {
      const double* k = K + ((size_t)bh * N + j) * d;
      const double* v = V + ((size_t)bh * N + j) * d;
      double* dj = dec ? dec + ((size_t)bh * N + j) * 4 : NULL;
      int32_t code = assign_one(k, par_h, ch_h, d, M0, C, dj);
      int32_t a = code < M0 ? code : (code - M0) / C;
      /* V-bar[a] += v; n[a] += 1 */
      for (int t = 0; t < d; ++t) vs[(size_t)a * d + t] += v[t];
      ns[a] += 1;
      /* masked add to the child */
      if (code >= M0) {
        for (int t = 0; t < d; ++t) vs[(size_t)code * d + t] += v[t];
        ns[code] += 1;
      }
      assign[(size_t)bh * N + j] = code;
    }
  }
}

/*
 * The aggregation of Algorithm 1 for given final codes:
 * used to check statistics against assignments made elsewhere.
 */
void avq_oracle_aggregate(int BH, int N, int d, int M0, int C,
                          const int32_t* assign, const double* V,
                          double* vsum, int64_t* counts) {
  const int Mt = M0 * (1 + C);
  for (int bh = 0; bh < BH; ++bh) {
    double* vs = vsum + (size_t)bh * Mt * d;
    int64_t* ns = counts + (size_t)bh * Mt;
    memset(vs, 0, sizeof(double) * (size_t)Mt * d);
    memset(ns, 0, sizeof(int64_t) * (size_t)Mt);
    for (int j = 0; j < N; ++j) {
      int32_t code = assign[(size_t)bh * N + j];
      int32_t a = code < M0 ? code : (code - M0) / C;
      const double* v = V + ((size_t)bh * N + j) * d;
      for (int t = 0; t < d; ++t) vs[(size_t)a * d + t] += v[t];
      ns[a] += 1;
      if (code >= M0) {
        for (int t = 0; t < d; ++t) vs[(size_t)code * d + t] += v[t];
        ns[code] += 1;
      }
    }
  }
}

/*
 * Top-P of the importance vector w[0..M0): the P largest entries in
 * descending order, ties to the lower index (the top-P of Algorithm 2).
 */
static void top_p(const double* w, int M0, int P, int32_t* out) {
  char* taken = (char*)calloc((size_t)M0, 1);
  for (int r = 0; r < P; ++r) {
    int best = -1;
    for (int j = 0; j < M0; ++j) {
      if (taken[j]) continue;
      if (best < 0 || w[j] > w[best]) best = j; /* strict: equal keeps lower index */
    }
    taken[best] = 1;
    out[r] = best;
  }
  free(taken);
}

/*
 * Algorithm 2 (Flash AVQ-Attention) for one query block I = [i0, i1) of one
 * head.  Coarse pass over the M0 parents with the masked running
 * max (Eq. 18), count-weighted denominator (Eq. 6) and importance (Eq. 7).
 * Top-P.  Then, for each selected parent: child logits, online
 * max merge, parent logit recovered as the mean of the child logits (Eq. 8),
 * correcting attention dA = exp(S_ic) - exp(S_ip) (Eq. 9) masked for empty
 * children, and the accumulator update.  Finally Y = x / z.
 */
static void attend_block(int d, int M0, int C, int P, double scale,
                         const double* Q, int i0, int i1,
                         const double* par_h, const double* ch_h,
                         const double* vs, const double* ns,
                         const int32_t* sel_in, double* O, int32_t* sel_out,
                         double* imp_out, int tile) {
  const int nI = i1 - i0;
  double* s = (double*)malloc(sizeof(double) * (size_t)nI * M0);
  double* A = (double*)malloc(sizeof(double) * (size_t)nI * M0);
  double* m = (double*)malloc(sizeof(double) * (size_t)nI);
  double* x = (double*)malloc(sizeof(double) * (size_t)nI * d);
  double* z = (double*)malloc(sizeof(double) * (size_t)nI);
  double* w = (double*)malloc(sizeof(double) * (size_t)M0);
  int32_t* S = (int32_t*)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
  double* sc = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));

  for (int r = 0; r < nI; ++r) {
    const double* q = Q + (size_t)(i0 + r) * d;
    /* s = q c^T over the parents */
    for (int j = 0; j < M0; ++j) s[(size_t)r * M0 + j] = scale * dot(q, par_h + (size_t)j * d, d);
    /* m = max over j with n_j > 0 (Eq. 18) */
    m[r] = -INFINITY;
    for (int j = 0; j < M0; ++j)
      if (ns[j] > 0 && s[(size_t)r * M0 + j] > m[r]) m[r] = s[(size_t)r * M0 + j];
    /* A = exp(s - m), A_j = 0 where n_j = 0 */
    for (int j = 0; j < M0; ++j)
      A[(size_t)r * M0 + j] = ns[j] > 0 ? exp(s[(size_t)r * M0 + j] - m[r]) : 0.0;
    /* x = A v-bar, z = sum_j A_j n_j  (Eq. 6) */
    for (int t = 0; t < d; ++t) x[(size_t)r * d + t] = 0.0;
    z[r] = 0.0;
    for (int j = 0; j < M0; ++j) {
      double a = A[(size_t)r * M0 + j];
      for (int t = 0; t < d; ++t) x[(size_t)r * d + t] += a * vs[(size_t)j * d + t];
      z[r] += a * ns[j];
    }
  }
  if (tile <= 0 || tile >= M0) {
    /* w_j = sum_i A_ij n_j / z_i  (Eq. 7) */
    for (int j = 0; j < M0; ++j) {
      w[j] = 0.0;
      for (int r = 0; r < nI; ++r) w[j] += A[(size_t)r * M0 + j] * ns[j] / z[r];
    }
  } else {
    /* Sec. B: the parents are visited in tiles of `tile` codes in index order;
     * the importance of the codes in tile J uses the count-extrapolated
     * denominator Z~_i(J) = (N / N_seen(J)) sum_{t <= J} Z_i(t)  (Eq. 13),
     * w_j = sum_i A_ij n_j / Z~_i(J)  (Eq. 14).  N is the number of keys, the
     * sum of the parents' counts; N_seen(J) the keys of parents in tiles <= J.
     * A common reference max cancels in A / Z~. */
    double ntot = 0.0;
    for (int j = 0; j < M0; ++j) ntot += ns[j];
    double* zpart = (double*)calloc((size_t)nI, sizeof(double));
    double nseen = 0.0;
    for (int j0 = 0; j0 < M0; j0 += tile) {
      const int j1 = j0 + tile < M0 ? j0 + tile : M0;
      for (int j = j0; j < j1; ++j) {
        nseen += ns[j];
        for (int r = 0; r < nI; ++r) zpart[r] += A[(size_t)r * M0 + j] * ns[j];
      }
      for (int j = j0; j < j1; ++j) {
        w[j] = 0.0;
        if (nseen <= 0.0) continue; /* every parent seen so far is empty: n_j = 0 */
        for (int r = 0; r < nI; ++r)
          if (zpart[r] > 0.0) w[j] += A[(size_t)r * M0 + j] * ns[j] / (ntot / nseen * zpart[r]);
      }
    }
    free(zpart);
  }
  if (imp_out) memcpy(imp_out, w, sizeof(double) * (size_t)M0);
  /* S = top-P(w), or the caller's selection */
  if (P > 0) {
    if (sel_in) memcpy(S, sel_in, sizeof(int32_t) * (size_t)P);
    else top_p(w, M0, P, S);
    if (sel_out) memcpy(sel_out, S, sizeof(int32_t) * (size_t)P);
  }
  /* child refinement (no-op when C == 0) */
  if (C > 0) {
    for (int r = 0; r < nI; ++r) {
      const double* q = Q + (size_t)(i0 + r) * d;
      for (int k = 0; k < P; ++k) {
        int p = S[k];
        const double* ch_p = ch_h + (size_t)p * C * d;
        const double* vc = vs + (size_t)(M0 + p * C) * d;
        const double* nc = ns + (M0 + p * C);
        /* s_c = q c_c^T */
        for (int c = 0; c < C; ++c) sc[c] = scale * dot(q, ch_p + (size_t)c * d, d);
        /* m' = max(m, max over c with n_c > 0 of s_c) */
        double mp = m[r];
        for (int c = 0; c < C; ++c)
          if (nc[c] > 0 && sc[c] > mp) mp = sc[c];
        /* rescale the accumulators to m' */
        double f = exp(m[r] - mp);
        for (int t = 0; t < d; ++t) x[(size_t)r * d + t] *= f;
        z[r] *= f;
        m[r] = mp;
        /* s_p = (1/C) sum_c s_c   (Eq. 8) */
        double sp = 0.0;
        for (int c = 0; c < C; ++c) sp += sc[c];
        sp /= C;
        /* dA = exp(s_c - m) - exp(s_p - m), zero where n_c = 0  (Eq. 9) */
        double Ap = exp(sp - m[r]);
        for (int c = 0; c < C; ++c) {
          double dA = nc[c] > 0 ? exp(sc[c] - m[r]) - Ap : 0.0;
          for (int t = 0; t < d; ++t) x[(size_t)r * d + t] += dA * vc[(size_t)c * d + t];
          z[r] += dA * nc[c];
        }
      }
    }
  }
  /* Y = x / z */
  for (int r = 0; r < nI; ++r)
    for (int t = 0; t < d; ++t) O[(size_t)(i0 + r) * d + t] = x[(size_t)r * d + t] / z[r];

  free(s); free(A); free(m); free(x); free(z); free(w); free(S); free(sc);
}

/*
 * Algorithm 2 over every (bh, query block), or over the listed ones only
 * (`blocks` holds nlist pairs (bh, block index); nullable = all).  `counts`
 * are passed as doubles.  `sel_in` (nullable) overrides the top-P selection:
 * [BH][nblk][P].  O rows of unlisted blocks are left untouched.
 */
/*
 * Stage 2 over all (or the listed) query blocks.  tile > 0 (and < M0) selects
 * the tiled importance with the count-extrapolated denominator of Sec. B
 * (Eqs. 13-14); everything else is unchanged by it.
 */
void avq_oracle_attention_tiled(int BH, int H, int N, int d, int M0, int C, int P, int block,
                                double scale, const double* Q,
                                const double* parents, const double* children,
                                const double* vsum, const double* counts,
                                const int32_t* sel_in, const int32_t* blocks, int nlist,
                                double* O, int32_t* sel_out, double* imp_out, int tile) {
  const int Mt = M0 * (1 + C);
  const int nblk = (N + block - 1) / block;
  const int total = blocks ? nlist : BH * nblk;
#pragma omp parallel for schedule(dynamic)
  for (int u = 0; u < total; ++u) {
    int bh = blocks ? blocks[2 * u] : u / nblk;
    int b = blocks ? blocks[2 * u + 1] : u % nblk;
    int h = bh % H;
    int i0 = b * block;
    int i1 = i0 + block < N ? i0 + block : N;
    size_t sb = (size_t)bh * nblk + b;
    attend_block(d, M0, C, P, scale, Q + (size_t)bh * N * d, i0, i1,
                 parents + (size_t)h * M0 * d, children + (size_t)h * M0 * C * d,
                 vsum + (size_t)bh * Mt * d, counts + (size_t)bh * Mt,
                 sel_in ? sel_in + sb * P : NULL, O + (size_t)bh * N * d,
                 sel_out ? sel_out + sb * P : NULL, imp_out ? imp_out + sb * M0 : NULL, tile);
  }
}

/* Stage 2 with the exact importance denominator (Eq. 7). */
void avq_oracle_attention(int BH, int H, int N, int d, int M0, int C, int P, int block,
                          double scale, const double* Q,
                          const double* parents, const double* children,
                          const double* vsum, const double* counts,
                          const int32_t* sel_in, const int32_t* blocks, int nlist,
                          double* O, int32_t* sel_out, double* imp_out) {
  avq_oracle_attention_tiled(BH, H, N, d, M0, C, P, block, scale, Q, parents, children, vsum, counts,
                             sel_in, blocks, nlist, O, sel_out, imp_out, 0);
}

int avq_oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the parallel loops above (host plumbing, no arithmetic). */
void avq_oracle_set_threads(int n) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/*
 * Codebook update of Sec. A ("Codeword Clustering During Training").
 * EMA statistics (Eq. 11), one set per head over the keys of every batch
 * entry:  S_x <- lambda S_x + (1 - lambda) sum_k k,  N_x <- lambda N_x +
 * (1 - lambda) |{k}|, over the keys quantised to code x, with the statistics
 * of Eq. 3 (a parent counts its whole cluster, a child the keys that moved to
 * it); ksum and counts are those statistics computed on the keys.
 * Parents take their unconstrained means C_p = S_p / N_p.  Children take the
 * mass-weighted projection of their means M_c = S_c / N_c onto the constraint
 * sum_c C_pc = C C_p (Eq. 12):  delta = sum_c M_c - C C_p,
 * sigma = sum_c 1 / N_c,  C_pc = M_c - delta / (N_c sigma).
 * Readings where the pages are silent:
 *   - a code with N_x = 0 after the update has no mean: it keeps its current
 *     position (parents_in / children_in) in place of M_x;
 *   - such massless children do not move; delta is spread over the children
 *     with N_c > 0 only (sigma over those); if no child has mass, all C
 *     children shift by -delta / C.
 * Layouts: ksum [B][H][Mt][d], counts [B][H][Mt]; S [H][Mt][d], Nst [H][Mt]
 * (updated in place); parents [H][M0][d], children [H][M0][C][d].
 */
void avq_oracle_codebook_update(int B, int H, int d, int M0, int C, double lambda,
                                const double* ksum, const double* counts, double* S, double* Nst,
                                const double* parents_in, const double* children_in,
                                double* parents_out, double* children_out) {
  const int Mt = M0 * (1 + C);
  /* Eq. 11 */
  for (int h = 0; h < H; ++h)
    for (int x = 0; x < Mt; ++x) {
      double n = 0.0;
      for (int b = 0; b < B; ++b) n += counts[((size_t)b * H + h) * Mt + x];
      Nst[(size_t)h * Mt + x] = lambda * Nst[(size_t)h * Mt + x] + (1.0 - lambda) * n;
      for (int t = 0; t < d; ++t) {
        double sk = 0.0;
        for (int b = 0; b < B; ++b) sk += ksum[(((size_t)b * H + h) * Mt + x) * d + t];
        double* sx = S + ((size_t)h * Mt + x) * d + t;
        *sx = lambda * *sx + (1.0 - lambda) * sk;
      }
    }
  double* Mc = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1) * d);
  for (int h = 0; h < H; ++h)
    for (int p = 0; p < M0; ++p) {
      /* parent: unconstrained mean */
      const double np = Nst[(size_t)h * Mt + p];
      double* cp = parents_out + ((size_t)h * M0 + p) * d;
      for (int t = 0; t < d; ++t)
        cp[t] = np > 0.0 ? S[((size_t)h * Mt + p) * d + t] / np : parents_in[((size_t)h * M0 + p) * d + t];
      if (C == 0) continue;
      /* children: means, then the projection (Eq. 12) */
      double sigma = 0.0;
      int massive = 0;
      for (int c = 0; c < C; ++c) {
        const int x = M0 + p * C + c;
        const double nc = Nst[(size_t)h * Mt + x];
        for (int t = 0; t < d; ++t)
          Mc[(size_t)c * d + t] = nc > 0.0 ? S[((size_t)h * Mt + x) * d + t] / nc
                                           : children_in[(((size_t)h * M0 + p) * C + c) * d + t];
        if (nc > 0.0) {
          sigma += 1.0 / nc;
          ++massive;
        }
      }
      for (int t = 0; t < d; ++t) {
        double delta = -C * cp[t];
        for (int c = 0; c < C; ++c) delta += Mc[(size_t)c * d + t];
        for (int c = 0; c < C; ++c) {
          const double nc = Nst[(size_t)h * Mt + M0 + p * C + c];
          double shift;
          if (massive > 0) shift = nc > 0.0 ? delta / (nc * sigma) : 0.0;
          else shift = delta / C;
          children_out[(((size_t)h * M0 + p) * C + c) * d + t] = Mc[(size_t)c * d + t] - shift;
        }
      }
    }
  free(Mc);
}

/* ------------------------------------------------------------------------
 * Depth-3 tree: the "deeper hierarchies" named as the next step in the
 * conclusion (Sec. 6).  Every child has C grandchildren and equals their
 * mean, as every parent equals the mean of its children (Eq. 5).  Code
 * layout per head: parents [0, M0), child (m, c) at M0 + m*C + c, grandchild
 * (m, c, g) at M0 + M0*C + (m*C + c)*C + g.
 *
 * Readings (the pages name the extension but give no algorithm; these are
 * Algorithms 1 and 2 applied once more, one level down):
 *   - Algorithm 1 descends one more level: a key that moved to child c*
 *     moves on to c*'s nearest grandchild (first strict minimum) only if that
 *     grandchild is strictly closer than c*.  Statistics (Eq. 3): a key counts
 *     at its parent, at its child if it moved, and at its grandchild if it
 *     moved twice.
 *   - Algorithm 2: after the child refinement of the top-P parents, each of
 *     the P*C refined children gets an importance like Eq. 7, using the
 *     logits and denominator of the attention after that refinement:
 *     w_c(I) = sum_{i in I} exp(s_ic - m_i) n_c / z_i; the top-P2 of them
 *     (descending, ties to the lower child code) are refined with their
 *     grandchildren exactly as parents are with their children: the child's
 *     logit is recovered as the mean of its grandchildren's (Eq. 8) and
 *     dA = exp(s_ig) - exp(s_ic) (Eq. 9), zero for empty grandchildren.
 * ---------------------------------------------------------------------- */

/* Algorithm 1, depth 3, for one key: `dec` (nullable) receives 6 decision
 * distances: the 4 of assign_one, then the best and second-best grandchild
 * distance (INFINITY when the key did not move to a child). */
static int32_t assign_one3(const double* k, const double* par_h, const double* ch_h,
                           const double* gc_h, int d, int M0, int C, double* dec) {
  int32_t code = assign_one(k, par_h, ch_h, d, M0, C, dec);
  if (dec) { dec[4] = INFINITY; dec[5] = INFINITY; }
  if (code < M0) return code;
  /* the key sits at child c = code - M0 (c = m*C + c'): scan its grandchildren */
  const int32_t c = code - M0;
  const double d_child = sqdist(k, ch_h + (size_t)c * d, d);
  double d_g = INFINITY, d_g2 = INFINITY;
  int32_t g_star = 0;
  for (int g = 0; g < C; ++g) {
    double dg = sqdist(k, gc_h + ((size_t)c * C + g) * d, d);
    if (dg < d_g) { /* first strict minimum */
      d_g2 = d_g;
      d_g = dg;
      g_star = g;
    } else if (dg < d_g2) {
      d_g2 = dg;
    }
  }
  if (dec) { dec[4] = d_g; dec[5] = d_g2; }
  /* moves to the grandchild only when strictly closer than the child */
  if (d_g < d_child) return M0 + M0 * C + c * C + g_star;
  return code;
}

void avq_oracle_quantize3(int BH, int H, int N, int d, int M0, int C,
                          const double* K, const double* V, const double* parents,
                          const double* children, const double* grandchildren,
                          int32_t* assign, double* vsum, int64_t* counts, double* dec) {
  const int M1 = M0 * C, Mt = M0 + M1 + M1 * C;
#pragma omp parallel for schedule(dynamic)
  for (int bh = 0; bh < BH; ++bh) {
    const int h = bh % H;
    const double* par_h = parents + (size_t)h * M0 * d;
    const double* ch_h = children + (size_t)h * M1 * d;
    const double* gc_h = grandchildren + (size_t)h * M1 * C * d;
    double* vs = vsum + (size_t)bh * Mt * d;
    int64_t* ns = counts + (size_t)bh * Mt;
    memset(vs, 0, sizeof(double) * (size_t)Mt * d);
    memset(ns, 0, sizeof(int64_t) * (size_t)Mt);
    for (int j = 0; j < N; ++j) {
      const double* k = K + ((size_t)bh * N + j) * d;
      const double* v = V + ((size_t)bh * N + j) * d;
      double* dj = dec ? dec + ((size_t)bh * N + j) * 6 : NULL;
      const int32_t code = assign_one3(k, par_h, ch_h, gc_h, d, M0, C, dj);
      /* the key's parent, and its child when it moved at least once */
      int32_t child = -1, a;
      if (code < M0) a = code;
      else if (code < M0 + M1) { child = code; a = (code - M0) / C; }
      else { child = M0 + (code - M0 - M1) / C; a = (child - M0) / C; }
      for (int t = 0; t < d; ++t) vs[(size_t)a * d + t] += v[t];
      ns[a] += 1;
      if (child >= 0) {
        for (int t = 0; t < d; ++t) vs[(size_t)child * d + t] += v[t];
        ns[child] += 1;
      }
      if (code >= M0 + M1) {
        for (int t = 0; t < d; ++t) vs[(size_t)code * d + t] += v[t];
        ns[code] += 1;
      }
      assign[(size_t)bh * N + j] = code;
    }
  }
}

/* top-P2 of the candidate children: descending importance, ties to the lower
 * child code */
static void top_p_codes(const double* w, const int32_t* code, int n, int P2, int32_t* out) {
  char* taken = (char*)calloc((size_t)(n > 0 ? n : 1), 1);
  for (int r = 0; r < P2; ++r) {
    int best = -1;
    for (int j = 0; j < n; ++j) {
      if (taken[j]) continue;
      if (best < 0 || w[j] > w[best] || (w[j] == w[best] && code[j] < code[best])) best = j;
    }
    taken[best] = 1;
    out[r] = best;
  }
  free(taken);
}

/* Algorithm 2, depth 3, for one query block of one head. */
static void attend_block3(int d, int M0, int C, int P, int P2, double scale,
                          const double* Q, int i0, int i1, const double* par_h,
                          const double* ch_h, const double* gc_h, const double* vs,
                          const double* ns, const int32_t* sel_in, const int32_t* sel2_in,
                          double* O, int32_t* sel_out, int32_t* sel2_out, double* imp_out,
                          double* imp2_out) {
  const int M1 = M0 * C;
  const int nI = i1 - i0, nc = P * C;
  double* s = (double*)malloc(sizeof(double) * (size_t)nI * M0);
  double* A = (double*)malloc(sizeof(double) * (size_t)nI * M0);
  double* m = (double*)malloc(sizeof(double) * (size_t)nI);
  double* x = (double*)malloc(sizeof(double) * (size_t)nI * d);
  double* z = (double*)malloc(sizeof(double) * (size_t)nI);
  double* w = (double*)malloc(sizeof(double) * (size_t)M0);
  int32_t* S = (int32_t*)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
  double* sc = (double*)malloc(sizeof(double) * (size_t)nI * (nc > 0 ? nc : 1));
  int32_t* ccode = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nc > 0 ? nc : 1));
  double* w2 = (double*)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
  int32_t* S2 = (int32_t*)malloc(sizeof(int32_t) * (size_t)(P2 > 0 ? P2 : 1));
  double* sg = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));

  /* coarse pass over the parents, as in attend_block */
  for (int r = 0; r < nI; ++r) {
    const double* q = Q + (size_t)(i0 + r) * d;
    for (int j = 0; j < M0; ++j) s[(size_t)r * M0 + j] = scale * dot(q, par_h + (size_t)j * d, d);
    m[r] = -INFINITY;
    for (int j = 0; j < M0; ++j)
      if (ns[j] > 0 && s[(size_t)r * M0 + j] > m[r]) m[r] = s[(size_t)r * M0 + j];
    for (int j = 0; j < M0; ++j)
      A[(size_t)r * M0 + j] = ns[j] > 0 ? exp(s[(size_t)r * M0 + j] - m[r]) : 0.0;
    for (int t = 0; t < d; ++t) x[(size_t)r * d + t] = 0.0;
    z[r] = 0.0;
    for (int j = 0; j < M0; ++j) {
      double a = A[(size_t)r * M0 + j];
      for (int t = 0; t < d; ++t) x[(size_t)r * d + t] += a * vs[(size_t)j * d + t];
      z[r] += a * ns[j];
    }
  }
  /* parents' importance (Eq. 7) and top-P */
  for (int j = 0; j < M0; ++j) {
    w[j] = 0.0;
    for (int r = 0; r < nI; ++r) w[j] += A[(size_t)r * M0 + j] * ns[j] / z[r];
  }
  if (imp_out) memcpy(imp_out, w, sizeof(double) * (size_t)M0);
  if (P > 0) {
    if (sel_in) memcpy(S, sel_in, sizeof(int32_t) * (size_t)P);
    else top_p(w, M0, P, S);
    if (sel_out) memcpy(sel_out, S, sizeof(int32_t) * (size_t)P);
  }
  /* child refinement of the selected parents (online max merge, Eqs. 8-9) */
  for (int k = 0; k < P; ++k)
    for (int c = 0; c < C; ++c) ccode[k * C + c] = M0 + S[k] * C + c;
  for (int r = 0; r < nI; ++r) {
    const double* q = Q + (size_t)(i0 + r) * d;
    for (int k = 0; k < P; ++k) {
      const int p = S[k];
      double* scr = sc + (size_t)r * nc + (size_t)k * C;
      for (int c = 0; c < C; ++c) scr[c] = scale * dot(q, ch_h + ((size_t)p * C + c) * d, d);
      double mp = m[r];
      for (int c = 0; c < C; ++c)
        if (ns[M0 + p * C + c] > 0 && scr[c] > mp) mp = scr[c];
      double f = exp(m[r] - mp);
      for (int t = 0; t < d; ++t) x[(size_t)r * d + t] *= f;
      z[r] *= f;
      m[r] = mp;
      double sp = 0.0;
      for (int c = 0; c < C; ++c) sp += scr[c];
      sp /= C;
      double Ap = exp(sp - m[r]);
      for (int c = 0; c < C; ++c) {
        const int x_c = M0 + p * C + c;
        double dA = ns[x_c] > 0 ? exp(scr[c] - m[r]) - Ap : 0.0;
        for (int t = 0; t < d; ++t) x[(size_t)r * d + t] += dA * vs[(size_t)x_c * d + t];
        z[r] += dA * ns[x_c];
      }
    }
  }
  /* the refined children's importance, with the logits and denominator of
   * the attention after the child refinement, and their top-P2 */
  for (int u = 0; u < nc; ++u) {
    w2[u] = 0.0;
    const double n_u = ns[ccode[u]];
    if (!(n_u > 0)) continue;
    for (int r = 0; r < nI; ++r) w2[u] += exp(sc[(size_t)r * nc + u] - m[r]) * n_u / z[r];
  }
  if (imp2_out) memcpy(imp2_out, w2, sizeof(double) * (size_t)nc);
  if (P2 > 0) {
    if (sel2_in) {
      /* caller's child codes -> candidate slots */
      for (int k = 0; k < P2; ++k) {
        S2[k] = 0;
        for (int u = 0; u < nc; ++u)
          if (ccode[u] == sel2_in[k]) S2[k] = u;
      }
    } else {
      top_p_codes(w2, ccode, nc, P2, S2);
    }
    if (sel2_out)
      for (int k = 0; k < P2; ++k) sel2_out[k] = ccode[S2[k]];
  }
  /* grandchild refinement of the selected children */
  for (int r = 0; r < nI; ++r) {
    const double* q = Q + (size_t)(i0 + r) * d;
    for (int k = 0; k < P2; ++k) {
      const int cc = ccode[S2[k]] - M0; /* child index m*C + c */
      for (int g = 0; g < C; ++g) sg[g] = scale * dot(q, gc_h + ((size_t)cc * C + g) * d, d);
      double mp = m[r];
      for (int g = 0; g < C; ++g)
        if (ns[M0 + M1 + cc * C + g] > 0 && sg[g] > mp) mp = sg[g];
      double f = exp(m[r] - mp);
      for (int t = 0; t < d; ++t) x[(size_t)r * d + t] *= f;
      z[r] *= f;
      m[r] = mp;
      /* the child's logit as the mean of its grandchildren's (Eq. 8) */
      double scm = 0.0;
      for (int g = 0; g < C; ++g) scm += sg[g];
      scm /= C;
      double Ac = exp(scm - m[r]);
      for (int g = 0; g < C; ++g) {
        const int x_g = M0 + M1 + cc * C + g;
        double dA = ns[x_g] > 0 ? exp(sg[g] - m[r]) - Ac : 0.0;
        for (int t = 0; t < d; ++t) x[(size_t)r * d + t] += dA * vs[(size_t)x_g * d + t];
        z[r] += dA * ns[x_g];
      }
    }
  }
  for (int r = 0; r < nI; ++r)
    for (int t = 0; t < d; ++t) O[(size_t)(i0 + r) * d + t] = x[(size_t)r * d + t] / z[r];

  free(s); free(A); free(m); free(x); free(z); free(w); free(S); free(sc); free(ccode);
  free(w2); free(S2); free(sg);
}

/* Stage 2, depth 3, over every (bh, query block).  sel [BH][nblk][P] parents,
 * sel2 [BH][nblk][P2] child codes, imp [BH][nblk][M0], imp2 [BH][nblk][P*C]
 * (candidate children in the order of sel, C each); sel_in / sel2_in
 * (nullable) override the two selections. */
void avq_oracle_attention3(int BH, int H, int N, int d, int M0, int C, int P, int P2, int block,
                           double scale, const double* Q, const double* parents,
                           const double* children, const double* grandchildren,
                           const double* vsum, const double* counts, const int32_t* sel_in,
                           const int32_t* sel2_in, double* O, int32_t* sel_out,
                           int32_t* sel2_out, double* imp_out, double* imp2_out) {
  const int M1 = M0 * C, Mt = M0 + M1 + M1 * C;
  const int nblk = (N + block - 1) / block;
#pragma omp parallel for schedule(dynamic)
  for (int u = 0; u < BH * nblk; ++u) {
    const int bh = u / nblk, b = u % nblk, h = bh % H;
    const int i0 = b * block, i1 = i0 + block < N ? i0 + block : N;
    const size_t sb = (size_t)bh * nblk + b;
    attend_block3(d, M0, C, P, P2, scale, Q + (size_t)bh * N * d, i0, i1,
                  parents + (size_t)h * M0 * d, children + (size_t)h * M1 * d,
                  grandchildren + (size_t)h * M1 * C * d, vsum + (size_t)bh * Mt * d,
                  counts + (size_t)bh * Mt, sel_in ? sel_in + sb * P : NULL,
                  sel2_in ? sel2_in + sb * P2 : NULL, O + (size_t)bh * N * d,
                  sel_out ? sel_out + sb * P : NULL, sel2_out ? sel2_out + sb * P2 : NULL,
                  imp_out ? imp_out + sb * M0 : NULL, imp2_out ? imp2_out + sb * P * C : NULL);
  }
}
