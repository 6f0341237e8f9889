/*
 * fp64 oracle for tree-indexed sparse decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  It shares no code,
 * header, table or helper with the CUDA path and never calls it.
 *
 * What it follows ("Subquadratic Attention with a Hierarchical Tree-Structured
 * Indexer" (ZHA), abstract: a tree of recursively compressed key summaries over
 * the KV cache, traversed top-down by each query to retrieve a sparse subset of
 * keys, whose tree grows in depth as the cache grows, followed by a final
 * attention over the retrieved keys; "ALHR" news item, technical features: a
 * static tree over the keys).  The open points are read as follows:
 *   - summary operator: leaf = arithmetic mean of the keys of its leaf block
 *     (tokens t < N only); node = unweighted mean of its existing children;
 *   - scoring: q . summary (unscaled; the 1/sqrt(d) factor does not change
 *     the order);
 *   - beam: the top-B candidates per level in total, ordered by score
 *     descending, lower node index first on equal scores;
 *   - levels: L = the smallest L >= 1 with b^L >= n0; the root (level L, one
 *     node) is not scored, routing starts from its children;
 *   - final attention: exact softmax over the union of the tokens of the
 *     selected leaves, two passes (max, then exp/sum/weighted V).
 *   - threshold descent ("Louver" explainer): bounding spheres centered on the
 *     summaries (leaf radius: farthest token; node radius: farthest child sphere),
 *     a child kept iff q . c + ||q|| r >= tau, exact check of the surviving
 *     leaves' tokens; pinned against a scan of all keys.
 *   - bf16-stored summaries (optional): each stored node is the bf16 rounding of
 *     its fp32-rounded fp64 mean, and parents average the stored children.
 *
 * Every computation is a plain loop in fp64 over inputs converted exactly
 * (bf16 -> fp64 and fp32 -> fp64 are exact).  One library routine is used:
 * qsort, for ordering candidates.  Single-threaded.
 *
 * Parity pins (tests/test_oracle.py): closed forms (root of a full tree =
 * mean of all tokens; constant keys), a hand-worked tree (tests/golden),
 * append == rebuild exactly on dyadic inputs, brute-force subset enumeration
 * of every beam step on tiny trees, q = 0 ties, monotone trees against a
 * library partial sort, beam >= n0 against a library softmax, single-token
 * attention and planted needles.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* dtype codes of the inputs: 0 = fp32, 1 = bf16 (raw 16-bit patterns). */
static double in_elem(const void *p, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float *)p)[i];
  uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
  float f;
  memcpy(&f, &bits, 4);
  return (double)f;
}

/* Number of leaves for N tokens with leaf block lb: ceil(N / lb). */
int64_t orc_num_leaves(int64_t N, int64_t lb) { return N <= 0 ? 0 : (N + lb - 1) / lb; }

/* Levels above the leaves: smallest L >= 1 with b^L >= n0 (0 for an empty tree). */
int orc_num_levels(int64_t n0, int64_t b) {
  if (n0 <= 0) return 0;
  int L = 1;
  int64_t span = b;
  while (span < n0) {
    span *= b;
    L++;
  }
  return L;
}

/*
 * Leaf summaries: out[(i - i0) * d + k] = mean over t in [i*lb, min(i*lb+lb, N))
 * of K[t*d + k], for leaves i in [i0, i1).  K is one (batch, KV-head) slice,
 * rows of d elements.
 */
void orc_leaf_means(const void *K, int dtype, int64_t d, int64_t N, int64_t lb, int64_t i0,
                    int64_t i1, double *out) {
  for (int64_t i = i0; i < i1; ++i) {
    int64_t t0 = i * lb;
    int64_t t1 = t0 + lb < N ? t0 + lb : N;
    double *o = out + (i - i0) * d;
    for (int64_t k = 0; k < d; ++k) {
      double s = 0.0;
      for (int64_t t = t0; t < t1; ++t) s += in_elem(K, dtype, t * d + k);
      o[k] = s / (double)(t1 - t0);
    }
  }
}

/*
 * Parent summaries: out[(i - i0) * d + k] = mean over the existing children
 * j in [b*i, min(b*i+b, n_child)) of child[j*d + k], for nodes i in [i0, i1).
 */
void orc_parent_means(const double *child, int64_t n_child, int64_t d, int64_t b, int64_t i0,
                      int64_t i1, double *out) {
  for (int64_t i = i0; i < i1; ++i) {
    int64_t j0 = b * i;
    int64_t j1 = j0 + b < n_child ? j0 + b : n_child;
    double *o = out + (i - i0) * d;
    for (int64_t k = 0; k < d; ++k) {
      double s = 0.0;
      for (int64_t j = j0; j < j1; ++j) s += child[j * d + k];
      o[k] = s / (double)(j1 - j0);
    }
  }
}

typedef struct {
  double score;
  int64_t idx;
} cand_t;

/* Descending score; on equal scores the lower node index comes first. */
static int by_score_then_index(const void *a, const void *b) {
  const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

static int by_index(const void *a, const void *b) {
  const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

/*
 * Top-down beam routing for nq queries over one tree.
 *   pyr: all levels of one tree, level l at rows [off[l], off[l] + cnt[l]),
 *        rows of d fp64 values; level L is the root (cnt[L] == 1).
 *   Q:   nq x d fp64 queries.
 * Outputs (per query):
 *   leaves[q*beam + j]: selected leaves, ascending, -1 padded;
 *   leaf_scores[q*beam + j]: q . S0[leaf] for those leaves (NaN on padding);
 *   bounds[(q*L + (L-1-l))*2 + {0,1}]: s_(B) and s_(B+1), the scores of the
 *        last kept and the first dropped candidate of level l in the order
 *        above (NaN, NaN when the level has at most B candidates);
 *   survivors[(q*L + (L-1-l))*beam + j]: the kept nodes of level l, ascending,
 *        -1 padded (may be NULL);
 *   ncand[q*L + (L-1-l)]: number of candidates scored at level l (may be NULL).
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int orc_route(const double *pyr, const int64_t *off, const int64_t *cnt, int L, int64_t d,
              int64_t b, const double *Q, int64_t nq, int64_t beam, int64_t *leaves,
              double *leaf_scores, double *bounds, int64_t *survivors, int64_t *ncand) {
  if (L < 1 || beam < 1 || b < 2) return -1;
  int64_t maxc = beam * b;
  cand_t *C = (cand_t *)malloc(sizeof(cand_t) * (size_t)maxc);
  int64_t *surv = (int64_t *)malloc(sizeof(int64_t) * (size_t)beam);
  if (!C || !surv) {
    free(C);
    free(surv);
    return -1;
  }
  for (int64_t qi = 0; qi < nq; ++qi) {
    const double *q = Q + qi * d;
    int64_t m = 1;
    surv[0] = 0; /* the root */
    for (int l = L - 1; l >= 0; --l) {
      const double *S = pyr + off[l] * d;
      int64_t nc = 0;
      for (int64_t s = 0; s < m; ++s) {
        int64_t c0 = b * surv[s];
        int64_t c1 = c0 + b < cnt[l] ? c0 + b : cnt[l];
        for (int64_t c = c0; c < c1; ++c) {
          double acc = 0.0;
          for (int64_t k = 0; k < d; ++k) acc += q[k] * S[c * d + k];
          C[nc].score = acc;
          C[nc].idx = c;
          nc++;
        }
      }
      qsort(C, (size_t)nc, sizeof(cand_t), by_score_then_index);
      int64_t keep = nc < beam ? nc : beam;
      int64_t lvl = qi * L + (L - 1 - l);
      if (bounds) {
        bounds[2 * lvl] = nc > beam ? C[keep - 1].score : NAN;
        bounds[2 * lvl + 1] = nc > beam ? C[keep].score : NAN;
      }
      if (ncand) ncand[lvl] = nc;
      qsort(C, (size_t)keep, sizeof(cand_t), by_index);
      for (int64_t j = 0; j < keep; ++j) surv[j] = C[j].idx;
      m = keep;
      if (survivors)
        for (int64_t j = 0; j < beam; ++j) survivors[lvl * beam + j] = j < keep ? surv[j] : -1;
      if (l == 0) {
        for (int64_t j = 0; j < beam; ++j) {
          leaves[qi * beam + j] = j < keep ? C[j].idx : -1;
          if (leaf_scores) leaf_scores[qi * beam + j] = j < keep ? C[j].score : NAN;
        }
      }
    }
  }
  free(C);
  free(surv);
  return 0;
}

/*
 * Exact softmax attention of one query over the tokens of the given leaves
 * (tokens t < N only; leaf indices < 0 are skipped):
 *   s_t = scale * q . K[t];  o = sum_t exp(s_t - max) V[t] / sum_t exp(s_t - max).
 * K, V: one (batch, KV-head) slice of rows of d elements.  Returns the number
 * of tokens attended.
 */
int64_t orc_attend(const double *q, const void *K, const void *V, int dtype, int64_t d, int64_t N,
                   int64_t lb, const int64_t *leaves, int64_t nleaves, double scale, double *out) {
  double mx = -INFINITY;
  int64_t ntok = 0;
  for (int64_t j = 0; j < nleaves; ++j) {
    if (leaves[j] < 0) continue;
    int64_t t0 = leaves[j] * lb, t1 = t0 + lb < N ? t0 + lb : N;
    for (int64_t t = t0; t < t1; ++t) {
      double s = 0.0;
      for (int64_t k = 0; k < d; ++k) s += q[k] * in_elem(K, dtype, t * d + k);
      s *= scale;
      if (s > mx) mx = s;
      ntok++;
    }
  }
  for (int64_t k = 0; k < d; ++k) out[k] = 0.0;
  if (ntok == 0) return 0;
  double den = 0.0;
  for (int64_t j = 0; j < nleaves; ++j) {
    if (leaves[j] < 0) continue;
    int64_t t0 = leaves[j] * lb, t1 = t0 + lb < N ? t0 + lb : N;
    for (int64_t t = t0; t < t1; ++t) {
      double s = 0.0;
      for (int64_t k = 0; k < d; ++k) s += q[k] * in_elem(K, dtype, t * d + k);
      double p = exp(s * scale - mx);
      den += p;
      for (int64_t k = 0; k < d; ++k) out[k] += p * in_elem(V, dtype, t * d + k);
    }
  }
  for (int64_t k = 0; k < d; ++k) out[k] /= den;
  return ntok;
}

/* Dense softmax attention of one query over all tokens t < N (same formula). */
void orc_dense(const double *q, const void *K, const void *V, int dtype, int64_t d, int64_t N,
               double scale, double *out) {
  double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  double mx = -INFINITY;
  for (int64_t t = 0; t < N; ++t) {
    double a = 0.0;
    for (int64_t k = 0; k < d; ++k) a += q[k] * in_elem(K, dtype, t * d + k);
    s[t] = a * scale;
    if (s[t] > mx) mx = s[t];
  }
  for (int64_t k = 0; k < d; ++k) out[k] = 0.0;
  double den = 0.0;
  for (int64_t t = 0; t < N; ++t) {
    double p = exp(s[t] - mx);
    den += p;
    for (int64_t k = 0; k < d; ++k) out[k] += p * in_elem(V, dtype, t * d + k);
  }
  if (N > 0)
    for (int64_t k = 0; k < d; ++k) out[k] /= den;
  free(s);
}

/*
 * Bounding spheres and threshold descent ("Louver" explainer, index design: every cluster
 * of keys is enclosed in a bounding sphere with a center and a radius; a query with
 * threshold tau wants every key in the halfspace {p : q . p >= tau}; a cluster whose sphere
 * misses the halfspace is pruned, the keys of the others are checked exactly, so no key
 * with q . k >= tau is missed).  On this tree the center of a node is its summary and the
 * radius covers every key of its subtree:
 *   leaf i:  r = max over its tokens t < N of ||k_t - c_i||
 *   node i:  r = max over its existing children j of (||c_j - c_i|| + r_j)
 * (a child's sphere lies inside the ball of radius ||c_j - c_i|| + r_j around c_i, by the
 * triangle inequality, so the node's sphere contains all of its subtree's keys).
 */

/* Radii of leaves [0, n0): centers [n0][d] (the leaf summaries). */
void orc_leaf_radii(const void *K, int dtype, int64_t d, int64_t N, int64_t lb, const double *centers,
                    int64_t n0, double *out) {
  for (int64_t i = 0; i < n0; ++i) {
    int64_t t0 = i * lb, t1 = t0 + lb < N ? t0 + lb : N;
    double best = 0.0;
    for (int64_t t = t0; t < t1; ++t) {
      double s = 0.0;
      for (int64_t k = 0; k < d; ++k) {
        double e = in_elem(K, dtype, t * d + k) - centers[i * d + k];
        s += e * e;
      }
      if (s > best) best = s;
    }
    out[i] = sqrt(best);
  }
}

/* Radii of the parents [0, n_parent) of children [0, n_child) (centers and radii given). */
void orc_parent_radii(const double *child_c, const double *child_r, int64_t n_child, const double *parent_c,
                      int64_t n_parent, int64_t d, int64_t b, double *out) {
  for (int64_t i = 0; i < n_parent; ++i) {
    int64_t j0 = i * b, j1 = j0 + b < n_child ? j0 + b : n_child;
    double best = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
      double s = 0.0;
      for (int64_t k = 0; k < d; ++k) {
        double e = child_c[j * d + k] - parent_c[i * d + k];
        s += e * e;
      }
      double r = sqrt(s) + child_r[j];
      if (r > best) best = r;
    }
    out[i] = best;
  }
}

/* Every token t < N with q . k_t >= tau, ascending (up to max_out written); returns the count. */
int64_t orc_threshold_brute(const void *K, int dtype, int64_t d, int64_t N, const double *q, double tau,
                            int64_t *out, int64_t max_out) {
  int64_t n = 0;
  for (int64_t t = 0; t < N; ++t) {
    double s = 0.0;
    for (int64_t k = 0; k < d; ++k) s += q[k] * in_elem(K, dtype, t * d + k);
    if (s >= tau) {
      if (n < max_out) out[n] = t;
      n++;
    }
  }
  return n;
}

/*
 * Threshold descent over a tree (pyr: every level's summaries, level l at rows off[l] ..,
 * cnt[l] nodes; radii in the same row order).  Survivors start as {root}; for l = L-1 .. 0
 * the children of the survivors are kept iff q . c + ||q|| r >= tau.  The tokens of the
 * surviving leaves are then checked exactly.  Writes the tokens found in ascending order (up
 * to max_out), returns their count; *tested = number of sphere tests.
 */
int64_t orc_threshold_descent(const double *pyr, const double *radii, const int64_t *off, const int64_t *cnt,
                              int L, int64_t d, int64_t b, int64_t lb, int64_t N, const void *K, int dtype,
                              const double *q, double tau, int64_t *out, int64_t max_out, int64_t *tested) {
  double qn = 0.0;
  for (int64_t k = 0; k < d; ++k) qn += q[k] * q[k];
  qn = sqrt(qn);
  int64_t cap = cnt[0] + 1;
  int64_t *cur = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
  int64_t *nxt = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
  int64_t m = 1, ntest = 0;
  cur[0] = 0;
  for (int l = L - 1; l >= 0; --l) {
    int64_t mn = 0;
    for (int64_t j = 0; j < m; ++j) {
      int64_t c0 = cur[j] * b, c1 = c0 + b < cnt[l] ? c0 + b : cnt[l];
      for (int64_t c = c0; c < c1; ++c) {
        const double *row = pyr + (off[l] + c) * d;
        double s = 0.0;
        for (int64_t k = 0; k < d; ++k) s += q[k] * row[k];
        ntest++;
        if (s + qn * radii[off[l] + c] >= tau) nxt[mn++] = c;
      }
    }
    int64_t *tmp = cur;
    cur = nxt;
    nxt = tmp;
    m = mn;
  }
  int64_t n = 0;
  for (int64_t j = 0; j < m; ++j) {
    int64_t t0 = cur[j] * lb, t1 = t0 + lb < N ? t0 + lb : N;
    for (int64_t t = t0; t < t1; ++t) {
      double s = 0.0;
      for (int64_t k = 0; k < d; ++k) s += q[k] * in_elem(K, dtype, t * d + k);
      if (s >= tau) {
        if (n < max_out) out[n] = t;
        n++;
      }
    }
  }
  free(cur);
  free(nxt);
  if (tested) *tested = ntest;
  return n;
}

/*
 * Summaries stored in bf16 (an option of the tree, halving the bytes a route reads).  The
 * pages fix no storage precision; the reading taken here: the stored value of a node is its
 * fp64 mean rounded to the nearest fp32 (ties to even) and that fp32 value rounded to the
 * nearest bf16 (ties to even) -- the bf16 rounding of what an fp32 tree would store -- and
 * every parent averages the STORED values of its children.  This replaces each x[i] by the
 * fp64 value of its stored bf16.  Rounding to bf16 by hand: keep the top 16 bits of the
 * fp32 pattern after adding half a bf16 unit (0x7FFF) plus the lowest kept bit (ties to
 * even); NaN stays NaN.
 */
void orc_round_bf16(double *x, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    float f = (float)x[i];
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) {
      u |= 0x00400000u;
    } else {
      u += 0x7FFFu + ((u >> 16) & 1u);
    }
    u &= 0xFFFF0000u;
    memcpy(&f, &u, 4);
    x[i] = (double)f;
  }
}
