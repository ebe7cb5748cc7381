/*
 * lsa_oracle.c -- plain, slow, fp64 CPU oracle for the Latent Sparse Attention
 * (LSA) hierarchical latent-key path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  The product
 * (the CUDA library and its binding) never calls it and shares no code with it.
 *
 * Sources followed (pages about "Latent Sparse Attention"):
 *  [P1] kongchang.com, "Latent Sparse Attention Breaks Through the Million-Token
 *       Context Bottleneck", section "How LSA Sidesteps Per-Key Scoring with
 *       Hierarchical Clustering" (latent projection of keys; tree whose root holds
 *       all keys and whose levels get finer; top-down walk scoring a few candidate
 *       clusters per level), and section "The Accuracy-Efficiency Dilemma"
 *       (sparse attention over k selected keys, O(nkd)).
 *  [P4] bdtechtalks.com, "Latent sparse attention", section "How latent sparse
 *       attention works" (centroid per cluster stored with references to the
 *       original keys; a fixed number of original keys retrieved from the chosen
 *       clusters; flat search vs hierarchical search with a fixed budget per
 *       level).
 * Where the pages leave a step open, the reading used is stated at the step.
 *
 * Every floating-point quantity here is double precision; inputs arrive as the
 * stored values (bf16 or fp32) widened to double by the caller.
 *
 * Parity pins: every function below is checked in the CPU test suite against
 * something other than itself (published generator vectors, brute-force
 * enumeration, closed forms, a library attention routine, finite differences).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_SHAPE 2
#define ORC_ERR_ALLOC 3
#define ORC_ERR_NONFINITE 5

#define ORC_MAX_LEVELS 8

/* ------------------------------------------------------------------------- */
/* SplitMix64 (Steele, Lea & Flood, "Fast Splittable Pseudorandom Number     */
/* Generators", OOPSLA 2014): the state advances by the odd constant gamma    */
/* and each output is the state passed through the variant-13 mixer.          */
/* The pages fix no initialisation for the k-means; this seeded hash is the   */
/* reading used for "seeded init".                                            */
/* ------------------------------------------------------------------------- */
static const uint64_t SM64_GAMMA = 0x9e3779b97f4a7c15ULL;

uint64_t orc_splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

/* Output number i (0-based) of the generator whose state starts at s. */
uint64_t orc_splitmix64_at(uint64_t s, uint64_t i) {
  return orc_splitmix64_mix(s + (i + 1) * SM64_GAMMA);
}

/* Hash that orders the members of a segment for the seeded initialisation of
 * level `level`: the level's stream state is output `level` of the stream
 * seeded with `seed`; the key at position `pos` gets output `pos` of it.  Both
 * maps are bijections, so distinct positions never tie. */
uint64_t orc_init_hash(uint64_t seed, int32_t level, int64_t pos) {
  uint64_t s = orc_splitmix64_at(seed, (uint64_t)level);
  return orc_splitmix64_at(s, (uint64_t)pos);
}

/* ------------------------------------------------------------------------- */
/* Latent projection [P1 "How LSA Sidesteps ...": keys are mapped into a      */
/* low-dimensional latent space].  Z[i,:] = X[i,:] . W  with W of shape [d,r].*/
/* ------------------------------------------------------------------------- */
int orc_project(const double *X, int64_t n, int32_t d, const double *W,
                int32_t r, double *Z) {
  if (!X || !W || !Z || n < 0 || d <= 0 || r <= 0) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    for (int32_t k = 0; k < r; ++k) {
      double acc = 0.0;
      for (int32_t j = 0; j < d; ++j) acc += X[i * d + j] * W[(int64_t)j * r + k];
      Z[i * r + k] = acc;
    }
  }
  return ORC_OK;
}

/* Query latent for one GQA group: the G query heads of a group share one
 * selection (the last-chunk prefill workload states that a group of 4 query
 * heads shares it), so the group's query is the mean of its G head rows,
 * projected with the same W as the keys.  Qg: [T, G, d] -> qlat: [T, r]. */
int orc_query_latent(const double *Qg, int64_t T, int32_t G, int32_t d,
                     const double *W, int32_t r, double *qlat) {
  if (!Qg || !W || !qlat || T < 0 || G <= 0 || d <= 0 || r <= 0) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double *mean = (double *)malloc(sizeof(double) * d);
    for (int32_t j = 0; j < d; ++j) {
      double s = 0.0;
      for (int32_t g = 0; g < G; ++g) s += Qg[(t * G + g) * d + j];
      mean[j] = s / (double)G;
    }
    for (int32_t k = 0; k < r; ++k) {
      double acc = 0.0;
      for (int32_t j = 0; j < d; ++j) acc += mean[j] * W[(int64_t)j * r + k];
      qlat[t * r + k] = acc;
    }
    free(mean);
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Balanced assignment of m keys to b clusters of capacity m/b.               */
/* Reading (the pages only say the tree is "similar to hierarchical k-means"  */
/* and the workloads fix an exact leaf size): rank every (key, cluster) pair  */
/* by (distance asc, key position asc, cluster asc); scan the pairs in that   */
/* order and give a key to a cluster when the key is still free and the       */
/* cluster still has room.  With preferences read off one global pair order,  */
/* this greedy result is the unique stable assignment.                        */
/* D: [m, b] distances; pos: [m] key positions; assign: [m] cluster in [0,b). */
/* ------------------------------------------------------------------------- */
typedef struct {
  double d;
  int64_t pos;
  int32_t c;
  int32_t i;
} orc_pair;

static int orc_pair_cmp(const void *a, const void *b) {
  const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
  if (x->d < y->d) return -1;
  if (x->d > y->d) return 1;
  if (x->pos < y->pos) return -1;
  if (x->pos > y->pos) return 1;
  return (x->c > y->c) - (x->c < y->c);
}

int orc_balanced_assign(const double *D, const int64_t *pos, int64_t m,
                        int32_t b, int32_t *assign) {
  if (!D || !pos || !assign || m <= 0 || b <= 0) return ORC_ERR_ARG;
  if (m % b != 0) return ORC_ERR_SHAPE;
  const int64_t cap = m / b;
  orc_pair *pairs = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(m * b));
  int64_t *count = (int64_t *)calloc((size_t)b, sizeof(int64_t));
  if (!pairs || !count) { free(pairs); free(count); return ORC_ERR_ALLOC; }
  for (int64_t i = 0; i < m; ++i) {
    assign[i] = -1;
    for (int32_t c = 0; c < b; ++c) {
      double v = D[i * b + c];
      if (isnan(v)) { free(pairs); free(count); return ORC_ERR_NONFINITE; }
      orc_pair p = {v, pos[i], c, (int32_t)i};
      pairs[i * b + c] = p;
    }
  }
  qsort(pairs, (size_t)(m * b), sizeof(orc_pair), orc_pair_cmp);
  for (int64_t k = 0; k < m * b; ++k) {
    const orc_pair *p = &pairs[k];
    if (assign[p->i] < 0 && count[p->c] < cap) {
      assign[p->i] = p->c;
      count[p->c] += 1;
    }
  }
  free(pairs);
  free(count);
  return ORC_OK;
}

/* Squared Euclidean distance of each member row to each centroid (k-means). */
int orc_distances(const double *Zs, int64_t m, int32_t r, const double *mu,
                  int32_t b, double *D) {
  if (!Zs || !mu || !D) return ORC_ERR_ARG;
  for (int64_t i = 0; i < m; ++i)
    for (int32_t c = 0; c < b; ++c) {
      double acc = 0.0;
      for (int32_t k = 0; k < r; ++k) {
        double diff = Zs[i * r + k] - mu[(int64_t)c * r + k];
        acc += diff * diff;
      }
      D[i * b + c] = acc;
    }
  return ORC_OK;
}

/* Seeded initialisation of the b children of one segment: child j starts at the
 * latent row of the member with the j-th smallest init hash. */
int orc_level_init(const double *Zs, const int64_t *pos, int64_t m, int32_t r,
                   int32_t b, uint64_t seed, int32_t level, double *mu) {
  if (!Zs || !pos || !mu || b > m) return ORC_ERR_ARG;
  char *taken = (char *)calloc((size_t)m, 1);
  if (!taken) return ORC_ERR_ALLOC;
  for (int32_t j = 0; j < b; ++j) {
    int64_t best = -1;
    uint64_t best_h = 0;
    for (int64_t i = 0; i < m; ++i) {
      if (taken[i]) continue;
      uint64_t h = orc_init_hash(seed, level, pos[i]);
      if (best < 0 || h < best_h) { best = i; best_h = h; }
    }
    taken[best] = 1;
    memcpy(&mu[(int64_t)j * r], &Zs[best * r], sizeof(double) * r);
  }
  free(taken);
  return ORC_OK;
}

/* Centroid = mean of the latent rows assigned to it ([P4 "How latent sparse
 * attention works": each cluster is represented by a centroid]). */
int orc_means(const double *Zs, int64_t m, int32_t r, const int32_t *assign,
              int32_t b, double *mu) {
  if (!Zs || !assign || !mu) return ORC_ERR_ARG;
  int64_t *cnt = (int64_t *)calloc((size_t)b, sizeof(int64_t));
  if (!cnt) return ORC_ERR_ALLOC;
  memset(mu, 0, sizeof(double) * (size_t)b * r);
  for (int64_t i = 0; i < m; ++i) {
    int32_t c = assign[i];
    cnt[c] += 1;
    for (int32_t k = 0; k < r; ++k) mu[(int64_t)c * r + k] += Zs[i * r + k];
  }
  for (int32_t c = 0; c < b; ++c)
    for (int32_t k = 0; k < r; ++k)
      mu[(int64_t)c * r + k] = cnt[c] ? mu[(int64_t)c * r + k] / (double)cnt[c] : 0.0;
  free(cnt);
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Tree build, top-down ([P1]: the root holds every key and the clusters get  */
/* finer toward the leaves; "similar to hierarchical k-means").               */
/* Level l splits every level-(l-1) node (the root for l = 0) into b_l        */
/* children numbered parent*b_l + j, by `iters` rounds of (balanced           */
/* assignment, mean update) from the seeded initialisation.  The stored       */
/* centroids are the means of the last assignment.                            */
/* Outputs: centroids of all levels concatenated ([N_0,r], [N_1,r], ...),     */
/* min_pos of all levels concatenated (smallest member position per node),    */
/* leaf_index [n] = keys of leaf 0 in ascending position, then leaf 1, ...    */
/* trace (optional): [levels, iters, n] node id of each key (indexed by key   */
/* position) after each assignment.                                           */
/* ------------------------------------------------------------------------- */
int orc_build_tree(const double *Z, int64_t n, int32_t r, const int32_t *branching,
                   int32_t levels, int32_t leaf_size, int32_t iters, uint64_t seed,
                   double *centroids, int32_t *min_pos, int32_t *leaf_index,
                   int32_t *trace) {
  if (!Z || !branching || !centroids || !min_pos || !leaf_index) return ORC_ERR_ARG;
  if (levels < 1 || levels > ORC_MAX_LEVELS || leaf_size < 1 || iters < 1 || r < 1)
    return ORC_ERR_ARG;
  int64_t prod = leaf_size;
  for (int32_t l = 0; l < levels; ++l) {
    if (branching[l] < 1) return ORC_ERR_ARG;
    prod *= branching[l];
  }
  if (prod != n) return ORC_ERR_SHAPE;

  int64_t *order = (int64_t *)malloc(sizeof(int64_t) * n);  /* keys in segment order */
  int64_t *next = (int64_t *)malloc(sizeof(int64_t) * n);
  if (!order || !next) { free(order); free(next); return ORC_ERR_ALLOC; }
  for (int64_t i = 0; i < n; ++i) order[i] = i;

  int64_t segs = 1, cent_off = 0, node_off = 0;
  int err = ORC_OK;
  for (int32_t l = 0; l < levels && err == ORC_OK; ++l) {
    const int32_t b = branching[l];
    const int64_t m = n / segs, cap = m / b;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t s = 0; s < segs; ++s) {
      const int64_t *pos = &order[s * m];
      double *Zs = (double *)malloc(sizeof(double) * m * r);
      double *D = (double *)malloc(sizeof(double) * m * b);
      double *mu = (double *)malloc(sizeof(double) * b * r);
      int32_t *a = (int32_t *)malloc(sizeof(int32_t) * m);
      int64_t *fill = (int64_t *)calloc((size_t)b, sizeof(int64_t));
      int e = (Zs && D && mu && a && fill) ? ORC_OK : ORC_ERR_ALLOC;
      if (e == ORC_OK) {
        for (int64_t i = 0; i < m; ++i) memcpy(&Zs[i * r], &Z[pos[i] * r], sizeof(double) * r);
        e = orc_level_init(Zs, pos, m, r, b, seed, l, mu);
      }
      for (int32_t t = 0; t < iters && e == ORC_OK; ++t) {
        orc_distances(Zs, m, r, mu, b, D);
        e = orc_balanced_assign(D, pos, m, b, a);
        if (e != ORC_OK) break;
        if (trace)
          for (int64_t i = 0; i < m; ++i)
            trace[((int64_t)l * iters + t) * n + pos[i]] = (int32_t)(s * b + a[i]);
        orc_means(Zs, m, r, a, b, mu);
      }
      if (e == ORC_OK) {
        for (int32_t j = 0; j < b; ++j) {
          memcpy(&centroids[cent_off + (s * b + j) * r], &mu[(int64_t)j * r], sizeof(double) * r);
          min_pos[node_off + s * b + j] = INT32_MAX;
        }
        /* stable split: members of child j keep ascending position order */
        for (int64_t i = 0; i < m; ++i) {
          int32_t j = a[i];
          next[(s * b + j) * cap + fill[j]] = pos[i];
          fill[j] += 1;
          if (pos[i] < min_pos[node_off + s * b + j]) min_pos[node_off + s * b + j] = (int32_t)pos[i];
        }
      }
      if (e != ORC_OK) {
#pragma omp critical
        err = e;
      }
      free(Zs); free(D); free(mu); free(a); free(fill);
    }
    int64_t *tmp = order; order = next; next = tmp;
    cent_off += segs * b * r;
    node_off += segs * b;
    segs *= b;
  }
  if (err == ORC_OK)
    for (int64_t i = 0; i < n; ++i) leaf_index[i] = (int32_t)order[i];
  free(order);
  free(next);
  return err;
}

/* ------------------------------------------------------------------------- */
/* Pooling of consecutive keys ([P4] "How latent sparse attention works": the  */
/* keys are first pooled into smaller representations, then clustered).       */
/* Reading (the pages give neither the pooling operator nor the block size):   */
/* block j holds the p consecutive keys at positions [j*p, (j+1)*p) and is     */
/* represented by the mean of their latent rows.                              */
/* Zp: [n/p, r].                                                               */
/* ------------------------------------------------------------------------- */
int orc_pool_keys(const double *Z, int64_t n, int32_t r, int32_t p, double *Zp) {
  if (!Z || !Zp || p < 1 || r < 1) return ORC_ERR_ARG;
  if (n % p) return ORC_ERR_SHAPE;
  for (int64_t j = 0; j < n / p; ++j)
    for (int32_t c = 0; c < r; ++c) {
      double s = 0.0;
      for (int32_t i = 0; i < p; ++i) s += Z[(j * p + i) * r + c];
      Zp[j * r + c] = s / p;
    }
  return ORC_OK;
}

/* Tree over pooled blocks: the build above runs on the n/p block rows (a      */
/* block's position is its index j, which orders pairs and seeds the start),  */
/* with leaf_size/p blocks per leaf.  The cluster then references the         */
/* original keys of its blocks ([P4]: centroids stored with references to the */
/* original keys): leaf_index lists, for each block j of a leaf in ascending  */
/* order, the keys j*p .. j*p+p-1, and min_pos is in key positions.            */
/* trace (optional): [levels, iters, n/p] node id of each block.               */
int orc_build_tree_pooled(const double *Z, int64_t n, int32_t r, int32_t p, const int32_t *branching,
                          int32_t levels, int32_t leaf_size, int32_t iters, uint64_t seed,
                          double *centroids, int32_t *min_pos, int32_t *leaf_index, int32_t *trace) {
  if (!Z || !branching || !centroids || !min_pos || !leaf_index || p < 1) return ORC_ERR_ARG;
  if (n % p || leaf_size % p) return ORC_ERR_SHAPE;
  if (levels < 1 || levels > ORC_MAX_LEVELS) return ORC_ERR_ARG;
  const int64_t nb = n / p;
  double *Zp = (double *)malloc(sizeof(double) * nb * r);
  int32_t *blocks = (int32_t *)malloc(sizeof(int32_t) * nb);
  if (!Zp || !blocks) { free(Zp); free(blocks); return ORC_ERR_ALLOC; }
  int err = orc_pool_keys(Z, n, r, p, Zp);
  if (err == ORC_OK)
    err = orc_build_tree(Zp, nb, r, branching, levels, leaf_size / p, iters, seed, centroids, min_pos, blocks,
                         trace);
  if (err == ORC_OK) {
    int64_t nodes = 0, level_nodes = 1;
    for (int32_t l = 0; l < levels; ++l) {
      level_nodes *= branching[l];
      nodes += level_nodes;
    }
    for (int64_t k = 0; k < nodes; ++k) min_pos[k] *= p;
    for (int64_t s = 0; s < nb; ++s)
      for (int32_t i = 0; i < p; ++i) leaf_index[s * p + i] = blocks[s] * p + i;
  }
  free(Zp);
  free(blocks);
  return err;
}

/* ------------------------------------------------------------------------- */
/* Tree update on append ([P1]: the tree can be precomputed and then updated). */
/* Reading (the pages give no update rule; every node of a level has the same */
/* fan-out, so only the top level can grow): once U = leaf_size * b_1 * ...  */
/* * b_{L-1} keys have been appended after the n_old indexed ones, they get a  */
/* subtree of their own -- the build above run on those U keys alone with     */
/* branching b_1..b_{L-1} (positions counted from the block's first key, the  */
/* same seed) -- attached as top-level node b_0.  Its root centroid is the    */
/* mean of the U keys' latent rows.  Every old node keeps its id and values;  */
/* the subtree's nodes follow the old ones on each level, and its min_pos and */
/* leaf_index are shifted by n_old.  One head; levels >= 2.                    */
/* Outputs use the grown tree's layout (b_0 + 1 top nodes); trace (optional): */
/* [levels-1, iters, U] of the subtree's build.                                */
/* ------------------------------------------------------------------------- */
int orc_tree_append(const double *old_cent, const int32_t *old_min_pos, const int32_t *old_leaf, int64_t n_old,
                    const double *Znew, int64_t U, int32_t r, const int32_t *branching, int32_t levels,
                    int32_t leaf_size, int32_t iters, uint64_t seed, double *cent, int32_t *min_pos,
                    int32_t *leaf_index, int32_t *trace) {
  if (!old_cent || !old_min_pos || !old_leaf || !Znew || !branching || !cent || !min_pos || !leaf_index)
    return ORC_ERR_ARG;
  if (levels < 2 || levels > ORC_MAX_LEVELS) return ORC_ERR_ARG;
  int64_t sub_nodes_total = 0, level_nodes = 1;
  for (int32_t l = 1; l < levels; ++l) {
    level_nodes *= branching[l];
    sub_nodes_total += level_nodes;
  }
  if (level_nodes * leaf_size != U) return ORC_ERR_SHAPE;
  double *sc = (double *)malloc(sizeof(double) * sub_nodes_total * r);
  int32_t *sm = (int32_t *)malloc(sizeof(int32_t) * sub_nodes_total);
  int32_t *sl = (int32_t *)malloc(sizeof(int32_t) * U);
  if (!sc || !sm || !sl) { free(sc); free(sm); free(sl); return ORC_ERR_ALLOC; }
  int err = orc_build_tree(Znew, U, r, branching + 1, levels - 1, leaf_size, iters, seed, sc, sm, sl, trace);
  if (err == ORC_OK) {
    int64_t old_off = 0, new_off = 0, sub_off = 0;   /* node offsets of the level in each array */
    int64_t old_nodes = branching[0], sub_nodes = 1;
    for (int32_t l = 0; l < levels; ++l) {
      if (l > 0) {
        old_nodes *= branching[l];
        sub_nodes *= branching[l];
      }
      memcpy(&cent[new_off * r], &old_cent[old_off * r], sizeof(double) * old_nodes * r);
      memcpy(&min_pos[new_off], &old_min_pos[old_off], sizeof(int32_t) * old_nodes);
      if (l == 0) {   /* the new top node: mean of every appended key */
        for (int32_t c = 0; c < r; ++c) {
          double s = 0.0;
          for (int64_t i = 0; i < U; ++i) s += Znew[i * r + c];
          cent[(new_off + old_nodes) * r + c] = s / (double)U;
        }
        min_pos[new_off + old_nodes] = (int32_t)n_old;
      } else {
        memcpy(&cent[(new_off + old_nodes) * r], &sc[sub_off * r], sizeof(double) * sub_nodes * r);
        for (int64_t k = 0; k < sub_nodes; ++k) min_pos[new_off + old_nodes + k] = sm[sub_off + k] + (int32_t)n_old;
        sub_off += sub_nodes;
      }
      old_off += old_nodes;
      new_off += old_nodes + sub_nodes;
    }
    memcpy(leaf_index, old_leaf, sizeof(int32_t) * n_old);
    for (int64_t i = 0; i < U; ++i) leaf_index[n_old + i] = sl[i] + (int32_t)n_old;
  }
  free(sc); free(sm); free(sl);
  return err;
}

/* ------------------------------------------------------------------------- */
/* Hierarchical search ([P1]: the query starts at the root, scores a few      */
/* candidate clusters per level and descends into a few branches; [P4]:       */
/* fixed search budget per level; a fixed number of original keys retrieved  */
/* from the chosen clusters).                                                  */
/* Score = inner product of the query latent with the centroid.  Level 0      */
/* candidates are all top nodes; level l candidates are all children of the   */
/* nodes kept at level l-1.  With q_pos given (causal), a node is a candidate */
/* only if its smallest member position is <= the query position.  Keep the   */
/* beam[l] best by (score desc, node id asc).  Output: the keys of the kept   */
/* leaves, leaf by leaf in that rank order, ascending positions inside a leaf,*/
/* padded with -1 to beam[L-1]*leaf_size.                                     */
/* beam_trace (optional): [levels, T, beam_max] kept node ids, -1 padded.     */
/* scored (optional): [T] number of nodes scored for the query.               */
/* ------------------------------------------------------------------------- */
typedef struct {
  double s;
  int64_t id;
} orc_cand;

static int orc_cand_cmp(const void *a, const void *b) {
  const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

int orc_select(const double *qlat, int64_t T, int32_t r, const int32_t *branching,
               int32_t levels, int32_t leaf_size, const double *centroids,
               const int32_t *min_pos, const int32_t *leaf_index, const int32_t *beam,
               const int32_t *q_pos, int32_t *idx_out, int32_t *beam_trace,
               int64_t *scored) {
  if (!qlat || !branching || !centroids || !min_pos || !leaf_index || !beam || !idx_out)
    return ORC_ERR_ARG;
  if (levels < 1 || levels > ORC_MAX_LEVELS) return ORC_ERR_ARG;
  int64_t nodes[ORC_MAX_LEVELS], cent_off[ORC_MAX_LEVELS], node_off[ORC_MAX_LEVELS];
  int64_t acc_nodes = 1, co = 0, no = 0;
  int32_t beam_max = 0;
  for (int32_t l = 0; l < levels; ++l) {
    acc_nodes *= branching[l];
    nodes[l] = acc_nodes;
    cent_off[l] = co;
    node_off[l] = no;
    co += acc_nodes * r;
    no += acc_nodes;
    int64_t avail = (l == 0) ? nodes[0] : (int64_t)beam[l - 1] * branching[l];
    if (beam[l] < 1 || beam[l] > avail) return ORC_ERR_SHAPE;
    if (beam[l] > beam_max) beam_max = beam[l];
  }
  const int64_t K_sel = (int64_t)beam[levels - 1] * leaf_size;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t t = 0; t < T; ++t) {
    int64_t max_cand = nodes[0];
    for (int32_t l = 1; l < levels; ++l)
      if ((int64_t)beam[l - 1] * branching[l] > max_cand) max_cand = (int64_t)beam[l - 1] * branching[l];
    orc_cand *cand = (orc_cand *)malloc(sizeof(orc_cand) * max_cand);
    int64_t *ids = (int64_t *)malloc(sizeof(int64_t) * max_cand);
    int64_t *kept = (int64_t *)malloc(sizeof(int64_t) * beam_max);
    int64_t n_ids = nodes[0], n_kept = 0, n_scored = 0;
    for (int64_t c = 0; c < n_ids; ++c) ids[c] = c;
    for (int32_t l = 0; l < levels; ++l) {
      int64_t n_c = 0;
      for (int64_t k = 0; k < n_ids; ++k) {
        int64_t id = ids[k];
        if (q_pos && min_pos[node_off[l] + id] > q_pos[t]) continue;
        const double *mu = &centroids[cent_off[l] + id * r];
        double s = 0.0;
        for (int32_t j = 0; j < r; ++j) s += qlat[t * r + j] * mu[j];
        if (isnan(s)) {
#pragma omp critical
          err = ORC_ERR_NONFINITE;
        }
        cand[n_c].s = s;
        cand[n_c].id = id;
        ++n_c;
      }
      n_scored += n_c;
      qsort(cand, (size_t)n_c, sizeof(orc_cand), orc_cand_cmp);
      n_kept = n_c < beam[l] ? n_c : beam[l];
      for (int64_t k = 0; k < n_kept; ++k) kept[k] = cand[k].id;
      if (beam_trace)
        for (int32_t k = 0; k < beam_max; ++k)
          beam_trace[((int64_t)l * T + t) * beam_max + k] = k < n_kept ? (int32_t)kept[k] : -1;
      if (l + 1 < levels) {
        n_ids = 0;
        for (int64_t k = 0; k < n_kept; ++k)
          for (int32_t j = 0; j < branching[l + 1]; ++j) ids[n_ids++] = kept[k] * branching[l + 1] + j;
      }
    }
    for (int64_t k = 0; k < beam[levels - 1]; ++k)
      for (int32_t q = 0; q < leaf_size; ++q)
        idx_out[t * K_sel + k * leaf_size + q] =
            k < n_kept ? leaf_index[kept[k] * leaf_size + q] : -1;
    if (scored) scored[t] = n_scored;
    free(cand);
    free(ids);
    free(kept);
  }
  return err;
}

/* ------------------------------------------------------------------------- */
/* Sparse attention over the selected keys ([P1 "The Accuracy-Efficiency     */
/* Dilemma": each query interacts with only k keys]; [P4]: the retrieved keys,*/
/* plus a dense range of recent positions).  One GQA group: the G query heads */
/* share the key index list.  Key j enters query t's softmax if it is listed  */
/* in idx[t] (>= 0) or lies in [tail_begin, tail_end), and, when causal, if   */
/* j <= q_pos[t].  logit = scale * <q, k_j>;  O = sum softmax * v_j;          */
/* LSE = log sum exp(logit).  No visible key: O = 0, LSE = -inf.              */
/* Q, O: [T, G, d];  K, V: [n_cap, d];  idx: [T, K_sel];  LSE: [T, G].        */
/* ------------------------------------------------------------------------- */
static int orc_cmp_i64(const void *x, const void *y) {
  const int64_t a = *(const int64_t *)x, b = *(const int64_t *)y;
  return (a > b) - (a < b);
}

/* Keys query t attends to: its index list, the dense tail range and, when n_sink
 * or window is positive, the first n_sink positions (sink tokens) and the window
 * positions q_pos - window + 1 .. q_pos (bdtechtalks.com, "Latent sparse
 * attention", section "How latent sparse attention works": the keys taken from
 * the chosen clusters are used together with a window of recent tokens and a few
 * initial sink tokens).  With sink or window the key set is a set: it is sorted and a
 * position listed twice counts once. */
static int64_t orc_visible_keys(int64_t t, const int32_t *idx, int32_t K_sel,
                                const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                                int64_t tail_end, int64_t n_cap, int32_t n_sink, int32_t window,
                                int64_t *out) {
  int64_t cnt = 0;
  for (int32_t k = 0; k < K_sel; ++k) {
    int64_t j = idx[t * K_sel + k];
    if (j < 0 || j >= n_cap) continue;
    if (causal && j > q_pos[t]) continue;
    out[cnt++] = j;
  }
  for (int64_t j = tail_begin; j < tail_end; ++j) {
    if (causal && j > q_pos[t]) continue;
    out[cnt++] = j;
  }
  if (n_sink == 0 && window == 0) return cnt;
  for (int64_t j = 0; j < n_sink && j < n_cap; ++j)
    if (j <= q_pos[t]) out[cnt++] = j;
  for (int64_t j = (int64_t)q_pos[t] - window + 1; j <= q_pos[t]; ++j)
    if (j >= 0 && j < n_cap) out[cnt++] = j;
  qsort(out, (size_t)cnt, sizeof(int64_t), orc_cmp_i64);
  int64_t u = 0;
  for (int64_t k = 0; k < cnt; ++k)
    if (u == 0 || out[k] != out[u - 1]) out[u++] = out[k];
  return u;
}

static int orc_attn_fwd_keys(const double *Q, int64_t T, int32_t G, int32_t d, const double *K,
                             const double *V, int64_t n_cap, const int32_t *idx, int32_t K_sel,
                             const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                             int64_t tail_end, int32_t n_sink, int32_t window, double scale,
                             double *O, double *LSE) {
  if (!Q || !K || !V || !O || !LSE || (K_sel > 0 && !idx) || (causal && !q_pos))
    return ORC_ERR_ARG;
  if (tail_begin < 0 || tail_end < tail_begin || tail_end > n_cap) return ORC_ERR_SHAPE;
  if (n_sink < 0 || window < 0 || ((n_sink > 0 || window > 0) && !causal)) return ORC_ERR_ARG;
  const int64_t max_keys = K_sel + (tail_end - tail_begin) + n_sink + window;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (max_keys + 1));
    double *logit = (double *)malloc(sizeof(double) * (max_keys + 1));
    int64_t cnt = orc_visible_keys(t, idx, K_sel, q_pos, causal, tail_begin, tail_end, n_cap, n_sink,
                                   window, keys);
    for (int32_t h = 0; h < G; ++h) {
      const double *q = &Q[(t * G + h) * d];
      double *o = &O[(t * G + h) * d];
      for (int32_t j = 0; j < d; ++j) o[j] = 0.0;
      if (cnt == 0) { LSE[t * G + h] = -INFINITY; continue; }
      double mx = -INFINITY;
      for (int64_t k = 0; k < cnt; ++k) {
        const double *kr = &K[keys[k] * d];
        double s = 0.0;
        for (int32_t j = 0; j < d; ++j) s += q[j] * kr[j];
        logit[k] = scale * s;
        if (logit[k] > mx) mx = logit[k];
      }
      double l = 0.0;
      for (int64_t k = 0; k < cnt; ++k) l += exp(logit[k] - mx);
      for (int64_t k = 0; k < cnt; ++k) {
        double p = exp(logit[k] - mx) / l;
        const double *vr = &V[keys[k] * d];
        for (int32_t j = 0; j < d; ++j) o[j] += p * vr[j];
      }
      LSE[t * G + h] = mx + log(l);
    }
    free(keys);
    free(logit);
  }
  return ORC_OK;
}

int orc_attn_fwd(const double *Q, int64_t T, int32_t G, int32_t d, const double *K,
                 const double *V, int64_t n_cap, const int32_t *idx, int32_t K_sel,
                 const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                 int64_t tail_end, double scale, double *O, double *LSE) {
  return orc_attn_fwd_keys(Q, T, G, d, K, V, n_cap, idx, K_sel, q_pos, causal, tail_begin, tail_end, 0, 0,
                           scale, O, LSE);
}

/* The same with the sink and recent-window keys added (causal). */
int orc_attn_fwd_sw(const double *Q, int64_t T, int32_t G, int32_t d, const double *K,
                    const double *V, int64_t n_cap, const int32_t *idx, int32_t K_sel,
                    const int32_t *q_pos, int64_t tail_begin, int64_t tail_end, int32_t n_sink,
                    int32_t window, double scale, double *O, double *LSE) {
  return orc_attn_fwd_keys(Q, T, G, d, K, V, n_cap, idx, K_sel, q_pos, 1, tail_begin, tail_end, n_sink,
                           window, scale, O, LSE);
}

/* Gradient of the same sparse attention for a fixed key selection, from the
 * upstream gradient dO (standard softmax-attention calculus restricted to the
 * visible (query, key) pairs):  P = softmax(logit);  dV_j += P_j dO;
 * dP_j = <dO, v_j>;  dS_j = P_j (dP_j - sum_i P_i dP_i);  dQ = scale sum_j dS_j k_j;
 * dK_j += scale dS_j q.  dK and dV ([n_cap, d]) are overwritten and sum over
 * the G heads of the group and over every query that sees key j. */
static int orc_attn_bwd_keys(const double *Q, int64_t T, int32_t G, int32_t d, const double *K,
                             const double *V, int64_t n_cap, const int32_t *idx, int32_t K_sel,
                             const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                             int64_t tail_end, int32_t n_sink, int32_t window, double scale,
                             const double *dO, double *dQ, double *dK, double *dV) {
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || (K_sel > 0 && !idx) || (causal && !q_pos))
    return ORC_ERR_ARG;
  if (tail_begin < 0 || tail_end < tail_begin || tail_end > n_cap) return ORC_ERR_SHAPE;
  if (n_sink < 0 || window < 0 || ((n_sink > 0 || window > 0) && !causal)) return ORC_ERR_ARG;
  memset(dK, 0, sizeof(double) * (size_t)(n_cap * d));
  memset(dV, 0, sizeof(double) * (size_t)(n_cap * d));
  const int64_t max_keys = K_sel + (tail_end - tail_begin) + n_sink + window;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (max_keys + 1));
    double *p = (double *)malloc(sizeof(double) * (max_keys + 1));
    double *dp = (double *)malloc(sizeof(double) * (max_keys + 1));
    int64_t cnt = orc_visible_keys(t, idx, K_sel, q_pos, causal, tail_begin, tail_end, n_cap, n_sink,
                                   window, keys);
    for (int32_t h = 0; h < G; ++h) {
      const double *q = &Q[(t * G + h) * d];
      const double *go = &dO[(t * G + h) * d];
      double *gq = &dQ[(t * G + h) * d];
      for (int32_t j = 0; j < d; ++j) gq[j] = 0.0;
      if (cnt == 0) continue;
      double mx = -INFINITY;
      for (int64_t k = 0; k < cnt; ++k) {
        const double *kr = &K[keys[k] * d];
        double s = 0.0;
        for (int32_t j = 0; j < d; ++j) s += q[j] * kr[j];
        p[k] = scale * s;
        if (p[k] > mx) mx = p[k];
      }
      double l = 0.0;
      for (int64_t k = 0; k < cnt; ++k) l += exp(p[k] - mx);
      double delta = 0.0;
      for (int64_t k = 0; k < cnt; ++k) {
        p[k] = exp(p[k] - mx) / l;
        const double *vr = &V[keys[k] * d];
        double s = 0.0;
        for (int32_t j = 0; j < d; ++j) s += go[j] * vr[j];
        dp[k] = s;
        delta += p[k] * s;
      }
      for (int64_t k = 0; k < cnt; ++k) {
        const double ds = p[k] * (dp[k] - delta);
        const double *kr = &K[keys[k] * d];
        double *gk = &dK[keys[k] * d];
        double *gv = &dV[keys[k] * d];
        for (int32_t j = 0; j < d; ++j) {
          gq[j] += scale * ds * kr[j];
#pragma omp atomic
          gk[j] += scale * ds * q[j];
#pragma omp atomic
          gv[j] += p[k] * go[j];
        }
      }
    }
    free(keys);
    free(p);
    free(dp);
  }
  return ORC_OK;
}

int orc_attn_bwd(const double *Q, int64_t T, int32_t G, int32_t d, const double *K,
                 const double *V, int64_t n_cap, const int32_t *idx, int32_t K_sel,
                 const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                 int64_t tail_end, double scale, const double *dO, double *dQ,
                 double *dK, double *dV) {
  return orc_attn_bwd_keys(Q, T, G, d, K, V, n_cap, idx, K_sel, q_pos, causal, tail_begin, tail_end, 0, 0,
                           scale, dO, dQ, dK, dV);
}

/* Backward of orc_attn_fwd_sw. */
int orc_attn_bwd_sw(const double *Q, int64_t T, int32_t G, int32_t d, const double *K,
                    const double *V, int64_t n_cap, const int32_t *idx, int32_t K_sel,
                    const int32_t *q_pos, int64_t tail_begin, int64_t tail_end, int32_t n_sink,
                    int32_t window, double scale, const double *dO, double *dQ, double *dK,
                    double *dV) {
  return orc_attn_bwd_keys(Q, T, G, d, K, V, n_cap, idx, K_sel, q_pos, 1, tail_begin, tail_end, n_sink,
                           window, scale, dO, dQ, dK, dV);
}
