/*
 * lsa.h -- C ABI of the B200 (sm_100a) library for the hot path of Latent Sparse
 * Attention (LSA) with a hierarchical latent-key index.
 *
 * What the path computes (pages about "Latent Sparse Attention"):
 *  - kongchang.com, "Latent Sparse Attention Breaks Through the Million-Token
 *    Context Bottleneck", section "How LSA Sidesteps Per-Key Scoring with
 *    Hierarchical Clustering": keys are projected into a low-dimensional latent
 *    space and grouped level by level into a tree whose root holds all keys;
 *    a query starts at the root, scores a few candidate clusters per level and
 *    descends into a few branches until it reaches leaf key subsets.
 *  - bdtechtalks.com, "Latent sparse attention", section "How latent sparse
 *    attention works": each cluster keeps a centroid next to references to its
 *    original keys; the query is compared with centroids, a fixed number of
 *    original keys is taken from the chosen clusters and attention runs over
 *    them (plus a window of recent tokens); hierarchical search keeps a fixed
 *    budget per level.
 *  - kongchang.com, section "The Accuracy-Efficiency Dilemma": sparse attention
 *    where each query interacts with only k keys.
 *
 * Conventions shared by every entry point
 *  - Device pointers are plain CUDA device addresses allocated by the caller;
 *    the library never allocates device memory.  Host pointers are marked "host".
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it; a call returns once its launches are
 *    queued.  Only lsa_status_check synchronises.
 *  - Every call validates its arguments on the host first and returns an
 *    lsa_status; on a validation error nothing is launched.  lsa_last_error()
 *    then holds a one-line explanation (thread-local).
 *  - `status` is a caller-allocated device int32 (zero it before use, e.g. with
 *    lsa_status_clear).  Kernels that detect a problem while running (a NaN score,
 *    a device loop that hit its round cap) write a nonzero lsa_status code there;
 *    the first code written wins.  Read it with lsa_status_check.
 *  - dtype: LSA_F32 or LSA_BF16; Q, K, V, W, O and dO of one call share it.
 *    Accumulation is fp32 throughout; gradients are fp32.
 *  - No call aborts, traps or throws.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LSA_VERSION 1
#define LSA_MAX_LEVELS 8
#define LSA_MAX_BRANCHING 16       /* children per node on a level the k-means build splits */
#define LSA_MAX_TOP_BRANCHING 512  /* top-level nodes a tree can reach through lsa_tree_append */
#define LSA_MAX_BEAM 32

typedef enum lsa_status {
  LSA_OK = 0,
  LSA_ERR_INVALID_ARG = 1, /* null pointer, unknown dtype, bad scalar            */
  LSA_ERR_SHAPE = 2,       /* sizes inconsistent or outside supported limits     */
  LSA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed               */
  LSA_ERR_TIMEOUT = 4,     /* a device loop or barrier hit its iteration cap     */
  LSA_ERR_NONFINITE = 5,   /* NaN met where an ordering decision was needed      */
  LSA_ERR_WORKSPACE = 6    /* workspace missing or smaller than required         */
} lsa_status;

typedef enum lsa_dtype { LSA_F32 = 0, LSA_BF16 = 1 } lsa_dtype;

/* Geometry and memory layout of a tree (one tree per KV head, all heads in one
 * buffer).  Filled by lsa_tree_describe; treat as read-only afterwards.
 * Layout of the tree buffer (byte offsets, every region 256-byte aligned):
 *   centroids of level l : float [n_heads][nodes[l]][r]   at off_centroids[l]
 *   min_pos of level l   : int32 [n_heads][nodes[l]]      at off_min_pos[l]
 *                          (smallest key position under the node)
 *   leaf_index           : int32 [n_heads][n_tree]        at off_leaf_index
 *                          (keys of leaf 0 in ascending position, then leaf 1, ...)
 * Node ids: level l has nodes[l] = b_0*...*b_l nodes; the children of node p of
 * level l-1 are p*b_l + j, j < b_l.  Leaves are the nodes of the last level and
 * each holds exactly leaf_size keys. */
typedef struct lsa_tree_desc {
  int32_t n_heads;
  int32_t r;
  int32_t levels;
  int32_t leaf_size;
  int64_t n_tree;                         /* = leaf_size * prod(branching)     */
  int32_t branching[LSA_MAX_LEVELS];
  int64_t nodes[LSA_MAX_LEVELS];
  uint64_t off_centroids[LSA_MAX_LEVELS];
  uint64_t off_min_pos[LSA_MAX_LEVELS];
  uint64_t off_leaf_index;
  uint64_t bytes;                         /* size of the tree buffer           */
} lsa_tree_desc;

/* Library version (LSA_VERSION). */
int lsa_version(void);

/* Static text for a status code; never NULL. */
const char *lsa_strerror(int status);

/* Detail of the last error returned on this thread ("" if none). */
const char *lsa_last_error(void);

/* Host only.  Fills *out for n_heads trees with latent dim r, `levels` levels of
 * fan-out branching[0..levels) (root to leaves; branching[0] in [2, 512], the others
 * in [2, 16]; lsa_build_tree itself needs branching[0] <= 16 too, wider top levels
 * come from lsa_tree_append) and leaves of leaf_size keys.  Limits: 1 <= levels <= 8, r in {16, 32, 64}, leaf_size in [8, 4096],
 * n_tree <= 2^30 and n_heads * n_tree < 2^31.
 * Returns LSA_ERR_SHAPE / LSA_ERR_INVALID_ARG on violations. */
int lsa_tree_describe(int32_t n_heads, int32_t r, const int32_t *branching /* host */,
                      int32_t levels, int32_t leaf_size, lsa_tree_desc *out /* host */);

/* Host only.  Device workspace bytes lsa_build_tree needs for keys of width d. */
int lsa_build_workspace_bytes(const lsa_tree_desc *tree, int32_t d, size_t *bytes /* host */);

/* Build the index (kongchang.com, "How LSA Sidesteps Per-Key Scoring with
 * Hierarchical Clustering": latent projection, then clustering level by level
 * from the root "similar to hierarchical k-means").
 *  K        : [n_heads][n_cap][d] keys; positions [0, n_tree) are indexed, the
 *             rest (decode appends) are left for the dense tail.
 *  W        : [n_heads][d][r] latent projection (same dtype as K).
 *  iters    : k-means rounds per level (>= 1).  Each round assigns every key of a
 *             parent node to one of its b_l children with exactly
 *             (parent size / b_l) keys per child -- the unique stable assignment
 *             under the pair order (squared distance asc, key position asc,
 *             child asc) -- then moves each child centroid to its members' mean.
 *             Round 1 starts from the members with the b_l smallest SplitMix64
 *             hashes of (seed, level, position).  Stored centroids are the means
 *             of the last round's assignment.
 *  trace    : optional (NULL) int32 [levels][iters][n_heads][n_tree]: node id of
 *             every key (indexed by position) after each round's assignment.
 *  tree_mem : tree->bytes of device memory, written completely (alignment gaps are zeroed).
 * Limits: d in {64, 128}; n_cap >= n_tree.  Writes LSA_ERR_TIMEOUT to *status if
 * an assignment needs more than 4096 proposal rounds (never seen in practice),
 * LSA_ERR_NONFINITE if a distance is NaN. */
int lsa_build_tree(const lsa_tree_desc *tree, void *tree_mem, const void *K, int64_t n_cap,
                   int32_t d, int32_t dtype, const void *W, int32_t iters, uint64_t seed,
                   void *workspace, size_t workspace_bytes, int32_t *trace, int32_t *status,
                   void *stream);

/* lsa_build_tree over pooled keys (bdtechtalks.com, "Latent sparse attention",
 * section "How latent sparse attention works": consecutive keys are pooled into
 * smaller representations, then clustered; each cluster keeps references to the
 * original keys).
 *  pool : keys per block, >= 1 and dividing tree->leaf_size.  Block j of a head
 *         holds keys [j*pool, (j+1)*pool) and is represented by the mean of their
 *         latent rows (fp32, summed in position order).  The k-means levels of
 *         lsa_build_tree run on the n_tree/pool blocks (a block's position is j)
 *         with leaf_size/pool blocks per leaf.
 * Output layout is that of lsa_build_tree: leaf_index lists, for the blocks of a
 * leaf in ascending order, their keys j*pool .. j*pool + pool - 1 (so every leaf
 * still holds leaf_size keys in ascending position), min_pos is a key position,
 * and every centroid is the mean of the latent rows of the keys under the node.
 *  trace : optional int32 [levels][iters][n_heads][n_tree/pool], node id of every
 *          block (indexed by block) after each round.
 * pool = 1 is lsa_build_tree.  Workspace: lsa_build_workspace_bytes of the same
 * tree.  Other arguments, limits and errors as lsa_build_tree; LSA_ERR_SHAPE if
 * pool does not divide leaf_size. */
int lsa_build_tree_pooled(const lsa_tree_desc *tree, void *tree_mem, const void *K, int64_t n_cap,
                          int32_t d, int32_t dtype, const void *W, int32_t pool, int32_t iters,
                          uint64_t seed, void *workspace, size_t workspace_bytes, int32_t *trace,
                          int32_t *status, void *stream);

/* Host only.  Device workspace bytes lsa_tree_append needs for keys of width d
 * (the subtree's buffer and its build workspace).  LSA_ERR_SHAPE if levels < 2. */
int lsa_tree_append_workspace_bytes(const lsa_tree_desc *tree, int32_t d, size_t *bytes /* host */);

/* Update of an index on append (kongchang.com, "How LSA Sidesteps Per-Key Scoring
 * with Hierarchical Clustering": the tree can be precomputed and then updated).
 * Every node of a level has the same fan-out, so only the top level can grow: once
 * U = leaf_size * branching[1] * ... * branching[levels-1] keys have been appended
 * after the tree->n_tree indexed ones, they get a subtree of their own, attached as
 * top-level node branching[0].
 *  tree, tree_mem   : the current index (read only; levels >= 2).
 *  grown            : lsa_tree_describe of the same heads, r, levels and leaf_size with
 *                     branching[0] + 1 (so grown->n_tree = tree->n_tree + U).
 *  grown_mem        : grown->bytes of device memory (not tree_mem), written completely.
 *  K, n_cap, d, dtype, W : as lsa_build_tree; keys [tree->n_tree, grown->n_tree) of
 *                     every head are the appended block (n_cap >= grown->n_tree).
 * The subtree is lsa_build_tree run on the U appended keys alone with branching
 * branching[1..levels) (same iters and seed; positions, for the seeded start and the
 * pair order, counted from the block's first key); its node ids follow the old ones
 * on every level, its min_pos and leaf_index are shifted by tree->n_tree, and the new
 * top node's centroid is the mean of its children's (= of the U keys' latent rows).
 * Every old node keeps its id, centroid, min_pos and keys.
 *  trace : optional int32 [levels-1][iters][n_heads][U] of the subtree's build.
 * Errors as lsa_build_tree; LSA_ERR_SHAPE if grown does not match tree. */
int lsa_tree_append(const lsa_tree_desc *tree, const void *tree_mem, const lsa_tree_desc *grown,
                    void *grown_mem, const void *K, int64_t n_cap, int32_t d, int32_t dtype,
                    const void *W, int32_t iters, uint64_t seed, void *workspace,
                    size_t workspace_bytes, int32_t *trace, int32_t *status, void *stream);

/* Hierarchical search (kongchang.com, "How LSA Sidesteps ..."; bdtechtalks.com,
 * "How latent sparse attention works": fixed budget per level, a fixed number
 * of original keys from the chosen clusters).
 *  Q       : [T][Hq][d] queries; Hq = G * n_heads, query head h belongs to group
 *            h / G and the G heads of a group share one selection.
 *  W       : the [n_heads][d][r] projection the tree was built with.
 *  beam    : host int32[levels]; beam[0] <= nodes[0], beam[l] <= beam[l-1]*b_l,
 *            every beam[l] in [1, 32].
 *  q_pos   : NULL (non-causal) or device int32[T] query positions; a node is a
 *            candidate only if its min_pos <= q_pos.
 * Per (group g, query t): q = (mean of the group's G query rows) . W[g] (fp32);
 * level-0 candidates are all top nodes, level-l candidates the children of the
 * nodes kept at level l-1; score = <q, centroid> (fp32); keep the beam[l] best by
 * (score desc, node id asc).
 *  idx_out : optional [n_heads][T][beam[levels-1] * leaf_size] int32 key positions
 *            of the kept leaves, leaf by leaf in rank order, ascending inside a
 *            leaf, -1 where fewer leaves were eligible.
 *  leaves_out: optional [n_heads][T][beam[levels-1]] int32 kept leaf ids in rank
 *            order, -1 padded (the input of lsa_tree_attn).  At least one of
 *            idx_out and leaves_out must be given.
 *  qlat_out: optional [T][n_heads][r] float query latents.
 *  beam_out: optional [levels][n_heads][T][max beam] int32 kept node ids per level
 *            in rank order, -1 padded.
 * Writes LSA_ERR_NONFINITE to *status if a score is NaN. */
int lsa_select(const lsa_tree_desc *tree, const void *tree_mem, const void *Q, int32_t T,
               int32_t Hq, int32_t d, int32_t dtype, const void *W, const int32_t *beam,
               const int32_t *q_pos, int32_t *idx_out, int32_t *leaves_out, float *qlat_out,
               int32_t *beam_out, int32_t *status, void *stream);

/* The same hierarchical search as lsa_select, scheduled for large query batches
 * (prefill, training): after the top level, every level scores the children of a
 * kept node for all the walks that kept it together (the (query, group, parent)
 * triples are grouped by parent first), then ranks each walk's candidates.  The
 * scores are the same fp32 expressions, so every output (idx_out, leaves_out,
 * qlat_out, beam_out, status) equals lsa_select's bit for bit.  Arguments as
 * lsa_select, plus:
 *  workspace: device memory of lsa_select_batched_workspace_bytes(tree, T, beam)
 *             bytes (NULL allowed when that is 0); contents need no initialisation
 *             and are scratch afterwards.  Not shared between concurrent calls.
 * T must be <= 2^26.  Errors as lsa_select; LSA_ERR_WORKSPACE if the workspace is
 * missing or too small.  With one level it runs lsa_select's kernel. */
int lsa_select_batched_workspace_bytes(const lsa_tree_desc *tree, int32_t T, const int32_t *beam,
                                       size_t *bytes /* host */);
int lsa_select_batched(const lsa_tree_desc *tree, const void *tree_mem, const void *Q, int32_t T,
                       int32_t Hq, int32_t d, int32_t dtype, const void *W, const int32_t *beam,
                       const int32_t *q_pos, int32_t *idx_out, int32_t *leaves_out,
                       float *qlat_out, int32_t *beam_out, void *workspace,
                       size_t workspace_bytes, int32_t *status, void *stream);

/* Flat search (bdtechtalks.com, "Latent sparse attention", section "How latent
 * sparse attention works": the first of the two search strategies compares the
 * query with all cluster centroids).  Arguments and outputs as lsa_select with a
 * single budget: per (group g, query t) every leaf of the last level is scored,
 * score = <q, leaf centroid> (fp32), a leaf is a candidate only if its min_pos <=
 * q_pos[t] (when q_pos is given), and the n_leaves best by (score desc, leaf id asc)
 * are kept, in that order.  idx_out [n_heads][T][n_leaves * leaf_size] and
 * leaves_out [n_heads][T][n_leaves] as in lsa_select; qlat_out optional.
 * n_leaves in [1, min(32, number of leaves)].  Quadratic in the context: every
 * query reads every leaf centroid of its group. */
int lsa_select_flat(const lsa_tree_desc *tree, const void *tree_mem, const void *Q, int32_t T,
                    int32_t Hq, int32_t d, int32_t dtype, const void *W, int32_t n_leaves,
                    const int32_t *q_pos, int32_t *idx_out, int32_t *leaves_out, float *qlat_out,
                    int32_t *status, void *stream);

/* Host only.  Workspace bytes lsa_sparse_attn needs for these sizes (0 when the
 * call runs without key splitting). */
int lsa_attn_workspace_bytes(int32_t T, int32_t Hq, int32_t n_heads, int32_t d, int32_t K_sel,
                             int64_t tail_len, size_t *bytes);

/* Sparse attention forward (kongchang.com, "The Accuracy-Efficiency Dilemma";
 * bdtechtalks.com, "How latent sparse attention works").
 *  Q [T][Hq][d];  K, V [n_heads][n_cap][d];  idx [n_heads][T][K_sel] key positions
 *  (-1 = none) shared by the G query heads of a group; the dense range
 *  [tail_begin, tail_end) of positions is attended by every query as well.
 *  causal: key j is visible to query t only if j <= q_pos[t] (q_pos device
 *  int32[T], required when causal).  logits = scale * <q, k>.
 *  O   [T][Hq][d] (dtype of Q) = softmax-weighted sum of V rows;
 *  LSE [T][Hq] float = natural log of the softmax denominator (-inf and O = 0 when
 *  a query sees no key).  Indices must lie in [0, n_cap) or be -1, and must not
 *  repeat within a row or fall inside the tail range. */
int lsa_sparse_attn(const void *Q, int32_t T, int32_t Hq, const void *K, const void *V,
                    int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype, const int32_t *idx,
                    int32_t K_sel, const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                    int64_t tail_end, float scale, void *O, float *LSE, void *workspace,
                    size_t workspace_bytes, int32_t *status, void *stream);

/* Largest sink and window sizes lsa_sparse_attn_sw accepts. */
#define LSA_MAX_SINK_WINDOW 65536

/* Host only.  Workspace bytes lsa_sparse_attn_sw needs: the extended key lists
 * ([n_heads][T][K_sel + n_sink + window] int32) and the split partials of the
 * attention over them. */
int lsa_sparse_attn_sw_workspace_bytes(int32_t T, int32_t Hq, int32_t n_heads, int32_t d, int32_t K_sel,
                                       int64_t tail_len, int32_t n_sink, int32_t window, size_t *bytes);

/* Sparse attention with sink and recent-window keys (bdtechtalks.com, "Latent
 * sparse attention", section "How latent sparse attention works": the keys taken
 * from the chosen clusters are attended together with a window of recent tokens
 * and a few initial sink tokens).  Arguments and outputs as lsa_sparse_attn with causal = 1
 * (q_pos required), plus
 *  n_sink : positions [0, n_sink) join every query's keys (where <= q_pos);
 *  window : positions [q_pos[t] - window + 1, q_pos[t]] join query t's keys.
 * Query t attends to the union of its index list, the tail range, the sink and
 * its window, each key once: an index-list entry that also lies in the tail, the
 * sink or the window is not counted twice.  n_sink, window in
 * [0, LSA_MAX_SINK_WINDOW], n_sink <= n_cap.  Key lists are extended by a kernel
 * into the workspace, then the key-list attention runs. */
int lsa_sparse_attn_sw(const void *Q, int32_t T, int32_t Hq, const void *K, const void *V,
                       int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype, const int32_t *idx,
                       int32_t K_sel, const int32_t *q_pos, int32_t n_sink, int32_t window,
                       int64_t tail_begin, int64_t tail_end, float scale, void *O, float *LSE,
                       void *workspace, size_t workspace_bytes, int32_t *status, void *stream);

/* Backward of lsa_sparse_attn_sw (conventions of lsa_sparse_attn_bwd).  Needs
 * workspace for the extended key lists: n_heads * T * (K_sel + n_sink + window)
 * int32, rounded up to 256 bytes. */
int lsa_sparse_attn_sw_bwd(const void *Q, int32_t T, int32_t Hq, const void *K, const void *V,
                           int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype, const void *O,
                           const float *LSE, const void *dO, const int32_t *idx, int32_t K_sel,
                           const int32_t *q_pos, int32_t n_sink, int32_t window, int64_t tail_begin,
                           int64_t tail_end, float scale, float *dQ, float *dK, float *dV,
                           void *workspace, size_t workspace_bytes, int32_t *status, void *stream);

/* Host only.  Workspace bytes lsa_tree_attn needs. */
int lsa_tree_attn_workspace_bytes(const lsa_tree_desc *tree, int32_t T, int32_t Hq, int32_t d,
                                  int32_t dtype, int32_t n_leaves, size_t *bytes);

/* Sparse attention over tree-structured selections (the same sources as
 * lsa_sparse_attn): query t of group g attends to the keys of the leaves
 * leaves[g][t][0..n_leaves) (-1 = none) of the index built by lsa_build_tree,
 * i.e. exactly lsa_sparse_attn with the expanded key lists and no tail.
 * Computed leaf by leaf: every selected leaf's K/V rows are read once per pass
 * and shared by all (query, head) rows that chose the leaf, with the products on
 * the tensor cores (bf16, d = 128, leaf size 64; other shapes run the generic
 * kernels on the expanded lists).  Outputs as lsa_sparse_attn.  While
 * T * Hq * n_leaves * d * 2 bytes stay within 24 GiB, every (row, leaf) pair
 * stores its leaf maximum, exp-sum and unnormalised output in the workspace and
 * a row's leaves are merged in a fixed order (results are reproducible bit for
 * bit); larger calls take a second pass over the leaves instead and accumulate
 * the outputs with fp32 atomic adds, whose order is not fixed, so results may
 * differ from run to run in the last bits.  n_leaves in [1, 32]. */
int lsa_tree_attn(const lsa_tree_desc *tree, const void *tree_mem, const void *Q, int32_t T,
                  int32_t Hq, const void *K, const void *V, int64_t n_cap, int32_t d,
                  int32_t dtype, const int32_t *leaves, int32_t n_leaves, const int32_t *q_pos,
                  int32_t causal, float scale, void *O, float *LSE, void *workspace,
                  size_t workspace_bytes, int32_t *status, void *stream);

/* Host only.  Workspace bytes lsa_tree_attn_sw needs. */
int lsa_tree_attn_sw_workspace_bytes(const lsa_tree_desc *tree, int32_t T, int32_t Hq, int32_t d,
                                     int32_t dtype, int32_t n_leaves, int32_t n_sink, int32_t window,
                                     size_t *bytes);

/* lsa_tree_attn (causal, q_pos required) with sink and recent-window keys as in
 * lsa_sparse_attn_sw: query t attends to the keys of its leaves, positions
 * [0, n_sink) and [q_pos[t] - window + 1, q_pos[t]], each key once.  On the leaf-by-
 * leaf path a leaf key inside the sink or the window is left out (a leaf lists its
 * keys in position order, so the kept keys are one index range) and the sink and
 * window keys are attended as one more partial, tile by tile on the tensor cores
 * (128 (query, head) rows of a KV group against the 64-position key blocks that any
 * of them needs), merged in the combine; other shapes run the key-list attention on
 * the expanded and extended lists.  n_sink, window in [0, LSA_MAX_SINK_WINDOW]. */
int lsa_tree_attn_sw(const lsa_tree_desc *tree, const void *tree_mem, const void *Q, int32_t T,
                     int32_t Hq, const void *K, const void *V, int64_t n_cap, int32_t d,
                     int32_t dtype, const int32_t *leaves, int32_t n_leaves, const int32_t *q_pos,
                     int32_t n_sink, int32_t window, float scale, void *O, float *LSE, void *workspace,
                     size_t workspace_bytes, int32_t *status, void *stream);

/* Host only.  Workspace bytes lsa_tree_attn_bwd needs. */
int lsa_tree_attn_bwd_workspace_bytes(const lsa_tree_desc *tree, int32_t T, int32_t Hq, int32_t d,
                                      int32_t dtype, int32_t n_leaves, size_t *bytes);

/* Backward of lsa_tree_attn for a fixed selection (the gradient of the same
 * attention as lsa_sparse_attn_bwd, with the same outputs and conventions):
 * computed leaf by leaf on the tensor cores, P and dS = P * (dP - rowsum(dO * O))
 * rounded to bf16 for the products; each leaf's dK and dV rows are written once
 * (a leaf owns its keys), dQ accumulates with fp32 red-adds (summation order not
 * fixed).  dQ, dK, dV are overwritten. */
int lsa_tree_attn_bwd(const lsa_tree_desc *tree, const void *tree_mem, const void *Q, int32_t T,
                      int32_t Hq, const void *K, const void *V, int64_t n_cap, int32_t d,
                      int32_t dtype, const void *O, const float *LSE, const void *dO,
                      const int32_t *leaves, int32_t n_leaves, const int32_t *q_pos, int32_t causal,
                      float scale, float *dQ, float *dK, float *dV, void *workspace,
                      size_t workspace_bytes, int32_t *status, void *stream);

/* Backward of lsa_sparse_attn for a fixed selection (same arguments), given the
 * forward's O and LSE and the upstream gradient dO ([T][Hq][d], dtype of Q).
 * Outputs (float): dQ [T][Hq][d]; dK, dV [n_heads][n_cap][d], overwritten (zero
 * where no query sees the key); dK/dV sum over the G heads of a group and over
 * every query that sees the key.  Needs no workspace. */
int lsa_sparse_attn_bwd(const void *Q, int32_t T, int32_t Hq, const void *K, const void *V,
                        int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype, const void *O,
                        const float *LSE, const void *dO, const int32_t *idx, int32_t K_sel,
                        const int32_t *q_pos, int32_t causal, int64_t tail_begin,
                        int64_t tail_end, float scale, float *dQ, float *dK, float *dV,
                        int32_t *status, void *stream);

/* Same computation and arguments as lsa_sparse_attn, for callers that cannot
 * allocate device memory: a plugin whose host framework passes it only its input
 * and output buffers, or a decode loop that must not call cudaMalloc (which can
 * synchronise the whole device) once serving has started.  The pages have no
 * counterpart of this call; it only changes where the split partials live.
 *  - Nothing is allocated: when the keys of a query are split over several CTAs
 *    (few queries, long key lists: decode), the partial results go to a built-in
 *    device array of LSA_NOALLOC_SCRATCH_BYTES (4 MiB).  Every GPU that loads the
 *    library holds that array until the process exits.  A call needing more
 *    (lsa_attn_workspace_bytes reports the need) returns LSA_ERR_WORKSPACE with
 *    nothing launched.  At d = 128 a call needs at most about G * 0.62 MB (G =
 *    query heads per KV head), so every call with G <= 4 fits, e.g. any number of
 *    decode tokens with 32 query heads over 8 KV heads; G = 8 can need up to about
 *    4.9 MB.  Calls that need no split use no scratch at all.
 *  - The first call on a device looks up that device's address of the array (once
 *    per device, with the device current); make that first call before any stream
 *    capture.  The address is kept for the life of the process: after
 *    cudaDeviceReset (or anything else that destroys and recreates the device's
 *    primary context) the kept address is stale, so do not call this entry point
 *    on that device again in the same process.
 *  - All calls share the one array and it keeps the last call's contents; every
 *    call overwrites the partials it reads, so nothing needs clearing, but calls
 *    that overlap on the GPU (other streams, other host threads) race on it. */
#define LSA_NOALLOC_SCRATCH_BYTES (4u << 20)
int lsa_sparse_attn_noalloc(const void *Q, int32_t T, int32_t Hq, const void *K, const void *V,
                            int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype,
                            const int32_t *idx, int32_t K_sel, const int32_t *q_pos, int32_t causal,
                            int64_t tail_begin, int64_t tail_end, float scale, void *O, float *LSE,
                            int32_t *status, void *stream);

/* One balanced k-means assignment step of the build (kongchang.com, "How LSA
 * Sidesteps Per-Key Scoring with Hierarchical Clustering": the tree is built like
 * hierarchical k-means), exposed on its own.  Segment s holds the m latent rows
 * Z[s*m .. s*m + m) (fp32, [nseg*m][r], device) and the b centroids
 * mu[s*b .. s*b + b) ([nseg*b][r], device).  Each row goes to one of its segment's
 * centroids, exactly m/b rows per centroid, by the unique stable assignment under
 * the order (squared distance asc, row index in the segment asc, centroid asc).
 * choice [nseg*m] uint8 (device) receives the centroid index of every row.
 * Rows are identified by their index inside the segment.
 *  b in [2, 16] dividing m; r in {16, 32, 64}; nseg * m < 2^31.
 *  max_rounds: cap on the proposal rounds of the parallel deferred acceptance
 *  (0 = the cap the build uses, 4096).  A segment whose assignment is still
 *  changing when the cap is reached leaves choice balanced or not and sets
 *  LSA_ERR_TIMEOUT in *status; the kernels return normally either way.  NaN
 *  distances set LSA_ERR_NONFINITE.
 *  workspace: lsa_balanced_assign_workspace_bytes(nseg, m, b) bytes (device). */
int lsa_balanced_assign_workspace_bytes(int64_t nseg, int64_t m, int32_t b, size_t *bytes);
int lsa_balanced_assign(const float *Z, const float *mu, int64_t nseg, int64_t m, int32_t b, int32_t r,
                        int32_t max_rounds, uint8_t *choice, void *workspace, size_t workspace_bytes,
                        int32_t *status, void *stream);

/* Latent projection of the keys (kongchang.com, "Latent Sparse Attention Breaks
 * Through the Million-Token Context Bottleneck", section "How LSA Sidesteps
 * Per-Key Scoring with Hierarchical Clustering": keys are first mapped into a
 * low-dimensional latent space).  The first step of lsa_build_tree, exposed on
 * its own:  Z[h][i][c] = sum_j K[h][i][j] * W[h][j][c]  for i < n.
 *  K : [n_heads][n_cap][d] (dtype), device;  W : [n_heads][d][r] (dtype), device;
 *  Z : [n_heads][n][r] fp32, device, overwritten (may be NULL when n = 0).
 *  d in {64, 128}, r in {16, 32, 64}, 0 <= n <= n_cap.  bf16 inputs run on the
 *  tensor cores (exact products, fp32 sums); fp32 inputs use fp32 FMAs.  An MMA
 *  that does not complete within a second sets LSA_ERR_TIMEOUT in *status (may be
 *  NULL).  Needs no workspace. */
int lsa_project_keys(const void *K, int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype,
                     const void *W, int32_t r, int64_t n, float *Z, int32_t *status, void *stream);

/* Decode append (bdtechtalks.com, "How latent sparse attention works": the
 * recent tokens join the attended keys): write the new key row and value row of
 * every KV head at position `pos` of the caches K, V [n_heads][n_cap][d].
 * K_rows, V_rows: [n_heads][d] in the caches' dtype.  One kernel launch. */
int lsa_kv_append(void *K, void *V, int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype,
                  int64_t pos, const void *K_rows, const void *V_rows, void *stream);

/* One decode step of a single request (kongchang.com, "The Accuracy-Efficiency
 * Dilemma of Sparse Attention": decode is memory-bound and latency-sensitive;
 * bdtechtalks.com, "How latent sparse attention works": the query is compared
 * with the centroids, a fixed number of keys is taken from the chosen clusters,
 * and the recent tokens join them).  For the token at position `pos` it
 *   1. appends K_row, V_row ([n_heads][d], device) at `pos` of the caches K, V
 *      ([n_heads][n_cap][d]) when they are non-NULL (both or neither);
 *   2. walks the index with the group query of Q ([1][Hq][d]), as lsa_select with
 *      q_pos = pos (every indexed key precedes the token), keeping beam[levels-1]
 *      leaves per KV group;
 *   3. attends to the keys of the kept leaves and to the tail [tail_begin, pos]:
 *      O [1][Hq][d] (dtype), LSE [Hq] fp32, as lsa_sparse_attn with causal = 1.
 * Two kernel launches; no host synchronisation.  Requires n_tree - 1 <= pos <
 * n_cap and n_tree <= tail_begin <= pos + 1.  leaves_out (optional, device,
 * [n_heads][beam[levels-1]]) receives the kept leaf ids (-1 pads).
 * The kept leaves' keys and the tail are attended in chunks of 64 keys, one CTA
 * each; one call handles up to 17408 / (8 G) chunks at d = 128 bf16 (544 at G = 4)
 * and returns LSA_ERR_SHAPE beyond that.
 * workspace: lsa_decode_step_workspace_bytes(tree, Hq, d, beam, tail_len_max)
 * bytes with tail_len_max >= pos + 1 - tail_begin; calls that share a workspace
 * must not overlap on the GPU. */
int lsa_decode_step_workspace_bytes(const lsa_tree_desc *tree, int32_t Hq, int32_t d, const int32_t *beam,
                                    int64_t tail_len_max, size_t *bytes);
int lsa_decode_step(const lsa_tree_desc *tree, const void *tree_mem, const void *W, const int32_t *beam,
                    void *K, void *V, int64_t n_cap, int32_t d, int32_t dtype, const void *Q, int32_t Hq,
                    const void *K_row, const void *V_row, int64_t pos, int64_t tail_begin, float scale,
                    void *O, float *LSE, int32_t *leaves_out, void *workspace, size_t workspace_bytes,
                    int32_t *status, void *stream);

/* Zero the device status word on `stream`. */
int lsa_status_clear(int32_t *status, void *stream);

/* Synchronise `stream`, copy the device status word to *host_out and return
 * LSA_OK, or LSA_ERR_CUDA if the stream reported an error. */
int lsa_status_check(const int32_t *status, void *stream, int32_t *host_out /* host */);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
