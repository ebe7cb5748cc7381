// api.cu -- C ABI of the LSA library: argument validation, workspace layout and
// dispatch to the kernels.  Every check runs on the host before any launch; no
// call aborts, traps or throws.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = '\0';
  return LSA_OK;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(LSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

bool valid_dtype(int dt) { return dt == LSA_F32 || dt == LSA_BF16; }

// Recompute a descriptor from its defining fields and compare, so a corrupted or
// hand-made struct is rejected.
int check_desc(const lsa_tree_desc* t) {
  if (!t) return fail(LSA_ERR_INVALID_ARG, "tree descriptor is NULL");
  lsa_tree_desc ref;
  int rc = lsa_tree_describe(t->n_heads, t->r, t->branching, t->levels, t->leaf_size, &ref);
  if (rc != LSA_OK) return rc;
  if (memcmp(&ref, t, sizeof(ref)) != 0)
    return fail(LSA_ERR_INVALID_ARG, "tree descriptor was not produced by lsa_tree_describe");
  return LSA_OK;
}

}  // namespace

namespace lsa {

// Record a message for lsa_last_error() on this thread and return `code`.
int report_error(int code, const char* msg) { return fail(code, "%s", msg); }

size_t build_workspace_layout(const lsa_tree_desc& t, char* base, BuildPlan* P) {
  const int64_t H = t.n_heads, n = t.n_tree, R = t.r, nslots = H * n;
  int bmax = 0;
  int64_t max_tiles = 0, max_partial = 0, max_grid_segc = 0, S = 1;
  for (int l = 0; l < t.levels; ++l) {
    const int b = t.branching[l];
    bmax = b > bmax ? b : bmax;
    const int64_t m = n / S, cap = m / b, nseg = H * S;
    const int64_t tiles = nseg * ceil_div(m, kTile);
    max_tiles = tiles > max_tiles ? tiles : max_tiles;
    const int64_t cpn = ceil_div(cap, kMeanChunk);
    const int64_t part = cpn > 1 ? nseg * b * cpn * R : 0;
    max_partial = part > max_partial ? part : max_partial;
    if (m > kCtaMaxSeg) max_grid_segc = nseg * b > max_grid_segc ? nseg * b : max_grid_segc;
    S *= b;
  }
  const int64_t max_nodes = H * t.nodes[t.levels - 1];
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    uint64_t at = off;
    off = align256(off + (bytes ? bytes : 1));
    return base ? base + at : nullptr;
  };
  char* p;
  p = take(nslots * R * 4);              if (P) P->Za = reinterpret_cast<float*>(p);
  p = take(nslots * R * 4);              if (P) P->Zb = reinterpret_cast<float*>(p);
  p = take(nslots * 4);                  if (P) P->pa = reinterpret_cast<int32_t*>(p);
  p = take(nslots * 4);                  if (P) P->pb = reinterpret_cast<int32_t*>(p);
  p = take(nslots * 4);                  if (P) P->order = reinterpret_cast<int32_t*>(p);
  p = take(nslots * bmax * 4);           if (P) P->D = reinterpret_cast<float*>(p);
  p = take(nslots * 8);                  if (P) P->pref = reinterpret_cast<uint64_t*>(p);
  p = take(nslots * 4);                  if (P) P->dbits = reinterpret_cast<uint32_t*>(p);
  p = take(nslots);                      if (P) P->choice = reinterpret_cast<uint8_t*>(p);
  p = take(nslots);                      if (P) P->ptr = reinterpret_cast<uint8_t*>(p);
  p = take(max_nodes * R * 4);           if (P) P->mu = reinterpret_cast<float*>(p);
  p = take(max_tiles * bmax * 4);        if (P) P->tcnt = reinterpret_cast<int32_t*>(p);
  p = take(max_tiles * bmax * 8);        if (P) P->toff = reinterpret_cast<int64_t*>(p);
  p = take(max_tiles * bmax * 8);        if (P) P->cand_h = reinterpret_cast<uint64_t*>(p);
  p = take(max_tiles * bmax * 8);        if (P) P->cand_slot = reinterpret_cast<int64_t*>(p);
  p = take(max_partial * 4);             if (P) P->partial = reinterpret_cast<float*>(p);
  p = take(max_grid_segc * 2048 * 4);    if (P) P->hist = reinterpret_cast<uint32_t*>(p);
  p = take(max_grid_segc * 8);           if (P) P->thr = reinterpret_cast<unsigned long long*>(p);
  p = take(max_grid_segc * 8);           if (P) P->prefix = reinterpret_cast<unsigned long long*>(p);
  p = take(max_grid_segc * 4);           if (P) P->need = reinterpret_cast<uint32_t*>(p);
  p = take(max_grid_segc * 4);           if (P) P->active = reinterpret_cast<int32_t*>(p);
  p = take(24 * 4);                      if (P) P->flags = reinterpret_cast<int32_t*>(p);
  p = take(sizeof(GridBarrier));         if (P) P->bar = reinterpret_cast<GridBarrier*>(p);
  return off;
}

size_t assign_workspace_layout(int64_t nseg, int64_t m, int b, char* base, BuildPlan* P) {
  const int64_t nslots = nseg * m, nnodes = nseg * b;
  const bool grid = m > kCtaMaxSeg;
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    uint64_t at = off;
    off = align256(off + (bytes ? bytes : 1));
    return base ? base + at : nullptr;
  };
  char* p;
  p = take(nslots * b * 4);                   if (P) P->D = reinterpret_cast<float*>(p);
  p = take(nslots * 8);                       if (P) P->pref = reinterpret_cast<uint64_t*>(p);
  p = take(nslots * 4);                       if (P) P->dbits = reinterpret_cast<uint32_t*>(p);
  p = take(nslots);                           if (P) P->ptr = reinterpret_cast<uint8_t*>(p);
  p = take(grid ? nnodes * 2048 * 4 : 0);     if (P) P->hist = reinterpret_cast<uint32_t*>(p);
  p = take(grid ? nnodes * 8 : 0);            if (P) P->thr = reinterpret_cast<unsigned long long*>(p);
  p = take(grid ? nnodes * 8 : 0);            if (P) P->prefix = reinterpret_cast<unsigned long long*>(p);
  p = take(grid ? nnodes * 4 : 0);            if (P) P->need = reinterpret_cast<uint32_t*>(p);
  p = take(grid ? nnodes * 4 : 0);            if (P) P->active = reinterpret_cast<int32_t*>(p);
  p = take(24 * 4);                           if (P) P->flags = reinterpret_cast<int32_t*>(p);
  p = take(sizeof(GridBarrier));              if (P) P->bar = reinterpret_cast<GridBarrier*>(p);
  return off;
}

}  // namespace lsa

extern "C" {

int lsa_version(void) { return LSA_VERSION; }

const char* lsa_strerror(int status) {
  switch (status) {
    case LSA_OK: return "ok";
    case LSA_ERR_INVALID_ARG: return "invalid argument";
    case LSA_ERR_SHAPE: return "unsupported or inconsistent shape";
    case LSA_ERR_CUDA: return "CUDA error";
    case LSA_ERR_TIMEOUT: return "device loop hit its iteration cap";
    case LSA_ERR_NONFINITE: return "NaN in an ordering decision";
    case LSA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

const char* lsa_last_error(void) { return g_err; }

int lsa_tree_describe(int32_t n_heads, int32_t r, const int32_t* branching, int32_t levels, int32_t leaf_size,
                      lsa_tree_desc* out) {
  if (!branching || !out) return fail(LSA_ERR_INVALID_ARG, "branching and out must be non-NULL");
  if (n_heads < 1) return fail(LSA_ERR_SHAPE, "n_heads must be >= 1 (got %d)", n_heads);
  if (r != 16 && r != 32 && r != 64) return fail(LSA_ERR_SHAPE, "r must be 16, 32 or 64 (got %d)", r);
  if (levels < 1 || levels > LSA_MAX_LEVELS) return fail(LSA_ERR_SHAPE, "levels must be in [1, 8] (got %d)", levels);
  if (leaf_size < 8 || leaf_size > 4096) return fail(LSA_ERR_SHAPE, "leaf_size must be in [8, 4096] (got %d)", leaf_size);
  lsa_tree_desc t;
  memset(&t, 0, sizeof(t));
  t.n_heads = n_heads;
  t.r = r;
  t.levels = levels;
  t.leaf_size = leaf_size;
  int64_t nodes = 1;
  for (int l = 0; l < levels; ++l) {
    const int bmax = l == 0 ? LSA_MAX_TOP_BRANCHING : LSA_MAX_BRANCHING;
    if (branching[l] < 2 || branching[l] > bmax)
      return fail(LSA_ERR_SHAPE, "branching[%d] must be in [2, %d] (got %d)", l, bmax, branching[l]);
    nodes *= branching[l];
    if (nodes * leaf_size > (int64_t(1) << 30)) return fail(LSA_ERR_SHAPE, "tree larger than 2^30 keys");
    t.branching[l] = branching[l];
    t.nodes[l] = nodes;
  }
  t.n_tree = nodes * leaf_size;
  if ((int64_t)n_heads * t.n_tree >= (int64_t(1) << 31))
    return fail(LSA_ERR_SHAPE, "n_heads * n_tree must stay below 2^31 (got %lld)", (long long)n_heads * t.n_tree);
  uint64_t off = 0;
  for (int l = 0; l < levels; ++l) {
    t.off_centroids[l] = off;
    off = align256(off + (uint64_t)n_heads * t.nodes[l] * r * sizeof(float));
  }
  for (int l = 0; l < levels; ++l) {
    t.off_min_pos[l] = off;
    off = align256(off + (uint64_t)n_heads * t.nodes[l] * sizeof(int32_t));
  }
  t.off_leaf_index = off;
  off = align256(off + (uint64_t)n_heads * t.n_tree * sizeof(int32_t));
  t.bytes = off;
  *out = t;
  return ok();
}

int lsa_build_workspace_bytes(const lsa_tree_desc* tree, int32_t d, size_t* bytes) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  *bytes = lsa::build_workspace_layout(*tree, nullptr, nullptr);
  return ok();
}

int lsa_build_tree(const lsa_tree_desc* tree, void* tree_mem, const void* K, int64_t n_cap, int32_t d,
                   int32_t dtype, const void* W, int32_t iters, uint64_t seed, void* workspace,
                   size_t workspace_bytes, int32_t* trace, int32_t* status, void* stream) {
  return lsa_build_tree_pooled(tree, tree_mem, K, n_cap, d, dtype, W, 1, iters, seed, workspace, workspace_bytes,
                               trace, status, stream);
}

int lsa_build_tree_pooled(const lsa_tree_desc* tree, void* tree_mem, const void* K, int64_t n_cap, int32_t d,
                          int32_t dtype, const void* W, int32_t pool, int32_t iters, uint64_t seed, void* workspace,
                          size_t workspace_bytes, int32_t* trace, int32_t* status, void* stream) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (pool < 1 || tree->leaf_size % pool != 0)
    return fail(LSA_ERR_SHAPE, "pool (%d) must be >= 1 and divide leaf_size (%d)", pool, tree->leaf_size);
  if (tree->branching[0] > LSA_MAX_BRANCHING)
    return fail(LSA_ERR_SHAPE, "the k-means build splits at most 16 ways (branching[0] = %d)", tree->branching[0]);
  if (!tree_mem || !K || !W) return fail(LSA_ERR_INVALID_ARG, "tree_mem, K and W must be non-NULL");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  if (n_cap < tree->n_tree) return fail(LSA_ERR_SHAPE, "n_cap (%lld) < n_tree (%lld)", (long long)n_cap, (long long)tree->n_tree);
  if (iters < 1 || iters > 1000) return fail(LSA_ERR_INVALID_ARG, "iters must be in [1, 1000] (got %d)", iters);
  const size_t need = lsa::build_workspace_layout(*tree, nullptr, nullptr);
  if (!workspace || workspace_bytes < need)
    return fail(LSA_ERR_WORKSPACE, "build needs %zu workspace bytes (got %zu)", need, workspace ? workspace_bytes : (size_t)0);
  lsa::BuildPlan P;
  lsa::build_workspace_layout(*tree, static_cast<char*>(workspace), &P);
  P.iters = iters;
  P.seed = seed;
  P.coop_blocks = lsa::da_grid_blocks();
  if (P.coop_blocks <= 0) return fail(LSA_ERR_CUDA, "cannot size the cooperative assignment grid");
  cudaError_t e = cudaMemsetAsync(tree_mem, 0, tree->bytes, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess)
    e = lsa::run_build(P, *tree, tree_mem, K, n_cap, d, dtype, W, pool, trace, status,
                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_build_tree_pooled");
  return ok();
}

static int append_subtree(const lsa_tree_desc* tree, lsa_tree_desc* sub) {
  if (tree->levels < 2) return fail(LSA_ERR_SHAPE, "an update on append needs levels >= 2 (got %d)", tree->levels);
  return lsa_tree_describe(tree->n_heads, tree->r, tree->branching + 1, tree->levels - 1, tree->leaf_size, sub);
}

int lsa_tree_append_workspace_bytes(const lsa_tree_desc* tree, int32_t d, size_t* bytes) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  lsa_tree_desc sub;
  if ((rc = append_subtree(tree, &sub)) != LSA_OK) return rc;
  *bytes = align256(sub.bytes) + lsa::build_workspace_layout(sub, nullptr, nullptr);
  return ok();
}

int lsa_tree_append(const lsa_tree_desc* tree, const void* tree_mem, const lsa_tree_desc* grown, void* grown_mem,
                    const void* K, int64_t n_cap, int32_t d, int32_t dtype, const void* W, int32_t iters,
                    uint64_t seed, void* workspace, size_t workspace_bytes, int32_t* trace, int32_t* status,
                    void* stream) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if ((rc = check_desc(grown)) != LSA_OK) return rc;
  lsa_tree_desc sub;
  if ((rc = append_subtree(tree, &sub)) != LSA_OK) return rc;
  bool match = grown->n_heads == tree->n_heads && grown->r == tree->r && grown->levels == tree->levels &&
               grown->leaf_size == tree->leaf_size && grown->branching[0] == tree->branching[0] + 1;
  for (int l = 1; l < tree->levels; ++l) match = match && grown->branching[l] == tree->branching[l];
  if (!match) return fail(LSA_ERR_SHAPE, "grown must describe the same tree with branching[0] + 1");
  if (!tree_mem || !grown_mem || !K || !W) return fail(LSA_ERR_INVALID_ARG, "tree_mem, grown_mem, K and W must be non-NULL");
  if (tree_mem == grown_mem) return fail(LSA_ERR_INVALID_ARG, "grown_mem must not be tree_mem");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  if (n_cap < grown->n_tree)
    return fail(LSA_ERR_SHAPE, "n_cap (%lld) < grown n_tree (%lld)", (long long)n_cap, (long long)grown->n_tree);
  if (iters < 1 || iters > 1000) return fail(LSA_ERR_INVALID_ARG, "iters must be in [1, 1000] (got %d)", iters);
  const size_t sub_bytes = align256(sub.bytes);
  const size_t need = sub_bytes + lsa::build_workspace_layout(sub, nullptr, nullptr);
  if (!workspace || workspace_bytes < need)
    return fail(LSA_ERR_WORKSPACE, "append needs %zu workspace bytes (got %zu)", need, workspace ? workspace_bytes : (size_t)0);
  char* sub_mem = static_cast<char*>(workspace);
  lsa::BuildPlan P;
  lsa::build_workspace_layout(sub, sub_mem + sub_bytes, &P);
  P.iters = iters;
  P.seed = seed;
  P.coop_blocks = lsa::da_grid_blocks();
  if (P.coop_blocks <= 0) return fail(LSA_ERR_CUDA, "cannot size the cooperative assignment grid");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t esz = dtype == LSA_BF16 ? 2 : 4;
  const char* Kb = static_cast<const char*>(K) + (size_t)tree->n_tree * d * esz;   // first appended key of head 0
  cudaError_t e = cudaMemsetAsync(grown_mem, 0, grown->bytes, st);
  if (e == cudaSuccess) e = lsa::run_build(P, sub, sub_mem, Kb, n_cap, d, dtype, W, 1, trace, status, st);
  if (e == cudaSuccess) e = lsa::run_tree_attach(*tree, tree_mem, sub, sub_mem, *grown, grown_mem, st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_tree_append");
  return ok();
}

// Beam checks shared by the select calls: fills a's per-level fields, returns
// LSA_OK or the failure code (beam_max through *bmax).
static int beam_checks(const lsa_tree_desc* tree, const int32_t* beam, lsa::SelectArgs& a, int* bmax) {
  if (!beam) return fail(LSA_ERR_INVALID_ARG, "beam must be non-NULL");
  int beam_max = 0;
  for (int l = 0; l < tree->levels; ++l) {
    const int64_t avail = l == 0 ? tree->nodes[0] : (int64_t)beam[l - 1] * tree->branching[l];
    if (beam[l] < 1 || beam[l] > LSA_MAX_BEAM || beam[l] > avail ||
        (l + 1 < tree->levels && (int64_t)beam[l] * tree->branching[l + 1] > 512))
      return fail(LSA_ERR_SHAPE, "beam[%d] = %d must be in [1, min(64, %lld)]", l, beam[l], (long long)avail);
    beam_max = beam[l] > beam_max ? beam[l] : beam_max;
    a.beam[l] = beam[l];
    a.branching[l] = tree->branching[l];
    a.nodes[l] = tree->nodes[l];
    a.off_c[l] = tree->off_centroids[l];
    a.off_m[l] = tree->off_min_pos[l];
  }
  *bmax = beam_max;
  return LSA_OK;
}

// Arguments of lsa_select and lsa_select_batched (same checks); *empty when T == 0.
static int select_setup(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                        int32_t d, int32_t dtype, const void* W, const int32_t* beam, const int32_t* q_pos,
                        int32_t* idx_out, int32_t* leaves_out, float* qlat_out, int32_t* beam_out, int32_t* status,
                        lsa::SelectArgs& a, bool* empty) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!beam) return fail(LSA_ERR_INVALID_ARG, "beam must be non-NULL");
  if (T < 0) return fail(LSA_ERR_SHAPE, "T must be >= 0");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  if (Hq < tree->n_heads || Hq % tree->n_heads) return fail(LSA_ERR_SHAPE, "Hq (%d) must be a multiple of n_heads (%d)", Hq, tree->n_heads);
  if (Hq / tree->n_heads > 64) return fail(LSA_ERR_SHAPE, "more than 64 query heads per group");
  memset(&a, 0, sizeof(a));
  int beam_max = 0;
  if ((rc = beam_checks(tree, beam, a, &beam_max)) != LSA_OK) return rc;
  a.T = T; a.Hq = Hq; a.Hkv = tree->n_heads; a.G = Hq / tree->n_heads; a.d = d; a.r = tree->r;
  a.levels = tree->levels; a.leaf = tree->leaf_size; a.beam_max = beam_max; a.n_tree = tree->n_tree;
  a.off_leaf = tree->off_leaf_index;
  *empty = T == 0;
  if (T == 0) return LSA_OK;
  if (!tree_mem || !Q || !W) return fail(LSA_ERR_INVALID_ARG, "tree_mem, Q and W must be non-NULL");
  if (!idx_out && !leaves_out) return fail(LSA_ERR_INVALID_ARG, "give idx_out, leaves_out or both");
  a.Q = Q; a.W = W; a.tree = static_cast<const char*>(tree_mem); a.q_pos = q_pos; a.idx_out = idx_out;
  a.leaves_out = leaves_out;
  a.qlat_out = qlat_out; a.beam_out = beam_out; a.status = status;
  return LSA_OK;
}

int lsa_select(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq, int32_t d,
               int32_t dtype, const void* W, const int32_t* beam, const int32_t* q_pos, int32_t* idx_out,
               int32_t* leaves_out, float* qlat_out, int32_t* beam_out, int32_t* status, void* stream) {
  lsa::SelectArgs a;
  bool empty = false;
  int rc = select_setup(tree, tree_mem, Q, T, Hq, d, dtype, W, beam, q_pos, idx_out, leaves_out, qlat_out, beam_out,
                        status, a, &empty);
  if (rc != LSA_OK) return rc;
  if (empty) return ok();
  cudaError_t e = lsa::run_select(a, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_select");
  return ok();
}

// the batched schedule packs (query, rank) into 32 bits: query * 32 + rank
static constexpr int32_t kBatchedMaxT = 1 << 26;

int lsa_select_batched_workspace_bytes(const lsa_tree_desc* tree, int32_t T, const int32_t* beam, size_t* bytes) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes must be non-NULL");
  if (T < 0 || T > kBatchedMaxT) return fail(LSA_ERR_SHAPE, "T must be in [0, 2^26] (got %d)", T);
  lsa::SelectArgs a;
  memset(&a, 0, sizeof(a));
  int beam_max = 0;
  if ((rc = beam_checks(tree, beam, a, &beam_max)) != LSA_OK) return rc;
  a.T = T; a.Hkv = tree->n_heads; a.r = tree->r; a.levels = tree->levels;
  *bytes = lsa::select_nodes_workspace_bytes(a);
  return ok();
}

int lsa_select_batched(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                       int32_t d, int32_t dtype, const void* W, const int32_t* beam, const int32_t* q_pos,
                       int32_t* idx_out, int32_t* leaves_out, float* qlat_out, int32_t* beam_out, void* workspace,
                       size_t workspace_bytes, int32_t* status, void* stream) {
  lsa::SelectArgs a;
  bool empty = false;
  int rc = select_setup(tree, tree_mem, Q, T, Hq, d, dtype, W, beam, q_pos, idx_out, leaves_out, qlat_out, beam_out,
                        status, a, &empty);
  if (rc != LSA_OK) return rc;
  if (T > kBatchedMaxT) return fail(LSA_ERR_SHAPE, "T must be <= 2^26 (got %d)", T);
  if (empty) return ok();
  const size_t need = lsa::select_nodes_workspace_bytes(a);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(LSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes);
  cudaError_t e = lsa::run_select_nodes(a, dtype, workspace, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_select_batched");
  return ok();
}

static int attn_common_checks(const void* Q, int32_t T, int32_t Hq, const void* K, const void* V, int32_t n_heads,
                              int64_t n_cap, int32_t d, int32_t dtype, const int32_t* idx, int32_t K_sel,
                              const int32_t* q_pos, int32_t causal, int64_t tail_begin, int64_t tail_end) {
  if (T < 0 || n_heads < 1 || Hq < n_heads || Hq % n_heads) return fail(LSA_ERR_SHAPE, "need T >= 0 and Hq a multiple of n_heads");
  const int G = Hq / n_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(LSA_ERR_SHAPE, "query heads per group must be 1, 2, 4 or 8 (got %d)", G);
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  if (n_cap < 1) return fail(LSA_ERR_SHAPE, "n_cap must be >= 1");
  if (K_sel < 0) return fail(LSA_ERR_SHAPE, "K_sel must be >= 0");
  if (tail_begin < 0 || tail_end < tail_begin || tail_end > n_cap)
    return fail(LSA_ERR_SHAPE, "tail range [%lld, %lld) must lie in [0, n_cap)", (long long)tail_begin, (long long)tail_end);
  if (T > 0) {
    if (!Q || !K || !V) return fail(LSA_ERR_INVALID_ARG, "Q, K and V must be non-NULL");
    if (K_sel > 0 && !idx) return fail(LSA_ERR_INVALID_ARG, "idx must be non-NULL when K_sel > 0");
    if (causal && !q_pos) return fail(LSA_ERR_INVALID_ARG, "q_pos is required when causal");
  }
  return LSA_OK;
}

int lsa_select_flat(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                    int32_t d, int32_t dtype, const void* W, int32_t n_leaves, const int32_t* q_pos,
                    int32_t* idx_out, int32_t* leaves_out, float* qlat_out, int32_t* status, void* stream) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (T < 0) return fail(LSA_ERR_SHAPE, "T must be >= 0");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  if (Hq < tree->n_heads || Hq % tree->n_heads) return fail(LSA_ERR_SHAPE, "Hq (%d) must be a multiple of n_heads (%d)", Hq, tree->n_heads);
  if (Hq / tree->n_heads > 64) return fail(LSA_ERR_SHAPE, "more than 64 query heads per group");
  const int L = tree->levels - 1;
  if (n_leaves < 1 || n_leaves > LSA_MAX_BEAM || n_leaves > tree->nodes[L])
    return fail(LSA_ERR_SHAPE, "n_leaves = %d must be in [1, min(%d, %lld)]", n_leaves, LSA_MAX_BEAM,
                (long long)tree->nodes[L]);
  if (T == 0) return ok();
  if (!tree_mem || !Q || !W) return fail(LSA_ERR_INVALID_ARG, "tree_mem, Q and W must be non-NULL");
  if (!idx_out && !leaves_out) return fail(LSA_ERR_INVALID_ARG, "give idx_out, leaves_out or both");
  lsa::SelectArgs a;
  memset(&a, 0, sizeof(a));
  for (int l = 0; l < tree->levels; ++l) {
    a.branching[l] = tree->branching[l];
    a.nodes[l] = tree->nodes[l];
    a.off_c[l] = tree->off_centroids[l];
    a.off_m[l] = tree->off_min_pos[l];
  }
  a.beam[L] = n_leaves;
  a.Q = Q; a.W = W; a.tree = static_cast<const char*>(tree_mem); a.q_pos = q_pos; a.idx_out = idx_out;
  a.leaves_out = leaves_out; a.qlat_out = qlat_out; a.status = status;
  a.T = T; a.Hq = Hq; a.Hkv = tree->n_heads; a.G = Hq / tree->n_heads; a.d = d; a.r = tree->r;
  a.levels = tree->levels; a.leaf = tree->leaf_size; a.beam_max = n_leaves; a.n_tree = tree->n_tree;
  a.off_leaf = tree->off_leaf_index;
  {   // a prime that does not divide the leaf count: i -> i * p mod n_leaves is a bijection
    const int64_t NL = tree->nodes[L];
    const int64_t primes[] = {1000003, 999983, 40503, 7919};
    a.flat_perm = 1;
    for (int64_t p : primes)
      if (NL % p != 0) { a.flat_perm = p % NL == 0 ? 1 : p; break; }
  }
  cudaError_t e = lsa::run_select_flat(a, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_select_flat");
  return ok();
}

int lsa_attn_workspace_bytes(int32_t T, int32_t Hq, int32_t n_heads, int32_t d, int32_t K_sel, int64_t tail_len,
                             size_t* bytes) {
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  if (T < 0 || n_heads < 1 || Hq < 1 || K_sel < 0 || tail_len < 0 || (d != 64 && d != 128))
    return fail(LSA_ERR_SHAPE, "bad sizes");
  const int ns = T > 0 ? lsa::attn_splits(T, n_heads, K_sel + tail_len) : 1;
  *bytes = ns > 1 ? (size_t)T * Hq * ns * (d + 2) * sizeof(float) : 0;
  return ok();
}

static void fill_attn(lsa::AttnArgs& a, const void* Q, int32_t T, int32_t Hq, const void* K, const void* V,
                      int32_t n_heads, int64_t n_cap, int32_t d, const int32_t* idx, int32_t K_sel,
                      const int32_t* q_pos, int32_t causal, int64_t tail_begin, int64_t tail_end, float scale,
                      int32_t* status) {
  memset(&a, 0, sizeof(a));
  a.Q = Q; a.K = K; a.V = V; a.idx = K_sel > 0 ? idx : nullptr; a.q_pos = q_pos; a.status = status;
  a.T = T; a.n_cap = n_cap; a.tail_begin = tail_begin; a.tail_end = tail_end;
  a.Hq = Hq; a.Hkv = n_heads; a.G = Hq / n_heads; a.d = d; a.K_sel = K_sel; a.causal = causal ? 1 : 0;
  const int64_t keys = K_sel + (tail_end - tail_begin);
  a.nsplit = lsa::attn_splits(T, n_heads, keys);
  int64_t kps = (keys + a.nsplit - 1) / a.nsplit;
  kps = (kps + 15) / 16 * 16;
  a.keys_per_split = (int32_t)(kps > 0 ? kps : 16);
  a.scale = scale;
  a.scale_log2 = scale * 1.44269504088896340736f;
}

int lsa_sparse_attn(const void* Q, int32_t T, int32_t Hq, const void* K, const void* V, int32_t n_heads,
                    int64_t n_cap, int32_t d, int32_t dtype, const int32_t* idx, int32_t K_sel, const int32_t* q_pos,
                    int32_t causal, int64_t tail_begin, int64_t tail_end, float scale, void* O, float* LSE,
                    void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = attn_common_checks(Q, T, Hq, K, V, n_heads, n_cap, d, dtype, idx, K_sel, q_pos, causal, tail_begin, tail_end);
  if (rc != LSA_OK) return rc;
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  if (T == 0) return ok();
  if (!O || !LSE) return fail(LSA_ERR_INVALID_ARG, "O and LSE must be non-NULL");
  lsa::AttnArgs a;
  fill_attn(a, Q, T, Hq, K, V, n_heads, n_cap, d, idx, K_sel, q_pos, causal, tail_begin, tail_end, scale, status);
  a.O = O;
  a.LSE = LSE;
  if (a.nsplit > 1) {
    const size_t need = (size_t)T * Hq * a.nsplit * (d + 2) * sizeof(float);
    if (!workspace || workspace_bytes < need)
      return fail(LSA_ERR_WORKSPACE, "attention needs %zu workspace bytes (got %zu)", need, workspace ? workspace_bytes : (size_t)0);
    a.part = static_cast<float*>(workspace);
  }
  cudaError_t e = lsa::run_attn_fwd(a, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn");
  return ok();
}

static int tree_attn_ws(const lsa_tree_desc* tree, int32_t T, int32_t Hq, int32_t d, int32_t dtype,
                        int32_t n_leaves, int32_t n_sink, int32_t window, size_t* bytes) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  if (T < 0 || Hq < tree->n_heads || Hq % tree->n_heads || n_leaves < 1 || n_leaves > LSA_MAX_BEAM ||
      (d != 64 && d != 128))
    return fail(LSA_ERR_SHAPE, "bad sizes");
  if (n_sink < 0 || window < 0 || n_sink > LSA_MAX_SINK_WINDOW || window > LSA_MAX_SINK_WINDOW)
    return fail(LSA_ERR_SHAPE, "n_sink and window must lie in [0, %d]", LSA_MAX_SINK_WINDOW);
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  const int G = Hq / tree->n_heads;
  const bool fast = lsa::tree_attn_fast_path(dtype, d, G, tree->leaf_size);
  *bytes = lsa::tree_attn_workspace(tree->n_heads, tree->nodes[tree->levels - 1], T, Hq, d, n_leaves,
                                    tree->leaf_size, fast, n_sink, window);
  return ok();
}

int lsa_tree_attn_workspace_bytes(const lsa_tree_desc* tree, int32_t T, int32_t Hq, int32_t d, int32_t dtype,
                                  int32_t n_leaves, size_t* bytes) {
  return tree_attn_ws(tree, T, Hq, d, dtype, n_leaves, 0, 0, bytes);
}

int lsa_tree_attn_sw_workspace_bytes(const lsa_tree_desc* tree, int32_t T, int32_t Hq, int32_t d, int32_t dtype,
                                     int32_t n_leaves, int32_t n_sink, int32_t window, size_t* bytes) {
  return tree_attn_ws(tree, T, Hq, d, dtype, n_leaves, n_sink, window, bytes);
}

static int tree_attn_call(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                          const void* K, const void* V, int64_t n_cap, int32_t d, int32_t dtype,
                          const int32_t* leaves, int32_t n_leaves, const int32_t* q_pos, int32_t causal,
                          int32_t n_sink, int32_t window, float scale, void* O, float* LSE, void* workspace,
                          size_t workspace_bytes, int32_t* status, void* stream, const char* name) {
  size_t need = 0;
  int rc = tree_attn_ws(tree, T, Hq, d, dtype, n_leaves, n_sink, window, &need);
  if (rc != LSA_OK) return rc;
  const int G = Hq / tree->n_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(LSA_ERR_SHAPE, "query heads per group must be 1, 2, 4 or 8");
  if (n_cap < tree->n_tree) return fail(LSA_ERR_SHAPE, "n_cap (%lld) < n_tree", (long long)n_cap);
  if (n_sink > n_cap) return fail(LSA_ERR_SHAPE, "n_sink (%d) > n_cap (%lld)", n_sink, (long long)n_cap);
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  if (T == 0) return ok();
  if (!tree_mem || !Q || !K || !V || !leaves || !O || !LSE)
    return fail(LSA_ERR_INVALID_ARG, "tree_mem, Q, K, V, leaves, O and LSE must be non-NULL");
  if (causal && !q_pos) return fail(LSA_ERR_INVALID_ARG, "q_pos is required when causal");
  if (!workspace || workspace_bytes < need)
    return fail(LSA_ERR_WORKSPACE, "tree attention needs %zu workspace bytes (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  lsa::TreeAttnCall c;
  memset(&c, 0, sizeof(c));
  c.Q = Q; c.K = K; c.V = V;
  c.leaf_index = reinterpret_cast<const int32_t*>(static_cast<const char*>(tree_mem) + tree->off_leaf_index);
  c.leaves = leaves; c.q_pos = q_pos; c.O = O; c.LSE = LSE; c.workspace = workspace; c.status = status;
  c.T = T; c.n_cap = n_cap; c.n_tree = tree->n_tree; c.NL = tree->nodes[tree->levels - 1];
  c.Hq = Hq; c.H = tree->n_heads; c.d = d; c.dtype = dtype; c.B = n_leaves; c.leaf = tree->leaf_size;
  c.causal = causal ? 1 : 0; c.scale = scale; c.n_sink = n_sink; c.window = window;
  cudaError_t e = lsa::run_tree_attn(c, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return ok();
}

int lsa_tree_attn(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                  const void* K, const void* V, int64_t n_cap, int32_t d, int32_t dtype, const int32_t* leaves,
                  int32_t n_leaves, const int32_t* q_pos, int32_t causal, float scale, void* O, float* LSE,
                  void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  return tree_attn_call(tree, tree_mem, Q, T, Hq, K, V, n_cap, d, dtype, leaves, n_leaves, q_pos, causal, 0, 0, scale,
                        O, LSE, workspace, workspace_bytes, status, stream, "lsa_tree_attn");
}

int lsa_tree_attn_sw(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                     const void* K, const void* V, int64_t n_cap, int32_t d, int32_t dtype, const int32_t* leaves,
                     int32_t n_leaves, const int32_t* q_pos, int32_t n_sink, int32_t window, float scale, void* O,
                     float* LSE, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  if (!q_pos && T > 0) return fail(LSA_ERR_INVALID_ARG, "q_pos is required with sink and window keys");
  return tree_attn_call(tree, tree_mem, Q, T, Hq, K, V, n_cap, d, dtype, leaves, n_leaves, q_pos, 1, n_sink, window,
                        scale, O, LSE, workspace, workspace_bytes, status, stream, "lsa_tree_attn_sw");
}

int lsa_tree_attn_bwd_workspace_bytes(const lsa_tree_desc* tree, int32_t T, int32_t Hq, int32_t d, int32_t dtype,
                                      int32_t n_leaves, size_t* bytes) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  if (T < 0 || Hq < tree->n_heads || Hq % tree->n_heads || n_leaves < 1 || n_leaves > LSA_MAX_BEAM ||
      (d != 64 && d != 128))
    return fail(LSA_ERR_SHAPE, "bad sizes");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  const bool fast = lsa::tree_attn_fast_path(dtype, d, Hq / tree->n_heads, tree->leaf_size);
  *bytes = lsa::tree_attn_bwd_workspace(tree->n_heads, tree->nodes[tree->levels - 1], T, Hq, d, n_leaves,
                                        tree->leaf_size, fast);
  return ok();
}

int lsa_tree_attn_bwd(const lsa_tree_desc* tree, const void* tree_mem, const void* Q, int32_t T, int32_t Hq,
                      const void* K, const void* V, int64_t n_cap, int32_t d, int32_t dtype, const void* O,
                      const float* LSE, const void* dO, const int32_t* leaves, int32_t n_leaves,
                      const int32_t* q_pos, int32_t causal, float scale, float* dQ, float* dK, float* dV,
                      void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  size_t need = 0;
  int rc = lsa_tree_attn_bwd_workspace_bytes(tree, T, Hq, d, dtype, n_leaves, &need);
  if (rc != LSA_OK) return rc;
  const int G = Hq / tree->n_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(LSA_ERR_SHAPE, "query heads per group must be 1, 2, 4 or 8");
  if (n_cap < tree->n_tree) return fail(LSA_ERR_SHAPE, "n_cap (%lld) < n_tree", (long long)n_cap);
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  if (!dK || !dV) return fail(LSA_ERR_INVALID_ARG, "dK and dV must be non-NULL");
  if (T > 0) {
    if (!tree_mem || !Q || !K || !V || !O || !LSE || !dO || !leaves || !dQ)
      return fail(LSA_ERR_INVALID_ARG, "tree_mem, Q, K, V, O, LSE, dO, leaves and dQ must be non-NULL");
    if (causal && !q_pos) return fail(LSA_ERR_INVALID_ARG, "q_pos is required when causal");
    if (!workspace || workspace_bytes < need)
      return fail(LSA_ERR_WORKSPACE, "tree attention backward needs %zu workspace bytes (got %zu)", need,
                  workspace ? workspace_bytes : (size_t)0);
  }
  lsa::TreeAttnCall c;
  memset(&c, 0, sizeof(c));
  c.Q = Q; c.K = K; c.V = V;
  c.leaf_index = tree_mem ? reinterpret_cast<const int32_t*>(static_cast<const char*>(tree_mem) + tree->off_leaf_index)
                          : nullptr;
  c.leaves = leaves; c.q_pos = q_pos; c.workspace = workspace; c.status = status;
  c.T = T; c.n_cap = n_cap; c.n_tree = tree->n_tree; c.NL = tree->nodes[tree->levels - 1];
  c.Hq = Hq; c.H = tree->n_heads; c.d = d; c.dtype = dtype; c.B = n_leaves; c.leaf = tree->leaf_size;
  c.causal = causal ? 1 : 0; c.scale = scale;
  cudaError_t e = lsa::run_tree_attn_bwd(c, O, LSE, dO, dQ, dK, dV, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_tree_attn_bwd");
  return ok();
}

int lsa_sparse_attn_bwd(const void* Q, int32_t T, int32_t Hq, const void* K, const void* V, int32_t n_heads,
                        int64_t n_cap, int32_t d, int32_t dtype, const void* O, const float* LSE, const void* dO,
                        const int32_t* idx, int32_t K_sel, const int32_t* q_pos, int32_t causal, int64_t tail_begin,
                        int64_t tail_end, float scale, float* dQ, float* dK, float* dV, int32_t* status,
                        void* stream) {
  int rc = attn_common_checks(Q, T, Hq, K, V, n_heads, n_cap, d, dtype, idx, K_sel, q_pos, causal, tail_begin, tail_end);
  if (rc != LSA_OK) return rc;
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  if (!dK || !dV) return fail(LSA_ERR_INVALID_ARG, "dK and dV must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t kv_bytes = (size_t)n_heads * n_cap * d * sizeof(float);
  cudaError_t e;
  if ((e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_bwd");
  if ((e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_bwd");
  if (T == 0) return ok();
  if (!O || !LSE || !dO || !dQ) return fail(LSA_ERR_INVALID_ARG, "O, LSE, dO and dQ must be non-NULL");
  lsa::AttnArgs a;
  fill_attn(a, Q, T, Hq, K, V, n_heads, n_cap, d, idx, K_sel, q_pos, causal, tail_begin, tail_end, scale, status);
  a.O = const_cast<void*>(O);
  a.LSE = const_cast<float*>(LSE);
  a.dO = dO;
  a.dQ = dQ;
  a.dK = dK;
  a.dV = dV;
  if (a.nsplit > 1 && (e = cudaMemsetAsync(dQ, 0, (size_t)T * Hq * d * sizeof(float), st)) != cudaSuccess)
    return cuda_fail(e, "lsa_sparse_attn_bwd");
  e = lsa::run_attn_bwd(a, dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_bwd");
  return ok();
}

static int sw_checks(int32_t n_sink, int32_t window, const int32_t* q_pos, int64_t n_cap) {
  if (n_sink < 0 || window < 0 || n_sink > LSA_MAX_SINK_WINDOW || window > LSA_MAX_SINK_WINDOW)
    return fail(LSA_ERR_SHAPE, "n_sink and window must lie in [0, %d]", LSA_MAX_SINK_WINDOW);
  if (n_sink > n_cap) return fail(LSA_ERR_SHAPE, "n_sink (%d) > n_cap (%lld)", n_sink, (long long)n_cap);
  if (!q_pos) return fail(LSA_ERR_INVALID_ARG, "q_pos is required with sink and window keys");
  return LSA_OK;
}

int lsa_sparse_attn_sw_workspace_bytes(int32_t T, int32_t Hq, int32_t n_heads, int32_t d, int32_t K_sel,
                                       int64_t tail_len, int32_t n_sink, int32_t window, size_t* bytes) {
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  if (n_sink < 0 || window < 0 || n_sink > LSA_MAX_SINK_WINDOW || window > LSA_MAX_SINK_WINDOW)
    return fail(LSA_ERR_SHAPE, "n_sink and window must lie in [0, %d]", LSA_MAX_SINK_WINDOW);
  const int32_t K2 = K_sel + n_sink + window;
  size_t attn = 0;
  int rc = lsa_attn_workspace_bytes(T, Hq, n_heads, d, K2, tail_len, &attn);
  if (rc != LSA_OK) return rc;
  *bytes = align256((size_t)n_heads * T * K2 * sizeof(int32_t)) + attn;
  return ok();
}

int lsa_sparse_attn_sw(const void* Q, int32_t T, int32_t Hq, const void* K, const void* V, int32_t n_heads,
                       int64_t n_cap, int32_t d, int32_t dtype, const int32_t* idx, int32_t K_sel,
                       const int32_t* q_pos, int32_t n_sink, int32_t window, int64_t tail_begin, int64_t tail_end,
                       float scale, void* O, float* LSE, void* workspace, size_t workspace_bytes, int32_t* status,
                       void* stream) {
  int rc = attn_common_checks(Q, T, Hq, K, V, n_heads, n_cap, d, dtype, idx, K_sel, q_pos, 1, tail_begin, tail_end);
  if (rc != LSA_OK) return rc;
  if ((rc = sw_checks(n_sink, window, q_pos, n_cap)) != LSA_OK) return rc;
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  if (T == 0) return ok();
  if (!O || !LSE) return fail(LSA_ERR_INVALID_ARG, "O and LSE must be non-NULL");
  size_t need = 0;
  if ((rc = lsa_sparse_attn_sw_workspace_bytes(T, Hq, n_heads, d, K_sel, tail_end - tail_begin, n_sink, window,
                                               &need)) != LSA_OK)
    return rc;
  if (!workspace || workspace_bytes < need)
    return fail(LSA_ERR_WORKSPACE, "attention with sink and window keys needs %zu workspace bytes (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  const int32_t K2 = K_sel + n_sink + window;
  int32_t* idx2 = static_cast<int32_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = lsa::run_attn_extend(K_sel > 0 ? idx : nullptr, K_sel, T, n_heads, q_pos, n_sink, window,
                                       tail_begin, tail_end, n_cap, idx2, st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_sw");
  lsa::AttnArgs a;
  fill_attn(a, Q, T, Hq, K, V, n_heads, n_cap, d, idx2, K2, q_pos, 1, tail_begin, tail_end, scale, status);
  a.O = O;
  a.LSE = LSE;
  if (a.nsplit > 1)
    a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256((size_t)n_heads * T * K2 * sizeof(int32_t)));
  e = lsa::run_attn_fwd(a, dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_sw");
  return ok();
}

int lsa_sparse_attn_sw_bwd(const void* Q, int32_t T, int32_t Hq, const void* K, const void* V, int32_t n_heads,
                           int64_t n_cap, int32_t d, int32_t dtype, const void* O, const float* LSE, const void* dO,
                           const int32_t* idx, int32_t K_sel, const int32_t* q_pos, int32_t n_sink, int32_t window,
                           int64_t tail_begin, int64_t tail_end, float scale, float* dQ, float* dK, float* dV,
                           void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = attn_common_checks(Q, T, Hq, K, V, n_heads, n_cap, d, dtype, idx, K_sel, q_pos, 1, tail_begin, tail_end);
  if (rc != LSA_OK) return rc;
  if ((rc = sw_checks(n_sink, window, q_pos, n_cap)) != LSA_OK) return rc;
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  if (!dK || !dV) return fail(LSA_ERR_INVALID_ARG, "dK and dV must be non-NULL");
  const int32_t K2 = K_sel + n_sink + window;
  const size_t need = align256((size_t)n_heads * T * K2 * sizeof(int32_t));
  if (T > 0 && (!workspace || workspace_bytes < need))
    return fail(LSA_ERR_WORKSPACE, "the backward with sink and window keys needs %zu workspace bytes (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t kv_bytes = (size_t)n_heads * n_cap * d * sizeof(float);
  cudaError_t e;
  if ((e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_sw_bwd");
  if ((e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_sw_bwd");
  if (T == 0) return ok();
  if (!O || !LSE || !dO || !dQ) return fail(LSA_ERR_INVALID_ARG, "O, LSE, dO and dQ must be non-NULL");
  int32_t* idx2 = static_cast<int32_t*>(workspace);
  e = lsa::run_attn_extend(K_sel > 0 ? idx : nullptr, K_sel, T, n_heads, q_pos, n_sink, window, tail_begin, tail_end,
                           n_cap, idx2, st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_sw_bwd");
  lsa::AttnArgs a;
  fill_attn(a, Q, T, Hq, K, V, n_heads, n_cap, d, idx2, K2, q_pos, 1, tail_begin, tail_end, scale, status);
  a.O = const_cast<void*>(O);
  a.LSE = const_cast<float*>(LSE);
  a.dO = dO;
  a.dQ = dQ;
  a.dK = dK;
  a.dV = dV;
  if (a.nsplit > 1 && (e = cudaMemsetAsync(dQ, 0, (size_t)T * Hq * d * sizeof(float), st)) != cudaSuccess)
    return cuda_fail(e, "lsa_sparse_attn_sw_bwd");
  e = lsa::run_attn_bwd(a, dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_sparse_attn_sw_bwd");
  return ok();
}

static size_t decode_ws_layout(int64_t Hkv, int B, int G, int d, int nsplit, char* base, int32_t** leaves,
                               int32_t** cnt, float** part) {
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    uint64_t at = off;
    off = align256(off + (bytes ? bytes : 1));
    return base ? base + at : nullptr;
  };
  char* p = take((uint64_t)Hkv * B * 4);
  if (leaves) *leaves = reinterpret_cast<int32_t*>(p);
  p = take((uint64_t)Hkv * 4);
  if (cnt) *cnt = reinterpret_cast<int32_t*>(p);
  p = take((uint64_t)Hkv * nsplit * G * (d + 4) * 4);   // partial rows padded to 16 bytes
  if (part) *part = reinterpret_cast<float*>(p);
  return off;
}

int lsa_decode_step_workspace_bytes(const lsa_tree_desc* tree, int32_t Hq, int32_t d, const int32_t* beam,
                                    int64_t tail_len_max, size_t* bytes) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  lsa::SelectArgs a;
  memset(&a, 0, sizeof(a));
  int bmax = 0;
  if ((rc = beam_checks(tree, beam, a, &bmax)) != LSA_OK) return rc;
  if (Hq < tree->n_heads || Hq % tree->n_heads) return fail(LSA_ERR_SHAPE, "Hq must be a multiple of n_heads");
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  if (tail_len_max < 0) return fail(LSA_ERR_SHAPE, "tail_len_max must be >= 0");
  const int B = beam[tree->levels - 1];
  const int nsplit = lsa::dec_splits(B, tree->leaf_size, tail_len_max);
  *bytes = decode_ws_layout(tree->n_heads, B, Hq / tree->n_heads, d, nsplit, nullptr, nullptr, nullptr, nullptr);
  return ok();
}

int lsa_decode_step(const lsa_tree_desc* tree, const void* tree_mem, const void* W, const int32_t* beam, void* K,
                    void* V, int64_t n_cap, int32_t d, int32_t dtype, const void* Q, int32_t Hq, const void* K_row,
                    const void* V_row, int64_t pos, int64_t tail_begin, float scale, void* O, float* LSE,
                    int32_t* leaves_out, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int rc = check_desc(tree);
  if (rc != LSA_OK) return rc;
  lsa::SelectArgs a;
  memset(&a, 0, sizeof(a));
  int bmax = 0;
  if ((rc = beam_checks(tree, beam, a, &bmax)) != LSA_OK) return rc;
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(LSA_ERR_SHAPE, "d must be 64 or 128 (got %d)", d);
  const int32_t H = tree->n_heads;
  if (Hq < H || Hq % H) return fail(LSA_ERR_SHAPE, "Hq (%d) must be a multiple of n_heads (%d)", Hq, H);
  const int G = Hq / H;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(LSA_ERR_SHAPE, "query heads per group must be 1, 2, 4 or 8");
  if (!tree_mem || !W || !K || !V || !Q || !O || !LSE)
    return fail(LSA_ERR_INVALID_ARG, "tree_mem, W, K, V, Q, O and LSE must be non-NULL");
  if ((K_row == nullptr) != (V_row == nullptr)) return fail(LSA_ERR_INVALID_ARG, "give both K_row and V_row or neither");
  if (n_cap < tree->n_tree) return fail(LSA_ERR_SHAPE, "n_cap is smaller than the indexed keys");
  if (pos < tree->n_tree - 1 || pos >= n_cap)
    return fail(LSA_ERR_SHAPE, "pos %lld must lie in [n_tree - 1, n_cap) (n_tree %lld)", (long long)pos,
                (long long)tree->n_tree);
  if (tail_begin < tree->n_tree || tail_begin > pos + 1)
    return fail(LSA_ERR_SHAPE, "tail_begin %lld must lie in [n_tree, pos + 1]", (long long)tail_begin);
  if (!std::isfinite(scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite");
  const int B = beam[tree->levels - 1];
  const int64_t tail_len = pos + 1 - tail_begin;
  const int nsplit = lsa::dec_splits(B, tree->leaf_size, tail_len);
  if (nsplit > lsa::dec_max_splits(dtype, d, G))
    return fail(LSA_ERR_SHAPE, "decode step: %d splits of 64 keys (kept leaves and tail) exceed the %d one call merges",
                nsplit, lsa::dec_max_splits(dtype, d, G));
  const size_t need = decode_ws_layout(H, B, G, d, nsplit, nullptr, nullptr, nullptr, nullptr);
  if (!workspace || workspace_bytes < need)
    return fail(LSA_ERR_WORKSPACE, "decode step needs %zu workspace bytes (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  int32_t *leaves = nullptr, *cnt = nullptr;
  float* part = nullptr;
  decode_ws_layout(H, B, G, d, nsplit, static_cast<char*>(workspace), &leaves, &cnt, &part);
  if (leaves_out) leaves = leaves_out;   // the kept leaves go straight to the caller's buffer
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // select (one CTA per KV group) with the append and the counter reset folded in
  a.Q = Q; a.W = W; a.tree = static_cast<const char*>(tree_mem); a.q_pos = nullptr; a.idx_out = nullptr;
  a.leaves_out = leaves; a.status = status;
  a.T = 1; a.Hq = Hq; a.Hkv = H; a.G = G; a.d = d; a.r = tree->r;
  a.levels = tree->levels; a.leaf = tree->leaf_size; a.beam_max = bmax; a.n_tree = tree->n_tree;
  a.off_leaf = tree->off_leaf_index;
  const int row_bytes = d * (dtype == LSA_BF16 ? 2 : 4);
  if (K_row) {
    a.app_K = K; a.app_V = V; a.app_Kr = K_row; a.app_Vr = V_row; a.app_pos = pos; a.app_ncap = n_cap;
    a.app_row_bytes = row_bytes;
  }
  a.zero_cnt = cnt;
  cudaError_t e = lsa::run_select(a, dtype, st);
  if (e == cudaSuccess) {
    lsa::DecAttnArgs b;
    memset(&b, 0, sizeof(b));
    b.Q = Q; b.K = K; b.V = V; b.leaves = leaves;
    b.leaf_index = reinterpret_cast<const int32_t*>(static_cast<const char*>(tree_mem) + tree->off_leaf_index);
    b.O = O; b.LSE = LSE; b.part = part; b.cnt = cnt;
    b.n_cap = n_cap; b.n_tree = tree->n_tree; b.tail_begin = tail_begin; b.tail_end = pos + 1;
    b.Hq = Hq; b.Hkv = H; b.B = B; b.leaf = tree->leaf_size; b.spl = (tree->leaf_size + 63) / 64;
    b.nsplit = nsplit; b.scale_log2 = scale * 1.44269504088896340736f;
    e = lsa::run_dec_attn(b, dtype, d, G, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "lsa_decode_step");
  return ok();
}

static int assign_checks(int64_t nseg, int64_t m, int32_t b) {
  if (nseg < 1 || m < 1) return fail(LSA_ERR_SHAPE, "need nseg >= 1 and m >= 1");
  if (b < 2 || b > LSA_MAX_BRANCHING || m % b != 0)
    return fail(LSA_ERR_SHAPE, "b must be in [2, 16] and divide m (b = %d, m = %lld)", b, (long long)m);
  if (nseg * m >= (int64_t(1) << 31)) return fail(LSA_ERR_SHAPE, "nseg * m must stay below 2^31");
  return LSA_OK;
}

int lsa_balanced_assign_workspace_bytes(int64_t nseg, int64_t m, int32_t b, size_t* bytes) {
  if (!bytes) return fail(LSA_ERR_INVALID_ARG, "bytes is NULL");
  int rc = assign_checks(nseg, m, b);
  if (rc != LSA_OK) return rc;
  *bytes = lsa::assign_workspace_layout(nseg, m, b, nullptr, nullptr);
  return ok();
}

int lsa_balanced_assign(const float* Z, const float* mu, int64_t nseg, int64_t m, int32_t b, int32_t r,
                        int32_t max_rounds, uint8_t* choice, void* workspace, size_t workspace_bytes,
                        int32_t* status, void* stream) {
  if (!Z || !mu || !choice) return fail(LSA_ERR_INVALID_ARG, "Z, mu and choice must be non-NULL");
  int rc = assign_checks(nseg, m, b);
  if (rc != LSA_OK) return rc;
  if (r != 16 && r != 32 && r != 64) return fail(LSA_ERR_SHAPE, "r must be 16, 32 or 64 (got %d)", r);
  if (max_rounds < 0) return fail(LSA_ERR_INVALID_ARG, "max_rounds must be >= 0 (0: the build's cap)");
  const size_t need = lsa::assign_workspace_layout(nseg, m, b, nullptr, nullptr);
  if (!workspace || workspace_bytes < need)
    return fail(LSA_ERR_WORKSPACE, "assignment needs %zu workspace bytes (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  lsa::BuildPlan P;
  memset(&P, 0, sizeof(P));
  lsa::assign_workspace_layout(nseg, m, b, static_cast<char*>(workspace), &P);
  P.mu = const_cast<float*>(mu);
  P.choice = choice;
  P.coop_blocks = lsa::da_grid_blocks();
  if (P.coop_blocks <= 0) return fail(LSA_ERR_CUDA, "cannot size the cooperative assignment grid");
  cudaError_t e = lsa::run_assign(P, Z, nseg, m, b, r, max_rounds ? max_rounds : lsa::kMaxRounds, status,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_balanced_assign");
  return ok();
}

int lsa_project_keys(const void* K, int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype, const void* W,
                     int32_t r, int64_t n, float* Z, int32_t* status, void* stream) {
  if (!K || !W || (!Z && n > 0)) return fail(LSA_ERR_INVALID_ARG, "K, W and Z must be non-NULL");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (n_heads < 1 || (d != 64 && d != 128) || (r != 16 && r != 32 && r != 64))
    return fail(LSA_ERR_SHAPE, "need n_heads >= 1, d in {64, 128} and r in {16, 32, 64}");
  if (n < 0 || n > n_cap) return fail(LSA_ERR_SHAPE, "n %lld outside [0, n_cap]", (long long)n);
  cudaError_t e = lsa::run_project(K, n_cap, W, n, n_heads, r, d, dtype, Z, nullptr, status,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_project_keys");
  return ok();
}

int lsa_kv_append(void* K, void* V, int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype, int64_t pos,
                  const void* K_rows, const void* V_rows, void* stream) {
  if (!K || !V || !K_rows || !V_rows) return fail(LSA_ERR_INVALID_ARG, "K, V, K_rows and V_rows must be non-NULL");
  if (!valid_dtype(dtype)) return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (n_heads < 1 || (d != 64 && d != 128)) return fail(LSA_ERR_SHAPE, "need n_heads >= 1 and d in {64, 128}");
  if (pos < 0 || pos >= n_cap) return fail(LSA_ERR_SHAPE, "pos %lld outside [0, n_cap)", (long long)pos);
  const int64_t row_bytes = (int64_t)d * (dtype == LSA_BF16 ? 2 : 4);
  cudaError_t e = lsa::run_kv_append(K, V, n_heads, n_cap, row_bytes, pos, K_rows, V_rows,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_kv_append");
  return ok();
}

int lsa_status_clear(int32_t* status, void* stream) {
  if (!status) return fail(LSA_ERR_INVALID_ARG, "status is NULL");
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lsa_status_clear");
  return ok();
}

int lsa_status_check(const int32_t* status, void* stream, int32_t* host_out) {
  if (!status || !host_out) return fail(LSA_ERR_INVALID_ARG, "status and host_out must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host_out, status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "lsa_status_check");
  return ok();
}

}  // extern "C"
