// select.cu -- hierarchical beam search over the latent-key tree.
//
// Method (kongchang.com, "Latent Sparse Attention Breaks Through the
// Million-Token Context Bottleneck", section "How LSA Sidesteps Per-Key Scoring
// with Hierarchical Clustering"): the query starts at the root, scores only a
// few candidate clusters per level and descends into a few branches;
// bdtechtalks.com, "Latent sparse attention", section "How latent sparse
// attention works": hierarchical search with a fixed budget per level, then a
// fixed number of original keys taken from the chosen clusters.
//
// One warp per (query t, KV group g).  Scores are fp32 inner products of the
// group's latent query with fp32 centroids (exact enough that ordering
// decisions only differ from an fp64 evaluation inside a ~1e-6 relative band).
// Candidates are ranked by a packed 64-bit key (orderable score, ~node id) so a
// descending sort gives (score desc, node id asc).  A level's candidates (at
// most beam * branching <= 512) are scored by lane groups that read whole
// centroid rows with coalesced loads, then sorted in registers by a warp-wide
// bitonic network (shuffles across lanes); the walk needs no CTA barrier, so
// many walks are in flight per SM to hide memory latency.

#include <climits>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

constexpr int kSelWarps = 8;       // (query, group) units per CTA, one warp each
constexpr int kSelMaxE = 16;       // sort width per lane: beam * branching <= 32 * 16
constexpr int kWideWarps = 16;     // warps of the small-batch kernel: 32 * 16 candidate slots
// Below this many (query, group) units the warp-per-unit kernel cannot fill the
// 148 SMs (8 units per CTA), and one CTA per unit is used instead.
constexpr int64_t kWideUnits = 148 * 8;

// Bitonic sort (descending) of 32*E keys held in registers, E per lane; element
// index i = lane * E + e.  Pairs closer than E sit in one lane; farther pairs are
// exchanged with a shuffle.
template <int E>
__device__ __forceinline__ void warp_sort_desc(unsigned long long (&v)[E]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int p = e ^ j;
          if (p > e) {
            const bool desc = ((lane * E + e) & k) == 0;
            const unsigned long long x = v[e], y = v[p];
            if (desc ? (x < y) : (x > y)) { v[e] = y; v[p] = x; }
          }
        }
      } else {
        const int lj = j / E;
        const bool lower = (lane & lj) == 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[e], lj);
          const bool desc = ((lane * E + e) & k) == 0;
          const bool take_max = lower == desc;
          v[e] = take_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
        }
      }
    }
  }
}

__device__ __forceinline__ int32_t key_id(unsigned long long k) {
  return (int32_t)(0xffffffffu - (uint32_t)(k & 0xffffffffull));
}

// Write the first B of a sorted register list (element index lane * E + e) as the
// kept set; returns (in every lane) how many of them are real candidates.
template <int E>
__device__ __forceinline__ int emit_kept(const unsigned long long (&v)[E], int B, int32_t* kept) {
  const int lane = threadIdx.x & 31;
  int cnt = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    if (i < B) {
      kept[i] = v[e] ? key_id(v[e]) : -1;
      cnt += v[e] != 0ull;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  return cnt;
}

// Shared-memory slot of sorted-list element i (lane i / E, register i % E): the
// register index is XORed with the lane so that the E-strided reads of one
// register index by the 32 lanes spread over all banks.
template <int E>
__device__ __forceinline__ int key_slot(int i) {
  const int ln = i / E, e = i % E;
  return ln * E + (e ^ (ln % E));
}

// Keep the best B (<= 64) of the keys v held by one warp (E per lane, element
// index lane * E + e): writes their node ids to next[0..B) in key order and returns
// how many are real candidates.  s_key: shared scratch of >= 64 keys that no lane
// of the warp still needs.
template <int E>
__device__ __forceinline__ int warp_keep_best(unsigned long long (&v)[E], int B, unsigned long long* s_key,
                                              int32_t* next) {
  const int lane = threadIdx.x & 31;
  if constexpr (E >= 8) {
    // Threshold first: the B-th largest of the lanes' two largest keys is a lower
    // bound of the B-th largest key overall (those 64 are keys of the level), so
    // every kept key is >= tau.  Keys are distinct, so sorting the keys >= tau
    // gives exactly the first B of the full order; when more than 64 pass, the
    // full sort runs instead.
    unsigned long long smp[2] = {0ull, 0ull};
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const unsigned long long x = v[e];
      const bool top = x > smp[0];
      smp[1] = top ? smp[0] : (x > smp[1] ? x : smp[1]);
      smp[0] = top ? x : smp[0];
    }
    warp_sort_desc<2>(smp);
    const unsigned long long tau = __shfl_sync(0xffffffffu, ((B - 1) & 1) ? smp[1] : smp[0], (B - 1) >> 1);
    int c = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) c += (v[e] != 0ull && v[e] >= tau);
    int inc = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += y;
    }
    const int total = __shfl_sync(0xffffffffu, inc, 31);
    if (total <= 64) {
      __syncwarp();                       // every lane has read its keys: s_key is free
      int o = inc - c;
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (v[e] != 0ull && v[e] >= tau) s_key[o++] = v[e];
      __syncwarp();
      unsigned long long w[2];
      w[0] = 2 * lane < total ? s_key[2 * lane] : 0ull;
      w[1] = 2 * lane + 1 < total ? s_key[2 * lane + 1] : 0ull;
      warp_sort_desc<2>(w);
      return emit_kept<2>(w, B, next);
    }
  }
  warp_sort_desc<E>(v);
  return emit_kept<E>(v, B, next);
}

// Centroid rows are scored by groups of LPR lanes; each lane holds F float4
// pieces of the latent query, so one warp-wide load covers 32 / LPR whole rows.
template <int R>
struct RowSplit {
  static constexpr int LPR = 4;
  static constexpr int F = R / (4 * LPR);
  static constexpr int RPI = 32 / LPR;
  static constexpr int U = F >= 8 ? 1 : (8 / F > 4 ? 4 : 8 / F);   // rows in flight per lane group
};

// One level of the walk: score the ncand children of the kept parents (all nodes
// on level 0), write their keys to s_key, sort them in registers (E per lane)
// and keep the first beam[l].  Returns the number of real candidates kept.
template <int R, int E>
__device__ __forceinline__ int level_pass(const SelectArgs& a, int l, int ncand, const float* cent,
                                          const int32_t* mpos, bool all_eligible, int64_t qpos,
                                          const float4 (&lat)[RowSplit<R>::F], const int32_t* kept, int b,
                                          unsigned long long* s_key, int32_t* next, bool& bad) {
  using RS = RowSplit<R>;
  constexpr int U = RS::U;
  const int lane = threadIdx.x & 31, sub = lane % RS::LPR, grp = lane / RS::LPR;
  for (int c0 = 0; c0 < ncand; c0 += RS::RPI * U) {
    float4 x[U][RS::F];
    bool ok[U];
    int64_t id[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * RS::RPI + grp;
      ok[u] = c < ncand;
      id[u] = 0;
      if (ok[u]) {
        id[u] = l == 0 ? c : (int64_t)kept[c / b] * b + (c % b);
        ok[u] = all_eligible || (int64_t)__ldg(&mpos[id[u]]) <= qpos;
      }
      const float4* cr = reinterpret_cast<const float4*>(cent + id[u] * R);
#pragma unroll
      for (int f = 0; f < RS::F; ++f) x[u][f] = ok[u] ? __ldg(&cr[f * RS::LPR + sub]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float sc = 0.f;
#pragma unroll
      for (int f = 0; f < RS::F; ++f) {
        sc = fmaf(lat[f].x, x[u][f].x, sc);
        sc = fmaf(lat[f].y, x[u][f].y, sc);
        sc = fmaf(lat[f].z, x[u][f].z, sc);
        sc = fmaf(lat[f].w, x[u][f].w, sc);
      }
#pragma unroll
      for (int o = 1; o < RS::LPR; o <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
      const int c = c0 + u * RS::RPI + grp;
      if (sub == 0 && c < ncand) {
        unsigned long long key = 0ull;
        if (ok[u]) {
          if (isnan(sc)) bad = true;
          else key = ((unsigned long long)orderable(sc) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)id[u]);
        }
        s_key[key_slot<E>(c)] = key;
      }
    }
  }
  __syncwarp();
  unsigned long long v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    v[e] = i < ncand ? s_key[key_slot<E>(i)] : 0ull;
  }
  return warp_keep_best<E>(v, a.beam[l], s_key, next);
}

// Latent arithmetic shared by every select kernel, so a query's latent (and its
// walk) does not depend on the kernel or the batch it is selected in: the group
// query q (mean of the G query heads, summed in head order) times W[g]; column c
// is the fixed pairwise sum of kLatParts partial sums, partial p running
// sequentially over the rows [p DK / kLatParts, (p + 1) DK / kLatParts).
constexpr int kLatParts = 8;

template <typename T, int R, int DK>
__device__ __forceinline__ float latent_partial(const float* q, const T* Wg, int c, int p) {
  constexpr int RPP = DK / kLatParts;
  float acc = 0.f;
#pragma unroll 4
  for (int jj = 0; jj < RPP; ++jj) {
    const int j = p * RPP + jj;
    acc = fmaf(q[j], to_f32(Wg[(int64_t)j * R + c]), acc);
  }
  return acc;
}
__device__ __forceinline__ float latent_combine(const float (&pp)[kLatParts]) {
  return ((pp[0] + pp[1]) + (pp[2] + pp[3])) + ((pp[4] + pp[5]) + (pp[6] + pp[7]));
}
template <typename T, int DK>
__device__ __forceinline__ float group_mean(const SelectArgs& a, int64_t t, int g, int j) {
  const T* Q = static_cast<const T*>(a.Q);
  float sum = 0.f;
  for (int i = 0; i < a.G; ++i) sum += to_f32(Q[(t * a.Hq + (int64_t)g * a.G + i) * DK + j]);
  return sum / (float)a.G;
}

// The latent of (t, g) computed by one warp (Wg: global or shared memory).
template <typename T, int R, int DK>
__device__ __forceinline__ void latent_query(const SelectArgs& a, int64_t t, int g, const T* Wg, float* s_q,
                                             float* s_lat) {
  constexpr int RPP = DK / kLatParts;
  const int lane = threadIdx.x & 31;
  for (int j = lane; j < DK; j += 32) s_q[j] = group_mean<T, DK>(a, t, g, j);
  __syncwarp();
  // lane: columns 2 c2 and 2 c2 + 1 (one 2-element load per row); per column the
  // same partial sums and pairwise order as latent_partial / latent_combine
  for (int c2 = lane; c2 < R / 2; c2 += 32) {
    auto part = [&](int p, float& x0, float& x1) {
      x0 = 0.f;
      x1 = 0.f;
#pragma unroll 4
      for (int jj = 0; jj < RPP; ++jj) {
        const int j = p * RPP + jj;
        float w[2];
        load2_generic(Wg + (int64_t)j * R + 2 * c2, w);
        x0 = fmaf(s_q[j], w[0], x0);
        x1 = fmaf(s_q[j], w[1], x1);
      }
    };
    float a0, a1, b0, b1, lo0, lo1, hi0, hi1, u0, u1;
    part(0, a0, a1); part(1, b0, b1); lo0 = a0 + b0; lo1 = a1 + b1;
    part(2, a0, a1); part(3, b0, b1); u0 = a0 + b0; u1 = a1 + b1; lo0 = lo0 + u0; lo1 = lo1 + u1;
    part(4, a0, a1); part(5, b0, b1); hi0 = a0 + b0; hi1 = a1 + b1;
    part(6, a0, a1); part(7, b0, b1); u0 = a0 + b0; u1 = a1 + b1; hi0 = hi0 + u0; hi1 = hi1 + u1;
    const float v0 = lo0 + hi0, v1 = lo1 + hi1;
    s_lat[2 * c2] = v0;
    s_lat[2 * c2 + 1] = v1;
    if (a.qlat_out) {
      a.qlat_out[(t * a.Hkv + g) * R + 2 * c2] = v0;
      a.qlat_out[(t * a.Hkv + g) * R + 2 * c2 + 1] = v1;
    }
  }
  __syncwarp();
}

// The same latent computed by a whole CTA of NT >= max(DK, R * kLatParts) threads
// (one partial sum per thread); every thread of the CTA must call it.
template <typename T, int R, int DK, int NT>
__device__ __forceinline__ void latent_query_cta(const SelectArgs& a, int64_t t, int g, const T* Wg, float* s_q,
                                                 float (*s_part)[R], float* s_lat) {
  static_assert(NT >= DK && NT >= R * kLatParts, "");
  const int tid = threadIdx.x;
  if (tid < DK) s_q[tid] = group_mean<T, DK>(a, t, g, tid);
  __syncthreads();
  if (tid < R * kLatParts) s_part[tid / R][tid % R] = latent_partial<T, R, DK>(s_q, Wg, tid % R, tid / R);
  __syncthreads();
  if (tid < R) {
    float pp[kLatParts];
#pragma unroll
    for (int p = 0; p < kLatParts; ++p) pp[p] = s_part[p][tid];
    const float v = latent_combine(pp);
    s_lat[tid] = v;
    if (a.qlat_out) a.qlat_out[(t * a.Hkv + g) * R + tid] = v;
  }
  __syncthreads();
}

// One warp per (query t, KV group g), kSelWarps queries of one group per CTA.
// The walk synchronises only its own warp.
template <typename T, int R, int DK>
__global__ void __launch_bounds__(kSelWarps * 32, 3) k_select(SelectArgs a) {
  using RS = RowSplit<R>;
  __shared__ unsigned long long s_key[kSelWarps][32 * kSelMaxE];
  __shared__ float s_q[kSelWarps][DK];
  __shared__ __align__(16) float s_lat[kSelWarps][R];
  __shared__ int32_t s_kept[kSelWarps][2][LSA_MAX_BEAM];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y;
  const int64_t t = (int64_t)blockIdx.x * kSelWarps + warp;
  if (t >= a.T) return;
  latent_query<T, R, DK>(a, t, g, static_cast<const T*>(a.W) + (int64_t)g * DK * R, s_q[warp], s_lat[warp]);
  float4 lat[RS::F];
#pragma unroll
  for (int f = 0; f < RS::F; ++f)
    lat[f] = reinterpret_cast<const float4*>(s_lat[warp])[f * RS::LPR + lane % RS::LPR];
  const int64_t qpos = a.q_pos ? (int64_t)a.q_pos[t] : (int64_t)LLONG_MAX;
  // a query at or past the last indexed position sees every node (decode): no
  // per-node eligibility load is needed
  const bool all_eligible = qpos >= a.n_tree - 1;
  unsigned long long* keys = s_key[warp];
  int ncand = (int)a.nodes[0];
  int n_kept = 0;
  int cur = 0;
  bool bad = false;
  for (int l = 0; l < a.levels; ++l) {
    const int b = a.branching[l];
    const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[l]) + (int64_t)g * a.nodes[l] * R;
    const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[l]) + (int64_t)g * a.nodes[l];
    const int32_t* kept = s_kept[warp][cur];
    int32_t* next = s_kept[warp][cur ^ 1];
    int valid;
#define LSA_LEVEL(EE) level_pass<R, EE>(a, l, ncand, cent, mpos, all_eligible, qpos, lat, kept, b, keys, next, bad)
    if (ncand <= 32) valid = LSA_LEVEL(1);
    else if (ncand <= 64) valid = LSA_LEVEL(2);
    else if (ncand <= 128) valid = LSA_LEVEL(4);
    else if (ncand <= 256) valid = LSA_LEVEL(8);
    else valid = LSA_LEVEL(16);
#undef LSA_LEVEL
    __syncwarp();
    if (a.beam_out && lane < a.beam_max) {
      const int32_t id = lane < valid ? next[lane] : -1;
      a.beam_out[(((int64_t)l * a.Hkv + g) * a.T + t) * a.beam_max + lane] = id;
    }
    n_kept = valid;
    cur ^= 1;
    ncand = l + 1 < a.levels ? valid * a.branching[l + 1] : 0;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, LSA_ERR_NONFINITE);
  const int32_t* kept = s_kept[warp][cur];
  const int leaf = a.leaf;
  const int B = a.beam[a.levels - 1];
  if (a.leaves_out && lane < B) a.leaves_out[((int64_t)g * a.T + t) * B + lane] = lane < n_kept ? kept[lane] : -1;
  if (a.idx_out) {
    const int64_t K_sel = (int64_t)B * leaf;
    const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
    int32_t* out = a.idx_out + ((int64_t)g * a.T + t) * K_sel;
    for (int64_t i = lane; i < K_sel; i += 32) {
      const int k = (int)(i / leaf), q = (int)(i % leaf);
      out[i] = k < n_kept ? __ldg(&li[(int64_t)kept[k] * leaf + q]) : -1;
    }
  }
}

// Small batches (decode): one CTA of kWideWarps warps per (query t, KV group g),
// so a level's candidates are scored in one or two memory round trips.  Each
// warp sorts a chunk of 32 keys; chunk lists are then merged pairwise keeping
// the first 32 (the elementwise max of one descending list and the other one
// reversed holds the top 32 of both as a bitonic sequence, which five shuffle
// steps sort).  Scores use the same lane-group sums as k_select.
template <typename T, int R, int DK>
__global__ void __launch_bounds__(kWideWarps * 32) k_select_wide(SelectArgs a) {
  using RS = RowSplit<R>;
  constexpr int NT = kWideWarps * 32;
  __shared__ unsigned long long s_key[32 * kWideWarps];
  __shared__ __align__(16) T s_w[DK * R];
  __shared__ float s_q[DK];
  __shared__ float s_part[kLatParts][R];
  __shared__ __align__(16) float s_lat[R];
  __shared__ int32_t s_kept[2][LSA_MAX_BEAM];
  __shared__ int s_valid;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.y;
  const int64_t t = blockIdx.x;
  // a kernel launched as this one's programmatic dependent (the decode step's
  // attention) may start now; it waits for this grid to finish before it reads
  // anything written here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (t == 0) {   // decode step: this head's new key and value rows, the attention's counter
    const int chunks = a.app_row_bytes / 16;
    if (a.app_K && tid < 2 * chunks) {
      const bool isv = tid >= chunks;
      const int c = isv ? tid - chunks : tid;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(isv ? a.app_Vr : a.app_Kr) +
                                                        (int64_t)g * a.app_row_bytes) + c;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(isv ? a.app_V : a.app_K) +
                                            ((int64_t)g * a.app_ncap + a.app_pos) * a.app_row_bytes) + c;
      *dst = __ldg(src);
    }
    if (a.zero_cnt && tid == 0) a.zero_cnt[g] = 0;
  }
  {  // W[g] staged by the whole CTA in one memory round trip; the top level's rows are
     // requested into L2 meanwhile (every walk scores all of them next)
    constexpr int VEC = 16 / sizeof(T);
    const T* W = static_cast<const T*>(a.W) + (int64_t)g * DK * R;
    const char* top = a.tree + a.off_c[0] + (int64_t)g * a.nodes[0] * R * sizeof(float);
    const int64_t top_lines = (a.nodes[0] * R * (int64_t)sizeof(float) + 127) / 128;
    for (int64_t x = tid; x < top_lines; x += NT) asm volatile("prefetch.global.L2 [%0];" ::"l"(top + x * 128));
    for (int i = tid * VEC; i < DK * R; i += NT * VEC)
      *reinterpret_cast<uint4*>(&s_w[i]) = __ldg(reinterpret_cast<const uint4*>(W + i));
  }
  __syncthreads();
  latent_query_cta<T, R, DK, NT>(a, t, g, s_w, s_q, s_part, s_lat);
  float4 lat[RS::F];
#pragma unroll
  for (int f = 0; f < RS::F; ++f) lat[f] = reinterpret_cast<const float4*>(s_lat)[f * RS::LPR + lane % RS::LPR];
  const int64_t qpos = a.q_pos ? (int64_t)a.q_pos[t] : (int64_t)LLONG_MAX;
  const bool all_eligible = qpos >= a.n_tree - 1;
  const int sub = lane % RS::LPR, gg = warp * RS::RPI + lane / RS::LPR;
  constexpr int GROUPS = kWideWarps * RS::RPI;
  int ncand = (int)a.nodes[0];
  int n_kept = 0;
  int cur = 0;
  bool bad = false;
  for (int l = 0; l < a.levels; ++l) {
    const int b = a.branching[l];
    const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[l]) + (int64_t)g * a.nodes[l] * R;
    const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[l]) + (int64_t)g * a.nodes[l];
    const int32_t* kept = s_kept[cur];
    constexpr int U = 32 * kWideWarps / GROUPS;   // every candidate slot in flight at once
    for (int c0 = 0; c0 < ncand; c0 += GROUPS * U) {
      float4 x[U][RS::F];
      bool ok[U];
      int64_t id[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * GROUPS + gg;
        ok[u] = c < ncand;
        id[u] = 0;
        if (ok[u]) {
          id[u] = l == 0 ? c : (int64_t)kept[c / b] * b + (c % b);
          ok[u] = all_eligible || (int64_t)__ldg(&mpos[id[u]]) <= qpos;
        }
        const float4* cr = reinterpret_cast<const float4*>(cent + id[u] * R);
#pragma unroll
        for (int f = 0; f < RS::F; ++f)
          x[u][f] = ok[u] ? __ldg(&cr[f * RS::LPR + sub]) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float sc = 0.f;
#pragma unroll
        for (int f = 0; f < RS::F; ++f) {
          sc = fmaf(lat[f].x, x[u][f].x, sc);
          sc = fmaf(lat[f].y, x[u][f].y, sc);
          sc = fmaf(lat[f].z, x[u][f].z, sc);
          sc = fmaf(lat[f].w, x[u][f].w, sc);
        }
#pragma unroll
        for (int o = 1; o < RS::LPR; o <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
        const int c = c0 + u * GROUPS + gg;
        if (sub == 0 && c < ncand) {
          unsigned long long key = 0ull;
          if (ok[u]) {
            if (isnan(sc)) bad = true;
            else key = ((unsigned long long)orderable(sc) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)id[u]);
          }
          s_key[c] = key;
        }
      }
    }
    __syncthreads();
    const int nchunks = (ncand + 31) / 32;
    unsigned long long v[1];
    v[0] = warp < nchunks && warp * 32 + lane < ncand ? s_key[warp * 32 + lane] : 0ull;
    if (warp < nchunks) warp_sort_desc<1>(v);
    // a warp's list replaces its own chunk, which only that warp has read
    for (int step = 1; step < nchunks; step <<= 1) {
      if (warp % (2 * step) == step && warp < nchunks) s_key[warp * 32 + lane] = v[0];
      __syncthreads();
      if (warp % (2 * step) == 0 && warp + step < nchunks) {
        const unsigned long long o = s_key[(warp + step) * 32 + 31 - lane];
        v[0] = v[0] > o ? v[0] : o;
#pragma unroll
        for (int j = 16; j; j >>= 1) {
          const unsigned long long p = __shfl_xor_sync(0xffffffffu, v[0], j);
          const bool lower = (lane & j) == 0;
          v[0] = lower ? (v[0] > p ? v[0] : p) : (v[0] < p ? v[0] : p);
        }
      }
      __syncthreads();
    }
    int32_t* next = s_kept[cur ^ 1];
    if (warp == 0) {
      const int valid = emit_kept<1>(v, a.beam[l], next);
      if (lane == 0) s_valid = valid;
    }
    __syncthreads();
    const int valid = s_valid;
    if (a.beam_out && tid < a.beam_max) {
      const int32_t id = tid < valid ? next[tid] : -1;
      a.beam_out[(((int64_t)l * a.Hkv + g) * a.T + t) * a.beam_max + tid] = id;
    }
    n_kept = valid;
    cur ^= 1;
    ncand = l + 1 < a.levels ? valid * a.branching[l + 1] : 0;
  }
  if (__syncthreads_or(bad) && tid == 0) set_status(a.status, LSA_ERR_NONFINITE);
  const int32_t* kept = s_kept[cur];
  const int leaf = a.leaf;
  const int B = a.beam[a.levels - 1];
  if (a.leaves_out && tid < B) a.leaves_out[((int64_t)g * a.T + t) * B + tid] = tid < n_kept ? kept[tid] : -1;
  if (a.idx_out) {
    const int64_t K_sel = (int64_t)B * leaf;
    const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
    int32_t* out = a.idx_out + ((int64_t)g * a.T + t) * K_sel;
    for (int64_t i = tid; i < K_sel; i += NT) {
      const int k = (int)(i / leaf), q = (int)(i % leaf);
      out[i] = k < n_kept ? __ldg(&li[(int64_t)kept[k] * leaf + q]) : -1;
    }
  }
}

template <typename T>
static cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  const bool wide = a.T * a.Hkv < kWideUnits;
  dim3 grid((unsigned)(wide ? a.T : ceil_div(a.T, kSelWarps)), (unsigned)a.Hkv);
#define LSA_SEL(RR, DD)                                                     \
  if (a.r == RR && a.d == DD) {                                             \
    if (wide) k_select_wide<T, RR, DD><<<grid, kWideWarps * 32, 0, st>>>(a); \
    else k_select<T, RR, DD><<<grid, kSelWarps * 32, 0, st>>>(a);           \
    return cudaGetLastError();                                              \
  }
  LSA_SEL(16, 64) LSA_SEL(32, 64) LSA_SEL(64, 64) LSA_SEL(16, 128) LSA_SEL(32, 128) LSA_SEL(64, 128)
#undef LSA_SEL
  return cudaErrorInvalidValue;
}

// ---- flat search: every leaf centroid scored ----------------------------------
//
// bdtechtalks.com, "Latent sparse attention", section "How latent sparse attention
// works" (first strategy): the query is compared against all cluster centroids.
// A CTA takes kFlatQ queries of one KV group and streams the group's leaf
// centroids through shared memory in tiles of kFlatTile leaves; a thread scores
// 4 queries x 8 leaves (sequential fp32 FMAs over the r dimensions).  Keys above a
// query's running threshold (its B-th best key so far) go to a shared buffer;
// when a buffer holds more than kFlatKeep keys a warp sorts it, keeps the best B
// and raises the threshold.  Keys as in the beam walk: (orderable score, ~leaf id),
// so the order is (score desc, leaf id asc).
constexpr int kFlatQ = 32;              // queries per CTA (4 per warp)
constexpr int kFlatTile = 256;          // leaves per tile (8 per lane)
constexpr int kFlatKeep = 160;          // buffer size that triggers a reduction
constexpr int kFlatCap = kFlatKeep + kFlatTile;

template <int R>
struct FlatSmem {
  float cent[kFlatTile][R + 4];          // padded rows: a quarter-warp's float4 reads hit distinct banks
  int32_t mpos[kFlatTile];
  unsigned long long buf[kFlatQ][kFlatCap];
  unsigned long long tau[kFlatQ];
  int32_t cnt[kFlatQ];
  __align__(16) float lat[kFlatQ][R];
  float q[kSelWarps][128];
  int32_t qpos[kFlatQ];
  int32_t kept[kFlatQ][LSA_MAX_BEAM];
  int32_t nkept[kFlatQ];
};

// Warp: the best B keys of query q's buffer into its first slots; returns how many.
template <int R>
__device__ __forceinline__ void flat_reduce(FlatSmem<R>& S, int q, int B) {
  const int lane = threadIdx.x & 31;
  const int n = S.cnt[q];
  unsigned long long v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int i = lane * 16 + e;
    v[e] = i < n ? S.buf[q][i] : 0ull;
  }
  warp_sort_desc<16>(v);
  __syncwarp();
  int valid = 0;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int i = lane * 16 + e;
    if (i < B) {
      S.buf[q][i] = v[e];
      valid += v[e] != 0ull;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) valid += __shfl_xor_sync(0xffffffffu, valid, o);
  const unsigned long long last = __shfl_sync(0xffffffffu, v[(B - 1) & 15], (B - 1) >> 4);
  __syncwarp();
  if (lane == 0) {
    S.cnt[q] = valid;
    S.tau[q] = valid >= B ? last : 0ull;
  }
  __syncwarp();
}

template <typename T, int R, int DK>
__global__ void __launch_bounds__(kSelWarps * 32, 1) k_select_flat(SelectArgs a) {
  extern __shared__ __align__(16) char flat_raw[];
  FlatSmem<R>& S = *reinterpret_cast<FlatSmem<R>*>(flat_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int g = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * kFlatQ;
  const int L = a.levels - 1, B = a.beam[L];
  const int64_t NL = a.nodes[L];
  const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[L]) + (int64_t)g * NL * R;
  const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[L]) + (int64_t)g * NL;
  const T* Wg = static_cast<const T*>(a.W) + (int64_t)g * DK * R;
  for (int qq = warp * 4; qq < warp * 4 + 4; ++qq) {   // latents of this warp's 4 queries
    const int64_t t = t0 + qq;
    if (t < a.T) {
      latent_query<T, R, DK>(a, t, g, Wg, S.q[warp], S.lat[qq]);
    } else {
      for (int k = lane; k < R; k += 32) S.lat[qq][k] = 0.f;
    }
    if (lane == 0) {
      S.cnt[qq] = 0;
      S.tau[qq] = 0ull;
      S.qpos[qq] = t < a.T ? (a.q_pos ? a.q_pos[t] : INT32_MAX) : -1;
    }
  }
  __syncthreads();
  bool bad = false;
  for (int64_t L0 = 0; L0 < NL; L0 += kFlatTile) {
    const int nt = (int)min64(kFlatTile, NL - L0);
    {  // all of a thread's loads in flight before its stores
      constexpr int PER = kFlatTile * (R / 4) / (kSelWarps * 32);
      float4 x[PER];
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int i = tid + j * kSelWarps * 32, l = i / (R / 4), kc = i % (R / 4);
        x[j] = l < nt ? __ldg(reinterpret_cast<const float4*>(cent + (L0 + l) * R) + kc) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int i = tid + j * kSelWarps * 32, l = i / (R / 4), kc = i % (R / 4);
        *reinterpret_cast<float4*>(&S.cent[l][kc * 4]) = x[j];
      }
    }
    for (int l = tid; l < kFlatTile; l += kSelWarps * 32) S.mpos[l] = l < nt ? __ldg(&mpos[L0 + l]) : INT32_MAX;
    __syncthreads();
    float acc[4][8];
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[qq][i] = 0.f;
#pragma unroll 2
    for (int k = 0; k < R; k += 4) {
      float4 lq[4], cl[8];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) lq[qq] = *reinterpret_cast<const float4*>(&S.lat[warp * 4 + qq][k]);
#pragma unroll
      for (int i = 0; i < 8; ++i) cl[i] = *reinterpret_cast<const float4*>(&S.cent[lane + 32 * i][k]);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc[qq][i] = fmaf(lq[qq].x, cl[i].x, acc[qq][i]);
          acc[qq][i] = fmaf(lq[qq].y, cl[i].y, acc[qq][i]);
          acc[qq][i] = fmaf(lq[qq].z, cl[i].z, acc[qq][i]);
          acc[qq][i] = fmaf(lq[qq].w, cl[i].w, acc[qq][i]);
        }
    }
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      const int q = warp * 4 + qq;
      const int64_t qp = S.qpos[q];
      if (qp < 0) continue;
      const unsigned long long tau = S.tau[q];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int l = lane + 32 * i;
        if (l >= nt || (int64_t)S.mpos[l] > qp) continue;
        const float sc = acc[qq][i];
        if (isnan(sc)) {
          bad = true;
          continue;
        }
        const unsigned long long key =
            ((unsigned long long)orderable(sc) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(L0 + l));
        if (key > tau) S.buf[q][atomicAdd(&S.cnt[q], 1)] = key;
      }
    }
    __syncthreads();
    const bool last = L0 + kFlatTile >= NL;
    for (int qq = warp * 4; qq < warp * 4 + 4; ++qq)
      if (S.qpos[qq] >= 0 && (S.cnt[qq] > kFlatKeep || (last && S.cnt[qq] > 0))) flat_reduce<R>(S, qq, B);
    __syncthreads();
  }
  if (__syncthreads_or(bad) && tid == 0) set_status(a.status, LSA_ERR_NONFINITE);
  // outputs: kept leaves in order, then their keys
  for (int qq = warp * 4; qq < warp * 4 + 4; ++qq) {
    const int64_t t = t0 + qq;
    if (t >= a.T) continue;
    const int n = S.cnt[qq];
    for (int i = lane; i < B; i += 32) {
      const int32_t leaf = i < n ? key_id(S.buf[qq][i]) : -1;
      S.kept[qq][i] = leaf;
      if (a.leaves_out) a.leaves_out[((int64_t)g * a.T + t) * B + i] = leaf;
    }
    __syncwarp();
    if (a.idx_out) {
      const int leaf = a.leaf;
      const int64_t K_sel = (int64_t)B * leaf;
      const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
      int32_t* out = a.idx_out + ((int64_t)g * a.T + t) * K_sel;
      for (int64_t i = lane; i < K_sel; i += 32) {
        const int k = (int)(i / leaf), q = (int)(i % leaf);
        out[i] = k < n ? __ldg(&li[(int64_t)S.kept[qq][k] * leaf + q]) : -1;
      }
    }
  }
}

template <typename T>
static cudaError_t launch_flat(const SelectArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(a.T, kFlatQ), (unsigned)a.Hkv);
#define LSA_FLAT(RR, DD)                                                                              \
  if (a.r == RR && a.d == DD) {                                                                       \
    const size_t smem = sizeof(FlatSmem<RR>);                                                         \
    cudaError_t e = cudaFuncSetAttribute(k_select_flat<T, RR, DD>,                                    \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
    if (e != cudaSuccess) return e;                                                                   \
    k_select_flat<T, RR, DD><<<grid, kSelWarps * 32, smem, st>>>(a);                                  \
    return cudaGetLastError();                                                                        \
  }
  LSA_FLAT(16, 64) LSA_FLAT(32, 64) LSA_FLAT(64, 64) LSA_FLAT(16, 128) LSA_FLAT(32, 128) LSA_FLAT(64, 128)
#undef LSA_FLAT
  return cudaErrorInvalidValue;
}

cudaError_t run_select_flat(const SelectArgs& a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (select_flat_tc_supported(a, dtype)) return run_select_flat_tc(a, st);
  return dtype == LSA_BF16 ? launch_flat<__nv_bfloat16>(a, st) : launch_flat<float>(a, st);
}

cudaError_t run_select(const SelectArgs& a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  return dtype == LSA_BF16 ? launch_select<__nv_bfloat16>(a, st) : launch_select<float>(a, st);
}

}  // namespace lsa
