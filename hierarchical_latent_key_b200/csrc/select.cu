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
#include "tc_sm100.cuh"

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
  if constexpr (E >= 4) {
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

// ---- node-major schedule for large batches ------------------------------------
//
// The same search, with the same arithmetic, as k_select, reordered for many
// queries.  At prefill every upper-level node is kept by hundreds of (query,
// group) walks, and a walk-by-walk schedule reads the node's children from L2
// once per walk.  Here every level after the first is one pass over the (walk,
// kept parent) pairs grouped by parent (a counting sort, like the attention's
// leaf lists): consecutive threads score the children of one parent, so those
// centroid rows are read once into L1 and then served from there.  Each score
// goes to the walk's candidate list at the slot the walk-by-walk kernel uses
// (rank of the parent x branching + child), and a warp per walk keeps the best
// beam[l] with the same ranking code.  A score is the fp32 expression of
// level_pass: four sequential FMA chains, chain s over the float4 pieces
// 4 f + s of the row, then (s0 + s1) + (s2 + s3), which is what its lane-group
// butterfly computes; so every kept list equals k_select's bit for bit.
struct NodeSel {
  SelectArgs a;
  float* lat;                 // [Hkv][T][r] latent queries
  int32_t* kept;              // [2][Hkv][T][32] kept node ids by level parity, -1 padded
  int32_t* nkept;             // [Hkv][T] number of real nodes kept at the last ranked level
  int32_t* cnt[2];            // [Hkv][max_par] walks per kept node, by level parity
  int32_t* off;               // [Hkv][max_par + 1] first grouped entry of each parent
  uint32_t* ent;              // [Hkv][T * 32] walk * 32 + rank of the parent, grouped by parent
  int32_t* epar;              // [Hkv][T * 32] the parent of each grouped entry
  unsigned long long* cand;   // [Hkv][T][cstride] candidate keys of the level being ranked
  int64_t max_par, cstride;
};

// Level l's kept nodes of walk (g, t), next[0, valid) in rank order: beam_out;
// then either the lists and parent counts for level l + 1 or, on the last level,
// the outputs (as k_select writes them).  Called by a whole warp.
__device__ __forceinline__ void sn_emit(const NodeSel& s, int l, int g, int64_t t, const int32_t* next, int valid) {
  const SelectArgs& a = s.a;
  const int lane = threadIdx.x & 31;
  if (a.beam_out && lane < a.beam_max)
    a.beam_out[(((int64_t)l * a.Hkv + g) * a.T + t) * a.beam_max + lane] = lane < valid ? next[lane] : -1;
  if (l + 1 < a.levels) {
    s.kept[(((int64_t)(l & 1) * a.Hkv + g) * a.T + t) * LSA_MAX_BEAM + lane] = lane < valid ? next[lane] : -1;
    if (lane == 0) s.nkept[(int64_t)g * a.T + t] = valid;
    if (lane < valid) atomicAdd(&s.cnt[l & 1][(int64_t)g * s.max_par + next[lane]], 1);
    return;
  }
  const int leaf = a.leaf;
  const int B = a.beam[l];
  if (a.leaves_out && lane < B) a.leaves_out[((int64_t)g * a.T + t) * B + lane] = lane < valid ? next[lane] : -1;
  if (a.idx_out) {
    const int64_t K_sel = (int64_t)B * leaf;
    const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
    int32_t* out = a.idx_out + ((int64_t)g * a.T + t) * K_sel;
    for (int64_t i = lane; i < K_sel; i += 32) {
      const int k = (int)(i / leaf), q = (int)(i % leaf);
      out[i] = k < valid ? __ldg(&li[(int64_t)next[k] * leaf + q]) : -1;
    }
  }
}

// Latents of kSnLatQ queries of one group per CTA: W[g] and the group means
// (transposed) in shared memory; a thread computes 4 queries x 4 columns, so two
// 16-byte shared loads feed 16 FMAs.  Per (query, column) the arithmetic is
// latent_query's: group mean summed in head order, kLatParts sequential partial
// sums, combined ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7)).
constexpr int kSnLatQ = 32;
template <typename T, int R, int DK>
__global__ void __launch_bounds__(128) k_sn_latent(NodeSel s) {
  const SelectArgs& a = s.a;
  constexpr int RPP = DK / kLatParts;
  static_assert(kLatParts == 8, "the combine below is written for 8 partial sums");
  __shared__ __align__(16) float s_w[DK * R];
  __shared__ __align__(16) float s_qt[DK][kSnLatQ];
  const int g = blockIdx.y, tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * kSnLatQ;
  const T* Wg = static_cast<const T*>(a.W) + (int64_t)g * DK * R;
  // every load of the two staging loops is independent of the others (4 elements each)
#pragma unroll
  for (int k = 0; k < DK * R / 4 / 128; ++k) {
    const int i = (k * 128 + tid) * 4;
    float v[4];
    load4(Wg + i, v);
    *reinterpret_cast<float4*>(&s_w[i]) = make_float4(v[0], v[1], v[2], v[3]);
  }
  const T* Q = static_cast<const T*>(a.Q);
#pragma unroll
  for (int k = 0; k < kSnLatQ * DK / 4 / 128; ++k) {
    const int i = k * 128 + tid;
    const int q = i % kSnLatQ, j = (i / kSnLatQ) * 4;   // a warp: 32 queries, one j block
    const int64_t t = t0 + q;
    float m[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < a.T) {   // group mean as group_mean: heads summed in order, then / G
      for (int h = 0; h < a.G; ++h) {
        float v[4];
        load4(Q + (t * a.Hq + (int64_t)g * a.G + h) * DK + j, v);
#pragma unroll
        for (int x = 0; x < 4; ++x) m[x] += v[x];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) m[x] = m[x] / (float)a.G;
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) s_qt[j + x][q] = m[x];
  }
  __syncthreads();
  for (int blk = tid; blk < (R / 4) * (kSnLatQ / 4); blk += 128) {
    const int c0 = (blk % (R / 4)) * 4, q0 = (blk / (R / 4)) * 4;
    float lo[4][4], hi[4][4], pr[4][4], cur[4][4];
    for (int p = 0; p < kLatParts; ++p) {
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) cur[x][y] = 0.f;
#pragma unroll 4
      for (int jj = 0; jj < RPP; ++jj) {
        const int j = p * RPP + jj;
        const float4 qv = *reinterpret_cast<const float4*>(&s_qt[j][q0]);
        const float4 wv = *reinterpret_cast<const float4*>(&s_w[j * R + c0]);
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) cur[x][y] = fmaf(qa[x], wa[y], cur[x][y]);
      }
      // pairwise tree: pr = p_even; then (p_even + p_odd) folded into lo / hi
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          if ((p & 1) == 0) {
            pr[x][y] = cur[x][y];
          } else {
            const float pair = pr[x][y] + cur[x][y];
            if (p == 1) lo[x][y] = pair;
            else if (p == 3) lo[x][y] = lo[x][y] + pair;
            else if (p == 5) hi[x][y] = pair;
            else hi[x][y] = hi[x][y] + pair;
          }
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int64_t t = t0 + q0 + x;
      if (t >= a.T) break;
      const float4 v = make_float4(lo[x][0] + hi[x][0], lo[x][1] + hi[x][1], lo[x][2] + hi[x][2],
                                   lo[x][3] + hi[x][3]);
      *reinterpret_cast<float4*>(s.lat + ((int64_t)g * a.T + t) * R + c0) = v;
      if (a.qlat_out) *reinterpret_cast<float4*>(a.qlat_out + (t * a.Hkv + g) * R + c0) = v;
    }
  }
}

// Level 0, one warp per walk (level_pass as in k_select, on the stored latent).
template <int R>
__global__ void __launch_bounds__(kSelWarps * 32) k_sn_top(NodeSel s) {
  using RS = RowSplit<R>;
  const SelectArgs& a = s.a;
  __shared__ unsigned long long s_key[kSelWarps][32 * kSelMaxE];
  __shared__ int32_t s_next[kSelWarps][LSA_MAX_BEAM];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y;
  const int64_t t = (int64_t)blockIdx.x * kSelWarps + warp;
  if (t >= a.T) return;
  const float4* lq = reinterpret_cast<const float4*>(s.lat + ((int64_t)g * a.T + t) * R);
  float4 lat[RS::F];
#pragma unroll
  for (int f = 0; f < RS::F; ++f) lat[f] = lq[f * RS::LPR + lane % RS::LPR];
  const int64_t qpos = a.q_pos ? (int64_t)a.q_pos[t] : (int64_t)LLONG_MAX;
  const bool all_eligible = qpos >= a.n_tree - 1;
  const int ncand = (int)a.nodes[0];
  const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[0]) + (int64_t)g * a.nodes[0] * R;
  const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[0]) + (int64_t)g * a.nodes[0];
  bool bad = false;
  int valid;
#define LSA_LEVEL0(EE) \
  level_pass<R, EE>(a, 0, ncand, cent, mpos, all_eligible, qpos, lat, nullptr, a.branching[0], s_key[warp], s_next[warp], bad)
  if (ncand <= 32) valid = LSA_LEVEL0(1);
  else if (ncand <= 64) valid = LSA_LEVEL0(2);
  else if (ncand <= 128) valid = LSA_LEVEL0(4);
  else if (ncand <= 256) valid = LSA_LEVEL0(8);
  else valid = LSA_LEVEL0(16);
#undef LSA_LEVEL0
  __syncwarp();
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, LSA_ERR_NONFINITE);
  sn_emit(s, 0, g, t, s_next[warp], valid);
}

// Per group: off = exclusive prefix sum of cnt over np parents (off[np] = total),
// cnt reset to 0 (the fill's cursors), and the next level's counts zeroed.
__global__ void __launch_bounds__(1024) k_sn_scan(int32_t* cnt, int32_t* cnt_next, int32_t* off, int64_t max_par,
                                                  int64_t np, int64_t n_next) {
  __shared__ int32_t s_warp[32];
  const int g = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* c = cnt + (int64_t)g * max_par;
  int32_t* o = off + (int64_t)g * (max_par + 1);
  const int64_t per = ceil_div(np, (int64_t)1024);
  const int64_t lo = min64((int64_t)tid * per, np), hi = min64(lo + per, np);
  constexpr int kBlk = 8;   // a block's loads are all issued before the first is used
  int32_t sum = 0;
  for (int64_t b0 = lo; b0 < hi; b0 += kBlk) {
    int32_t v[kBlk];
#pragma unroll
    for (int k = 0; k < kBlk; ++k) v[k] = b0 + k < hi ? c[b0 + k] : 0;
#pragma unroll
    for (int k = 0; k < kBlk; ++k) sum += v[k];
  }
  int32_t inc = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += y;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int32_t w = s_warp[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  int32_t run = inc - sum + (warp ? s_warp[warp - 1] : 0);
  for (int64_t b0 = lo; b0 < hi; b0 += kBlk) {
    int32_t v[kBlk];
#pragma unroll
    for (int k = 0; k < kBlk; ++k) v[k] = b0 + k < hi ? c[b0 + k] : 0;
#pragma unroll
    for (int k = 0; k < kBlk; ++k)
      if (b0 + k < hi) {
        o[b0 + k] = run;
        run += v[k];
        c[b0 + k] = 0;
      }
  }
  if (tid == 1023) o[np] = s_warp[31];
  int32_t* cn = cnt_next + (int64_t)g * max_par;
  for (int64_t i = tid; i < n_next; i += 1024) cn[i] = 0;
}

// (walk, rank) pairs of level l - 1's kept lists grouped by parent: a CTA takes
// kSnFillWalks walks, counts its pairs per parent in shared memory, reserves one
// range per parent it met with a single global atomic, then places its pairs (the
// order inside a parent's range is arbitrary; nothing depends on it).  Above
// kSnFillPar parents every pair reserves its slot with its own atomic.
constexpr int kSnFillWalks = 128;
constexpr int kSnFillPar = 4096;
__global__ void __launch_bounds__(256) k_sn_fill(NodeSel s, int l) {
  const SelectArgs& a = s.a;
  __shared__ int32_t s_h[kSnFillPar];
  const int g = blockIdx.y, tid = threadIdx.x;
  const int Bp = a.beam[l - 1];
  const int64_t np = a.nodes[l - 1];
  const int64_t w0 = (int64_t)blockIdx.x * kSnFillWalks;
  const int64_t nw = min64(kSnFillWalks, a.T - w0);
  const int32_t* kept = s.kept + (((int64_t)((l - 1) & 1) * a.Hkv + g) * a.T + w0) * LSA_MAX_BEAM;
  const int32_t* off = s.off + (int64_t)g * (s.max_par + 1);
  int32_t* cur = s.cnt[(l - 1) & 1] + (int64_t)g * s.max_par;
  uint32_t* ent = s.ent + (int64_t)g * a.T * LSA_MAX_BEAM;
  int32_t* epar = s.epar + (int64_t)g * a.T * LSA_MAX_BEAM;
  const int64_t ne = nw * Bp;
  if (np > kSnFillPar) {
    for (int64_t i = tid; i < ne; i += 256) {
      const int64_t w = i / Bp;
      const int rank = (int)(i % Bp);
      const int32_t p = kept[w * LSA_MAX_BEAM + rank];
      if (p < 0) continue;
      const int64_t pos = off[p] + atomicAdd(&cur[p], 1);
      ent[pos] = (uint32_t)((w0 + w) * LSA_MAX_BEAM + rank);
      epar[pos] = p;
    }
    return;
  }
  // this thread's pairs i = tid + 256 k, their parents read at once and kept in registers
  constexpr int kPer = kSnFillWalks * LSA_MAX_BEAM / 256;
  int32_t pv[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int64_t i = tid + 256 * k;
    pv[k] = i < ne ? kept[(i / Bp) * LSA_MAX_BEAM + i % Bp] : -1;
  }
  for (int64_t p = tid; p < np; p += 256) s_h[p] = 0;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kPer; ++k)
    if (pv[k] >= 0) atomicAdd(&s_h[pv[k]], 1);
  __syncthreads();
  for (int64_t p = tid; p < np; p += 256) {
    const int32_t c = s_h[p];
    s_h[p] = c > 0 ? off[p] + atomicAdd(&cur[p], c) : 0;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int64_t i = tid + 256 * k;
    const int32_t p = pv[k];
    if (p < 0) continue;
    const int32_t pos = atomicAdd(&s_h[p], 1);
    ent[pos] = (uint32_t)((w0 + i / Bp) * LSA_MAX_BEAM + i % Bp);
    epar[pos] = p;
  }
}

// Children j0 + 4 c + jl (c < CPL) of one entry: level_pass's score (four FMA
// chains, chain = float4 piece index mod 4, pieces in order, then (s0 + s1) +
// (s2 + s3)) and key, written to out[j].  An index past b reads child b - 1 and is
// dropped.  Returns whether a score was NaN.
template <int R, int CPL>
__device__ __forceinline__ bool score_children(const float4* q, const float* rows, int stride,
                                               const int32_t* mp, int64_t id0, int b, int j0, int jl,
                                               bool all_eligible, int64_t qpos, unsigned long long* out) {
  const float4* r4[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const int j = min(j0 + 4 * c + jl, b - 1);
    r4[c] = reinterpret_cast<const float4*>(rows + (int64_t)j * stride);
  }
  float acc[CPL][4];
#pragma unroll
  for (int c = 0; c < CPL; ++c)
#pragma unroll
    for (int h = 0; h < 4; ++h) acc[c][h] = 0.f;
#pragma unroll
  for (int k = 0; k < R / 4; ++k) {
    const float4 w = q[k];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const float4 x = r4[c][k];
      float& y = acc[c][k & 3];
      y = fmaf(w.x, x.x, y);
      y = fmaf(w.y, x.y, y);
      y = fmaf(w.z, x.z, y);
      y = fmaf(w.w, x.w, y);
    }
  }
  bool bad = false;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const int j = j0 + 4 * c + jl;
    if (j < b) {
      unsigned long long key = 0ull;
      if (all_eligible || (int64_t)mp[j] <= qpos) {
        const float sc = (acc[c][0] + acc[c][1]) + (acc[c][2] + acc[c][3]);
        if (isnan(sc)) bad = true;
        else key = ((unsigned long long)orderable(sc) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(id0 + j));
      }
      out[j] = key;
    }
  }
  return bad;
}

// Level l: a CTA takes `chunk` consecutive grouped entries; their parents form a
// contiguous id range whose children are contiguous rows of the level, staged in
// shared memory when they fit (they do unless the parents have very few walks
// each).  A warp scores 8 entries at a time, 4 lanes per entry: lane jl takes the
// children jl, jl + 4, ... (CPL = ceil(b / 4) of them, up to 4 at a time), and the
// 4 lanes of an entry store consecutive keys.  The entries' latents reach a
// per-warp double buffer with cp.async (each lane copies a quarter): the next
// group's copies and the entries of the group after it are in flight while the
// current group is scored.
constexpr int kSnChunk = 512;   // entries per CTA at most (the host may pick fewer)
constexpr int kSnRows = 128;    // staged child rows
constexpr int kSnWarps = 4;     // warps per CTA (three CTAs per SM: registers for the whole step, no spills)
template <int R>
struct SnScoreSmem {
  static constexpr int RP = R + 4;   // row stride in floats: the 8 rows a warp reads at once hit different banks
  static constexpr size_t kRows = 0;
  static constexpr size_t kLat = kRows + (size_t)kSnRows * RP * 4;
  static constexpr size_t kMp = kLat + (size_t)kSnWarps * 2 * 8 * RP * 4;
  static constexpr size_t kBytes = kMp + (size_t)kSnRows * 4;
};
template <int R, int CPL>
__global__ void __launch_bounds__(kSnWarps * 32, 3) k_sn_score(NodeSel s, int l, int chunk) {
  using S = SnScoreSmem<R>;
  constexpr int RP = S::RP;
  constexpr int QP = R / 16;  // latent pieces (float4) a lane copies
  const SelectArgs& a = s.a;
  extern __shared__ __align__(16) char sn_smem[];
  float* s_row = reinterpret_cast<float*>(sn_smem + S::kRows);
  int32_t* s_mp = reinterpret_cast<int32_t*>(sn_smem + S::kMp);
  const int g = blockIdx.y, tid = threadIdx.x;
  const int64_t n = s.off[(int64_t)g * (s.max_par + 1) + a.nodes[l - 1]];
  const int64_t e0 = (int64_t)blockIdx.x * chunk;
  if (e0 >= n) return;
  const int64_t e1 = min64(e0 + chunk, n);
  const uint32_t* ent = s.ent + (int64_t)g * a.T * LSA_MAX_BEAM;
  const int32_t* epar = s.epar + (int64_t)g * a.T * LSA_MAX_BEAM;
  const int b = a.branching[l];
  const int64_t pa = epar[e0], pb = epar[e1 - 1];
  const int64_t nrows = (pb - pa + 1) * b;
  const bool staged = nrows <= kSnRows;
  const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[l]) + (int64_t)g * a.nodes[l] * R;
  const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[l]) + (int64_t)g * a.nodes[l];
  if (staged) {   // rows pa*b .. pa*b + nrows - 1, contiguous in the level
    const float4* src = reinterpret_cast<const float4*>(cent + pa * b * R);
    for (int i = tid; i < nrows * (R / 4); i += kSnWarps * 32)
      reinterpret_cast<float4*>(s_row)[(i / (R / 4)) * (RP / 4) + i % (R / 4)] = __ldg(&src[i]);
    for (int i = tid; i < nrows; i += kSnWarps * 32) s_mp[i] = __ldg(&mpos[pa * b + i]);
  }
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5, jl = lane & 3, el = lane >> 2;
  constexpr int kStep = kSnWarps * 8;   // entries per CTA round
  const float* lat = s.lat + (int64_t)g * a.T * R;
  float* wl = reinterpret_cast<float*>(sn_smem + S::kLat) + warp * 2 * 8 * RP;   // [2][8][RP]
  bool bad = false;
  // group k of this warp: entries e0 + (warp + kSnWarps k) * 8 + el
  auto entry_of = [&](int64_t i, int64_t& t, int& rank, int64_t& p) {
    t = -1; rank = 0; p = 0;
    if (i < e1) {
      const uint32_t e = ent[i];
      p = epar[i];
      t = e / LSA_MAX_BEAM;
      rank = (int)(e % LSA_MAX_BEAM);
    }
  };
  // this lane's quarter of walk t's latent into buffer buf, entry slot el
  auto copy_lat = [&](int64_t t, int buf) {
    if (t >= 0) {
#pragma unroll
      for (int k = 0; k < QP; ++k)
        cp_async16(smem_u32(wl + (buf * 8 + el) * RP + (k * 4 + jl) * 4), lat + t * R + (k * 4 + jl) * 4);
    }
    cp_async_commit();
  };
  auto pos_of = [&](int64_t t) { return t >= 0 && a.q_pos ? (int64_t)a.q_pos[t] : (int64_t)LLONG_MAX; };
  int64_t i = e0 + warp * 8 + el;
  int64_t t_c, p_c, t_n, p_n;
  int r_c, r_n;
  entry_of(i, t_c, r_c, p_c);
  copy_lat(t_c, 0);
  int64_t qp_c = pos_of(t_c);
  entry_of(i + kStep, t_n, r_n, p_n);
  for (int buf = 0; i - el < e1; i += kStep, buf ^= 1) {
    // in flight while this group is scored: the next group's latents and position,
    // the entries of the group after it
    copy_lat(t_n, buf ^ 1);
    const int64_t qp_n = pos_of(t_n);
    int64_t t_f, p_f;
    int r_f;
    entry_of(i + 2 * kStep, t_f, r_f, p_f);
    cp_async_wait_prev();   // this lane's copies of the current group have landed
    __syncwarp();
    if (t_c >= 0) {
      const bool all_eligible = qp_c >= a.n_tree - 1;
      unsigned long long* out = s.cand + ((int64_t)g * a.T + t_c) * s.cstride + (int64_t)r_c * b;
      const float4* q = reinterpret_cast<const float4*>(wl + (buf * 8 + el) * RP);
      // two call sites, so that the staged rows are read with shared-memory loads
      if (staged) {
        const int64_t loc = (p_c - pa) * b;
        for (int j0 = 0; j0 < b; j0 += 4 * CPL)
          bad |= score_children<R, CPL>(q, s_row + loc * RP, RP, s_mp + loc, p_c * b, b, j0, jl, all_eligible,
                                        qp_c, out);
      } else {
        for (int j0 = 0; j0 < b; j0 += 4 * CPL)
          bad |= score_children<R, CPL>(q, cent + p_c * b * R, R, mpos + p_c * b, p_c * b, b, j0, jl, all_eligible,
                                        qp_c, out);
      }
    }
    __syncwarp();   // this buffer is refilled two groups later
    t_c = t_n; r_c = r_n; p_c = p_n; qp_c = qp_n;
    t_n = t_f; r_n = r_f; p_n = p_f;
  }
  cp_async_drain();
  if (bad) set_status(a.status, LSA_ERR_NONFINITE);
}

// Level l: one warp per walk keeps the best beam[l] of its candidate list.
template <int E>
__global__ void __launch_bounds__(kSelWarps * 32) k_sn_rank(NodeSel s, int l) {
  const SelectArgs& a = s.a;
  __shared__ unsigned long long s_key[kSelWarps][64];
  __shared__ int32_t s_next[kSelWarps][LSA_MAX_BEAM];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y;
  const int64_t t = (int64_t)blockIdx.x * kSelWarps + warp;
  if (t >= a.T) return;
  const int ncand = s.nkept[(int64_t)g * a.T + t] * a.branching[l];
  const unsigned long long* cl = s.cand + ((int64_t)g * a.T + t) * s.cstride;
  // candidate e * 32 + lane in register e: coalesced loads, and a lane's keys come
  // from different parents, so the threshold of warp_keep_best (the beam-th best of
  // the lanes' two best keys) usually leaves at most 64 keys to sort.  The kept set
  // and its order depend only on the keys, not on where they sit.
  unsigned long long v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = e * 32 + lane;
    v[e] = i < ncand ? cl[i] : 0ull;
  }
  const int valid = warp_keep_best<E>(v, a.beam[l], s_key[warp], s_next[warp]);
  __syncwarp();
  sn_emit(s, l, g, t, s_next[warp], valid);
}

// Workspace regions (256-byte aligned) of the node-major schedule.
struct NodeSelLayout {
  size_t lat, kept, nkept, cnt0, cnt1, off, ent, epar, cand, bytes;
  int64_t max_par, cstride;
};
static NodeSelLayout node_sel_layout(const SelectArgs& a) {
  NodeSelLayout L{};
  L.max_par = 1;
  L.cstride = 1;
  for (int l = 1; l < a.levels; ++l) {
    L.max_par = a.nodes[l - 1] > L.max_par ? a.nodes[l - 1] : L.max_par;
    const int64_t c = (int64_t)a.beam[l - 1] * a.branching[l];
    L.cstride = c > L.cstride ? c : L.cstride;
  }
  const int64_t HT = (int64_t)a.Hkv * a.T;
  size_t o = 0;
  auto take = [&](size_t n) { const size_t r = o; o += (n + 255) & ~(size_t)255; return r; };
  L.lat = take((size_t)HT * a.r * 4);
  L.kept = take((size_t)2 * HT * LSA_MAX_BEAM * 4);
  L.nkept = take((size_t)HT * 4);
  L.cnt0 = take((size_t)a.Hkv * L.max_par * 4);
  L.cnt1 = take((size_t)a.Hkv * L.max_par * 4);
  L.off = take((size_t)a.Hkv * (L.max_par + 1) * 4);
  L.ent = take((size_t)HT * LSA_MAX_BEAM * 4);
  L.epar = take((size_t)HT * LSA_MAX_BEAM * 4);
  L.cand = take((size_t)HT * L.cstride * 8);
  L.bytes = o;
  return L;
}

size_t select_nodes_workspace_bytes(const SelectArgs& a) {
  if (a.levels < 2 || a.T == 0) return 0;
  return node_sel_layout(a).bytes;
}

template <typename T>
static cudaError_t launch_select_nodes(const SelectArgs& a, void* ws, cudaStream_t st) {
  const NodeSelLayout L = node_sel_layout(a);
  char* w = static_cast<char*>(ws);
  NodeSel s;
  s.a = a;
  s.lat = reinterpret_cast<float*>(w + L.lat);
  s.kept = reinterpret_cast<int32_t*>(w + L.kept);
  s.nkept = reinterpret_cast<int32_t*>(w + L.nkept);
  s.cnt[0] = reinterpret_cast<int32_t*>(w + L.cnt0);
  s.cnt[1] = reinterpret_cast<int32_t*>(w + L.cnt1);
  s.off = reinterpret_cast<int32_t*>(w + L.off);
  s.ent = reinterpret_cast<uint32_t*>(w + L.ent);
  s.epar = reinterpret_cast<int32_t*>(w + L.epar);
  s.cand = reinterpret_cast<unsigned long long*>(w + L.cand);
  s.max_par = L.max_par;
  s.cstride = L.cstride;
  cudaError_t e = cudaMemsetAsync(s.cnt[0], 0, (size_t)a.Hkv * L.max_par * 4, st);
  if (e != cudaSuccess) return e;
  const dim3 gw((unsigned)ceil_div(a.T, kSelWarps), (unsigned)a.Hkv);
  const dim3 gl((unsigned)ceil_div(a.T, kSnLatQ), (unsigned)a.Hkv);
  bool launched = false;
#define LSA_SN(RR, DD)                                                   \
  if (a.r == RR && a.d == DD) {                                          \
    k_sn_latent<T, RR, DD><<<gl, 128, 0, st>>>(s);                       \
    k_sn_top<RR><<<gw, kSelWarps * 32, 0, st>>>(s);                      \
    launched = true;                                                     \
  }
  LSA_SN(16, 64) LSA_SN(32, 64) LSA_SN(64, 64) LSA_SN(16, 128) LSA_SN(32, 128) LSA_SN(64, 128)
#undef LSA_SN
  if (!launched) return cudaErrorInvalidValue;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int l = 1; l < a.levels; ++l) {
    const int64_t n_next = l + 1 < a.levels ? a.nodes[l] : 0;
    k_sn_scan<<<(unsigned)a.Hkv, 1024, 0, st>>>(s.cnt[(l - 1) & 1], s.cnt[l & 1], s.off, s.max_par, a.nodes[l - 1],
                                                n_next);
    k_sn_fill<<<dim3((unsigned)ceil_div(a.T, kSnFillWalks), (unsigned)a.Hkv), 256, 0, st>>>(s, l);
    // entries per CTA: the chunk's parents (about chunk / walks-per-parent + 1 of them)
    // should have their children fit the staged rows
    const int64_t per_par = ceil_div(a.T * a.beam[l - 1], a.nodes[l - 1]);
    int chunk = kSnChunk;
    while (chunk > 128 && (chunk / per_par + 2) * a.branching[l] > kSnRows) chunk >>= 1;
    // and enough CTAs for about four waves of three per SM (a last partial wave of
    // one or two leaves most SMs idle)
    const int64_t pairs = a.T * a.beam[l - 1] * a.Hkv;
    while (chunk > 128 && pairs / chunk < 4 * 3 * (int64_t)sm_count()) chunk >>= 1;
    const dim3 gs((unsigned)ceil_div(a.T * a.beam[l - 1], chunk), (unsigned)a.Hkv);
    // children per lane: ceil(b / 4), at most 4 per pass (larger branchings take several)
    const int cpl = (a.branching[l] + 3) / 4;
#define LSA_SNS1(RR, CC)                                                                          \
  {                                                                                               \
    const int sm = (int)SnScoreSmem<RR>::kBytes;                                                  \
    if ((e = cudaFuncSetAttribute(k_sn_score<RR, CC>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                  sm)) != cudaSuccess)                                            \
      return e;                                                                                   \
    k_sn_score<RR, CC><<<gs, kSnWarps * 32, sm, st>>>(s, l, chunk);                               \
  }
#define LSA_SNS(RR)                                     \
  if (a.r == RR) {                                      \
    if (cpl == 1) LSA_SNS1(RR, 1)                       \
    else if (cpl == 2) LSA_SNS1(RR, 2)                  \
    else if (cpl == 3) LSA_SNS1(RR, 3)                  \
    else LSA_SNS1(RR, 4)                                \
  }
    LSA_SNS(16) LSA_SNS(32) LSA_SNS(64)
#undef LSA_SNS
#undef LSA_SNS1
    const int64_t nc = (int64_t)a.beam[l - 1] * a.branching[l];
    if (nc <= 32) k_sn_rank<1><<<gw, kSelWarps * 32, 0, st>>>(s, l);
    else if (nc <= 64) k_sn_rank<2><<<gw, kSelWarps * 32, 0, st>>>(s, l);
    else if (nc <= 128) k_sn_rank<4><<<gw, kSelWarps * 32, 0, st>>>(s, l);
    else if (nc <= 256) k_sn_rank<8><<<gw, kSelWarps * 32, 0, st>>>(s, l);
    else k_sn_rank<16><<<gw, kSelWarps * 32, 0, st>>>(s, l);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t run_select_nodes(const SelectArgs& a, int dtype, void* ws, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (a.levels < 2) return run_select(a, dtype, st);
  return dtype == LSA_BF16 ? launch_select_nodes<__nv_bfloat16>(a, ws, st) : launch_select_nodes<float>(a, ws, st);
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
