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
// One CTA (4 warps) per (query t, KV group g).  Scores are fp32 inner products
// of the group's latent query with fp32 centroids (exact enough that ordering
// decisions only differ from an fp64 evaluation inside a ~1e-6 relative band).
// Candidates are ranked by a packed 64-bit key (orderable score, ~node id) so a
// descending sort gives (score desc, node id asc).  All threads score candidates
// into shared memory, each warp sorts a slice of 128 in registers (bitonic
// network, shuffles across lanes), and one warp sorts the concatenated per-warp
// heads: four CTA barriers per level instead of one per sorting-network stage.

#include <climits>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

constexpr int kSelThreads = 128;   // 4 warps x 128 candidates >= beam * branching (32 * 16)

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

template <int E>
__device__ __forceinline__ int merge_sorted(const unsigned long long* src, int m, int B, int32_t* kept) {
  const int lane = threadIdx.x & 31;
  unsigned long long v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    v[e] = i < m ? src[i] : 0ull;
  }
  warp_sort_desc<E>(v);
  return emit_kept<E>(v, B, kept);
}

template <typename T, int R, int DK>
__global__ void __launch_bounds__(kSelThreads, 4) k_select(SelectArgs a) {
  __shared__ float s_q[DK];
  __shared__ float s_part[kSelThreads];
  __shared__ __align__(16) T s_w[DK * R];
  __shared__ __align__(16) float s_lat[R];
  __shared__ unsigned long long s_cand[(kSelThreads / 32) * 128];
  __shared__ unsigned long long s_merge[(kSelThreads / 32) * LSA_MAX_BEAM];
  __shared__ int32_t s_kept[LSA_MAX_BEAM];
  __shared__ int32_t s_next[LSA_MAX_BEAM];
  __shared__ int s_nkept;
  const int64_t t = blockIdx.x;
  const int g = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* Q = static_cast<const T*>(a.Q);

  // group query: mean of the G query heads of the group
  for (int j = tid; j < DK; j += kSelThreads) {
    float s = 0.f;
    for (int i = 0; i < a.G; ++i) s += to_f32(Q[(t * a.Hq + (int64_t)g * a.G + i) * DK + j]);
    s_q[j] = s / (float)a.G;
  }
  __syncthreads();
  // latent query = group query . W[g]: W[g] is staged in shared memory with
  // 16-byte loads (one memory round trip), then thread (k, part) sums a slice of d
  {
    constexpr int PARTS = kSelThreads / R;
    constexpr int SPAN = DK / PARTS;
    constexpr int VEC = 16 / sizeof(T);
    const T* W = static_cast<const T*>(a.W) + (int64_t)g * DK * R;
#pragma unroll
    for (int i = tid * VEC; i < DK * R; i += kSelThreads * VEC)
      *reinterpret_cast<uint4*>(&s_w[i]) = __ldg(reinterpret_cast<const uint4*>(W + i));
    __syncthreads();
    const int k = tid % R, p = tid / R;
    float acc = 0.f;
#pragma unroll 16
    for (int j = p * SPAN; j < (p + 1) * SPAN; ++j) acc = fmaf(s_q[j], to_f32(s_w[j * R + k]), acc);
    s_part[tid] = acc;
    __syncthreads();
    if (tid < R) {
      float v = 0.f;
      for (int q = 0; q < PARTS; ++q) v += s_part[q * R + tid];
      s_lat[tid] = v;
      if (a.qlat_out) a.qlat_out[(t * a.Hkv + g) * R + tid] = v;
    }
    __syncthreads();
  }
  const int64_t qpos = a.q_pos ? (int64_t)a.q_pos[t] : (int64_t)LLONG_MAX;
  // a query at or past the last indexed position sees every node (decode): no
  // per-node eligibility load is needed
  const bool all_eligible = qpos >= a.n_tree - 1;
  int ncand = (int)a.nodes[0];
  int n_kept = 0;
  for (int l = 0; l < a.levels; ++l) {
    const int b = a.branching[l];
    const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[l]) + (int64_t)g * a.nodes[l] * R;
    const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[l]) + (int64_t)g * a.nodes[l];
    // all threads score (one candidate each per pass) into shared memory; then each
    // warp sorts a slice of 128 candidates (4 per lane) in registers
    const int nw_act = (ncand + 127) / 128;
    constexpr int KW = LSA_MAX_BEAM;                    // per-warp list kept for the merge
    bool bad = false;
    for (int i = tid; i < nw_act * 128; i += kSelThreads) {
      unsigned long long key = 0ull;
      if (i < ncand) {
        const int64_t id = l == 0 ? i : (int64_t)s_kept[i / b] * b + (i % b);
        if (all_eligible || (int64_t)__ldg(&mpos[id]) <= qpos) {
          const float4* cr = reinterpret_cast<const float4*>(cent + id * R);
          float sc = 0.f;
#pragma unroll
          for (int k = 0; k < R / 4; ++k) {
            const float4 c = __ldg(&cr[k]);
            sc = fmaf(s_lat[4 * k], c.x, sc);
            sc = fmaf(s_lat[4 * k + 1], c.y, sc);
            sc = fmaf(s_lat[4 * k + 2], c.z, sc);
            sc = fmaf(s_lat[4 * k + 3], c.w, sc);
          }
          if (isnan(sc)) bad = true;
          else key = ((unsigned long long)orderable(sc) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)id);
        }
      }
      s_cand[i] = key;
    }
    __syncthreads();
    if (warp < nw_act) {
      unsigned long long v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = s_cand[warp * 128 + lane * 4 + e];
      warp_sort_desc<4>(v);
      if (nw_act == 1) {
        const int cnt = emit_kept<4>(v, a.beam[l], s_next);
        if (lane == 0) s_nkept = cnt;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = lane * 4 + e;
          if (i < KW) s_merge[warp * KW + i] = v[e];
        }
      }
    }
    if (bad) set_status(a.status, LSA_ERR_NONFINITE);
    __syncthreads();
    if (nw_act > 1 && warp == 0) {
      const int m = nw_act * KW;
      const int cnt = merge_sorted<4>(s_merge, m, a.beam[l], s_next);   // m <= 4 * 32
      if (lane == 0) s_nkept = cnt;
    }
    __syncthreads();
    const int valid = s_nkept;
    if (tid < LSA_MAX_BEAM) {
      const int32_t id = tid < valid ? s_next[tid] : -1;
      s_kept[tid] = id;
      if (a.beam_out && tid < a.beam_max)
        a.beam_out[(((int64_t)l * a.Hkv + g) * a.T + t) * a.beam_max + tid] = id;
    }
    __syncthreads();
    n_kept = valid;
    ncand = l + 1 < a.levels ? valid * a.branching[l + 1] : 0;
  }
  const int leaf = a.leaf;
  const int B = a.beam[a.levels - 1];
  if (a.leaves_out && tid < B) a.leaves_out[((int64_t)g * a.T + t) * B + tid] = tid < n_kept ? s_kept[tid] : -1;
  if (a.idx_out) {
    const int64_t K_sel = (int64_t)B * leaf;
    const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
    int32_t* out = a.idx_out + ((int64_t)g * a.T + t) * K_sel;
    for (int64_t i = tid; i < K_sel; i += kSelThreads) {
      const int k = (int)(i / leaf), q = (int)(i % leaf);
      out[i] = k < n_kept ? __ldg(&li[(int64_t)s_kept[k] * leaf + q]) : -1;
    }
  }
}

template <typename T>
static cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)a.T, (unsigned)a.Hkv);
#define LSA_SEL(RR, DD)                                                     \
  if (a.r == RR && a.d == DD) {                                             \
    k_select<T, RR, DD><<<grid, kSelThreads, 0, st>>>(a);                   \
    return cudaGetLastError();                                              \
  }
  LSA_SEL(16, 64) LSA_SEL(32, 64) LSA_SEL(64, 64) LSA_SEL(16, 128) LSA_SEL(32, 128) LSA_SEL(64, 128)
#undef LSA_SEL
  return cudaErrorInvalidValue;
}

cudaError_t run_select(const SelectArgs& a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  return dtype == LSA_BF16 ? launch_select<__nv_bfloat16>(a, st) : launch_select<float>(a, st);
}

}  // namespace lsa
