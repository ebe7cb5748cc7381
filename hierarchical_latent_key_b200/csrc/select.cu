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
// One CTA per (query t, KV group g).  Scores are fp32 inner products of the
// group's latent query with fp32 centroids (exact enough that ordering
// decisions only differ from an fp64 evaluation inside a ~1e-6 relative band).
// Candidates are ranked by a packed 64-bit key (orderable score, ~node id) so
// one descending sort gives (score desc, node id asc).

#include <climits>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

constexpr int kSelThreads = 256;
constexpr int kMaxCand = LSA_MAX_BEAM * LSA_MAX_BRANCHING;

__device__ __forceinline__ void bitonic_desc(unsigned long long* s, int npad) {
  for (int k = 2; k <= npad; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < npad; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const unsigned long long x = s[i], y = s[p];
          const bool desc = (i & k) == 0;
          if (desc ? (x < y) : (x > y)) { s[i] = y; s[p] = x; }
        }
      }
      __syncthreads();
    }
  }
}

template <typename T, int R, int DK>
__global__ void __launch_bounds__(kSelThreads) k_select(SelectArgs a) {
  __shared__ float s_q[DK];
  __shared__ float s_part[kSelThreads];
  __shared__ __align__(16) float s_lat[R];
  __shared__ unsigned long long s_key[kMaxCand];
  __shared__ int32_t s_kept[LSA_MAX_BEAM];
  const int64_t t = blockIdx.x;
  const int g = blockIdx.y, tid = threadIdx.x;
  const T* Q = static_cast<const T*>(a.Q);

  // group query: mean of the G query heads of the group
  for (int j = tid; j < DK; j += kSelThreads) {
    float s = 0.f;
    for (int i = 0; i < a.G; ++i) s += to_f32(Q[(t * a.Hq + (int64_t)g * a.G + i) * DK + j]);
    s_q[j] = s / (float)a.G;
  }
  __syncthreads();
  // latent query = group query . W[g]; thread (k, part) sums a slice of d
  {
    constexpr int PARTS = kSelThreads / R;
    constexpr int SPAN = DK / PARTS;
    const int k = tid % R, p = tid / R;
    const T* W = static_cast<const T*>(a.W) + (int64_t)g * DK * R;
    float acc = 0.f;
    for (int j = p * SPAN; j < (p + 1) * SPAN; ++j) acc = fmaf(s_q[j], to_f32(W[j * R + k]), acc);
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
  int ncand = (int)a.nodes[0];
  int n_kept = 0;
  for (int l = 0; l < a.levels; ++l) {
    const int b = a.branching[l];
    int npad = 2;
    while (npad < ncand) npad <<= 1;
    const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[l]) + (int64_t)g * a.nodes[l] * R;
    const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[l]) + (int64_t)g * a.nodes[l];
    bool bad = false;
    for (int i = tid; i < npad; i += kSelThreads) {
      unsigned long long key = 0ull;
      if (i < ncand) {
        const int64_t id = l == 0 ? i : (int64_t)s_kept[i / b] * b + (i % b);
        if ((int64_t)__ldg(&mpos[id]) <= qpos) {
          const float4* cr = reinterpret_cast<const float4*>(cent + id * R);
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < R / 4; ++k) {
            const float4 c = __ldg(&cr[k]);
            s = fmaf(s_lat[4 * k], c.x, s);
            s = fmaf(s_lat[4 * k + 1], c.y, s);
            s = fmaf(s_lat[4 * k + 2], c.z, s);
            s = fmaf(s_lat[4 * k + 3], c.w, s);
          }
          if (isnan(s)) bad = true;
          else key = ((unsigned long long)orderable(s) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)id);
        }
      }
      s_key[i] = key;
    }
    if (bad) set_status(a.status, LSA_ERR_NONFINITE);
    __syncthreads();
    bitonic_desc(s_key, npad);
    const int B = a.beam[l];
    const int valid = __syncthreads_count(tid < B && tid < npad && s_key[tid] != 0ull);
    if (tid < LSA_MAX_BEAM) {
      const bool ok = tid < valid;
      const int32_t id = ok ? (int32_t)(0xffffffffu - (uint32_t)(s_key[tid] & 0xffffffffull)) : -1;
      s_kept[tid] = id;
      if (a.beam_out && tid < a.beam_max)
        a.beam_out[(((int64_t)l * a.Hkv + g) * a.T + t) * a.beam_max + tid] = id;
    }
    n_kept = valid;
    ncand = l + 1 < a.levels ? valid * a.branching[l + 1] : 0;
    __syncthreads();
  }
  const int leaf = a.leaf;
  const int64_t K_sel = (int64_t)a.beam[a.levels - 1] * leaf;
  const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
  int32_t* out = a.idx_out + ((int64_t)g * a.T + t) * K_sel;
  for (int64_t i = tid; i < K_sel; i += kSelThreads) {
    const int k = (int)(i / leaf), q = (int)(i % leaf);
    out[i] = k < n_kept ? __ldg(&li[(int64_t)s_kept[k] * leaf + q]) : -1;
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
