// decode.cu -- attention of one decode token over its selected leaves and the
// dense tail, in one launch.
//
// bdtechtalks.com, "Latent sparse attention", section "How latent sparse
// attention works": the query retrieves a fixed number of original keys from the
// clusters whose centroids it chose, and attention runs over them together with
// the recent tokens; kongchang.com, "Latent Sparse Attention Breaks Through the
// Million-Token Context Bottleneck", section "The Accuracy-Efficiency Dilemma":
// decode is memory-bound and latency-sensitive.
//
// Decode has one query token, so the work of a KV group is split over CTAs to
// reach the whole GPU: split s of group g takes 64 keys (a chunk of one kept
// leaf, read through leaf_index, or a chunk of the tail).  A CTA fetches its key
// positions, then all 64 K and V rows at once with 16-byte cp.async into padded
// shared-memory rows (one memory round trip), scores them for the G query heads
// of the group, and writes a partial (max, sum, unnormalised output) per head.
// The CTA that arrives last at the group's counter (atomicAdd after a fence; no
// CTA ever waits for another) merges the group's partials into O and LSE and
// re-arms the counter for the next call.
#include <cmath>

#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tc_sm100.cuh"

namespace lsa {

namespace {

constexpr int kDT = 128;         // threads per CTA
constexpr int kDKeys = 64;       // keys per split
constexpr float kLn2f = 0.69314718055994530942f;

template <typename T, int DK>
struct DecSmem {
  static constexpr int kRowBytes = DK * (int)sizeof(T) + 16;   // padded: rows shift by 16 B mod 128 B
  static constexpr size_t kKV = (size_t)kDKeys * kRowBytes;
  static constexpr size_t kBytes = 2 * kKV;
};

template <int N>
__device__ __forceinline__ void unpack(const uint4& x, const float*, float (&v)[N]) {
  static_assert(N == 4, "");
  v[0] = __uint_as_float(x.x); v[1] = __uint_as_float(x.y); v[2] = __uint_as_float(x.z); v[3] = __uint_as_float(x.w);
}
template <int N>
__device__ __forceinline__ void unpack(const uint4& x, const __nv_bfloat16*, float (&v)[N]) {
  static_assert(N == 8, "");
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(h[q]);
    v[2 * q] = f.x; v[2 * q + 1] = f.y;
  }
}

template <typename T, int DK, int G>
__global__ void __launch_bounds__(kDT) k_dec_attn(DecAttnArgs a) {
  using S = DecSmem<T, DK>;
  constexpr int EPC = 16 / (int)sizeof(T);        // elements per 16-byte chunk
  constexpr int CPR = DK / EPC;                   // chunks per row
  extern __shared__ __align__(16) char smem[];
  char* sK = smem;
  char* sV = smem + S::kKV;
  __shared__ int64_t s_pos[kDKeys];
  __shared__ float s_q[G][DK];
  __shared__ float s_p[G][kDKeys];
  __shared__ float s_m[G], s_l[G];
  __shared__ int s_n, s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, g = blockIdx.y;
  const T* Q = static_cast<const T*>(a.Q);
  const char* Kh = static_cast<const char*>(a.K) + (int64_t)g * a.n_cap * DK * sizeof(T);
  const char* Vh = static_cast<const char*>(a.V) + (int64_t)g * a.n_cap * DK * sizeof(T);

  // key positions of this split
  if (tid < kDKeys) {
    int64_t p = -1;
    const int n_leaf_splits = a.B * a.spl;
    if (s < n_leaf_splits) {
      const int k = s / a.spl, c = s % a.spl;
      const int32_t leaf = __ldg(&a.leaves[(int64_t)g * a.B + k]);
      const int i = c * kDKeys + tid;
      if (leaf >= 0 && i < a.leaf) p = __ldg(&a.leaf_index[(int64_t)g * a.n_tree + (int64_t)leaf * a.leaf + i]);
    } else {
      const int64_t j = a.tail_begin + (int64_t)(s - n_leaf_splits) * kDKeys + tid;
      if (j < a.tail_end) p = j;
    }
    s_pos[tid] = (p >= 0 && p < a.n_cap) ? p : -1;
  }
  for (int x = tid; x < G * DK; x += kDT) {
    const int h = x / DK, dim = x % DK;
    s_q[h][dim] = to_f32(Q[((int64_t)g * G + h) * DK + dim]) * a.scale_log2;
  }
  __syncthreads();
  // all K and V rows of the split in flight at once (absent keys: zero rows)
  for (int x = tid; x < kDKeys * CPR; x += kDT) {
    const int k = x / CPR, c = x % CPR;
    const int64_t p = s_pos[k];
    const uint32_t dk = smem_u32(sK + k * S::kRowBytes + c * 16), dv = smem_u32(sV + k * S::kRowBytes + c * 16);
    if (p >= 0) {
      cp_async16(dk, Kh + (p * DK + c * EPC) * sizeof(T));
      cp_async16(dv, Vh + (p * DK + c * EPC) * sizeof(T));
    } else {
      *reinterpret_cast<uint4*>(sK + k * S::kRowBytes + c * 16) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sV + k * S::kRowBytes + c * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_async_wait_all();
  __syncthreads();
  // scores: thread = (key, heads hg, hg + 2, ...)
  {
    const int k = tid % kDKeys, hg = tid / kDKeys;
    const bool valid = s_pos[k] >= 0;
    for (int h = hg; h < G; h += kDT / kDKeys) {
      float acc = 0.f;
#pragma unroll 4
      for (int c = 0; c < CPR; ++c) {
        float kv[EPC];
        unpack<EPC>(*reinterpret_cast<const uint4*>(sK + k * S::kRowBytes + c * 16), (const T*)nullptr, kv);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc = fmaf(s_q[h][c * EPC + e], kv[e], acc);
      }
      s_p[h][k] = valid ? acc : -INFINITY;
    }
  }
  __syncthreads();
  // per head: max and exp-sum over the 64 keys (one warp per head at a time)
  for (int h = warp; h < G; h += kDT / 32) {
    const float x0 = s_p[h][lane], x1 = s_p[h][lane + 32];
    float m = fmaxf(x0, x1);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float p0 = m == -INFINITY ? 0.f : exp2f(x0 - m), p1 = m == -INFINITY ? 0.f : exp2f(x1 - m);
    s_p[h][lane] = p0;
    s_p[h][lane + 32] = p1;
    float l = p0 + p1;
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) { s_m[h] = m; s_l[h] = l; }
  }
  __syncthreads();
  // unnormalised output of the split: thread = (head, dim) pairs
  float* part = a.part + ((int64_t)g * a.nsplit + s) * G * (DK + 2);
  for (int x = tid; x < G * DK; x += kDT) {
    const int h = x / DK, dim = x % DK;
    float o = 0.f;
    if (s_l[h] > 0.f) {
#pragma unroll 8
      for (int k = 0; k < kDKeys; ++k)
        o = fmaf(s_p[h][k], to_f32(*reinterpret_cast<const T*>(sV + k * S::kRowBytes + dim * sizeof(T))), o);
    }
    part[h * (DK + 2) + dim] = o;
    if (dim == 0) { part[h * (DK + 2) + DK] = s_m[h]; part[h * (DK + 2) + DK + 1] = s_l[h]; }
  }
  // arrival: the last CTA of the group merges every split
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&a.cnt[g], 1) == a.nsplit - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* pg = a.part + (int64_t)g * a.nsplit * G * (DK + 2);
  for (int x = tid; x < G * DK; x += kDT) {
    const int h = x / DK, dim = x % DK;
    float M = -INFINITY;
    for (int q = 0; q < a.nsplit; ++q) {
      const float* pp = pg + ((int64_t)q * G + h) * (DK + 2);
      if (__ldcg(&pp[DK + 1]) > 0.f) M = fmaxf(M, __ldcg(&pp[DK]));
    }
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int q = 0; q < a.nsplit; ++q) {
        const float* pp = pg + ((int64_t)q * G + h) * (DK + 2);
        const float l = __ldcg(&pp[DK + 1]);
        if (l > 0.f) {
          const float f = exp2f(__ldcg(&pp[DK]) - M);
          L = fmaf(l, f, L);
          o = fmaf(__ldcg(&pp[dim]), f, o);
        }
      }
    }
    const int64_t row = (int64_t)g * G + h;
    static_cast<T*>(a.O)[row * DK + dim] = from_f32<T>(L > 0.f ? o / L : 0.f);
    if (dim == 0) a.LSE[row] = L > 0.f ? (M + log2f(L)) * kLn2f : -INFINITY;
  }
  if (tid == 0) a.cnt[g] = 0;   // re-armed for the next call on this workspace
}

template <typename T>
cudaError_t launch_dec(const DecAttnArgs& a, int d, int G, cudaStream_t st) {
  const dim3 grid((unsigned)a.nsplit, (unsigned)a.Hkv);
#define LSA_DEC(DD, GG)                                                                              \
  if (d == DD && G == GG) {                                                                          \
    const size_t smem = DecSmem<T, DD>::kBytes;                                                      \
    cudaError_t e = cudaFuncSetAttribute(k_dec_attn<T, DD, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         (int)smem);                                                 \
    if (e != cudaSuccess) return e;                                                                  \
    k_dec_attn<T, DD, GG><<<grid, kDT, smem, st>>>(a);                                               \
    return cudaGetLastError();                                                                       \
  }
  LSA_DEC(64, 1) LSA_DEC(64, 2) LSA_DEC(64, 4) LSA_DEC(64, 8)
  LSA_DEC(128, 1) LSA_DEC(128, 2) LSA_DEC(128, 4) LSA_DEC(128, 8)
#undef LSA_DEC
  return cudaErrorInvalidValue;
}

}  // namespace

int dec_splits(int B, int leaf, int64_t tail_len) {
  const int spl = (leaf + kDKeys - 1) / kDKeys;
  return B * spl + (int)((tail_len + kDKeys - 1) / kDKeys);
}

cudaError_t run_dec_attn(const DecAttnArgs& a, int dtype, int d, int G, cudaStream_t st) {
  if (a.nsplit <= 0) return cudaSuccess;
  return dtype == LSA_BF16 ? launch_dec<__nv_bfloat16>(a, d, G, st) : launch_dec<float>(a, d, G, st);
}

}  // namespace lsa
