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
  constexpr int kPS = DK + 4;   // floats per partial row: d outputs, max, sum, 2 pad (16-byte rows)
  constexpr int EPC = 16 / (int)sizeof(T);        // elements per 16-byte chunk
  constexpr int CPR = DK / EPC;                   // chunks per row
  extern __shared__ __align__(16) char smem[];
  char* sK = smem;
  char* sV = smem + S::kKV;
  __shared__ int64_t s_pos[kDKeys];
  __shared__ __align__(16) float s_q[G][DK];
  __shared__ float s_p[G][kDKeys];
  __shared__ float s_m[G], s_l[G];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, g = blockIdx.y;
  const T* Q = static_cast<const T*>(a.Q);
  const char* Kh = static_cast<const char*>(a.K) + (int64_t)g * a.n_cap * DK * sizeof(T);
  const char* Vh = static_cast<const char*>(a.V) + (int64_t)g * a.n_cap * DK * sizeof(T);

  // Launched as a programmatic dependent of the select kernel: the query rows are
  // read before waiting for it; the kept leaves, the appended K/V row and the
  // re-armed counter after.
  for (int x = tid; x < G * DK; x += kDT) {
    const int h = x / DK, dim = x % DK;
    s_q[h][dim] = to_f32(Q[((int64_t)g * G + h) * DK + dim]) * a.scale_log2;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  // scores: two threads per key (halves of the row), every head of the group
  {
    const int k = tid >> 1, hh = tid & 1;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 4
    for (int cc = 0; cc < CPR / 2; ++cc) {
      const int c = hh * (CPR / 2) + cc;
      float kv[EPC];
      unpack<EPC>(*reinterpret_cast<const uint4*>(sK + k * S::kRowBytes + c * 16), (const T*)nullptr, kv);
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int e4 = 0; e4 < EPC / 4; ++e4) {
          const float4 q4 = *reinterpret_cast<const float4*>(&s_q[h][c * EPC + 4 * e4]);
          acc[h] = fmaf(q4.x, kv[4 * e4], acc[h]);
          acc[h] = fmaf(q4.y, kv[4 * e4 + 1], acc[h]);
          acc[h] = fmaf(q4.z, kv[4 * e4 + 2], acc[h]);
          acc[h] = fmaf(q4.w, kv[4 * e4 + 3], acc[h]);
        }
      }
    }
    const bool valid = s_pos[k] >= 0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float v = acc[h] + __shfl_xor_sync(0xffffffffu, acc[h], 1);
      if (hh == 0) s_p[h][k] = valid ? v : -INFINITY;
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
  // unnormalised output: thread = (pair of dims, slice of the keys), every head;
  // the key slices are summed through shared memory (the K tile is free now)
  {
    constexpr int DP = DK / 2, KS = kDT / DP, KPS = kDKeys / KS;
    const int dp = tid % DP, ks = tid / DP;
    float o[G][2];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h][0] = o[h][1] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < KPS; ++kk) {
      const int k = ks * KPS + kk;
      float v2[2];
      load2_generic(reinterpret_cast<const T*>(sV + k * S::kRowBytes) + 2 * dp, v2);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pk = s_p[h][k];
        o[h][0] = fmaf(pk, v2[0], o[h][0]);
        o[h][1] = fmaf(pk, v2[1], o[h][1]);
      }
    }
    float* s_red = reinterpret_cast<float*>(sK);      // [KS][G][DK]
#pragma unroll
    for (int h = 0; h < G; ++h) {
      s_red[(ks * G + h) * DK + 2 * dp] = o[h][0];
      s_red[(ks * G + h) * DK + 2 * dp + 1] = o[h][1];
    }
  }
  __syncthreads();
  float* part = a.part + ((int64_t)g * a.nsplit + s) * G * kPS;
  {
    constexpr int KS = kDT / (DK / 2);
    const float* s_red = reinterpret_cast<const float*>(sK);
    for (int x = tid; x < G * DK; x += kDT) {
      const int h = x / DK, dim = x % DK;
      float o = 0.f;
#pragma unroll
      for (int q = 0; q < KS; ++q) o += s_red[(q * G + h) * DK + dim];
      part[h * kPS + dim] = s_l[h] > 0.f ? o : 0.f;
      if (dim == 0) { part[h * kPS + DK] = s_m[h]; part[h * kPS + DK + 1] = s_l[h]; }
    }
  }
  // arrival: the last CTA of the group merges every split
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&a.cnt[g], 1) == a.nsplit - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge: (max, sum) of every (split, head) in one round of loads, per-head weights
  // by one warp per head, then the outputs with every split's partial in flight
  const float* pg = a.part + (int64_t)g * a.nsplit * G * kPS;
  float* s_w = reinterpret_cast<float*>(sK);          // [nsplit][G] (max, then weight; sum)
  for (int x = tid; x < a.nsplit * G; x += kDT) {
    const float* pp = pg + (int64_t)x * kPS;
    const float m = __ldcg(&pp[DK]), l = __ldcg(&pp[DK + 1]);
    s_w[2 * x] = l > 0.f ? m : -INFINITY;
    s_w[2 * x + 1] = l;
  }
  __syncthreads();
  for (int h = warp; h < G; h += kDT / 32) {
    float M = -INFINITY;
    for (int q = lane; q < a.nsplit; q += 32) M = fmaxf(M, s_w[2 * (q * G + h)]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int q = lane; q < a.nsplit; q += 32) {
      const int x = q * G + h;
      const float f = M == -INFINITY || s_w[2 * x + 1] <= 0.f ? 0.f : exp2f(s_w[2 * x] - M);
      L = fmaf(s_w[2 * x + 1], f, L);
      s_w[2 * x] = f;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) { s_m[h] = M; s_l[h] = L; }
  }
  __syncthreads();
  for (int x = tid; x < G * DK / 4; x += kDT) {     // (head, 4 dims)
    const int h = x / (DK / 4), d4 = x % (DK / 4);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q0 = 0; q0 < a.nsplit; q0 += 16) {
      float4 v[16];
#pragma unroll
      for (int qq = 0; qq < 16; ++qq) {
        const int q = q0 + qq;
        v[qq] = q < a.nsplit ? __ldcg(reinterpret_cast<const float4*>(pg + ((int64_t)q * G + h) * kPS) + d4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int qq = 0; qq < 16; ++qq) {
        const int q = q0 + qq;
        const float f = q < a.nsplit ? s_w[2 * (q * G + h)] : 0.f;
        o.x = fmaf(v[qq].x, f, o.x);
        o.y = fmaf(v[qq].y, f, o.y);
        o.z = fmaf(v[qq].z, f, o.z);
        o.w = fmaf(v[qq].w, f, o.w);
      }
    }
    const float L = s_l[h];
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int64_t row = (int64_t)g * G + h;
    T* Or = static_cast<T*>(a.O) + row * DK + 4 * d4;
    Or[0] = from_f32<T>(o.x * inv);
    Or[1] = from_f32<T>(o.y * inv);
    Or[2] = from_f32<T>(o.z * inv);
    Or[3] = from_f32<T>(o.w * inv);
    if (d4 == 0) a.LSE[row] = L > 0.f ? (s_m[h] + log2f(L)) * kLn2f : -INFINITY;
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
    cudaLaunchConfig_t cfg = {};                                                                     \
    cudaLaunchAttribute attr[1];                                                                     \
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;                                 \
    attr[0].val.programmaticStreamSerializationAllowed = 1;                                          \
    cfg.gridDim = grid; cfg.blockDim = dim3(kDT); cfg.dynamicSmemBytes = smem; cfg.stream = st;      \
    cfg.attrs = attr; cfg.numAttrs = 1;                                                              \
    e = cudaLaunchKernelEx(&cfg, k_dec_attn<T, DD, GG>, a);                                          \
    if (e != cudaSuccess) return e;                                                                  \
    return cudaGetLastError();                                                                       \
  }
  LSA_DEC(64, 1) LSA_DEC(64, 2) LSA_DEC(64, 4) LSA_DEC(64, 8)
  LSA_DEC(128, 1) LSA_DEC(128, 2) LSA_DEC(128, 4) LSA_DEC(128, 8)
#undef LSA_DEC
  return cudaErrorInvalidValue;
}

}  // namespace

int dec_max_splits(int dtype, int d, int G) {
  const size_t bytes = dtype == LSA_BF16 ? (d == 64 ? DecSmem<__nv_bfloat16, 64>::kKV : DecSmem<__nv_bfloat16, 128>::kKV)
                                         : (d == 64 ? DecSmem<float, 64>::kKV : DecSmem<float, 128>::kKV);
  return (int)(bytes / (2 * sizeof(float) * G));   // the merge keeps (max, weight) per (split, head) in the K tile
}

int dec_splits(int B, int leaf, int64_t tail_len) {
  const int spl = (leaf + kDKeys - 1) / kDKeys;
  return B * spl + (int)((tail_len + kDKeys - 1) / kDKeys);
}

cudaError_t run_dec_attn(const DecAttnArgs& a, int dtype, int d, int G, cudaStream_t st) {
  if (a.nsplit <= 0) return cudaSuccess;
  return dtype == LSA_BF16 ? launch_dec<__nv_bfloat16>(a, d, G, st) : launch_dec<float>(a, d, G, st);
}

}  // namespace lsa
