// attn.cu -- sparse attention over the selected keys (forward and backward).
//
// Method (kongchang.com, "Latent Sparse Attention Breaks Through the
// Million-Token Context Bottleneck", section "The Accuracy-Efficiency Dilemma":
// each query interacts with only k selected keys; bdtechtalks.com, "Latent
// sparse attention", section "How latent sparse attention works": attention over
// the keys retrieved from the chosen clusters plus a window of recent tokens).
//
// Work unit: one (query t, KV group g); the G query heads of the group share
// the key list, so every gathered K/V row serves G heads.  Inside a CTA each
// warp is split into four 8-lane groups; a group owns one key at a time, each
// lane holding d/8 consecutive elements of the K and V rows (16-byte loads), so
// a group reads a row with fully used sectors and the dot products reduce over
// 8 lanes only.  Every 8-lane group keeps its own online-softmax state (base-2
// exponent, scale folded into the query); states are merged at the end of the
// CTA and, when the keys are split over CTAs (decode), by a combine kernel.

#include <cmath>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kKeysPerIter = kAttnWarps * 4;
constexpr float kLn2 = 0.69314718055994530942f;

template <int N>
__device__ __forceinline__ void load_row(const float* p, float (&v)[N]) {
#pragma unroll
  for (int e = 0; e < N; e += 4) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p + e));
    v[e] = x.x; v[e + 1] = x.y; v[e + 2] = x.z; v[e + 3] = x.w;
  }
}
template <int N>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&v)[N]) {
#pragma unroll
  for (int e = 0; e < N; e += 8) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(p + e));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h[q]);
      v[e + 2 * q] = f.x; v[e + 2 * q + 1] = f.y;
    }
  }
}

__device__ __forceinline__ float group8_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;
}

// Key number i of a unit: the selected list first, then the dense tail.
__device__ __forceinline__ int64_t unit_key(const AttnArgs& a, const int32_t* ix, int64_t i) {
  return i < a.K_sel ? (int64_t)__ldg(&ix[i]) : a.tail_begin + (i - a.K_sel);
}

template <typename T, int DK, int G>
__global__ void __launch_bounds__(kAttnThreads) k_attn_fwd(AttnArgs a) {
  constexpr int EPL = DK / 8;
  __shared__ float s_m[kAttnWarps][G], s_l[kAttnWarps][G];
  __shared__ float s_acc[kAttnWarps][G][DK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane >> 3, sl = lane & 7;
  const int64_t t = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int g = blockIdx.y;
  const T* Q = static_cast<const T*>(a.Q);
  const T* Kh = static_cast<const T*>(a.K) + (int64_t)g * a.n_cap * DK;
  const T* Vh = static_cast<const T*>(a.V) + (int64_t)g * a.n_cap * DK;
  const int32_t* ix = a.idx ? a.idx + ((int64_t)g * a.T + t) * a.K_sel : nullptr;
  const int64_t nkeys = a.K_sel + (a.tail_end - a.tail_begin);
  const int64_t k_begin = (int64_t)split * a.keys_per_split;
  const int64_t k_end = min64(nkeys, k_begin + a.keys_per_split);
  const int64_t qpos = a.causal ? (int64_t)a.q_pos[t] : INT64_MAX;

  float q[G][EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    load_row<EPL>(Q + (t * a.Hq + (int64_t)g * G + h) * DK + sl * EPL, q[h]);
#pragma unroll
    for (int e = 0; e < EPL; ++e) q[h][e] *= a.scale_log2;
  }
  float m[G], l[G], acc[G][EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[h][e] = 0.f;
  }
  for (int64_t base = k_begin + warp * 4; base < k_end; base += kKeysPerIter) {
    const int64_t i = base + sub;
    const int64_t j = i < k_end ? unit_key(a, ix, i) : -1;
    const bool ok = j >= 0 && j < a.n_cap && j <= qpos;
    float kv[EPL], vv[EPL];
    if (ok) {
      load_row<EPL>(Kh + j * DK + sl * EPL, kv);
      load_row<EPL>(Vh + j * DK + sl * EPL, vv);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) { kv[e] = 0.f; vv[e] = 0.f; }
    }
    float s[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float x = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) x = fmaf(q[h][e], kv[e], x);
      s[h] = group8_sum(x);
    }
    if (ok) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mn = fmaxf(m[h], s[h]);
        const float corr = exp2f(m[h] - mn);
        const float p = exp2f(s[h] - mn);
        l[h] = l[h] * corr + p;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[h][e] = fmaf(p, vv[e], acc[h][e] * corr);
        m[h] = mn;
      }
    }
  }
  // merge the four 8-lane groups of the warp
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = m[h];
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 8));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
    const float f = M == -INFINITY ? 0.f : exp2f(m[h] - M);
    float L = l[h] * f;
    L += __shfl_xor_sync(0xffffffffu, L, 8);
    L += __shfl_xor_sync(0xffffffffu, L, 16);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float v = acc[h][e] * f;
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[h][e] = v;
    }
    if (lane == 0) { s_m[warp][h] = M; s_l[warp][h] = L; }
    if (sub == 0) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) s_acc[warp][h][sl * EPL + e] = acc[h][e];
    }
  }
  __syncthreads();
  // merge warps; thread handles (head, dim) pairs
  for (int x = threadIdx.x; x < G * DK; x += kAttnThreads) {
    const int h = x / DK, dim = x % DK;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][h]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float f = exp2f(s_m[w][h] - M);
        L += s_l[w][h] * f;
        o += s_acc[w][h][dim] * f;
      }
    }
    const int64_t row = t * a.Hq + (int64_t)g * G + h;
    if (a.nsplit == 1) {
      T* O = static_cast<T*>(a.O);
      O[row * DK + dim] = from_f32<T>(L > 0.f ? o / L : 0.f);
      if (dim == 0) a.LSE[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    } else {
      float* p = a.part + (row * a.nsplit + split) * (DK + 2);
      p[dim] = o;
      if (dim == 0) { p[DK] = M; p[DK + 1] = L; }
    }
  }
}

template <typename T, int DK>
__global__ void k_attn_combine(AttnArgs a) {
  const int64_t row = blockIdx.x;  // t * Hq + head
  const int dim = threadIdx.x;
  const float* p = a.part + row * a.nsplit * (DK + 2);
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, p[s * (DK + 2) + DK]);
  float L = 0.f, o = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.nsplit; ++s) {
      const float f = exp2f(p[s * (DK + 2) + DK] - M);
      L += p[s * (DK + 2) + DK + 1] * f;
      o += p[s * (DK + 2) + dim] * f;
    }
  }
  T* O = static_cast<T*>(a.O);
  O[row * DK + dim] = from_f32<T>(L > 0.f ? o / L : 0.f);
  if (dim == 0) a.LSE[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  atomicAdd(reinterpret_cast<float4*>(p), make_float4(a, b, c, d));
}

template <typename T, int DK, int G>
__global__ void __launch_bounds__(kAttnThreads) k_attn_bwd(AttnArgs a) {
  constexpr int EPL = DK / 8;
  __shared__ float s_dq[kAttnWarps][G][DK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane >> 3, sl = lane & 7;
  const int64_t t = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int g = blockIdx.y;
  const T* Q = static_cast<const T*>(a.Q);
  const T* O = static_cast<const T*>(a.O);
  const T* dO = static_cast<const T*>(a.dO);
  const T* Kh = static_cast<const T*>(a.K) + (int64_t)g * a.n_cap * DK;
  const T* Vh = static_cast<const T*>(a.V) + (int64_t)g * a.n_cap * DK;
  float* dKh = a.dK + (int64_t)g * a.n_cap * DK;
  float* dVh = a.dV + (int64_t)g * a.n_cap * DK;
  const int32_t* ix = a.idx ? a.idx + ((int64_t)g * a.T + t) * a.K_sel : nullptr;
  const int64_t nkeys = a.K_sel + (a.tail_end - a.tail_begin);
  const int64_t k_begin = (int64_t)split * a.keys_per_split;
  const int64_t k_end = min64(nkeys, k_begin + a.keys_per_split);
  const int64_t qpos = a.causal ? (int64_t)a.q_pos[t] : INT64_MAX;
  constexpr float kLog2e = 1.44269504088896340736f;

  float q[G][EPL], go[G][EPL], lse2[G], delta[G], dq[G][EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const int64_t row = t * a.Hq + (int64_t)g * G + h;
    load_row<EPL>(Q + row * DK + sl * EPL, q[h]);
    load_row<EPL>(dO + row * DK + sl * EPL, go[h]);
    float ov[EPL];
    load_row<EPL>(O + row * DK + sl * EPL, ov);
    float x = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) x = fmaf(go[h][e], ov[e], x);
    delta[h] = group8_sum(x);
    lse2[h] = a.LSE[row] * kLog2e;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dq[h][e] = 0.f;
  }
  for (int64_t base = k_begin + warp * 4; base < k_end; base += kKeysPerIter) {
    const int64_t i = base + sub;
    const int64_t j = i < k_end ? unit_key(a, ix, i) : -1;
    const bool ok = j >= 0 && j < a.n_cap && j <= qpos;
    float kv[EPL], vv[EPL];
    if (ok) {
      load_row<EPL>(Kh + j * DK + sl * EPL, kv);
      load_row<EPL>(Vh + j * DK + sl * EPL, vv);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) { kv[e] = 0.f; vv[e] = 0.f; }
    }
    float p[G], ds[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        x = fmaf(q[h][e], kv[e], x);
        y = fmaf(go[h][e], vv[e], y);
      }
      x = group8_sum(x);
      y = group8_sum(y);
      p[h] = ok ? exp2f(x * a.scale_log2 - lse2[h]) : 0.f;
      ds[h] = p[h] * (y - delta[h]);
#pragma unroll
      for (int e = 0; e < EPL; ++e) dq[h][e] = fmaf(ds[h], kv[e], dq[h][e]);
    }
    if (ok) {
#pragma unroll
      for (int e = 0; e < EPL; e += 4) {
        float gk[4], gv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float xk = 0.f, xv = 0.f;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            xk = fmaf(ds[h], q[h][e + c], xk);
            xv = fmaf(p[h], go[h][e + c], xv);
          }
          gk[c] = xk * a.scale;
          gv[c] = xv;
        }
        red_add4(dKh + j * DK + sl * EPL + e, gk[0], gk[1], gk[2], gk[3]);
        red_add4(dVh + j * DK + sl * EPL + e, gv[0], gv[1], gv[2], gv[3]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float v = dq[h][e];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      if (sub == 0) s_dq[warp][h][sl * EPL + e] = v;
    }
  __syncthreads();
  for (int x = threadIdx.x; x < G * DK; x += kAttnThreads) {
    const int h = x / DK, dim = x % DK;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) v += s_dq[w][h][dim];
    v *= a.scale;
    const int64_t row = t * a.Hq + (int64_t)g * G + h;
    if (a.nsplit == 1) a.dQ[row * DK + dim] = v;
    else atomicAdd(&a.dQ[row * DK + dim], v);
  }
}

int attn_splits(int64_t T, int Hkv, int64_t keys) {
  const int64_t units = T * Hkv;
  const int64_t target = 4 * 148;
  if (units >= target || keys <= 64) return 1;
  int64_t s = (target + units - 1) / units;
  const int64_t max_s = (keys + 63) / 64;
  return (int)(s < max_s ? s : max_s);
}

template <typename T>
static cudaError_t launch_fwd(const AttnArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)(a.T * a.nsplit), (unsigned)a.Hkv);
#define LSA_FWD(DD, GG)                                                               \
  if (a.d == DD && a.G == GG) {                                                       \
    k_attn_fwd<T, DD, GG><<<grid, kAttnThreads, 0, st>>>(a);                          \
    if (a.nsplit > 1) k_attn_combine<T, DD><<<(unsigned)(a.T * a.Hq), DD, 0, st>>>(a); \
    return cudaGetLastError();                                                        \
  }
  LSA_FWD(64, 1) LSA_FWD(64, 2) LSA_FWD(64, 4) LSA_FWD(64, 8)
  LSA_FWD(128, 1) LSA_FWD(128, 2) LSA_FWD(128, 4) LSA_FWD(128, 8)
#undef LSA_FWD
  return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t launch_bwd(const AttnArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)(a.T * a.nsplit), (unsigned)a.Hkv);
#define LSA_BWD(DD, GG)                                            \
  if (a.d == DD && a.G == GG) {                                    \
    k_attn_bwd<T, DD, GG><<<grid, kAttnThreads, 0, st>>>(a);       \
    return cudaGetLastError();                                     \
  }
  LSA_BWD(64, 1) LSA_BWD(64, 2) LSA_BWD(64, 4) LSA_BWD(64, 8)
  LSA_BWD(128, 1) LSA_BWD(128, 2) LSA_BWD(128, 4) LSA_BWD(128, 8)
#undef LSA_BWD
  return cudaErrorInvalidValue;
}

cudaError_t run_attn_fwd(const AttnArgs& a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  return dtype == LSA_BF16 ? launch_fwd<__nv_bfloat16>(a, st) : launch_fwd<float>(a, st);
}

cudaError_t run_attn_bwd(const AttnArgs& a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  return dtype == LSA_BF16 ? launch_bwd<__nv_bfloat16>(a, st) : launch_bwd<float>(a, st);
}

}  // namespace lsa
