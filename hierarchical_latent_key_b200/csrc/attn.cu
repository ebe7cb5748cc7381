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
// warp is split into groups of LPK = d/8 lanes; a group owns one key at a time,
// each lane holding 8 consecutive elements of the K and V rows (16-byte loads for
// bf16), so a group reads a row with fully used sectors and the dot products
// reduce over the group only.  Every group keeps its own online-softmax state
// (base-2 exponent, scale folded into the query); states are merged at the end
// of the CTA and, when the keys are split over CTAs (decode), by a combine kernel.

#include <cmath>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
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

// Sum over the LPK lanes that share a key (xor offsets stay inside the group).
template <int LPK>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = LPK / 2; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Key number i of a unit: the selected list first, then the dense tail.
__device__ __forceinline__ int64_t unit_key(const AttnArgs& a, const int32_t* ix, int64_t i) {
  return i < a.K_sel ? (int64_t)__ldg(&ix[i]) : a.tail_begin + (i - a.K_sel);
}

// Fetch K and V slices of the key at virtual position i of the unit (zeros and
// ok = false when the key is absent, out of range or in the causal future).
template <typename T, int EPL>
__device__ __forceinline__ bool fetch_kv(const AttnArgs& a, const int32_t* ix, const T* Kh, const T* Vh,
                                         int64_t i, int64_t k_end, int64_t qpos, int off,
                                         float (&kv)[EPL], float (&vv)[EPL]) {
  const int64_t j = i < k_end ? unit_key(a, ix, i) : -1;
  const bool ok = j >= 0 && j < a.n_cap && j <= qpos;
  if (ok) {
    load_row<EPL>(Kh + j * a.d + off, kv);
    load_row<EPL>(Vh + j * a.d + off, vv);
  } else {
#pragma unroll
    for (int e = 0; e < EPL; ++e) { kv[e] = 0.f; vv[e] = 0.f; }
  }
  return ok;
}

// LPK lanes own one key at a time (EPL = d / LPK elements each); a warp holds
// 32 / LPK keys per step, and the next step's rows are loaded before the current
// ones are used, so two rows per lane group are in flight.
template <typename T, int DK, int G, int LPK>
__global__ void __launch_bounds__(kAttnThreads) k_attn_fwd(AttnArgs a) {
  constexpr int EPL = DK / LPK;
  constexpr int KPW = 32 / LPK;                 // keys per warp per step
  constexpr int KPI = KPW * kAttnWarps;         // keys per CTA per step
  __shared__ float s_m[kAttnWarps][G], s_l[kAttnWarps][G];
  __shared__ float s_acc[kAttnWarps][G][DK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane / LPK, sl = lane % LPK;
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
  const int off = sl * EPL;

  float q[G][EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    load_row<EPL>(Q + (t * a.Hq + (int64_t)g * G + h) * DK + off, q[h]);
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
  int64_t base = k_begin + warp * KPW;
  float kv[EPL], vv[EPL];
  bool ok = fetch_kv<T, EPL>(a, ix, Kh, Vh, base + sub, k_end, qpos, off, kv, vv);
  for (; base < k_end; base += KPI) {
    float kn[EPL], vn[EPL];
    const bool okn = fetch_kv<T, EPL>(a, ix, Kh, Vh, base + KPI + sub, k_end, qpos, off, kn, vn);
    float s[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float x = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) x = fmaf(q[h][e], kv[e], x);
      s[h] = group_sum<LPK>(x);
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
#pragma unroll
    for (int e = 0; e < EPL; ++e) { kv[e] = kn[e]; vv[e] = vn[e]; }
    ok = okn;
  }
  // merge the key groups of the warp
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = m[h];
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = M == -INFINITY ? 0.f : exp2f(m[h] - M);
    float L = l[h] * f;
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float v = acc[h][e] * f;
#pragma unroll
      for (int o = LPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[h][e] = v;
    }
    if (lane == 0) { s_m[warp][h] = M; s_l[warp][h] = L; }
    if (sub == 0) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) s_acc[warp][h][off + e] = acc[h][e];
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

// Merge the split partials of one (query, head) row: the splits' maxima and sums
// are read by one thread each, the d outputs by one thread each with all split
// loads issued together.
template <typename T, int DK>
__global__ void __launch_bounds__(DK) k_attn_combine(AttnArgs a) {
  __shared__ float s_f[1024];
  __shared__ float s_M, s_L;
  const int64_t row = blockIdx.x;  // t * Hq + head
  const int dim = threadIdx.x;
  const int ns = a.nsplit;
  const float* p = a.part + row * ns * (DK + 2);
  float m = -INFINITY;
  for (int s = dim; s < ns; s += DK) m = fmaxf(m, p[s * (DK + 2) + DK]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((dim & 31) == 0) s_f[dim >> 5] = m;
  __syncthreads();
  if (dim == 0) {
    float M = -INFINITY;
    for (int w = 0; w < DK / 32; ++w) M = fmaxf(M, s_f[w]);
    s_M = M;
  }
  __syncthreads();
  const float M = s_M;
  float l = 0.f;
  for (int s = dim; s < ns; s += DK) {
    const float f = M == -INFINITY ? 0.f : exp2f(p[s * (DK + 2) + DK] - M);
    s_f[32 + s] = f;
    l += p[s * (DK + 2) + DK + 1] * f;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  __syncthreads();
  if ((dim & 31) == 0) s_f[dim >> 5] = l;
  __syncthreads();
  if (dim == 0) {
    float L = 0.f;
    for (int w = 0; w < DK / 32; ++w) L += s_f[w];
    s_L = L;
  }
  __syncthreads();
  const float L = s_L;
  float o = 0.f;
#pragma unroll 8
  for (int s = 0; s < ns; ++s) o += p[s * (DK + 2) + dim] * s_f[32 + s];
  T* O = static_cast<T*>(a.O);
  O[row * DK + dim] = from_f32<T>(L > 0.f ? o / L : 0.f);
  if (dim == 0) a.LSE[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  atomicAdd(reinterpret_cast<float4*>(p), make_float4(a, b, c, d));
}

template <typename T, int DK, int G, int LPK>
__global__ void __launch_bounds__(kAttnThreads) k_attn_bwd(AttnArgs a) {
  constexpr int EPL = DK / LPK;
  constexpr int KPW = 32 / LPK;
  constexpr int KPI = KPW * kAttnWarps;
  __shared__ float s_dq[kAttnWarps][G][DK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane / LPK, sl = lane % LPK;
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
  const int off = sl * EPL;
  constexpr float kLog2e = 1.44269504088896340736f;

  float q[G][EPL], go[G][EPL], lse2[G], delta[G], dq[G][EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const int64_t row = t * a.Hq + (int64_t)g * G + h;
    load_row<EPL>(Q + row * DK + off, q[h]);
    load_row<EPL>(dO + row * DK + off, go[h]);
    float ov[EPL];
    load_row<EPL>(O + row * DK + off, ov);
    float x = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) x = fmaf(go[h][e], ov[e], x);
    delta[h] = group_sum<LPK>(x);
    lse2[h] = a.LSE[row] * kLog2e;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dq[h][e] = 0.f;
  }
  for (int64_t base = k_begin + warp * KPW; base < k_end; base += KPI) {
    const int64_t i = base + sub;
    const int64_t j = i < k_end ? unit_key(a, ix, i) : -1;
    float kv[EPL], vv[EPL];
    const bool ok = fetch_kv<T, EPL>(a, ix, Kh, Vh, i, k_end, qpos, off, kv, vv);
    float p[G], ds[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        x = fmaf(q[h][e], kv[e], x);
        y = fmaf(go[h][e], vv[e], y);
      }
      x = group_sum<LPK>(x);
      y = group_sum<LPK>(y);
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
        red_add4(dKh + j * DK + off + e, gk[0], gk[1], gk[2], gk[3]);
        red_add4(dVh + j * DK + off + e, gv[0], gv[1], gv[2], gv[3]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float v = dq[h][e];
#pragma unroll
      for (int o = LPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (sub == 0) s_dq[warp][h][off + e] = v;
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

// one 16-byte chunk per thread: rows of every head for K, then for V
__global__ void k_kv_append(char* K, char* V, int64_t n_cap, int64_t row_bytes, int64_t pos, const char* Kr,
                            const char* Vr, int64_t n_heads) {
  const int64_t chunks = row_bytes / 16;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * n_heads * chunks) return;
  const int64_t which = i / (n_heads * chunks), rem = i % (n_heads * chunks);
  const int64_t h = rem / chunks, c = rem % chunks;
  char* dst = (which ? V : K) + (h * n_cap + pos) * row_bytes + c * 16;
  const char* src = (which ? Vr : Kr) + h * row_bytes + c * 16;
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
}

cudaError_t run_kv_append(void* K, void* V, int64_t n_heads, int64_t n_cap, int64_t row_bytes, int64_t pos,
                          const void* Kr, const void* Vr, cudaStream_t st) {
  const int64_t n = 2 * n_heads * (row_bytes / 16);
  k_kv_append<<<(unsigned)ceil_div(n, 256), 256, 0, st>>>(static_cast<char*>(K), static_cast<char*>(V), n_cap,
                                                          row_bytes, pos, static_cast<const char*>(Kr),
                                                          static_cast<const char*>(Vr), n_heads);
  return cudaGetLastError();
}

// Key lists with the sink and recent-window keys (bdtechtalks.com, "Latent sparse
// attention", section "How latent sparse attention works": the keys taken from the
// chosen clusters are used together with a window of recent tokens and a few
// initial sink tokens).  Row (g, t) of idx2 = the K_sel listed keys, then n_sink
// sink slots, then `window` window slots; a position that the tail range attends
// already, or that the sink or the window holds, is dropped from the earlier parts,
// so every key of the union appears once (the sink wins over the window, the tail
// over both).  Positions past q_pos are left to the attention's causal mask.
__global__ void k_attn_extend(const int32_t* __restrict__ idx, int32_t K_sel, int64_t T, const int32_t* __restrict__ q_pos,
                              int32_t n_sink, int32_t window, int64_t tail_begin, int64_t tail_end, int64_t n_cap,
                              int32_t* __restrict__ idx2, int32_t K2) {
  const int64_t g = blockIdx.y, t = blockIdx.x;
  const int64_t q = q_pos[t];
  const int64_t w_lo = q - window + 1;
  auto in_tail = [&](int64_t j) { return j >= tail_begin && j < tail_end; };
  const int32_t* src = idx + (g * T + t) * K_sel;
  int32_t* dst = idx2 + (g * T + t) * K2;
  for (int i = threadIdx.x; i < K2; i += blockDim.x) {
    int64_t out = -1;
    if (i < K_sel) {
      const int64_t j = src[i];
      if (j >= 0 && !(j < n_sink || (j >= w_lo && j <= q) || in_tail(j))) out = j;
    } else if (i < K_sel + n_sink) {
      const int64_t j = i - K_sel;
      if (j <= q && j < n_cap && !in_tail(j)) out = j;
    } else {
      const int64_t j = w_lo + (i - K_sel - n_sink);
      if (j >= n_sink && j >= 0 && j <= q && j < n_cap && !in_tail(j)) out = j;
    }
    dst[i] = (int32_t)out;
  }
}

cudaError_t run_attn_extend(const int32_t* idx, int32_t K_sel, int64_t T, int32_t n_heads, const int32_t* q_pos,
                            int32_t n_sink, int32_t window, int64_t tail_begin, int64_t tail_end, int64_t n_cap,
                            int32_t* idx2, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  k_attn_extend<<<dim3((unsigned)T, (unsigned)n_heads), 256, 0, st>>>(idx, K_sel, T, q_pos, n_sink, window, tail_begin,
                                                                      tail_end, n_cap, idx2, K_sel + n_sink + window);
  return cudaGetLastError();
}

int attn_splits(int64_t T, int Hkv, int64_t keys) {
  const int64_t units = T * Hkv;
  const int64_t target = 4 * 148;
  if (units <= 0 || units >= target || keys <= 64) return 1;
  int64_t s = (target + units - 1) / units;
  const int64_t max_s = (keys + 63) / 64;
  return (int)(s < max_s ? s : max_s);
}

template <typename T>
static cudaError_t launch_fwd(const AttnArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)(a.T * a.nsplit), (unsigned)a.Hkv);
#define LSA_FWD(DD, GG)                                                               \
  if (a.d == DD && a.G == GG) {                                                       \
    k_attn_fwd<T, DD, GG, DD / 8><<<grid, kAttnThreads, 0, st>>>(a);                  \
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
    k_attn_bwd<T, DD, GG, DD / 8><<<grid, kAttnThreads, 0, st>>>(a); \
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
