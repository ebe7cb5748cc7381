// build.cu -- kernels that build the hierarchical latent-key index.
//
// Method (kongchang.com, "Latent Sparse Attention Breaks Through the
// Million-Token Context Bottleneck", section "How LSA Sidesteps Per-Key
// Scoring with Hierarchical Clustering"): keys are projected into a latent
// space and clustered level by level from a root holding every key ("similar to
// hierarchical k-means"); bdtechtalks.com, "Latent sparse attention", section
// "How latent sparse attention works": every cluster keeps a centroid and
// references to its original keys.
//
// Data layout during a build (all KV heads at once; "slot" = index into the
// level's segment order, head h owns slots [h*n, (h+1)*n)):
//   Z[slot][r]   fp32 latent rows, grouped by parent node (segment) of the level
//   pos[slot]    key position of the slot (ascending inside a segment)
//   a segment is the m = n / S consecutive slots of one parent node.
// Each k-means round: distances + preference lists -> balanced assignment by
// deferred acceptance -> stable partition of every segment by child -> child
// means over the partitioned order (fixed summation order, so deterministic).

#include <cooperative_groups.h>
#include <type_traits>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

// ---------------------------------------------------------------------------
// latent projection of keys: Z[h][i] = K[h][i] . W[h], pos = i
// ---------------------------------------------------------------------------
template <typename T, int R, int DK>
__global__ void __launch_bounds__(256) k_project_keys(const T* __restrict__ K, int64_t n_cap,
                                                      const T* __restrict__ W, int64_t n,
                                                      float* __restrict__ Z, int32_t* __restrict__ pos) {
  constexpr int ROWS = 64;                  // rows per CTA; thread = (row, quarter of the columns)
  constexpr int CQ = R / 4;                 // columns per thread
  extern __shared__ float smem[];
  float* sW = smem;                         // [DK][R]
  float* sK = smem + DK * R;                // [ROWS][DK + 1]
  const int h = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * ROWS;
  const T* Wh = W + (int64_t)h * DK * R;
  for (int i = threadIdx.x; i < DK * R; i += 256) sW[i] = to_f32(Wh[i]);
  const T* Kh = K + (int64_t)h * n_cap * DK;
  for (int i = threadIdx.x; i < ROWS * DK; i += 256) {
    const int rr = i / DK, cc = i % DK;
    const int64_t row = row0 + rr;
    sK[rr * (DK + 1) + cc] = row < n ? to_f32(Kh[row * DK + cc]) : 0.f;
  }
  __syncthreads();
  const int rr = threadIdx.x >> 2, q = threadIdx.x & 3;
  float acc[CQ];
#pragma unroll
  for (int c = 0; c < CQ; ++c) acc[c] = 0.f;
  for (int j = 0; j < DK; ++j) {
    const float kv = sK[rr * (DK + 1) + j];
#pragma unroll
    for (int c = 0; c < CQ; ++c) acc[c] = fmaf(kv, sW[j * R + q * CQ + c], acc[c]);
  }
  const int64_t row = row0 + rr;
  if (row < n) {
    float* zr = Z + ((int64_t)h * n + row) * R + q * CQ;
#pragma unroll
    for (int c = 0; c < CQ; c += 4) *reinterpret_cast<float4*>(zr + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
    if (q == 0 && pos) pos[(int64_t)h * n + row] = (int32_t)row;
  }
}

// ---------------------------------------------------------------------------
// seeded start: child j of a segment starts at the member with the j-th
// smallest SplitMix64 hash of its position (stream state = output `level` of
// the stream seeded with `seed`).  Tile pass keeps each tile's b smallest.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void block_min_u64(uint64_t& v, int64_t& who, uint64_t* s_v, int64_t* s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    uint64_t ov = __shfl_xor_sync(0xffffffffu, v, o);
    int64_t ow = __shfl_xor_sync(0xffffffffu, who, o);
    if (ov < v) { v = ov; who = ow; }
  }
  if (lane == 0) { s_v[warp] = v; s_w[warp] = who; }
  __syncthreads();
  if (warp == 0) {
    v = lane < nw ? s_v[lane] : ~0ull;
    who = lane < nw ? s_w[lane] : -1;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      uint64_t ov = __shfl_xor_sync(0xffffffffu, v, o);
      int64_t ow = __shfl_xor_sync(0xffffffffu, who, o);
      if (ov < v) { v = ov; who = ow; }
    }
    if (lane == 0) { s_v[0] = v; s_w[0] = who; }
  }
  __syncthreads();
  v = s_v[0];
  who = s_w[0];
  __syncthreads();
}

__global__ void __launch_bounds__(kTile) k_init_tile(const int32_t* __restrict__ pos, int64_t m, int64_t tps,
                                                     int b, uint64_t stream_state, uint64_t* __restrict__ cand_h,
                                                     int64_t* __restrict__ cand_slot) {
  __shared__ uint64_t s_v[32];
  __shared__ int64_t s_w[32];
  const int64_t tile = blockIdx.x, seg = tile / tps, t = tile % tps;
  const int64_t lo = seg * m + t * kTile, hi = seg * m + min64(m, (t + 1) * kTile);
  const int64_t slot = lo + threadIdx.x;
  const uint64_t my = slot < hi ? splitmix64_at(stream_state, (uint64_t)pos[slot]) : ~0ull;
  uint64_t last = 0;
  bool have_last = false;
  for (int j = 0; j < b; ++j) {
    uint64_t v = (my != ~0ull && (!have_last || my > last)) ? my : ~0ull;
    int64_t w = v != ~0ull ? slot : -1;
    block_min_u64(v, w, s_v, s_w);
    if (threadIdx.x == 0) { cand_h[tile * b + j] = v; cand_slot[tile * b + j] = w; }
    last = v;
    have_last = true;
  }
}

template <int R>
__global__ void __launch_bounds__(1024) k_init_merge(const uint64_t* __restrict__ cand_h,
                                                     const int64_t* __restrict__ cand_slot, int64_t tps, int b,
                                                     int64_t m, const float* __restrict__ Z, float* __restrict__ mu) {
  __shared__ uint64_t s_v[32];
  __shared__ int64_t s_w[32];
  __shared__ int64_t s_pick[LSA_MAX_BRANCHING];
  const int64_t seg = blockIdx.x;
  const int64_t nc = tps * b;
  const uint64_t* ch = cand_h + seg * nc;
  const int64_t* cs = cand_slot + seg * nc;
  uint64_t last = 0;
  for (int j = 0; j < b; ++j) {
    uint64_t v = ~0ull;
    int64_t w = -1;
    for (int64_t i = threadIdx.x; i < nc; i += blockDim.x) {
      uint64_t x = ch[i];
      if (x != ~0ull && (j == 0 || x > last) && x < v) { v = x; w = cs[i]; }
    }
    block_min_u64(v, w, s_v, s_w);
    if (threadIdx.x == 0) s_pick[j] = w >= 0 ? w : seg * m + j;  // w < 0 only if a hash equals ~0
    last = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < b * R; i += blockDim.x) {
    int j = i / R, k = i % R;
    mu[(seg * b + j) * R + k] = Z[s_pick[j] * R + k];
  }
}

// ---------------------------------------------------------------------------
// distances to the segment's b children and each key's preference list
// (children ordered by (distance asc, child asc), 4 bits per rank)
// ---------------------------------------------------------------------------
template <int R>
__global__ void __launch_bounds__(256) k_dist_pref(const float* __restrict__ Z, const float* __restrict__ mu,
                                                   int64_t nslots, int64_t m, int b, float* __restrict__ D,
                                                   uint64_t* __restrict__ pref, uint8_t* __restrict__ choice,
                                                   uint8_t* __restrict__ ptr, uint32_t* __restrict__ dbits,
                                                   int32_t* status) {
  extern __shared__ float s_mu[];
  const int64_t k0 = (int64_t)blockIdx.x * blockDim.x;
  const int64_t k1 = min64(nslots, k0 + blockDim.x);
  const int64_t seg_lo = k0 / m, seg_hi = (k1 - 1) / m;
  const int64_t rows = (seg_hi - seg_lo + 1) * b;
  for (int64_t i = threadIdx.x; i < rows * R; i += blockDim.x) s_mu[i] = mu[seg_lo * b * R + i];
  __syncthreads();
  const int64_t slot = k0 + threadIdx.x;
  if (slot >= nslots) return;
  const float* mrow = s_mu + (slot / m - seg_lo) * b * R;
  float z[R];
#pragma unroll
  for (int k = 0; k < R; k += 4) {
    float4 v = *reinterpret_cast<const float4*>(&Z[slot * R + k]);
    z[k] = v.x; z[k + 1] = v.y; z[k + 2] = v.z; z[k + 3] = v.w;
  }
  float dist[LSA_MAX_BRANCHING];
  int ord[LSA_MAX_BRANCHING];
  bool bad = false;
  for (int c = 0; c < b; ++c) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < R; ++k) {
      float df = z[k] - mrow[c * R + k];
      acc = fmaf(df, df, acc);
    }
    if (isnan(acc)) { bad = true; acc = __int_as_float(0x7f800000); }
    D[slot * b + c] = acc;
    // insertion by (distance, child): later children go after equal distances
    int p = c;
    while (p > 0 && dist[p - 1] > acc) { dist[p] = dist[p - 1]; ord[p] = ord[p - 1]; --p; }
    dist[p] = acc;
    ord[p] = c;
  }
  if (bad) set_status(status, LSA_ERR_NONFINITE);
  uint64_t pk = 0;
  for (int c = 0; c < b; ++c) pk |= (uint64_t)ord[c] << (4 * c);
  pref[slot] = pk;
  choice[slot] = (uint8_t)ord[0];
  ptr[slot] = 0;
  dbits[slot] = __float_as_uint(dist[0]);
}

// ---------------------------------------------------------------------------
// balanced assignment by key-proposing deferred acceptance.
// Key order inside a child: composite (distance bits << 32 | segment-local
// index); distances are >= 0 so their bits order like the floats, and the
// local index orders like the position.  Each round every over-full child
// keeps its `cap` smallest composites among the keys currently proposing to it
// (found by radix select) and rejects the rest, which move to their next
// preference.  Stops when no child is over-full.  Because preferences come from
// one global pair order, the stable assignment is unique, so the result equals
// the greedy scan of the sorted pairs.
// ---------------------------------------------------------------------------

// Small segments: one CTA holds the whole segment (m <= 8192), KPT keys per thread.
template <int KPT>
__global__ void __launch_bounds__(1024) k_da_cta(const uint64_t* __restrict__ pref, const float* __restrict__ D,
                                                 uint8_t* __restrict__ choice_out, int64_t m, int b, int64_t cap,
                                                 int max_rounds, int32_t* status) {
  __shared__ uint32_t hist[LSA_MAX_BRANCHING][256];
  __shared__ unsigned long long s_thr[LSA_MAX_BRANCHING], s_prefix[LSA_MAX_BRANCHING];
  __shared__ uint32_t s_need[LSA_MAX_BRANCHING];
  __shared__ int s_active[LSA_MAX_BRANCHING];
  __shared__ int s_any, s_changed;
  const int64_t base = (int64_t)blockIdx.x * m;
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
  uint64_t pf[KPT], key[KPT];
  int ch[KPT], pt[KPT];
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    int64_t l = tid + (int64_t)k * nt;
    pt[k] = 0;
    if (l < m) {
      pf[k] = pref[base + l];
      ch[k] = (int)(pf[k] & 15);
      key[k] = ((uint64_t)__float_as_uint(D[(base + l) * b + ch[k]]) << 32) | (uint64_t)l;
    } else {
      pf[k] = 0; ch[k] = -1; key[k] = 0;
    }
  }
  int round = 0;
  for (; round < max_rounds; ++round) {
    for (int i = tid; i < b * 256; i += nt) hist[i >> 8][i & 255] = 0;
    if (tid == 0) { s_any = 0; s_changed = 0; }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < KPT; ++k)
      if (ch[k] >= 0) atomicAdd(&hist[ch[k]][key[k] >> 56], 1u);
    __syncthreads();
    // digit 0 resolve: one warp per child
    for (int c = warp; c < b; c += nwarps) {
      uint32_t v[8];
      uint32_t s = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { v[q] = hist[c][lane * 8 + q]; s += v[q]; }
      uint32_t inc = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const uint32_t total = __shfl_sync(0xffffffffu, inc, 31);
      if ((int64_t)total <= cap) {
        if (lane == 0) { s_thr[c] = ~0ull; s_active[c] = 0; }
      } else {
        const uint32_t want = (uint32_t)cap;  // rank (1-based) of the last kept key
        const unsigned hit = __ballot_sync(0xffffffffu, inc >= want);
        const int src = __ffs(hit) - 1;
        if (lane == src) {
          uint32_t before = inc - s;
          int B = 0;
          for (int q = 0; q < 8; ++q) {
            if (before + v[q] >= want) { B = lane * 8 + q; break; }
            before += v[q];
          }
          const uint32_t need = want - before, cnt = hist[c][B];
          if (cnt == need) {
            s_thr[c] = ((unsigned long long)B << 56) | ((1ull << 56) - 1);
            s_active[c] = 0;
          } else {
            s_prefix[c] = B; s_need[c] = need; s_active[c] = 1; s_any = 1;
          }
        }
      }
    }
    __syncthreads();
    int any = s_any;
    for (int dg = 1; any && dg < 8; ++dg) {
      const int shift = 56 - 8 * dg;
      __syncthreads();
      if (tid == 0) s_any = 0;
      for (int i = tid; i < b * 256; i += nt)
        if (s_active[i >> 8]) hist[i >> 8][i & 255] = 0;
      __syncthreads();
#pragma unroll
      for (int k = 0; k < KPT; ++k)
        if (ch[k] >= 0 && s_active[ch[k]] && (key[k] >> (shift + 8)) == s_prefix[ch[k]])
          atomicAdd(&hist[ch[k]][(key[k] >> shift) & 255], 1u);
      __syncthreads();
      for (int c = warp; c < b; c += nwarps) {
        if (!s_active[c]) continue;
        uint32_t v[8];
        uint32_t s = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) { v[q] = hist[c][lane * 8 + q]; s += v[q]; }
        uint32_t inc = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        const uint32_t want = s_need[c];
        const unsigned hit = __ballot_sync(0xffffffffu, inc >= want);
        const int src = __ffs(hit) - 1;
        __syncwarp();
        if (lane == src) {
          uint32_t before = inc - s;
          int B = 0;
          for (int q = 0; q < 8; ++q) {
            if (before + v[q] >= want) { B = lane * 8 + q; break; }
            before += v[q];
          }
          const uint32_t need = want - before, cnt = hist[c][B];
          const unsigned long long pre = (s_prefix[c] << 8) | (unsigned)B;
          if (cnt == need) {
            s_thr[c] = (pre << shift) | (shift ? ((1ull << shift) - 1ull) : 0ull);
            s_active[c] = 0;
          } else {
            s_prefix[c] = pre; s_need[c] = need; s_any = 1;
          }
        }
      }
      __syncthreads();
      any = s_any;
    }
    // reject every key above its child's threshold
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      if (ch[k] >= 0 && key[k] > s_thr[ch[k]]) {
        int64_t l = tid + (int64_t)k * nt;
        if (pt[k] + 1 >= b) {
          set_status(status, LSA_ERR_TIMEOUT);  // cannot happen when sum(cap) == m
        } else {
          ++pt[k];
          ch[k] = (int)((pf[k] >> (4 * pt[k])) & 15);
          key[k] = ((uint64_t)__float_as_uint(D[(base + l) * b + ch[k]]) << 32) | (uint64_t)l;
          s_changed = 1;
        }
      }
    }
    __syncthreads();
    if (!s_changed) break;
  }
  if (round >= max_rounds && tid == 0) set_status(status, LSA_ERR_TIMEOUT);
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    int64_t l = tid + (int64_t)k * nt;
    if (l < m) choice_out[base + l] = (uint8_t)ch[k];
  }
}

// Large segments: every CTA of a cooperative grid takes part in every round;
// phases are separated by a grid barrier whose waits are bounded in time.
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ bool grid_barrier(GridBarrier* bar, unsigned nblocks, int32_t* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    volatile unsigned* vgen = &bar->gen;
    volatile int* vabort = &bar->abort;
    const unsigned g = *vgen;
    __threadfence();
    const unsigned a = atomicAdd(&bar->arrive, 1u);
    if (a == nblocks - 1) {
      atomicExch(&bar->arrive, 0u);
      __threadfence();
      atomicAdd(&bar->gen, 1u);
    } else {
      const uint64_t t0 = global_ns();
      while (*vgen == g) {
        if (*vabort) { ok = 0; break; }
        if (global_ns() - t0 > kBarrierTimeoutNs) {
          atomicExch(&bar->abort, 1);
          set_status(status, LSA_ERR_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

struct DaGridArgs {
  const uint64_t* pref;
  const float* D;
  uint8_t* choice;
  uint8_t* ptr;
  uint32_t* dbits;
  uint32_t* hist;     // [nsegc][2048]
  unsigned long long* thr;
  unsigned long long* prefix;
  uint32_t* need;
  int32_t* active;
  int32_t* flags;     // [3][8]
  GridBarrier* bar;
  int64_t nslots, m, cap, nsegc;
  int b, max_rounds;
  int32_t* status;
};

__constant__ int c_dshift[6] = {53, 42, 32, 21, 10, 0};
__constant__ int c_dbits[6] = {11, 11, 10, 11, 11, 10};

__device__ __forceinline__ uint64_t grid_key(const DaGridArgs& a, int64_t slot) {
  return ((uint64_t)a.dbits[slot] << 32) | (uint64_t)(slot % a.m);
}

// Resolve one child's digit: find the bin holding the `want`-th smallest key.
__device__ __forceinline__ void grid_resolve(const DaGridArgs& a, int64_t sc, int dg, bool first, int32_t* fl) {
  const int lane = threadIdx.x & 31;
  uint32_t* hb = a.hist + sc * 2048;
  const int nb = 1 << c_dbits[dg];
  const int per = nb / 32;
  uint32_t s = 0;
  for (int q = 0; q < per; ++q) s += __ldcg(&hb[lane * per + q]);
  uint32_t inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, inc, 31);
  uint32_t want;
  if (first) {
    if ((int64_t)total <= a.cap) {
      if (lane == 0) { __stcg(&a.thr[sc], ~0ull); __stcg(&a.active[sc], 0); }
      want = 0;
    } else {
      want = (uint32_t)a.cap;
    }
  } else {
    want = __ldcg(&a.need[sc]);
  }
  if (want) {
    const unsigned hit = __ballot_sync(0xffffffffu, inc >= want);
    const int src = __ffs(hit) - 1;
    if (lane == src) {
      uint32_t before = inc - s;
      int B = 0;
      for (int q = 0; q < per; ++q) {
        uint32_t v = __ldcg(&hb[lane * per + q]);
        if (before + v >= want) { B = lane * per + q; break; }
        before += v;
      }
      const uint32_t need = want - before, cnt = __ldcg(&hb[B]);
      const int shift = c_dshift[dg];
      const unsigned long long pre =
          first ? (unsigned long long)B : ((__ldcg(&a.prefix[sc]) << c_dbits[dg]) | (unsigned)B);
      if (cnt == need) {
        __stcg(&a.thr[sc], (pre << shift) | (shift ? ((1ull << shift) - 1ull) : 0ull));
        __stcg(&a.active[sc], 0);
      } else {
        __stcg(&a.prefix[sc], pre);
        __stcg(&a.need[sc], need);
        __stcg(&a.active[sc], 1);
        atomicExch(&fl[dg], 1);
      }
    }
  }
  __syncwarp();
  for (int q = 0; q < per; ++q) __stcg(&hb[lane * per + q], 0u);
}

__global__ void __launch_bounds__(512) k_da_grid(DaGridArgs a) {
  const unsigned nblocks = gridDim.x;
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t gstride = (int64_t)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  const int64_t gwarp = gtid >> 5, nwarps_g = gstride >> 5;
  int round = 0;
  for (; round < a.max_rounds; ++round) {
    int32_t* fl = a.flags + (round % 3) * 8;
    if (gtid == 0) {
      int32_t* nf = a.flags + ((round + 1) % 3) * 8;
      for (int i = 0; i < 8; ++i) __stcg(&nf[i], 0);
    }
    // digit 0 histogram over all keys (warp-aggregated atomics)
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < a.nslots; base += gstride) {
      const int64_t slot = base + threadIdx.x;
      const bool ok = slot < a.nslots;
      uint64_t tag = ~0ull;
      if (ok) {
        const int64_t sc = (slot / a.m) * a.b + a.choice[slot];
        tag = ((uint64_t)sc << 11) | (grid_key(a, slot) >> 53);
      }
      const unsigned peers = __match_any_sync(0xffffffffu, tag);
      if (ok && lane == __ffs(peers) - 1) atomicAdd(&a.hist[(tag >> 11) * 2048 + (tag & 2047)], __popc(peers));
    }
    if (!grid_barrier(a.bar, nblocks, a.status)) return;
    for (int64_t sc = gwarp; sc < a.nsegc; sc += nwarps_g) grid_resolve(a, sc, 0, true, fl);
    if (!grid_barrier(a.bar, nblocks, a.status)) return;
    for (int dg = 1; dg < 6; ++dg) {
      if (!__ldcg(&fl[dg - 1])) break;
      const int pshift = c_dshift[dg - 1], shift = c_dshift[dg];
      const uint64_t mask = (1ull << c_dbits[dg]) - 1;
      for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < a.nslots; base += gstride) {
        const int64_t slot = base + threadIdx.x;
        uint64_t tag = ~0ull;
        if (slot < a.nslots) {
          const int64_t sc = (slot / a.m) * a.b + a.choice[slot];
          if (__ldcg(&a.active[sc])) {
            const uint64_t key = grid_key(a, slot);
            if ((key >> pshift) == __ldcg(&a.prefix[sc])) tag = ((uint64_t)sc << 11) | ((key >> shift) & mask);
          }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, tag);
        if (tag != ~0ull && lane == __ffs(peers) - 1)
          atomicAdd(&a.hist[(tag >> 11) * 2048 + (tag & 2047)], __popc(peers));
      }
      if (!grid_barrier(a.bar, nblocks, a.status)) return;
      for (int64_t sc = gwarp; sc < a.nsegc; sc += nwarps_g)
        if (__ldcg(&a.active[sc])) grid_resolve(a, sc, dg, false, fl);
      if (!grid_barrier(a.bar, nblocks, a.status)) return;
    }
    // reject
    for (int64_t slot = gtid; slot < a.nslots; slot += gstride) {
      const int64_t sc = (slot / a.m) * a.b + a.choice[slot];
      if (grid_key(a, slot) > __ldcg(&a.thr[sc])) {
        const int p = a.ptr[slot] + 1;
        if (p >= a.b) {
          set_status(a.status, LSA_ERR_TIMEOUT);
        } else {
          const int c = (int)((a.pref[slot] >> (4 * p)) & 15);
          a.ptr[slot] = (uint8_t)p;
          a.choice[slot] = (uint8_t)c;
          a.dbits[slot] = __float_as_uint(a.D[slot * a.b + c]);
          atomicExch(&fl[7], 1);
        }
      }
    }
    if (!grid_barrier(a.bar, nblocks, a.status)) return;
    if (!__ldcg(&fl[7])) break;
  }
  if (round >= a.max_rounds && gtid == 0) set_status(a.status, LSA_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
// stable partition of every segment by child: order[seg*m + c*cap + k] = slot
// of the k-th member (in slot order) of child c.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kTile) k_part_count(const uint8_t* __restrict__ choice, int64_t m, int64_t tps,
                                                      int b, int32_t* __restrict__ tcnt) {
  __shared__ int32_t s_cnt[LSA_MAX_BRANCHING];
  const int64_t tile = blockIdx.x, seg = tile / tps, t = tile % tps;
  const int64_t lo = seg * m + t * kTile, hi = seg * m + min64(m, (t + 1) * kTile);
  if (threadIdx.x < b) s_cnt[threadIdx.x] = 0;
  __syncthreads();
  const int64_t slot = lo + threadIdx.x;
  if (slot < hi) atomicAdd(&s_cnt[choice[slot]], 1);
  __syncthreads();
  if (threadIdx.x < b) tcnt[tile * b + threadIdx.x] = s_cnt[threadIdx.x];
}

__global__ void k_part_scan(const int32_t* __restrict__ tcnt, int64_t tps, int b, int64_t cap,
                            int64_t* __restrict__ toff) {
  const int64_t seg = blockIdx.x;
  const int c = threadIdx.x;
  if (c >= b) return;
  int64_t run = (int64_t)c * cap;
  for (int64_t t = 0; t < tps; ++t) {
    const int64_t tile = seg * tps + t;
    toff[tile * b + c] = run;
    run += tcnt[tile * b + c];
  }
}

__global__ void __launch_bounds__(kTile) k_part_scatter(const uint8_t* __restrict__ choice, int64_t m, int64_t tps,
                                                        int b, int64_t cap, const int64_t* __restrict__ toff,
                                                        int32_t* __restrict__ order, int32_t* status) {
  __shared__ int32_t s_wcnt[kTile / 32][LSA_MAX_BRANCHING];
  const int64_t tile = blockIdx.x, seg = tile / tps, t = tile % tps;
  const int64_t lo = seg * m + t * kTile, hi = seg * m + min64(m, (t + 1) * kTile);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t slot = lo + threadIdx.x;
  const bool ok = slot < hi;
  const int c = ok ? choice[slot] : 0xff;
  for (int i = threadIdx.x; i < (kTile / 32) * LSA_MAX_BRANCHING; i += blockDim.x) (&s_wcnt[0][0])[i] = 0;
  __syncthreads();
  const unsigned peers = __match_any_sync(0xffffffffu, c);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (ok && rank == 0) s_wcnt[warp][c] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < b) {  // exclusive scan over warps, per child
    int run = 0;
    for (int w = 0; w < kTile / 32; ++w) {
      int v = s_wcnt[w][threadIdx.x];
      s_wcnt[w][threadIdx.x] = run;
      run += v;
    }
  }
  __syncthreads();
  if (ok) {
    const int64_t at = toff[tile * b + c] + s_wcnt[warp][c] + rank;  // c * cap + rank inside child c
    if (at - (int64_t)c * cap < cap) order[seg * m + at] = (int32_t)slot;
    else set_status(status, LSA_ERR_TIMEOUT);  // only reachable after a failed assignment
  }
}

// ---------------------------------------------------------------------------
// child means over the partitioned order, in a fixed summation order
// ---------------------------------------------------------------------------
template <int R>
__global__ void __launch_bounds__(256) k_means_chunk(const float* __restrict__ Z, const int32_t* __restrict__ order,
                                                     int64_t nslots, int64_t nnodes, int64_t cap, int64_t cpn,
                                                     float* __restrict__ partial, float* __restrict__ mu) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= nnodes * cpn) return;
  const int64_t node = w / cpn, chunk = w % cpn;
  const int64_t lo = node * cap + chunk * kMeanChunk;
  const int64_t hi = node * cap + min64(cap, (chunk + 1) * kMeanChunk);
  constexpr int PER = (R + 31) / 32;
  float acc[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) acc[q] = 0.f;
  for (int64_t i = lo; i < hi; ++i) {
    const int64_t src = order[i];
    const float* zr = Z + ((uint64_t)src < (uint64_t)nslots ? src : 0) * R;
#pragma unroll
    for (int q = 0; q < PER; ++q)
      if (lane + 32 * q < R) acc[q] += zr[lane + 32 * q];
  }
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int k = lane + 32 * q;
    if (k >= R) continue;
    if (cpn == 1) mu[node * R + k] = acc[q] / (float)cap;
    else partial[w * R + k] = acc[q];
  }
}

template <int R>
__global__ void k_means_final(const float* __restrict__ partial, int64_t nnodes, int64_t cap, int64_t cpn,
                              float* __restrict__ mu) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nnodes * R) return;
  const int64_t node = i / R, k = i % R;
  float s = 0.f;
  for (int64_t c = 0; c < cpn; ++c) s += partial[(node * cpn + c) * R + k];
  mu[i] = s / (float)cap;
}

// trace[h][pos] = node id inside head h after an assignment round
__global__ void k_trace(const uint8_t* __restrict__ choice, const int32_t* __restrict__ pos, int64_t nslots,
                        int64_t n, int64_t m, int b, int64_t nodes_per_head, int32_t* __restrict__ trace) {
  const int64_t slot = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (slot >= nslots) return;
  const int64_t h = slot / n;
  const int64_t node = (slot / m) * b + choice[slot] - h * nodes_per_head;
  trace[h * n + pos[slot]] = (int32_t)node;
}

// next level's segment order: slot q takes the key at order[q]
template <int R>
__global__ void k_level_gather(const int32_t* __restrict__ order, const float* __restrict__ Za,
                               const int32_t* __restrict__ pa, int64_t nslots, float* __restrict__ Zb,
                               int32_t* __restrict__ pb) {
  constexpr int V = R / 4;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nslots * V) return;
  const int64_t q = i / V, part = i % V;
  int64_t src = order[q];
  if ((uint64_t)src >= (uint64_t)nslots) src = 0;  // only after a failed assignment
  reinterpret_cast<float4*>(Zb)[q * V + part] = reinterpret_cast<const float4*>(Za)[src * V + part];
  if (part == 0) pb[q] = pa[src];
}

// smallest key position of each node = that of its first member (ascending);
// a member is a key, or with pooling a block of `pool` keys starting at pa * pool
__global__ void k_min_pos(const int32_t* __restrict__ order, const int32_t* __restrict__ pa, int64_t nnodes,
                          int64_t cap, int32_t pool, int32_t* __restrict__ min_pos) {
  const int64_t node = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (node >= nnodes) return;
  int64_t src = order[node * cap];
  if ((uint64_t)src >= (uint64_t)(nnodes * cap)) src = 0;  // only after a failed assignment
  min_pos[node] = pa[src] * pool;
}

// ---------------------------------------------------------------------------
// pooling (bdtechtalks.com, "Latent sparse attention", section "How latent
// sparse attention works": consecutive keys pooled into smaller
// representations before the clustering): block j of a head is the mean of the
// latent rows of keys [j*pool, (j+1)*pool), summed in position order; its
// position is j.
// ---------------------------------------------------------------------------
template <int R>
__global__ void k_pool_keys(const float* __restrict__ Z, int64_t nblocks, int64_t per_head, int32_t pool,
                            float* __restrict__ Zp, int32_t* __restrict__ pos) {
  constexpr int V = R / 4;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // (head * nblocks + block) * V + part
  if (i >= nblocks * V) return;
  const int64_t blk = i / V, part = i % V;
  const float4* src = reinterpret_cast<const float4*>(Z) + blk * pool * V + part;
  float4 acc = src[0];
  for (int k = 1; k < pool; ++k) {
    const float4 v = src[(int64_t)k * V];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  const float inv = 1.f / (float)pool;
  reinterpret_cast<float4*>(Zp)[i] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (part == 0) pos[blk] = (int32_t)(blk % per_head);
}

// leaf_index of a pooled tree: block slot s (ascending inside its leaf) lists
// the keys b*pool .. b*pool + pool - 1 of its block b
__global__ void k_expand_leaves(const int32_t* __restrict__ blocks, int64_t nslots, int32_t pool,
                                int32_t* __restrict__ leaf_index) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nslots * pool) return;
  leaf_index[i] = blocks[i / pool] * pool + (int32_t)(i % pool);
}

// ---------------------------------------------------------------------------
// host driver
// ---------------------------------------------------------------------------
// One balanced assignment of every segment: distances and preference lists
// (k_dist_pref), then deferred acceptance, one CTA per segment up to kCtaMaxSeg
// keys, else the cooperative grid kernel.  Writes P.choice [nslots].  A segment
// still moving after max_rounds proposal rounds sets LSA_ERR_TIMEOUT.
template <int R>
static cudaError_t assign_round(const BuildPlan& P, const float* Za, int64_t nslots, int64_t m, int b,
                                int max_rounds, int32_t* status, cudaStream_t st) {
  const int64_t nseg = nslots / m, cap = m / b, nnodes = nseg * b;
  cudaError_t e;
  {
    // centroids of every segment a CTA's 256 slots touch: (256 / m + 1) * b rows,
    // at most (256 + b) * R floats (about 70 KB) when a segment holds b members
    const int64_t rows = (ceil_div(256, m) + 1) * b;
    const size_t smem = (size_t)rows * R * sizeof(float);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(k_dist_pref<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_dist_pref<R><<<(unsigned)ceil_div(nslots, 256), 256, smem, st>>>(Za, P.mu, nslots, m, b, P.D, P.pref,
                                                                      P.choice, P.ptr, P.dbits, status);
  }
  if (m <= kCtaMaxSeg) {
    const int kpt = m <= 1024 ? 1 : m <= 2048 ? 2 : m <= 4096 ? 4 : 8;
    const int nt = (int)((ceil_div(ceil_div(m, kpt), 32)) * 32);
    switch (kpt) {
      case 1: k_da_cta<1><<<(unsigned)nseg, nt, 0, st>>>(P.pref, P.D, P.choice, m, b, cap, max_rounds, status); break;
      case 2: k_da_cta<2><<<(unsigned)nseg, nt, 0, st>>>(P.pref, P.D, P.choice, m, b, cap, max_rounds, status); break;
      case 4: k_da_cta<4><<<(unsigned)nseg, nt, 0, st>>>(P.pref, P.D, P.choice, m, b, cap, max_rounds, status); break;
      default: k_da_cta<8><<<(unsigned)nseg, nt, 0, st>>>(P.pref, P.D, P.choice, m, b, cap, max_rounds, status); break;
    }
    return cudaGetLastError();
  }
  DaGridArgs a;
  a.pref = P.pref; a.D = P.D; a.choice = P.choice; a.ptr = P.ptr; a.dbits = P.dbits;
  a.hist = P.hist; a.thr = P.thr; a.prefix = P.prefix; a.need = P.need; a.active = P.active;
  a.flags = P.flags; a.bar = P.bar; a.nslots = nslots; a.m = m; a.cap = cap; a.nsegc = nnodes;
  a.b = b; a.max_rounds = max_rounds; a.status = status;
  if ((e = cudaMemsetAsync(P.hist, 0, (size_t)nnodes * 2048 * sizeof(uint32_t), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(P.flags, 0, 24 * sizeof(int32_t), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(P.bar, 0, sizeof(GridBarrier), st)) != cudaSuccess) return e;
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel((const void*)k_da_grid, dim3(P.coop_blocks), dim3(512), args, 0, st);
}

template <int R>
static cudaError_t build_levels(const BuildPlan& P, const lsa_tree_desc& t, char* tree_mem, int32_t* trace,
                                int32_t* status, int32_t pool, cudaStream_t st) {
  const int64_t H = t.n_heads, n = t.n_tree, nslots = H * n;
  float* Za = P.Za;
  float* Zb = P.Zb;
  int32_t* pa = P.pa;
  int32_t* pb = P.pb;
  cudaError_t e;
  int64_t S = 1;
  for (int l = 0; l < t.levels; ++l) {
    const int b = t.branching[l];
    const int64_t nseg = H * S, m = n / S, cap = m / b;
    const int64_t tps = ceil_div(m, kTile), ntiles = nseg * tps;
    const uint64_t stream_state = splitmix64_at(P.seed, (uint64_t)l);
    k_init_tile<<<(unsigned)ntiles, kTile, 0, st>>>(pa, m, tps, b, stream_state, P.cand_h, P.cand_slot);
    k_init_merge<R><<<(unsigned)nseg, 1024, 0, st>>>(P.cand_h, P.cand_slot, tps, b, m, Za, P.mu);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t nnodes = nseg * b;
    const int64_t cpn = ceil_div(cap, kMeanChunk);
    for (int it = 0; it < P.iters; ++it) {
      if ((e = assign_round<R>(P, Za, nslots, m, b, kMaxRounds, status, st)) != cudaSuccess) return e;
      k_part_count<<<(unsigned)ntiles, kTile, 0, st>>>(P.choice, m, tps, b, P.tcnt);
      k_part_scan<<<(unsigned)nseg, 32, 0, st>>>(P.tcnt, tps, b, cap, P.toff);
      k_part_scatter<<<(unsigned)ntiles, kTile, 0, st>>>(P.choice, m, tps, b, cap, P.toff, P.order, status);
      {
        const int64_t warps = nnodes * cpn;
        k_means_chunk<R><<<(unsigned)ceil_div(warps * 32, 256), 256, 0, st>>>(Za, P.order, nslots, nnodes, cap, cpn,
                                                                               P.partial, P.mu);
        if (cpn > 1)
          k_means_final<R><<<(unsigned)ceil_div(nnodes * R, 256), 256, 0, st>>>(P.partial, nnodes, cap, cpn, P.mu);
      }
      if (trace)
        k_trace<<<(unsigned)ceil_div(nslots, 256), 256, 0, st>>>(
            P.choice, pa, nslots, n, m, b, t.nodes[l], trace + ((int64_t)l * P.iters + it) * nslots);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // tree outputs of this level, then the next level's segment order
    float* cent = reinterpret_cast<float*>(tree_mem + t.off_centroids[l]);
    int32_t* mpos = reinterpret_cast<int32_t*>(tree_mem + t.off_min_pos[l]);
    if ((e = cudaMemcpyAsync(cent, P.mu, (size_t)nnodes * R * sizeof(float), cudaMemcpyDeviceToDevice, st)) !=
        cudaSuccess)
      return e;
    k_min_pos<<<(unsigned)ceil_div(nnodes, 256), 256, 0, st>>>(P.order, pa, nnodes, cap, pool, mpos);
    k_level_gather<R><<<(unsigned)ceil_div(nslots * (R / 4), 256), 256, 0, st>>>(P.order, Za, pa, nslots, Zb, pb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    float* tz = Za; Za = Zb; Zb = tz;
    int32_t* tp = pa; pa = pb; pb = tp;
    S *= b;
  }
  int32_t* leaf = reinterpret_cast<int32_t*>(tree_mem + t.off_leaf_index);
  if (pool == 1) return cudaMemcpyAsync(leaf, pa, (size_t)nslots * sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
  k_expand_leaves<<<(unsigned)ceil_div(nslots * pool, 256), 256, 0, st>>>(pa, nslots, pool, leaf);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t project(const void* K, int64_t n_cap, const void* W, int64_t n, int32_t n_heads, int r, int d,
                           float* Z, int32_t* pos, int32_t* status, cudaStream_t st) {
  // bf16 keys: tensor-core product (project.cu); fp32 keys keep fp32 FMAs, since a
  // tf32 product would round the operands to 10 mantissa bits
  if (project_tc_supported(std::is_same<T, float>::value ? LSA_F32 : LSA_BF16, r, d))
    return run_project_tc(K, n_cap, W, n, n_heads, r, d, Z, pos, status, st);
  if (n <= 0) return cudaSuccess;
  dim3 grid((unsigned)ceil_div(n, 64), (unsigned)n_heads);
  const T* k = static_cast<const T*>(K);
  const T* w = static_cast<const T*>(W);
#define LSA_PROJ(RR, DD)                                                                           \
  if (r == RR && d == DD) {                                                                        \
    const size_t smem = (size_t)(DD * RR + 64 * (DD + 1)) * sizeof(float);                         \
    cudaFuncSetAttribute(k_project_keys<T, RR, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                         (int)smem);                                                               \
    k_project_keys<T, RR, DD><<<grid, 256, smem, st>>>(k, n_cap, w, n, Z, pos);                   \
    return cudaGetLastError();                                                                     \
  }
  LSA_PROJ(16, 64) LSA_PROJ(32, 64) LSA_PROJ(64, 64) LSA_PROJ(16, 128) LSA_PROJ(32, 128) LSA_PROJ(64, 128)
#undef LSA_PROJ
  return cudaErrorInvalidValue;
}

cudaError_t run_assign(const BuildPlan& P, const float* Z, int64_t nseg, int64_t m, int b, int r, int max_rounds,
                       int32_t* status, cudaStream_t st) {
  const int64_t nslots = nseg * m;
  switch (r) {
    case 16: return assign_round<16>(P, Z, nslots, m, b, max_rounds, status, st);
    case 32: return assign_round<32>(P, Z, nslots, m, b, max_rounds, status, st);
    default: return assign_round<64>(P, Z, nslots, m, b, max_rounds, status, st);
  }
}

cudaError_t run_project(const void* K, int64_t n_cap, const void* W, int64_t n, int32_t n_heads, int r, int d,
                        int dtype, float* Z, int32_t* pos, int32_t* status, cudaStream_t st) {
  return dtype == LSA_BF16 ? project<__nv_bfloat16>(K, n_cap, W, n, n_heads, r, d, Z, pos, status, st)
                           : project<float>(K, n_cap, W, n, n_heads, r, d, Z, pos, status, st);
}

cudaError_t run_build(const BuildPlan& P, const lsa_tree_desc& t, void* tree_mem, const void* K, int64_t n_cap,
                      int d, int dtype, const void* W, int32_t pool, int32_t* trace, int32_t* status,
                      cudaStream_t st) {
  cudaError_t e = run_project(K, n_cap, W, t.n_tree, t.n_heads, t.r, d, dtype, P.Za, P.pa, status, st);
  if (e != cudaSuccess) return e;
  char* tm = static_cast<char*>(tree_mem);
  // with pooling the levels cluster the blocks: same nodes and tree buffer,
  // n_tree / pool members with leaf_size / pool per leaf
  BuildPlan Q = P;
  lsa_tree_desc tb = t;
  if (pool > 1) {
    const int64_t per_head = t.n_tree / pool, nblocks = t.n_heads * per_head;
    const unsigned grid = (unsigned)ceil_div(nblocks * (t.r / 4), 256);
    switch (t.r) {
      case 16: k_pool_keys<16><<<grid, 256, 0, st>>>(P.Za, nblocks, per_head, pool, P.Zb, P.pb); break;
      case 32: k_pool_keys<32><<<grid, 256, 0, st>>>(P.Za, nblocks, per_head, pool, P.Zb, P.pb); break;
      default: k_pool_keys<64><<<grid, 256, 0, st>>>(P.Za, nblocks, per_head, pool, P.Zb, P.pb); break;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    Q.Za = P.Zb; Q.Zb = P.Za;
    Q.pa = P.pb; Q.pb = P.pa;
    tb.n_tree = t.n_tree / pool;
    tb.leaf_size = t.leaf_size / pool;
  }
  switch (t.r) {
    case 16: return build_levels<16>(Q, tb, tm, trace, status, pool, st);
    case 32: return build_levels<32>(Q, tb, tm, trace, status, pool, st);
    default: return build_levels<64>(Q, tb, tm, trace, status, pool, st);
  }
}

// ---------------------------------------------------------------------------
// update on append: one level of the grown tree -- the old nodes, then the
// subtree's (its min_pos shifted by n_old); on the top level the subtree is one
// node whose centroid is the mean of the subtree's top centroids (its children,
// all of the same size) and whose min_pos is n_old
// ---------------------------------------------------------------------------
__global__ void k_attach_level(const float* __restrict__ oc, const int32_t* __restrict__ om, int64_t old_nodes,
                               const float* __restrict__ sc, const int32_t* __restrict__ sm, int64_t sub_nodes,
                               int root_children, int64_t H, int R, int32_t n_old, float* __restrict__ nc,
                               int32_t* __restrict__ nm) {
  const int64_t per = old_nodes + sub_nodes;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // (head * per + node) * R + column
  if (i >= H * per * R) return;
  const int64_t h = i / (per * R), node = (i / R) % per;
  const int c = (int)(i % R);
  float v;
  int32_t mp;
  if (node < old_nodes) {
    v = oc[(h * old_nodes + node) * R + c];
    mp = om[h * old_nodes + node];
  } else if (root_children > 0) {
    float s = 0.f;
    for (int j = 0; j < root_children; ++j) s += sc[(h * root_children + j) * R + c];
    v = s / (float)root_children;
    mp = n_old;
  } else {
    const int64_t k = node - old_nodes;
    v = sc[(h * sub_nodes + k) * R + c];
    mp = sm[h * sub_nodes + k] + n_old;
  }
  nc[i] = v;
  if (c == 0) nm[h * per + node] = mp;
}

__global__ void k_attach_leaves(const int32_t* __restrict__ ol, const int32_t* __restrict__ sl, int64_t H,
                                int64_t n_old, int64_t U, int32_t* __restrict__ nl) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * (n_old + U)) return;
  const int64_t h = i / (n_old + U), k = i % (n_old + U);
  nl[i] = k < n_old ? ol[h * n_old + k] : sl[h * U + (k - n_old)] + (int32_t)n_old;
}

cudaError_t run_tree_attach(const lsa_tree_desc& old_t, const void* old_mem, const lsa_tree_desc& sub,
                            const void* sub_mem, const lsa_tree_desc& grown, void* grown_mem, cudaStream_t st) {
  const char* om = static_cast<const char*>(old_mem);
  const char* sb = static_cast<const char*>(sub_mem);
  char* gm = static_cast<char*>(grown_mem);
  const int64_t H = old_t.n_heads;
  const int R = old_t.r;
  for (int l = 0; l < old_t.levels; ++l) {
    const int64_t on = old_t.nodes[l], sn = l == 0 ? 1 : sub.nodes[l - 1];
    const int sl = l == 0 ? 0 : l - 1;   // subtree level feeding this one (its top for the new root)
    const int64_t total = H * (on + sn) * R;
    k_attach_level<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(
        reinterpret_cast<const float*>(om + old_t.off_centroids[l]),
        reinterpret_cast<const int32_t*>(om + old_t.off_min_pos[l]), on,
        reinterpret_cast<const float*>(sb + sub.off_centroids[sl]),
        reinterpret_cast<const int32_t*>(sb + sub.off_min_pos[sl]), sn, l == 0 ? (int)sub.nodes[0] : 0, H, R,
        (int32_t)old_t.n_tree, reinterpret_cast<float*>(gm + grown.off_centroids[l]),
        reinterpret_cast<int32_t*>(gm + grown.off_min_pos[l]));
  }
  const int64_t total = H * grown.n_tree;
  k_attach_leaves<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(
      reinterpret_cast<const int32_t*>(om + old_t.off_leaf_index), reinterpret_cast<const int32_t*>(sb + sub.off_leaf_index),
      H, old_t.n_tree, sub.n_tree, reinterpret_cast<int32_t*>(gm + grown.off_leaf_index));
  return cudaGetLastError();
}

int da_grid_blocks() {
  int dev = 0, sms = 0, per = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_da_grid, 512, 0) != cudaSuccess) return 0;
  per = per > 2 ? 2 : per;
  return sms * per;
}

}  // namespace lsa
