// flat_tc.cu -- flat search on the tensor cores.
//
// bdtechtalks.com, "Latent sparse attention", section "How latent sparse
// attention works" (the first strategy): the query is compared against every
// cluster centroid.  For a KV group that is a dense product of the group
// latents [T x r] with the leaf centroids [leaves x r], followed by a top-B per
// query; the best B leaves are kept by (score desc, leaf id asc), a leaf being
// a candidate only if its smallest key position is visible to the query.
//
// Scores must rank like fp32 inner products (the near-tie band of the ranking is
// 1e-5 relative), so every fp32 operand x is split exactly into three bf16 parts
// x = x1 + x2 + x3 (x1 = bf16(x), x2 = bf16(x - x1), x3 = bf16(x - x1 - x2)) and
// the six products x_i y_j with i + j <= 4 are accumulated in fp32 by
// tcgen05.mma kind::f16; the terms left out are below 2^-24 of |x||y|.
//
// One CTA of 128 threads per (tile of 128 queries, KV group):
//   prologue: the group queries (mean of the G heads, split in three) times
//     W[g] on the tensor cores give the 128 latents in TMEM; each thread reads
//     its query's latent, splits it, and stores the three A tiles;
//   main loop over tiles of 128 leaves: the leaf centroids are read as fp32 rows,
//     split into three B tiles (double-buffered), and the six products of tile
//     j + 1 are issued before the scores of tile j are read from TMEM (two
//     128-column buffers); each thread keeps its query's best B keys in a
//     sorted list in shared memory.
#include <climits>

#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tc_sm100.cuh"

namespace lsa {

namespace {

constexpr int kFT = 128;               // queries per CTA = TMEM lanes
constexpr int kFTh = 2 * kFT;          // threads: two per query (halves of every leaf tile)
constexpr int kFN = 128;               // leaves per tile (MMA N)
constexpr int kFR = 64;                // latent dimension of this path
constexpr int kFMaxB = 32;             // longest kept list of this path
constexpr uint32_t kTileB = kFT * 128; // one [128 rows x 64 bf16] SW128 tile (16 KB)

template <int DK>
struct FlatTcSmem {
  // [A0 A1 A2 | B(0) 3 tiles | B(1) 3 tiles | W^T | lists | mpos(2)]
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = 3 * kTileB;
  static constexpr uint32_t kW = kB + 6 * kTileB;                 // [64 rows x DK] bf16, K-major
  static constexpr uint32_t kList = kW + kFR * DK * 2;
  static constexpr uint32_t kMpos = kList + kFMaxB * kFT * 8;   // list region: fp32 row staging, then the lists
  static constexpr size_t kBytes = 1024 + kMpos + 2 * kFN * 8;   // (min position, leaf id) per column and buffer
};

// Exact three-way bf16 split of an fp32 value.
__device__ __forceinline__ void split3(float x, __nv_bfloat16& a, __nv_bfloat16& b, __nv_bfloat16& c) {
  a = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(a);
  b = __float2bfloat16_rn(r1);
  c = __float2bfloat16_rn(r1 - __bfloat162float(b));
}

// 16-byte chunk c of row r of a [rows x 64 bf16] SW128 tile.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// Store 8 consecutive fp32 values (columns 8c .. 8c + 7 of row r) as their three
// bf16 parts into three tiles at base + {0, 1, 2} * stride.
__device__ __forceinline__ void store_split8(char* base, uint32_t stride, int r, int c, const float (&x)[8]) {
  uint32_t w[3][4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat16 a0, b0, c0, a1, b1, c1;
    split3(x[2 * q], a0, b0, c0);
    split3(x[2 * q + 1], a1, b1, c1);
    w[0][q] = pack2(a0, a1);
    w[1][q] = pack2(b0, b1);
    w[2][q] = pack2(c0, c1);
  }
  const uint32_t off = tile_off(r, c);
#pragma unroll
  for (int i = 0; i < 3; ++i)
    *reinterpret_cast<uint4*>(base + i * stride + off) = make_uint4(w[i][0], w[i][1], w[i][2], w[i][3]);
}

// v[i] for a run-time i, by a tree of selects (no local-memory indexing).
__device__ __forceinline__ float pick32(const float (&v)[32], int i) {
  float a16[16], a8[8], a4[4], a2[2];
#pragma unroll
  for (int k = 0; k < 16; ++k) a16[k] = (i & 16) ? v[k + 16] : v[k];
#pragma unroll
  for (int k = 0; k < 8; ++k) a8[k] = (i & 8) ? a16[k + 8] : a16[k];
#pragma unroll
  for (int k = 0; k < 4; ++k) a4[k] = (i & 4) ? a8[k + 4] : a8[k];
#pragma unroll
  for (int k = 0; k < 2; ++k) a2[k] = (i & 2) ? a4[k + 2] : a4[k];
  return (i & 1) ? a2[1] : a2[0];
}

template <int DK>
__global__ void __launch_bounds__(kFTh, 1) k_select_flat_tc(SelectArgs a) {
  using S = FlatTcSmem<DK>;
  constexpr int NH = DK / 64;                      // 64-column halves of a query / W^T row
  extern __shared__ char smem_raw[];
  __shared__ __align__(8) uint64_t s_mbar[3];      // [0, 1]: score buffers; [2]: latent
  __shared__ uint32_t s_taddr;
  __shared__ int s_bad;
  char* base = align1024(smem_raw);
  const uint32_t sbase = smem_u32(base);
  int2* s_ml = reinterpret_cast<int2*>(base + S::kMpos);   // [2][128] (min position, leaf id or -1)
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kFT - 1), hf = tid / kFT;   // query row (TMEM lane) and half of the columns
  const int g = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * kFT;
  const int L = a.levels - 1;
  const int64_t NL = a.nodes[L];
  const int B = a.beam[L];
  const float* cent = reinterpret_cast<const float*>(a.tree + a.off_c[L]) + (int64_t)g * NL * kFR;
  const int32_t* mpos = reinterpret_cast<const int32_t*>(a.tree + a.off_m[L]) + (int64_t)g * NL;
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.Q);
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.W) + (int64_t)g * DK * kFR;

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&s_mbar[i]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;");
    s_bad = 0;
  }
  alloc_tmem(&s_taddr, 2 * kFN);

  // ---- prologue: the group queries, split in three, and W^T into shared memory ----
  for (int x = tid; x < kFT * (DK / 8); x += kFTh) {
    const int r = x / (DK / 8), c = x % (DK / 8);
    const int64_t t = t0 + r;
    float q[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = 0.f;
    if (t < a.T) {
      for (int h = 0; h < a.G; ++h) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(Q + (t * a.Hq + (int64_t)g * a.G + h) * DK + c * 8));
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          q[2 * e] += f.x;
          q[2 * e + 1] += f.y;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] /= (float)a.G;
    }
    // split i of half (c / 8) at tile (i * NH + c / 8) of the B region
    store_split8(base + S::kB + (c >> 3) * kTileB, NH * kTileB, r, c & 7, q);
  }
  for (int e = tid; e < kFR * DK; e += kFTh) {      // W^T: row = latent column, K-major over d
    const int c = e % kFR, j = e / kFR;
    *reinterpret_cast<__nv_bfloat16*>(base + S::kW + (j >> 6) * (kFR * 128) + tile_off(c, (j & 63) >> 3) +
                                      (j & 7) * 2) = W[e];
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  bool ok = true;
  if (tid == 0) {   // latent [128 x 64] = sum_i Qbar_i . W, fp32 in TMEM columns [0, 64)
    constexpr uint32_t id_lat = idesc_bf16(128, kFR, false, false);
    int n = 0;
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t koff = (uint32_t)((kk & 3) * 32);
        const uint64_t da = sdesc_sw128(sbase + S::kB + (i * NH + (kk >> 2)) * kTileB + koff, 16, 1024);
        const uint64_t db = sdesc_sw128(sbase + S::kW + (kk >> 2) * (kFR * 128) + koff, 16, 1024);
        tc_mma(tmem, da, db, id_lat, n++ > 0 ? 1u : 0u);
      }
    tc_commit(smem_u32(&s_mbar[2]));
  }
  ok = __syncthreads_and(mbar_wait(smem_u32(&s_mbar[2]), 0));
  tc_fence_after();
  const int64_t t = t0 + row;
  const int64_t qpos = t < a.T ? (a.q_pos ? (int64_t)a.q_pos[t] : (int64_t)LLONG_MAX) : -1;
  // the same test as min position <= qpos, in 32 bits (every position fits an int32)
  const int32_t qlim = (int32_t)min64(qpos, (int64_t)INT32_MAX);
  const bool qok = qpos >= 0;
  if (ok) {   // this thread's half of its query's latent: split into the three A tiles
    float lat[32];
    tmem_ld32(tmem + lane_base + hf * 32, lat);
    if (a.qlat_out && t < a.T) {
      float* qo = a.qlat_out + (t * a.Hkv + g) * kFR + hf * 32;
#pragma unroll
      for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(qo + c) = make_float4(lat[c], lat[c + 1], lat[c + 2], lat[c + 3]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = lat[c * 8 + e];
      store_split8(base + S::kA, kTileB, row, hf * 4 + c, x);
    }
  }

  // ---- main loop over tiles of kFN leaves ----
  const int ntile = (int)ceil_div(NL, kFN);
  // the best 32 keys of this thread's query, sorted descending (0 = empty), in registers
  unsigned long long top[kFMaxB];
#pragma unroll
  for (int i = 0; i < kFMaxB; ++i) top[i] = 0ull;
  unsigned long long tau = 0ull;      // top[31]: a key must beat it to enter
  bool bad = false;
  int32_t cmp = 0, cleaf = -1;
  // fp32 centroid rows are staged with cp.async in the list region (row tid, its 16-byte
  // chunks XOR-swizzled by the row so that the row reads spread over the banks)
  char* stage = base + S::kList + row * (kFR * 4);
  auto stage_off = [&](int f) { return (uint32_t)((f ^ (row & 15)) << 4); };
  // tile j holds the leaves (i * perm) mod NL for i in [j kFN, (j + 1) kFN): neighbouring
  // leaves score alike, and a scan in tree order would raise each query's threshold slowly
  auto load_row = [&](int j) {
    const int64_t i = (int64_t)j * kFN + row;
    const int64_t l = i < NL ? (i * a.flat_perm) % NL : 0;
    cleaf = i < NL ? (int32_t)l : -1;
    const float* src = cent + l * kFR;
#pragma unroll
    for (int ff = 0; ff < kFR / 8; ++ff) {   // this half's 8 of the row's 16 chunks
      const int f = hf * (kFR / 8) + ff;
      cp_async16(smem_u32(stage + stage_off(f)), src + 4 * f);
    }
    cp_async_commit();
    cmp = __ldg(&mpos[l]);
  };
  auto store_row = [&](int j) {
    const int buf = j & 1;
    char* bt = base + S::kB + buf * 3 * kTileB;
    cp_async_wait_prev_n<0>();
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = hf * 4 + cc;
      const float4 u = *reinterpret_cast<const float4*>(stage + stage_off(2 * c));
      const float4 v = *reinterpret_cast<const float4*>(stage + stage_off(2 * c + 1));
      const float x[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
      store_split8(bt, kTileB, row, c, x);
    }
    if (hf == 0) s_ml[buf * kFN + row] = make_int2(cmp, cleaf);
  };
  auto issue = [&](int j) {           // one thread: the six products of tile j
    const int buf = j & 1;
    const uint32_t bt = sbase + S::kB + buf * 3 * kTileB;
    constexpr uint32_t id_s = idesc_bf16(128, kFN, false, false);
    constexpr int pi[6] = {0, 0, 1, 0, 1, 2}, pj[6] = {0, 1, 0, 2, 1, 0};
    tc_fence_after();
#pragma unroll
    for (int p = 0; p < 6; ++p)
#pragma unroll
      for (int kk = 0; kk < kFR / 16; ++kk) {
        const uint32_t koff = (uint32_t)(kk * 32);
        tc_mma(tmem + buf * kFN, sdesc_sw128(sbase + S::kA + pi[p] * kTileB + koff, 16, 1024),
               sdesc_sw128(bt + pj[p] * kTileB + koff, 16, 1024), id_s, (p | kk) ? 1u : 0u);
      }
    tc_commit(smem_u32(&s_mbar[buf]));
  };
  if (ok) {
    load_row(0);
    store_row(0);
    if (ntile > 1) load_row(1);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (ok && tid == 0) issue(0);
  for (int j = 0; j < ntile && ok; ++j) {
    if (j + 1 < ntile) {
      // buffer (j + 1) & 1 was read by the products of tile j - 1, which completed
      // before the scores of tile j - 1 were read; its TMEM columns are free too
      store_row(j + 1);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) issue(j + 1);
      if (j + 2 < ntile) load_row(j + 2);
    }
    ok = __syncthreads_and(mbar_wait(smem_u32(&s_mbar[j & 1]), (uint32_t)(j >> 1) & 1u));
    tc_fence_after();
    if (!ok) break;
    const int buf = j & 1;
#pragma unroll 1
    for (int part = hf * 2; part < hf * 2 + 2; ++part) {   // this half's 64 columns
      float sc[32];
      tmem_ld32(tmem + buf * kFN + lane_base + part * 32, sc);   // every lane: .sync.aligned
      // candidates against the threshold at the start of the part (a later insert only
      // raises it, and a key below the current threshold leaves the list unchanged)
      uint32_t mask = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int2 ml = s_ml[buf * kFN + part * 32 + i];   // one 8-byte broadcast read
        const int32_t leaf = ml.y;
        const bool elig = qok && leaf >= 0 && ml.x <= qlim;
        const bool nan = isnan(sc[i]);
        bad |= elig && nan;
        const unsigned long long key =
            ((unsigned long long)orderable(sc[i]) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)leaf);
        mask |= (elig && !nan && key > tau) ? (1u << i) : 0u;
      }
      // one pending candidate per lane per pass through the insertion network: the warp
      // makes as many passes as its busiest lane has candidates (key 0 changes nothing)
      while (__any_sync(0xffffffffu, mask != 0u)) {
        unsigned long long key = 0ull;
        if (mask) {
          const int i = __ffs(mask) - 1;
          mask &= mask - 1u;
          const int32_t leaf = s_ml[buf * kFN + part * 32 + i].y;
          key = ((unsigned long long)orderable(pick32(sc, i)) << 32) |
                (unsigned long long)(0xffffffffu - (uint32_t)leaf);
        }
#pragma unroll
        for (int k = kFMaxB - 1; k > 0; --k) top[k] = top[k] > key ? top[k] : (top[k - 1] > key ? key : top[k - 1]);
        top[0] = top[0] > key ? top[0] : key;
        tau = top[kFMaxB - 1];
      }
    }
    tc_fence_before();
    __syncthreads();   // this tile's leaf ids and min positions are rewritten next iteration
  }
  cp_async_drain();    // nothing in flight into the staging rows (a timed-out loop may leave one)
  __syncthreads();     // every product has completed: the B tiles are free
  // each half's best 32 (B region, [2][32][128]), merged per query into the list region
  unsigned long long* halves = reinterpret_cast<unsigned long long*>(base + S::kB);
#pragma unroll
  for (int i = 0; i < kFMaxB; ++i) halves[(hf * kFMaxB + i) * kFT + row] = top[i];
  __syncthreads();
  unsigned long long* list = reinterpret_cast<unsigned long long*>(base + S::kList);   // [32][128]
  __shared__ int32_t s_nk[kFT];
  if (hf == 0) {
    int ia = 0, ib = 0, nkept = 0;
    for (int i = 0; i < kFMaxB; ++i) {
      const unsigned long long x = halves[ia * kFT + row], y = halves[(kFMaxB + ib) * kFT + row];
      const unsigned long long v = x > y ? x : y;
      if (x > y) ++ia; else ++ib;
      list[i * kFT + row] = v;
      nkept += (i < B && v != 0ull);
    }
    s_nk[row] = qpos >= 0 ? nkept : 0;
  }
  if (bad) s_bad = 1;
  if (!ok && tid == 0) set_status(a.status, LSA_ERR_TIMEOUT);
  __syncthreads();
  if (s_bad && tid == 0) set_status(a.status, LSA_ERR_NONFINITE);
  // outputs: kept leaves in key order (-1 pads), then their keys
  if (hf == 0 && qpos >= 0 && a.leaves_out) {
    const int nkept = s_nk[row];
    for (int i = 0; i < B; ++i)
      a.leaves_out[((int64_t)g * a.T + t) * B + i] =
          i < nkept ? (int32_t)(0xffffffffu - (uint32_t)(list[i * kFT + row] & 0xffffffffull)) : -1;
  }
  if (a.idx_out) {
    const int lane = tid & 31;
    const int leafn = a.leaf;
    const int64_t K_sel = (int64_t)B * leafn;
    const int32_t* li = reinterpret_cast<const int32_t*>(a.tree + a.off_leaf) + (int64_t)g * a.n_tree;
    for (int r = warp; r < kFT; r += kFTh / 32) {
      const int64_t tr = t0 + r;
      if (tr >= a.T) break;
      const int nk = s_nk[r];
      int32_t* out = a.idx_out + ((int64_t)g * a.T + tr) * K_sel;
      for (int64_t i = lane; i < K_sel; i += 32) {
        const int k = (int)(i / leafn), q = (int)(i % leafn);
        int32_t v = -1;
        if (k < nk) {
          const int32_t lf = (int32_t)(0xffffffffu - (uint32_t)(list[k * kFT + r] & 0xffffffffull));
          v = __ldg(&li[(int64_t)lf * leafn + q]);
        }
        out[i] = v;
      }
    }
  }
  // every product issued above has completed before TMEM is released
  if (tid == 0) tc_commit(smem_u32(&s_mbar[2]));
  mbar_wait(smem_u32(&s_mbar[2]), 1);
  tc_fence_after();
  __syncthreads();
  free_tmem(tmem, 2 * kFN);
}

}  // namespace

bool select_flat_tc_supported(const SelectArgs& a, int dtype) {
  const int L = a.levels - 1;
  return dtype == LSA_BF16 && a.r == kFR && (a.d == 64 || a.d == 128) && a.beam[L] <= kFMaxB;
}

cudaError_t run_select_flat_tc(const SelectArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const dim3 grid((unsigned)ceil_div(a.T, kFT), (unsigned)a.Hkv);
#define LSA_FLAT_TC(DD)                                                                                       \
  if (a.d == DD) {                                                                                            \
    const size_t smem = FlatTcSmem<DD>::kBytes;                                                               \
    cudaError_t e = cudaFuncSetAttribute(k_select_flat_tc<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                         (int)smem);                                                          \
    if (e != cudaSuccess) return e;                                                                           \
    k_select_flat_tc<DD><<<grid, kFTh, smem, st>>>(a);                                                         \
    return cudaGetLastError();                                                                                \
  }
  LSA_FLAT_TC(64) LSA_FLAT_TC(128)
#undef LSA_FLAT_TC
  return cudaErrorInvalidValue;
}

}  // namespace lsa
