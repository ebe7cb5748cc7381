// project.cu -- latent projection of the keys on the tensor cores.
//
// kongchang.com, "Latent Sparse Attention Breaks Through the Million-Token
// Context Bottleneck", section "How LSA Sidesteps Per-Key Scoring with
// Hierarchical Clustering": keys are first mapped into a low-dimensional latent
// space, and the tree is built there.  Per KV head h and key i:
//     Z[h][i][c] = sum_j K[h][i][j] * W[h][j][c],   pos[h][i] = i.
//
// For bf16 keys and weights this is a dense [n x d] . [d x r] product with r a
// multiple of 16, so it runs as tcgen05.mma kind::f16 (bf16 x bf16 products are
// exact in fp32; only the order of the fp32 sums differs from a sequential loop).
// One persistent CTA per SM walks a contiguous range of 128-key tiles:
//   * K tiles (128 rows x d, 128-byte swizzled, K-major) stream through a ring of
//     kStages shared-memory stages with 16-byte cp.async (a tile of a head is one
//     contiguous block of 128 * d * 2 bytes in HBM);
//   * W[h] is held transposed ([r rows x d], K-major) in shared memory and reloaded
//     only when the range crosses into the next head;
//   * one thread issues the d/16 MMAs (M = 128, N = r, K = 16) into r TMEM columns
//     and commits them to an mbarrier; the 128 threads then read their row from
//     TMEM (thread = TMEM lane = key) and store it with 16-byte stores.
// Algorithmic bytes per key: d * 2 read + r * 4 + 4 written.
#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tc_sm100.cuh"

namespace lsa {

namespace {

constexpr int kPT = 128;       // threads per CTA = keys per tile = TMEM lanes
constexpr int kStages = 4;     // K-tile ring depth

template <int R, int DK>
struct ProjSmem {
  static constexpr uint32_t kTile = kPT * DK * 2;          // one K tile (bytes)
  static constexpr uint32_t kW = R * DK * 2;               // W[h] transposed
  static constexpr size_t kBytes = 1024 + (size_t)kStages * kTile + kW;
};

// R fp32 columns of this thread's TMEM lane (R = 16, 32 or 64).
template <int R>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[R]) {
  if constexpr (R == 16) {
    tmem_ld16(taddr, v);
  } else {
#pragma unroll
    for (int p = 0; p < R / 32; ++p) {
      float t[32];
      tmem_ld32(taddr + p * 32, t);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[p * 32 + i] = t[i];
    }
  }
}

template <int R, int DK>
__global__ void __launch_bounds__(kPT, 1)
    k_project_tc(const __nv_bfloat16* __restrict__ K, int64_t n_cap, const __nv_bfloat16* __restrict__ W,
                 int64_t n, int32_t n_heads, float* __restrict__ Z, int32_t* __restrict__ pos,
                 int32_t* __restrict__ status) {
  using S = ProjSmem<R, DK>;
  constexpr int kChunks = DK / 8;                  // 16-byte chunks per key row
  constexpr uint32_t kTmemCols = R < 32 ? 32 : R;  // allocation: a power of two >= 32
  extern __shared__ char smem_raw[];
  __shared__ __align__(8) uint64_t s_mbar;
  __shared__ uint32_t s_taddr;
  char* base = align1024(smem_raw);
  const uint32_t sK = smem_u32(base);
  const uint32_t sW = sK + kStages * S::kTile;
  const uint32_t mbar = smem_u32(&s_mbar);
  const int tid = threadIdx.x, warp = tid >> 5;

  // this CTA's contiguous range of (head, tile) pairs, head-major
  const int64_t tiles_per_head = ceil_div(n, kPT);
  const int64_t total = tiles_per_head * n_heads;
  const int64_t t_lo = total * blockIdx.x / gridDim.x, t_hi = total * (blockIdx.x + 1) / gridDim.x;
  const int64_t my = t_hi - t_lo;
  if (my <= 0) return;

  if (tid == 0) {
    mbar_init(mbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  alloc_tmem(&s_taddr, kTmemCols);

  // copy tile k of the range into stage k % kStages (rows past n repeat row n - 1)
  auto load_tile = [&](int64_t k) {
    const int64_t t = t_lo + k;
    const int64_t h = t / tiles_per_head, row0 = (t % tiles_per_head) * kPT;
    const __nv_bfloat16* Kh = K + h * n_cap * DK;
    const uint32_t dst = sK + (uint32_t)(k % kStages) * S::kTile;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int q = tid + i * kPT;
      const int r = q / kChunks, c = q % kChunks;
      const int64_t row = min64(row0 + r, n - 1);
      cp_async16(dst + sw128_off(r, c, kPT * 128), Kh + row * DK + c * 8);
    }
  };
  // W[h] transposed into sW: row c (latent column), K-major over d
  auto load_w = [&](int64_t h) {
    const __nv_bfloat16* Wh = W + h * DK * R;
    char* w = reinterpret_cast<char*>(base) + kStages * S::kTile;
    for (int e = tid; e < R * DK; e += kPT) {
      const int c = e % R, j = e / R;
      *reinterpret_cast<__nv_bfloat16*>(w + sw128_off(c, j >> 3, R * 128) + (j & 7) * 2) = Wh[e];
    }
  };

#pragma unroll
  for (int k = 0; k < kStages - 1; ++k) {
    if (k < my) load_tile(k);
    cp_async_commit();
  }
  int64_t w_head = -1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t idesc = idesc_bf16(128, R, false, false);
  bool ok = true;
  uint32_t phase = 0;
  for (int64_t k = 0; k < my && ok; ++k, phase ^= 1) {
    const int64_t t = t_lo + k;
    const int64_t h = t / tiles_per_head, row0 = (t % tiles_per_head) * kPT;
    // the stage of tile k - 1 is free: its MMA completed before the last epilogue
    if (k + kStages - 1 < my) load_tile(k + kStages - 1);
    cp_async_commit();
    if (h != w_head) {   // every MMA of the previous head has completed
      load_w(h);
      w_head = h;
    }
    cp_async_wait_prev_n<kStages - 1>();
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a0 = sK + (uint32_t)(k % kStages) * S::kTile;
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t koff = (uint32_t)((kk & 3) * 32);
        const uint64_t da = sdesc_sw128(a0 + (kk >> 2) * (kPT * 128) + koff, 16, 1024);
        const uint64_t db = sdesc_sw128(sW + (kk >> 2) * (R * 128) + koff, 16, 1024);
        tc_mma(tmem, da, db, idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(mbar);
    }
    ok = __syncthreads_and(mbar_wait(mbar, phase));
    tc_fence_after();
    if (ok) {
      float v[R];
      tmem_ld_row<R>(tmem + lane_base, v);
      const int64_t row = row0 + tid;
      if (row < n) {
        float* zr = Z + (h * n + row) * R;
#pragma unroll
        for (int c = 0; c < R; c += 4)
          *reinterpret_cast<float4*>(zr + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
        if (pos) pos[h * n + row] = (int32_t)row;
      }
    } else if (tid == 0) {
      set_status(status, LSA_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
  }
  cp_async_drain();
  if (!ok) mbar_wait(mbar, phase ^ 1);   // the phase that timed out (bounded): let a late MMA finish first
  tc_fence_after();
  free_tmem(tmem, kTmemCols);
}

}  // namespace

int sm_count() {
  static int count[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (!count[dev]) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c < 1) c = 148;
    count[dev] = c;
  }
  return count[dev];
}

bool project_tc_supported(int dtype, int r, int d) {
  return dtype == LSA_BF16 && (r == 16 || r == 32 || r == 64) && (d == 64 || d == 128);
}

cudaError_t run_project_tc(const void* K, int64_t n_cap, const void* W, int64_t n, int32_t n_heads, int r, int d,
                           float* Z, int32_t* pos, int32_t* status, cudaStream_t st) {
  if (n <= 0 || n_heads <= 0) return cudaSuccess;
  const int64_t tiles = ceil_div(n, kPT) * n_heads;
  const unsigned grid = (unsigned)min64(tiles, sm_count());
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(K);
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(W);
#define LSA_PROJ_TC(RR, DD)                                                                          \
  if (r == RR && d == DD) {                                                                          \
    const size_t smem = ProjSmem<RR, DD>::kBytes;                                                    \
    cudaError_t e = cudaFuncSetAttribute(k_project_tc<RR, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         (int)smem);                                                 \
    if (e != cudaSuccess) return e;                                                                  \
    k_project_tc<RR, DD><<<grid, kPT, smem, st>>>(k, n_cap, w, n, n_heads, Z, pos, status);          \
    return cudaGetLastError();                                                                       \
  }
  LSA_PROJ_TC(16, 64) LSA_PROJ_TC(32, 64) LSA_PROJ_TC(64, 64)
  LSA_PROJ_TC(16, 128) LSA_PROJ_TC(32, 128) LSA_PROJ_TC(64, 128)
#undef LSA_PROJ_TC
  return cudaErrorInvalidValue;
}

}  // namespace lsa
