// tree_attn.cu -- sparse attention over tree-structured selections, leaf by leaf.
//
// Method (kongchang.com, "Latent Sparse Attention Breaks Through the
// Million-Token Context Bottleneck", sections "How LSA Sidesteps Per-Key
// Scoring with Hierarchical Clustering" and "The Accuracy-Efficiency Dilemma";
// bdtechtalks.com, "Latent sparse attention", section "How latent sparse
// attention works"): each query attends to the original keys of the leaves its
// walk kept.  The result equals lsa_sparse_attn on the expanded key lists.
//
// Schedule: instead of gathering every query's 2048 keys (each selected leaf is
// re-read by every query that chose it), work is grouped by leaf: one CTA loads a
// leaf's 64 K and V rows once and serves every (query, head) row that selected
// it, with the products on the 5th-generation tensor cores (tcgen05.mma, bf16
// operands in 128B-swizzled shared memory, fp32 accumulators in tensor memory).
//   pass A: S = Q_rows . K_leaf^T -> per row, max and sum of exp over the leaf
//   combine: per (query, head) the softmax denominator over all its leaves
//   pass B: S again, P = exp(S - LSE) (bf16), O_rows += P . V_leaf (fp32 red-adds)
// Rows of one CTA chunk: up to 128 (query, head) pairs of queries that chose the
// leaf.  Shapes served here: bf16, d = 128, leaf size 64, G in {1, 2, 4, 8};
// other shapes expand the leaves into key lists and use the generic kernels.
#include <climits>
#include <cstring>

#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tc_sm100.cuh"

namespace lsa {

namespace {

constexpr int kTL = 128;            // threads per CTA (one TMEM lane / row each)
constexpr int kLeafKeys = 64;
constexpr int kDim = 128;

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  atomicAdd(reinterpret_cast<float4*>(p), make_float4(a, b, c, d));
}

struct TreeAttnArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const int32_t* leaf_index;   // [H][n_tree]
  const int32_t* leaves;       // [H][T][B]
  const int32_t* q_pos;
  int32_t* cnt;                // [H][NL]
  int32_t* off;                // [H][NL + 1]
  int32_t* ent;                // [H][T * B] (query << 6 | rank), grouped by leaf
  float2* stats;               // [T][Hq][B] (max, sum) in base 2
  float* lse2;                 // [T][Hq]
  float* oacc;                 // [T][Hq][d] (red-add mode)
  __nv_bfloat16* part;         // [T][Hq][B][d] leaf outputs over their own exp-sum (partial mode)
  int32_t* entq;               // [H][T * B] query position of each entry (INT_MAX: not causal)
  int32_t* coff;               // [H][NL] first chunk of each leaf within its head
  int32_t* ctotal;             // [H] chunks per head
  int4* cdesc;                 // chunk descriptors {head, leaf, first entry, entries}
  int32_t epc;                 // entries per chunk (rows / G)
  int32_t n_sink, window;      // leaf keys in [0, n_sink) or [q_pos - window + 1, q_pos] are left out
  const __nv_bfloat16* Od;     // [T][Hq][d] attention over the sink and window keys (or null)
  const float* LSEd;           // [T][Hq] its natural-log softmax denominator
  __nv_bfloat16* O;
  float* LSE;
  int32_t* status;
  int64_t T, n_cap, n_tree, NL;
  int32_t Hq, H, G, B, causal;
  float scale_log2;
};

// ---- leaf lists (counting sort of (query, rank) by leaf) ---------------------

__global__ void k_tl_count(TreeAttnArgs a) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)a.H * a.T * a.B) return;
  const int64_t g = i / (a.T * a.B);
  const int32_t leaf = a.leaves[i];
  if (leaf >= 0 && leaf < a.NL) atomicAdd(&a.cnt[g * a.NL + leaf], 1);
}

// A thread's range of a single-CTA scan is read kScanBlk elements at a time, every
// load of a block issued before the first is used (a one-by-one loop would wait
// out one memory round trip per element).
constexpr int kScanBlk = 16;

// Elements [b0, b0 + kScanBlk) of p below hi (0 past it): a full, 16-byte aligned
// block is read with four unconditional 16-byte loads.
__device__ __forceinline__ void load_blk(const int32_t* p, int64_t b0, int64_t hi, int32_t (&v)[kScanBlk]) {
  if (b0 + kScanBlk <= hi && ((reinterpret_cast<uintptr_t>(p + b0) & 15) == 0)) {
#pragma unroll
    for (int k = 0; k < kScanBlk / 4; ++k) {
      const int4 x = reinterpret_cast<const int4*>(p + b0)[k];
      v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < kScanBlk; ++k) v[k] = b0 + k < hi ? p[b0 + k] : 0;
  }
}

__global__ void __launch_bounds__(1024) k_tl_scan(TreeAttnArgs a) {
  __shared__ int32_t s_warp[32];
  const int64_t g = blockIdx.x;
  int32_t* c = a.cnt + g * a.NL;
  int32_t* o = a.off + g * (a.NL + 1);
  const int64_t per = ceil_div(a.NL, 1024);
  const int64_t lo = min64(threadIdx.x * per, a.NL), hi = min64(a.NL, lo + per);
  int32_t s = 0;
  for (int64_t b0 = lo; b0 < hi; b0 += kScanBlk) {
    int32_t v[kScanBlk];
    load_blk(c, b0, hi, v);
#pragma unroll
    for (int k = 0; k < kScanBlk; ++k) s += v[k];
  }
  // block exclusive scan of the per-thread sums
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t inc = s;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int32_t y = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += y;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int32_t w = s_warp[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  int32_t run = inc - s + (warp ? s_warp[warp - 1] : 0);
  for (int64_t b0 = lo; b0 < hi; b0 += kScanBlk) {
    int32_t v[kScanBlk];
    load_blk(c, b0, hi, v);
#pragma unroll
    for (int k = 0; k < kScanBlk; ++k)
      if (b0 + k < hi) {
        o[b0 + k] = run;
        run += v[k];
        c[b0 + k] = 0;  // becomes the fill cursor
      }
  }
  if (threadIdx.x == 1023) o[a.NL] = s_warp[31];
}

__global__ void k_tl_fill(TreeAttnArgs a) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)a.H * a.T * a.B) return;
  const int64_t g = i / (a.T * a.B), rem = i % (a.T * a.B);
  const int64_t t = rem / a.B, k = rem % a.B;
  const int32_t leaf = a.leaves[i];
  if (leaf < 0 || leaf >= a.NL) return;
  const int32_t pos = a.off[g * (a.NL + 1) + leaf] + atomicAdd(&a.cnt[g * a.NL + leaf], 1);
  a.ent[g * a.T * a.B + pos] = (int32_t)((t << 6) | k);
  if (a.entq) a.entq[g * a.T * a.B + pos] = a.causal ? a.q_pos[t] : INT_MAX;
}

// Chunk lists for the pipelined pass: per head, the first chunk of each leaf
// (ceil(entries / epc) chunks per leaf) and the head's total.
__global__ void __launch_bounds__(1024) k_tl_cscan(TreeAttnArgs a) {
  __shared__ int32_t s_warp[32];
  const int64_t g = blockIdx.x;
  const int32_t* o = a.off + g * (a.NL + 1);
  int32_t* c = a.coff + g * a.NL;
  const int64_t per = ceil_div(a.NL, 1024);
  const int64_t lo = min64(threadIdx.x * per, a.NL), hi = min64(a.NL, lo + per);
  // chunks of leaf i: ceil((o[i + 1] - o[i]) / epc), blocks of kScanBlk leaves read at once
  auto chunks_of = [&](int64_t b0, int32_t (&v)[kScanBlk]) {
    int32_t e[kScanBlk];
    load_blk(o, b0, hi + 1, e);   // o[b0 .. min(b0 + kScanBlk, hi + 1)): o has NL + 1 entries
    const int32_t last = b0 + kScanBlk <= hi ? o[b0 + kScanBlk] : 0;
#pragma unroll
    for (int k = 0; k < kScanBlk; ++k) {
      const int32_t next = k + 1 < kScanBlk ? e[k + 1] : last;
      v[k] = b0 + k < hi ? (next - e[k] + a.epc - 1) / a.epc : 0;
    }
  };
  int32_t s = 0;
  for (int64_t b0 = lo; b0 < hi; b0 += kScanBlk) {
    int32_t v[kScanBlk];
    chunks_of(b0, v);
#pragma unroll
    for (int k = 0; k < kScanBlk; ++k) s += v[k];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t inc = s;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int32_t y = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += y;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int32_t w = s_warp[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  int32_t run = inc - s + (warp ? s_warp[warp - 1] : 0);
  for (int64_t b0 = lo; b0 < hi; b0 += kScanBlk) {
    int32_t v[kScanBlk];
    chunks_of(b0, v);
#pragma unroll
    for (int k = 0; k < kScanBlk; ++k)
      if (b0 + k < hi) {
        c[b0 + k] = run;
        run += v[k];
      }
  }
  if (threadIdx.x == 1023) a.ctotal[g] = s_warp[31];
}

__global__ void k_tl_chunks(TreeAttnArgs a) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)a.H * a.NL) return;
  const int64_t g = i / a.NL, leaf = i % a.NL;
  int64_t base = a.coff[i];
  for (int64_t h = 0; h < g; ++h) base += a.ctotal[h];
  const int32_t e0 = a.off[g * (a.NL + 1) + leaf], n = a.off[g * (a.NL + 1) + leaf + 1] - e0;
  for (int32_t c = 0; c * a.epc < n; ++c)
    a.cdesc[base + c] = make_int4((int)g, (int)leaf, e0 + c * a.epc, min(a.epc, n - c * a.epc));
}

// ---- shared pieces of the two passes ----------------------------------------

struct LeafSmem {
  uint32_t sA, sK, sV, sP;       // shared addresses (1024-B aligned)
  int32_t* pos;                  // [64] key positions of the leaf
  uint32_t mbar;
  uint32_t* taddr_slot;
};

// This thread's row of a chunk: query index (or -1), rank of the leaf in that
// query's list, and head within the group.
__device__ __forceinline__ void row_of(const TreeAttnArgs& a, const int32_t* ent, int64_t n_ent, int64_t e0,
                                       int64_t& tq, int& rank, int& h) {
  const int64_t e = e0 + threadIdx.x / a.G;
  h = threadIdx.x % a.G;
  tq = -1;
  rank = 0;
  if (e < n_ent) {
    const int32_t v = ent[e];
    tq = v >> 6;
    rank = v & 63;
  }
}

// Copy this thread's query row into row threadIdx.x of the A tile.
__device__ __forceinline__ void copy_row(const TreeAttnArgs& a, int64_t g, int64_t tq, int h, uint32_t sA) {
  if (tq < 0) return;
  const __nv_bfloat16* q = a.Q + (tq * a.Hq + g * a.G + h) * kDim;
#pragma unroll
  for (int c = 0; c < 16; ++c) cp_async16(sA + sw128_off(threadIdx.x, c, kTL * 128), q + c * 8);
}

// Copy the leaf's K (and V) rows (positions already in smem) into the tiles.
__device__ __forceinline__ void copy_leaf(const TreeAttnArgs& a, int64_t g, const LeafSmem& s, bool with_v) {
  const __nv_bfloat16* Kh = a.K + g * a.n_cap * kDim;
  const __nv_bfloat16* Vh = a.V + g * a.n_cap * kDim;
  const int r = threadIdx.x >> 1, c0 = (threadIdx.x & 1) * 8;
  const int64_t j = s.pos[r];
#pragma unroll
  for (int c = c0; c < c0 + 8; ++c) {
    cp_async16(s.sK + sw128_off(r, c, kLeafKeys * 128), Kh + j * kDim + c * 8);
    if (with_v) cp_async16(s.sV + sw128_off(r, c, kLeafKeys * 128), Vh + j * kDim + c * 8);
  }
}

// S[128 rows x 64 keys] = A . K_leaf^T into TMEM columns [col, col + 64).
__device__ __forceinline__ void issue_qk(const LeafSmem& s, uint32_t tmem, int col) {
  constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t koff = (uint32_t)((kk & 3) * 32);
    const uint64_t da = sdesc_sw128(s.sA + (kk >> 2) * (kTL * 128) + koff, 16, 1024);
    const uint64_t db = sdesc_sw128(s.sK + (kk >> 2) * (kLeafKeys * 128) + koff, 16, 1024);
    tc_mma(tmem + col, da, db, idesc, kk > 0 ? 1u : 0u);
  }
}

// Number of a leaf's keys visible at query position qp.  A leaf lists its keys
// in ascending position order (the index build keeps position order inside
// every node), so the visible keys are a prefix; a branch-free binary search
// finds its length and the masks below are register compares.
__device__ __forceinline__ int visible_prefix(const int32_t* pos, int64_t qp) {
  if ((int64_t)pos[kLeafKeys - 1] <= qp) return kLeafKeys;
  int c = 0;   // < 64 from here on: steps 32 + 16 + ... + 1 reach 63 at most
#pragma unroll
  for (int step = kLeafKeys / 2; step; step >>= 1)
    if ((int64_t)pos[c + step - 1] <= qp) c += step;
  return c;
}

// This thread's 64 scores (base-2 scaled, causally masked) from TMEM.
__device__ __forceinline__ void read_scores(const TreeAttnArgs& a, const LeafSmem& s, uint32_t tmem, int64_t tq,
                                            float (&sc)[64]) {
  const int warp = threadIdx.x >> 5;
  float v[32];
  const int64_t qp = (a.causal && tq >= 0) ? (int64_t)a.q_pos[tq] : INT64_MAX;
  const int nvis = visible_prefix(s.pos, qp);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + half * 32, v);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int key = half * 32 + i;
      sc[key] = key < nvis ? v[i] * a.scale_log2 : -INFINITY;
    }
  }
}

// ---- pass A: per-row max and exp-sum over each selected leaf -----------------

__global__ void __launch_bounds__(kTL) k_tl_stats(TreeAttnArgs a) {
  extern __shared__ char smem_raw[];
  __shared__ int32_t s_pos[kLeafKeys];
  __shared__ __align__(8) uint64_t s_mbar;
  __shared__ uint32_t s_taddr;
  const int64_t g = blockIdx.y, leaf = blockIdx.x;
  const int32_t* offg = a.off + g * (a.NL + 1);
  const int64_t e_lo = offg[leaf], n_ent = offg[leaf + 1] - e_lo;
  if (n_ent == 0) return;
  const int32_t* ent = a.ent + g * a.T * a.B + e_lo;
  char* base = align1024(smem_raw);
  LeafSmem s;
  s.sA = smem_u32(base);
  s.sK = s.sA + kTL * 256;
  s.sV = 0;
  s.sP = 0;
  s.pos = s_pos;
  s.mbar = smem_u32(&s_mbar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(s.mbar));
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  // first chunk's row and the leaf's key positions: independent loads in flight together
  int64_t tq;
  int rank, h;
  row_of(a, ent, n_ent, 0, tq, rank, h);
  if (threadIdx.x < kLeafKeys) s_pos[threadIdx.x] = a.leaf_index[g * a.n_tree + leaf * kLeafKeys + threadIdx.x];
  __syncthreads();
  copy_leaf(a, g, s, false);
  alloc_tmem(&s_taddr, 64);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;
  uint32_t phase = 0;
  bool ok = true;
  for (int64_t e0 = 0; e0 < n_ent && ok; e0 += kTL / a.G) {
    if (e0 > 0) row_of(a, ent, n_ent, e0, tq, rank, h);
    copy_row(a, g, tq, h, s.sA);
    cp_async_wait_all();
    fence_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_qk(s, tmem, 0);
      tc_commit(s.mbar);
    }
    ok = __syncthreads_and(mbar_wait(s.mbar, phase));
    phase ^= 1;
    tc_fence_after();
    if (ok) {
      float sc[64];
      read_scores(a, s, tmem, tq, sc);
      if (tq >= 0) {
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < 64; ++i) m = fmaxf(m, sc[i]);
        float l = 0.f;
        if (m != -INFINITY) {
#pragma unroll
          for (int i = 0; i < 64; ++i) l += exp2f(sc[i] - m);
        }
        a.stats[(tq * a.Hq + g * a.G + h) * a.B + rank] = make_float2(m, l);
      }
    } else {
      set_status(a.status, LSA_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
  }
  free_tmem(tmem, 64);
}

// ---- combine: softmax denominator of every (query, head) over its leaves -----

__global__ void k_tl_lse(TreeAttnArgs a) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // t * Hq + head
  if (row >= a.T * a.Hq) return;
  const int64_t t = row / a.Hq, head = row % a.Hq, g = head / a.G;
  const int32_t* lv = a.leaves + (g * a.T + t) * a.B;
  const float2* st = a.stats + row * a.B;
  float M = -INFINITY;
  for (int k = 0; k < a.B; ++k)
    if (lv[k] >= 0) M = fmaxf(M, st[k].x);
  float L = 0.f;
  if (M != -INFINITY)
    for (int k = 0; k < a.B; ++k)
      if (lv[k] >= 0 && st[k].y > 0.f) L += st[k].y * exp2f(st[k].x - M);
  a.lse2[row] = L > 0.f ? M + log2f(L) : INFINITY;   // +inf: no visible key, P = 0
  a.LSE[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

// ---- pass B: O_rows += softmax(S) . V_leaf ------------------------------------

__global__ void __launch_bounds__(kTL) k_tl_out(TreeAttnArgs a) {
  extern __shared__ char smem_raw[];
  __shared__ int32_t s_pos[kLeafKeys];
  __shared__ __align__(8) uint64_t s_mbar;
  __shared__ uint32_t s_taddr;
  const int64_t g = blockIdx.y, leaf = blockIdx.x;
  const int32_t* offg = a.off + g * (a.NL + 1);
  const int64_t e_lo = offg[leaf], n_ent = offg[leaf + 1] - e_lo;
  if (n_ent == 0) return;
  const int32_t* ent = a.ent + g * a.T * a.B + e_lo;
  char* base = align1024(smem_raw);
  LeafSmem s;
  s.sA = smem_u32(base);                       // 32 KB: rows x d
  s.sK = s.sA + kTL * 256;                     // 16 KB
  s.sV = s.sK + kLeafKeys * 256;               // 16 KB
  s.sP = s.sA;                                 // P (rows x 64 keys) overwrites the consumed Q tile
  s.pos = s_pos;
  s.mbar = smem_u32(&s_mbar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(s.mbar));
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  // first chunk's row (and its LSE) and the leaf's key positions in flight together
  int64_t tq;
  int rank, h;
  row_of(a, ent, n_ent, 0, tq, rank, h);
  float lse = tq >= 0 ? a.lse2[tq * a.Hq + g * a.G + h] : INFINITY;
  if (threadIdx.x < kLeafKeys) s_pos[threadIdx.x] = a.leaf_index[g * a.n_tree + leaf * kLeafKeys + threadIdx.x];
  __syncthreads();
  copy_leaf(a, g, s, true);
  alloc_tmem(&s_taddr, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;
  const int warp = threadIdx.x >> 5;
  uint32_t phase = 0;
  bool ok = true;
  char* sP_gen = base;
  for (int64_t e0 = 0; e0 < n_ent && ok; e0 += kTL / a.G) {
    if (e0 > 0) {
      row_of(a, ent, n_ent, e0, tq, rank, h);
      lse = tq >= 0 ? a.lse2[tq * a.Hq + g * a.G + h] : INFINITY;
    }
    copy_row(a, g, tq, h, s.sA);
    cp_async_wait_all();
    fence_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_qk(s, tmem, 0);
      tc_commit(s.mbar);
    }
    ok = __syncthreads_and(mbar_wait(s.mbar, phase));
    phase ^= 1;
    tc_fence_after();
    if (ok) {
      float sc[64];
      read_scores(a, s, tmem, tq, sc);
      // P row (bf16) into the K-major A tile of the second product
      const int r = threadIdx.x;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p0 = exp2f(sc[c * 8 + 2 * q] - lse), p1 = exp2f(sc[c * 8 + 2 * q + 1] - lse);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          w[q] = *reinterpret_cast<uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(sP_gen + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (ok && threadIdx.x == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc_sw128(s.sP + kk * 32, 16, 1024);
        const uint64_t db = sdesc_sw128(s.sV + kk * 2048, kLeafKeys * 128, 1024);
        tc_mma(tmem, da, db, idesc, kk > 0 ? 1u : 0u);   // O over S's columns: S is in P now
      }
      tc_commit(s.mbar);
    }
    if (ok) {
      ok = __syncthreads_and(mbar_wait(s.mbar, phase));
      phase ^= 1;
    }
    tc_fence_after();
    if (ok) {
      // every lane takes part in the (warp-collective) TMEM loads; only rows of
      // real queries are added to the output
      float* dst = tq >= 0 ? a.oacc + (tq * a.Hq + g * a.G + h) * kDim : nullptr;
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + part * 32, v);
        if (dst) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) red_add_v4(dst + part * 32 + i, v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
    } else {
      set_status(a.status, LSA_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
  }
  free_tmem(tmem, 128);
}

__global__ void k_tl_finish(TreeAttnArgs a) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.T * a.Hq * (kDim / 4)) return;
  const float4 v = reinterpret_cast<const float4*>(a.oacc)[i];
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  reinterpret_cast<uint2*>(a.O)[i] = w;
}

// ---- partial mode: per (row, leaf) partial outputs, then combine ---------------
//
// Each (row, leaf) pair writes its leaf max m (base 2), exp-sum l and the
// leaf output P.V / l with P = exp2(S - m), rounded to bf16 (a convex
// combination of the leaf's V rows, so bf16 keeps it to 2^-9 of their scale);
// k_tl_combine merges a row's leaves with weights 2^(m - M) l.  No pass over the
// statistics first and no atomics, at the cost of T * Hq * n_leaves * d * 2
// bytes of partials.

// One warp per (query, head) row: O = sum_k w_k o_k / sum_k w_k with
// w_k = 2^(m_k - M) l_k over the row's leaves, in a fixed order (even ranks and
// odd ranks, each in rank order, then their sum).
// 16 bytes through the non-coherent path; volatile, so that every partial of a row
// is requested before the first is used (the compiler would otherwise sink each
// load to its use and keep only a few in flight)
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__global__ void k_tl_combine(TreeAttnArgs a) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;   // t * Hq + head
  const int lane = threadIdx.x & 31;
  if (row >= a.T * a.Hq) return;
  const int64_t t = row / a.Hq, head = row % a.Hq, g = head / a.G;
  // half-warp h reads the partials of ranks h, h + 2, ...; lane (mod 16) owns dims
  // [8 (lane mod 16), +8); all of them are requested at once, with the statistics
  // (ranks without a partial are read too, the workspace is readable, and skipped)
  const int half = lane >> 4, sl = lane & 15;
  const __nv_bfloat16* pr = a.part + row * a.B * kDim + sl * 8;
  uint4 raw[LSA_MAX_BEAM / 2];
#pragma unroll
  for (int i = 0; i < LSA_MAX_BEAM / 2; ++i) {
    const int k = 2 * i + half;
    raw[i] = k < a.B ? ld_nc_v4(pr + (int64_t)k * kDim) : make_uint4(0u, 0u, 0u, 0u);
  }
  bool valid = false;
  float mk = -INFINITY, lk = 0.f;
  if (lane < a.B && a.leaves[(g * a.T + t) * a.B + lane] >= 0) {
    const float2 st = a.stats[row * a.B + lane];
    valid = st.y > 0.f;
    mk = st.x;
    lk = st.y;
  }
  // the sink/window part (if any) is one more partial: base-2 max = its LSE / ln 2, l = 1
  const float md = a.LSEd ? a.LSEd[row] * 1.44269504088896340736f : -INFINITY;
  float M = valid ? mk : -INFINITY;
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  M = fmaxf(M, md);
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  const float wk = valid ? exp2f(mk - M) * lk : 0.f;
  // L: butterfly sum (each step adds the same two values on both lanes: every lane
  // ends with the same bits)
  float L = wk;
#pragma unroll
  for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int i = 0; i < LSA_MAX_BEAM / 2; ++i) {   // this half's ranks in order
    const int k = 2 * i + half;
    const float w = __shfl_sync(0xffffffffu, wk, k & 31);
    if ((vmask >> k) & 1u) {
      const uint32_t wd[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[q]));
        acc[2 * q] = fmaf(w, f.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(w, f.y, acc[2 * q + 1]);
      }
    }
  }
  // even ranks + odd ranks (the same sum on both halves)
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  if (md != -INFINITY) {   // after the leaves, in a fixed order
    const float w = exp2f(md - M);
    float v0[4], v1[4];
    load4(a.Od + row * kDim + sl * 8, v0);
    load4(a.Od + row * kDim + sl * 8 + 4, v1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[e] = fmaf(w, v0[e], acc[e]);
      acc[e + 4] = fmaf(w, v1[e], acc[e + 4]);
    }
    L += w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (half == 0) {
    uint32_t w4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q] * inv, acc[2 * q + 1] * inv);
      w4[q] = *reinterpret_cast<uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(a.O + row * kDim + sl * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  if (lane == 0) a.LSE[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

// ---- dense part: the sink and window keys, tile by tile -----------------------
//
// A CTA holds kTL rows, (query, head) pairs of one KV group: 128 / G consecutive
// queries with their G heads.  Each row attends densely to the sink [0, n_sink)
// and the window (q_pos - window, q_pos], each key once and none past q_pos or
// the cache.  The CTA walks the 64-position key blocks that any of its rows
// needs, twice: first for every row's softmax max and sum, then for
// P = 2^(s - lse) and O = P.V on the tensor cores (O already normalised).

struct BandArgs {
  const __nv_bfloat16 *Q, *K, *V;
  const int32_t* q_pos;
  __nv_bfloat16* Od;           // [T][Hq][d]
  float* LSEd;                 // [T][Hq] natural log (-inf: no dense key)
  int32_t* status;
  int64_t T, n_cap;
  int32_t Hq, H, G, n_sink, window;
  float scale_log2;
};
constexpr size_t kBandSmem = 1024 + kTL * 256 + 4 * kLeafKeys * 256;   // Q 32 KB; two {K, V} buffers

__global__ void __launch_bounds__(kTL) k_tl_band(BandArgs a) {
  extern __shared__ char smem_raw[];
  __shared__ __align__(8) uint64_t s_mbar;
  __shared__ uint32_t s_taddr;
  __shared__ int32_t s_red[kTL / 32];
  char* base = align1024(smem_raw);
  // two buffers of {K, V} (16 KB each): a block's copies land in one while the
  // previous block is computed from the other; P overlays the K tile of its own
  // block once S = Q.K^T has completed
  auto gK = [&](int buf) { return base + kTL * 256 + buf * 2 * kLeafKeys * 256; };
  auto gV = [&](int buf) { return gK(buf) + kLeafKeys * 256; };
  LeafSmem s;
  s.sA = smem_u32(base);
  s.mbar = smem_u32(&s_mbar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = blockIdx.y;
  const int64_t t = (int64_t)blockIdx.x * (kTL / a.G) + threadIdx.x / a.G;
  const int hh = threadIdx.x % a.G;
  const bool valid = t < a.T;
  const int64_t q = valid ? (int64_t)a.q_pos[t] : -1;
  // this row's dense keys: [0, s_hi) and [w_lo, w_hi]
  const int64_t s_hi = valid ? min(min((int64_t)a.n_sink, a.n_cap), q + 1) : 0;
  const int64_t w_lo = max(max(q - a.window + 1, (int64_t)a.n_sink), (int64_t)0);
  const int64_t w_hi = valid && a.window > 0 ? min(q, a.n_cap - 1) : -1;
  // first block at or after b that this row needs (INT_MAX: none)
  auto next_block = [&](int b) -> int {
    if ((int64_t)b * kLeafKeys < s_hi) return b;
    if (w_lo <= w_hi && (int64_t)b <= (w_hi >> 6)) return (int)max((int64_t)b, w_lo >> 6);
    return INT_MAX;
  };
  auto cta_min = [&](int v) -> int {
    v = __reduce_min_sync(0xffffffffu, v);
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    int r = s_red[0];
#pragma unroll
    for (int w = 1; w < kTL / 32; ++w) r = min(r, s_red[w]);
    __syncthreads();
    return r;
  };
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(s.mbar));
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  // positions past every row's query are never attended, and the cache rows there
  // may hold anything: their V rows are zeros (0 x NaN would still be NaN)
  const int64_t qmax = -(int64_t)cta_min(valid ? -(int)q : INT_MAX);
  if (valid) {   // lands with the first block's group
    const __nv_bfloat16* qr = a.Q + (t * a.Hq + g * a.G + hh) * kDim;
#pragma unroll
    for (int c = 0; c < 16; ++c) cp_async16(s.sA + sw128_off(threadIdx.x, c, kTL * 128), qr + c * 8);
  }
  // copies of block b into buffer buf (issued, not waited for)
  auto load_block = [&](int b, int buf, bool with_v) {
    const int r = threadIdx.x >> 1, c0 = (threadIdx.x & 1) * 8;
    const int64_t j = (int64_t)b * kLeafKeys + r;
    const uint32_t sK = smem_u32(gK(buf)), sV = smem_u32(gV(buf));
    if (j <= qmax && j < a.n_cap) {
      const __nv_bfloat16* kr = a.K + (g * a.n_cap + j) * kDim;
      const __nv_bfloat16* vr = a.V + (g * a.n_cap + j) * kDim;
#pragma unroll
      for (int c = c0; c < c0 + 8; ++c) {
        cp_async16(sK + sw128_off(r, c, kLeafKeys * 128), kr + c * 8);
        if (with_v) cp_async16(sV + sw128_off(r, c, kLeafKeys * 128), vr + c * 8);
      }
    } else {
#pragma unroll
      for (int c = c0; c < c0 + 8; ++c) {
        *reinterpret_cast<uint4*>(gK(buf) + sw128_off(r, c, kLeafKeys * 128)) = make_uint4(0u, 0u, 0u, 0u);
        if (with_v) *reinterpret_cast<uint4*>(gV(buf) + sw128_off(r, c, kLeafKeys * 128)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
  // this row's 64 scores of block b (base-2 scaled; -inf outside its dense keys)
  auto scores = [&](int b, uint32_t tmem, float (&sc)[64]) {
    const int64_t j0 = (int64_t)b * kLeafKeys;
    const int64_t sh = s_hi - j0, wl = w_lo - j0, wh = w_hi - j0;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + half * 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int k = half * 32 + i;
        sc[k] = (k < sh || (k >= wl && k <= wh)) ? v[i] * a.scale_log2 : -INFINITY;
      }
    }
  };
  alloc_tmem(&s_taddr, 256);   // S in columns [0, 64), O in [64, 192)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;
  uint32_t phase = 0;
  bool ok = true;
  // product on the tensor cores from buffer buf, then every thread waits for it
  auto run_mma = [&](int buf, bool pv, bool accumulate) {
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      if (!pv) {
        LeafSmem cs = s;
        cs.sK = smem_u32(gK(buf));
        issue_qk(cs, tmem, 0);
      } else {
        constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
        const uint32_t sP = smem_u32(gK(buf)), sV = smem_u32(gV(buf));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma(tmem + 64, sdesc_sw128(sP + kk * 32, 16, 1024), sdesc_sw128(sV + kk * 2048, kLeafKeys * 128, 1024),
                 idesc, (accumulate || kk > 0) ? 1u : 0u);
      }
      tc_commit(s.mbar);
    }
    ok = __syncthreads_and(mbar_wait(s.mbar, phase));
    phase ^= 1;
    tc_fence_after();
  };
  // sweep 1: max and sum of every row
  float m = -INFINITY, l = 0.f;
  {
    int b = cta_min(next_block(0)), cur = 0;
    if (b != INT_MAX) load_block(b, cur, false);
    cp_async_commit();
    while (b != INT_MAX && ok) {
      const int nb = cta_min(next_block(b + 1));   // also: every thread is done with the other buffer
      if (nb != INT_MAX) load_block(nb, cur ^ 1, false);
      cp_async_commit();
      cp_async_wait_prev();
      fence_async_smem();
      run_mma(cur, false, false);
      if (!ok) break;
      float sc[64];
      scores(b, tmem, sc);
      float bm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) bm = fmaxf(bm, sc[i]);
      const float mn = fmaxf(m, bm);
      if (mn != -INFINITY) {
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) sum += exp2f(sc[i] - mn);
        l = (m == -INFINITY ? 0.f : l * exp2f(m - mn)) + sum;
        m = mn;
      }
      tc_fence_before();
      b = nb;
      cur ^= 1;
    }
    cp_async_drain();
  }
  const float lse2 = l > 0.f ? m + log2f(l) : INFINITY;   // +inf: P = 0
  // sweep 2: O = sum over blocks of 2^(s - lse) . V
  bool any = false;
  if (ok) {
    __syncthreads();   // sweep 1's buffers are free
    int b = cta_min(next_block(0)), cur = 0;
    if (b != INT_MAX) load_block(b, cur, true);
    cp_async_commit();
    while (b != INT_MAX && ok) {
      const int nb = cta_min(next_block(b + 1));
      if (nb != INT_MAX) load_block(nb, cur ^ 1, true);
      cp_async_commit();
      cp_async_wait_prev();
      fence_async_smem();
      run_mma(cur, false, false);
      if (!ok) break;
      float sc[64];
      scores(b, tmem, sc);
      const int r = threadIdx.x;
      char* gP = gK(cur);   // S = Q.K^T has completed: P takes the K tile's place
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(exp2f(sc[c * 8 + 2 * i] - lse2), exp2f(sc[c * 8 + 2 * i + 1] - lse2));
          w[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(gP + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_async_smem();
      tc_fence_before();
      run_mma(cur, true, any);
      any = true;
      tc_fence_before();
      b = nb;
      cur ^= 1;
    }
    cp_async_drain();
  }
  if (!ok) set_status(a.status, LSA_ERR_TIMEOUT);
  if (ok) {   // CTA-uniform: the TMEM loads are warp-collective, the stores per row
    const int64_t row = t * a.Hq + g * a.G + hh;
    __nv_bfloat16* dst = valid ? a.Od + row * kDim : nullptr;
#pragma unroll
    for (int part = 0; part < 4; ++part) {
      float v[32];
      if (any) {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 64 + part * 32, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(v[i + 2 * k], v[i + 2 * k + 1]);
          w[k] = *reinterpret_cast<uint32_t*>(&b2);
        }
        if (dst) *reinterpret_cast<uint4*>(dst + part * 32 + i) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    if (valid) a.LSEd[row] = l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  free_tmem(tmem, 256);
}

// ---- partial mode, pipelined ------------------------------------------------
//
// Persistent CTAs (one per SM), each walking a contiguous range of chunks with
// four warp roles joined by mbarriers:
//   warps 8 and 11, 9 and 14 (two loader groups, alternate chunks): chunk
//     metadata into shared memory and 16-byte cp.async copies of the chunk's Q
//     rows and the leaf's K and V rows into one of kPipeStages stages
//     (128B-swizzled tiles), after an L2 prefetch of the K/V rows two chunks
//     earlier;
//   warp 10 (one lane, MMA): S = Q.K^T into one of kPipeBufs TMEM buffers, and
//     once P is in shared memory, O = P.V over the same columns;
//   warps 0-1 and 2-3 (P, even and odd chunks, one TMEM lane per row): P and
//     the (m, l) statistics from S;
//   warps 4-5 and 6-7 (epilogue, even and odd chunks, same lanes): O from TMEM
//     to the partial outputs.
// A warp reaches only the TMEM lane quarter (warp mod 4), so the rows of even
// chunks sit in lanes 0-63 and those of odd chunks in lanes 64-127: their M = 128
// products read the Q (then P) tile from 8 KB below the stage, which puts the
// chunk's 64 rows in tile rows 64-127.  The softmax and epilogue work of the two
// parities then runs on all four SM sub-partitions instead of two.
// Every wait is bounded; on a timeout the CTA records LSA_ERR_TIMEOUT, stops
// its roles, waits for its copies and MMAs in flight and frees TMEM.

constexpr int kPipeStages = 4;
constexpr int kPipeBufs = 4;                       // TMEM buffers of 128 columns
constexpr int kChunkRows = 64;                     // rows of a chunk (TMEM lanes 0-63 or 64-127)
constexpr int kPipeLoaders = 64;                   // threads of a loader group (warps 2-3, 6-7)
constexpr int kPipeThreads = 15 * 32;              // warps 12 and 13 have no role
// Stage: Q/P tile [0, 16 KB), K [16, 32 KB), V [32, 48 KB).  The M = 128 products
// read 128 tile rows; rows 64-127 fall on the next 8 KB of the same stage and
// belong to no chunk row (their results are never used).
constexpr uint32_t kStageBytes = 49152;
constexpr uint32_t kQHalf = kChunkRows * 128;     // bytes between the two 64-column halves of Q
// odd chunks use odd stages, whose tiles have a whole stage below them to read from
static_assert(kPipeStages % 2 == 0 && kPipeBufs % 2 == 0 && kQHalf <= kStageBytes, "chunk parity layout");

struct PipeMeta {
  int32_t ent[kPipeStages][kChunkRows];
  int32_t lpos[2][2][kLeafKeys];                   // per loader group and iteration parity: key positions
  int32_t lqrow[2][2][kChunkRows];                 // and the global Q row of each tile row (loaders only)
  int32_t nvis[kPipeStages][kChunkRows];           // visible keys of each entry: [vlo, nvis)
  int32_t vlo[kPipeStages][kChunkRows];
  int32_t info[kPipeStages][2];                    // head, entries
  int32_t prow[kPipeBufs][kChunkRows];             // partial row of each TMEM lane (-1: none)
  float2 stat[kPipeBufs][kChunkRows];              // (m, l) of each TMEM lane
  uint64_t full[kPipeStages], sempty[kPipeStages], pready[kPipeStages];
  uint64_t sfull[kPipeBufs], ofull[kPipeBufs], tempty[kPipeBufs], mready[kPipeBufs];
  uint64_t done;
  uint32_t taddr;
  int32_t abort;
};
constexpr size_t kPipeSmem = 1024 + kPipeStages * kStageBytes + sizeof(PipeMeta);

// Barrier of one loader group (named barrier 1 + group) that also returns, in
// every one of its threads, whether any of them passed `v`: their stop decisions
// agree, so none waits at the barrier for a loader that has left.
__device__ __forceinline__ bool loaders_any(bool v, int group) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\nbar.red.or.pred q, %2, %3, p;\nselp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + group), "n"(kPipeLoaders)
      : "memory");
  return r != 0;
}

// Metadata one loader thread needs for one chunk.
struct LoadMeta {
  int g, leaf, e_lo, ne;
  int32_t pos;      // position of key (lt mod 64)
  int32_t qent;     // entry of Q row lt (or -1)
  int32_t ev, eq;   // entry lt and its query position (metadata)
};

__global__ void __launch_bounds__(kPipeThreads, 1) k_tl_pipe(TreeAttnArgs a) {
  extern __shared__ char smem_raw[];
  char* base = align1024(smem_raw);
  PipeMeta& M = *reinterpret_cast<PipeMeta*>(base + kPipeStages * kStageBytes);
  const uint32_t sbase = smem_u32(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t C = 0;
  for (int h = 0; h < a.H; ++h) C += a.ctotal[h];
  const int64_t k0 = C * blockIdx.x / gridDim.x, k1 = C * (blockIdx.x + 1) / gridDim.x;
  const int N = (int)(k1 - k0);
  if (N == 0) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPipeStages; ++s) {
      mbar_init(smem_u32(&M.full[s]), 2 * kPipeLoaders);
      mbar_init(smem_u32(&M.sempty[s]), 1);
      mbar_init(smem_u32(&M.pready[s]), kChunkRows);
    }
    for (int b = 0; b < kPipeBufs; ++b) {
      mbar_init(smem_u32(&M.sfull[b]), 1);
      mbar_init(smem_u32(&M.ofull[b]), 1);
      mbar_init(smem_u32(&M.tempty[b]), kChunkRows);
      mbar_init(smem_u32(&M.mready[b]), kChunkRows);
    }
    mbar_init(smem_u32(&M.done), 1);
    M.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  alloc_tmem(&M.taddr, 128 * kPipeBufs);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.taddr;
  volatile int32_t* abort_flag = &M.abort;
  // warp-uniform view of the abort flag (the warps' collectives must not diverge)
  auto aborted = [&]() { return __any_sync(0xffffffffu, *abort_flag != 0); };
  auto fail = [&]() {
    *abort_flag = 1;
    set_status(a.status, LSA_ERR_TIMEOUT);
  };

  if (warp == 8 || warp == 9 || warp == 11 || warp == 14) {
    // ---- loaders: two groups of 64 threads take alternate chunks (and stages);
    // in a group, lanes (j & 15) x rows (j >> 4) + 4 i copy 16-byte pieces.  The
    // warps of a group sit on different SM sub-partitions. ----
    const int lt = (warp == 8 ? 0 : warp == 11 ? 1 : warp == 9 ? 2 : 3) * 32 + lane;
    const int group = lt >> 6, j = lt & 63;
    // descriptors come 32 at a time (one per lane) and are broadcast by shuffles;
    // a chunk's metadata is fetched two group iterations before its copies
    int4 dcur = lane < N ? a.cdesc[k0 + lane] : make_int4(0, 0, 0, 0);
    int4 dnxt = 32 + lane < N ? a.cdesc[k0 + 32 + lane] : make_int4(0, 0, 0, 0);
    int blk = 0;
    // descriptor of chunk kk (in block blk or the next)
    auto desc = [&](int kk) -> int4 {
      const int4& dr = (kk >> 5) == blk ? dcur : dnxt;
      const int q = kk & 31;
      return make_int4(__shfl_sync(0xffffffffu, dr.x, q), __shfl_sync(0xffffffffu, dr.y, q),
                       __shfl_sync(0xffffffffu, dr.z, q), __shfl_sync(0xffffffffu, dr.w, q));
    };
    auto fetch = [&](int kk, LoadMeta& L) {
      const int4 d = desc(kk);
      L.g = d.x; L.leaf = d.y; L.e_lo = d.z; L.ne = d.w;
      const int32_t* entg = a.ent + (int64_t)L.g * a.T * a.B + L.e_lo;
      L.pos = a.leaf_index[(int64_t)L.g * a.n_tree + (int64_t)L.leaf * kLeafKeys + j];
      const int n_rows = L.ne * a.G;
      L.qent = j < n_rows ? entg[j / a.G] : -1;
      L.ev = j < L.ne ? entg[j] : -1;
      L.eq = j < L.ne ? a.entq[(int64_t)L.g * a.T * a.B + L.e_lo + j] : 0;
    };
    // L2 prefetch of the K/V rows two group iterations ahead (no shared memory
    // needed); the row position is loaded one iteration before the prefetch
    int32_t pf_pos = 0, pf_g = 0;
    auto pf_issue = [&]() {
      const int64_t row = ((int64_t)pf_g * a.n_cap + pf_pos) * kDim;
      asm volatile("prefetch.global.L2 [%0];\nprefetch.global.L2 [%1];\nprefetch.global.L2 [%2];\nprefetch.global.L2 [%3];"
                   ::"l"(a.K + row), "l"(a.K + row + 64), "l"(a.V + row), "l"(a.V + row + 64));
    };
    auto pf_load = [&](int kk) {
      const int4 d = desc(kk);
      pf_g = d.x;
      pf_pos = a.leaf_index[(int64_t)pf_g * a.n_tree + (int64_t)d.y * kLeafKeys + j];
    };
    if (group + 2 < N) {   // the group's second chunk right away
      pf_load(group + 2);
      pf_issue();
    }
    if (group + 4 < N) pf_load(group + 4);
    LoadMeta cur, n1, n2;
    if (group < N) fetch(group, cur);
    if (group + 2 < N) fetch(group + 2, n1);
    for (int k = group; k < N; k += 2) {
      if ((k >> 5) != blk) {   // entering block k / 32: shift the descriptor window
        blk = k >> 5;
        dcur = dnxt;
        const int64_t nb = (int64_t)(blk + 1) * 32 + lane;
        dnxt = nb < N ? a.cdesc[k0 + nb] : make_int4(0, 0, 0, 0);
      }
      if (k + 4 < N) {
        pf_issue();
        if (k + 6 < N) pf_load(k + 6);
      }
      if (k + 4 < N) fetch(k + 4, n2);
      const int s = k % kPipeStages;
      const uint32_t st = sbase + s * kStageBytes;
      // row addresses through the group's own shared buffers (alternating by
      // iteration), so that 16 lanes copy one 256-B row; everything that does not
      // touch the stage is done before waiting for it
      const int n_rows = cur.ne * a.G;
      int32_t* lpos = M.lpos[group][(k >> 1) & 1];
      int32_t* lqrow = M.lqrow[group][(k >> 1) & 1];
      lpos[j] = cur.pos;
      lqrow[j] = j < n_rows ? (cur.qent >> 6) * a.Hq + cur.g * a.G + j % a.G : -1;
      asm volatile("bar.sync %0, %1;" ::"r"(1 + group), "n"(kPipeLoaders) : "memory");
      // visible keys of entry j: position <= q_pos, outside the sink [0, n_sink)
      // and the window (q_pos - window, q_pos], whose keys the dense part attends
      int nvis = 0, vlo = 0;
      if (j < a.epc && cur.ev >= 0) {
        const int hi = visible_prefix(lpos, (int64_t)cur.eq - a.window);
        vlo = a.n_sink > 0 ? visible_prefix(lpos, (int64_t)a.n_sink - 1) : 0;
        nvis = hi > vlo ? hi : vlo;
      }
      const int c = j & 15, rg = j >> 4;
      const int64_t kv_base = (int64_t)cur.g * a.n_cap;
      // all row addresses first: each copy's asm is a compiler memory barrier, so a
      // shared-memory read between two copies would wait out its full latency
      int32_t kpos[16], qr[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        kpos[i] = lpos[rg + 4 * i];
        qr[i] = lqrow[rg + 4 * i];
      }
      const bool ok = k < kPipeStages || mbar_wait(smem_u32(&M.sempty[s]), ((k / kPipeStages) - 1) & 1);
      if (loaders_any(!ok || *abort_flag != 0, group)) {   // every thread of the group agrees
        if (!ok) fail();
        break;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {   // K and V rows rg, rg + 4, ..., chunk c
        const int kr2 = rg + 4 * i;
        const int64_t row = kv_base + kpos[i];
        cp_async16(st + 16384u + sw128_off(kr2, c, kLeafKeys * 128), a.K + row * kDim + c * 8);
        cp_async16(st + 32768u + sw128_off(kr2, c, kLeafKeys * 128), a.V + row * kDim + c * 8);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)   // Q rows rg, rg + 4, ... below n_rows
        if (qr[i] >= 0) cp_async16(st + sw128_off(rg + 4 * i, c, kQHalf), a.Q + (int64_t)qr[i] * kDim + c * 8);
      const uint32_t bar = smem_u32(&M.full[s]);
      cp_async_arrive(bar);
      if (j < a.epc) {
        M.ent[s][j] = cur.ev;
        M.nvis[s][j] = nvis;
        M.vlo[s][j] = vlo;
      }
      if (j == 0) {
        M.info[s][0] = cur.g;
        M.info[s][1] = cur.ne;
      }
      mbar_arrive(bar);
      cur = n1;
      n1 = n2;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // nothing in flight when the CTA exits
  } else if (warp == 10) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 64, false, false);
      constexpr uint32_t id_pv = idesc_bf16(128, 128, false, true);
      auto qk = [&](int k) {
        const int s = k % kPipeStages, b = k % kPipeBufs;
        fence_async_smem();    // the loaders' cp.async writes, seen through the barrier, before the MMA reads
        tc_fence_after();
        // odd chunks: tile rows 64-127 are the chunk's rows (the 8 KB below the stage
        // feed rows 0-63, whose results are never read)
        const uint32_t sA = sbase + s * kStageBytes - (k & 1) * kQHalf, sK = sbase + s * kStageBytes + 16384;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          tc_mma(tmem + b * 128, sdesc_sw128(sA + (kk >> 2) * kQHalf + koff, 16, 1024),
                 sdesc_sw128(sK + (kk >> 2) * (kLeafKeys * 128) + koff, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&M.sfull[b]));
      };
      auto pv = [&](int k) {
        const int s = k % kPipeStages, b = k % kPipeBufs;
        tc_fence_after();
        const uint32_t sP = sbase + s * kStageBytes - (k & 1) * kQHalf, sV = sbase + s * kStageBytes + 32768;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma(tmem + b * 128, sdesc_sw128(sP + kk * 32, 16, 1024),
                 sdesc_sw128(sV + kk * 2048, kLeafKeys * 128, 1024), id_pv, kk > 0 ? 1u : 0u);
        tc_commit(smem_u32(&M.ofull[b]));
        tc_commit(smem_u32(&M.sempty[s]));
      };
      // issue whichever product is ready: P.V of the oldest chunk whose P is in
      // shared memory, else S of the next chunk whose stage has landed and whose
      // TMEM buffer is free; give up after kWaitNs without progress
      int nq = 0, np = 0, idle = 0;
      bool ok = true;
      uint64_t t_idle = 0;
      while (np < N) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        bool progressed = false;
        if (np < nq && mbar_test(smem_u32(&M.pready[np % kPipeStages]), (np / kPipeStages) & 1)) {
          pv(np++);
          progressed = true;
        } else if (nq < N && mbar_test(smem_u32(&M.full[nq % kPipeStages]), (nq / kPipeStages) & 1) &&
                   (nq < kPipeBufs || mbar_test(smem_u32(&M.tempty[nq % kPipeBufs]), ((nq / kPipeBufs) - 1) & 1))) {
          qk(nq++);
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if ((++idle & 63) == 0) {   // the timer is read once every 64 idle polls
          const uint64_t t = now_ns();
          if (idle == 64) {
            t_idle = t;
          } else if (t - t_idle > kWaitNs) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) fail();
      tc_commit(smem_u32(&M.done));    // every MMA issued above has completed
      if (!mbar_wait(smem_u32(&M.done), 0)) fail();
    }
    __syncwarp();
  } else if (warp < 4) {
    // ---- P: warps 0-1 take the even chunks (TMEM lanes 0-63), warps 2-3 the odd
    // ones (lanes 64-127); r = the row within the chunk ----
    const int r = (warp & 1) * 32 + lane;
    const int pgrp = warp >> 1;
    const int e = r / a.G, hh = r % a.G;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    for (int k = pgrp; k < N; k += 2) {
      if (aborted()) break;
      const int s = k % kPipeStages, b = k % kPipeBufs;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&M.full[s]), (k / kPipeStages) & 1));
      if (!ok) break;
      const int g = M.info[s][0];
      const int v = M.ent[s][e];
      const int64_t tq = v >= 0 ? (v >> 6) : -1;
      const int nvis = M.nvis[s][e], vlo = M.vlo[s][e];
      const int prow = tq >= 0 ? (int)((tq * a.Hq + g * a.G + hh) * a.B + (v & 63)) : -1;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&M.sfull[b]), (k / kPipeBufs) & 1));
      if (!ok) break;
      tc_fence_after();
      float m = -INFINITY, l = 0.f;
      if (__any_sync(0xffffffffu, tq >= 0)) {   // a warp without chunk rows leaves its P rows unused
        float sc[64];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float t32[32];
          tmem_ld32(tmem + b * 128 + lane_base + half * 32, t32);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            sc[half * 32 + i] = half * 32 + i < nvis && half * 32 + i >= vlo ? t32[i] * a.scale_log2 : -INFINITY;
        }
        float mx[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) mx[i] = fmaxf(fmaxf(sc[4 * i], sc[4 * i + 1]), fmaxf(sc[4 * i + 2], sc[4 * i + 3]));
#pragma unroll
        for (int w = 8; w; w >>= 1)
#pragma unroll
          for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
        m = mx[0];
        const float mref = m == -INFINITY ? 0.f : m;
        float ls[8];
        char* sP = base + s * kStageBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
          float lc = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float p0 = exp2f(sc[c * 8 + 2 * q] - mref), p1 = exp2f(sc[c * 8 + 2 * q + 1] - mref);
            lc += p0 + p1;
            __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
            w[q] = *reinterpret_cast<uint32_t*>(&b2);
          }
          ls[c] = lc;
          *reinterpret_cast<uint4*>(sP + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        l = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      }
      M.prow[b][r] = prow;
      M.stat[b][r] = make_float2(m, l);
      mbar_arrive(smem_u32(&M.mready[b]));
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&M.pready[s]));
    }
    if (!ok && lane == 0) fail();
  } else if (warp < 8) {
    // ---- epilogue: warps 4-5 take the even chunks, warps 6-7 the odd ones (the
    // TMEM lanes of their P warps); r = the row within the chunk ----
    const int r = (warp & 1) * 32 + lane;
    const int egrp = (warp >> 1) & 1;
    bool ok = true;
    for (int k = egrp; k < N; k += 2) {
      if (aborted()) break;
      const int b = k % kPipeBufs;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&M.mready[b]), (k / kPipeBufs) & 1) &&
                                       mbar_wait(smem_u32(&M.ofull[b]), (k / kPipeBufs) & 1));
      if (!ok) break;
      tc_fence_after();
      const int prow = M.prow[b][r];
      const float2 st = M.stat[b][r];
      __nv_bfloat16* dst = prow >= 0 ? a.part + (int64_t)prow * kDim : nullptr;
      const float inv_l = st.y > 0.f ? 1.f / st.y : 0.f;
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        float v[32];
        tmem_ld32(tmem + b * 128 + ((uint32_t)((warp & 3) * 32) << 16) + part * 32, v);
        if (dst) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(v[i + 2 * q] * inv_l, v[i + 2 * q + 1] * inv_l);
              w[q] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(dst + part * 32 + i) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (prow >= 0) a.stats[prow] = st;
      tc_fence_before();
      mbar_arrive(smem_u32(&M.tempty[b]));
    }
    if (!ok && lane == 0) fail();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  free_tmem(tmem, 128 * kPipeBufs);
}

// ---- backward, leaf by leaf -------------------------------------------------
//
// Same leaf lists as the forward.  Per leaf CTA and chunk of up to 128 rows:
//   S = Q . K_leaf^T, dP = dO . V_leaf^T                   (tcgen05, TMEM cols 0..127)
//   P = exp(S - LSE), dS = P * (dP - delta)                (bf16 tiles in smem)
//   dV_leaf^T += dO^T . P,  dK_leaf^T += Q^T . dS          (TMEM accumulators, all chunks)
//   dQ_rows = dS . K_leaf                                  (TMEM cols 0..127, fp32 red-adds)
// A leaf owns its keys, so dK/dV of the leaf are stored once, without atomics.
// delta = rowsum(dO * O) and the base-2 LSE come from k_tlb_rows.

struct TreeBwdArgs {
  TreeAttnArgs f;              // lists, Q/K/V, positions, sizes
  const __nv_bfloat16* O;
  const __nv_bfloat16* dO;
  const float* LSE;
  float* delta;                // [T][Hq]
  float* lse2b;                // [T][Hq]
  float* dQ;
  float* dK;
  float* dV;
  float scale;
};

__global__ void k_tlb_rows(TreeBwdArgs b) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;   // one warp per row
  const int lane = threadIdx.x & 31;
  if (row >= b.f.T * b.f.Hq) return;
  float v[4], o[4];
  load4(b.dO + row * kDim + lane * 4, v);
  load4(b.O + row * kDim + lane * 4, o);
  float x = v[0] * o[0] + v[1] * o[1] + v[2] * o[2] + v[3] * o[3];
#pragma unroll
  for (int s = 16; s; s >>= 1) x += __shfl_xor_sync(0xffffffffu, x, s);
  if (lane == 0) {
    b.delta[row] = x;
    const float L = b.LSE[row];
    b.lse2b[row] = L == -INFINITY ? INFINITY : L * 1.44269504088896340736f;
  }
}

__global__ void __launch_bounds__(kTL) k_tlb_leaf(TreeBwdArgs b) {
  extern __shared__ char smem_raw[];
  __shared__ int32_t s_pos[kLeafKeys];
  __shared__ __align__(8) uint64_t s_mbar;
  __shared__ uint32_t s_taddr;
  const TreeAttnArgs& a = b.f;
  const int64_t g = blockIdx.y, leaf = blockIdx.x;
  const int32_t* offg = a.off + g * (a.NL + 1);
  const int64_t e_lo = offg[leaf], n_ent = offg[leaf + 1] - e_lo;
  if (n_ent == 0) return;
  const int32_t* ent = a.ent + g * a.T * a.B + e_lo;
  char* base = align1024(smem_raw);
  const uint32_t sQ = smem_u32(base);            // 32 KB  rows x d
  const uint32_t sdO = sQ + kTL * 256;           // 32 KB  rows x d
  const uint32_t sK = sdO + kTL * 256;           // 16 KB  keys x d
  const uint32_t sV = sK + kLeafKeys * 256;      // 16 KB  keys x d
  const uint32_t sP = sV + kLeafKeys * 256;      // 16 KB  rows x keys
  const uint32_t sdS = sP + kTL * 128;           // 16 KB  rows x keys
  char* gP = base + (sP - sQ);
  char* gdS = base + (sdS - sQ);
  const uint32_t mbar = smem_u32(&s_mbar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar));
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  int64_t tq;
  int rank, h;
  row_of(a, ent, n_ent, 0, tq, rank, h);
  int64_t row = tq >= 0 ? tq * a.Hq + g * a.G + h : -1;
  float dlt = row >= 0 ? b.delta[row] : 0.f, lse = row >= 0 ? b.lse2b[row] : INFINITY;
  if (threadIdx.x < kLeafKeys) s_pos[threadIdx.x] = a.leaf_index[g * a.n_tree + leaf * kLeafKeys + threadIdx.x];
  __syncthreads();
  {
    LeafSmem ls;
    ls.sK = sK;
    ls.sV = sV;
    ls.pos = s_pos;
    copy_leaf(a, g, ls, true);
  }
  alloc_tmem(&s_taddr, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_taddr;
  const int warp = threadIdx.x >> 5;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  uint32_t phase = 0;
  bool ok = true;
  bool first = true;
  const int64_t qp = 0;
  (void)qp;
  for (int64_t e0 = 0; e0 < n_ent && ok; e0 += kTL / a.G) {
    if (e0 > 0) {
      row_of(a, ent, n_ent, e0, tq, rank, h);
      row = tq >= 0 ? tq * a.Hq + g * a.G + h : -1;
      dlt = row >= 0 ? b.delta[row] : 0.f;
      lse = row >= 0 ? b.lse2b[row] : INFINITY;
    }
    if (row >= 0) {
      const __nv_bfloat16* q = a.Q + row * kDim;
      const __nv_bfloat16* go = b.dO + row * kDim;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        cp_async16(sQ + sw128_off(threadIdx.x, c, kTL * 128), q + c * 8);
        cp_async16(sdO + sw128_off(threadIdx.x, c, kTL * 128), go + c * 8);
      }
    }
    cp_async_wait_all();
    fence_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      constexpr uint32_t id_s = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ko = (uint32_t)(kk & 3) * 32;
        tc_mma(tmem, sdesc_sw128(sQ + (kk >> 2) * (kTL * 128) + ko, 16, 1024),
               sdesc_sw128(sK + (kk >> 2) * (kLeafKeys * 128) + ko, 16, 1024), id_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ko = (uint32_t)(kk & 3) * 32;
        tc_mma(tmem + 64, sdesc_sw128(sdO + (kk >> 2) * (kTL * 128) + ko, 16, 1024),
               sdesc_sw128(sV + (kk >> 2) * (kLeafKeys * 128) + ko, 16, 1024), id_s, kk > 0 ? 1u : 0u);
      }
      tc_commit(mbar);
    }
    ok = __syncthreads_and(mbar_wait(mbar, phase));
    phase ^= 1;
    tc_fence_after();
    if (!ok) {
      set_status(a.status, LSA_ERR_TIMEOUT);
      break;
    }
    {
      const int64_t qpos = (a.causal && tq >= 0) ? (int64_t)a.q_pos[tq] : INT64_MAX;
      const int nvis = row >= 0 ? visible_prefix(s_pos, qpos) : 0;
      const int r = threadIdx.x;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float sv[32], dv[32];
        tmem_ld32(tmem + lane_base + half * 32, sv);
        tmem_ld32(tmem + lane_base + 64 + half * 32, dv);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t wp[4], wd[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float p2[2], d2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int i = c * 8 + 2 * q + u, key = half * 32 + i;
              const bool vis = key < nvis;
              const float p = vis ? exp2f(sv[i] * a.scale_log2 - lse) : 0.f;
              p2[u] = p;
              d2[u] = p * (dv[i] - dlt);
            }
            __nv_bfloat162 bp = __floats2bfloat162_rn(p2[0], p2[1]);
            __nv_bfloat162 bd = __floats2bfloat162_rn(d2[0], d2[1]);
            wp[q] = *reinterpret_cast<uint32_t*>(&bp);
            wd[q] = *reinterpret_cast<uint32_t*>(&bd);
          }
          const int chunk = half * 4 + c;
          const uint32_t off = (r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(gP + off) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
          *reinterpret_cast<uint4*>(gdS + off) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      // dV^T (d x keys) += dO^T . P ; dK^T += Q^T . dS   (both operands MN-major)
      constexpr uint32_t id_t = idesc_bf16(128, 64, true, true);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = (first && kk == 0) ? 0u : 1u;
        tc_mma(tmem + 128, sdesc_sw128(sdO + kk * 2048, kTL * 128, 1024), sdesc_sw128(sP + kk * 2048, kTL * 128, 1024),
               id_t, acc);
        tc_mma(tmem + 192, sdesc_sw128(sQ + kk * 2048, kTL * 128, 1024), sdesc_sw128(sdS + kk * 2048, kTL * 128, 1024),
               id_t, acc);
      }
      // dQ rows (rows x d) = dS . K_leaf   (dS K-major, K_leaf as MN-major B)
      constexpr uint32_t id_q = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc_mma(tmem, sdesc_sw128(sdS + kk * 32, 16, 1024), sdesc_sw128(sK + kk * 2048, kLeafKeys * 128, 1024),
               id_q, kk > 0 ? 1u : 0u);
      tc_commit(mbar);
    }
    first = false;
    ok = __syncthreads_and(mbar_wait(mbar, phase));
    phase ^= 1;
    tc_fence_after();
    if (!ok) {
      set_status(a.status, LSA_ERR_TIMEOUT);
      break;
    }
    {
      float* dst = row >= 0 ? b.dQ + row * kDim : nullptr;
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        float v[32];
        tmem_ld32(tmem + lane_base + part * 32, v);
        if (dst) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            red_add_v4(dst + part * 32 + i, v[i] * b.scale, v[i + 1] * b.scale, v[i + 2] * b.scale,
                       v[i + 3] * b.scale);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  if (ok) {
    // lane t holds dimension t of every key's gradient: store the leaf's rows once
    tc_fence_after();
    float* dKh = b.dK + g * a.n_cap * kDim;
    float* dVh = b.dV + g * a.n_cap * kDim;
    const int t = threadIdx.x;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float vv[32], kv[32];
      tmem_ld32(tmem + lane_base + 128 + half * 32, vv);
      tmem_ld32(tmem + lane_base + 192 + half * 32, kv);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int64_t j = s_pos[half * 32 + i];
        dVh[j * kDim + t] = vv[i];
        dKh[j * kDim + t] = kv[i] * b.scale;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  free_tmem(tmem, 256);
}

// expand leaves into key lists (fallback shapes)
__global__ void k_tl_expand(const int32_t* leaves, const int32_t* leaf_index, int64_t H, int64_t T, int B, int leaf,
                            int64_t n_tree, int32_t* idx) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t K_sel = (int64_t)B * leaf;
  if (i >= H * T * K_sel) return;
  const int64_t g = i / (T * K_sel), rem = i % (T * K_sel), t = rem / K_sel, k = rem % K_sel;
  const int32_t lf = leaves[(g * T + t) * B + k / leaf];
  idx[i] = lf >= 0 ? leaf_index[g * n_tree + (int64_t)lf * leaf + k % leaf] : -1;
}

constexpr size_t kStatsSmem = 1024 + kTL * 256 + kLeafKeys * 256;
constexpr size_t kOutSmem = 1024 + kTL * 256 + 2 * kLeafKeys * 256;
constexpr size_t kBwdSmem = 1024 + 2 * kTL * 256 + 2 * kLeafKeys * 256 + 2 * kTL * 128;

}  // namespace

// Partial mode while its per-(row, leaf) outputs stay within this many bytes.
constexpr size_t kPartialMaxBytes = size_t(24) << 30;   // an eighth of a 180 GB part

static bool partial_fits(int64_t T, int64_t Hq, int B) { return (size_t)T * Hq * B * kDim * 2 <= kPartialMaxBytes; }

static int64_t max_chunks(int64_t H, int64_t NL, int64_t T, int B, int epc) {
  return H * NL + ceil_div(H * T * B, (int64_t)epc);
}

size_t tree_attn_workspace(int64_t H, int64_t NL, int64_t T, int64_t Hq, int d, int B, int leaf, bool fast,
                           int n_sink, int window) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const bool sw = n_sink > 0 || window > 0;
  const size_t expand = al((size_t)H * T * B * leaf * 4);
  if (!fast || (sw && !partial_fits(T, Hq, B)))   // key lists (extended with the sink and window keys)
    return expand + (sw ? al((size_t)H * T * ((size_t)B * leaf + n_sink + window) * 4) : 0);
  const size_t lists = al(H * NL * 4) + al(H * (NL + 1) * 4) + al((size_t)H * T * B * 4) + al((size_t)T * Hq * B * 8);
  const size_t red = lists + al((size_t)T * Hq * 4) + al((size_t)T * Hq * d * 4);
  if (!partial_fits(T, Hq, B)) return red;
  const int epc = kChunkRows / (int)(Hq / H);
  size_t part = lists + al((size_t)T * Hq * B * d * 2) + al((size_t)H * T * B * 4) + al(H * NL * 4) +
                al(H * 4) + al((size_t)max_chunks(H, NL, T, B, epc) * 16);
  if (sw) part += al((size_t)T * Hq * d * 2) + al((size_t)T * Hq * 4);   // dense part: output and LSE
  return part > red ? part : red;
}

size_t tree_attn_bwd_workspace(int64_t H, int64_t NL, int64_t T, int64_t Hq, int d, int B, int leaf, bool fast) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  if (!fast) return al((size_t)H * T * B * leaf * 4);
  return al(H * NL * 4) + al(H * (NL + 1) * 4) + al((size_t)H * T * B * 4) + 2 * al((size_t)T * Hq * 4);
}

bool tree_attn_fast_path(int dtype, int d, int G, int leaf) {
  return dtype == LSA_BF16 && d == kDim && leaf == kLeafKeys && (G == 1 || G == 2 || G == 4 || G == 8);
}

cudaError_t run_tree_attn(const TreeAttnCall& c, cudaStream_t st) {
  if (c.T == 0) return cudaSuccess;
  const int G = c.Hq / c.H;
  const bool fast = tree_attn_fast_path(c.dtype, c.d, G, c.leaf);
  char* ws = static_cast<char*>(c.workspace);
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  cudaError_t e;
  const bool sw = c.n_sink > 0 || c.window > 0;
  // key-list attention over given lists (one CTA per (query, group): no split workspace)
  auto keylist_attn = [&](const int32_t* idx, int32_t K_sel, void* O, float* LSE, float* part) {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.Q = c.Q; a.K = c.K; a.V = c.V; a.idx = idx; a.q_pos = c.q_pos; a.O = O; a.LSE = LSE;
    a.status = c.status; a.T = c.T; a.n_cap = c.n_cap; a.Hq = c.Hq; a.Hkv = c.H; a.G = G; a.d = c.d;
    a.K_sel = K_sel; a.causal = c.causal;
    a.nsplit = part ? attn_splits(c.T, c.H, K_sel) : 1;
    int64_t kps = (K_sel + a.nsplit - 1) / a.nsplit;
    kps = (kps + 15) / 16 * 16;
    a.keys_per_split = (int32_t)(kps > 0 ? kps : 16);
    a.part = part;
    a.scale = c.scale; a.scale_log2 = c.scale * 1.44269504088896340736f;
    return run_attn_fwd(a, c.dtype, st);
  };
  if (!fast || (sw && !partial_fits(c.T, c.Hq, c.B))) {
    int32_t* idx = reinterpret_cast<int32_t*>(ws);
    const int64_t total = (int64_t)c.H * c.T * c.B * c.leaf;
    k_tl_expand<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(c.leaves, c.leaf_index, c.H, c.T, c.B, c.leaf,
                                                                c.n_tree, idx);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (!sw) return keylist_attn(idx, c.B * c.leaf, c.O, c.LSE, nullptr);
    int32_t* idx2 = reinterpret_cast<int32_t*>(ws + al((size_t)total * 4));
    if ((e = run_attn_extend(idx, c.B * c.leaf, c.T, c.H, c.q_pos, c.n_sink, c.window, 0, 0, c.n_cap, idx2, st)) !=
        cudaSuccess)
      return e;
    return keylist_attn(idx2, c.B * c.leaf + c.n_sink + c.window, c.O, c.LSE, nullptr);
  }
  TreeAttnArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(c.Q);
  a.K = static_cast<const __nv_bfloat16*>(c.K);
  a.V = static_cast<const __nv_bfloat16*>(c.V);
  a.leaf_index = c.leaf_index;
  a.leaves = c.leaves;
  a.q_pos = c.q_pos;
  size_t o = 0;
  a.cnt = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * c.NL * 4);
  a.off = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * (c.NL + 1) * 4);
  a.ent = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * c.T * c.B * 4);
  a.stats = reinterpret_cast<float2*>(ws + o); o += al((size_t)c.T * c.Hq * c.B * 8);
  a.lse2 = a.oacc = nullptr;
  a.part = nullptr;
  a.entq = a.coff = a.ctotal = nullptr;
  a.cdesc = nullptr;
  a.epc = kChunkRows / G;
  a.n_sink = c.n_sink;
  a.window = c.window;
  a.Od = nullptr;
  a.LSEd = nullptr;
  const bool partial = partial_fits(c.T, c.Hq, c.B);
  const size_t o_lists = o;
  if (partial) {
    a.part = reinterpret_cast<__nv_bfloat16*>(ws + o); o += al((size_t)c.T * c.Hq * c.B * kDim * 2);
    a.entq = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * c.T * c.B * 4);
    a.coff = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * c.NL * 4);
    a.ctotal = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * 4);
    a.cdesc = reinterpret_cast<int4*>(ws + o);
    o += al((size_t)max_chunks(c.H, c.NL, c.T, c.B, a.epc) * 16);
    if (sw) {   // dense part: the sink and window keys, 64-position blocks on the tensor cores
      BandArgs d;
      d.Q = a.Q; d.K = a.K; d.V = a.V; d.q_pos = c.q_pos;
      d.Od = reinterpret_cast<__nv_bfloat16*>(ws + o); o += al((size_t)c.T * c.Hq * kDim * 2);
      d.LSEd = reinterpret_cast<float*>(ws + o); o += al((size_t)c.T * c.Hq * 4);
      d.status = c.status; d.T = c.T; d.n_cap = c.n_cap;
      d.Hq = (int32_t)c.Hq; d.H = (int32_t)c.H; d.G = G; d.n_sink = c.n_sink; d.window = c.window;
      d.scale_log2 = c.scale * 1.44269504088896340736f;
      cudaFuncSetAttribute(k_tl_band, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBandSmem);
      k_tl_band<<<dim3((unsigned)ceil_div(c.T, (int64_t)(kTL / G)), (unsigned)c.H), kTL, kBandSmem, st>>>(d);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      a.Od = d.Od;
      a.LSEd = d.LSEd;
    }
  } else {
    o = o_lists;
    a.lse2 = reinterpret_cast<float*>(ws + o); o += al((size_t)c.T * c.Hq * 4);
    a.oacc = reinterpret_cast<float*>(ws + o);
  }
  a.O = static_cast<__nv_bfloat16*>(c.O);
  a.LSE = c.LSE;
  a.status = c.status;
  a.T = c.T; a.n_cap = c.n_cap; a.n_tree = c.n_tree; a.NL = c.NL;
  a.Hq = c.Hq; a.H = c.H; a.G = G; a.B = c.B; a.causal = c.causal;
  a.scale_log2 = c.scale * 1.44269504088896340736f;
  const int64_t n_sel = (int64_t)c.H * c.T * c.B;
  if ((e = cudaMemsetAsync(a.cnt, 0, (size_t)c.H * c.NL * 4, st)) != cudaSuccess) return e;
  k_tl_count<<<(unsigned)ceil_div(n_sel, 256), 256, 0, st>>>(a);
  k_tl_scan<<<(unsigned)c.H, 1024, 0, st>>>(a);
  k_tl_fill<<<(unsigned)ceil_div(n_sel, 256), 256, 0, st>>>(a);
  if (partial) {
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    k_tl_cscan<<<(unsigned)c.H, 1024, 0, st>>>(a);
    k_tl_chunks<<<(unsigned)ceil_div((int64_t)c.H * c.NL, 256), 256, 0, st>>>(a);
    cudaFuncSetAttribute(k_tl_pipe, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPipeSmem);
    k_tl_pipe<<<(unsigned)nsm, kPipeThreads, kPipeSmem, st>>>(a);
    k_tl_combine<<<(unsigned)ceil_div(c.T * c.Hq * 32, 256), 256, 0, st>>>(a);
    return cudaGetLastError();
  }
  if ((e = cudaMemsetAsync(a.oacc, 0, (size_t)c.T * c.Hq * kDim * 4, st)) != cudaSuccess) return e;
  cudaFuncSetAttribute(k_tl_stats, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStatsSmem);
  cudaFuncSetAttribute(k_tl_out, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOutSmem);
  dim3 grid((unsigned)c.NL, (unsigned)c.H);
  k_tl_stats<<<grid, kTL, kStatsSmem, st>>>(a);
  k_tl_lse<<<(unsigned)ceil_div(c.T * c.Hq, 256), 256, 0, st>>>(a);
  k_tl_out<<<grid, kTL, kOutSmem, st>>>(a);
  k_tl_finish<<<(unsigned)ceil_div(c.T * c.Hq * (kDim / 4), 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t run_tree_attn_bwd(const TreeAttnCall& c, const void* O, const float* LSE, const void* dO, float* dQ,
                              float* dK, float* dV, cudaStream_t st) {
  const int G = c.Hq / c.H;
  const bool fast = tree_attn_fast_path(c.dtype, c.d, G, c.leaf);
  char* ws = static_cast<char*>(c.workspace);
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  cudaError_t e;
  const size_t kv_bytes = (size_t)c.H * c.n_cap * c.d * sizeof(float);
  if ((e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return e;
  if (c.T == 0) return cudaSuccess;
  if (!fast) {
    int32_t* idx = reinterpret_cast<int32_t*>(ws);
    const int64_t total = (int64_t)c.H * c.T * c.B * c.leaf;
    k_tl_expand<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(c.leaves, c.leaf_index, c.H, c.T, c.B, c.leaf,
                                                                c.n_tree, idx);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.Q = c.Q; a.K = c.K; a.V = c.V; a.idx = idx; a.q_pos = c.q_pos; a.O = const_cast<void*>(O);
    a.LSE = const_cast<float*>(LSE); a.dO = dO; a.dQ = dQ; a.dK = dK; a.dV = dV; a.status = c.status;
    a.T = c.T; a.n_cap = c.n_cap; a.Hq = c.Hq; a.Hkv = c.H; a.G = G; a.d = c.d; a.K_sel = c.B * c.leaf;
    a.causal = c.causal; a.nsplit = 1; a.keys_per_split = (int32_t)((a.K_sel + 15) / 16 * 16);
    a.scale = c.scale; a.scale_log2 = c.scale * 1.44269504088896340736f;
    return run_attn_bwd(a, c.dtype, st);
  }
  TreeBwdArgs b;
  memset(&b, 0, sizeof(b));
  TreeAttnArgs& a = b.f;
  a.Q = static_cast<const __nv_bfloat16*>(c.Q);
  a.K = static_cast<const __nv_bfloat16*>(c.K);
  a.V = static_cast<const __nv_bfloat16*>(c.V);
  a.leaf_index = c.leaf_index;
  a.leaves = c.leaves;
  a.q_pos = c.q_pos;
  size_t o = 0;
  a.cnt = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * c.NL * 4);
  a.off = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * (c.NL + 1) * 4);
  a.ent = reinterpret_cast<int32_t*>(ws + o); o += al((size_t)c.H * c.T * c.B * 4);
  b.delta = reinterpret_cast<float*>(ws + o); o += al((size_t)c.T * c.Hq * 4);
  b.lse2b = reinterpret_cast<float*>(ws + o);
  a.status = c.status;
  a.T = c.T; a.n_cap = c.n_cap; a.n_tree = c.n_tree; a.NL = c.NL;
  a.Hq = c.Hq; a.H = c.H; a.G = G; a.B = c.B; a.causal = c.causal;
  a.scale_log2 = c.scale * 1.44269504088896340736f;
  b.O = static_cast<const __nv_bfloat16*>(O);
  b.dO = static_cast<const __nv_bfloat16*>(dO);
  b.LSE = LSE;
  b.dQ = dQ; b.dK = dK; b.dV = dV; b.scale = c.scale;
  const int64_t n_sel = (int64_t)c.H * c.T * c.B;
  if ((e = cudaMemsetAsync(a.cnt, 0, (size_t)c.H * c.NL * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dQ, 0, (size_t)c.T * c.Hq * kDim * 4, st)) != cudaSuccess) return e;
  k_tl_count<<<(unsigned)ceil_div(n_sel, 256), 256, 0, st>>>(a);
  k_tl_scan<<<(unsigned)c.H, 1024, 0, st>>>(a);
  k_tl_fill<<<(unsigned)ceil_div(n_sel, 256), 256, 0, st>>>(a);
  k_tlb_rows<<<(unsigned)ceil_div(c.T * c.Hq * 32, 256), 256, 0, st>>>(b);
  cudaFuncSetAttribute(k_tlb_leaf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwdSmem);
  k_tlb_leaf<<<dim3((unsigned)c.NL, (unsigned)c.H), kTL, kBwdSmem, st>>>(b);
  return cudaGetLastError();
}

}  // namespace lsa
