// lsa_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/lsa.h"

namespace lsa {

constexpr int kTile = 1024;           // keys per tile in partition / init passes
constexpr int64_t kCtaMaxSeg = 8192;  // segments up to this size: one CTA runs the whole assignment
constexpr int kMeanChunk = 256;       // keys summed by one warp before a second-stage sum
constexpr int kMaxRounds = 4096;      // proposal-round cap of the balanced assignment
constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;  // grid-barrier wait cap (2 s)

struct GridBarrier {
  unsigned arrive;
  unsigned gen;
  int abort;
  int pad;
};

// Device workspace of one tree build, carved out of the caller's buffer.
struct BuildPlan {
  float* Za;
  float* Zb;
  int32_t* pa;
  int32_t* pb;
  int32_t* order;
  float* D;
  uint64_t* pref;
  uint32_t* dbits;
  uint8_t* choice;
  uint8_t* ptr;
  float* mu;
  int32_t* tcnt;
  int64_t* toff;
  uint64_t* cand_h;
  int64_t* cand_slot;
  float* partial;
  uint32_t* hist;
  unsigned long long* thr;
  unsigned long long* prefix;
  uint32_t* need;
  int32_t* active;
  int32_t* flags;
  GridBarrier* bar;
  int iters;
  uint64_t seed;
  int coop_blocks;
};

// Byte sizes of every region of a build workspace (layout shared by the size
// query and the carving of a caller buffer).
size_t build_workspace_layout(const lsa_tree_desc& t, char* base, BuildPlan* plan);

// One balanced assignment (distances, preference lists, deferred acceptance) of
// nseg segments of m latent rows Z [nseg*m][r] to the b centroids of their segment
// (P.mu [nseg*b][r]); the result goes to P.choice.  P needs D, pref, dbits, ptr and,
// for m > kCtaMaxSeg, the grid fields.
cudaError_t run_assign(const BuildPlan& P, const float* Z, int64_t nseg, int64_t m, int b, int r, int max_rounds,
                       int32_t* status, cudaStream_t st);
size_t assign_workspace_layout(int64_t nseg, int64_t m, int b, char* base, BuildPlan* P);

// Latent projection of keys on the tensor cores (bf16, r in {16, 32, 64}, d in {64, 128}):
// Z[h][i] = K[h][i] . W[h] and pos[h][i] = i for i < n.
// run_project picks the tensor-core kernel where supported, fp32 FMAs otherwise.
bool project_tc_supported(int dtype, int r, int d);
cudaError_t run_project(const void* K, int64_t n_cap, const void* W, int64_t n, int32_t n_heads, int r, int d,
                        int dtype, float* Z, int32_t* pos, int32_t* status, cudaStream_t st);
cudaError_t run_project_tc(const void* K, int64_t n_cap, const void* W, int64_t n, int32_t n_heads, int r, int d,
                           float* Z, int32_t* pos, int32_t* status, cudaStream_t st);

cudaError_t run_build(const BuildPlan& P, const lsa_tree_desc& t, void* tree_mem, const void* K, int64_t n_cap,
                      int d, int dtype, const void* W, int32_t pool, int32_t* trace, int32_t* status,
                      cudaStream_t st);
int da_grid_blocks();
// The grown tree of an update on append: old levels as prefixes, the subtree's
// nodes after them, the new top node = mean of the subtree's top centroids.
cudaError_t run_tree_attach(const lsa_tree_desc& old_t, const void* old_mem, const lsa_tree_desc& sub,
                            const void* sub_mem, const lsa_tree_desc& grown, void* grown_mem, cudaStream_t st);

struct SelectArgs {
  const void* Q;
  const void* W;
  const char* tree;
  const int32_t* q_pos;
  int32_t* idx_out;
  int32_t* leaves_out;
  float* qlat_out;
  int32_t* beam_out;
  int32_t* status;
  int64_t T;
  int32_t Hq, Hkv, G, d, r, levels, leaf, beam_max;
  int64_t n_tree;
  int32_t branching[LSA_MAX_LEVELS];
  int32_t beam[LSA_MAX_LEVELS];
  int64_t nodes[LSA_MAX_LEVELS];
  uint64_t off_c[LSA_MAX_LEVELS];
  uint64_t off_m[LSA_MAX_LEVELS];
  uint64_t off_leaf;
  // decode step only (the small-batch kernel): append one K/V row per KV head at
  // app_pos before selecting, and zero the attention's arrival counters
  void* app_K;
  void* app_V;
  const void* app_Kr;
  const void* app_Vr;
  int64_t app_pos, app_ncap;
  int32_t app_row_bytes;
  int32_t* zero_cnt;
  // flat search on the tensor cores: leaves are scanned in the order i -> (i * perm) mod
  // n_leaves (perm coprime with n_leaves), so a query's running threshold rises fast
  int64_t flat_perm;
};
// Streaming multiprocessors of the current device (cached per device; 148 if unknown).
int sm_count();
cudaError_t run_select(const SelectArgs& a, int dtype, cudaStream_t st);
// The same search scheduled level by level over (walk, parent) pairs grouped by
// parent, for large batches; kept lists and outputs equal run_select's bit for bit.
// ws: select_nodes_workspace_bytes(a) bytes of device memory (a.levels >= 2).
size_t select_nodes_workspace_bytes(const SelectArgs& a);
cudaError_t run_select_nodes(const SelectArgs& a, int dtype, void* ws, cudaStream_t st);

// Decode attention (decode.cu): one query token, keys = the kept leaves of every
// KV group (leaf_index slices) + the tail [tail_begin, tail_end), split into
// chunks of 64 keys over CTAs; the last CTA of a group merges the partials.
struct DecAttnArgs {
  const void* Q;              // [Hq][d]
  const void* K;
  const void* V;              // [Hkv][n_cap][d]
  const int32_t* leaves;      // [Hkv][B]
  const int32_t* leaf_index;  // [Hkv][n_tree]
  void* O;                    // [Hq][d]
  float* LSE;                 // [Hq]
  float* part;                // [Hkv][nsplit][G][d + 4] (d outputs, max, sum, 2 pad)
  int32_t* cnt;               // [Hkv], zero on entry, re-zeroed by the last CTA
  int64_t n_cap, n_tree, tail_begin, tail_end;
  int32_t Hq, Hkv, B, leaf, spl, nsplit;
  float scale_log2;
};
int dec_splits(int B, int leaf, int64_t tail_len);
int dec_max_splits(int dtype, int d, int G);
cudaError_t run_dec_attn(const DecAttnArgs& a, int dtype, int d, int G, cudaStream_t st);
// flat search: every leaf of the last level scored, the best beam[levels - 1] kept
cudaError_t run_select_flat(const SelectArgs& a, int dtype, cudaStream_t st);
// flat search on the tensor cores (bf16 inputs, r = 64, at most 32 kept leaves)
bool select_flat_tc_supported(const SelectArgs& a, int dtype);
cudaError_t run_select_flat_tc(const SelectArgs& a, cudaStream_t st);

struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* idx;
  const int32_t* q_pos;
  void* O;
  float* LSE;
  float* part;        // split partials [T][Hq][nsplit][d + 2]
  const void* dO;
  float* dQ;
  float* dK;
  float* dV;
  int32_t* status;
  int64_t T, n_cap, tail_begin, tail_end;
  int32_t Hq, Hkv, G, d, K_sel, causal, nsplit, keys_per_split;
  float scale_log2;   // scale * log2(e)
  float scale;
};
struct TreeAttnCall {
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* leaf_index;
  const int32_t* leaves;
  const int32_t* q_pos;
  void* O;
  float* LSE;
  void* workspace;
  int32_t* status;
  int64_t T, n_cap, n_tree, NL;
  int32_t Hq, H, d, dtype, B, leaf, causal;
  int32_t n_sink, window;     // sink and recent-window keys (0: none; causal calls only)
  float scale;
};
size_t tree_attn_workspace(int64_t H, int64_t NL, int64_t T, int64_t Hq, int d, int B, int leaf, bool fast,
                           int n_sink = 0, int window = 0);
bool tree_attn_fast_path(int dtype, int d, int G, int leaf);
cudaError_t run_tree_attn(const TreeAttnCall& c, cudaStream_t st);
size_t tree_attn_bwd_workspace(int64_t H, int64_t NL, int64_t T, int64_t Hq, int d, int B, int leaf, bool fast);
cudaError_t run_tree_attn_bwd(const TreeAttnCall& c, const void* O, const float* LSE, const void* dO, float* dQ,
                              float* dK, float* dV, cudaStream_t st);
int attn_splits(int64_t T, int Hkv, int64_t keys);
int report_error(int code, const char* msg);
cudaError_t run_kv_append(void* K, void* V, int64_t n_heads, int64_t n_cap, int64_t row_bytes, int64_t pos,
                          const void* Kr, const void* Vr, cudaStream_t st);
cudaError_t run_attn_fwd(const AttnArgs& a, int dtype, cudaStream_t st);
cudaError_t run_attn_bwd(const AttnArgs& a, int dtype, cudaStream_t st);
// idx2 [n_heads][T][K_sel + n_sink + window]: the key lists with the sink and window keys
cudaError_t run_attn_extend(const int32_t* idx, int32_t K_sel, int64_t T, int32_t n_heads, const int32_t* q_pos,
                            int32_t n_sink, int32_t window, int64_t tail_begin, int64_t tail_end, int64_t n_cap,
                            int32_t* idx2, cudaStream_t st);

}  // namespace lsa
