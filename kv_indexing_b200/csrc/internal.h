// Internal launch interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "lsa.h"

namespace lsa {

// ----------------------------------------------------------------- indexer --
// One work item = one 128-key tile against one query group (NQ queries x H
// heads = N MMA columns). FLAT: key rows [128 j, 128 j + 128) of sequence b.
// GATHER: the 128 candidate slots [128 j, 128 j + 128) of query row r, made of
// 128 / P recalled pages (page ids from `pages`).
struct IndexerArgs {
  int B, T, H, d;
  int L_rows;            // key rows per sequence in the key array
  int L_max;             // token capacity per sequence (seq_len clamp; gather rows)
  int NQ, N, G;          // queries per tile, MMA N (= NQ * H), query groups per sequence
  int n_tiles;           // tiles per group (FLAT) or per query row (GATHER)
  int vis_shift;         // FLAT: key s visible to pos iff s < (pos + 1) >> vis_shift (rows of 2^shift tokens)
  int gather;            // 0 = FLAT, 1 = GATHER
  int multi_group;       // FLAT with several query groups per sequence (prefill):
                         // the score rows are streamed out past L2
  int stages, nbuf_b;    // A-tile ring depth, B-tile buffers (1 or 2)
  int n_acc;             // TMEM accumulators (2 or 4)
  long long n_items;
  const int* seq_len;
  const float* w;
  const float* q_scale;  // e4m3 only
  const float* k_scale;  // e4m3 only (indexed by b * L_rows + s)
  float* out;
  long long out_row_stride;
  float inv_sqrt_d;
  // GATHER
  const int* pages;
  int M, P, sink, window;
  // FLAT, feeding the selection's filter launch (gmax != null): per query row
  // the maximum score key over each group of 2^g0_shift slots that are dynamic
  // candidates (sink and window excluded, visible only), and the selection's
  // per-row counters cleared
  uint32_t* gmax;
  int gmax_stride, g0_shift;
  unsigned* sel_counters;
  int* status;           // per-device status word
};

size_t indexer_smem_bytes(int d, bool fp8, int N, int stages, int nbuf_b);
void indexer_pick_pipeline(int d, bool fp8, int N, int* stages, int* nbuf_b);
int indexer_n_acc(int N);
cudaError_t launch_indexer(const CUtensorMap& tm_k, const CUtensorMap& tm_q, const IndexerArgs& a,
                           bool fp8, int grid, cudaStream_t stream);

// --------------------------------------------------------- streaming select --
// Order-preserving key of a score: larger score, larger key; -inf -> 0 (not a
// candidate), -0 ranks as +0. NaN is not supported.
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                         // -0 ranks as +0
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return k <= 0x007FFFFFu ? 0u : k;                     // -inf: not a candidate
}
#endif

enum SelectMode { kSelectTokens = 0, kSelectHierTokens = 1, kSelectPages = 2 };

struct SelectArgs {
  int mode;
  int B, T;
  int L_max;
  const int* seq_len;
  const float* scores;
  long long row_stride;   // floats between consecutive (b, t) rows
  int n_slots;            // slots per row
  int k, sink, window;    // token budget
  int P, M;               // pages / hier
  int entry_shift;        // > 0: slots are entries of 2^shift tokens (kSelectTokens); the
                          // query's slot position is its last complete entry
  const int* pages;       // kSelectHierTokens: [B*T, M]
  int* out;
  int out_len;            // k (tokens) or M (pages)
  // scratch (workspace): per-CTA candidate lists and per-row arrival counters
  uint32_t* cand_keys;    // [rows, C, cand_cap]
  int* cand_slots;        // [rows, C, cand_cap]
  unsigned* row_arrivals; // [rows]
  int cand_cap;
  int final_in_smem;
  // grid-cooperative path: per-row coordination blocks
  void* grid_ws;
  size_t grid_row_bytes;
  // filter path: group maxima of 2^g0_shift slots (written by group_max_kernel
  // or by the indexer's epilogue), the per-row pool of kept candidates, the
  // per-warp segment table and the per-row counters (arrivals, pool fill)
  uint32_t* gmax;         // [rows][gmax_stride] order-preserving keys, 0 = no candidate
  int gmax_stride;
  int g0_shift, fold;     // the lower bound uses groups of 2^g0_shift * fold slots
  uint32_t* pool_keys;    // [rows][pool_cap]
  int* pool_slots;        // [rows][pool_cap]
  int pool_cap;
  uint4* wtab;            // [rows][C * warps]: (pool base, kept, equal to the bound, 0)
  unsigned* counters;     // [rows][2]
  int* status;
};

// C CTAs per row, `seg` slots each; each keeps at most `cand_cap` candidates.
struct SelectPlan {
  int C, seg, cand_cap;
  bool final_in_smem;
  bool grid;              // grid-cooperative launch (rows * C CTAs co-resident)
  bool cluster;           // one thread-block cluster of C CTAs per row (no workspace)
  int cluster_rc;         // cluster path: keys per thread (4, 8, 16, 32 or 64)
  bool filter;            // filter path: group-maximum bound, C CTAs per row, last CTA finishes
  bool row;               // row path: one CTA per row, the row's keys in registers
  int row_rc;             // row path: keys per thread (8 or 16)
  int g0_shift, fold, gmax_stride, pool_cap;
};

// Workspace layout of the filter path (offsets from the selection workspace).
struct FilterLayout {
  size_t gmax, pool_keys, pool_slots, wtab, counters, total;
};
FilterLayout filter_layout(int rows, const SelectPlan& p);

// d_bound: an upper bound on the dynamic budget of any row (k - sink - window for
// token selection, M for page recall).
SelectPlan select_plan(int rows, int n_slots, int d_bound, int num_sms);
size_t select_ws_bytes(int rows, const SelectPlan& p);
// gmax_ready: the group maxima are already in the workspace and the row
// counters cleared (the indexer's epilogue did both); otherwise a pre-pass
// computes them from the scores.
cudaError_t launch_select(const SelectArgs& a, const SelectPlan& p, void* ws, cudaStream_t stream,
                          bool gmax_ready = false);

// ------------------------------------------------------------------ pooling --
cudaError_t launch_pool(const uint16_t* k, const int* seq_len, int B, int L_max, int d, int P,
                        uint16_t* page_keys, cudaStream_t stream);
// d must be 128 (one warp of four columns per page).
cudaError_t launch_pool_e4m3(const uint8_t* k8, const float* k_scale, const int* seq_len, int B, int L_max, int d,
                             int P, uint8_t* page_codes, float* page_scales, cudaStream_t stream);

// ---------------------------------------------------------- sparse attention --
struct AttnArgs {
  int B, T, Hq, L_max;
  int d_qk, d_v;
  int k;                  // index row length
  float scale_log2;       // scale * log2(e)
  const int* idx;
  const uint16_t* q;      // [rows, Hq, d_qk] bf16
  const uint16_t* kp;     // K rows
  const uint16_t* vp;     // V rows (may alias kp)
  long long k_stride, v_stride;
  int sep_v;              // V rows loaded separately (not a prefix of the K row)
  int kv8;                // MLA: K = V rows are e4m3 codes (row stride in bytes), times k_scale
  const float* k_scale;   // kv8: per-token scale [B * L_max]
  int n_split, blocks_per_split;
  int fixed_blocks, fixed_splits, bps_fixed;   // splits [0, fixed_splits) cover blocks [0, fixed_blocks) in
                                               // bps_fixed-block pieces; the others blocks_per_split each
  int stream_sink, stream_window;   // > 0: index rows start with this streaming prefix (computed, not read)
  const int* seq_len;               // [B] (streaming prefix only)
  uint16_t* out;          // [rows, Hq, d_v] bf16
  float* lse;             // [rows, Hq] or null
  uint16_t* part_o;       // [rows, n_split, Hq, d_v] bf16, each split normalised by its own sum
  float* part_m;          // [rows, n_split, Hq]
  float* part_l;          // [rows, n_split, Hq]
  int* status;            // per-device status word
};

constexpr int kAttnBN = 32;  // KV rows per block (d_qk = 64)
constexpr int kAttnBNMla = 64;  // KV rows per block (MLA, d_qk = 576)

// TMA descriptors of one attention launch: q tiles [128 heads x 64], K/V row
// tiles [32 rows x 64] (contiguous blocks) and one-row boxes for row gathers.
struct AttnMaps {
  CUtensorMap q, k_tile, k_rows, v_tile, v_rows;
};

// One launch may cover several layers of a cross-layer group that share the
// index rows, B, T, L_max, Hq, the head dims and the split plan; each layer has
// its own q, latent rows, scale, outputs and split partials. maps[i] / args[i]
// describe layer i (the shared fields of args[0] are used). MLA only when n > 1.
constexpr int kMaxLaunchLayers = 4;
cudaError_t launch_attn(const AttnMaps* maps, const AttnArgs* args, int n, cudaStream_t stream);
cudaError_t launch_attn_combine(const AttnArgs* args, int n, cudaStream_t stream);

// --------------------------------------------------------------------- misc --
int device_sm_count();
// Records a one-line reason for lsa_last_error() and returns `st`.
lsa_status_t set_error(lsa_status_t st, const char* fmt, ...);
int* device_status_ptr();
// Device address of a __device__ symbol of this library in the current context,
// looked up once per device and context (thread-safe). nullptr and *err on failure.
struct SymbolCache {
  static constexpr int kDevices = 64;
  std::mutex mu;
  unsigned long long ctx[kDevices] = {};
  void* ptr[kDevices] = {};
};
void* symbol_address_cached(SymbolCache* cache, const void* symbol, cudaError_t* err);
cudaError_t set_max_smem(const void* func, size_t bytes);
// Launch with programmatic stream serialization (plus up to two extra launch
// attributes): the kernel may start while the previous kernel in the stream
// finishes, and orders itself with pdl_wait before reading shared inputs.
cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, void** args,
                       const cudaLaunchAttribute* extra = nullptr, int n_extra = 0);

}  // namespace lsa
