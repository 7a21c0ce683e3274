// C ABI of the LSA hot path (declarations and contracts in include/lsa.h).
//
// Host side only: argument validation, workspace layout, TMA tensor-map
// encoding and kernel launches. Nothing here allocates device memory or
// synchronises the stream (except lsa_device_status, which exists to do so).
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "lsa.h"
#include "ptx.cuh"

namespace lsa {

// Per-device status word: kernels that give up waiting OR LSA_ERR_TIMEOUT into it.
__device__ int g_device_status = 0;

namespace {

thread_local char g_err[512] = {0};

lsa_status_t fail(lsa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

lsa_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(LSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define LSA_CHECK_CUDA(expr, what)                  \
  do {                                              \
    cudaError_t _e = (expr);                        \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool is_pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

// ------------------------------------------------------------ tensor maps --
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, inner] with 128-byte swizzled boxes [box_rows, box_inner].
lsa_status_t make_tmap(CUtensorMap* m, const void* base, bool fp8, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const uint32_t elt = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * elt};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LSA_OK;
}

// bf16 rows of `inner` elements spaced `row_stride` elements apart.
lsa_status_t make_tmap_strided(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride,
                               uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LSA_ERR_CUDA, "cuTensorMapEncodeTiled (rows) failed (%d)", static_cast<int>(r));
  return LSA_OK;
}

// --------------------------------------------------------------- validation --
lsa_status_t check_budget(lsa_budget_t bu) {
  if (bu.k < 1 || bu.k > 8192) return fail(LSA_ERR_UNSUPPORTED, "budget k=%d outside [1, 8192]", bu.k);
  if (bu.sink < 0 || bu.window < 0) return fail(LSA_ERR_INVALID_ARG, "negative sink/window");
  if (static_cast<long long>(bu.sink) + bu.window > bu.k)
    return fail(LSA_ERR_INVALID_ARG, "sink (%d) + window (%d) exceed the budget k=%d", bu.sink, bu.window, bu.k);
  return LSA_OK;
}

lsa_status_t check_indexer(const lsa_indexer_in_t* in, bool allow_fp8) {
  if (!in) return fail(LSA_ERR_INVALID_ARG, "null indexer descriptor");
  if (in->B < 1 || in->T < 1 || in->L_max < 1) return fail(LSA_ERR_INVALID_ARG, "B, T and L_max must be >= 1");
  if (in->d != 64 && in->d != 128) return fail(LSA_ERR_UNSUPPORTED, "indexer d=%d not in {64, 128}", in->d);
  if (!is_pow2_in(in->H, 4, 128)) return fail(LSA_ERR_UNSUPPORTED, "indexer H=%d not in {4,...,128} (power of 2)", in->H);
  if (in->L_max % 128 != 0) return fail(LSA_ERR_UNSUPPORTED, "L_max=%d must be a multiple of 128", in->L_max);
  if (static_cast<long long>(in->B) * in->L_max >= (1ll << 31) ||
      static_cast<long long>(in->B) * in->T * in->H >= (1ll << 31))
    return fail(LSA_ERR_UNSUPPORTED, "tensor too large for 32-bit row coordinates");
  if (!in->seq_len || !in->q || !in->w || !in->k) return fail(LSA_ERR_INVALID_ARG, "null indexer tensor");
  if (!aligned16(in->q) || !aligned16(in->k) || !aligned16(in->w))
    return fail(LSA_ERR_INVALID_ARG, "indexer tensors must be 16-byte aligned");
  if (in->dtype == LSA_E4M3) {
    if (!allow_fp8) return fail(LSA_ERR_UNSUPPORTED, "e4m3 inputs are supported by flat indexing only");
    if (in->d != 128) return fail(LSA_ERR_UNSUPPORTED, "e4m3 indexer requires d = 128");
    if (!in->q_scale || !in->k_scale) return fail(LSA_ERR_INVALID_ARG, "e4m3 inputs need q_scale and k_scale");
  } else if (in->dtype != LSA_BF16) {
    return fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(in->dtype));
  }
  return LSA_OK;
}

lsa_status_t check_attn(const lsa_attn_in_t* at, int k) {
  if (!at) return fail(LSA_ERR_INVALID_ARG, "null attention descriptor");
  if (at->B < 1 || at->T < 1 || at->L_max < 1) return fail(LSA_ERR_INVALID_ARG, "B, T and L_max must be >= 1");
  if (at->Hq < 1 || at->Hq > 128) return fail(LSA_ERR_UNSUPPORTED, "Hq=%d outside [1, 128]", at->Hq);
  const bool mla = at->d_qk == 576 && at->d_v == 512;
  const bool small = at->d_qk == 64 && at->d_v == 64;
  if (!mla && !small) return fail(LSA_ERR_UNSUPPORTED, "(d_qk, d_v) = (%d, %d) unsupported", at->d_qk, at->d_v);
  if (!at->seq_len || !at->q || !at->k || !at->v) return fail(LSA_ERR_INVALID_ARG, "null attention tensor");
  if (!aligned16(at->q) || !aligned16(at->k) || !aligned16(at->v))
    return fail(LSA_ERR_INVALID_ARG, "attention tensors must be 16-byte aligned");
  if (at->k_row_stride < at->d_qk || at->k_row_stride % 8 || at->v_row_stride < at->d_v || at->v_row_stride % 8)
    return fail(LSA_ERR_INVALID_ARG, "row strides must cover the row and be multiples of 8 elements");
  const bool alias = at->v == at->k && at->v_row_stride == at->k_row_stride;
  if (mla && !alias) return fail(LSA_ERR_UNSUPPORTED, "d_qk=576/d_v=512 requires v == k (MLA latent rows)");
  if (at->kv_dtype != LSA_BF16 && at->kv_dtype != LSA_E4M3)
    return fail(LSA_ERR_INVALID_ARG, "kv_dtype %d is neither LSA_BF16 nor LSA_E4M3", at->kv_dtype);
  if (at->kv_dtype == LSA_E4M3) {
    if (!mla) return fail(LSA_ERR_UNSUPPORTED, "e4m3 KV needs the MLA shape (d_qk=576, d_v=512)");
    if (!at->k_scale || (reinterpret_cast<uintptr_t>(at->k_scale) & 3u))
      return fail(LSA_ERR_INVALID_ARG, "e4m3 KV needs k_scale (fp32, 4-byte aligned)");
    if (at->k_row_stride % 16) return fail(LSA_ERR_INVALID_ARG, "e4m3 KV row stride must be a multiple of 16 bytes");
  } else if (at->k_scale) {
    return fail(LSA_ERR_INVALID_ARG, "k_scale is for e4m3 KV only");
  }
  if (!(at->scale > 0.f) || !std::isfinite(at->scale)) return fail(LSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (k < 1 || k > 8192) return fail(LSA_ERR_UNSUPPORTED, "index row length %d outside [1, 8192]", k);
  if (at->stream_sink < -1 || at->stream_window < -1)
    return fail(LSA_ERR_INVALID_ARG, "stream_sink / stream_window below -1");
  if (at->stream_sink > 0 || at->stream_window > 0) {
    if (at->stream_sink < 0 || at->stream_window < 0 ||
        static_cast<long long>(at->stream_sink) + at->stream_window > k)
      return fail(LSA_ERR_INVALID_ARG, "streaming prefix (sink %d + window %d) must fit the index row of %d",
                  at->stream_sink, at->stream_window, k);
  }
  if (static_cast<long long>(at->B) * at->T * at->Hq >= (1ll << 31))
    return fail(LSA_ERR_UNSUPPORTED, "too many query rows");
  return LSA_OK;
}

// ---------------------------------------------------------- plan helpers --
struct FlatPlan {
  int NQ, N, G, n_tiles;
};

FlatPlan flat_plan(int T, int H, int L_rows) {
  FlatPlan p;
  int n = 16;
  while (n < 256 && n < T * H) n <<= 1;
  if (n < H) n = H;
  p.N = n;
  p.NQ = n / H;
  p.G = (T + p.NQ - 1) / p.NQ;
  p.n_tiles = (L_rows + 127) / 128;
  return p;
}

struct AttnPlan {
  int n_split, bps, nvp;
  int fixed_blocks, fixed_splits, bps_fixed;   // streaming-prefix blocks and their own splits
};

// `layers`: layers that share the launch (their CTAs split the GPU between them).
AttnPlan attn_plan(const lsa_attn_in_t* at, int k, int layers = 1) {
  AttnPlan p;
  const int rows = at->B * at->T;
  p.nvp = at->d_v >= 512 ? 2 : 1;
  const int bn = at->d_qk == 576 ? kAttnBNMla : kAttnBN;   // KV rows per kernel block
  const int nblk = (k + bn - 1) / bn;
  int ns = device_sm_count() / (rows * layers * p.nvp);
  if (ns < 1) ns = 1;
  if (ns > nblk) ns = nblk;
  if (ns > 64) ns = 64;   // the split combine merges at most 64 partials
  p.bps = (nblk + ns - 1) / ns;
  p.n_split = (nblk + p.bps - 1) / p.bps;
  p.fixed_blocks = p.fixed_splits = p.bps_fixed = 0;
  // MLA with the streaming-prefix promise: the prefix splits run while the top-k
  // still works, so the rest of the row is the critical path -- give it splits of
  // half the size (the prefix keeps the plain size).
  const int prefix = (at->stream_sink > 0 ? at->stream_sink : 0) + (at->stream_window > 0 ? at->stream_window : 0);
  if (at->d_qk == 576 && prefix / bn >= 2 && p.bps >= 2) {
    const int F = std::min(nblk, prefix / bn);
    const int bps_d = p.bps / 2;
    const int fs = (F + p.bps - 1) / p.bps;
    const int ds = (nblk - F + bps_d - 1) / bps_d;
    if (fs + ds <= 64) {
      p.fixed_blocks = F;
      p.fixed_splits = fs;
      p.bps_fixed = p.bps;
      p.bps = bps_d;
      p.n_split = fs + ds;
    }
  }
  return p;
}

size_t attn_ws_bytes(const lsa_attn_in_t* at, int k, int layers = 1) {
  const AttnPlan p = attn_plan(at, k, layers);
  if (p.n_split <= 1) return 0;
  const size_t rows = static_cast<size_t>(at->B) * at->T;
  const size_t nm = rows * p.n_split * at->Hq;
  return align_up(nm * at->d_v * 2, 256) + 2 * align_up(nm * 4, 256);
}

// Layers [i, i + n) of a group that go into one attention launch: consecutive
// MLA layers with the same head count and KV type, at most kMaxLaunchLayers.
int group_launch_layers(const lsa_attn_in_t* layers, int i, int n_layers) {
  const lsa_attn_in_t& f = layers[i];
  if (!(f.d_qk == 576 && f.d_v == 512)) return 1;
  int n = 1;
  while (n < kMaxLaunchLayers && i + n < n_layers && layers[i + n].d_qk == 576 && layers[i + n].d_v == 512 &&
         layers[i + n].Hq == f.Hq && layers[i + n].kv_dtype == f.kv_dtype)
    ++n;
  return n;
}

// The group's layer i as launched: its own selection wrote the index rows, so
// their streaming prefix is known.
lsa_attn_in_t group_layer(const lsa_attn_in_t* layers, int i, lsa_budget_t bu) {
  lsa_attn_in_t lay = layers[i];
  lay.stream_sink = bu.sink;
  lay.stream_window = bu.window;
  return lay;
}

SelectPlan token_select_plan(int rows, int n_slots, lsa_budget_t bu) {
  return select_plan(rows, n_slots, std::max(0, bu.k - bu.sink - bu.window), device_sm_count());
}

SelectPlan page_select_plan(int rows, int n_pages, int M) { return select_plan(rows, n_pages, M, device_sm_count()); }

size_t hier_ws_bytes(const lsa_indexer_in_t* in, int P, int M, lsa_budget_t bu, bool pages_external) {
  const int rows = in->B * in->T;
  size_t s = align_up(static_cast<size_t>(rows) * (in->L_max / P) * 4, 256);   // page scores
  if (!pages_external) s += align_up(static_cast<size_t>(rows) * M * 4, 256);   // recalled pages
  s += align_up(static_cast<size_t>(rows) * M * P * 4, 256);                     // fine candidate scores
  s += std::max(select_ws_bytes(rows, page_select_plan(rows, in->L_max / P, M)),
                select_ws_bytes(rows, token_select_plan(rows, M * P, bu)));      // selection scratch
  return s;
}

// Entries of m tokens per sequence, and the selection's entry shift log2(m).
int entry_shift_of(int m) {
  int sh = 0;
  while ((1 << sh) < m) ++sh;
  return sh;
}

size_t compressed_ws_bytes(const lsa_indexer_in_t* in, int m, lsa_budget_t bu, bool scores_external) {
  const int rows = in->B * in->T;
  const int n_e = in->L_max / m;
  size_t s = scores_external ? 0 : align_up(static_cast<size_t>(rows) * n_e * 4, 256);
  return s + select_ws_bytes(rows, token_select_plan(rows, n_e, bu));
}

size_t flat_ws_bytes(const lsa_indexer_in_t* in, lsa_budget_t bu, bool scores_external) {
  const int rows = in->B * in->T;
  size_t s = scores_external ? 0 : align_up(static_cast<size_t>(rows) * in->L_max * 4, 256);
  return s + select_ws_bytes(rows, token_select_plan(rows, in->L_max, bu));
}

// ------------------------------------------------------------ launchers --
// Where the indexer writes the selection's group maxima (FLAT scores feeding a
// filter-launch selection), or nothing.
struct FusedSummary {
  uint32_t* gmax = nullptr;
  int gmax_stride = 0, g0_shift = 0;
  unsigned* counters = nullptr;
  int sink = 0, window = 0;
};

lsa_status_t run_flat_scores(const lsa_indexer_in_t* in, const void* keys, int L_rows, int vis_shift,
                             float* scores, cudaStream_t st, const FusedSummary& fs = FusedSummary{}) {
  const bool fp8 = in->dtype == LSA_E4M3;
  const FlatPlan fp = flat_plan(in->T, in->H, L_rows);
  CUtensorMap tm_k, tm_q;
  const uint32_t box_inner = fp8 ? 128 : 64;
  lsa_status_t s = make_tmap(&tm_k, keys, fp8, in->d, static_cast<uint64_t>(in->B) * L_rows, box_inner, 128);
  if (s != LSA_OK) return s;
  s = make_tmap(&tm_q, in->q, fp8, in->d, static_cast<uint64_t>(in->B) * in->T * in->H, box_inner, fp.N);
  if (s != LSA_OK) return s;
  IndexerArgs a{};
  a.B = in->B; a.T = in->T; a.H = in->H; a.d = in->d;
  a.L_rows = L_rows; a.L_max = in->L_max;
  a.NQ = fp.NQ; a.N = fp.N; a.G = fp.G; a.n_tiles = fp.n_tiles;
  a.vis_shift = vis_shift; a.gather = 0;
  a.multi_group = fp.G > 1;
  indexer_pick_pipeline(in->d, fp8, fp.N, &a.stages, &a.nbuf_b);
  a.n_acc = indexer_n_acc(fp.N);
  a.n_items = static_cast<long long>(in->B) * fp.G * fp.n_tiles;
  a.seq_len = in->seq_len; a.w = in->w; a.q_scale = in->q_scale; a.k_scale = in->k_scale;
  a.out = scores; a.out_row_stride = L_rows;
  a.inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(in->d));
  a.gmax = fs.gmax; a.gmax_stride = fs.gmax_stride; a.g0_shift = fs.g0_shift; a.sel_counters = fs.counters;
  if (fs.gmax) { a.sink = fs.sink; a.window = fs.window; }
  a.status = device_status_ptr();
  const int grid = static_cast<int>(std::min<long long>(a.n_items, device_sm_count()));
  if (grid < 1) return LSA_OK;
  LSA_CHECK_CUDA(launch_indexer(tm_k, tm_q, a, fp8, grid, st), "indexer launch");
  return LSA_OK;
}

lsa_status_t run_select(int mode, int B, int T, int L_max, const int* seq_len, const float* scores,
                        long long row_stride, int n_slots, lsa_budget_t bu, int P, int M, const int* pages,
                        int* out, int out_len, void* sws, cudaStream_t st, int entry_shift = 0,
                        bool summary_ready = false) {
  SelectArgs a{};
  a.mode = mode; a.B = B; a.T = T; a.L_max = L_max; a.seq_len = seq_len;
  a.entry_shift = entry_shift;
  a.scores = scores; a.row_stride = row_stride; a.n_slots = n_slots;
  a.k = bu.k; a.sink = bu.sink; a.window = bu.window; a.P = P; a.M = M; a.pages = pages;
  a.out = out; a.out_len = out_len;
  a.status = device_status_ptr();
  const SelectPlan p = mode == kSelectPages ? page_select_plan(B * T, n_slots, M)
                                            : token_select_plan(B * T, n_slots, bu);
  LSA_CHECK_CUDA(launch_select(a, p, sws, st, summary_ready && p.filter), "select launch");
  return LSA_OK;
}

// The indexer-side half of the fused decode selection: when token selection
// over n_slots will take the filter launch, the FLAT indexer writes its group
// maxima (and clears its counters) into the selection workspace `sws`.
FusedSummary fused_summary(int rows, int n_slots, lsa_budget_t bu, void* sws) {
  FusedSummary fs;
  const SelectPlan p = token_select_plan(rows, n_slots, bu);
  if (!p.filter) return fs;
  const FilterLayout Ly = filter_layout(rows, p);
  uint8_t* w = static_cast<uint8_t*>(sws);
  fs.gmax = reinterpret_cast<uint32_t*>(w + Ly.gmax);
  fs.gmax_stride = p.gmax_stride;
  fs.g0_shift = p.g0_shift;
  fs.counters = reinterpret_cast<unsigned*>(w + Ly.counters);
  fs.sink = bu.sink;
  fs.window = bu.window;
  return fs;
}

// Hierarchical indexing; e4m3 inputs (in->dtype) come with page_scales, the
// per-page fp32 scales of the e4m3 page codes.
lsa_status_t run_hier(const lsa_indexer_in_t* in, const void* page_keys, int P, int M, lsa_budget_t bu,
                      int* idx, int* pages_out, void* ws, cudaStream_t st, const float* page_scales = nullptr) {
  const bool fp8 = in->dtype == LSA_E4M3;
  const size_t rows = static_cast<size_t>(in->B) * in->T;
  const int n_pages = in->L_max / P;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* page_scores = reinterpret_cast<float*>(w);
  w += align_up(rows * n_pages * 4, 256);
  int* pages = pages_out;
  if (!pages) {
    pages = reinterpret_cast<int*>(w);
    w += align_up(rows * M * 4, 256);
  }
  float* cand = reinterpret_cast<float*>(w);
  w += align_up(rows * static_cast<size_t>(M) * P * 4, 256);
  void* sws = w;   // selection scratch (reused by both selections)

  // 1) coarse scores over full, fully visible pages
  int p_shift = 0;
  while ((1 << p_shift) < P) ++p_shift;
  lsa_indexer_in_t pin = *in;   // the page keys (and, for e4m3, their scales) take the keys' place
  pin.k_scale = page_scales;
  lsa_status_t s = run_flat_scores(&pin, page_keys, n_pages, p_shift, page_scores, st);
  if (s != LSA_OK) return s;
  // 2) recall: forced sink/window pages + top pages of the dynamic region (ascending)
  s = run_select(kSelectPages, in->B, in->T, in->L_max, in->seq_len, page_scores, n_pages, n_pages, bu, P, M,
                 nullptr, pages, M, sws, st);
  if (s != LSA_OK) return s;
  // 3) fine scores over the recalled pages' tokens
  {
    CUtensorMap tm_k, tm_q;
    const uint32_t box_inner = fp8 ? 128 : 64;   // one 128-byte swizzle span per box row
    s = make_tmap(&tm_k, in->k, fp8, in->d, static_cast<uint64_t>(in->B) * in->L_max, box_inner, P);
    if (s != LSA_OK) return s;
    const int N = in->H < 16 ? 16 : in->H;
    s = make_tmap(&tm_q, in->q, fp8, in->d, static_cast<uint64_t>(in->B) * in->T * in->H, box_inner, N);
    if (s != LSA_OK) return s;
    IndexerArgs a{};
    a.B = in->B; a.T = in->T; a.H = in->H; a.d = in->d;
    a.L_rows = in->L_max; a.L_max = in->L_max;
    a.NQ = 1; a.N = N; a.G = in->T;
    a.n_tiles = (M * P + 127) / 128;
    a.vis_shift = 0; a.gather = 1;
    indexer_pick_pipeline(in->d, fp8, N, &a.stages, &a.nbuf_b);
    a.n_acc = indexer_n_acc(N);
    a.n_items = static_cast<long long>(rows) * a.n_tiles;
    a.seq_len = in->seq_len; a.w = in->w; a.q_scale = in->q_scale; a.k_scale = in->k_scale;
    a.out = cand; a.out_row_stride = static_cast<long long>(M) * P;
    a.inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(in->d));
    a.pages = pages; a.M = M; a.P = P; a.sink = bu.sink; a.window = bu.window;
    a.status = device_status_ptr();
    const int grid = static_cast<int>(std::min<long long>(a.n_items, device_sm_count()));
    LSA_CHECK_CUDA(launch_indexer(tm_k, tm_q, a, fp8, grid, st), "fine indexer launch");
  }
  // 4) token selection restricted to the recalled pages
  return run_select(kSelectHierTokens, in->B, in->T, in->L_max, in->seq_len, cand, static_cast<long long>(M) * P,
                    M * P, bu, P, M, pages, idx, bu.k, sws, st);
}

// Attention of n layers (1 <= n <= kMaxLaunchLayers) over the same index rows
// in one launch; layer i writes outs[i] / lses[i] and keeps its split
// partials in wss[i] (attn_ws_bytes(&ats[i], k, n) bytes each).
lsa_status_t run_attn(const lsa_attn_in_t* ats, int n, const int* idx, int k, void* const* outs, float* const* lses,
                      uint8_t* const* wss, cudaStream_t st) {
  const AttnPlan p = attn_plan(&ats[0], k, n);
  AttnMaps maps[kMaxLaunchLayers];
  AttnArgs args[kMaxLaunchLayers];
  for (int i = 0; i < n; ++i) {
    const lsa_attn_in_t* at = &ats[i];
    AttnMaps& m = maps[i];
    lsa_status_t s = make_tmap(&m.q, at->q, false, at->d_qk, static_cast<uint64_t>(at->B) * at->T * at->Hq, 64, 128);
    if (s != LSA_OK) return s;
    const uint64_t kv_rows = static_cast<uint64_t>(at->B) * at->L_max;
    m.k_tile = m.k_rows = m.v_tile = m.v_rows = CUtensorMap{};   // e4m3 KV: rows staged by the producer threads
    if (at->kv_dtype != LSA_E4M3) {
      if ((s = make_tmap_strided(&m.k_tile, at->k, at->d_qk, kv_rows, at->k_row_stride, 64, kAttnBN)) != LSA_OK)
        return s;
      if ((s = make_tmap_strided(&m.k_rows, at->k, at->d_qk, kv_rows, at->k_row_stride, 64, 1)) != LSA_OK) return s;
      if ((s = make_tmap_strided(&m.v_tile, at->v, at->d_v, kv_rows, at->v_row_stride, 64, kAttnBN)) != LSA_OK)
        return s;
      if ((s = make_tmap_strided(&m.v_rows, at->v, at->d_v, kv_rows, at->v_row_stride, 64, 1)) != LSA_OK) return s;
    }
    AttnArgs& a = args[i];
    a = AttnArgs{};
    a.B = at->B; a.T = at->T; a.Hq = at->Hq; a.L_max = at->L_max;
    a.d_qk = at->d_qk; a.d_v = at->d_v; a.k = k;
    a.scale_log2 = at->scale * 1.4426950408889634f;
    a.idx = idx;
    a.q = static_cast<const uint16_t*>(at->q);
    a.kp = static_cast<const uint16_t*>(at->k);
    a.vp = static_cast<const uint16_t*>(at->v);
    a.k_stride = at->k_row_stride; a.v_stride = at->v_row_stride;
    a.sep_v = !(at->v == at->k && at->v_row_stride == at->k_row_stride);
    a.kv8 = at->kv_dtype == LSA_E4M3;
    a.k_scale = at->k_scale;
    a.n_split = p.n_split; a.blocks_per_split = p.bps;
    a.fixed_blocks = p.fixed_blocks; a.fixed_splits = p.fixed_splits; a.bps_fixed = p.bps_fixed;
    a.stream_sink = at->stream_sink > 0 ? at->stream_sink : 0;
    a.stream_window = at->stream_window > 0 ? at->stream_window : 0;
    a.seq_len = at->seq_len;
    a.out = static_cast<uint16_t*>(outs[i]);
    a.lse = lses ? lses[i] : nullptr;
    a.status = device_status_ptr();
    if (p.n_split > 1) {
      const size_t nm = static_cast<size_t>(at->B) * at->T * p.n_split * at->Hq;
      uint8_t* w = wss[i];
      a.part_o = reinterpret_cast<uint16_t*>(w);
      w += align_up(nm * at->d_v * 2, 256);
      a.part_m = reinterpret_cast<float*>(w);
      w += align_up(nm * 4, 256);
      a.part_l = reinterpret_cast<float*>(w);
    }
  }
  LSA_CHECK_CUDA(launch_attn(maps, args, n, st), "attention launch");
  if (p.n_split > 1) LSA_CHECK_CUDA(launch_attn_combine(args, n, st), "attention combine launch");
  return LSA_OK;
}

lsa_status_t check_ws(void* ws, size_t have, size_t need) {
  if (have < need) return fail(LSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", have, need);
  if (need > 0 && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return fail(LSA_ERR_INVALID_ARG, "workspace must be non-null and 256-byte aligned");
  return LSA_OK;
}

lsa_status_t check_entry_size(const lsa_indexer_in_t* in, int m) {
  if (!is_pow2_in(m, 1, 128)) return fail(LSA_ERR_UNSUPPORTED, "entry size m=%d not a power of 2 in [1, 128]", m);
  if (in->L_max % m) return fail(LSA_ERR_INVALID_ARG, "L_max must be a multiple of m");
  return LSA_OK;
}

lsa_status_t check_hier_params(const lsa_indexer_in_t* in, int P, int M, lsa_budget_t bu) {
  if (!is_pow2_in(P, 16, 128)) return fail(LSA_ERR_UNSUPPORTED, "page size P=%d not in {16,32,64,128}", P);
  if (in->L_max % P) return fail(LSA_ERR_INVALID_ARG, "L_max must be a multiple of P");
  const int forced_max = (bu.sink + P - 1) / P + (bu.window + P - 1) / P + 1;
  if (M < forced_max) return fail(LSA_ERR_INVALID_ARG, "M=%d below the %d pages sink/window can force", M, forced_max);
  if (M > 8192) return fail(LSA_ERR_UNSUPPORTED, "recall M=%d above 8192", M);
  if (static_cast<long long>(M) * P > (1 << 24)) return fail(LSA_ERR_UNSUPPORTED, "M * P too large");
  return LSA_OK;
}

}  // namespace

lsa_status_t set_error(lsa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

// Identity of the CUDA context current on this host thread, 0 if there is none
// yet (or the driver cannot say). The device address of a __device__ symbol is
// valid only in the context that loaded this library's module, so per-device
// caches of such addresses are keyed by it: after cudaDeviceReset (or any other
// new context) the address is looked up again.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

void* symbol_address_cached(SymbolCache* cache, const void* symbol, cudaError_t* err) {
  *err = cudaSuccess;
  int dev = 0;
  if ((*err = cudaGetDevice(&dev)) != cudaSuccess) return nullptr;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(cache->mu);
  if (dev >= 0 && dev < SymbolCache::kDevices && ctx != 0 && cache->ctx[dev] == ctx) return cache->ptr[dev];
  void* p = nullptr;
  if ((*err = cudaGetSymbolAddress(&p, symbol)) != cudaSuccess) return nullptr;
  if (!p) {
    *err = cudaErrorInvalidSymbol;
    return nullptr;
  }
  // the lookup made the device's primary context current if none was
  const unsigned long long now = ctx != 0 ? ctx : current_context_id();
  if (dev >= 0 && dev < SymbolCache::kDevices && now != 0) {
    cache->ctx[dev] = now;
    cache->ptr[dev] = p;
  }
  return p;
}

int* device_status_ptr() {
  static SymbolCache cache;
  cudaError_t e;
  return static_cast<int*>(symbol_address_cached(&cache, &g_device_status, &e));   // kernels skip a null word
}

// SM counts per device ordinal, filled on first use; safe under concurrent calls
// (both racers store the same value). Ordinals beyond the table are looked up
// on every call.
constexpr int kCachedDevices = 64;

int device_sm_count() {
  static std::atomic<int> cache[kCachedDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;   // no device: plans are only sized (workspace queries)
  const bool cached = dev >= 0 && dev < kCachedDevices;
  if (cached) {
    if (const int c = cache[dev].load(std::memory_order_relaxed)) return c;
  }
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (cached) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, void** args,
                       const cudaLaunchAttribute* extra, int n_extra) {
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  for (int i = 0; i < n_extra && n < 3; ++i) attr[n++] = extra[i];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t set_max_smem(const void* func, size_t bytes) {
  return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

}  // namespace lsa

using namespace lsa;

extern "C" {

const char* lsa_status_string(lsa_status_t s) {
  switch (s) {
    case LSA_OK: return "ok";
    case LSA_ERR_INVALID_ARG: return "invalid argument";
    case LSA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case LSA_ERR_WORKSPACE: return "workspace too small";
    case LSA_ERR_CUDA: return "CUDA error";
    case LSA_ERR_TIMEOUT: return "kernel gave up waiting on a barrier";
  }
  return "unknown status";
}

const char* lsa_last_error(void) { return g_err; }

lsa_status_t lsa_workspace_size(lsa_op_t op, const lsa_op_args_t* args, size_t* bytes) {
  if (!args || !bytes) return fail(LSA_ERR_INVALID_ARG, "null argument");
  *bytes = 0;
  lsa_status_t s;
  switch (op) {
    case LSA_OP_INDEX_FLAT:
      if ((s = check_indexer(args->indexer, true)) != LSA_OK) return s;
      if ((s = check_budget(args->budget)) != LSA_OK) return s;
      *bytes = flat_ws_bytes(args->indexer, args->budget, args->scores_external != 0);
      return LSA_OK;
    case LSA_OP_INDEX_COMPRESSED:
      if ((s = check_indexer(args->indexer, true)) != LSA_OK) return s;
      if ((s = check_entry_size(args->indexer, args->m)) != LSA_OK) return s;
      if ((s = check_budget(args->budget)) != LSA_OK) return s;
      *bytes = compressed_ws_bytes(args->indexer, args->m, args->budget, args->scores_external != 0);
      return LSA_OK;
    case LSA_OP_INDEX_HIER:
      if ((s = check_indexer(args->indexer, true)) != LSA_OK) return s;
      if ((s = check_hier_params(args->indexer, args->P, args->M, args->budget)) != LSA_OK) return s;
      if ((s = check_budget(args->budget)) != LSA_OK) return s;
      *bytes = hier_ws_bytes(args->indexer, args->P, args->M, args->budget, false);
      return LSA_OK;
    case LSA_OP_SELECT:
      if ((s = check_budget(args->budget)) != LSA_OK) return s;
      if (args->B < 1 || args->T < 1 || args->L_max < 1) return fail(LSA_ERR_INVALID_ARG, "B, T and L_max must be >= 1");
      *bytes = select_ws_bytes(args->B * args->T, token_select_plan(args->B * args->T, args->L_max, args->budget));
      return LSA_OK;
    case LSA_OP_SPARSE_ATTN:
      if ((s = check_attn(args->attn, args->budget.k)) != LSA_OK) return s;
      *bytes = attn_ws_bytes(args->attn, args->budget.k);
      return LSA_OK;
    case LSA_OP_LAYER_GROUP: {
      if ((s = check_indexer(args->indexer, args->P == 0)) != LSA_OK) return s;
      if (args->n_layers < 1 || !args->attn) return fail(LSA_ERR_INVALID_ARG, "need n_layers >= 1 attention inputs");
      const lsa_indexer_in_t* in = args->indexer;
      size_t idx_bytes = align_up(static_cast<size_t>(in->B) * in->T * args->budget.k * 4, 256);
      size_t ix = 0;
      if (args->P) {
        if ((s = check_hier_params(in, args->P, args->M, args->budget)) != LSA_OK) return s;
        ix = hier_ws_bytes(in, args->P, args->M, args->budget, false);
      } else {
        ix = flat_ws_bytes(in, args->budget, false);
      }
      for (int i = 0; i < args->n_layers; ++i)
        if ((s = check_attn(&args->attn[i], args->budget.k)) != LSA_OK) return s;
      // Every layer keeps its split partials in a region of its own, apart from
      // the selection's scratch: with the streaming-prefix promise a launch's
      // first splits may run while the kernel before it (the selection, or the
      // previous launch's combine) still reads its own buffers.
      size_t at = 0;
      for (int i = 0; i < args->n_layers;) {
        const int n = group_launch_layers(args->attn, i, args->n_layers);
        for (int j = i; j < i + n; ++j) {
          const lsa_attn_in_t lay = group_layer(args->attn, j, args->budget);
          at += attn_ws_bytes(&lay, args->budget.k, n);
        }
        i += n;
      }
      *bytes = idx_bytes + ix + at;
      return LSA_OK;
    }
  }
  return fail(LSA_ERR_INVALID_ARG, "unknown op %d", static_cast<int>(op));
}

lsa_status_t lsa_index_flat(const lsa_indexer_in_t* in, lsa_budget_t budget, int32_t* idx, float* scores_out,
                            void* workspace, size_t workspace_bytes, lsa_stream_t stream) {
  lsa_status_t s;
  if ((s = check_indexer(in, true)) != LSA_OK) return s;
  if ((s = check_budget(budget)) != LSA_OK) return s;
  if (!idx && !scores_out) return fail(LSA_ERR_INVALID_ARG, "need idx or scores_out");
  if ((idx && !aligned16(idx)) || (scores_out && !aligned16(scores_out)))
    return fail(LSA_ERR_INVALID_ARG, "outputs must be 16-byte aligned");
  const size_t need = flat_ws_bytes(in, budget, scores_out != nullptr);
  if ((s = check_ws(workspace, workspace_bytes, need)) != LSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* scores = scores_out;
  if (!scores) {
    scores = reinterpret_cast<float*>(w);
    w += align_up(static_cast<size_t>(in->B) * in->T * in->L_max * 4, 256);
  }
  const FusedSummary fs = idx ? fused_summary(in->B * in->T, in->L_max, budget, w) : FusedSummary{};
  if ((s = run_flat_scores(in, in->k, in->L_max, 0, scores, st, fs)) != LSA_OK) return s;
  if (idx)
    return run_select(kSelectTokens, in->B, in->T, in->L_max, in->seq_len, scores, in->L_max, in->L_max, budget, 0,
                      0, nullptr, idx, budget.k, w, st, 0, fs.gmax != nullptr);
  return LSA_OK;
}

lsa_status_t lsa_index_compressed(const lsa_indexer_in_t* in, int32_t m, lsa_budget_t budget, int32_t* idx,
                                  float* scores_out, void* workspace, size_t workspace_bytes, lsa_stream_t stream) {
  lsa_status_t s;
  if ((s = check_indexer(in, true)) != LSA_OK) return s;
  if ((s = check_entry_size(in, m)) != LSA_OK) return s;
  if ((s = check_budget(budget)) != LSA_OK) return s;
  if (!idx && !scores_out) return fail(LSA_ERR_INVALID_ARG, "need idx or scores_out");
  if ((idx && !aligned16(idx)) || (scores_out && !aligned16(scores_out)))
    return fail(LSA_ERR_INVALID_ARG, "outputs must be 16-byte aligned");
  const size_t need = compressed_ws_bytes(in, m, budget, scores_out != nullptr);
  if ((s = check_ws(workspace, workspace_bytes, need)) != LSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int n_e = in->L_max / m;
  const int shift = entry_shift_of(m);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* scores = scores_out;
  if (!scores) {
    scores = reinterpret_cast<float*>(w);
    w += align_up(static_cast<size_t>(in->B) * in->T * n_e * 4, 256);
  }
  const FusedSummary fs = idx ? fused_summary(in->B * in->T, n_e, budget, w) : FusedSummary{};
  if ((s = run_flat_scores(in, in->k, n_e, shift, scores, st, fs)) != LSA_OK) return s;
  if (idx)
    return run_select(kSelectTokens, in->B, in->T, in->L_max, in->seq_len, scores, n_e, n_e, budget, 0, 0, nullptr,
                      idx, budget.k, w, st, shift, fs.gmax != nullptr);
  return LSA_OK;
}

lsa_status_t lsa_select_streaming(const float* scores, const int32_t* seq_len, int32_t B, int32_t T,
                                  int32_t L_max, lsa_budget_t budget, int32_t* idx, void* workspace,
                                  size_t workspace_bytes, lsa_stream_t stream) {
  lsa_status_t s;
  if ((s = check_budget(budget)) != LSA_OK) return s;
  if (!scores || !seq_len || !idx) return fail(LSA_ERR_INVALID_ARG, "null tensor");
  if (B < 1 || T < 1 || L_max < 1) return fail(LSA_ERR_INVALID_ARG, "B, T and L_max must be >= 1");
  if (static_cast<long long>(B) * T > 65535) return fail(LSA_ERR_UNSUPPORTED, "at most 65535 query rows per call");
  const size_t need = select_ws_bytes(B * T, token_select_plan(B * T, L_max, budget));
  if ((s = check_ws(workspace, workspace_bytes, need)) != LSA_OK) return s;
  return run_select(kSelectTokens, B, T, L_max, seq_len, scores, L_max, L_max, budget, 0, 0, nullptr, idx,
                    budget.k, workspace, reinterpret_cast<cudaStream_t>(stream));
}

lsa_status_t lsa_pool_pages(const void* k, const int32_t* seq_len, int32_t B, int32_t L_max, int32_t d, int32_t P,
                            void* page_keys, lsa_stream_t stream) {
  if (!k || !seq_len || !page_keys) return fail(LSA_ERR_INVALID_ARG, "null tensor");
  if (!aligned16(k) || !aligned16(page_keys)) return fail(LSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (B < 1 || L_max < 1) return fail(LSA_ERR_INVALID_ARG, "B and L_max must be >= 1");
  if (d != 64 && d != 128) return fail(LSA_ERR_UNSUPPORTED, "d=%d not in {64, 128}", d);
  if (!is_pow2_in(P, 16, 128)) return fail(LSA_ERR_UNSUPPORTED, "page size P=%d not in {16,32,64,128}", P);
  if (L_max % P) return fail(LSA_ERR_INVALID_ARG, "L_max must be a multiple of P");
  LSA_CHECK_CUDA(launch_pool(static_cast<const uint16_t*>(k), seq_len, B, L_max, d, P,
                             static_cast<uint16_t*>(page_keys), reinterpret_cast<cudaStream_t>(stream)),
                 "pool launch");
  return LSA_OK;
}

lsa_status_t lsa_index_hier(const lsa_indexer_in_t* in, const void* page_keys, int32_t P, int32_t M,
                            lsa_budget_t budget, int32_t* idx, int32_t* pages_out, void* workspace,
                            size_t workspace_bytes, lsa_stream_t stream) {
  lsa_status_t s;
  if (in && in->dtype == LSA_E4M3)
    return fail(LSA_ERR_UNSUPPORTED, "e4m3 inputs: use lsa_index_hier_e4m3 (page keys come with page scales)");
  if ((s = check_indexer(in, false)) != LSA_OK) return s;
  if ((s = check_budget(budget)) != LSA_OK) return s;
  if ((s = check_hier_params(in, P, M, budget)) != LSA_OK) return s;
  if (!page_keys || !idx) return fail(LSA_ERR_INVALID_ARG, "null page_keys or idx");
  if (!aligned16(page_keys) || !aligned16(idx) || (pages_out && !aligned16(pages_out)))
    return fail(LSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (static_cast<long long>(in->B) * in->T > 65535) return fail(LSA_ERR_UNSUPPORTED, "at most 65535 query rows per call");
  const size_t need = hier_ws_bytes(in, P, M, budget, pages_out != nullptr);
  if ((s = check_ws(workspace, workspace_bytes, need)) != LSA_OK) return s;
  return run_hier(in, page_keys, P, M, budget, idx, pages_out, workspace, reinterpret_cast<cudaStream_t>(stream));
}

lsa_status_t lsa_pool_pages_e4m3(const void* k8, const float* k_scale, const int32_t* seq_len, int32_t B,
                                 int32_t L_max, int32_t d, int32_t P, void* page_codes, float* page_scales,
                                 lsa_stream_t stream) {
  if (!k8 || !k_scale || !seq_len || !page_codes || !page_scales) return fail(LSA_ERR_INVALID_ARG, "null tensor");
  if (!aligned16(k8) || !aligned16(page_codes) || !aligned16(k_scale) || !aligned16(page_scales))
    return fail(LSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (B < 1 || L_max < 1) return fail(LSA_ERR_INVALID_ARG, "B and L_max must be >= 1");
  if (d != 128) return fail(LSA_ERR_UNSUPPORTED, "e4m3 page pooling requires d = 128");
  if (!is_pow2_in(P, 16, 128)) return fail(LSA_ERR_UNSUPPORTED, "page size P=%d not in {16,32,64,128}", P);
  if (L_max % P) return fail(LSA_ERR_INVALID_ARG, "L_max must be a multiple of P");
  LSA_CHECK_CUDA(launch_pool_e4m3(static_cast<const uint8_t*>(k8), k_scale, seq_len, B, L_max, d, P,
                                  static_cast<uint8_t*>(page_codes), page_scales,
                                  reinterpret_cast<cudaStream_t>(stream)),
                 "e4m3 pool launch");
  return LSA_OK;
}

lsa_status_t lsa_index_hier_e4m3(const lsa_indexer_in_t* in, const void* page_codes, const float* page_scales,
                                 int32_t P, int32_t M, lsa_budget_t budget, int32_t* idx, int32_t* pages_out,
                                 void* workspace, size_t workspace_bytes, lsa_stream_t stream) {
  lsa_status_t s;
  if ((s = check_indexer(in, true)) != LSA_OK) return s;
  if (in->dtype != LSA_E4M3) return fail(LSA_ERR_INVALID_ARG, "lsa_index_hier_e4m3 takes e4m3 inputs");
  if ((s = check_budget(budget)) != LSA_OK) return s;
  if ((s = check_hier_params(in, P, M, budget)) != LSA_OK) return s;
  if (!page_codes || !page_scales || !idx) return fail(LSA_ERR_INVALID_ARG, "null page codes, page scales or idx");
  if (!aligned16(page_codes) || !aligned16(page_scales) || !aligned16(idx) || (pages_out && !aligned16(pages_out)))
    return fail(LSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (static_cast<long long>(in->B) * in->T > 65535) return fail(LSA_ERR_UNSUPPORTED, "at most 65535 query rows per call");
  const size_t need = hier_ws_bytes(in, P, M, budget, pages_out != nullptr);
  if ((s = check_ws(workspace, workspace_bytes, need)) != LSA_OK) return s;
  return run_hier(in, page_codes, P, M, budget, idx, pages_out, workspace, reinterpret_cast<cudaStream_t>(stream),
                  page_scales);
}

lsa_status_t lsa_sparse_attn(const lsa_attn_in_t* in, const int32_t* idx, int32_t k, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, lsa_stream_t stream) {
  lsa_status_t s;
  if ((s = check_attn(in, k)) != LSA_OK) return s;
  if (!idx || !out) return fail(LSA_ERR_INVALID_ARG, "null idx or out");
  if (!aligned16(out) || (lse && !aligned16(lse))) return fail(LSA_ERR_INVALID_ARG, "outputs must be 16-byte aligned");
  if (static_cast<long long>(in->B) * in->T > 65535) return fail(LSA_ERR_UNSUPPORTED, "at most 65535 query rows per call");
  if ((s = check_ws(workspace, workspace_bytes, attn_ws_bytes(in, k))) != LSA_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return run_attn(in, 1, idx, k, &out, &lse, &ws, reinterpret_cast<cudaStream_t>(stream));
}

lsa_status_t lsa_layer_group(const lsa_indexer_in_t* in, const void* page_keys, int32_t P, int32_t M,
                             lsa_budget_t budget, int32_t n_layers, const lsa_attn_in_t* layers, void* const* outs,
                             float* const* lse_outs, int32_t* idx, void* workspace, size_t workspace_bytes,
                             lsa_stream_t stream) {
  lsa_status_t s;
  if ((s = check_indexer(in, P == 0)) != LSA_OK) return s;
  if ((s = check_budget(budget)) != LSA_OK) return s;
  if (n_layers < 1 || !layers || !outs) return fail(LSA_ERR_INVALID_ARG, "need n_layers >= 1 layers and outputs");
  if (P) {
    if ((s = check_hier_params(in, P, M, budget)) != LSA_OK) return s;
    if (!page_keys) return fail(LSA_ERR_INVALID_ARG, "hierarchical group needs page_keys");
  }
  if (static_cast<long long>(in->B) * in->T > 65535) return fail(LSA_ERR_UNSUPPORTED, "at most 65535 query rows per call");
  for (int i = 0; i < n_layers; ++i) {
    if ((s = check_attn(&layers[i], budget.k)) != LSA_OK) return s;
    if (layers[i].B != in->B || layers[i].T != in->T || layers[i].L_max != in->L_max)
      return fail(LSA_ERR_INVALID_ARG, "layer %d shapes differ from the indexer's", i);
    if (!outs[i] || !aligned16(outs[i])) return fail(LSA_ERR_INVALID_ARG, "layer %d output null or unaligned", i);
  }
  // Layers' outputs may be written concurrently (one launch, or a launch whose
  // streaming-prefix splits start before the previous one ends): no overlaps,
  // and none with the index rows the selection writes meanwhile.
  auto span = [&](int i, uintptr_t* lo, uintptr_t* hi) {
    *lo = reinterpret_cast<uintptr_t>(outs[i]);
    *hi = *lo + static_cast<uintptr_t>(layers[i].B) * layers[i].T * layers[i].Hq * layers[i].d_v * 2;
  };
  for (int i = 0; i < n_layers; ++i) {
    uintptr_t a0, a1;
    span(i, &a0, &a1);
    for (int j = i + 1; j < n_layers; ++j) {
      uintptr_t b0, b1;
      span(j, &b0, &b1);
      if (a0 < b1 && b0 < a1) return fail(LSA_ERR_INVALID_ARG, "outputs of layers %d and %d overlap", i, j);
    }
    if (idx) {
      const uintptr_t i0 = reinterpret_cast<uintptr_t>(idx);
      const uintptr_t i1 = i0 + static_cast<uintptr_t>(in->B) * in->T * budget.k * 4;
      if (a0 < i1 && i0 < a1) return fail(LSA_ERR_INVALID_ARG, "output of layer %d overlaps idx", i);
    }
  }
  lsa_op_args_t wa{};
  wa.indexer = in; wa.attn = layers; wa.budget = budget; wa.P = P; wa.M = M; wa.n_layers = n_layers;
  size_t need = 0;
  if ((s = lsa_workspace_size(LSA_OP_LAYER_GROUP, &wa, &need)) != LSA_OK) return s;
  if ((s = check_ws(workspace, workspace_bytes, need)) != LSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int32_t* idx_buf = idx ? idx : reinterpret_cast<int32_t*>(w);
  w += align_up(static_cast<size_t>(in->B) * in->T * budget.k * 4, 256);
  uint8_t* attn_ws = w + (P ? hier_ws_bytes(in, P, M, budget, false) : flat_ws_bytes(in, budget, false));
  if (P) {
    if ((s = run_hier(in, page_keys, P, M, budget, idx_buf, nullptr, w, st)) != LSA_OK) return s;
  } else {
    float* scores = reinterpret_cast<float*>(w);
    uint8_t* sws = w + align_up(static_cast<size_t>(in->B) * in->T * in->L_max * 4, 256);
    const FusedSummary fs = fused_summary(in->B * in->T, in->L_max, budget, sws);
    if ((s = run_flat_scores(in, in->k, in->L_max, 0, scores, st, fs)) != LSA_OK) return s;
    if ((s = run_select(kSelectTokens, in->B, in->T, in->L_max, in->seq_len, scores, in->L_max, in->L_max, budget,
                        0, 0, nullptr, idx_buf, budget.k, sws, st, 0, fs.gmax != nullptr)) != LSA_OK)
      return s;
  }
  for (int i = 0; i < n_layers;) {
    const int n = group_launch_layers(layers, i, n_layers);
    lsa_attn_in_t lays[kMaxLaunchLayers];
    float* lses[kMaxLaunchLayers];
    uint8_t* wss[kMaxLaunchLayers];
    for (int j = 0; j < n; ++j) {
      lays[j] = group_layer(layers, i + j, budget);
      lses[j] = lse_outs ? lse_outs[i + j] : nullptr;
      wss[j] = attn_ws;
      attn_ws += attn_ws_bytes(&lays[j], budget.k, n);
    }
    if ((s = run_attn(lays, n, idx_buf, budget.k, outs + i, lses, wss, st)) != LSA_OK) return s;
    i += n;
  }
  return LSA_OK;
}

lsa_status_t lsa_device_status(lsa_stream_t stream) {
  LSA_CHECK_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream synchronize");
  int v = 0;
  LSA_CHECK_CUDA(cudaMemcpyFromSymbol(&v, lsa::g_device_status, sizeof(int)), "status read");
  const int zero = 0;
  LSA_CHECK_CUDA(cudaMemcpyToSymbol(lsa::g_device_status, &zero, sizeof(int)), "status reset");
  if (v & kStatusTimeout) return fail(LSA_ERR_TIMEOUT, "a kernel gave up waiting on a barrier");
  if (v & kStatusInternal) return fail(LSA_ERR_CUDA, "a selection candidate pool bound did not hold");
  if (v & kStatusBadIndex)
    return fail(LSA_ERR_INVALID_ARG, "an attention index row held an entry >= L_max (it was skipped)");
  return LSA_OK;
}

}  // extern "C"
