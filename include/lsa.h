/*
 * lsa.h -- C ABI of the LSA (LongCat Sparse Attention) hot path on B200 (sm_100a).
 *
 * The path: lightning-indexer scores -> streaming-aware top-k (flat, or
 * hierarchical over mean-pooled pages) -> gathered-KV sparse MQA/MLA attention,
 * with one index set reusable across a group of layers.
 *
 * Sources for what each call computes:
 *   [LSA]   "LongCat Sparse Attention: Taming the Lightning via Streaming-aware
 *           Hierarchical Cross-Layer Indexing" (arXiv 2608.01662, summary page):
 *           abstract (1) Streaming-Aware, (2) Cross-Layer, (3) Hierarchical
 *           Indexing; key contributions (HI cuts per-query selection from O(L)
 *           to O(L/P + MP); CLI cuts indexing to 1/N); limitations (SI gives 50%
 *           of the budget to fixed regions).
 *   [CARD]  "LongCat-Flash-Lite-Sparse" model card: the SI / CLI / HI bullets.
 *   [DSA]   "DSA Lightning Indexer" article (Baidu AI Cloud): "Lightweight
 *           Scoring Module", "Dynamic Token Selector", "Sparse Attention
 *           Calculator".
 *
 * Conventions (all calls):
 *   - Every tensor argument is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or retains memory. Scratch space is the
 *     caller's `workspace` (size from lsa_workspace_size); it may be NULL when
 *     the required size is 0.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises the host.
 *   - Arguments are validated on the host before anything is launched; a call
 *     that returns an error has launched nothing and written nothing.
 *     lsa_last_error() then holds a one-line reason (thread-local).
 *   - Tensors are dense, row-major, in the shapes stated. bf16 = IEEE bfloat16,
 *     e4m3 = OCP FP8 E4M3 ("e4m3fn"). Every pointer must be 16-byte aligned.
 *   - seq_len[b] (device int32) is the number of cached tokens of sequence b;
 *     the T queries of sequence b sit at absolute positions
 *     pos(t) = seq_len[b] - T + t. Values are clamped to [0, L_max]; a query with
 *     pos < 0 yields an all -1 index row.
 *   - Kernels that wait on on-chip barriers give up after a bounded number of
 *     polls, record a timeout in a per-device status word and return;
 *     lsa_device_status() reads (and clears) it. The attention records there
 *     too any index entry it skipped for being >= L_max.
 *   - No exceptions cross the ABI.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lsa_stream_t; /* same type as cudaStream_t */

typedef enum lsa_status {
  LSA_OK = 0,
  LSA_ERR_INVALID_ARG = 1, /* bad pointer, shape, budget or alignment */
  LSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported limits below */
  LSA_ERR_WORKSPACE = 3,   /* workspace smaller than lsa_workspace_size() */
  LSA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  LSA_ERR_TIMEOUT = 5      /* a kernel gave up waiting on a barrier */
} lsa_status_t;

typedef enum lsa_dtype {
  LSA_BF16 = 0,
  LSA_E4M3 = 1
} lsa_dtype_t;

/* Streaming-aware budget [LSA abstract (1); LSA limitations; CARD "SI"]:
 * k selected tokens per query = the attention sink (first `sink` tokens) + the
 * local window (the `window` most recent visible tokens, minus any already in
 * the sink) + the dynamic top-(k - |sink| - |window|) of the remaining visible
 * tokens by indexer score (ties to the lower index).
 * Requires 0 <= sink, 0 <= window, sink + window <= k, 1 <= k <= 8192. */
typedef struct lsa_budget {
  int32_t k;
  int32_t sink;
  int32_t window;
} lsa_budget_t;

/* Lightning-indexer inputs [DSA "Lightweight Scoring Module"; LSA section 2.2]:
 *   score[b,t,s] = (1/sqrt(d)) * sum_h w[b,t,h] * ReLU(q[b,t,h,:] . k[b,s,:])
 * for s <= pos(t); invisible keys are excluded (score -inf).
 *   q        [B,T,H,d]   bf16, or e4m3 codes with q_scale [B,T,H] (fp32 > 0)
 *   w        [B,T,H]     fp32
 *   k        [B,L_max,d] bf16, or e4m3 codes with k_scale [B,L_max] (fp32 > 0)
 *   seq_len  [B]         int32
 * With e4m3, q and k stand for code * scale (row scales). Supported:
 * d in {64, 128}; H in {4, 8, 16, 32, 64, 128}; L_max % 128 == 0; T >= 1. */
typedef struct lsa_indexer_in {
  int32_t B, T, H, d, L_max;
  lsa_dtype_t dtype;
  const int32_t* seq_len;
  const void* q;
  const float* q_scale; /* e4m3 only, else NULL */
  const float* w;
  const void* k;
  const float* k_scale; /* e4m3 only, else NULL */
} lsa_indexer_in_t;

/* Sparse attention inputs [DSA "Sparse Attention Calculator"; LSA abstract]:
 *   o[b,t,h,:] = sum_j softmax_j(scale * q[b,t,h,:] . K[b,idx_j,:]) V[b,idx_j,:]
 * over the valid (>= 0) entries of the index row; lse = log of the softmax
 * denominator plus the max (natural log). K row (b,s) starts at
 * k + (b*L_max + s)*k_row_stride (d_qk elements); V row at
 * v + (b*L_max + s)*v_row_stride (d_v elements). For MLA (one latent row per
 * token) pass v = k: V is then the first d_v columns of the latent row.
 *   q [B,T,Hq,d_qk] bf16; K, V bf16. Strides in elements, multiples of 8.
 * Supported: (d_qk, d_v) in {(64, 64), (576, 512)}; 1 <= Hq <= 128.
 * FP8 KV (kv_dtype = LSA_E4M3, MLA only; the quantised storage of the DSA
 * article's "Quantized computation" applied to the latent cache): k = v holds
 * e4m3 codes (row stride in elements = bytes, a multiple of 16) and k_scale
 * [B*L_max] the fp32 scale of each token's row, so K = V = code * scale.
 * Scores and outputs are those of the formula above on those values. */
typedef struct lsa_attn_in {
  int32_t B, T, Hq, d_qk, d_v, L_max;
  float scale;
  const int32_t* seq_len;
  const void* q;
  const void* k;
  const void* v;
  int64_t k_row_stride;
  int64_t v_row_stride;
  /* Optional layout promise (0 / 0 or -1 / -1 = none): every index row starts
   * with the streaming prefix lsa_select_streaming writes for this sink and
   * window -- the sink tokens [0, min(sink, pos+1)) ascending, then the window
   * tokens up to pos ascending (LSA abstract (1), SI). The MLA kernel then
   * computes those entries instead of reading them, and its work on them may
   * overlap the kernel in the same stream that writes the rest of idx: that
   * kernel may write idx only, and must not read or write this call's
   * workspace or outputs (q, k, v and seq_len are read before it ends). A row
   * that breaks the promise gives undefined results. */
  int32_t stream_sink, stream_window;
  int32_t kv_dtype;        /* LSA_BF16 (0, the default) or LSA_E4M3 */
  const float* k_scale;    /* LSA_E4M3: per-token scale [B*L_max]; else NULL */
} lsa_attn_in_t;

typedef enum lsa_op {
  LSA_OP_INDEX_FLAT = 0,
  LSA_OP_INDEX_HIER = 1,
  LSA_OP_SELECT = 2,
  LSA_OP_SPARSE_ATTN = 3,
  LSA_OP_LAYER_GROUP = 4,
  LSA_OP_INDEX_COMPRESSED = 5
} lsa_op_t;

/* Arguments of lsa_workspace_size; fill the members the op uses. */
typedef struct lsa_op_args {
  const lsa_indexer_in_t* indexer; /* INDEX_FLAT, INDEX_HIER, LAYER_GROUP, INDEX_COMPRESSED */
  const lsa_attn_in_t* attn;       /* SPARSE_ATTN; LAYER_GROUP: n_layers entries */
  lsa_budget_t budget;             /* INDEX_*, SELECT, LAYER_GROUP; SPARSE_ATTN uses k */
  int32_t P, M;                    /* INDEX_HIER; LAYER_GROUP (P = 0: flat) */
  int32_t n_layers;                /* LAYER_GROUP */
  int32_t B, T, L_max;             /* SELECT */
  int32_t scores_external;         /* INDEX_FLAT, INDEX_COMPRESSED: 1 if the caller passes scores_out */
  int32_t m;                       /* INDEX_COMPRESSED: tokens per entry */
} lsa_op_args_t;

/* One-line description of a status code (static storage). */
const char* lsa_status_string(lsa_status_t status);

/* Reason for the last failed call on this host thread ("" if none). */
const char* lsa_last_error(void);

/* Bytes of workspace `op` needs for `args`. Pure host arithmetic. */
lsa_status_t lsa_workspace_size(lsa_op_t op, const lsa_op_args_t* args, size_t* bytes);

/* Flat indexing [DSA "Lightweight Scoring Module" + "Dynamic Token Selector";
 * LSA abstract (1)]: indexer scores of every visible key, then the streaming
 * selection per query.
 *   idx        [B,T,k] int32 out: sink ascending, window ascending, dynamic
 *              ascending, then -1 padding (fewer than k visible tokens => all
 *              visible tokens). May be NULL (scores only; scores_out required).
 *   scores_out [B,T,L_max] fp32 out, optional: the scores (-inf where invisible).
 *              When NULL the scores live in the workspace. */
lsa_status_t lsa_index_flat(const lsa_indexer_in_t* in, lsa_budget_t budget, int32_t* idx,
                            float* scores_out, void* workspace, size_t workspace_bytes,
                            lsa_stream_t stream);

/* Indexing over compressed entries [DSA article, "Technical Evolution and
 * Applications": the indexer picks the top-k of compressed historical
 * entries]. in->k holds one key per entry, [B, L_max/m, d] (bf16, or e4m3
 * with k_scale [B, L_max/m]); entry e stands for tokens [e m, e m + m) and
 * the query at pos sees it once all of them are cached: (e + 1) m <= pos + 1.
 * in->L_max and seq_len count tokens. Scores are lsa_index_flat's on the entry
 * keys; the streaming selection runs over entries, at the query's last
 * complete entry, with budget.k, sink and window counted in entries. The
 * pages name no compressor: the entry keys are inputs.
 *   m          tokens per entry: a power of 2 in [1, 128] (m = 1 is
 *              lsa_index_flat); L_max % 128 == 0 as for every indexer call
 *   idx        [B,T,k] int32 entry ids out, laid out as lsa_index_flat's (a
 *              query with no complete entry gets -1 everywhere). May be NULL
 *              (scores only; scores_out required).
 *   scores_out [B,T,L_max/m] fp32 out, optional (-inf at entries not yet
 *              complete); else kept in the workspace.
 * Attention over the chosen entries is lsa_sparse_attn on the compressed KV
 * rows [B, L_max/m, d_qk] with these idx. */
lsa_status_t lsa_index_compressed(const lsa_indexer_in_t* in, int32_t m, lsa_budget_t budget,
                                  int32_t* idx, float* scores_out, void* workspace,
                                  size_t workspace_bytes, lsa_stream_t stream);

/* Streaming selection alone [DSA "Dynamic Token Selector"; LSA abstract (1)]
 * over given scores [B,T,L_max] fp32 (-inf = not a candidate; NaN unsupported;
 * -0 ranks equal to +0). Output as lsa_index_flat. Bit-exact for given scores. */
lsa_status_t lsa_select_streaming(const float* scores, const int32_t* seq_len, int32_t B,
                                  int32_t T, int32_t L_max, lsa_budget_t budget, int32_t* idx,
                                  void* workspace, size_t workspace_bytes, lsa_stream_t stream);

/* Size of the static device scratch used by lsa_select_streaming_noalloc:
 * 16 MiB, held on every GPU that loads this library until the process exits. */
#define LSA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* lsa_select_streaming without a workspace: same arguments minus the
 * workspace, same output, same contract. No counterpart in the paper; it is
 * for callers that cannot allocate device memory where they select (a plugin
 * in a serving engine whose memory is pre-reserved for its KV cache, or a
 * latency-critical path that cannot afford cudaMalloc/cudaFree, which may
 * block the host and synchronise the device). It allocates nothing: the
 * selection's scratch is a fixed LSA_NOALLOC_SCRATCH_BYTES buffer compiled
 * into the library.
 *   - Shapes whose scratch (lsa_workspace_size with LSA_OP_SELECT) exceeds
 *     LSA_NOALLOC_SCRATCH_BYTES are rejected with LSA_ERR_WORKSPACE before
 *     anything is launched. Rows of up to 262144 score slots need no
 *     scratch at all (any number of rows); longer rows do: with k=2048 and
 *     sink+window=1024 on a 148-SM B200, L_max=1M admits up to 20 rows.
 *   - The first call on a device (and the first after its context changes,
 *     e.g. after cudaDeviceReset) looks up the buffer's device address, which
 *     may load the library's device code onto that device; make that first
 *     call, per device, before any stream capture begins.
 *   - Every call on a device shares the buffer. Calls whose kernels may
 *     overlap on the GPU (different streams without ordering) race on it and
 *     give undefined results: order them on one stream. Each call clears on
 *     `stream` the parts of the buffer that must start at zero. */
lsa_status_t lsa_select_streaming_noalloc(const float* scores, const int32_t* seq_len, int32_t B,
                                          int32_t T, int32_t L_max, lsa_budget_t budget,
                                          int32_t* idx, lsa_stream_t stream);

/* Page pooling for Hierarchical Indexing [LSA abstract (3); CARD "HI"]:
 *   page_keys[b,p,:] = bf16_rne( (sum_{j<P} k[b, pP+j, :]) / P )
 * summed in fp32 in ascending j, for every full page (pP + P <= seq_len[b]);
 * other page rows are left untouched. k [B,L_max,d] bf16; page_keys
 * [B,L_max/P,d] bf16. P in {16,32,64,128}; L_max % P == 0; d in {64,128}.
 * Called when pages fill, not per query. */
lsa_status_t lsa_pool_pages(const void* k, const int32_t* seq_len, int32_t B, int32_t L_max,
                            int32_t d, int32_t P, void* page_keys, lsa_stream_t stream);

/* Hierarchical indexing [LSA abstract (3), key contributions; CARD "HI"]:
 * coarse scores on page_keys, recall of M pages (pages holding sink or window
 * tokens are forced in; the rest are the top full, fully visible pages of the
 * dynamic region by page score, ties to the lower page), then fine token
 * scores inside the recalled pages and the streaming selection restricted to
 * them. bf16 inputs (e4m3: lsa_index_hier_e4m3). Requires
 * M >= ceil(sink/P) + ceil(window/P) + 1.
 *   idx       [B,T,k] int32 out (layout as lsa_index_flat)
 *   pages_out [B,T,M] int32 out, optional: recalled pages ascending, -1 padded. */
lsa_status_t lsa_index_hier(const lsa_indexer_in_t* in, const void* page_keys, int32_t P,
                            int32_t M, lsa_budget_t budget, int32_t* idx, int32_t* pages_out,
                            void* workspace, size_t workspace_bytes, lsa_stream_t stream);

/* FP8 page pooling for Hierarchical Indexing [LSA abstract (3); DSA "Quantized
 * computation"]: page keys of e4m3 token keys, themselves in e4m3 with one fp32
 * scale per page. For every full page (pP + P <= seq_len[b]):
 *   mean[i]  = (sum_{j<P} fp32(code(k8[b,pP+j,i]) * k_scale[b,pP+j])) / P
 *              (fp32 products and sum, ascending j, one division)
 *   scale    = max_i |mean[i]| / 448 (fp32), or 1 for an all-zero page
 *   code[i]  = e4m3(mean[i] / scale), round to nearest even, saturating to 448
 * page_codes [B,L_max/P,d] e4m3 codes; page_scales [B,L_max/P] fp32; rows of
 * pages that are not full are left untouched. d = 128; P in {16,32,64,128};
 * L_max % P == 0. Called when pages fill, not per query. */
lsa_status_t lsa_pool_pages_e4m3(const void* k8, const float* k_scale, const int32_t* seq_len, int32_t B,
                                 int32_t L_max, int32_t d, int32_t P, void* page_codes, float* page_scales,
                                 lsa_stream_t stream);

/* FP8 hierarchical indexing [LSA abstract (3); DSA "Quantized computation"]:
 * lsa_index_hier on e4m3 inputs (in->dtype == LSA_E4M3: q codes with q_scale,
 * token key codes with k_scale) and e4m3 page keys with their page scales as
 * lsa_pool_pages_e4m3 writes them. Page scores and fine scores are the
 * indexer's formula on the dequantized values (code times scale); recall and
 * selection as lsa_index_hier. Workspace: lsa_workspace_size with
 * LSA_OP_INDEX_HIER and the same descriptor. Requires d = 128. */
lsa_status_t lsa_index_hier_e4m3(const lsa_indexer_in_t* in, const void* page_codes, const float* page_scales,
                                 int32_t P, int32_t M, lsa_budget_t budget, int32_t* idx, int32_t* pages_out,
                                 void* workspace, size_t workspace_bytes, lsa_stream_t stream);

/* Sparse MQA/MLA attention over an index set [DSA "Sparse Attention
 * Calculator"]: idx [B,T,k] int32 (entries < 0 are skipped; entries >= L_max
 * are skipped too and make the next lsa_device_status() return
 * LSA_ERR_INVALID_ARG: the device checks every entry). out [B,T,Hq,d_v] bf16;
 * lse [B,T,Hq] fp32 optional (-inf and out = 0 when a row has no valid index). */
lsa_status_t lsa_sparse_attn(const lsa_attn_in_t* in, const int32_t* idx, int32_t k, void* out,
                             float* lse, void* workspace, size_t workspace_bytes,
                             lsa_stream_t stream);

/* Cross-layer group [LSA abstract (2), key contributions; CARD "CLI"]: one
 * indexing pass (flat if P == 0, else hierarchical over page_keys) whose index
 * set feeds the sparse attention of n_layers layers.
 *   layers [n_layers] attention inputs (own q and KV per layer, same B, T,
 *          L_max and seq_len as the indexer); outs[i] [B,T,Hq,d_v] bf16;
 *   lse_outs NULL or n_layers pointers (each may be NULL);
 *   idx [B,T,k] int32 out, optional (else kept in the workspace).
 * Consecutive MLA layers (d_qk=576, d_v=512) with the same Hq run as one
 * attention launch (up to 4 layers each), so their work overlaps; the
 * attention of every layer starts on its streaming-prefix entries while the
 * selection still runs. Hence the layers' outputs must not overlap one
 * another or idx (LSA_ERR_INVALID_ARG, checked for outs and idx). The split
 * plan of a shared launch differs from a single lsa_sparse_attn call's, so the
 * outputs agree with that call within rounding, not bit for bit. */
lsa_status_t lsa_layer_group(const lsa_indexer_in_t* in, const void* page_keys, int32_t P,
                             int32_t M, lsa_budget_t budget, int32_t n_layers,
                             const lsa_attn_in_t* layers, void* const* outs,
                             float* const* lse_outs, int32_t* idx, void* workspace,
                             size_t workspace_bytes, lsa_stream_t stream);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device, for everything since the last call: LSA_OK; LSA_ERR_TIMEOUT
 * if a kernel gave up waiting; LSA_ERR_INVALID_ARG if an attention index row
 * held an entry >= L_max; LSA_ERR_CUDA if an internal bound did not hold. */
lsa_status_t lsa_device_status(lsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
