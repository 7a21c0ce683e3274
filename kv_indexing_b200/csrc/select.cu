// Streaming-aware top-k selection (LSA paper abstract (1) and the model card's
// "SI" bullet: a fixed attention sink and a local sliding window take part of
// the budget, dynamic top-k by indexer score fills the rest; the DSA Lightning
// Indexer article's "Dynamic Token Selector" for the top-k itself).
//
// Per query row: sink tokens [0, min(S, pos+1)), the window (the W most recent
// visible tokens not already in the sink), then the top D = k - |sink| - |window|
// dynamic candidates by (score descending, index ascending), written in
// ascending index order, then -1 padding. The same kernels select pages for
// Hierarchical Indexing (forced sink/window pages + the top pages of the
// dynamic region, all ascending) and the fine token set over recalled pages.
//
// Scores map to order-preserving uint32 keys (-inf -> 0 = not a candidate,
// -0 -> +0); ties go to the lower slot, so every path equals the definition
// exactly. Launch shapes, chosen by select_plan in this order:
//   row      rows of <= 8192 dynamic slots: one CTA per row, keys in registers,
//            range-radix threshold, ordered emission (select_row_kernel)
//   cluster  rows of <= 8 x 512 x 64 slots: one thread-block cluster of up to
//            8 CTAs per row, 4..64 keys per thread in shared memory, agreement
//            through DSMEM and cluster barriers (select_cluster_kernel)
//   grid     longer rows when rows x CTAs fit the GPU at once: one cooperative
//            launch, agreement through per-row blocks in global memory
//            (select_grid_kernel)
//   filter   rows too long for a cluster, few enough for two CTAs each: a
//            bound from per-group maxima (written by the indexer when fused),
//            per-warp candidate runs, the last CTA of the row finishes
//            (select_filter_kernel)
//   two-level otherwise: each CTA keeps its segment's local top-D candidates,
//            the last CTA of the row merges them (select_kernel)
// None but grid, filter and two-level use a workspace.
#include "internal.h"
#include "ptx.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kDigitBits = 13;   // register-path radix digit
constexpr int kDigits = 1 << kDigitBits;
constexpr int kPer = 8;          // consecutive elements per thread per compaction chunk (fallback)
constexpr int kRL = 16;          // keys per thread, local phase
constexpr int kRF = 32;          // keys per thread, merge phase


struct Plan {
  bool valid;
  int lead_a_lo, lead_a_n, lead_b_lo, lead_b_n;   // fixed outputs at [0, lead_a_n + lead_b_n)
  int dyn_lo, dyn_hi, D, dyn_off;                 // dynamic slots, budget, output offset
  int trail_lo, trail_n;                          // fixed outputs after the dynamic block
};

__device__ __forceinline__ Plan make_plan(const SelectArgs& a, int r) {
  Plan p{};
  const int b = r / a.T, t = r % a.T;
  int L = __ldg(a.seq_len + b);
  L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
  int pos = L - a.T + t;
  if (a.entry_shift > 0) pos = ((pos + 1) >> a.entry_shift) - 1;   // last complete entry
  p.valid = pos >= 0;
  if (!p.valid) return p;
  const int sink_end = min(a.sink, pos + 1);
  const int w_lo = max(sink_end, pos - a.window + 1);
  const int win_n = pos + 1 - w_lo;
  if (a.mode != kSelectPages) {
    p.lead_a_lo = 0;
    p.lead_a_n = sink_end;
    p.lead_b_lo = w_lo;
    p.lead_b_n = win_n;
    p.D = a.k - sink_end - win_n;
    p.dyn_off = sink_end + win_n;
    if (a.mode == kSelectTokens) {
      p.dyn_lo = sink_end;
      p.dyn_hi = min(w_lo, a.n_slots);
    } else {
      p.dyn_lo = 0;
      p.dyn_hi = a.n_slots;
    }
    p.trail_n = 0;
  } else {
    const int P = a.P;
    const int e_lo = (sink_end + P - 1) / P;
    int wp_lo, wp_hi, e_hi;
    if (win_n > 0) {
      wp_lo = max(w_lo / P, e_lo);
      wp_hi = max(pos / P + 1, wp_lo);
      e_hi = w_lo / P;
    } else {
      wp_lo = wp_hi = e_lo;
      e_hi = (pos + 1) / P;
    }
    e_hi = max(min(e_hi, a.n_slots), e_lo);
    p.lead_a_lo = 0;
    p.lead_a_n = e_lo;
    p.lead_b_lo = 0;
    p.lead_b_n = 0;
    p.trail_lo = wp_lo;
    p.trail_n = wp_hi - wp_lo;
    p.D = a.M - e_lo - p.trail_n;
    p.dyn_lo = e_lo;
    p.dyn_hi = e_hi;
    p.dyn_off = e_lo;
  }
  if (p.D < 0) p.D = 0;
  if (p.dyn_hi < p.dyn_lo) p.dyn_hi = p.dyn_lo;
  return p;
}

// Inclusive scan of one value per thread (thread order). Uses `tmp` [kWarps].
__device__ __noinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kWarps ? tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) tmp[lane] = w;
  }
  __syncthreads();
  const uint32_t res = x + (warp > 0 ? tmp[warp - 1] : 0u);
  if (total) *total = tmp[kWarps - 1];
  __syncthreads();
  return res;
}

struct Thr {
  uint32_t thr;       // exact key of the D-th best candidate
  uint32_t need_eq;   // how many keys equal to thr are taken (lowest index first)
  bool all;           // every candidate is taken (fewer than D of them)
};

struct Shared {
  alignas(16) uint32_t hist[kDigits];   // 16-byte aligned: read four bins at a time
  uint32_t tmp[32];
  uint32_t red[3][kWarps];
  uint32_t cnt, mn, mx;
  int bin;
  uint32_t above;
  int last;
};

// Block-wide count / min / max of per-thread partials (into sh.cnt, sh.mn, sh.mx).
__device__ __noinline__ void block_cnt_min_max(uint32_t c, uint32_t mn, uint32_t mx, Shared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sh.red[0][warp] = c;
    sh.red[1][warp] = mn;
    sh.red[2][warp] = mx;
  }
  __syncthreads();
  if (warp == 0) {
    c = lane < kWarps ? sh.red[0][lane] : 0u;
    mn = lane < kWarps ? sh.red[1][lane] : 0xFFFFFFFFu;
    mx = lane < kWarps ? sh.red[2][lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c += __shfl_xor_sync(0xffffffffu, c, o);
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
      sh.cnt = c;
      sh.mn = mn;
      sh.mx = mx;
    }
  }
  __syncthreads();
}

// Exact threshold of the D-th best key of key(0) .. key(n - 1) (key 0 = not a
// candidate); `key` reads element i (shared or global memory).
template <class K>
__device__ Thr cta_threshold_by(K&& key, int n, uint32_t D, Shared& sh) {
  const int tid = threadIdx.x;
  Thr r{0u, 0u, false};
  uint32_t c = 0u;
  for (int i = tid; i < n; i += kThreads) c += key(i) != 0u ? 1u : 0u;
  uint32_t total = 0u;
  block_incl_scan(c, sh.tmp, &total);
  if (total <= D) {
    r.all = true;
    return r;
  }
  if (D == 0u) {
    r.thr = 0xFFFFFFFFu;
    return r;
  }
  uint32_t prefix = 0u, mask = 0u, need = D;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t dmask = static_cast<uint32_t>(nb - 1);
    for (int i = tid; i < nb; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t k = key(i);
      if (k != 0u && (k & mask) == prefix) atomicAdd(&sh.hist[(k >> shift) & dmask], 1u);
    }
    __syncthreads();
    const int per = nb / kThreads;             // bins per thread (4 or 2), counted from the top
    const int hi_bin = nb - per * tid;
    uint32_t local = 0u;
    for (int q = 1; q <= per; ++q) local += sh.hist[hi_bin - q];
    const uint32_t incl = block_incl_scan(local, sh.tmp, nullptr);
    const uint32_t excl = incl - local;
    if (excl < need && need <= incl) {
      uint32_t above = excl;
      for (int q = 1; q <= per; ++q) {
        const int bb = hi_bin - q;
        if (above + sh.hist[bb] >= need) {
          sh.bin = bb;
          sh.above = above;
          break;
        }
        above += sh.hist[bb];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sh.bin) << shift;
    mask |= dmask << shift;
    need -= sh.above;
    __syncthreads();
  }
  r.thr = prefix;
  r.need_eq = need;
  return r;
}

__device__ Thr cta_threshold(const uint32_t* keys, int n, uint32_t D, Shared& sh) {
  return cta_threshold_by([&](int i) { return keys[i]; }, n, D, sh);
}

// Emit the selected elements of keys[0, n) in index order: emit(out_pos, i).
// Returns how many were selected.
template <class F>
__device__ uint32_t cta_emit(const uint32_t* keys, int n, const Thr& t, Shared& sh, F&& emit) {
  const int tid = threadIdx.x;
  uint32_t eq_total = 0u;
  if (!t.all) {
    uint32_t e = 0u;
    for (int i = tid; i < n; i += kThreads) e += (keys[i] == t.thr && keys[i] != 0u) ? 1u : 0u;
    block_incl_scan(e, sh.tmp, &eq_total);
  }
  const bool tie_scan = !t.all && t.need_eq > 0u && t.need_eq < eq_total;
  const bool ties_all = t.need_eq >= eq_total;
  uint32_t eq_run = 0u, sel_run = 0u;
  for (int c0 = 0; c0 < n; c0 += kThreads * kPer) {
    const int i0 = c0 + tid * kPer;
    uint32_t kk[kPer];
    uint32_t ne = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      kk[e] = i0 + e < n ? keys[i0 + e] : 0u;
      ne += (kk[e] == t.thr && kk[e] != 0u) ? 1u : 0u;
    }
    uint32_t eq_tot = 0u, er = 0u;
    if (tie_scan) er = block_incl_scan(ne, sh.tmp, &eq_tot) - ne + eq_run;
    uint32_t selmask = 0u, ns = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const uint32_t k = kk[e];
      bool s = false;
      if (k != 0u) {
        if (t.all || k > t.thr) {
          s = true;
        } else if (k == t.thr) {
          s = tie_scan ? (er < t.need_eq) : ties_all;
          ++er;
        }
      }
      if (s) {
        selmask |= 1u << e;
        ++ns;
      }
    }
    uint32_t sel_tot = 0u;
    uint32_t pos = block_incl_scan(ns, sh.tmp, &sel_tot) - ns + sel_run;
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (selmask & (1u << e)) emit(pos++, i0 + e);
    eq_run += eq_tot;
    sel_run += sel_tot;
  }
  return sel_run;
}


// Exact threshold of the D-th best key among the nonzero keys held in
// registers (thread t holds keys[t*R .. t*R+R)).
template <int R>
__device__ Thr reg_threshold(const uint32_t (&k)[R], uint32_t D, Shared& sh) {
  const int tid = threadIdx.x;
  uint32_t c = 0u, mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
  for (int j = 0; j < R; ++j)
    if (k[j] != 0u) {
      ++c;
      mn = min(mn, k[j]);
      mx = max(mx, k[j]);
    }
  block_cnt_min_max(c, mn, mx, sh);
  Thr r{0u, 0u, false};
  const uint32_t total = sh.cnt, kmin = sh.mn, kmax = sh.mx;
  if (total <= D) {
    r.all = true;
    return r;
  }
  if (D == 0u) {
    r.thr = 0xFFFFFFFFu;
    return r;
  }
  if (kmin == kmax) {
    r.thr = kmax;
    r.need_eq = D;
    return r;
  }
  const int bits = 32 - __clz(kmax - kmin);              // every rel = key - kmin is < 2^bits
  int prev = bits;                                        // keys in play satisfy rel >> prev == hi
  int shift = bits > kDigitBits ? bits - kDigitBits : 0;
  uint32_t hi = 0u, need = D;
  while (true) {
    const int width = prev - shift;                       // digit bits this pass (<= 13)
    const int nb = 1 << width;
    const uint32_t dmask = static_cast<uint32_t>(nb - 1);
    for (int i = tid; i < nb; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const uint32_t rel = k[j] - kmin;
      const bool in = k[j] != 0u && (prev >= 32 || (rel >> prev) == hi);
      if (in) atomicAdd(&sh.hist[(rel >> shift) & dmask], 1u);
    }
    __syncthreads();
    const int per = (nb + kThreads - 1) / kThreads;       // bins per thread, counted from the top
    const int top = nb - per * tid;
    uint32_t local = 0u;
    for (int q = 1; q <= per; ++q)
      if (top - q >= 0) local += sh.hist[top - q];
    const uint32_t incl = block_incl_scan(local, sh.tmp, nullptr);
    const uint32_t excl = incl - local;
    if (excl < need && need <= incl) {
      uint32_t above = excl;
      for (int q = 1; q <= per; ++q) {
        const int bb = top - q;
        if (bb < 0) break;
        if (above + sh.hist[bb] >= need) {
          sh.bin = bb;
          sh.above = above;
          break;
        }
        above += sh.hist[bb];
      }
    }
    __syncthreads();
    hi = (width >= 32 ? 0u : (hi << width)) | static_cast<uint32_t>(sh.bin);
    need -= sh.above;
    __syncthreads();
    if (shift == 0) break;
    prev = shift;
    shift = shift > kDigitBits ? shift - kDigitBits : 0;
  }
  r.thr = kmin + hi;
  r.need_eq = need;
  return r;
}

// Emit the selected register-held keys in index order: emit(out_pos, j).
// Layout (warp-striped): lane l of warp w holds element w*32*R + 32*j + l in
// k[j], so index order is (warp, j, lane). Positions come from per-stripe warp
// ballots plus one exclusive scan over the warps' counts.
template <int R, class F>
__device__ uint32_t reg_emit(const uint32_t (&k)[R], const Thr& t, Shared& sh, F&& emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t gtm[R], eqm[R];
  uint32_t n_gt = 0u, n_eq = 0u;
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const bool nz = k[j] != 0u;
    gtm[j] = __ballot_sync(0xffffffffu, nz && (t.all || k[j] > t.thr));
    eqm[j] = __ballot_sync(0xffffffffu, nz && !t.all && k[j] == t.thr);
    n_gt += __popc(gtm[j]);
    n_eq += __popc(eqm[j]);
  }
  // ties before this warp -> this warp's share of the need_eq lowest-index ties
  if (lane == 0) sh.red[0][warp] = n_eq;
  __syncthreads();
  uint32_t eq_before = 0u;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) eq_before += w < warp ? sh.red[0][w] : 0u;
  const uint32_t take = t.need_eq > eq_before ? min(t.need_eq - eq_before, n_eq) : 0u;
  if (lane == 0) sh.red[1][warp] = n_gt + take;
  __syncthreads();
  uint32_t pos = 0u, total = 0u;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t v = sh.red[1][w];
    pos += w < warp ? v : 0u;
    total += v;
  }
  uint32_t eq_run = 0u;
#pragma unroll
  for (int j = 0; j < R; ++j) {
    // ties of this stripe with warp-local rank < take are selected
    uint32_t tk = 0u;
    if (eqm[j]) {
      const uint32_t rank = eq_run + __popc(eqm[j] & lt);
      tk = __ballot_sync(0xffffffffu, ((eqm[j] >> lane) & 1u) && rank < take);
    }
    const uint32_t sel = gtm[j] | tk;
    if ((sel >> lane) & 1u) emit(pos + __popc(sel & lt), j);
    pos += __popc(sel);
    eq_run += __popc(eqm[j]);
  }
  __syncthreads();   // sh.red is reused by the next call
  return total;
}

__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelectArgs a) {
  pdl_wait();
  pdl_trigger();
  const int C = gridDim.x;
  const int c = blockIdx.x;
  const int r = blockIdx.y;
  const int tid = threadIdx.x;
  __shared__ Shared sh;
  extern __shared__ uint32_t dyn[];   // keys (local phase) / keys + slots (final phase)

  const Plan pl = make_plan(a, r);
  int* out = a.out + static_cast<long long>(r) * a.out_len;
  if (!pl.valid) {
    if (c == 0)
      for (int i = tid; i < a.out_len; i += kThreads) out[i] = -1;
    return;   // every CTA of the row takes this branch; the arrival counter is untouched
  }

  // ---------------------------------------------------------- local phase --
  const int len = pl.dyn_hi - pl.dyn_lo;
  const int seg = (len + C - 1) / C;
  int my_lo = pl.dyn_lo + c * seg;
  if (my_lo > pl.dyn_hi) my_lo = pl.dyn_hi;
  const int my_n = min(pl.dyn_hi, my_lo + seg) - my_lo;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride + my_lo;
  const long long cbase = (static_cast<long long>(r) * C + c) * a.cand_cap;
  uint32_t* ck = a.cand_keys + cbase;
  int* cs = a.cand_slots + cbase;
  uint32_t n_loc = 0u;
  if (my_n <= kThreads * kRL) {
    uint32_t k[kRL];
    const int i0 = (tid >> 5) * 32 * kRL + (tid & 31);   // element of k[j]: i0 + 32 * j
    float v[kRL];
#pragma unroll
    for (int j = 0; j < kRL; ++j) v[j] = i0 + 32 * j < my_n ? __ldg(row + i0 + 32 * j) : -INFINITY;
#pragma unroll
    for (int j = 0; j < kRL; ++j) k[j] = score_key(v[j]);
    const Thr tl = reg_threshold<kRL>(k, static_cast<uint32_t>(pl.D), sh);
    n_loc = reg_emit<kRL>(k, tl, sh, [&](uint32_t p, int j) {
      ck[p] = k[j];
      cs[p] = my_lo + i0 + 32 * j;
    });
  } else {
    uint32_t* keys = dyn;
    for (int i0 = 0; i0 < my_n; i0 += kThreads * 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kThreads + tid;
        v[u] = i < my_n ? __ldg(row + i) : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kThreads + tid;
        if (i < my_n) keys[i] = score_key(v[u]);
      }
    }
    __syncthreads();
    const Thr tl = cta_threshold(keys, my_n, static_cast<uint32_t>(pl.D), sh);
    n_loc = cta_emit(keys, my_n, tl, sh, [&](uint32_t p, int i) {
      ck[p] = keys[i];
      cs[p] = my_lo + i;
    });
  }
  for (int i = static_cast<int>(n_loc) + tid; i < a.cand_cap; i += kThreads) ck[i] = 0u;   // unused: no candidate

  // ------------------------------------------------- last CTA of the row --
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(a.row_arrivals + r, 1u) == static_cast<unsigned>(C - 1);
  __syncthreads();
  if (!sh.last) return;
  __threadfence();

  const int n_all = C * a.cand_cap;
  const uint32_t* gk = a.cand_keys + static_cast<long long>(r) * n_all;
  const int* gs = a.cand_slots + static_cast<long long>(r) * n_all;
  int* dyn_out = out + pl.dyn_off;
  const int M = a.M, P = a.P;
  const long long prow = static_cast<long long>(r) * M;
  auto token = [&](int slot) {
    return a.mode == kSelectHierTokens ? __ldg(a.pages + prow + slot / P) * P + slot % P : slot;
  };
  uint32_t n_sel = 0u;
  if (n_all <= kThreads * kRF) {
    uint32_t k[kRF];
    int sl[kRF];
    const int i0 = (tid >> 5) * 32 * kRF + (tid & 31);   // element of k[j]: i0 + 32 * j
#pragma unroll
    for (int j = 0; j < kRF; ++j) {
      const bool ok = i0 + 32 * j < n_all;
      k[j] = ok ? __ldcg(gk + i0 + 32 * j) : 0u;
      sl[j] = ok ? __ldcg(gs + i0 + 32 * j) : 0;
    }
    const Thr tf = reg_threshold<kRF>(k, static_cast<uint32_t>(pl.D), sh);
    n_sel = reg_emit<kRF>(k, tf, sh, [&](uint32_t p, int j) { dyn_out[p] = token(sl[j]); });
  } else {
    const Thr tf = cta_threshold(gk, n_all, static_cast<uint32_t>(pl.D), sh);
    n_sel = cta_emit(gk, n_all, tf, sh, [&](uint32_t p, int i) { dyn_out[p] = token(__ldcg(gs + i)); });
  }
  for (int i = tid; i < pl.lead_a_n; i += kThreads) out[i] = pl.lead_a_lo + i;
  for (int i = tid; i < pl.lead_b_n; i += kThreads) out[pl.lead_a_n + i] = pl.lead_b_lo + i;
  const int tr0 = pl.dyn_off + static_cast<int>(n_sel);
  for (int i = tid; i < pl.trail_n; i += kThreads) out[tr0 + i] = pl.trail_lo + i;
  for (int i = tr0 + pl.trail_n + tid; i < a.out_len; i += kThreads) out[i] = -1;
  if (tid == 0) a.row_arrivals[r] = 0u;   // ready for the next call on this workspace
}


// ---------------------------------------------------------------------------
// Grid-cooperative variant (all CTAs of the launch co-resident, one CTA per SM).
// The CTAs of a row hold their segment's keys in registers and cooperate
// through a per-row block in the workspace: a CTA arrives on a counter, the
// last to arrive does the row-wide step and releases the others through a flag
// (bounded spin). Steps:
//   S0  row max key (atomicMax).
//   A   histogram of d = (max - key) >> 13 over 2048 bins, i.e. the two
//       binades of key space below the max; scores of one row sit close
//       together, so the D-th best is almost always inside. S1: the last CTA
//       finds the bin b1 holding the D-th best and the count above it.
//   B   each CTA lists its few keys in bin b1. S2: the last CTA resolves the
//       exact D-th key from the lists and gives every CTA its output offset and
//       its share of the ties (lowest index first).
// If fewer than D candidates fall in the window, or a list overflows, the row
// switches (uniformly) to three exact radix rounds over the full key (11/11/10
// bits) with the same arrive/release steps. Every CTA then writes its own
// selections in index order.
// ---------------------------------------------------------------------------

constexpr int kSubHist = 4;       // round-A sub-histograms (warp w uses w % 4)
constexpr int kWHStride = 2052;   // sub-histogram stride (words), bank-staggered
constexpr int kListCap = 256;     // round-B list capacity per CTA
constexpr int kRangeShift = 13;   // round-A bin width: 2^13 key units (2048 bins = 2 binades)
constexpr int kMaxGridC = 64;     // CTAs per row on the grid path

enum : unsigned { kModeRange = 0u, kModeAll = 1u, kModeNone = 2u, kModeRadix = 3u };

// Flags are 64-bit words released with their payload (bit 63 = released), so a
// waiting CTA receives the row-wide result in the same load that releases it.
constexpr unsigned long long kReleased = 1ull << 63;

struct GridRow {                      // per row, zeroed before each launch
  unsigned arrive[8];
  unsigned maxkey, overflow;
  unsigned long long flag[8];         // S0: max key; S1: mode/bin/need; radix rounds: bin/need
  unsigned long long fl[kMaxGridC];   // per CTA: threshold | offset | ties taken
  unsigned histA[2048];               // round A window histogram
};

// per-row, per-CTA arrays following the GridRow blocks (written before being read)
struct GridCta {
  unsigned* cnt;      // [C] candidates
  unsigned* inr;      // [C] candidates inside the round-A window
  unsigned* def;      // [C] keys above the bin / prefix (definitely selected)
  unsigned* ln;       // [C] round-B list lengths
  unsigned* lists;    // [C][kListCap] round-B (max - key) values
  unsigned* h3;       // [C][1024] fallback round-3 histograms
  unsigned* hist1;    // [2048] fallback round-1 histogram (zeroed when the fallback starts)
  unsigned* hist2;    // [2048] fallback round-2 histogram
};

__host__ __device__ constexpr size_t grid_blocks_bytes(int rows) {
  return (sizeof(GridRow) * static_cast<size_t>(rows) + 255) / 256 * 256;
}
__host__ __device__ constexpr size_t grid_row_bytes(int C) {
  return (static_cast<size_t>(C) * (4 * 4 + kListCap * 4 + 1024 * 4) + 2 * 2048 * 4 + 255) / 256 * 256;
}

__device__ __forceinline__ GridCta grid_cta(uint8_t* base, int C) {
  GridCta g;
  g.cnt = reinterpret_cast<unsigned*>(base);
  g.inr = g.cnt + C;
  g.def = g.inr + C;
  g.ln = g.def + C;
  g.lists = g.ln + C;
  g.h3 = g.lists + static_cast<size_t>(C) * kListCap;
  g.hist1 = g.h3 + static_cast<size_t>(C) * 1024;
  g.hist2 = g.hist1 + 2048;
  return g;
}

__device__ __forceinline__ unsigned long long ld_acquire64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

struct GShared {
  unsigned long long v64;
  unsigned u[4];
  int ok;
};

// True in every thread of the CTA that arrives last on `counter` (of `n`).
__device__ __noinline__ bool arrive_last(unsigned* counter, unsigned n, Shared& sh) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) sh.last = atomicAdd(counter, 1u) == n - 1u;
  __syncthreads();
  if (sh.last) __threadfence();
  return sh.last != 0;
}

// Wait (bounded) for a released flag; every thread gets the payload. False on timeout.
__device__ __noinline__ bool wait64(const unsigned long long* flag, unsigned long long* val, int* status,
                                    GShared& gs) {
  if (threadIdx.x == 0) {
    const unsigned long long t0 = globaltimer_ns();
    unsigned long long v;
    gs.ok = 1;
    while (!((v = ld_acquire64(flag)) & kReleased)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_timeout(status);
        gs.ok = 0;
        break;
      }
    }
    gs.v64 = v;
  }
  __syncthreads();
  *val = gs.v64;
  const bool ok = gs.ok != 0;
  __syncthreads();
  return ok;
}

// Release a payload flag (after the CTA's published writes).
__device__ __forceinline__ void release64(unsigned long long* flag, unsigned long long payload) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) st_release64(flag, kReleased | payload);
}

// Row-wide step: the last CTA runs `work` (returns the payload, uniform) and
// releases; the others wait. Every thread gets the payload.
template <class W>
__device__ __forceinline__ bool row_step(unsigned* arrive, unsigned long long* flag, unsigned C, int* status,
                                         Shared& sh, GShared& gs, unsigned long long* val, W&& work) {
  if (arrive_last(arrive, C, sh)) {
    const unsigned long long v = work();
    release64(flag, v);
    *val = kReleased | v;
    return true;
  }
  return wait64(flag, val, status, gs);
}

__device__ __forceinline__ unsigned long long pack_cta(unsigned thr, unsigned offset, unsigned take, unsigned mode) {
  return (static_cast<unsigned long long>(mode == kModeAll) << 62) |
         (static_cast<unsigned long long>(mode == kModeNone) << 61) |
         (static_cast<unsigned long long>(thr) << 28) | (static_cast<unsigned long long>(offset & 0x3FFFu) << 14) |
         (take & 0x3FFFu);
}

// Bin where the running count over bins [0, nb) reaches `need`, scanning from
// the top (descending keys) or from bin 0 (when bin 0 holds the largest keys).
template <bool FROM_TOP, bool GLOBAL>
__device__ __noinline__ void find_bin(const unsigned* h, int nb, unsigned need, Shared& sh) {
  const int tid = threadIdx.x;
  const int per = nb / kThreads;
  unsigned vals[16];
  unsigned local = 0u;
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    if (q < per) {
      const int bb = FROM_TOP ? nb - 1 - (per * tid + q) : per * tid + q;
      vals[q] = GLOBAL ? __ldcg(h + bb) : h[bb];
      local += vals[q];
    }
  }
  const unsigned incl = block_incl_scan(local, sh.tmp, nullptr);
  const unsigned excl = incl - local;
  if (excl < need && need <= incl) {
    unsigned above = excl;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      if (q < per) {
        if (above + vals[q] >= need) {
          sh.bin = FROM_TOP ? nb - 1 - (per * tid + q) : per * tid + q;
          sh.above = above;
          break;
        }
        above += vals[q];
      }
    }
  }
  __syncthreads();
}

// Per-CTA offsets and tie shares from per-CTA (definite, tie) counts held by
// threads cc < C; writes the packed per-CTA flags (released).
__device__ __noinline__ void publish_ctas(GridRow* G, unsigned C, unsigned def, unsigned eq, unsigned need_eq,
                                          unsigned thr, unsigned mode, Shared& sh) {
  const int tid = threadIdx.x;
  const unsigned my_eq = tid < static_cast<int>(C) ? eq : 0u;
  const unsigned eq_before = block_incl_scan(my_eq, sh.tmp, nullptr) - my_eq;
  const unsigned tk = need_eq > eq_before ? min(need_eq - eq_before, my_eq) : 0u;
  const unsigned n = tid < static_cast<int>(C) ? def + tk : 0u;
  const unsigned off = block_incl_scan(n, sh.tmp, nullptr) - n;
  __threadfence();
  __syncthreads();
  if (tid < static_cast<int>(C)) st_release64(&G->fl[tid], kReleased | pack_cta(thr, off, tk, mode));
}

// Ordered emission of the selected keys of this CTA (keys in shared memory,
// warp-striped: element w*32*kRL + 32*j + lane). Two rolled passes: per-warp
// counts, then positions from per-stripe ballots.
template <int R, class F>
__device__ __forceinline__ uint32_t smem_emit(const uint32_t* keys, const Thr& t, Shared& sh, F&& emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int base = warp * 32 * R + lane;
  uint32_t n_gt = 0u, n_eq = 0u;
#pragma unroll 4
  for (int j = 0; j < R; ++j) {
    const uint32_t k = keys[base + 32 * j];
    n_gt += __popc(__ballot_sync(0xffffffffu, k != 0u && (t.all || k > t.thr)));
    n_eq += __popc(__ballot_sync(0xffffffffu, k != 0u && !t.all && k == t.thr));
  }
  if (lane == 0) sh.red[0][warp] = n_eq;
  __syncthreads();
  uint32_t eq_before = 0u;
  for (int w = 0; w < warp; ++w) eq_before += sh.red[0][w];
  const uint32_t take = t.need_eq > eq_before ? min(t.need_eq - eq_before, n_eq) : 0u;
  if (lane == 0) sh.red[1][warp] = n_gt + take;
  __syncthreads();
  uint32_t pos = 0u, total = 0u;
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t v = sh.red[1][w];
    pos += w < warp ? v : 0u;
    total += v;
  }
  uint32_t eq_run = 0u;
#pragma unroll 2
  for (int j = 0; j < R; ++j) {
    const uint32_t k = keys[base + 32 * j];
    const uint32_t gtm = __ballot_sync(0xffffffffu, k != 0u && (t.all || k > t.thr));
    const bool is_eq = k != 0u && !t.all && k == t.thr;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t tk = __ballot_sync(0xffffffffu, is_eq && eq_run + __popc(eqm & lt) < take);
    const uint32_t sel = gtm | tk;
    if ((sel >> lane) & 1u) emit(pos + __popc(sel & lt), base + 32 * j);
    pos += __popc(sel);
    eq_run += __popc(eqm);
  }
  __syncthreads();   // sh.red is reused
  return total;
}

__global__ void __launch_bounds__(kThreads, 1) select_grid_kernel(const SelectArgs a) {
  pdl_wait();
  pdl_trigger();
  const unsigned C = gridDim.x;
  const int c = blockIdx.x;
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ Shared sh;
  __shared__ GShared gs;
  __shared__ unsigned s_cnt;
  extern __shared__ uint32_t dsm[];
  uint32_t* keys = dsm;                                  // [kThreads * kRL] warp-striped
  uint32_t* sub = dsm + kThreads * kRL;                  // [kSubHist][kWHStride] round-A histograms

  const Plan pl = make_plan(a, r);
  int* out = a.out + static_cast<long long>(r) * a.out_len;
  if (!pl.valid) {
    if (c == 0)
      for (int i = tid; i < a.out_len; i += kThreads) out[i] = -1;
    return;   // every CTA of the row returns; the row's block is untouched
  }
  GridRow* G = reinterpret_cast<GridRow*>(a.grid_ws) + r;
  const GridCta X = grid_cta(reinterpret_cast<uint8_t*>(a.grid_ws) + grid_blocks_bytes(a.B * a.T) +
                                 static_cast<size_t>(r) * a.grid_row_bytes, C);
  const unsigned D = static_cast<unsigned>(pl.D);

  // keys of this CTA's segment (element e at keys[e], e < kThreads * kRL)
  const int len = pl.dyn_hi - pl.dyn_lo;
  const int seg = (len + static_cast<int>(C) - 1) / static_cast<int>(C);
  int my_lo = pl.dyn_lo + c * seg;
  if (my_lo > pl.dyn_hi) my_lo = pl.dyn_hi;
  const int my_n = min(pl.dyn_hi, my_lo + seg) - my_lo;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride + my_lo;
  const int base = warp * 32 * kRL + lane;   // this thread's elements: base + 32 * j
  uint32_t nz = 0u, mx = 0u;
#pragma unroll 8
  for (int j = 0; j < kRL; ++j) {
    const int e = base + 32 * j;
    const uint32_t k = score_key(e < my_n ? __ldg(row + e) : -INFINITY);
    keys[e] = k;
    nz += k != 0u ? 1u : 0u;
    mx = max(mx, k);
  }
  {
    uint4* z = reinterpret_cast<uint4*>(sub);
    for (int i = tid; i < kSubHist * kWHStride / 4; i += kThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  unsigned long long fv = 0ull;

  // ---- S0: row max key and candidate counts ----
  block_cnt_min_max(nz, 0xFFFFFFFFu, mx, sh);
  if (tid == 0) {
    X.cnt[c] = sh.cnt;
    if (sh.cnt) atomicMax(&G->maxkey, sh.mx);
  }
  if (!row_step(&G->arrive[0], &G->flag[0], C, a.status, sh, gs, &fv, [&] {
        return static_cast<unsigned long long>(__ldcg(&G->maxkey));
      }))
    return;
  const uint32_t kmax = static_cast<uint32_t>(fv);

  // ---- round A: window histogram ----
  {
    uint32_t* h = sub + (warp % kSubHist) * kWHStride;
    uint32_t nin = 0u;
#pragma unroll 4
    for (int j = 0; j < kRL; ++j) {
      const uint32_t k = keys[base + 32 * j];
      const uint32_t d = (kmax - k) >> kRangeShift;
      if (k != 0u && d < 2048u) {
        ++nin;
        atomicAdd(&h[d], 1u);
      }
    }
    uint32_t my_in = 0u;
    block_incl_scan(nin, sh.tmp, &my_in);   // barrier: sub-histograms complete
    for (int bin = tid; bin < 2048; bin += kThreads) {
      const unsigned sum = sub[bin] + sub[kWHStride + bin] + sub[2 * kWHStride + bin] + sub[3 * kWHStride + bin];
      if (sum) atomicAdd(&G->histA[bin], sum);
    }
    if (tid == 0) X.inr[c] = my_in;
  }
  if (!row_step(&G->arrive[1], &G->flag[1], C, a.status, sh, gs, &fv, [&]() -> unsigned long long {
        const unsigned cn = tid < static_cast<int>(C) ? __ldcg(X.cnt + tid) : 0u;
        const unsigned ci = tid < static_cast<int>(C) ? __ldcg(X.inr + tid) : 0u;
        unsigned total = 0u, total_in = 0u;
        block_incl_scan(cn, sh.tmp, &total);
        block_incl_scan(ci, sh.tmp, &total_in);
        if (total <= D || D == 0u) {
          const unsigned mode = D == 0u ? kModeNone : kModeAll;
          publish_ctas(G, C, D == 0u ? 0u : cn, 0u, 0u, 0u, mode, sh);
          return static_cast<unsigned long long>(mode) << 48;
        }
        if (total_in < D) {
          for (int i = tid; i < 4096; i += kThreads) X.hist1[i] = 0u;   // hist1 and hist2
          return static_cast<unsigned long long>(kModeRadix) << 48;
        }
        find_bin<false, true>(G->histA, 2048, D, sh);
        return (static_cast<unsigned long long>(kModeRange) << 48) |
               (static_cast<unsigned long long>(sh.bin) << 16) | (D - sh.above);
      }))
    return;
  unsigned mode = static_cast<unsigned>(fv >> 48) & 3u;

  if (mode == kModeRange) {
    // ---- round B: list this CTA's keys in bin b1 ----
    const unsigned b1 = static_cast<unsigned>(fv >> 16) & 0xFFFFu, need1 = static_cast<unsigned>(fv & 0xFFFFu);
    if (tid == 0) s_cnt = 0u;
    __syncthreads();
    unsigned* lst = X.lists + static_cast<size_t>(c) * kListCap;
    uint32_t nd = 0u;
#pragma unroll 4
    for (int j = 0; j < kRL; ++j) {
      const uint32_t k = keys[base + 32 * j];
      const uint32_t rel = kmax - k;
      const uint32_t d = rel >> kRangeShift;
      if (k != 0u && d < b1) {
        ++nd;
      } else if (k != 0u && d == b1) {
        const unsigned p = atomicAdd(&s_cnt, 1u);
        if (p < kListCap) lst[p] = rel;
      }
    }
    uint32_t my_def = 0u;
    block_incl_scan(nd, sh.tmp, &my_def);
    if (tid == 0) {
      X.def[c] = my_def;
      X.ln[c] = s_cnt;
      if (s_cnt > kListCap) atomicOr(&G->overflow, 1u);
    }
    if (arrive_last(&G->arrive[2], C, sh)) {
      if (__ldcg(&G->overflow)) {
        for (int i = tid; i < 4096; i += kThreads) X.hist1[i] = 0u;
        release64(&G->flag[2], static_cast<unsigned long long>(kModeRadix) << 48);
      } else {
        // exact D-th key: histogram of the listed keys' low 13 bits of (max - key)
        for (int i = tid; i < (1 << kRangeShift); i += kThreads) sh.hist[i] = 0u;
        __syncthreads();
        for (unsigned cc = warp; cc < C; cc += kWarps) {
          const unsigned n = __ldcg(X.ln + cc);
          for (unsigned i = lane; i < n; i += 32)
            atomicAdd(&sh.hist[__ldcg(X.lists + cc * kListCap + i) & ((1u << kRangeShift) - 1u)], 1u);
        }
        __syncthreads();
        find_bin<false, false>(sh.hist, 1 << kRangeShift, need1, sh);
        const unsigned thr_rel = (b1 << kRangeShift) | static_cast<unsigned>(sh.bin);
        const unsigned need_eq = need1 - sh.above;
        // per CTA: keys strictly above the threshold and ties equal to it
        for (unsigned cc = warp; cc < C; cc += kWarps) {
          const unsigned n = __ldcg(X.ln + cc);
          unsigned lo = 0u, eq = 0u;
          for (unsigned i = lane; i < n; i += 32) {
            const unsigned rel = __ldcg(X.lists + cc * kListCap + i);
            lo += rel < thr_rel ? 1u : 0u;
            eq += rel == thr_rel ? 1u : 0u;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            lo += __shfl_xor_sync(0xffffffffu, lo, o);
            eq += __shfl_xor_sync(0xffffffffu, eq, o);
          }
          if (lane == 0) {
            sh.hist[8192 - 1 - 2 * cc] = lo;
            sh.hist[8192 - 2 - 2 * cc] = eq;
          }
        }
        __syncthreads();
        const unsigned def = tid < static_cast<int>(C) ? __ldcg(X.def + tid) + sh.hist[8192 - 1 - 2 * tid] : 0u;
        const unsigned eq = tid < static_cast<int>(C) ? sh.hist[8192 - 2 - 2 * tid] : 0u;
        publish_ctas(G, C, def, eq, need_eq, kmax - thr_rel, kModeRange, sh);
        release64(&G->flag[2], static_cast<unsigned long long>(kModeRange) << 48);
      }
    }
    if (!wait64(&G->flag[2], &fv, a.status, gs)) return;
    mode = static_cast<unsigned>(fv >> 48) & 3u;
  }

  if (mode == kModeRadix) {
    // ---- fallback: three exact radix rounds over the full key ----
    for (int i = tid; i < 2048; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    for (int j = 0; j < kRL; ++j) {
      const uint32_t k = keys[base + 32 * j];
      if (k != 0u) atomicAdd(&sh.hist[k >> 21], 1u);
    }
    __syncthreads();
    for (int bin = tid; bin < 2048; bin += kThreads)
      if (sh.hist[bin]) atomicAdd(&X.hist1[bin], sh.hist[bin]);
    if (!row_step(&G->arrive[3], &G->flag[3], C, a.status, sh, gs, &fv, [&] {
          find_bin<true, true>(X.hist1, 2048, D, sh);
          return (static_cast<unsigned long long>(sh.bin) << 16) | (D - sh.above);
        }))
      return;
    const unsigned b1 = static_cast<unsigned>(fv >> 16) & 0xFFFFu, need1 = static_cast<unsigned>(fv & 0xFFFFu);
    for (int i = tid; i < 2048; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    for (int j = 0; j < kRL; ++j) {
      const uint32_t k = keys[base + 32 * j];
      if (k != 0u && (k >> 21) == b1) atomicAdd(&sh.hist[(k >> 10) & 2047u], 1u);
    }
    __syncthreads();
    for (int bin = tid; bin < 2048; bin += kThreads)
      if (sh.hist[bin]) atomicAdd(&X.hist2[bin], sh.hist[bin]);
    if (!row_step(&G->arrive[4], &G->flag[4], C, a.status, sh, gs, &fv, [&] {
          find_bin<true, true>(X.hist2, 2048, need1, sh);
          return (static_cast<unsigned long long>(sh.bin) << 16) | (need1 - sh.above);
        }))
      return;
    const unsigned p22 = (b1 << 11) | (static_cast<unsigned>(fv >> 16) & 0xFFFFu);
    const unsigned need2 = static_cast<unsigned>(fv & 0xFFFFu);
    unsigned* h3 = X.h3 + static_cast<size_t>(c) * 1024;
    for (int i = tid; i < 1024; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    uint32_t ngt = 0u;
    for (int j = 0; j < kRL; ++j) {
      const uint32_t k = keys[base + 32 * j];
      if (k == 0u) continue;
      const uint32_t hi22 = k >> 10;
      if (hi22 > p22) ++ngt;
      else if (hi22 == p22) atomicAdd(&sh.hist[k & 1023u], 1u);
    }
    uint32_t my_gt = 0u;
    block_incl_scan(ngt, sh.tmp, &my_gt);
    for (int i = tid; i < 1024; i += kThreads) h3[i] = sh.hist[i];
    if (tid == 0) X.def[c] = my_gt;
    if (arrive_last(&G->arrive[5], C, sh)) {
      for (int i = tid; i < 1024; i += kThreads) {
        unsigned sum = 0u;
        for (unsigned cc = 0; cc < C; ++cc) sum += __ldcg(X.h3 + cc * 1024 + i);
        sh.hist[i] = sum;
      }
      __syncthreads();
      find_bin<true, false>(sh.hist, 1024, need2, sh);
      const unsigned b3 = static_cast<unsigned>(sh.bin);
      const unsigned need_eq = need2 - sh.above;
      for (unsigned cc = warp; cc < C; cc += kWarps) {
        unsigned above = 0u;
        for (int i = lane; i < 1024; i += 32)
          if (static_cast<unsigned>(i) > b3) above += __ldcg(X.h3 + cc * 1024 + i);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
        if (lane == 0) {
          sh.hist[2048 + 2 * cc] = above + __ldcg(X.def + cc);
          sh.hist[2048 + 2 * cc + 1] = __ldcg(X.h3 + cc * 1024 + b3);
        }
      }
      __syncthreads();
      const unsigned def = tid < static_cast<int>(C) ? sh.hist[2048 + 2 * tid] : 0u;
      const unsigned eq = tid < static_cast<int>(C) ? sh.hist[2048 + 2 * tid + 1] : 0u;
      publish_ctas(G, C, def, eq, need_eq, (p22 << 10) | b3, kModeRange, sh);
    }
  }

  // ---- emit this CTA's selections in index order ----
  if (!wait64(&G->fl[c], &fv, a.status, gs)) return;
  Thr t{0u, 0u, false};
  if ((fv >> 62) & 1ull) {
    t.all = true;
  } else if ((fv >> 61) & 1ull) {
    t.thr = 0xFFFFFFFFu;   // nothing is taken
  } else {
    t.thr = static_cast<unsigned>(fv >> 28);
  }
  t.need_eq = static_cast<unsigned>(fv & 0x3FFFu);
  const int off = static_cast<int>((fv >> 14) & 0x3FFFu);
  int* dyn_out = out + pl.dyn_off + off;
  const long long prow = static_cast<long long>(r) * a.M;
  const bool hier = a.mode == kSelectHierTokens;
  const uint32_t n_mine = smem_emit<kRL>(keys, t, sh, [&](uint32_t p, int e) {
    const int slot = my_lo + e;
    dyn_out[p] = hier ? __ldg(a.pages + prow + slot / a.P) * a.P + slot % a.P : slot;
  });
  if (c == static_cast<int>(C) - 1) {
    // the last segment ends the dynamic block: its end is the selected count
    const int n_sel = off + static_cast<int>(n_mine);
    for (int i = tid; i < pl.lead_a_n; i += kThreads) out[i] = pl.lead_a_lo + i;
    for (int i = tid; i < pl.lead_b_n; i += kThreads) out[pl.lead_a_n + i] = pl.lead_b_lo + i;
    const int tr0 = pl.dyn_off + n_sel;
    for (int i = tid; i < pl.trail_n; i += kThreads) out[tr0 + i] = pl.trail_lo + i;
    for (int i = tr0 + pl.trail_n + tid; i < a.out_len; i += kThreads) out[i] = -1;
  }
}


// ------------------------------------------------------------ cluster path --
// One thread-block cluster of C <= 8 CTAs per row, each holding up to 16384
// consecutive dynamic slots' keys in shared memory. The CTAs agree on the
// exact D-th key through distributed shared memory and hardware cluster
// barriers: (1) every CTA broadcasts its max key and candidate count into
// every CTA's slots; (2) each builds a 2048-bin histogram of
// (max - key) >> 13 and every CTA sums the cluster's histograms to find the
// boundary bin; (3) each lists its keys in that bin and every CTA resolves the
// exact key (and the tie count) from all lists, then the per-CTA output
// offsets; (4) each CTA writes its selections in index order. If the window
// of the histogram holds fewer than D keys, or a boundary list overflows, all
// CTAs take three exact radix rounds over the full key instead (the decision
// is made from the same cluster-wide data in every CTA, so the barriers stay
// uniform). No global workspace and no spin waits: only barriers.
constexpr int kClusterMax = 8;    // CTAs per row cluster (the portable maximum)
constexpr int kListCapC = 512;                  // boundary-bin keys per CTA
enum { kXMax = 0, kXCnt = 1, kXIn = 2, kXDef = 3, kXLen = 4, kXGt = 5, kXEq = 6, kXSlots = 7 };

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Thread t < C writes v into slot [kind][c] of cluster CTA t.
__device__ __forceinline__ void cluster_broadcast(uint32_t* xs, int kind, int c, int C, uint32_t v) {
  if (static_cast<int>(threadIdx.x) < C)
    st_cluster_u32(mapa_shared(smem_u32(xs + kind * kClusterMax + c), threadIdx.x), v);
}

// Sum over the cluster of h[0, nb) (each CTA's copy; nb <= 4 * kThreads) into
// the local dst: one 16-byte load per CTA per thread, all in flight together.
__device__ __forceinline__ void cluster_sum(const uint32_t* h, int nb, int C, uint32_t* dst) {
  const int i = threadIdx.x * 4;
  if (i >= nb) return;
  const uint32_t a0 = smem_u32(h) + 4u * i;
  uint4 v[kClusterMax];
#pragma unroll
  for (int cc = 0; cc < kClusterMax; ++cc)
    v[cc] = cc < C ? ld_cluster_v4(mapa_shared(a0, cc)) : make_uint4(0u, 0u, 0u, 0u);
  uint4 sum = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int cc = 0; cc < kClusterMax; ++cc) {
    sum.x += v[cc].x;
    sum.y += v[cc].y;
    sum.z += v[cc].z;
    sum.w += v[cc].w;
  }
  *reinterpret_cast<uint4*>(dst + i) = sum;
}

// Per-CTA output offsets and tie shares from per-CTA (greater, equal) counts:
// CTA cc takes gt[cc] + take[cc] where ties go to the lower CTAs first.
__device__ __forceinline__ void cluster_offsets(const uint32_t* gt, const uint32_t* eq, int C, uint32_t need_eq,
                                                int c, uint32_t* off, uint32_t* take, uint32_t* total) {
  uint32_t run = 0u, eq_before = 0u;
  for (int cc = 0; cc < C; ++cc) {
    const uint32_t tk = need_eq > eq_before ? min(need_eq - eq_before, eq[cc]) : 0u;
    if (cc == c) {
      *off = run;
      *take = tk;
    }
    run += gt[cc] + tk;
    eq_before += eq[cc];
  }
  *total = run;
}

// Inclusive scan of one value per thread, inlined (cluster path).
__device__ __noinline__ uint32_t scan_incl(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kWarps ? tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) tmp[lane] = w;
  }
  __syncthreads();
  const uint32_t res = x + (warp > 0 ? tmp[warp - 1] : 0u);
  if (total) *total = tmp[kWarps - 1];
  __syncthreads();
  return res;
}

// Bin of a local histogram h[0, PER * kThreads) where the running count from
// bin 0 (FROM_TOP = false) or from the last bin reaches `need`: *bin and the
// count strictly before it (*above). Uniform result in every thread.
template <int PER, bool FROM_TOP>
__device__ __noinline__ void find_bin_c(const uint32_t* h, uint32_t need, Shared& sh, uint32_t* bin,
                                           uint32_t* above) {
  constexpr int nb = PER * kThreads;
  const int tid = threadIdx.x;
  uint32_t vals[PER];
  uint32_t local = 0u;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int bb = FROM_TOP ? nb - 1 - (PER * tid + q) : PER * tid + q;
    vals[q] = h[bb];
    local += vals[q];
  }
  const uint32_t incl = scan_incl(local, sh.tmp, nullptr);
  const uint32_t excl = incl - local;
  if (excl < need && need <= incl) {
    uint32_t run = excl;
    bool done = false;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      if (!done && run + vals[q] >= need) {
        sh.bin = FROM_TOP ? nb - 1 - (PER * tid + q) : PER * tid + q;
        sh.above = run;
        done = true;
      }
      run += vals[q];
    }
  }
  __syncthreads();
  *bin = static_cast<uint32_t>(sh.bin);
  *above = sh.above;
  __syncthreads();
}

// Element e of a CTA's segment sits at keys[e + 4 (e / RC)]: thread t owns the
// RC consecutive elements [RC t, RC t + RC) at keys[(RC + 4) t ...]. The
// warp-coalesced fill writes 32 consecutive words; the per-thread passes read
// 16 bytes at a time, and with a stride of 4 (mod 32) words the eight threads
// of each quarter-warp phase hit distinct bank quads: no conflicts either way.
template <int RC, int UNROLL, class F>
__device__ __forceinline__ void for_keys(const uint32_t* run, F&& f) {
  const uint4* p = reinterpret_cast<const uint4*>(run);
#pragma unroll UNROLL
  for (int j4 = 0; j4 < RC / 4; ++j4) {
    const uint4 v = p[j4];
    f(v.x, 4 * j4);
    f(v.y, 4 * j4 + 1);
    f(v.z, 4 * j4 + 2);
    f(v.w, 4 * j4 + 3);
  }
}

//
// Dynamic shared memory of a CTA holding RC keys per thread: the keys,
// two histograms, the outgoing list, the broadcast slots and the round-A
// sub-histograms (whose space the copies of every CTA's list reuse later).
constexpr size_t cluster_smem_words(int RC) {
  return static_cast<size_t>(kThreads) * (RC + 4) + 2048 + 2048 + kListCapC +
         kXSlots * kClusterMax + kSubHist * kWHStride;
}
static_assert(kClusterMax * kListCapC <= kSubHist * kWHStride, "list copies fit the sub-histogram space");

// RC keys per thread: 4, 8, 16, 32 or 64 (2048 .. 32768 slots per CTA).
template <int RC>
__global__ void __launch_bounds__(kThreads, 1) select_cluster_kernel(const SelectArgs a) {
  static_assert(RC == 4 || RC == 8 || RC == 16 || RC == 32 || RC == 64, "keys per thread");
  pdl_wait();
  pdl_trigger();
  const int C = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(cluster_ctarank());
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ Shared sh;
  __shared__ unsigned s_cnt;
  extern __shared__ __align__(16) uint32_t cluster_dsm[];   // 16-byte loads and DSMEM copies
  uint32_t* dsm = cluster_dsm;
  uint32_t* keys = dsm;                              // [kThreads][RC + 4]: each thread's run, then 4 pad words
  uint32_t* histA = keys + kThreads * (RC + 4);      // [2048]  read by the cluster
  uint32_t* fbh = histA + 2048;                      // [2048]  fallback rounds, read by the cluster
  uint32_t* list = fbh + 2048;                       // [kListCapC] read by the cluster
  uint32_t* xs = list + kListCapC;                   // [kXSlots][kClusterMax] broadcast slots
  uint32_t* sub = xs + kXSlots * kClusterMax;        // [kSubHist][kWHStride] local, round A only
  uint32_t* lists = sub;                             // [kClusterMax][kListCapC] local copies of every list (after round A)

  const Plan pl = make_plan(a, r);                   // identical in every CTA of the cluster
  int* out = a.out + static_cast<long long>(r) * a.out_len;
  if (!pl.valid) {
    if (c == 0)
      for (int i = tid; i < a.out_len; i += kThreads) out[i] = -1;
    return;   // the whole cluster returns before touching shared memory of another CTA
  }
  cluster_arrive_release();   // this CTA has started: its shared memory may be written by the others
  const uint32_t D = static_cast<uint32_t>(pl.D);
  const int len = pl.dyn_hi - pl.dyn_lo;
  const int seg = (len + C - 1) / C;
  int my_lo = pl.dyn_lo + c * seg;
  if (my_lo > pl.dyn_hi) my_lo = pl.dyn_hi;
  const int my_n = min(pl.dyn_hi, my_lo + seg) - my_lo;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride + my_lo;

  // ---- (1) keys (coalesced fill), local max and count; broadcast
  uint32_t nz = 0u, mx = 0u;
  constexpr int kBatch = RC < 32 ? RC : 32;   // loads in flight per thread at a time
#pragma unroll 1
  for (int h = 0; h < RC / kBatch; ++h) {
    const int e0 = warp * 32 * RC + lane + 32 * kBatch * h;
    float f[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) f[j] = e0 + 32 * j < my_n ? __ldg(row + e0 + 32 * j) : -INFINITY;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const uint32_t k = score_key(f[j]);
      const int e = e0 + 32 * j;
      keys[e + 4 * (e / RC)] = k;
      nz += k != 0u ? 1u : 0u;
      mx = max(mx, k);
    }
  }
  {
    uint4* z = reinterpret_cast<uint4*>(sub);
    for (int i = tid; i < kSubHist * kWHStride / 4; i += kThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  block_cnt_min_max(nz, 0xFFFFFFFFu, mx, sh);        // also orders the fill before the per-thread passes
  cluster_wait_acquire();     // every CTA of the cluster has started
  cluster_broadcast(xs, kXMax, c, C, sh.mx);
  cluster_broadcast(xs, kXCnt, c, C, sh.cnt);
  cluster_sync_all();

  const uint32_t* kvb = keys + (RC + 4) * tid;   // this thread's RC consecutive elements (16-byte aligned)

  uint32_t kmax = 0u, total = 0u;
  for (int cc = 0; cc < C; ++cc) {
    kmax = max(kmax, xs[kXMax * kClusterMax + cc]);
    total += xs[kXCnt * kClusterMax + cc];
  }
  Thr t{0u, 0u, false};
  uint32_t my_off = 0u;
  if (total <= D || D == 0u) {
    // every candidate is taken (or none): offsets are candidate-count prefixes
    t.all = D != 0u;
    if (!t.all) t.thr = 0xFFFFFFFFu;
    for (int cc = 0; cc < c && t.all; ++cc) my_off += xs[kXCnt * kClusterMax + cc];
  } else {
    bool radix = false;
    // ---- (2) window histogram of (max - key) >> 13: bin 0 holds the largest keys
    {
      uint32_t* h = sub + (warp % kSubHist) * kWHStride;
      uint32_t nin = 0u;
      for_keys<RC, 2>(kvb, [&](uint32_t k, int) {
        const uint32_t d = (kmax - k) >> kRangeShift;
        if (k != 0u && d < 2048u) {
          ++nin;
          atomicAdd(&h[d], 1u);
        }
      });
      uint32_t my_in = 0u;
      scan_incl(nin, sh.tmp, &my_in);                // barrier: sub-histograms complete
      for (int bin = tid; bin < 2048; bin += kThreads)
        histA[bin] = sub[bin] + sub[kWHStride + bin] + sub[2 * kWHStride + bin] + sub[3 * kWHStride + bin];
      cluster_broadcast(xs, kXIn, c, C, my_in);
    }
    cluster_sync_all();
    uint32_t total_in = 0u;
    for (int cc = 0; cc < C; ++cc) total_in += xs[kXIn * kClusterMax + cc];
    radix = total_in < D;
    uint32_t b1 = 0u, need1 = 0u;
    if (!radix) {
      cluster_sum(histA, 2048, C, sh.hist);
      __syncthreads();
      uint32_t above = 0u;
      find_bin_c<2048 / kThreads, false>(sh.hist, D, sh, &b1, &above);
      need1 = D - above;
      // ---- (3) list this CTA's keys in the boundary bin (as max - key)
      if (tid == 0) s_cnt = 0u;
      __syncthreads();
      uint32_t nd = 0u;
      const uint32_t lt = (1u << lane) - 1u;
      for_keys<RC, 2>(kvb, [&](uint32_t k, int) {   // warp-uniform: every thread holds RC keys
        const uint32_t rel = kmax - k;
        const uint32_t d = rel >> kRangeShift;
        nd += (k != 0u && d < b1) ? 1u : 0u;
        // boundary-bin keys: one shared-counter reservation per warp (the list is
        // unordered), so a crowded bin does not serialise on the counter
        const bool inb = k != 0u && d == b1;
        const uint32_t m = __ballot_sync(0xffffffffu, inb);
        if (m != 0u) {
          const int leader = __ffs(m) - 1;
          unsigned base = 0u;
          if (lane == leader) base = atomicAdd(&s_cnt, static_cast<unsigned>(__popc(m)));
          base = __shfl_sync(0xffffffffu, base, leader);
          const unsigned p = base + static_cast<unsigned>(__popc(m & lt));
          if (inb && p < kListCapC) list[p] = rel;
        }
      });
      uint32_t my_def = 0u;
      scan_incl(nd, sh.tmp, &my_def);
      cluster_broadcast(xs, kXDef, c, C, my_def);
      cluster_broadcast(xs, kXLen, c, C, s_cnt);
    }
    cluster_sync_all();
    if (!radix)
      for (int cc = 0; cc < C; ++cc) radix = radix || xs[kXLen * kClusterMax + cc] > static_cast<uint32_t>(kListCapC);
    if (!radix) {
      // copy every CTA's list here (16-byte loads, all in flight), then the
      // exact key: histogram of the low 13 bits of (max - key)
      {
        constexpr int kV = kListCapC / 4;                    // uint4 per list
        const uint32_t l0 = smem_u32(list);
        uint4 v[kClusterMax * kV / kThreads];
#pragma unroll
        for (int q = 0; q < kClusterMax * kV / kThreads; ++q) {
          const int g = tid + q * kThreads, cc = g / kV, u = g % kV;
          v[q] = (cc < C && 4u * u < xs[kXLen * kClusterMax + cc]) ? ld_cluster_v4(mapa_shared(l0 + 16u * u, cc))
                                                                  : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < kClusterMax * kV / kThreads; ++q)
          reinterpret_cast<uint4*>(lists)[tid + q * kThreads] = v[q];
      }
      {
        uint4* z = reinterpret_cast<uint4*>(sh.hist);
        for (int i = tid; i < (1 << kRangeShift) / 4; i += kThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncthreads();
      for (int cc = 0; cc < C; ++cc) {
        const uint32_t n = xs[kXLen * kClusterMax + cc];
        for (uint32_t i = tid; i < n; i += kThreads)
          atomicAdd(&sh.hist[lists[cc * kListCapC + i] & ((1u << kRangeShift) - 1u)], 1u);
      }
      __syncthreads();
      uint32_t b2 = 0u, above2 = 0u;
      find_bin_c<(1 << kRangeShift) / kThreads, false>(sh.hist, need1, sh, &b2, &above2);
      const uint32_t thr_rel = (b1 << kRangeShift) | b2;
      const uint32_t need_eq = need1 - above2;
      // per CTA: keys strictly above the exact key, and ties equal to it
      if (warp < C) {
        const uint32_t n = xs[kXLen * kClusterMax + warp];
        uint32_t lo = 0u, eq = 0u;
        for (uint32_t i = lane; i < n; i += 32) {
          const uint32_t rel = lists[warp * kListCapC + i];
          lo += rel < thr_rel ? 1u : 0u;
          eq += rel == thr_rel ? 1u : 0u;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          lo += __shfl_xor_sync(0xffffffffu, lo, o);
          eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        if (lane == 0) {
          sh.red[0][warp] = xs[kXDef * kClusterMax + warp] + lo;
          sh.red[1][warp] = eq;
        }
      }
      __syncthreads();
      uint32_t tot = 0u;
      cluster_offsets(sh.red[0], sh.red[1], C, need_eq, c, &my_off, &t.need_eq, &tot);
      t.thr = kmax - thr_rel;
    } else {
      // ---- fallback: three exact radix rounds over the full key
      uint32_t prefix = 0u, mask = 0u, need = D;
      for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        const uint32_t dmask = static_cast<uint32_t>(nb - 1);
        if (pass > 0) cluster_sync_all();           // the previous round's histogram has been read
        for (int i = tid; i < nb; i += kThreads) fbh[i] = 0u;
        __syncthreads();
        for_keys<RC, 1>(kvb, [&](uint32_t k, int) {
          if (k != 0u && (k & mask) == prefix) atomicAdd(&fbh[(k >> shift) & dmask], 1u);
        });
        cluster_sync_all();
        cluster_sum(fbh, nb, C, sh.hist);
        __syncthreads();
        uint32_t bin = 0u, above = 0u;
        if (nb == 2048)
          find_bin_c<2048 / kThreads, true>(sh.hist, need, sh, &bin, &above);
        else
          find_bin_c<1024 / kThreads, true>(sh.hist, need, sh, &bin, &above);
        prefix |= bin << shift;
        mask |= dmask << shift;
        need -= above;
      }
      uint32_t gt = 0u, eq = 0u;
      for_keys<RC, 1>(kvb, [&](uint32_t k, int) {
        gt += (k != 0u && k > prefix) ? 1u : 0u;
        eq += (k != 0u && k == prefix) ? 1u : 0u;
      });
      uint32_t my_gt = 0u, my_eq = 0u;
      scan_incl(gt, sh.tmp, &my_gt);
      scan_incl(eq, sh.tmp, &my_eq);
      cluster_broadcast(xs, kXGt, c, C, my_gt);
      cluster_broadcast(xs, kXEq, c, C, my_eq);
      cluster_sync_all();
      uint32_t tot = 0u;
      cluster_offsets(xs + kXGt * kClusterMax, xs + kXEq * kClusterMax, C, need, c, &my_off, &t.need_eq, &tot);
      t.thr = prefix;
    }
  }

  // ---- (4) this CTA's selections in index order: per-thread counts, two scans
  uint32_t n_gt = 0u, n_eq = 0u;
  for_keys<RC, 2>(kvb, [&](uint32_t k, int) {
    const bool cand = k != 0u;
    n_gt += (cand && (t.all || k > t.thr)) ? 1u : 0u;
    n_eq += (cand && !t.all && k == t.thr) ? 1u : 0u;
  });
  uint32_t eq_tot = 0u;
  const uint32_t eq_before = scan_incl(n_eq, sh.tmp, &eq_tot) - n_eq;      // ties in lower elements of this CTA
  const uint32_t take = t.need_eq > eq_before ? min(t.need_eq - eq_before, n_eq) : 0u;
  uint32_t n_mine = 0u;
  uint32_t pos = scan_incl(n_gt + take, sh.tmp, &n_mine) - (n_gt + take);
  int* dyn_out = out + pl.dyn_off + my_off;
  const long long prow = static_cast<long long>(r) * a.M;
  const bool hier = a.mode == kSelectHierTokens;
  if (n_gt + take > 0u) {
    uint32_t taken = 0u;
    for_keys<RC, 1>(kvb, [&](uint32_t k, int j) {
      bool s = false;
      if (k != 0u) {
        if (t.all || k > t.thr) {
          s = true;
        } else if (k == t.thr && taken < take) {
          s = true;
          ++taken;
        }
      }
      if (s) {
        const int slot = my_lo + RC * tid + j;
        dyn_out[pos++] = hier ? __ldg(a.pages + prow + slot / a.P) * a.P + slot % a.P : slot;
      }
    });
  }
  if (c == C - 1) {
    // the last segment ends the dynamic block: its end is the selected count
    const int n_sel = static_cast<int>(my_off + n_mine);
    for (int i = tid; i < pl.lead_a_n; i += kThreads) out[i] = pl.lead_a_lo + i;
    for (int i = tid; i < pl.lead_b_n; i += kThreads) out[pl.lead_a_n + i] = pl.lead_b_lo + i;
    const int tr0 = pl.dyn_off + n_sel;
    for (int i = tid; i < pl.trail_n; i += kThreads) out[tr0 + i] = pl.trail_lo + i;
    for (int i = tr0 + pl.trail_n + tid; i < a.out_len; i += kThreads) out[i] = -1;
  }
  cluster_sync_all();   // no CTA leaves while another may still read its lists or histograms
}

// ===========================================================================
// Filter path (few rows, each split over C CTAs; no spin waits).
//
// A lower bound on the threshold comes from group maxima. Cut a row's slots
// into groups of G and take each group's maximum key over its dynamic
// candidates; let v be the D-th largest of these maxima. At least D groups have
// a candidate >= v, so the D-th best candidate is >= v. And every candidate
// strictly above v lies in one of the fewer than D groups whose maximum
// exceeds v, so fewer than D * G candidates are above v (when at most D groups
// hold candidates v = 0 and every candidate counts, again fewer than D * G + 1).
// Each CTA finds v from the row's group maxima (the same v in every CTA),
// streams its segment of the row and keeps the candidates above v in one run
// per warp, in slot order, in a per-row pool; it also counts those equal to v.
// The last CTA of the row to finish takes the exact top D of the kept
// candidates -- or, when fewer than D are above v, all of them and the
// lowest-slot candidates equal to v -- and writes the row.
// ===========================================================================

// Range-radix thresholds: the exact D-th best nonzero key by rounds of 11-bit
// digits over key - kmin, each a 2048-bin shared histogram whose target bin is
// found by a conflict-free warp-chunked scan from the top.
constexpr int kFastBits = 11, kFastBins = 1 << kFastBits;   // 2048 bins: 128 per warp, 4 per lane

// After a round's histogram (kFastBins bins in sh.hist, counted from the top):
// the bin holding the need-th key (sh.bin) and the keys above it (sh.above).
// Warp w owns bins [kFastBins - 128 (w + 1), kFastBins - 128 w); lane l reads
// four of them as one 16-byte load (conflict-free). Not inlined: every caller
// shares one copy of the code.
__device__ __noinline__ void pick_bin_from_top(uint32_t need, Shared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint4* h4 = reinterpret_cast<const uint4*>(sh.hist);
  const int b0 = kFastBins - 128 * (warp + 1) + 4 * (31 - lane);   // lowest of the lane's four bins
  const uint4 v = h4[b0 >> 2];
  const uint32_t lsum = v.x + v.y + v.z + v.w;
  uint32_t incl = lsum;                                  // inclusive scan from the top within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.red[0][warp] = incl;
  __syncthreads();
  uint32_t before = 0u;                                  // bins above this warp's chunk
#pragma unroll
  for (int w = 0; w < kWarps; ++w) before += w < warp ? sh.red[0][w] : 0u;
  const uint32_t excl = before + incl - lsum;
  if (excl < need && need <= excl + lsum) {
    const uint32_t cnt[4] = {v.w, v.z, v.y, v.x};       // top bin first
    uint32_t above = excl;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (above + cnt[q] >= need) {
        sh.bin = b0 + 3 - q;
        sh.above = above;
        break;
      }
      above += cnt[q];
    }
  }
  __syncthreads();
}

// The rounds of a range-radix threshold: digits of
// rel = key - kmin from the top, kFastBits at a time. `count(prev, hi, shift,
// dmask)` adds this round's in-play keys (rel >> prev == hi) to sh.hist.
template <class Count>
__device__ Thr range_rounds(uint32_t total, uint32_t kmin, uint32_t kmax, uint32_t D, Shared& sh, Count&& count) {
  const int tid = threadIdx.x;
  Thr r{0u, 0u, false};
  if (total <= D) {
    r.all = true;
    return r;
  }
  if (D == 0u) {
    r.thr = 0xFFFFFFFFu;
    return r;
  }
  if (kmin == kmax) {
    r.thr = kmax;
    r.need_eq = D;
    return r;
  }
  const int bits = 32 - __clz(kmax - kmin);               // every rel = key - kmin is < 2^bits
  int prev = bits;                                         // keys in play satisfy rel >> prev == hi
  int shift = bits > kFastBits ? bits - kFastBits : 0;
  uint32_t hi = 0u, need = D;
  uint4* h4 = reinterpret_cast<uint4*>(sh.hist);
  while (true) {
    const int width = prev - shift;                        // digit bits this round (<= 11)
    const uint32_t dmask = (1u << width) - 1u;
    if (tid < kFastBins / 4) h4[tid] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    count(prev, hi, shift, dmask);
    __syncthreads();
    pick_bin_from_top(need, sh);
    hi = (width >= 32 ? 0u : (hi << width)) | static_cast<uint32_t>(sh.bin);
    need -= sh.above;
    __syncthreads();
    if (shift == 0) break;
    prev = shift;
    shift = shift > kFastBits ? shift - kFastBits : 0;
  }
  r.thr = kmin + hi;
  r.need_eq = need;
  return r;
}

// Exact threshold of the D-th best of key(0) .. key(n - 1) (key 0 = not a
// candidate), read through an accessor (shared memory), by range-radix
// rounds. Rolled loops: code that runs once per CTA pays more for instruction
// fetch than for loop overhead.
template <class K>
__device__ Thr range_threshold_by(K&& key, int n, uint32_t D, Shared& sh) {
  uint32_t c = 0u, mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll 4
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint32_t k = key(i);
    if (k != 0u) {
      ++c;
      mn = min(mn, k);
      mx = max(mx, k);
    }
  }
  block_cnt_min_max(c, mn, mx, sh);
  const uint32_t kmin = sh.mn;
  return range_rounds(sh.cnt, kmin, sh.mx, D, sh, [&](int prev, uint32_t hi, int shift, uint32_t dmask) {
#pragma unroll 4
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const uint32_t k = key(i);
      const uint32_t rel = k - kmin;
      if (k != 0u && (prev >= 32 || (rel >> prev) == hi)) atomicAdd(&sh.hist[(rel >> shift) & dmask], 1u);
    }
  });
}

// The same over keys held in registers, R per thread (any layout).
template <int R>
__device__ Thr fast_threshold(const uint32_t (&k)[R], uint32_t D, Shared& sh) {
  uint32_t c = 0u, mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
  for (int j = 0; j < R; ++j)
    if (k[j] != 0u) {
      ++c;
      mn = min(mn, k[j]);
      mx = max(mx, k[j]);
    }
  block_cnt_min_max(c, mn, mx, sh);
  const uint32_t kmin = sh.mn;
  return range_rounds(sh.cnt, kmin, sh.mx, D, sh, [&](int prev, uint32_t hi, int shift, uint32_t dmask) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const uint32_t rel = k[j] - kmin;
      if (k[j] != 0u && (prev >= 32 || (rel >> prev) == hi)) atomicAdd(&sh.hist[(rel >> shift) & dmask], 1u);
    }
  });
}

constexpr int kStageCap = 8192;                   // kept candidates staged in shared memory by the finisher
constexpr int kWarpSlots = 1024;                  // slots per warp in phase 2 (held in registers)
constexpr int kPhase1Per = 32;                    // folded group maxima per thread in phase 1
constexpr int kPhase1Cap = kThreads * kPhase1Per; // 16384 per row

// gmax[r][g] = max key over slots [g G0, g G0 + G0) of row r that are dynamic
// candidates (0 if none); entries past the row's groups are 0.
__global__ void __launch_bounds__(256) group_max_kernel(const SelectArgs a) {
  pdl_wait();   // the scores come from the previous kernel
  pdl_trigger();
  const int r = blockIdx.y;
  const Plan pl = make_plan(a, r);
  const int G0 = 1 << a.g0_shift;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride;
  uint32_t* gm = a.gmax + static_cast<long long>(r) * a.gmax_stride;
  const int lo = pl.valid ? pl.dyn_lo : 0, hi = pl.valid ? pl.dyn_hi : 0;
  if (blockIdx.x == 0 && threadIdx.x < 2) a.counters[2 * r + threadIdx.x] = 0u;   // arrivals, pool fill
  for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < a.gmax_stride; g += gridDim.x * blockDim.x) {
    const int s0 = g << a.g0_shift;
    uint32_t m = 0u;
    if (s0 < hi && s0 + G0 > lo) {
      for (int i = 0; i < G0; ++i) {
        const int s = s0 + i;
        if (s >= lo && s < hi) m = max(m, score_key(__ldg(row + s)));
      }
    }
    gm[g] = m;
  }
}

// Slot range [lo, hi) of warp `w` of CTA `c` (C CTAs, kWarps warps each) within
// the row's dynamic region.
struct WarpRange {
  int lo, hi;
};
__device__ __forceinline__ WarpRange warp_range(const Plan& pl, int C, int c, int w) {
  const int len = pl.dyn_hi - pl.dyn_lo;
  const int seg = (len + C - 1) / C;
  const int c_lo = pl.dyn_lo + min(len, c * seg), c_hi = pl.dyn_lo + min(len, (c + 1) * seg);
  const int sub = (seg + kWarps - 1) / kWarps;
  const int lo = min(c_hi, c_lo + w * sub);
  return WarpRange{lo, min(c_hi, lo + sub)};
}

// The D-th largest of the row's n_fold group maxima (each the maximum of F
// consecutive stored maxima), R per thread; 0 when at most D are nonzero.
// Loads are predicated and all in flight at once. Rows of maxima start on
// 16-byte boundaries and hold a multiple of max(F, 4).
template <int R>
__device__ uint32_t phase1_bound(const uint32_t* gm, int F, int n_fold, uint32_t D, Shared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t k[R];
  const int e0 = warp * 32 * R + lane;   // element of k[j]: e0 + 32 j
  if (F == 1) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int e = e0 + 32 * j;
      k[j] = e < n_fold ? __ldcg(gm + e) : 0u;
    }
  } else if (F == 2) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int e = e0 + 32 * j;
      const uint2 q = e < n_fold ? __ldcg(reinterpret_cast<const uint2*>(gm) + e) : make_uint2(0u, 0u);
      k[j] = max(q.x, q.y);
    }
  } else {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int e = e0 + 32 * j;
      const uint4 q = e < n_fold ? __ldcg(reinterpret_cast<const uint4*>(gm + e * F)) : make_uint4(0u, 0u, 0u, 0u);
      k[j] = max(max(q.x, q.y), max(q.z, q.w));
    }
    if (F == 8) {
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int e = e0 + 32 * j;
        const uint4 q = e < n_fold ? __ldcg(reinterpret_cast<const uint4*>(gm + e * F + 4)) : make_uint4(0u, 0u, 0u, 0u);
        k[j] = max(k[j], max(max(q.x, q.y), max(q.z, q.w)));
      }
    }
  }
  const Thr t = fast_threshold<R>(k, D, sh);
  return t.all ? 0u : t.thr;
}

__global__ void __launch_bounds__(kThreads, 1) select_filter_kernel(const SelectArgs a) {
  pdl_wait();   // scores and group maxima come from the previous kernel(s)
  pdl_trigger();
  const int C = static_cast<int>(gridDim.x);
  const int c = blockIdx.x, r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  __shared__ Shared sh;
  extern __shared__ __align__(16) uint32_t filt_dsm[];

  const Plan pl = make_plan(a, r);
  int* out = a.out + static_cast<long long>(r) * a.out_len;
  if (!pl.valid) {
    if (c == 0)
      for (int i = tid; i < a.out_len; i += kThreads) out[i] = -1;
    return;   // every CTA of the row returns; the row's counters are untouched
  }
  const uint32_t D = static_cast<uint32_t>(pl.D);
  const int nreg = C * kWarps;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride;
  const long long pbase = static_cast<long long>(r) * a.pool_cap;
  uint4* wt_row = a.wtab + static_cast<long long>(r) * nreg;

  // ---- phase 1: the D-th largest group maximum v (0: keep every candidate)
  uint32_t v = 0u;
  if (D > 0u) {
    const uint32_t* gm = a.gmax + static_cast<long long>(r) * a.gmax_stride;
    const int n_fold = a.gmax_stride / a.fold;
    v = n_fold <= kThreads * 16 ? phase1_bound<16>(gm, a.fold, n_fold, D, sh)
                                : phase1_bound<kPhase1Per>(gm, a.fold, n_fold, D, sh);
  }

  // ---- phase 2: keep this warp's candidates above v (slot order), count those equal to v.
  // The warp's slots (at most kWarpSlots: the plan gives every row enough CTAs)
  // are loaded once, all in flight, and stay in registers for both passes.
  if (D > 0u) {
    const WarpRange wr = warp_range(pl, C, c, warp);
    uint32_t kk[kWarpSlots / 32];
#pragma unroll
    for (int j = 0; j < kWarpSlots / 32; ++j) {
      const int s = wr.lo + lane + 32 * j;
      kk[j] = s < wr.hi ? score_key(__ldcg(row + s)) : 0u;
    }
    uint32_t kept = 0u, n_eq = 0u;
#pragma unroll
    for (int j = 0; j < kWarpSlots / 32; ++j) {
      kept += __popc(__ballot_sync(0xffffffffu, kk[j] > v));
      n_eq += __popc(__ballot_sync(0xffffffffu, v != 0u && kk[j] == v));
    }
    uint32_t base = 0u;
    if (lane == 0 && kept) base = atomicAdd(a.counters + 2 * r + 1, kept);
    base = __shfl_sync(0xffffffffu, base, 0);
    if (base + kept > static_cast<uint32_t>(a.pool_cap)) {   // cannot happen (see above); never write past the pool
      if (lane == 0) record_internal(a.status);
      kept = 0u;
    }
    if (kept) {
      uint32_t run = base;
#pragma unroll
      for (int j = 0; j < kWarpSlots / 32; ++j) {
        const uint32_t m = __ballot_sync(0xffffffffu, kk[j] > v);
        if (kk[j] > v) {
          const uint32_t p = run + __popc(m & lt);
          a.pool_keys[pbase + p] = kk[j];
          a.pool_slots[pbase + p] = wr.lo + lane + 32 * j;
        }
        run += __popc(m);
      }
    }
    if (lane == 0) wt_row[c * kWarps + warp] = make_uint4(base, kept, n_eq, 0u);
  }

  // ---- phase 3: the last CTA of the row finishes it
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(a.counters + 2 * r, 1u) == static_cast<unsigned>(C - 1);
  __syncthreads();
  if (!sh.last) return;
  __threadfence();

  uint4* wt = reinterpret_cast<uint4*>(filt_dsm);                 // [nreg] this row's warp table
  uint32_t* sel = reinterpret_cast<uint32_t*>(wt + nreg);         // [nreg] selected per warp run
  uint32_t* take = sel + nreg;                                    // [nreg] ties taken per warp run
  uint32_t* off = take + nreg;                                    // [nreg] output offset per warp run
  const int M = a.M, P = a.P;
  const long long prow = static_cast<long long>(r) * M;
  auto token = [&](int slot) {
    return a.mode == kSelectHierTokens ? __ldg(a.pages + prow + slot / P) * P + slot % P : slot;
  };
  int* dyn_out = out + pl.dyn_off;
  // Exclusive prefix over the warp runs of x(i) into pre[i] (each thread a
  // contiguous chunk of runs); returns the total.
  auto run_prefix = [&](auto&& x, uint32_t* pre) -> uint32_t {
    const int per = (nreg + kThreads - 1) / kThreads;
    const int i0 = tid * per;
    uint32_t loc = 0u;
    for (int q = 0; q < per; ++q)
      if (i0 + q < nreg) loc += x(i0 + q);
    uint32_t total = 0u;
    uint32_t run = block_incl_scan(loc, sh.tmp, &total) - loc;
    for (int q = 0; q < per; ++q)
      if (i0 + q < nreg) {
        const uint32_t xv = x(i0 + q);
        pre[i0 + q] = run;
        run += xv;
      }
    __syncthreads();
    return total;
  };
  // Ties to the lowest slots (the runs are in slot order): run i takes
  // min(eq_i, need - ties before it); then output offsets of (above_i + take_i).
  auto place = [&](auto&& above, uint32_t need) -> uint32_t {
    run_prefix([&](int i) { return take[i]; }, off);   // off[i] = ties before run i
    const int per = (nreg + kThreads - 1) / kThreads;
    for (int q = 0; q < per; ++q) {
      const int i = tid * per + q;
      if (i < nreg) take[i] = need > off[i] ? min(take[i], need - off[i]) : 0u;
    }
    __syncthreads();
    return run_prefix([&](int i) { return above(i) + take[i]; }, off);
  };
  uint32_t n_sel = 0u;
  if (D > 0u) {
    uint32_t g_loc = 0u;
    for (int i = tid; i < nreg; i += kThreads) {
      const uint4 e = __ldcg(wt_row + i);
      wt[i] = e;
      g_loc += e.y;
    }
    uint32_t G = 0u;
    block_incl_scan(g_loc, sh.tmp, &G);   // also orders the table fill before its use
    const uint32_t* pk = a.pool_keys + pbase;
    const int* ps = a.pool_slots + pbase;
    // the kept candidates in slot order: run i's land at sk[at[i] ..]; each
    // thread copies whole runs, its loads independent of one another
    uint32_t* at = sel;
    run_prefix([&](int i) { return wt[i].y; }, at);
    uint32_t* sk = off + nreg;                                   // [kStageCap] keys
    int* ss = reinterpret_cast<int*>(sk + kStageCap);            // [kStageCap] slots
    const bool staged = G <= static_cast<uint32_t>(kStageCap);
    if (staged) {
      for (int i = tid; i < nreg; i += kThreads) {
        const uint4 e = wt[i];
        const uint32_t d0 = at[i];
        for (uint32_t j0 = 0; j0 < e.y; j0 += 8) {
          uint32_t kv[8];
          int sv[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const bool in = j0 + q < e.y;
            kv[q] = in ? __ldcg(pk + e.x + j0 + q) : 0u;
            sv[q] = in ? __ldcg(ps + e.x + j0 + q) : 0;
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (j0 + q < e.y) {
              sk[d0 + j0 + q] = kv[q];
              ss[d0 + j0 + q] = sv[q];
            }
        }
      }
      __syncthreads();
    }
    if (G >= D && staged) {
      // the exact D-th best is among the kept candidates, staged in slot order
      const Thr t = range_threshold_by([&](int i) { return sk[i]; }, static_cast<int>(G), D, sh);
      n_sel = cta_emit(sk, static_cast<int>(G), t, sh, [&](uint32_t p, int i) { dyn_out[p] = token(ss[i]); });
    } else if (G >= D) {
      // more kept candidates than shared memory holds (not expected for scores
      // that are not adversarial): the same from the pool in global memory
      const Thr t = cta_threshold_by([&](int i) { return __ldcg(pk + i); }, static_cast<int>(G), D, sh);
      for (int i = warp; i < nreg; i += kWarps) {
        const uint4 e = wt[i];
        uint32_t gt = 0u, eq = 0u;
        for (uint32_t j0 = 0; j0 < e.y; j0 += 32) {
          const uint32_t kk = j0 + lane < e.y ? __ldcg(pk + e.x + j0 + lane) : 0u;
          gt += __popc(__ballot_sync(0xffffffffu, kk != 0u && (t.all || kk > t.thr)));
          eq += __popc(__ballot_sync(0xffffffffu, kk != 0u && !t.all && kk == t.thr));
        }
        if (lane == 0) {
          sel[i] = gt;
          take[i] = eq;
        }
      }
      __syncthreads();
      n_sel = place([&](int i) { return sel[i]; }, t.all ? 0u : t.need_eq);
      for (int i = warp; i < nreg; i += kWarps) {
        const uint4 e = wt[i];
        uint32_t pos = off[i], eq_run = 0u;
        const uint32_t tk = take[i];
        for (uint32_t j0 = 0; j0 < e.y; j0 += 32) {
          const bool in = j0 + lane < e.y;
          const uint32_t kk = in ? __ldcg(pk + e.x + j0 + lane) : 0u;
          const bool gt = kk != 0u && (t.all || kk > t.thr);
          const bool eq = kk != 0u && !t.all && kk == t.thr;
          const uint32_t em = __ballot_sync(0xffffffffu, eq);
          const bool s = gt || (eq && eq_run + __popc(em & lt) < tk);
          const uint32_t sm = __ballot_sync(0xffffffffu, s);
          if (s) dyn_out[pos + __popc(sm & lt)] = token(__ldcg(ps + e.x + j0 + lane));
          pos += __popc(sm);
          eq_run += __popc(em);
        }
      }
    } else {
      // every kept candidate (G < D <= kStageCap, so they are staged), and the
      // lowest-slot candidates equal to v
      const bool ties = v != 0u;                                  // v = 0: the kept candidates are all there are
      for (int i = tid; i < nreg; i += kThreads) take[i] = ties ? wt[i].z : 0u;
      __syncthreads();
      // at[] (staged offsets) is overwritten by place(); keep the runs' staged starts in wt[i].w
      for (int i = tid; i < nreg; i += kThreads) wt[i].w = at[i];
      __syncthreads();
      n_sel = place([&](int i) { return wt[i].y; }, ties ? D - G : 0u);
      for (int i = warp; i < nreg; i += kWarps) {
        const uint4 e = wt[i];
        uint32_t pos = off[i];
        const uint32_t tk = take[i];
        if (tk == 0u) {
          for (uint32_t j0 = lane; j0 < e.y; j0 += 32) dyn_out[pos + j0] = token(ss[e.w + j0]);
        } else {
          // this run holds some of the ties: rescan its slots
          const WarpRange wr = warp_range(pl, C, i / kWarps, i % kWarps);
          uint32_t eq_run = 0u;
          for (int s0 = wr.lo; s0 < wr.hi; s0 += 32) {
            const int s = s0 + lane;
            const uint32_t kk = s < wr.hi ? score_key(__ldcg(row + s)) : 0u;
            const bool eq = kk == v;
            const uint32_t em = __ballot_sync(0xffffffffu, eq);
            const bool sl = kk > v || (eq && eq_run + __popc(em & lt) < tk);
            const uint32_t sm = __ballot_sync(0xffffffffu, sl);
            if (sl) dyn_out[pos + __popc(sm & lt)] = token(s);
            pos += __popc(sm);
            eq_run += __popc(em);
          }
        }
      }
    }
  }
  for (int i = tid; i < pl.lead_a_n; i += kThreads) out[i] = pl.lead_a_lo + i;
  for (int i = tid; i < pl.lead_b_n; i += kThreads) out[pl.lead_a_n + i] = pl.lead_b_lo + i;
  const int tr0 = pl.dyn_off + static_cast<int>(n_sel);
  for (int i = tid; i < pl.trail_n; i += kThreads) out[tr0 + i] = pl.trail_lo + i;
  for (int i = tr0 + pl.trail_n + tid; i < a.out_len; i += kThreads) out[i] = -1;
}

// One CTA per row for rows of at most kThreads * RC dynamic slots: the keys
// stay in registers (warp-striped: lane l of warp w holds element
// w 32 RC + 32 j + l in k[j]), the exact D-th key comes from range-radix
// rounds over one shared histogram, and the selection is emitted in index
// order. No cluster barriers, no distributed shared memory, no workspace.
template <int RC>
__global__ void __launch_bounds__(kThreads, 1) select_row_kernel(const SelectArgs a) {
  pdl_wait();   // the scores come from the previous kernel
  pdl_trigger();
  __shared__ Shared sh;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Plan pl = make_plan(a, r);
  int* out = a.out + static_cast<long long>(r) * a.out_len;
  if (!pl.valid) {
    for (int i = tid; i < a.out_len; i += kThreads) out[i] = -1;
    return;
  }
  const int len = pl.dyn_hi - pl.dyn_lo;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride + pl.dyn_lo;
  const int e0 = warp * 32 * RC + lane;
  uint32_t k[RC];
#pragma unroll
  for (int j = 0; j < RC; ++j) {
    const int e = e0 + 32 * j;
    k[j] = e < len ? score_key(__ldg(row + e)) : 0u;
  }
  const Thr t = fast_threshold<RC>(k, static_cast<uint32_t>(pl.D), sh);
  int* dyn_out = out + pl.dyn_off;
  const long long prow = static_cast<long long>(r) * a.M;
  const bool hier = a.mode == kSelectHierTokens;
  const uint32_t n_sel = reg_emit<RC>(k, t, sh, [&](uint32_t p, int j) {
    const int slot = pl.dyn_lo + e0 + 32 * j;
    dyn_out[p] = hier ? __ldg(a.pages + prow + slot / a.P) * a.P + slot % a.P : slot;
  });
  for (int i = tid; i < pl.lead_a_n; i += kThreads) out[i] = pl.lead_a_lo + i;
  for (int i = tid; i < pl.lead_b_n; i += kThreads) out[pl.lead_a_n + i] = pl.lead_b_lo + i;
  const int tr0 = pl.dyn_off + static_cast<int>(n_sel);
  for (int i = tid; i < pl.trail_n; i += kThreads) out[tr0 + i] = pl.trail_lo + i;
  for (int i = tr0 + pl.trail_n + tid; i < a.out_len; i += kThreads) out[i] = -1;
}

}  // namespace

SelectPlan select_plan(int rows, int n_slots, int d_bound, int num_sms) {
  const int kLocalRegs = kThreads * kRL;    // segment that fits the register path
  const int kMergeRegs = kThreads * kRF;    // merged candidates that fit the register path
  constexpr int kSegMax = 32768;            // fallback: keys per CTA in shared memory
  SelectPlan p{};
  auto seg_of = [&](int C) { return (n_slots + C - 1) / C; };
  // row path: rows of at most 8192 slots, one CTA each, keys in registers.
  // Measured: faster than a cluster up to 8192 slots; at 16384 (32 keys per
  // thread on one SM) the 8-CTA cluster with 4 keys per thread is faster
  for (const int rc : {8, 16}) {
    if (n_slots <= kThreads * rc) {
      p.row = true;
      p.row_rc = rc;
      p.C = 1;
      p.seg = n_slots;
      return p;
    }
  }
  // cluster path: one cluster of up to 8 CTAs per row, any number of rows. The
  // cost of a CTA's passes grows with its keys per thread (each pass is
  // instruction-bound on one SM), so few rows spread over more CTAs with fewer
  // keys each (down to 4 per thread); many rows keep 32 (up to 131072 slots)
  // or 64 (up to 262144) to bound the CTA count
  for (const int rc : {4, 8, 16, 32, 64}) {
    const int cta_keys = kThreads * rc;
    const int C = (n_slots + cta_keys - 1) / cta_keys;
    if (C <= kClusterMax && (rows * C <= num_sms || rc >= 32)) {
      p.cluster = true;
      p.cluster_rc = rc;
      p.C = std::max(1, (n_slots + cta_keys - 1) / cta_keys);
      p.seg = seg_of(p.C);
      return p;
    }
  }
  // grid-cooperative path: register-sized segments, one CTA per SM, all co-resident
  const int Cg = std::max(1, (n_slots + kLocalRegs - 1) / kLocalRegs);
  int Cgrid = Cg;
  while (rows * Cgrid * 2 <= num_sms && seg_of(Cgrid * 2) >= 1024 && Cgrid * 2 <= kMaxGridC)
    Cgrid *= 2;   // more CTAs for latency, within the coordination block's capacity
  if (rows * Cgrid <= num_sms && Cgrid <= kMaxGridC) {
    p.grid = true;
    p.C = Cgrid;
    p.seg = seg_of(Cgrid);
    p.cand_cap = 0;
    return p;
  }
  // filter path: rows too long for one cluster and for the grid launch, few enough
  // that each gets two or more CTAs
  if (d_bound >= 1 && n_slots > kClusterMax * kThreads * 64 && n_slots <= (1 << 21) && 2 * rows <= num_sms) {
    p.filter = true;
    const int c_min = (n_slots + kWarps * kWarpSlots - 1) / (kWarps * kWarpSlots);   // warp slices fit registers
    p.C = std::max(c_min, std::min((n_slots + 4095) / 4096, num_sms / rows));
    p.seg = seg_of(p.C);
    // groups of G slots: the bound is tight when there are many groups per
    // dynamic slot (G <= n / (8 D)); phase 1 holds at most kPhase1Cap of them
    int G = 1;
    while (G < 64 && 16ll * G * d_bound <= 2ll * n_slots) G *= 2;   // largest G <= n / (8 D)
    while (true) {
      const int g0 = std::min(G, 16);
      int sh = 0;
      while ((1 << sh) < g0) ++sh;
      const int fold = G / g0;
      const int ng0 = (n_slots + g0 - 1) / g0;
      const int unit = std::max(fold, 4);
      const int stride = (ng0 + unit - 1) / unit * unit;
      if (stride / fold <= kPhase1Cap) {
        p.g0_shift = sh;
        p.fold = fold;
        p.gmax_stride = stride;
        break;
      }
      G *= 2;
    }
    p.pool_cap = d_bound * G + 32;
    return p;
  }
  // few rows: ~2K keys per CTA for latency; rows alone fill the GPU: register-sized segments
  int C = rows >= num_sms ? std::max(1, (n_slots + kLocalRegs - 1) / kLocalRegs)
                          : std::max(1, std::min(64, (n_slots + 2047) / 2048));
  while (seg_of(C) > kLocalRegs && C < 1024) C *= 2;                   // local keys in registers
  while (C > 1 && C * std::min(d_bound, seg_of(C)) > kMergeRegs && seg_of(C / 2) <= kLocalRegs) C /= 2;
  while (seg_of(C) > kSegMax) C *= 2;
  p.C = C;
  p.seg = seg_of(C);
  p.cand_cap = std::max(1, std::min(d_bound, p.seg));
  p.final_in_smem = false;
  return p;
}

FilterLayout filter_layout(int rows, const SelectPlan& p) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  FilterLayout L{};
  size_t o = 0;
  L.gmax = o;
  o += al(static_cast<size_t>(rows) * p.gmax_stride * 4);
  L.pool_keys = o;
  o += al(static_cast<size_t>(rows) * p.pool_cap * 4);
  L.pool_slots = o;
  o += al(static_cast<size_t>(rows) * p.pool_cap * 4);
  L.wtab = o;
  o += al(static_cast<size_t>(rows) * p.C * kWarps * 16);
  L.counters = o;
  o += al(static_cast<size_t>(rows) * 8);
  L.total = o;
  return L;
}

size_t select_ws_bytes(int rows, const SelectPlan& p) {
  if (p.filter) return filter_layout(rows, p).total;
  if (p.cluster || p.row) return 0;
  if (p.grid) return grid_blocks_bytes(rows) + grid_row_bytes(p.C) * rows;
  const size_t n = static_cast<size_t>(rows) * p.C * p.cand_cap;
  return ((n * 8 + rows * 4 + 255) / 256) * 256;
}

cudaError_t launch_select(const SelectArgs& a0, const SelectPlan& p, void* ws, cudaStream_t stream,
                          bool gmax_ready) {
  SelectArgs a = a0;
  const int rows = a.B * a.T;
  if (p.filter) {
    const FilterLayout Ly = filter_layout(rows, p);
    uint8_t* w = static_cast<uint8_t*>(ws);
    a.gmax = reinterpret_cast<uint32_t*>(w + Ly.gmax);
    a.gmax_stride = p.gmax_stride;
    a.g0_shift = p.g0_shift;
    a.fold = p.fold;
    a.pool_keys = reinterpret_cast<uint32_t*>(w + Ly.pool_keys);
    a.pool_slots = reinterpret_cast<int*>(w + Ly.pool_slots);
    a.pool_cap = p.pool_cap;
    a.wtab = reinterpret_cast<uint4*>(w + Ly.wtab);
    a.counters = reinterpret_cast<unsigned*>(w + Ly.counters);
    void* args[] = {&a};
    if (!gmax_ready) {
      const int blocks = std::min((p.gmax_stride + 255) / 256, 64);
      cudaError_t e = launch_pdl(reinterpret_cast<const void*>(&group_max_kernel), dim3(blocks, rows), dim3(256), 0,
                                 stream, args);
      if (e != cudaSuccess) return e;
    }
    const size_t smem = static_cast<size_t>(p.C) * kWarps * 28 + static_cast<size_t>(kStageCap) * 8;
    const void* fn = reinterpret_cast<const void*>(&select_filter_kernel);
    cudaError_t e = set_max_smem(fn, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(fn, dim3(p.C, rows), dim3(kThreads), smem, stream, args);
  }
  if (p.row) {
    const void* fn = p.row_rc == 16 ? reinterpret_cast<const void*>(&select_row_kernel<16>)
                                    : reinterpret_cast<const void*>(&select_row_kernel<8>);
    void* args[] = {&a};
    return launch_pdl(fn, dim3(rows, 1, 1), dim3(kThreads, 1, 1), 0, stream, args);
  }
  if (p.cluster) {
    const size_t smem = cluster_smem_words(p.cluster_rc) * 4;
    const void* fn = p.cluster_rc == 64   ? reinterpret_cast<const void*>(&select_cluster_kernel<64>)
                     : p.cluster_rc == 32 ? reinterpret_cast<const void*>(&select_cluster_kernel<32>)
                     : p.cluster_rc == 16 ? reinterpret_cast<const void*>(&select_cluster_kernel<16>)
                     : p.cluster_rc == 8  ? reinterpret_cast<const void*>(&select_cluster_kernel<8>)
                                          : reinterpret_cast<const void*>(&select_cluster_kernel<4>);
    cudaError_t e = set_max_smem(fn, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    void* args[] = {&a};
    return launch_pdl(fn, dim3(p.C, rows, 1), dim3(kThreads, 1, 1), smem, stream, args, attr, 1);
  }
  if (p.grid) {
    a.grid_ws = ws;
    a.grid_row_bytes = grid_row_bytes(p.C);
    // reset the rows' coordination blocks (counters, flags, window histograms)
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(GridRow) * static_cast<size_t>(rows), stream);
    if (e != cudaSuccess) return e;
    const size_t smem = (static_cast<size_t>(kThreads) * kRL + static_cast<size_t>(kSubHist) * kWHStride) * 4;
    const void* fn = reinterpret_cast<const void*>(&select_grid_kernel);
    e = set_max_smem(fn, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.C, rows, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs co-resident: rows wait on each other
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&a};
    return cudaLaunchKernelExC(&cfg, fn, args);
  }
  const size_t n = static_cast<size_t>(rows) * p.C * p.cand_cap;
  a.cand_cap = p.cand_cap;
  a.final_in_smem = p.final_in_smem ? 1 : 0;
  a.cand_keys = static_cast<uint32_t*>(ws);
  a.cand_slots = reinterpret_cast<int*>(a.cand_keys + n);
  a.row_arrivals = reinterpret_cast<unsigned*>(a.cand_slots + n);
  cudaError_t e = cudaMemsetAsync(a.row_arrivals, 0, rows * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  const size_t smem = p.seg > kThreads * kRL ? static_cast<size_t>(p.seg) * 4 : 0;   // fallback keys
  const void* fn = reinterpret_cast<const void*>(&select_kernel);
  e = set_max_smem(fn, smem);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  return launch_pdl(fn, dim3(p.C, rows), dim3(kThreads), smem, stream, args);
}

}  // namespace lsa
