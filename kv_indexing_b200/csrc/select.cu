// Streaming-aware top-k selection (LSA paper abstract (1) and the model card's
// "SI" bullet: a fixed attention sink and a local sliding window take part of
// the budget, dynamic top-k by indexer score fills the rest; the DSA Lightning
// Indexer article's "Dynamic Token Selector" for the top-k itself).
//
// Per query row: sink tokens [0, min(S, pos+1)), the window (the W most recent
// visible tokens not already in the sink), then the top D = k - |sink| - |window|
// dynamic candidates by (score descending, index ascending), written in
// ascending index order, then -1 padding. The same kernel selects pages for
// Hierarchical Indexing (forced sink/window pages + the top pages of the
// dynamic region, all ascending) and the fine token set over recalled pages.
//
// Algorithm: scores map to order-preserving uint32 keys (-inf -> 0 = not a
// candidate, -0 -> +0). A cluster of C CTAs splits the row's dynamic range
// into C contiguous segments; three radix passes (11, 11, 10 bits) build
// per-CTA histograms, merged across the cluster through distributed shared
// memory, that narrow down the exact key of the D-th best candidate. Every
// candidate above that key is taken, plus the lowest-index candidates equal to
// it; an ordered compaction (block scans, cluster-wide segment offsets) writes
// them in ascending index order. The result does not depend on C.
#include <cooperative_groups.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace lsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kPerThread = 8;   // consecutive elements per thread in the compaction

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                         // -0 ranks as +0
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return k <= 0x007FFFFFu ? 0u : k;                     // -inf: not a candidate
}

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
  const int pos = L - a.T + t;
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

// Inclusive scan of one value per thread (thread order). Uses `tmp` [kWarps+1].
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
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

// Histogram update with warp aggregation (lanes hitting the same bin add once).
__device__ __forceinline__ void hist_add(uint32_t* h, uint32_t bin, bool active) {
  const uint32_t key = active ? bin : 0xFFFFFFFFu;
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  const int leader = __ffs(peers) - 1;
  if (active && (threadIdx.x & 31) == leader) atomicAdd(&h[bin], static_cast<uint32_t>(__popc(peers)));
}

template <bool IN_SMEM>
__device__ __forceinline__ uint32_t key_at(const uint32_t* keys, const float* row, int my_lo, int i) {
  if (IN_SMEM) return keys[i];
  return score_key(__ldg(row + my_lo + i));
}

template <bool IN_SMEM>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelectArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int r = blockIdx.y;
  const int tid = threadIdx.x;

  extern __shared__ uint32_t sm[];
  uint32_t* hist[2] = {sm, sm + kBins};
  uint32_t* ghist = sm + 2 * kBins;
  uint32_t* tmp = ghist + kBins;          // kWarps + 1 scan scratch
  uint32_t* pub = tmp + 32;               // [0] = gt count, [1] = eq count (read by the cluster)
  uint32_t* keys = pub + 32;
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const Plan pl = make_plan(a, r);
  int* out = a.out + static_cast<long long>(r) * a.out_len;
  const float* row = a.scores + static_cast<long long>(r) * a.row_stride;
  if (!pl.valid) {
    if (rank == 0)
      for (int i = tid; i < a.out_len; i += kThreads) out[i] = -1;
    return;   // every CTA of the cluster takes this branch (same row)
  }

  const int len = pl.dyn_hi - pl.dyn_lo;
  const int seg = (len + C - 1) / C;
  int my_lo = pl.dyn_lo + rank * seg;
  if (my_lo > pl.dyn_hi) my_lo = pl.dyn_hi;
  const int my_hi = min(pl.dyn_hi, my_lo + seg);
  const int my_n = my_hi - my_lo;

  // ---- pass 0: load keys (cache in shared memory) + top-digit histogram ----
  for (int i = tid; i < kBins; i += kThreads) hist[0][i] = 0u;
  __syncthreads();
  for (int i0 = 0; i0 < my_n; i0 += kThreads) {
    const int i = i0 + tid;
    uint32_t k = 0u;
    if (i < my_n) {
      k = score_key(__ldg(row + my_lo + i));
      if (IN_SMEM) keys[i] = k;
    }
    hist_add(hist[0], k >> 21, k != 0u);
  }
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u, need = static_cast<uint32_t>(pl.D);
  uint32_t thr = 0u, need_eq = 0u;
  bool take_all = false;
  uint32_t n_cand = 0u;

  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const int nb = 1 << widths[pass];
    const uint32_t dmask = static_cast<uint32_t>(nb - 1);
    uint32_t* h = hist[pass & 1];
    if (pass > 0) {
      for (int i = tid; i < nb; i += kThreads) h[i] = 0u;
      __syncthreads();
      for (int i0 = 0; i0 < my_n; i0 += kThreads) {
        const int i = i0 + tid;
        const uint32_t k = i < my_n ? key_at<IN_SMEM>(keys, row, my_lo, i) : 0u;
        const bool act = k != 0u && (k & mask) == prefix;
        hist_add(h, (k >> shift) & dmask, act);
      }
      __syncthreads();
    }
    // merge the cluster's histograms
    cluster.sync();
    for (int i = tid; i < nb; i += kThreads) {
      uint32_t s = 0u;
      for (int c = 0; c < C; ++c) s += cluster.map_shared_rank(h, c)[i];
      ghist[i] = s;
    }
    __syncthreads();

    const int per = nb / kThreads;             // bins per thread (4 or 2)
    const int hi_bin = nb - per * tid;         // this thread owns bins [hi_bin - per, hi_bin)
    uint32_t local = 0u;
    for (int q = 1; q <= per; ++q) local += ghist[hi_bin - q];
    uint32_t total = 0u;
    const uint32_t incl = block_incl_scan(local, tmp, &total);

    if (pass == 0) {
      n_cand = total;
      // fixed outputs and padding (rank 0), now that the dynamic count is known
      if (rank == 0) {
        const int n_sel = min(static_cast<uint32_t>(pl.D), n_cand);
        for (int i = tid; i < pl.lead_a_n; i += kThreads) out[i] = pl.lead_a_lo + i;
        for (int i = tid; i < pl.lead_b_n; i += kThreads) out[pl.lead_a_n + i] = pl.lead_b_lo + i;
        const int tr0 = pl.dyn_off + n_sel;
        for (int i = tid; i < pl.trail_n; i += kThreads) out[tr0 + i] = pl.trail_lo + i;
        for (int i = tr0 + pl.trail_n + tid; i < a.out_len; i += kThreads) out[i] = -1;
      }
      if (n_cand <= need) {
        take_all = true;
        break;
      }
      if (need == 0u) break;
    }

    const uint32_t excl = incl - local;
    if (excl < need && need <= incl) {
      uint32_t above = excl;
      for (int q = 1; q <= per; ++q) {
        const int bb = hi_bin - q;
        if (above + ghist[bb] >= need) {
          s_bin = bb;
          s_above = above;
          break;
        }
        above += ghist[bb];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(s_bin) << shift;
    mask |= dmask << shift;
    need -= s_above;
    __syncthreads();
  }

  if (take_all) {
    thr = 0u;          // every candidate (key > 0)
    need_eq = 0u;
  } else if (pl.D == 0) {
    thr = 0xFFFFFFFFu;
    need_eq = 0u;
  } else {
    thr = prefix;      // exact key of the D-th best candidate
    need_eq = need;    // how many candidates equal to it are taken (lowest index first)
  }

  // ---- counts per segment, published to the cluster ----
  uint32_t gt = 0u, eq = 0u;
  for (int i = tid; i < my_n; i += kThreads) {
    const uint32_t k = key_at<IN_SMEM>(keys, row, my_lo, i);
    gt += (k > thr && k != 0u) ? 1u : 0u;
    eq += (k == thr && k != 0u) ? 1u : 0u;
  }
  uint32_t tgt = 0u, teq = 0u;
  block_incl_scan(gt, tmp, &tgt);
  block_incl_scan(eq, tmp, &teq);
  if (tid == 0) {
    pub[0] = tgt;
    pub[1] = teq;
  }
  cluster.sync();
  uint32_t base_sel = 0u, eq_before = 0u, my_take = 0u;
  for (int c = 0; c < C; ++c) {
    const uint32_t* rp = cluster.map_shared_rank(pub, c);
    const uint32_t g_c = rp[0], e_c = rp[1];
    const uint32_t take_c = need_eq > eq_before ? min(need_eq - eq_before, e_c) : 0u;
    if (c < rank) base_sel += g_c + take_c;
    if (c == rank) my_take = take_c;
    eq_before += e_c;
  }

  // ---- ordered compaction of this segment ----
  const int chunk = kThreads * kPerThread;
  uint32_t eq_run = 0u, sel_run = 0u;
  int* dyn_out = out + pl.dyn_off + base_sel;
  for (int c0 = 0; c0 < my_n; c0 += chunk) {
    const int i0 = c0 + tid * kPerThread;
    uint32_t kk[kPerThread];
    uint32_t ne = 0u;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const int i = i0 + e;
      kk[e] = i < my_n ? key_at<IN_SMEM>(keys, row, my_lo, i) : 0u;
      ne += (kk[e] == thr && kk[e] != 0u) ? 1u : 0u;
    }
    uint32_t eq_tot = 0u;
    const uint32_t eq_ex = block_incl_scan(ne, tmp, &eq_tot) - ne + eq_run;
    uint32_t ns = 0u, er = eq_ex;
    uint32_t selmask = 0u;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const uint32_t k = kk[e];
      bool s = false;
      if (k != 0u) {
        if (k > thr) {
          s = true;
        } else if (k == thr) {
          s = er < my_take;
          ++er;
        }
      }
      if (s) {
        selmask |= 1u << e;
        ++ns;
      }
    }
    uint32_t sel_tot = 0u;
    uint32_t pos_out = block_incl_scan(ns, tmp, &sel_tot) - ns + sel_run;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      if (selmask & (1u << e)) {
        const int slot = my_lo + i0 + e;
        int tok = slot;
        if (a.mode == kSelectHierTokens) {
          const int page = __ldg(a.pages + static_cast<long long>(r) * a.M + slot / a.P);
          tok = page * a.P + slot % a.P;
        }
        dyn_out[pos_out++] = tok;
      }
    }
    eq_run += eq_tot;
    sel_run += sel_tot;
  }
  cluster.sync();   // peers may still read this CTA's published counts
}

}  // namespace

int select_cluster_size(int rows, int max_dyn, int num_sms, int* cap) {
  const int kCapMax = 40960;   // keys cached per CTA (160 KB)
  int C = 1;
  while (C < 8 && rows * C * 2 <= num_sms) C *= 2;
  while (C < 8 && (max_dyn + C - 1) / C > kCapMax) C *= 2;
  const int seg = (max_dyn + C - 1) / C;
  *cap = seg <= kCapMax ? seg : 0;
  return C;
}

cudaError_t launch_select(const SelectArgs& a, int C, cudaStream_t stream) {
  const bool in_smem = a.cap > 0;
  const void* fn = in_smem ? reinterpret_cast<const void*>(&select_kernel<true>)
                           : reinterpret_cast<const void*>(&select_kernel<false>);
  const size_t smem = (3 * kBins + 64) * sizeof(uint32_t) + static_cast<size_t>(a.cap) * sizeof(uint32_t);
  cudaError_t e = set_max_smem(fn, smem);
  if (e != cudaSuccess) return e;
  const int rows = a.B * a.T;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, rows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {const_cast<SelectArgs*>(&a)};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace lsa
