// Lightning-indexer scores on tcgen05 tensor cores.
//
// What it computes (DSA Lightning Indexer article, "Lightweight Scoring
// Module": ReLU of the scaled q.k product; LSA paper section 2.2: the DSA
// indexer sums heads with per-query weights):
//
//   score[b,t,s] = (1/sqrt(d)) * sum_h w[b,t,h] * ReLU(q[b,t,h,:] . k[b,s,:])
//
// for keys s visible to query t (s < (pos(t)+1) / vis_div), -inf otherwise.
// With e4m3 inputs q and k stand for code * row scale; both scales are > 0, so
// ReLU(qs*ks*x) = qs*ks*ReLU(x): qs folds into w and ks multiplies the head sum.
//
// Mapping: keys on the MMA M dimension (128 TMEM lanes), (query, head) pairs on
// N (N = NQ * H <= 256), K = d. Each epilogue thread owns one key row, so the
// ReLU, the head-weighted sum and the causal mask are thread-local and the
// [keys x heads] product never leaves the SM.
//
// Roles (320 threads, one CTA per SM, persistent over a contiguous tile range):
//   warp 0      TMA producer: key tiles into an S-stage ring, query tiles into
//               1-2 buffers (re-loaded only when the query group changes)
//   warp 1      TMEM owner + single-thread UMMA issuer; 2 or 4 accumulators
//   warps 2..9  two epilogue warpgroups taking alternate tiles:
//               TMEM -> registers -> fp32 scores in global memory
//
// Two tile sources: FLAT (128 consecutive key rows of one sequence) and
// GATHER (the recalled pages of one query, 128 / P pages per tile, used by the
// fine stage of Hierarchical Indexing).
#include "internal.h"
#include "ptx.cuh"

namespace lsa {
namespace {

constexpr int kEpiWG = 2;                      // epilogue warpgroups
constexpr int kThreads = 64 + 128 * kEpiWG;
constexpr int kTileM = 128;

template <int DK, bool FP8>
struct Cfg {
  static constexpr int kElt = FP8 ? 1 : 2;
  static constexpr int kRowBytes = DK * kElt;          // bytes of one key / query row
  static constexpr int kBoxes = kRowBytes / 128;       // 128-byte swizzle boxes per row
  static constexpr int kBoxElems = 128 / kElt;         // elements per box row
  static constexpr int kATileBytes = kTileM * kRowBytes;
  static constexpr int kKSteps = kRowBytes / 32;       // one MMA consumes 32 bytes of K
  static_assert(kBoxes >= 1, "row must span at least one 128-byte box");
};

__device__ __forceinline__ int clamp_len(const int* seq_len, int b, int L_max) {
  int L = __ldg(seq_len + b);
  return L < 0 ? 0 : (L > L_max ? L_max : L);
}

// Per query group (FLAT: NQ queries of one sequence; GATHER: one query row).
struct Group {
  int b, q0, nq;      // sequence, first query, valid queries
  int pos0;           // absolute position of query q0 (may be negative)
  int n_live;         // tiles of this group that hold visible keys
};

__device__ __forceinline__ Group make_group(const IndexerArgs& a, long long grp) {
  Group g;
  if (!a.gather) {
    g.b = static_cast<int>(grp / a.G);
    g.q0 = static_cast<int>(grp - static_cast<long long>(g.b) * a.G) * a.NQ;
    g.nq = min(a.NQ, a.T - g.q0);
    g.pos0 = clamp_len(a.seq_len, g.b, a.L_max) - a.T + g.q0;
    const int pos_last = g.pos0 + g.nq - 1;
    const int nvis = pos_last < 0 ? 0 : (pos_last + 1) >> a.vis_shift;
    g.n_live = min(a.n_tiles, (nvis + kTileM - 1) / kTileM);
  } else {
    const int r = static_cast<int>(grp);
    g.b = r / a.T;
    g.q0 = r - g.b * a.T;
    g.nq = 1;
    g.pos0 = clamp_len(a.seq_len, g.b, a.L_max) - a.T + g.q0;
    g.n_live = g.pos0 >= 0 ? a.n_tiles : 0;
  }
  return g;
}

// Walks this CTA's contiguous range of (group, tile) items without divisions.
struct TileIter {
  long long item, end, grp;
  int j;
  Group g;
  __device__ __forceinline__ void begin(const IndexerArgs& a, long long b0, long long e0) {
    item = b0;
    end = e0;
    grp = b0 / a.n_tiles;
    j = static_cast<int>(b0 - grp * a.n_tiles);
    g = make_group(a, grp);
  }
  __device__ __forceinline__ bool valid() const { return item < end; }
  __device__ __forceinline__ bool live() const { return j < g.n_live; }
  __device__ __forceinline__ void next(const IndexerArgs& a) {
    ++item;
    if (++j == a.n_tiles) {
      j = 0;
      ++grp;
      if (item < end) g = make_group(a, grp);
    }
  }
};

__device__ __forceinline__ void spin_ns(unsigned long long ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

// acc[i % 8] += w[i] * max(v[i], 0): eight independent FMA chains.
template <int NV>
__device__ __forceinline__ void relu_dot_acc(const float* wcol, const uint32_t (&v)[NV], float (&acc)[8]) {
#pragma unroll
  for (int i = 0; i < NV; i += 4) {
    const float4 wv = *reinterpret_cast<const float4*>(wcol + i);
    acc[(i + 0) & 7] = fmaf(wv.x, fmaxf(__uint_as_float(v[i + 0]), 0.f), acc[(i + 0) & 7]);
    acc[(i + 1) & 7] = fmaf(wv.y, fmaxf(__uint_as_float(v[i + 1]), 0.f), acc[(i + 1) & 7]);
    acc[(i + 2) & 7] = fmaf(wv.z, fmaxf(__uint_as_float(v[i + 2]), 0.f), acc[(i + 2) & 7]);
    acc[(i + 3) & 7] = fmaf(wv.w, fmaxf(__uint_as_float(v[i + 3]), 0.f), acc[(i + 3) & 7]);
  }
}

// Selection summary written beside a FLAT score (the selection's filter launch
// reads it): the maximum score key of each group of 2^g0_shift consecutive
// slots over the query's dynamic candidates -- visible, neither sink nor
// window -- from the 32 consecutive slots of this warp (one per lane).
// Warp-uniform: every lane calls it.
__device__ __forceinline__ void flat_group_max(const IndexerArgs& a, long long qrow, int s, int nvis, float v,
                                               int lane) {
  const int pe = nvis - 1;                           // the query's last visible slot
  const int sink_end = min(a.sink, max(pe + 1, 0));
  const int w_lo = max(sink_end, pe - a.window + 1);
  uint32_t key = (s >= sink_end && s < w_lo) ? score_key(v) : 0u;
  for (int o = 1; o < (1 << a.g0_shift); o <<= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, o));
  if ((lane & ((1 << a.g0_shift) - 1)) == 0) a.gmax[qrow * a.gmax_stride + (s >> a.g0_shift)] = key;
}

// A FLAT score. Rows of a multi-group (prefill) launch are far larger than L2
// and read only by a later selection, so they bypass it (streaming store);
// decode rows stay in L2 for the selection that follows at once.
__device__ __forceinline__ void store_score(const IndexerArgs& a, long long i, float v) {
  if (a.multi_group)
    __stcs(a.out + i, v);
  else
    a.out[i] = v;
}

__device__ __forceinline__ float sum8(const float (&a)[8]) {
  return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

// The eight chains of relu_dot_acc held as four packed pairs (chain 2j in the
// low half of acc2[j], 2j + 1 in the high half), advanced with the paired fp32
// FMA: each lane is an ordinary round-to-nearest fmaf, so the chains and their
// sum equal relu_dot_acc's bit for bit.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void relu_dot_acc2(const float* wcol, const uint32_t (&v)[32], uint64_t (&acc2)[4]) {
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float4 wv = *reinterpret_cast<const float4*>(wcol + i);
    const uint64_t r01 = pack2(fmaxf(__uint_as_float(v[i + 0]), 0.f), fmaxf(__uint_as_float(v[i + 1]), 0.f));
    const uint64_t r23 = pack2(fmaxf(__uint_as_float(v[i + 2]), 0.f), fmaxf(__uint_as_float(v[i + 3]), 0.f));
    uint64_t& a01 = acc2[(i & 7) >> 1];
    uint64_t& a23 = acc2[((i + 2) & 7) >> 1];
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a01) : "l"(pack2(wv.x, wv.y)), "l"(r01));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a23) : "l"(pack2(wv.z, wv.w)), "l"(r23));
  }
}

__device__ __forceinline__ float sum8x2(const uint64_t (&acc2)[4]) {
  float a[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) asm("mov.b64 {%0, %1}, %2;" : "=f"(a[2 * j]), "=f"(a[2 * j + 1]) : "l"(acc2[j]));
  return sum8(a);
}

template <int DK, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                   const IndexerArgs a) {
  using C = Cfg<DK, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages, NB = a.nbuf_b, N = a.N, NACC = a.n_acc;
  uint8_t* sA = base;
  uint8_t* sB = sA + static_cast<size_t>(S) * C::kATileBytes;
  float* wcol_all = reinterpret_cast<float*>(sB + static_cast<size_t>(NB) * N * C::kRowBytes);  // [8][N]
  uint64_t* a_full = reinterpret_cast<uint64_t*>(wcol_all + 4 * kEpiWG * N);
  uint64_t* a_empty = a_full + S;
  uint64_t* b_full = a_empty + S;
  uint64_t* b_empty = b_full + 2;
  uint64_t* acc_full = b_empty + 2;
  uint64_t* acc_empty = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long per = a.n_items / gridDim.x, rem = a.n_items % gridDim.x;
  const long long it_begin = blockIdx.x * per + min(static_cast<long long>(blockIdx.x), rem);
  const long long it_end = it_begin + per + (blockIdx.x < rem ? 1 : 0);

  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(NACC * N)) tmem_cols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);    // the four warps of the epilogue warpgroup owning the slot
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();   // inputs may come from the previous kernel in the stream
  pdl_trigger();
  if (a.sel_counters && blockIdx.x == 0)   // the selection that follows starts from zero counters
    for (int i = threadIdx.x; i < 2 * a.B * a.T; i += blockDim.x) a.sel_counters[i] = 0u;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      const uint64_t pol = policy_evict_first();   // recalled pages' keys are read once
      long long na = 0, ng = 0, cur = -1;
      TileIter it;
      for (it.begin(a, it_begin, it_end); it.valid(); it.next(a)) {
        if (!it.live()) continue;
        if (*abort_flag) break;
        if (it.grp != cur) {
          const int bs = static_cast<int>(ng % NB);
          const uint32_t ph = static_cast<uint32_t>((ng / NB) & 1);
          if (!mbar_wait(&b_empty[bs], ph ^ 1, a.status)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&b_full[bs], N * C::kRowBytes);
          const int qrow = (it.g.b * a.T + it.g.q0) * a.H;
          uint8_t* dst = sB + static_cast<size_t>(bs) * N * C::kRowBytes;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_2d(dst + bx * N * 128, &tm_q, &b_full[bs], bx * C::kBoxElems, qrow);
          cur = it.grp;
          ++ng;
        }
        const int s = static_cast<int>(na % S);
        const uint32_t ph = static_cast<uint32_t>((na / S) & 1);
        if (!mbar_wait(&a_empty[s], ph ^ 1, a.status)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&a_full[s], C::kATileBytes);
        uint8_t* dst = sA + static_cast<size_t>(s) * C::kATileBytes;
        if (!a.gather) {
          // default L2 policy: measured faster than evict-first for keys read
          // once, and a prefill chunk's other query groups re-read them from L2
          const int y = it.g.b * a.L_rows + kTileM * it.j;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_2d(dst + bx * kTileM * 128, &tm_k, &a_full[s], bx * C::kBoxElems, y);
        } else {
          const int per_tile = kTileM / a.P;
          const long long r = it.grp;
          for (int sub = 0; sub < per_tile; ++sub) {
            const int pi = it.j * per_tile + sub;
            int page = pi < a.M ? __ldg(a.pages + r * a.M + pi) : -1;
            if (page < 0) page = 0;   // masked in the epilogue
            const int y = it.g.b * a.L_max + page * a.P;
#pragma unroll
            for (int bx = 0; bx < C::kBoxes; ++bx)
              tma_load_2d_hint(dst + bx * kTileM * 128 + sub * a.P * 128, &tm_k, &a_full[s], bx * C::kBoxElems,
                               y, pol);
          }
        }
        ++na;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc = FP8 ? make_idesc(0, 0, kTileM, N, 0, 0) : make_idesc(1, 1, kTileM, N, 0, 0);
      long long na = 0, ng = 0, nt = 0, cur = -1;
      int bs = 0;
      TileIter it;
      for (it.begin(a, it_begin, it_end); it.valid(); it.next(a)) {
        if (!it.live()) continue;
        if (*abort_flag) break;
        if (it.grp != cur) {
          if (cur >= 0) umma_commit(&b_empty[bs]);   // old query tile free once its MMAs finish
          bs = static_cast<int>(ng % NB);
          const uint32_t ph = static_cast<uint32_t>((ng / NB) & 1);
          if (!mbar_wait(&b_full[bs], ph, a.status)) { *abort_flag = 1; break; }
          cur = it.grp;
          ++ng;
        }
        const int acc = static_cast<int>(nt % NACC);
        const uint32_t aph = static_cast<uint32_t>((nt / NACC) & 1);
        if (!mbar_wait(&acc_empty[acc], aph ^ 1, a.status)) { *abort_flag = 1; break; }
        const int s = static_cast<int>(na % S);
        const uint32_t ph = static_cast<uint32_t>((na / S) & 1);
        if (!mbar_wait(&a_full[s], ph, a.status)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + static_cast<size_t>(s) * C::kATileBytes);
        const uint32_t b0 = smem_u32(sB + static_cast<size_t>(bs) * N * C::kRowBytes);
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * N);
#pragma unroll
        for (int ks = 0; ks < C::kKSteps; ++ks) {
          const int bx = ks >> 2, off = (ks & 3) * 32;
          const uint64_t ad = make_sdesc(a0 + bx * kTileM * 128 + off, 16, 1024, kLayoutSW128);
          const uint64_t bd = make_sdesc(b0 + bx * N * 128 + off, 16, 1024, kLayoutSW128);
          if (FP8)
            umma_f8(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
          else
            umma_f16(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        umma_commit(&a_empty[s]);
        umma_commit(&acc_full[acc]);
        ++na;
        ++nt;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int ew = warp - 2;              // 0..7
    const int wg = ew >> 2;               // epilogue warpgroup: takes live tiles with nt % 2 == wg
    const int qw = warp & 3;              // TMEM lane quarter of this warp
    const int row = qw * 32 + lane;       // key row of the tile owned by this thread
    float* wcol = wcol_all + ew * N;      // per-warp copy: no cross-warp barrier needed
    long long nt = 0, cur = -1;
    int sink_end = 0, w_lo = 0;
    TileIter it;
    for (it.begin(a, it_begin, it_end); it.valid(); it.next(a)) {
      const bool live = it.live();
      const bool mine = live ? ((nt & 1) == wg) : ((it.j & 1) == wg);
      if (!mine) {
        nt += live ? 1 : 0;
        continue;
      }
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;   // warp-uniform exit
      const Group& g = it.g;
      if (it.grp != cur) {
        __syncwarp();
        for (int c = lane; c < N; c += 32) {
          const int qi = c / a.H, h = c - qi * a.H;
          float wv = 0.f;
          if (qi < g.nq) {
            const long long wi = (static_cast<long long>(g.b) * a.T + g.q0 + qi) * a.H + h;
            wv = __ldg(a.w + wi) * a.inv_sqrt_d;
            if (FP8) wv *= __ldg(a.q_scale + wi);
          }
          wcol[c] = wv;
        }
        __syncwarp();
        if (a.gather && g.pos0 >= 0) {
          sink_end = min(a.sink, g.pos0 + 1);
          w_lo = max(sink_end, g.pos0 - a.window + 1);
        }
        cur = it.grp;
      }
      const int s = kTileM * it.j + row;                       // key row (FLAT) or slot (GATHER)
      const long long orow = (static_cast<long long>(g.b) * a.T + g.q0) * a.out_row_stride;
      if (!live) {
        if (!a.gather) {
          if (s < a.L_rows)
            for (int qi = 0; qi < g.nq; ++qi) store_score(a, orow + qi * a.out_row_stride + s, -INFINITY);
          if (a.gmax && (lane & ((1 << a.g0_shift) - 1)) == 0)
            for (int qi = 0; qi < g.nq; ++qi)
              a.gmax[(static_cast<long long>(g.b) * a.T + g.q0 + qi) * a.gmax_stride + (s >> a.g0_shift)] = 0u;
        } else if (s < a.M * a.P) {
          a.out[orow + s] = -INFINITY;
        }
        continue;
      }
      const int acc = static_cast<int>(nt % NACC);
      const uint32_t aph = static_cast<uint32_t>((nt / NACC) & 1);
      ++nt;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], aph, a.status))) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(acc * N);
      float kscale = 1.f;
      if (FP8 && !a.gather && s < a.L_rows) kscale = __ldg(a.k_scale + static_cast<long long>(g.b) * a.L_rows + s);
      // the score of query qi of the group from its head sum sc
      auto finish = [&](int qi, float sc) {
        if (qi >= g.nq) return;
        if (!a.gather) {
          const int pos = g.pos0 + qi;   // key s visible iff s < (pos + 1) >> vis_shift
          const int nvis = pos < 0 ? 0 : (pos + 1) >> a.vis_shift;
          const float v = s < nvis ? sc * kscale : -INFINITY;
          if (s < a.L_rows) store_score(a, orow + qi * a.out_row_stride + s, v);
          if (a.gmax) flat_group_max(a, static_cast<long long>(g.b) * a.T + g.q0 + qi, s, nvis, v, lane);
        } else if (s < a.M * a.P) {
          const int page = __ldg(a.pages + (static_cast<long long>(g.b) * a.T + g.q0) * a.M + s / a.P);
          const int tok = page * a.P + (s & (a.P - 1));
          // e4m3: the recalled token's own key scale
          const float ks = (FP8 && page >= 0) ? __ldg(a.k_scale + static_cast<long long>(g.b) * a.L_max + tok) : 1.f;
          a.out[orow + s] = (page >= 0 && tok >= sink_end && tok < w_lo) ? sc * ks : -INFINITY;
        }
      };
      if ((a.H & 63) == 0) {
        // 64 columns per load round, summed with paired FMAs
        for (int qi = 0; qi < a.NQ; ++qi) {
          uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
          for (int c0 = qi * a.H; c0 < (qi + 1) * a.H; c0 += 64) {
            uint32_t v0[32], v1[32];
            tmem_ld32(tbase + c0, v0);
            tmem_ld32(tbase + c0 + 32, v1);
            tmem_ld_wait();
            relu_dot_acc2(wcol + c0, v0, acc2);
            relu_dot_acc2(wcol + c0 + 32, v1, acc2);
          }
          finish(qi, sum8x2(acc2));
        }
      } else if (a.H >= 16) {
        for (int qi = 0; qi < a.NQ; ++qi) {
          float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          const int c_end = (qi + 1) * a.H;
          for (int c0 = qi * a.H; c0 < c_end;) {
            if (c_end - c0 >= 32) {
              uint32_t v0[32];
              tmem_ld32(tbase + c0, v0);
              tmem_ld_wait();
              relu_dot_acc<32>(wcol + c0, v0, acc8);
              c0 += 32;
            } else {
              uint32_t v0[16];
              tmem_ld16(tbase + c0, v0);
              tmem_ld_wait();
              relu_dot_acc<16>(wcol + c0, v0, acc8);
              c0 += 16;
            }
          }
          finish(qi, sum8(acc8));
        }
      } else {
        // H in {4, 8}: one 16-column load covers 16 / H queries
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tbase + c0, v);
          tmem_ld_wait();
          const int per = 16 / a.H;
          for (int qq = 0; qq < per; ++qq) {
            float sc = 0.f;
            for (int i = 0; i < a.H; ++i)
              sc = fmaf(wcol[c0 + qq * a.H + i], fmaxf(__uint_as_float(v[qq * a.H + i]), 0.f), sc);
            finish(c0 / a.H + qq, sc);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) spin_ns(50000);   // let in-flight copies and MMAs land before TMEM is released
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

template <int DK, bool FP8>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(&indexer_kernel<DK, FP8>);
}

}  // namespace

size_t indexer_smem_bytes(int d, bool fp8, int N, int stages, int nbuf_b) {
  const size_t row = static_cast<size_t>(d) * (fp8 ? 1 : 2);
  return 1024 + stages * 128 * row + nbuf_b * N * row + 4 * kEpiWG * N * 4 + (2 * stages + 12) * 8 + 16;
}

// The key ring is what keeps HBM busy (bytes in flight per SM); a second
// query buffer only hides the reload at a query-group change, so it is kept
// only when it costs no key stage.
void indexer_pick_pipeline(int d, bool fp8, int N, int* stages, int* nbuf_b) {
  const size_t kMax = 232448;
  const int kMaxStages = 4;   // measured: deeper key rings only add queueing latency at the HBM read ceiling
  auto fit = [&](int nb) {
    int s = kMaxStages;
    while (s > 2 && indexer_smem_bytes(d, fp8, N, s, nb) > kMax) --s;
    return s;
  };
  const int s2 = fit(2), s1 = fit(1);
  *nbuf_b = s2 >= s1 ? 2 : 1;
  *stages = s2 >= s1 ? s2 : s1;
}

int indexer_n_acc(int N) { return 4 * N <= 512 ? 4 : 2; }

cudaError_t launch_indexer(const CUtensorMap& tm_k, const CUtensorMap& tm_q, const IndexerArgs& a, bool fp8,
                           int grid, cudaStream_t stream) {
  const void* fn = nullptr;
  if (fp8) {
    if (a.d != 128) return cudaErrorInvalidValue;
    fn = kernel_ptr<128, true>();
  } else {
    fn = a.d == 128 ? kernel_ptr<128, false>() : kernel_ptr<64, false>();
  }
  size_t smem = indexer_smem_bytes(a.d, fp8, a.N, a.stages, a.nbuf_b);
  if (smem < 120 * 1024) smem = 120 * 1024;   // one CTA per SM: TMEM allocation never contends
  cudaError_t e = set_max_smem(fn, smem);
  if (e != cudaSuccess) return e;
  void* args[] = {const_cast<CUtensorMap*>(&tm_k), const_cast<CUtensorMap*>(&tm_q), const_cast<IndexerArgs*>(&a)};
  return launch_pdl(fn, dim3(grid), dim3(kThreads), smem, stream, args);
}

}  // namespace lsa
