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
// Roles (192 threads, one CTA per SM, persistent over a contiguous item range):
//   warp 0      TMA producer: key tiles into an S-stage ring, query tiles into
//               1-2 buffers (re-loaded only when the query group changes)
//   warp 1      TMEM owner + single-thread UMMA issuer, double-buffered accumulator
//   warps 2..5  epilogue: TMEM -> registers -> fp32 scores in global memory
//
// Two tile sources: FLAT (128 consecutive key rows of one sequence) and
// GATHER (the recalled pages of one query, 128 / P pages per tile, used by the
// fine stage of Hierarchical Indexing).
#include "internal.h"
#include "ptx.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 192;
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

struct Item {
  int b, t_or_g, j, q0;
  long long group;
  bool live;
};

__device__ __forceinline__ int clamp_len(const int* seq_len, int b, int L_max) {
  int L = __ldg(seq_len + b);
  return L < 0 ? 0 : (L > L_max ? L_max : L);
}

__device__ __forceinline__ Item decode_item(const IndexerArgs& a, long long item) {
  Item it;
  it.j = static_cast<int>(item % a.n_tiles);
  const long long grp = item / a.n_tiles;
  it.group = grp;
  if (!a.gather) {
    const int g = static_cast<int>(grp % a.G);
    const int b = static_cast<int>(grp / a.G);
    it.b = b;
    it.t_or_g = g;
    it.q0 = g * a.NQ;
    const int Lb = clamp_len(a.seq_len, b, a.L_max);
    const int t_last = min(a.T - 1, it.q0 + a.NQ - 1);
    const int pos_last = Lb - a.T + t_last;
    const int nvis = pos_last < 0 ? 0 : (pos_last + 1) / a.vis_div;
    it.live = static_cast<long long>(kTileM) * it.j < nvis;
  } else {
    const int r = static_cast<int>(grp);
    const int b = r / a.T, t = r % a.T;
    it.b = b;
    it.t_or_g = t;
    it.q0 = t;
    it.live = clamp_len(a.seq_len, b, a.L_max) - a.T + t >= 0;
  }
  return it;
}

// Write one score (or -inf) for query `qi` of the tile, key row `row`.
template <bool FP8>
__device__ __forceinline__ void emit_score(const IndexerArgs& a, const Item& it, int qi, int row, float score,
                                           bool dead) {
  if (!a.gather) {
    const int t = it.q0 + qi;
    if (qi >= a.NQ || t >= a.T) return;
    const int s = kTileM * it.j + row;
    if (s >= a.L_rows) return;
    const int pos = clamp_len(a.seq_len, it.b, a.L_max) - a.T + t;
    const int nvis = pos < 0 ? 0 : (pos + 1) / a.vis_div;
    float v = -INFINITY;
    if (!dead && s < nvis) {
      v = score;
      if (FP8) v *= __ldg(a.k_scale + static_cast<long long>(it.b) * a.L_rows + s);
    }
    a.out[(static_cast<long long>(it.b) * a.T + t) * a.out_row_stride + s] = v;
  } else {
    if (qi != 0) return;
    const int slot = kTileM * it.j + row;
    if (slot >= a.M * a.P) return;
    const int r = it.b * a.T + it.t_or_g;
    const int pos = clamp_len(a.seq_len, it.b, a.L_max) - a.T + it.t_or_g;
    float v = -INFINITY;
    if (!dead && pos >= 0) {
      const int page = __ldg(a.pages + static_cast<long long>(r) * a.M + slot / a.P);
      const int tok = page * a.P + slot % a.P;
      const int sink_end = min(a.sink, pos + 1);
      const int w_lo = max(sink_end, pos - a.window + 1);
      // only dynamic candidates (visible, in neither the sink nor the window)
      if (page >= 0 && tok >= sink_end && tok < w_lo) v = score;
    }
    a.out[static_cast<long long>(r) * a.out_row_stride + slot] = v;
  }
}

__device__ __forceinline__ float relu_dot16(const float* wcol, const uint32_t (&v)[16]) {
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) acc = fmaf(wcol[i], fmaxf(__uint_as_float(v[i]), 0.f), acc);
  return acc;
}

__device__ __forceinline__ float relu_dot32(const float* wcol, const uint32_t (&v)[32]) {
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) acc = fmaf(wcol[i], fmaxf(__uint_as_float(v[i]), 0.f), acc);
  return acc;
}

__device__ __forceinline__ void spin_ns(unsigned long long ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

template <int DK, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                   const IndexerArgs a) {
  using C = Cfg<DK, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages, NB = a.nbuf_b, N = a.N;
  uint8_t* sA = base;
  uint8_t* sB = sA + static_cast<size_t>(S) * C::kATileBytes;
  float* wcol_all = reinterpret_cast<float*>(sB + static_cast<size_t>(NB) * N * C::kRowBytes);  // [4][N]
  uint64_t* a_full = reinterpret_cast<uint64_t*>(wcol_all + 4 * N);
  uint64_t* a_empty = a_full + S;
  uint64_t* b_full = a_empty + S;
  uint64_t* b_empty = b_full + 2;
  uint64_t* acc_full = b_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long per = a.n_items / gridDim.x, rem = a.n_items % gridDim.x;
  const long long it_begin = blockIdx.x * per + min(static_cast<long long>(blockIdx.x), rem);
  const long long it_end = it_begin + per + (blockIdx.x < rem ? 1 : 0);

  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(2 * N)) tmem_cols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      const uint64_t pol = policy_evict_first();   // keys are streamed once
      long long na = 0, ng = 0, cur = -1;
      for (long long item = it_begin; item < it_end; ++item) {
        if (*abort_flag) break;
        const Item it = decode_item(a, item);
        if (!it.live) continue;
        if (it.group != cur) {
          const int bs = static_cast<int>(ng % NB);
          const uint32_t ph = static_cast<uint32_t>((ng / NB) & 1);
          if (!mbar_wait(&b_empty[bs], ph ^ 1, a.status)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&b_full[bs], N * C::kRowBytes);
          const int qrow = (it.b * a.T + it.q0) * a.H;
          uint8_t* dst = sB + static_cast<size_t>(bs) * N * C::kRowBytes;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_2d(dst + bx * N * 128, &tm_q, &b_full[bs], bx * C::kBoxElems, qrow);
          cur = it.group;
          ++ng;
        }
        const int s = static_cast<int>(na % S);
        const uint32_t ph = static_cast<uint32_t>((na / S) & 1);
        if (!mbar_wait(&a_empty[s], ph ^ 1, a.status)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&a_full[s], C::kATileBytes);
        uint8_t* dst = sA + static_cast<size_t>(s) * C::kATileBytes;
        if (!a.gather) {
          const int y = it.b * a.L_rows + kTileM * it.j;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_2d_hint(dst + bx * kTileM * 128, &tm_k, &a_full[s], bx * C::kBoxElems, y, pol);
        } else {
          const int per_tile = kTileM / a.P;
          const long long r = static_cast<long long>(it.b) * a.T + it.t_or_g;
          for (int sub = 0; sub < per_tile; ++sub) {
            const int pi = it.j * per_tile + sub;
            int page = pi < a.M ? __ldg(a.pages + r * a.M + pi) : -1;
            if (page < 0) page = 0;   // masked in the epilogue
            const int y = it.b * a.L_max + page * a.P;
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
      for (long long item = it_begin; item < it_end; ++item) {
        if (*abort_flag) break;
        const Item it = decode_item(a, item);
        if (!it.live) continue;
        if (it.group != cur) {
          if (cur >= 0) umma_commit(&b_empty[bs]);   // old query tile free once its MMAs finish
          bs = static_cast<int>(ng % NB);
          const uint32_t ph = static_cast<uint32_t>((ng / NB) & 1);
          if (!mbar_wait(&b_full[bs], ph, a.status)) { *abort_flag = 1; break; }
          cur = it.group;
          ++ng;
        }
        const int acc = static_cast<int>(nt & 1);
        const uint32_t aph = static_cast<uint32_t>((nt >> 1) & 1);
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
    const int qw = warp & 3;              // TMEM lane quarter of this warp
    const int row = qw * 32 + lane;       // key row of the tile owned by this thread
    float* wcol = wcol_all + qw * N;      // per-warp copy: no cross-warp barrier needed
    long long nt = 0, cur = -1;
    for (long long item = it_begin; item < it_end; ++item) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;   // warp-uniform exit
      const Item it = decode_item(a, item);
      if (it.group != cur) {
        __syncwarp();
        for (int c = lane; c < N; c += 32) {
          const int qi = c / a.H, h = c % a.H, t = it.q0 + qi;
          float wv = 0.f;
          if (qi < a.NQ && t < a.T) {
            const long long wi = (static_cast<long long>(it.b) * a.T + t) * a.H + h;
            wv = __ldg(a.w + wi) * a.inv_sqrt_d;
            if (FP8) wv *= __ldg(a.q_scale + wi);
          }
          wcol[c] = wv;
        }
        __syncwarp();
        cur = it.group;
      }
      if (!it.live) {
        for (int qi = 0; qi < a.NQ; ++qi) emit_score<FP8>(a, it, qi, row, 0.f, true);
        continue;
      }
      const int acc = static_cast<int>(nt & 1);
      const uint32_t aph = static_cast<uint32_t>((nt >> 1) & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], aph, a.status))) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(acc * N);
      if (a.H >= 16) {
        for (int qi = 0; qi < a.NQ; ++qi) {
          const int c_end = (qi + 1) * a.H;
          float sc = 0.f;
          for (int c0 = qi * a.H; c0 < c_end;) {
            if (c_end - c0 >= 64) {
              uint32_t v0[32], v1[32];
              tmem_ld32(tbase + c0, v0);
              tmem_ld32(tbase + c0 + 32, v1);
              tmem_ld_wait();
              sc += relu_dot32(wcol + c0, v0) + relu_dot32(wcol + c0 + 32, v1);
              c0 += 64;
            } else if (c_end - c0 >= 32) {
              uint32_t v0[32];
              tmem_ld32(tbase + c0, v0);
              tmem_ld_wait();
              sc += relu_dot32(wcol + c0, v0);
              c0 += 32;
            } else {
              uint32_t v0[16];
              tmem_ld16(tbase + c0, v0);
              tmem_ld_wait();
              sc += relu_dot16(wcol + c0, v0);
              c0 += 16;
            }
          }
          emit_score<FP8>(a, it, qi, row, sc, false);
        }
      } else {
        // H in {4, 8}: one 16-column load covers 16 / H queries
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tbase + c0, v);
          tmem_ld_wait();
          if (a.H == 8) {
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
              float sc = 0.f;
#pragma unroll
              for (int i = 0; i < 8; ++i)
                sc = fmaf(wcol[c0 + qq * 8 + i], fmaxf(__uint_as_float(v[qq * 8 + i]), 0.f), sc);
              emit_score<FP8>(a, it, c0 / 8 + qq, row, sc, false);
            }
          } else {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              float sc = 0.f;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                sc = fmaf(wcol[c0 + qq * 4 + i], fmaxf(__uint_as_float(v[qq * 4 + i]), 0.f), sc);
              emit_score<FP8>(a, it, c0 / 4 + qq, row, sc, false);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      ++nt;
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
  return 1024 + stages * 128 * row + nbuf_b * N * row + 4 * N * 4 + (2 * stages + 8) * 8 + 16;
}

void indexer_pick_pipeline(int d, bool fp8, int N, int* stages, int* nbuf_b) {
  const size_t kMax = 232448;
  const size_t row = static_cast<size_t>(d) * (fp8 ? 1 : 2);
  const size_t a_tile = 128 * row, b_tile = N * row;
  int nb = 2;
  if (indexer_smem_bytes(d, fp8, N, 3, 2) > kMax) nb = 1;
  int s = 8;
  while (s > 2 && indexer_smem_bytes(d, fp8, N, s, nb) > kMax) --s;
  (void)a_tile;
  (void)b_tile;
  *stages = s;
  *nbuf_b = nb;
}

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
  return cudaLaunchKernel(fn, dim3(grid), dim3(kThreads), args, smem, stream);
}

}  // namespace lsa
