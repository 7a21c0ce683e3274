// Gathered-KV sparse MQA / MLA attention (DSA Lightning Indexer article,
// "Sparse Attention Calculator": attention computed only over the selected
// top-k entries; LSA paper abstract: the selection reads only those KV rows).
//
//   o[r, h, :] = sum_j softmax_j(scale * q[r, h, :] . K[idx_j, :]) V[idx_j, :]
//
// over the valid (>= 0) entries idx_j of query row r; lse = log of the softmax
// denominator plus the max. For MLA one latent row per token serves as K
// (d_qk = 576) and its first d_v = 512 columns as V.
//
// One CTA = (v part, KV split, query row). Heads (<= 128, zero-padded) sit on
// the MMA M dimension; q is resident in shared memory. KV rows arrive 32 at a
// time by TMA (tiled boxes for contiguous runs, tile::gather4 row gathers
// otherwise) into 128-byte-swizzled tiles (double buffered), used K-major for S = q K^T and MN-major for O += P V. S (32
// columns) and O (d_v / n_parts <= 256 columns, the fp32 accumulator) live in
// TMEM; one thread per head runs the online softmax on its S row (lazy
// rescaling: the running max moves only when a block raises it by > 2^8) and
// writes bf16 P to shared memory for the PV MMA. With several KV splits each
// CTA writes an unnormalised partial (O, m, l) and a combine kernel merges them.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace lsa {
namespace {

// Outputs of one layer of a launch (see launch_attn).
struct LayerOut {
  uint16_t* out;          // [rows, Hq, d_v] bf16
  float* lse;             // [rows, Hq] or null
  uint16_t* part_o;       // [rows, n_split, Hq, d_v] bf16 split partials
  float* part_m;          // [rows, n_split, Hq]
  float* part_l;          // [rows, n_split, Hq]
  float scale_log2;       // the layer's softmax scale * log2(e)
  const uint8_t* kv8;     // e4m3 KV: the layer's latent rows of codes (else null)
  long long kv8_stride;   // bytes between consecutive latent rows
  const float* k_scale;   // e4m3 KV: per-token scale [B * L_max]
};
struct LayerOuts {
  LayerOut l[kMaxLaunchLayers];
  int n;
};

LayerOuts layer_outs(const AttnArgs* args, int n) {
  LayerOuts lo{};
  lo.n = n;
  for (int i = 0; i < n; ++i)
    lo.l[i] = LayerOut{args[i].out,
                       args[i].lse,
                       args[i].part_o,
                       args[i].part_m,
                       args[i].part_l,
                       args[i].scale_log2,
                       args[i].kv8 ? reinterpret_cast<const uint8_t*>(args[i].kp) : nullptr,
                       args[i].k_stride,
                       args[i].k_scale};
  return lo;
}

constexpr int kThreads = 128;
constexpr int BN = kAttnBN;

template <int DQK, int DV, bool SEP_V>
struct ACfg {
  static constexpr int kQChunks = DQK / 64;
  static constexpr int kVN = DV < 256 ? DV : 256;
  static constexpr int kNVP = DV / kVN;
  static constexpr int kQBytes = kQChunks * 128 * 128;
  static constexpr int kChunkBytes = BN * 128;
  static constexpr int kKVBytes = kQChunks * kChunkBytes;
  static constexpr int kVBytes = SEP_V ? (DV / 64) * kChunkBytes : 0;
  static constexpr int kPBytes = 128 * BN * 2;
  static constexpr int kSCol = kVN;
  static constexpr int kTmemCols = (kVN + BN) <= 128 ? 128 : ((kVN + BN) <= 256 ? 256 : 512);
  static constexpr size_t kSmem = 1024 + kQBytes + 2 * kKVBytes + 2 * kVBytes + kPBytes + 2 * BN * 4 + 80;
};

__device__ __forceinline__ void spin_ns(unsigned long long ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

template <int DQK, int DV, bool SEP_V>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
                const __grid_constant__ CUtensorMap tm_kg, const __grid_constant__ CUtensorMap tm_vt,
                const __grid_constant__ CUtensorMap tm_vg, const AttnArgs a) {
  using C = ACfg<DQK, DV, SEP_V>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sKV = sQ + C::kQBytes;
  uint8_t* sV = sKV + 2 * C::kKVBytes;
  uint8_t* sP = sV + 2 * C::kVBytes;
  int* idx_s = reinterpret_cast<int*>(sP + C::kPBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(idx_s + 2 * BN);
  uint64_t* q_full = bars;
  uint64_t* s_full = bars + 1;
  uint64_t* pv_done = bars + 2;
  uint64_t* kv_full = bars + 3;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int vp = blockIdx.x, split = blockIdx.y, r = blockIdx.z;
  const int b = r / a.T;
  const int h = tid;

  const int nblk_total = (a.k + BN - 1) / BN;
  const int blk0 = split * a.blocks_per_split;
  const int nblk = max(0, min(a.blocks_per_split, nblk_total - blk0));
  const int* idx_row = a.idx + static_cast<long long>(r) * a.k;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(pv_done, 1);
    mbar_init(&kv_full[0], 1);
    mbar_init(&kv_full[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();   // inputs may come from the previous kernel in the stream
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tO = tmem;
  const uint32_t tS = tmem + C::kSCol;

  if (tid == 0 && nblk > 0) {
    prefetch_tmap(&tm_q);
    mbar_arrive_expect_tx(q_full, C::kQBytes);
    for (int c = 0; c < C::kQChunks; ++c) tma_load_2d(sQ + c * 16384, &tm_q, q_full, c * 64, r * a.Hq);
  }

  // Gathers run on TMA, issued by warp 0: lane j holds entry j of the next
  // block's indices (prefetched one block ahead). A block of 32 consecutive
  // valid rows (the sink and window parts of a streaming index set) loads as
  // tiled boxes; any other block as tile::gather4 row gathers (4 rows each).
  // Invalid entries gather row 0 of the sequence (finite; masked in the softmax).
  auto idx_at = [&](int blk) -> int {
    const int ip = (blk0 + blk) * BN + tid;
    int id = (blk < nblk && ip < a.k) ? __ldg(idx_row + ip) : -1;
    if (id >= a.L_max) {   // out of range: skipped, and flagged in the status word
      record_bad_index(a.status);
      id = -1;
    }
    return id;
  };
  int idx_reg = tid < BN ? idx_at(0) : -1;
  constexpr uint32_t kBlockBytes = BN * (DQK + (SEP_V ? DV : 0)) * 2;
  auto load_block = [&](int blk, int buf) {
    if (warp == 0) {
      const int id = idx_reg;
      idx_s[buf * BN + tid] = id;
      idx_reg = idx_at(blk + 1);
      const int id0 = __shfl_sync(0xffffffffu, id, 0);
      const bool contiguous = __all_sync(0xffffffffu, id0 >= 0 && id == id0 + tid);
      const int row0 = b * a.L_max;
      const int y = row0 + (id >= 0 ? id : 0);
      int ys[BN];
#pragma unroll
      for (int j = 0; j < BN; ++j) ys[j] = __shfl_sync(0xffffffffu, y, j);
      if (tid == 0) {
        mbar_arrive_expect_tx(&kv_full[buf], kBlockBytes);
        uint8_t* kv = sKV + buf * C::kKVBytes;
        uint8_t* vv = sV + buf * C::kVBytes;
        if (contiguous) {
          for (int c = 0; c < C::kQChunks; ++c) tma_load_2d(kv + c * C::kChunkBytes, &tm_kt, &kv_full[buf], c * 64, row0 + id0);
          if (SEP_V)
            for (int c = 0; c < DV / 64; ++c) tma_load_2d(vv + c * C::kChunkBytes, &tm_vt, &kv_full[buf], c * 64, row0 + id0);
        } else {
          for (int c = 0; c < C::kQChunks; ++c)
#pragma unroll
            for (int g = 0; g < BN / 4; ++g)
              tma_gather4(kv + c * C::kChunkBytes + g * 512, &tm_kg, &kv_full[buf], c * 64, ys[4 * g], ys[4 * g + 1],
                          ys[4 * g + 2], ys[4 * g + 3]);
          if (SEP_V)
            for (int c = 0; c < DV / 64; ++c)
#pragma unroll
              for (int g = 0; g < BN / 4; ++g)
                tma_gather4(vv + c * C::kChunkBytes + g * 512, &tm_vg, &kv_full[buf], c * 64, ys[4 * g],
                            ys[4 * g + 1], ys[4 * g + 2], ys[4 * g + 3]);
        }
      }
    }
  };

  const uint32_t idesc_qk = make_idesc(1, 1, 128, BN, 0, 0);
  const uint32_t idesc_pv = make_idesc(1, 1, 128, C::kVN, 0, 1);
  float m_run = -INFINITY, l_run = 0.f;   // log2 domain

  // Failure decisions are block-uniform (__syncthreads_and), so no thread can
  // be left waiting at a barrier the others skipped.
  bool fail = false;
  if (nblk > 0) load_block(0, 0);
  for (int blk = 0; blk < nblk; ++blk) {
    const int buf = blk & 1;
    const bool pv_ok = blk >= 1 ? mbar_wait(pv_done, (blk - 1) & 1, a.status) : true;   // frees buf^1, P and O
    if (!__syncthreads_and(pv_ok)) { fail = true; break; }
    if (blk + 1 < nblk) load_block(blk + 1, buf ^ 1);
    const bool kv_ok = mbar_wait(&kv_full[buf], (blk >> 1) & 1, a.status);
    if (!__syncthreads_and(kv_ok)) { fail = true; break; }
    if (tid == 0) {
      const bool q_ok = blk > 0 || mbar_wait(q_full, 0, a.status);
      if (!q_ok) {
        *abort_flag = 1;
      } else {
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sKV + buf * C::kKVBytes);
#pragma unroll 1
        for (int c = 0; c < C::kQChunks; ++c) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = make_sdesc(q0 + c * 16384 + ks * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = make_sdesc(k0 + c * C::kChunkBytes + ks * 32, 16, 1024, kLayoutSW128);
            umma_f16(tS, ad, bd, idesc_qk, (c | ks) ? 1u : 0u);
          }
        }
        umma_commit(s_full);
      }
    }
    __syncthreads();
    if (*abort_flag) { fail = true; break; }
    const bool s_ok = mbar_wait(s_full, blk & 1, a.status);
    if (!__syncthreads_and(s_ok)) { fail = true; break; }
    tc_fence_after();

    uint32_t sv[32];
    tmem_ld32(tS + lane_off, sv);
    tmem_ld_wait();
    float x[32];
    float mb = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool valid = idx_s[buf * BN + j] >= 0;
      x[j] = valid ? __uint_as_float(sv[j]) * a.scale_log2 : -INFINITY;
      mb = fmaxf(mb, x[j]);
    }
    const float m_new = fmaxf(m_run, mb);
    const bool move = m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + 8.f);
    float corr = 1.f;
    if (move) {
      corr = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
      l_run *= corr;
      m_run = m_new;
    }
    // O holds data from earlier blocks: rescale it (warp-uniform TMEM access)
    if (blk > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
      for (int c0 = 0; c0 < C::kVN; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32(tO + lane_off + c0, ov);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
        tmem_st32(tO + lane_off + c0, ov);
      }
      tmem_st_wait();
    }
    float psum = 0.f;
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float p0 = m_run == -INFINITY ? 0.f : exp2f(x[j] - m_run);
      const float p1 = m_run == -INFINITY ? 0.f : exp2f(x[j + 1] - m_run);
      psum += p0 + p1;
      const __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
      pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&v2);
    }
    l_run += psum;
    uint8_t* prow = sP + (h >> 3) * 512 + (h & 7) * 16;
#pragma unroll
    for (int kc = 0; kc < 4; ++kc)
      *reinterpret_cast<uint4*>(prow + kc * 128) = make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t p0 = smem_u32(sP);
      const uint32_t v0 = SEP_V ? smem_u32(sV + buf * C::kVBytes)
                                : smem_u32(sKV + buf * C::kKVBytes) + vp * (C::kVN / 64) * C::kChunkBytes;
#pragma unroll
      for (int ks = 0; ks < BN / 16; ++ks) {
        const uint64_t ad = make_sdesc(p0 + ks * 256, 128, 512, kLayoutNone);
        const uint64_t bd = make_sdesc(v0 + ks * 2048, C::kChunkBytes, 1024, kLayoutSW128);
        umma_f16(tO, ad, bd, idesc_pv, (blk > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(pv_done);
    }
  }
  {
    const bool last_ok = (!fail && nblk > 0) ? mbar_wait(pv_done, (nblk - 1) & 1, a.status) : true;
    if (!__syncthreads_and(last_ok)) fail = true;
  }
  if (fail && tid == 0) *abort_flag = 1;
  __syncthreads();
  tc_fence_after();

  const bool have = nblk > 0 && !*abort_flag;
  const bool write_row = h < a.Hq;
  if (a.n_split == 1) {
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    uint16_t* orow = a.out + (static_cast<long long>(r) * a.Hq + h) * DV + vp * C::kVN;
#pragma unroll 1
    for (int c0 = 0; c0 < C::kVN; c0 += 32) {
      uint32_t ov[32];
      if (have) {
        tmem_ld32(tO + lane_off + c0, ov);
        tmem_ld_wait();
      }
      if (write_row) {
        uint32_t pkd[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float o0 = have ? __uint_as_float(ov[i]) * inv_l : 0.f;
          const float o1 = have ? __uint_as_float(ov[i + 1]) * inv_l : 0.f;
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(o0, o1);
          pkd[i >> 1] = *reinterpret_cast<const uint32_t*>(&v2);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pkd[4 * q], pkd[4 * q + 1], pkd[4 * q + 2], pkd[4 * q + 3]);
      }
    }
    if (vp == 0 && write_row && a.lse)
      a.lse[static_cast<long long>(r) * a.Hq + h] =
          l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
  } else {
    const long long prow = (static_cast<long long>(r) * a.n_split + split) * a.Hq + h;
    uint16_t* po = a.part_o + prow * DV + vp * C::kVN;
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < C::kVN; c0 += 32) {
      uint32_t ov[32];
      if (have) {
        tmem_ld32(tO + lane_off + c0, ov);
        tmem_ld_wait();
      }
      if (write_row) {
        uint32_t pkd[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float o0 = have ? __uint_as_float(ov[i]) * inv_l : 0.f;
          const float o1 = have ? __uint_as_float(ov[i + 1]) * inv_l : 0.f;
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(o0, o1);
          pkd[i >> 1] = *reinterpret_cast<const uint32_t*>(&v2);
        }
        uint4* dst = reinterpret_cast<uint4*>(po + c0);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pkd[4 * q], pkd[4 * q + 1], pkd[4 * q + 2], pkd[4 * q + 3]);
      }
    }
    if (vp == 0 && write_row) {
      a.part_m[prow] = have ? m_run : -INFINITY;
      a.part_l[prow] = have ? l_run : 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) spin_ns(50000);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// MLA decode (d_qk = 576, d_v = 512): one CTA pair (a cluster of 2) per (KV
// split, query row). The pair splits the q.K contraction: CTA 0 holds q
// columns [0, 320) and CTA 1 columns [320, 576), both in tensor memory (the A
// operand of the score MMA, so q is never re-read from shared memory). Each
// CTA loads five 64-column chunks of every gathered KV row (CTA 0 columns
// [0, 320), CTA 1 columns [256, 576)), computes a partial score block, sends
// it to its partner through distributed shared memory (one bulk copy per
// block, counted on the partner's mbarrier) and adds the partner's: both CTAs
// then hold the same
// scores (fp32 addition commutes), run the same online softmax and each
// accumulates its half of the output columns (O += P V over 256 of the 512
// latent columns, with P in tensor memory as the MMA A operand).
//
// Roles (352 threads):
//   warps 0, 10 TMA producers, each for half of every block (rows 0-31 and
//               32-63): index entries (prefetched one ring ahead) -> validity
//               mask, tiled boxes for contiguous runs, tile::gather4 row
//               gathers otherwise, into a kStages-deep ring of 64-row blocks.
//               Two warps issue the 80 gather operations of a block: measured
//               on B200, one issuing warp is what limits a random-row gather
//               (3.2 us per 64-row block against 2.2 us with two)
//   warp 1      TMEM owner; lane 0 issues QK(b) then PV(b - 1)
//   warps 2..9  softmax: two threads per head, each on 32 of a block's 64
//               columns. Software-pipelined: the partial scores of block b + 1
//               go to the partner before block b's softmax runs, so the
//               exchange latency hides behind a whole iteration. The two
//               threads of a head agree on the block max through a tagged
//               shared-memory slot (bounded wait, no block-wide barrier).
namespace mla {
constexpr int kThreads = 352;
constexpr int kSoftThreads = 256;
constexpr int kProducer2 = 10;                      // the second producer warp
constexpr int BN = 64;                              // KV rows per block
constexpr int kStages = 3;
constexpr int kChunks = 5;                          // 64-column chunks per CTA and block
constexpr int kChunkBytes = BN * 128;
constexpr int kStageBytes = kChunks * kChunkBytes;
constexpr int kXBytes = 128 * BN * 4;               // exchange rows of 256 B, 16-byte units XOR-swizzled by row
constexpr int kXTotalBytes = 128 * BN * 4;          // bytes the partner sends per block
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352;
constexpr int kOffX = kStages * kStageBytes;        // [2] receive buffers
constexpr int kOffSend = kOffX + 2 * kXBytes;       // outgoing partial scores (same layout)
constexpr int kOffTag = kOffSend + kXBytes;         // [2][2][128] u64 tagged max slots + [2][128] u64 sums
constexpr int kOffMask = kOffTag + (4 * 128 + 2 * 128) * 8;
constexpr int kOffKScale = kOffMask + kStages * 8;   // e4m3 KV: [kStages][BN] token scales of the staged rows
constexpr int kOffBars = kOffKScale + kStages * BN * 4;
constexpr int kNumBars = 2 * kStages + 13;
constexpr int kOffMisc = kOffBars + kNumBars * 8;
constexpr size_t kSmem = 1024 + kOffMisc + 16;
static_assert(kOffBars % 8 == 0, "mbarriers need 8-byte alignment");
static_assert(kSmem <= 227 * 1024, "shared memory budget");
static_assert(kStageBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");

// Bounded wait that also gives up when another thread of the CTA has aborted.
template <bool CLUSTER>
__device__ __forceinline__ bool wait_ph(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  auto probe = [&] { return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (probe()) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (probe()) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      record_timeout(status);
      *abort_flag = 1;
      return false;
    }
  }
}

// Publish (tag, value) in a shared slot; read the partner's slot once its tag
// matches. Bounded like the barrier waits.
__device__ __forceinline__ void put_tagged(volatile unsigned long long* slot, uint32_t tag, float v) {
  *slot = (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
}
__device__ __forceinline__ bool get_tagged(const volatile unsigned long long* slot, uint32_t tag, float* v,
                                           int* status, volatile int* abort_flag) {
  unsigned long long x = *slot;
  if (static_cast<uint32_t>(x >> 32) != tag) {
    const unsigned long long t0 = globaltimer_ns();
    while (static_cast<uint32_t>((x = *slot) >> 32) != tag) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_timeout(status);
        *abort_flag = 1;
        return false;
      }
    }
  }
  *v = __uint_as_float(static_cast<uint32_t>(x));
  return true;
}

// K/V tile and row-gather maps and q maps of every layer of a launch.
struct MapSet {
  CUtensorMap kt[kMaxLaunchLayers], kg[kMaxLaunchLayers], q[kMaxLaunchLayers];
};

// e4m3 pair -> bf16 pair, exact (every e4m3 value is a bf16 value): through
// the paired e4m3 -> f16 conversion and fp32. (A bit-level f16 -> bf16 step
// measured slower: the staging is bound by instruction issue.)
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two_codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two_codes)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// KV8: the latent rows are e4m3 codes with a per-token scale. The producer
// threads stage each block's codes as bf16 (exact) in the same swizzled tiles
// and the token scales beside them; the softmax multiplies each score column
// by its token's scale, and P by it before the PV product (V = code * scale).
template <bool KV8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_pair_kernel(const __grid_constant__ MapSet maps, const __grid_constant__ LayerOuts lo, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sStage = base;
  uint8_t* sX = base + kOffX;
  uint8_t* sSend = base + kOffSend;
  volatile unsigned long long* tag_max = reinterpret_cast<volatile unsigned long long*>(base + kOffTag);  // [2][2][128]
  volatile unsigned long long* tag_sum = tag_max + 4 * 128;                                              // [2][128]
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(base + kOffMask);                                       // [kStages][2]
  float* kscale_s = reinterpret_cast<float*>(base + kOffKScale);                                         // [kStages][BN]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* pv_done = p_full + 1;
  uint64_t* x_full = pv_done + 1;     // [2]
  uint64_t* q_ready = x_full + 2;
  uint64_t* send_full = q_ready + 1;  // the outgoing buffer is written
  uint64_t* send_free = send_full + 1;  // the bulk copy has read it
  uint64_t* q_full = send_free + 1;     // q chunks staged in shared memory
  uint64_t* x_free = q_full + 1;        // [2] the partner has read what this CTA sent into its buffer i
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  // z = split * layers + layer: splits outermost, so the streaming-prefix splits of all layers launch first
  const int layer = static_cast<int>(blockIdx.z) % lo.n;
  const int r = blockIdx.y, split = static_cast<int>(blockIdx.z) / lo.n;
  const LayerOut& Lo = lo.l[layer];
  const CUtensorMap* tm_kt = &maps.kt[layer];
  const CUtensorMap* tm_kg = &maps.kg[layer];
  const CUtensorMap* tm_q = &maps.q[layer];
  const int b = r / a.T;
  const int chunk0 = rank ? 4 : 0;        // global 64-column chunk of local chunk 0
  const int nq = rank ? 4 : 5;            // q chunks held (and score chunks multiplied)
  const int qk_local0 = rank ? 1 : 0;     // local chunk of the first score chunk
  const int q_chunk0 = rank ? 5 : 0;

  const int nblk_total = (a.k + BN - 1) / BN;
  const bool prefix_split = split < a.fixed_splits;
  const int blk0 = prefix_split ? split * a.bps_fixed
                                : a.fixed_blocks + (split - a.fixed_splits) * a.blocks_per_split;
  const int nblk = max(0, prefix_split ? min(a.bps_fixed, a.fixed_blocks - blk0)
                                       : min(a.blocks_per_split, nblk_total - blk0));
  const int* idx_row = a.idx + static_cast<long long>(r) * a.k;
  // Streaming prefix: with the layout promise, a split whose entries all lie
  // in the row's sink + window prefix computes them (sink s at entry s, window
  // token w_lo + j at entry sink_end + j) and never reads idx, so it need not
  // wait for the kernel that writes the rest of the row.
  bool fixed = false;
  int f_sink_end = 0, f_wlo = 0;
  if (a.stream_sink + a.stream_window > 0 && nblk > 0) {
    int L = __ldg(a.seq_len + b);
    L = L < 0 ? 0 : (L > a.L_max ? a.L_max : L);
    const int pos = L - a.T + (r - b * a.T);
    if (pos >= 0) {
      f_sink_end = min(a.stream_sink, pos + 1);
      f_wlo = max(f_sink_end, pos - a.stream_window + 1);
      const int n_fixed = f_sink_end + (pos + 1 - f_wlo);
      fixed = min(a.k, (blk0 + nblk) * BN) <= n_fixed;
    }
  }

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], KV8 ? 64 : 2);   // KV8: every producer thread; else one expect_tx arrive per warp
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftThreads);
    mbar_init(p_full, kSoftThreads);
    mbar_init(pv_done, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&x_full[i], 1);   // own expect_tx arrive + the partner's copy bytes
    mbar_init(q_ready, kSoftThreads);
    mbar_init(send_full, kSoftThreads);
    mbar_init(send_free, 1);
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&x_free[i], 1);   // the partner's MMA issuer, remotely
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < 6 * 128; i += kThreads) tag_max[i] = 0ull;   // tags start at 0 (never a live tag)
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();   // the partner's barriers are initialised before any remote arrive
  // The index rows come from the previous kernel in the stream. The last cluster
  // waits in any case, so this grid never completes before that kernel does.
  if (!fixed || (blockIdx.y == gridDim.y - 1 && blockIdx.z == gridDim.z - 1)) pdl_wait();
  pdl_trigger();
  // Second cluster phase: q is staged in the exchange buffers, so the partner
  // may copy scores into them only after this CTA has moved q into TMEM. The
  // softmax threads arrive after that move and wait before their first send;
  // the other warps never touch those buffers and arrive right away.
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + kColO, tQ = tmem + kColQ, tS = tmem + kColS, tP = tmem + kColP;

  if (warp == 0 || warp == kProducer2) {
    // ----------------------------------------------------------- producers --
    const int part = warp == 0 ? 0 : 1;   // rows [32 part, 32 part + 32) of every block
    if (part == 0 && lane == 0) {
      // q rows [r Hq, r Hq + 128) x this CTA's chunks, 128-byte swizzled, into the exchange buffers
      mbar_arrive_expect_tx(q_full, nq * 16384);
      for (int j = 0; j < nq; ++j) tma_load_2d(sX + j * 16384, tm_q, q_full, (q_chunk0 + j) * 64, r * a.Hq);
    }
    __syncwarp();
    cluster_arrive_release();
    if (!KV8) {   // e4m3 KV: no K tensor maps (the rows are staged by these threads)
      prefetch_tmap(tm_kt);
      prefetch_tmap(tm_kg);
    }
    const int row0 = b * a.L_max;
    // index entry e of block `bb`, -1 outside the split / row
    auto load_id = [&](int bb, int e) -> int {
      const int ip = (blk0 + bb) * BN + e;
      if (bb >= nblk || ip >= a.k) return -1;
      if (fixed) return ip < f_sink_end ? ip : f_wlo + (ip - f_sink_end);
      const int v = __ldg(idx_row + ip);
      if (v >= a.L_max) {   // out of range: skipped, and flagged in the status word
        record_bad_index(a.status);
        return -1;
      }
      return v;
    };
    int ids_lo[kStages], ids_hi[kStages];   // entries lane and lane + 32 of the next kStages blocks
#pragma unroll
    for (int j = 0; j < kStages; ++j) {
      ids_lo[j] = load_id(j, lane);
      ids_hi[j] = load_id(j, lane + 32);
    }
    bool run = true;
    for (int g = 0; run && g < nblk; g += kStages) {
#pragma unroll
      for (int j = 0; j < kStages; ++j) {
        const int blk = g + j;
        if (blk >= nblk) {
          run = false;
          break;
        }
        if (blk >= kStages) {
          const bool ok = wait_ph<false>(&kv_empty[j], ((blk / kStages) - 1) & 1, a.status, abort_flag);
          if (!__all_sync(0xffffffffu, ok)) {
            run = false;
            break;
          }
        }
        const int id_lo = ids_lo[j], id_hi = ids_hi[j];
        ids_lo[j] = load_id(blk + kStages, lane);
        ids_hi[j] = load_id(blk + kStages, lane + 32);
        const uint32_t valid_lo = __ballot_sync(0xffffffffu, id_lo >= 0);
        const uint32_t valid_hi = __ballot_sync(0xffffffffu, id_hi >= 0);
        const int id0 = __shfl_sync(0xffffffffu, id_lo, 0);
        const bool contiguous =
            __all_sync(0xffffffffu, id0 >= 0 && id_lo == id0 + lane && id_hi == id0 + 32 + lane);
        if constexpr (KV8) {
          // this lane's row of the block, 320 codes of it (this CTA's columns),
          // staged as bf16 in the swizzled tile; invalid entries stage row 0 of
          // the sequence (finite, masked out) with scale 0
          const int id = part == 0 ? id_lo : id_hi;
          const int row = 32 * part + lane;
          const int y = id >= 0 ? id : 0;
          if (lane == 0 && part == 0) {
            mask_s[2 * j] = valid_lo;
            mask_s[2 * j + 1] = valid_hi;
          }
          kscale_s[j * BN + row] = id >= 0 ? __ldg(Lo.k_scale + row0 + y) : 0.f;
          const uint4* src = reinterpret_cast<const uint4*>(Lo.kv8 + static_cast<long long>(row0 + y) * Lo.kv8_stride +
                                                            chunk0 * 64);
          uint8_t* trow = sStage + j * kStageBytes + row * 128;
          const int swz = row & 7;
          // all 20 loads in flight first (the shared-memory stores below would
          // otherwise keep the compiler from hoisting them), then convert
          uint4 v[kChunks * 4];
#pragma unroll
          for (int i = 0; i < kChunks * 4; ++i) v[i] = __ldg(src + i);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {   // codes 16q .. 16q + 15 of chunk c -> bf16 units 2q, 2q + 1
              const uint4 e = v[4 * c + q];
              const uint4 u0 = make_uint4(e4m3x2_to_bf16x2(e.x), e4m3x2_to_bf16x2(e.x >> 16), e4m3x2_to_bf16x2(e.y),
                                          e4m3x2_to_bf16x2(e.y >> 16));
              const uint4 u1 = make_uint4(e4m3x2_to_bf16x2(e.z), e4m3x2_to_bf16x2(e.z >> 16), e4m3x2_to_bf16x2(e.w),
                                          e4m3x2_to_bf16x2(e.w >> 16));
              *reinterpret_cast<uint4*>(trow + c * kChunkBytes + (((2 * q) ^ swz) << 4)) = u0;
              *reinterpret_cast<uint4*>(trow + c * kChunkBytes + (((2 * q + 1) ^ swz) << 4)) = u1;
            }
          }
          fence_proxy_async_smem();   // generic-proxy stores, read by the tensor cores
          mbar_arrive(&kv_full[j]);
          continue;
        }
        const int y_mine = row0 + (part == 0 ? (id_lo >= 0 ? id_lo : 0) : (id_hi >= 0 ? id_hi : 0));
        int yg[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)   // lane g < 8 gathers block rows 32 part + 4g .. + 3
          yg[q] = __shfl_sync(0xffffffffu, y_mine, (4 * lane + q) & 31);
        if (lane == 0) {
          if (part == 0) {
            mask_s[2 * j] = valid_lo;
            mask_s[2 * j + 1] = valid_hi;
          }
          mbar_arrive_expect_tx(&kv_full[j], kStageBytes / 2);
        }
        __syncwarp();
        uint8_t* st = sStage + j * kStageBytes;
        if (contiguous) {
          if (lane < kChunks)   // one 32-row box per chunk
            tma_load_2d(st + lane * kChunkBytes + part * (kChunkBytes / 2), tm_kt, &kv_full[j],
                        (chunk0 + lane) * 64, row0 + id0 + 32 * part);
        } else if (lane < BN / 8) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
            tma_gather4(st + c * kChunkBytes + (8 * part + lane) * 512, tm_kg, &kv_full[j], (chunk0 + c) * 64,
                        yg[0], yg[1], yg[2], yg[3]);
        }
      }
    }
    cluster_wait_acquire();
  } else if (warp == 1) {
    cluster_arrive_release();
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0 && nblk > 0) {
      const uint32_t idesc_qk = make_idesc(1, 1, 128, BN, 0, 0);
      const uint32_t idesc_pv = make_idesc(1, 1, 128, 256, 0, 1);
      const uint32_t peer_xfree = mapa_shared(smem_u32(x_free), peer);
      auto issue_pv = [&](int pb) -> bool {
        if (!wait_ph<false>(p_full, pb & 1, a.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sStage + (pb % kStages) * kStageBytes);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t bd = make_sdesc(vb + ks * 2048, kChunkBytes, 1024, kLayoutSW128);
          umma_f16_ts(tO, tP + ks * 8, bd, idesc_pv, (pb > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(pv_done);
        umma_commit(&kv_empty[pb % kStages]);
        // P(pb) is stored, so every softmax thread has read block pb's partial
        // scores from exchange buffer pb & 1: the partner may copy block pb + 2
        // into it (a cumulative release of what p_full acquired)
        mbar_arrive_remote(peer_xfree + (pb & 1) * 8);
        return true;
      };
      bool ok = wait_ph<false>(q_ready, 0, a.status, abort_flag);
      for (int blk = 0; ok && blk < nblk; ++blk) {
        const int s = blk % kStages;
        ok = wait_ph<false>(&kv_full[s], (blk / kStages) & 1, a.status, abort_flag);
        if (ok && blk >= 1) ok = wait_ph<false>(s_free, (blk - 1) & 1, a.status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(sStage + s * kStageBytes);
#pragma unroll 1
        for (int j = 0; j < nq; ++j) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bd = make_sdesc(kb + (qk_local0 + j) * kChunkBytes + ks * 32, 16, 1024, kLayoutSW128);
            umma_f16_ts(tS, tQ + j * 32 + ks * 8, bd, idesc_qk, (j | ks) ? 1u : 0u);
          }
        }
        umma_commit(s_full);
        if (blk >= 1) ok = issue_pv(blk - 1);
      }
      if (ok) issue_pv(nblk - 1);
    }
    __syncwarp();
    cluster_wait_acquire();
  } else {
    // ------------------------------------------------- softmax / epilogue --
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;            // columns [32 half, 32 half + 32) of a block
    const int h = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    // q row h -> TMEM columns (two bf16 per column, k ascending) from the
    // swizzled staging tiles; the two threads of a head take alternate chunks.
    // Rows h >= Hq hold finite values of other rows (or zeros) and are never written out.
    ok = __all_sync(0xffffffffu, wait_ph<false>(q_full, 0, a.status, abort_flag));
    if (ok) {
#pragma unroll
      for (int jj = 0; jj < 3; ++jj) {
        const int j = 2 * jj + half;
        if (j < nq) {
          const uint4* row = reinterpret_cast<const uint4*>(sX + j * 16384 + h * 128);
          uint32_t v[32];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const uint4 w = row[t ^ (h & 7)];
            v[4 * t] = w.x;
            v[4 * t + 1] = w.y;
            v[4 * t + 2] = w.z;
            v[4 * t + 3] = w.w;
          }
          tmem_st32(tQ + lane_base + j * 32, v);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    cluster_arrive_release();   // this CTA's exchange buffers are free
    cluster_wait_acquire();     // and so are the partner's
    const uint32_t col_off = static_cast<uint32_t>(half * 32);
    const int swz = h & 7;   // unit t of this thread's half-row sits at unit t ^ swz
    const uint32_t peer_x = mapa_shared(smem_u32(sX), peer);
    const uint32_t peer_xfull = mapa_shared(smem_u32(x_full), peer);
    const bool leader = h == 0 && half == 0;
    uint4* send_row = reinterpret_cast<uint4*>(sSend + h * (BN * 4) + half * 128);
    // Partial scores of block bb: TMEM -> registers, free S, stage them in the
    // outgoing buffer; the leader ships the whole block with one bulk copy.
    auto fetch_send = [&](int bb, uint32_t (&sv)[32]) -> bool {
      if (!__all_sync(0xffffffffu, wait_ph<false>(s_full, bb & 1, a.status, abort_flag))) return false;
      tc_fence_after();
      tmem_ld32(tS + lane_base + col_off, sv);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free);
      if (bb >= 1) {
        if (leader) {
          bulk_wait_read();   // the previous block's copy has read the outgoing buffer
          mbar_arrive(send_free);
        }
        if (!__all_sync(0xffffffffu, wait_ph<false>(send_free, (bb - 1) & 1, a.status, abort_flag))) return false;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) send_row[t ^ swz] = make_uint4(sv[4 * t], sv[4 * t + 1], sv[4 * t + 2], sv[4 * t + 3]);
      fence_proxy_async_smem();
      mbar_arrive(send_full);
      const int i = bb & 1;
      bool lok = true;
      if (leader) {
        mbar_arrive_expect_tx(&x_full[i], kXTotalBytes);
        lok = wait_ph<false>(send_full, bb & 1, a.status, abort_flag);
        // the partner's buffer i still holds block bb - 2 until its readers have
        // signalled (remote arrivals on this CTA's x_free[i])
        if (lok && bb >= 2) lok = wait_ph<true>(&x_free[i], ((bb - 2) >> 1) & 1, a.status, abort_flag);
        if (lok) {
          bulk_copy_to_peer(peer_x + i * kXBytes, sSend, kXBytes, peer_xfull + i * 8);
          bulk_commit();
        }
      }
      return __all_sync(0xffffffffu, lok);   // warp-uniform outcome
    };
    float m_run = -INFINITY, l_part = 0.f;   // log2 domain; l_part: this thread's columns
    uint32_t sv_cur[32], sv_nxt[32];
    if (ok && nblk > 0) ok = fetch_send(0, sv_cur);
    for (int blk = 0; ok && blk < nblk; ++blk) {
      const int s = blk % kStages, i = blk & 1;
      // Block blk + 1's partial leaves before block blk's softmax: the
      // partner's reply then has a whole iteration to arrive. The partner has
      // finished reading its buffer (blk + 1) & 1 (block blk - 1) before it
      // sent block blk, which this thread receives below only after sending:
      // ordering comes from the previous iteration's receive.
      if (blk + 1 < nblk) {
        ok = fetch_send(blk + 1, sv_nxt);
        if (!ok) break;
      }
      ok = __all_sync(0xffffffffu, wait_ph<true>(&x_full[i], (blk >> 1) & 1, a.status, abort_flag));
      if (!ok) break;
      float x[32];
      {
        const float4* src = reinterpret_cast<const float4*>(sX + i * kXBytes + h * (BN * 4) + half * 128);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float4 w = src[t ^ swz];
          x[4 * t] = __uint_as_float(sv_cur[4 * t]) + w.x;
          x[4 * t + 1] = __uint_as_float(sv_cur[4 * t + 1]) + w.y;
          x[4 * t + 2] = __uint_as_float(sv_cur[4 * t + 2]) + w.z;
          x[4 * t + 3] = __uint_as_float(sv_cur[4 * t + 3]) + w.w;
        }
      }
      ok = __all_sync(0xffffffffu, wait_ph<false>(&kv_full[s], (blk / kStages) & 1, a.status, abort_flag));
      if (!ok) break;
      const uint32_t valid = mask_s[2 * s + half];
      const float4* ks4 = reinterpret_cast<const float4*>(kscale_s + s * BN + 32 * half);   // KV8: token scales
      float mloc[8];
      if constexpr (KV8) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float4 k4 = ks4[t];
          const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * t + e;
            x[j] = ((valid >> j) & 1u) ? x[j] * kk[e] * Lo.scale_log2 : -INFINITY;
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = ((valid >> j) & 1u) ? x[j] * Lo.scale_log2 : -INFINITY;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) mloc[t] = fmaxf(fmaxf(x[4 * t], x[4 * t + 1]), fmaxf(x[4 * t + 2], x[4 * t + 3]));
      const float mb_mine = fmaxf(fmaxf(fmaxf(mloc[0], mloc[1]), fmaxf(mloc[2], mloc[3])),
                                  fmaxf(fmaxf(mloc[4], mloc[5]), fmaxf(mloc[6], mloc[7])));
      // the other half of the row's block max (tag = block + 1)
      put_tagged(tag_max + (i * 2 + half) * 128 + h, static_cast<uint32_t>(blk + 1), mb_mine);
      float mb_other;
      ok = __all_sync(0xffffffffu, get_tagged(tag_max + (i * 2 + (half ^ 1)) * 128 + h, static_cast<uint32_t>(blk + 1),
                                              &mb_other, a.status, abort_flag));
      if (!ok) break;
      const float mb = fmaxf(mb_mine, mb_other);
      const float m_new = fmaxf(m_run, mb);
      const bool move = m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + 8.f);
      float corr = 1.f;
      if (move) {
        corr = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
        l_part *= corr;
        m_run = m_new;
      }
      if (__any_sync(0xffffffffu, move && blk > 0)) {
        // O holds earlier blocks: rescale this thread's 128 columns once PV(blk - 1) has landed
        ok = __all_sync(0xffffffffu, wait_ph<false>(pv_done, (blk - 1) & 1, a.status, abort_flag));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + lane_base + c0, ov);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) ov[t] = __float_as_uint(__uint_as_float(ov[t]) * corr);
          tmem_st32(tO + lane_base + c0, ov);
        }
        tmem_st_wait();
      }
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float p0 = m_run == -INFINITY ? 0.f : exp2f(x[j] - m_run);
        const float p1 = m_run == -INFINITY ? 0.f : exp2f(x[j + 1] - m_run);
        ps[(j >> 1) & 3] += p0 + p1;
        float w0 = p0, w1 = p1;
        if constexpr (KV8) {   // V row = code * scale: the scale rides on P
          const float2 k2 = reinterpret_cast<const float2*>(ks4)[j >> 1];
          w0 *= k2.x;
          w1 *= k2.y;
        }
        const __nv_bfloat162 v2 = __floats2bfloat162_rn(w0, w1);
        pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&v2);
      }
      l_part += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      // P lives in TMEM (one block): free once PV(blk - 1) has completed
      if (blk >= 1) {
        ok = __all_sync(0xffffffffu, wait_ph<false>(pv_done, (blk - 1) & 1, a.status, abort_flag));
        if (!ok) break;
      }
      tc_fence_after();
      tmem_st16(tP + lane_base + half * 16, pk);   // keys [32 half, 32 half + 32) of row h
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
#pragma unroll
      for (int t = 0; t < 32; ++t) sv_cur[t] = sv_nxt[t];
    }
    if (ok && nblk > 0)
      ok = __all_sync(0xffffffffu, wait_ph<false>(pv_done, (nblk - 1) & 1, a.status, abort_flag));
    // row sum over both halves (fixed order: both threads get the same value)
    float l_run = 0.f;
    if (ok) {
      put_tagged(tag_sum + half * 128 + h, 0xFFFFFFFFu, l_part);
      float l_other;
      ok = __all_sync(0xffffffffu, get_tagged(tag_sum + (half ^ 1) * 128 + h, 0xFFFFFFFFu, &l_other, a.status,
                                              abort_flag));
      l_run = half == 0 ? l_part + l_other : l_other + l_part;
    }
    // ---- epilogue: this thread's 128 output columns, staged per warp for coalesced stores
    if (ok) {
      tc_fence_after();
      const bool have = nblk > 0;
      const bool final_out = a.n_split == 1;
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      float* tile = reinterpret_cast<float*>(sX) + (warp - 2) * 32 * 36;   // [32 rows][36]
#pragma unroll 1
      for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
        uint32_t ov[32];
        if (have) {
          tmem_ld32(tO + lane_base + c0, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) ov[t] = 0u;
        }
        const float f = inv_l;   // final output and split partials are both normalised
        float4* trow = reinterpret_cast<float4*>(tile + lane * 36);
#pragma unroll
        for (int t = 0; t < 8; ++t)
          trow[t] = make_float4(__uint_as_float(ov[4 * t]) * f, __uint_as_float(ov[4 * t + 1]) * f,
                                __uint_as_float(ov[4 * t + 2]) * f, __uint_as_float(ov[4 * t + 3]) * f);
        __syncwarp();
        // 8 rows per instruction, 64 bytes (32 bf16) per row
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int rr = t * 8 + (lane >> 2), seg = lane & 3;
          const int hh = quarter * 32 + rr;
          const float4* srcp = reinterpret_cast<const float4*>(tile + rr * 36 + seg * 8);
          const float4 v0 = srcp[0], v1 = srcp[1];
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(v0.x, v0.y), b1 = __floats2bfloat162_rn(v0.z, v0.w);
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v1.x, v1.y), b3 = __floats2bfloat162_rn(v1.z, v1.w);
          if (hh < a.Hq) {
            const long long orow = final_out ? static_cast<long long>(r) * a.Hq + hh
                                             : (static_cast<long long>(r) * a.n_split + split) * a.Hq + hh;
            uint16_t* dstp = (final_out ? Lo.out : Lo.part_o) + orow * 512 + rank * 256 + c0 + seg * 8;
            *reinterpret_cast<uint4*>(dstp) =
                make_uint4(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1),
                           *reinterpret_cast<const uint32_t*>(&b2), *reinterpret_cast<const uint32_t*>(&b3));
          }
        }
        __syncwarp();
      }
      if (rank == 0 && half == 0 && h < a.Hq) {
        if (final_out) {
          if (Lo.lse)
            Lo.lse[static_cast<long long>(r) * a.Hq + h] =
                l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
        } else {
          const long long prow = (static_cast<long long>(r) * a.n_split + split) * a.Hq + h;
          Lo.part_m[prow] = have ? m_run : -INFINITY;
          Lo.part_l[prow] = have ? l_run : 0.f;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) spin_ns(50000);   // let copies and MMAs in flight land before the exit
  cluster_sync_all();                 // the partner has finished writing into this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch(const AttnMaps* m, const AttnArgs* a, int n, cudaStream_t stream) {
  for (int i = 1; i < n; ++i)
    if (a[i].kv8 != a[0].kv8) return cudaErrorInvalidValue;   // one KV type per launch
  const void* fn = a[0].kv8 ? reinterpret_cast<const void*>(&mla_pair_kernel<true>)
                            : reinterpret_cast<const void*>(&mla_pair_kernel<false>);
  cudaError_t e = set_max_smem(fn, kSmem);
  if (e != cudaSuccess) return e;
  MapSet maps{};
  for (int i = 0; i < n; ++i) {
    maps.kt[i] = m[i].k_tile;
    maps.kg[i] = m[i].k_rows;
    maps.q[i] = m[i].q;
  }
  LayerOuts lo = layer_outs(a, n);
  AttnArgs shared = a[0];
  void* args[] = {&maps, &lo, &shared};
  return launch_pdl(fn, dim3(2, a[0].B * a[0].T, a[0].n_split * n), dim3(kThreads, 1, 1), kSmem, stream, args);
}
}  // namespace mla

// Merge KV-split partials (o_s = O_s / l_s in bf16, with m_s and l_s):
//   f_s = l_s 2^(m_s - m*),  m* = max m_s;  o = sum f_s o_s / sum f_s.
template <int kInFlight>
__global__ void __launch_bounds__(128) combine_kernel(const __grid_constant__ LayerOuts lo, const AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_f[64];
  __shared__ float s_den;
  const int r = blockIdx.x, h = blockIdx.y;
  const LayerOut& Lo = lo.l[blockIdx.z];
  const int ns = a.n_split;
  const long long base = static_cast<long long>(r) * ns * a.Hq + h;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float m[2], l[2];
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int sidx = lane + 32 * q;
      m[q] = -INFINITY;
      l[q] = 0.f;
      if (sidx < ns) {
        const long long i = base + static_cast<long long>(sidx) * a.Hq;
        l[q] = Lo.part_l[i];
        m[q] = l[q] > 0.f ? Lo.part_m[i] : -INFINITY;
      }
      M = fmaxf(M, m[q]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float f = l[q] > 0.f ? l[q] * exp2f(m[q] - M) : 0.f;
      if (lane + 32 * q < 64) s_f[lane + 32 * q] = f;
      den += f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) {
      s_den = den;
      if (Lo.lse) Lo.lse[static_cast<long long>(r) * a.Hq + h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  __syncthreads();
  const int c = threadIdx.x * 4;
  if (c >= a.d_v) return;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (kInFlight <= 4) {
#pragma unroll 4
    for (int sidx = 0; sidx < ns; ++sidx) {
      const float f = s_f[sidx];
      const uint2 o = *reinterpret_cast<const uint2*>(Lo.part_o + (base + static_cast<long long>(sidx) * a.Hq) * a.d_v + c);
      acc[0] = fmaf(__uint_as_float(o.x << 16), f, acc[0]);
      acc[1] = fmaf(__uint_as_float(o.x & 0xFFFF0000u), f, acc[1]);
      acc[2] = fmaf(__uint_as_float(o.y << 16), f, acc[2]);
      acc[3] = fmaf(__uint_as_float(o.y & 0xFFFF0000u), f, acc[3]);
    }
  } else {
    // many splits: their partials are independent loads, kInFlight in flight
    // per thread, then accumulated in split order (the same arithmetic)
    const uint16_t* po = Lo.part_o + base * a.d_v + c;
    const long long sstride = static_cast<long long>(a.Hq) * a.d_v;
    for (int s0 = 0; s0 < ns; s0 += kInFlight) {
      uint2 o[kInFlight];
#pragma unroll
      for (int j = 0; j < kInFlight; ++j)
        o[j] = s0 + j < ns ? *reinterpret_cast<const uint2*>(po + (s0 + j) * sstride) : make_uint2(0u, 0u);
#pragma unroll
      for (int j = 0; j < kInFlight; ++j) {
        if (s0 + j >= ns) break;
        const float f = s_f[s0 + j];
        acc[0] = fmaf(__uint_as_float(o[j].x << 16), f, acc[0]);
        acc[1] = fmaf(__uint_as_float(o[j].x & 0xFFFF0000u), f, acc[1]);
        acc[2] = fmaf(__uint_as_float(o[j].y << 16), f, acc[2]);
        acc[3] = fmaf(__uint_as_float(o[j].y & 0xFFFF0000u), f, acc[3]);
      }
    }
  }
  const float inv = s_den > 0.f ? 1.f / s_den : 0.f;
  const __nv_bfloat162 v01 = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  const __nv_bfloat162 v23 = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&v01);
  pk.y = *reinterpret_cast<const uint32_t*>(&v23);
  *reinterpret_cast<uint2*>(Lo.out + (static_cast<long long>(r) * a.Hq + h) * a.d_v + c) = pk;
}

template <int DQK, int DV, bool SEP_V>
cudaError_t launch_t(const AttnMaps& m, const AttnArgs& a, cudaStream_t stream) {
  using C = ACfg<DQK, DV, SEP_V>;
  const void* fn = reinterpret_cast<const void*>(&attn_kernel<DQK, DV, SEP_V>);
  size_t smem = C::kSmem;
  if (smem < 60 * 1024) smem = 60 * 1024;   // at most 3 CTAs per SM: TMEM demand stays <= 512 columns
  cudaError_t e = set_max_smem(fn, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(C::kNVP, a.n_split, a.B * a.T);
  void* args[] = {const_cast<CUtensorMap*>(&m.q), const_cast<CUtensorMap*>(&m.k_tile),
                  const_cast<CUtensorMap*>(&m.k_rows), const_cast<CUtensorMap*>(&m.v_tile),
                  const_cast<CUtensorMap*>(&m.v_rows), const_cast<AttnArgs*>(&a)};
  return launch_pdl(fn, grid, dim3(kThreads), smem, stream, args);
}

}  // namespace

cudaError_t launch_attn(const AttnMaps* m, const AttnArgs* args, int n, cudaStream_t stream) {
  if (n < 1 || n > kMaxLaunchLayers) return cudaErrorInvalidValue;
  const AttnArgs& a = args[0];
  if (a.d_qk == 576 && a.d_v == 512) {
    for (int i = 0; i < n; ++i)
      if (args[i].sep_v) return cudaErrorNotSupported;   // MLA keeps V inside the latent row
    return mla::launch(m, args, n, stream);
  }
  if (n != 1) return cudaErrorNotSupported;
  if (a.d_qk == 64 && a.d_v == 64) {
    if (a.sep_v) return launch_t<64, 64, true>(m[0], a, stream);
    return launch_t<64, 64, false>(m[0], a, stream);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_attn_combine(const AttnArgs* args, int n, cudaStream_t stream) {
  const AttnArgs& a = args[0];
  if (a.n_split > 64 || n < 1 || n > kMaxLaunchLayers) return cudaErrorInvalidValue;
  LayerOuts lo = layer_outs(args, n);
  AttnArgs shared = a;
  const dim3 grid(a.B * a.T, a.Hq, n);
  void* kargs[] = {&lo, &shared};
  // rows with many splits (few rows on the GPU) take 16 partial loads in flight
  // per thread; many rows keep 4 (registers: the grid is rows x heads CTAs)
  const void* fn = a.n_split >= 24 ? reinterpret_cast<const void*>(&combine_kernel<16>)
                                   : reinterpret_cast<const void*>(&combine_kernel<4>);
  return launch_pdl(fn, grid, dim3(a.d_v / 4 < 32 ? 32 : a.d_v / 4),
                    0, stream, kargs);
}

}  // namespace lsa
