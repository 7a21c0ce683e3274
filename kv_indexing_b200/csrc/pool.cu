// Mean-pooled page keys for Hierarchical Indexing (LSA paper abstract (3) and
// the model card's "HI" bullet: coarse scores over blocks of keys first).
//
//   page_keys[b, p, :] = bf16_rne( (sum_{j<P} k[b, pP + j, :]) / P )
//
// for every full page (pP + P <= seq_len[b]). The sum is fp32 in ascending j
// (one thread per 8 columns of a page, sequential over the page's rows), then
// one correctly rounded division by P, then round-to-nearest-even to bf16 --
// so the stored codes do not depend on thread scheduling. An e4m3 variant
// (below) pools dequantized e4m3 keys into e4m3 page keys with page scales.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace lsa {
namespace {

__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ k, const int* __restrict__ seq_len,
                                                   int L_max, int d, int P, uint16_t* __restrict__ pk) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int vec_per_row = d / 8;   // 16-byte vectors per key row
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int page = static_cast<int>(gid / vec_per_row);
  const int v = static_cast<int>(gid % vec_per_row);
  int L = __ldg(seq_len + b);
  L = L < 0 ? 0 : (L > L_max ? L_max : L);
  if (static_cast<long long>(page + 1) * P > L) return;
  const uint4* src = reinterpret_cast<const uint4*>(k + (static_cast<long long>(b) * L_max + static_cast<long long>(page) * P) * d) + v;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int j = 0; j < P; ++j) {
    const uint4 x = __ldg(src + static_cast<long long>(j) * vec_per_row);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] = __fadd_rn(acc[2 * e], __uint_as_float(w[e] << 16));
      acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], __uint_as_float(w[e] & 0xFFFF0000u));
    }
  }
  const float fP = static_cast<float>(P);
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint16_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(acc[2 * e], fP)));
    const uint16_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(acc[2 * e + 1], fP)));
    o[e] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(pk + (static_cast<long long>(b) * (L_max / P) + page) * d) + v;
  *dst = make_uint4(o[0], o[1], o[2], o[3]);
}

// FP8 page keys (the e4m3 variant of Hierarchical Indexing): one warp per page,
// four columns per lane. A token element is its e4m3 code's value times the
// token's fp32 scale, rounded to fp32; the page mean is the fp32 sum in
// ascending row order divided by P; the page scale is amax / 448 (1 when the
// page is all zero) and each element is stored as e4m3(mean / scale), round to
// nearest even, saturating to the largest finite magnitude. Every rounding is
// explicit (no contraction into fused multiply-adds), so the codes do not
// depend on the compiler.
__global__ void __launch_bounds__(256) pool_e4m3_kernel(const uint8_t* __restrict__ k8, const float* __restrict__ ks,
                                                        const int* __restrict__ seq_len, int L_max, int d, int P,
                                                        uint8_t* __restrict__ pc, float* __restrict__ psc) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int page = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  int L = __ldg(seq_len + b);
  L = L < 0 ? 0 : (L > L_max ? L_max : L);
  if (static_cast<long long>(page + 1) * P > L) return;   // warp-uniform
  const long long row0 = static_cast<long long>(b) * L_max + static_cast<long long>(page) * P;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < P; ++j) {
    const uint32_t c4 = __ldg(reinterpret_cast<const uint32_t*>(k8 + (row0 + j) * d) + lane);
    const float sc = __ldg(ks + row0 + j);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half_raw hv = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>((c4 >> (8 * e)) & 0xFFu), __NV_E4M3);
      acc[e] = __fadd_rn(acc[e], __fmul_rn(__half2float(__half(hv)), sc));
    }
  }
  const float fP = static_cast<float>(P);
  float mean[4], amax = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    mean[e] = __fdiv_rn(acc[e], fP);
    amax = fmaxf(amax, fabsf(mean[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint32_t out = 0u;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    out |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(mean[e], scale), __NV_SATFINITE, __NV_E4M3)) << (8 * e);
  const long long prow = static_cast<long long>(b) * (L_max / P) + page;
  reinterpret_cast<uint32_t*>(pc + prow * d)[lane] = out;
  if (lane == 0) psc[prow] = scale;
}

}  // namespace

cudaError_t launch_pool_e4m3(const uint8_t* k8, const float* k_scale, const int* seq_len, int B, int L_max, int d,
                             int P, uint8_t* page_codes, float* page_scales, cudaStream_t stream) {
  const int pages = L_max / P;
  const int per_block = 8;   // warps (pages) per 256-thread block
  const dim3 grid(static_cast<unsigned>((pages + per_block - 1) / per_block), B);
  void* args[] = {(void*)&k8, (void*)&k_scale, (void*)&seq_len, &L_max, &d, &P, &page_codes, &page_scales};
  return launch_pdl(reinterpret_cast<const void*>(&pool_e4m3_kernel), grid, dim3(256), 0, stream, args);
}

cudaError_t launch_pool(const uint16_t* k, const int* seq_len, int B, int L_max, int d, int P, uint16_t* page_keys,
                        cudaStream_t stream) {
  const long long n = static_cast<long long>(L_max / P) * (d / 8);
  const int threads = 256;
  const dim3 grid(static_cast<unsigned>((n + threads - 1) / threads), B);
  void* args[] = {(void*)&k, (void*)&seq_len, &L_max, &d, &P, &page_keys};
  return launch_pdl(reinterpret_cast<const void*>(&pool_kernel), grid, dim3(threads), 0, stream, args);
}

}  // namespace lsa
