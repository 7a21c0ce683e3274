// Mean-pooled page keys for Hierarchical Indexing (LSA paper abstract (3) and
// the model card's "HI" bullet: coarse scores over blocks of keys first).
//
//   page_keys[b, p, :] = bf16_rne( (sum_{j<P} k[b, pP + j, :]) / P )
//
// for every full page (pP + P <= seq_len[b]). The sum is fp32 in ascending j
// (one thread per 8 columns of a page, sequential over the page's rows), then
// one correctly rounded division by P, then round-to-nearest-even to bf16 --
// so the stored codes do not depend on thread scheduling.
#include <cuda_bf16.h>

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

}  // namespace

cudaError_t launch_pool(const uint16_t* k, const int* seq_len, int B, int L_max, int d, int P, uint16_t* page_keys,
                        cudaStream_t stream) {
  const long long n = static_cast<long long>(L_max / P) * (d / 8);
  const int threads = 256;
  const dim3 grid(static_cast<unsigned>((n + threads - 1) / threads), B);
  void* args[] = {(void*)&k, (void*)&seq_len, &L_max, &d, &P, &page_keys};
  return launch_pdl(reinterpret_cast<const void*>(&pool_kernel), grid, dim3(threads), 0, stream, args);
}

}  // namespace lsa
