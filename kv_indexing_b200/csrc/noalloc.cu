// lsa_select_streaming_noalloc: the streaming top-k selection with its scratch
// in a fixed buffer compiled into the library instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where
// they select. A plugin inside a serving engine that has reserved (nearly) all
// HBM for its own KV-cache pool up front has nowhere to cudaMalloc from, and
// code on a latency-critical decode path cannot afford cudaMalloc/cudaFree,
// which may block the host and (cudaFree) synchronise the whole device. This
// entry point allocates nothing: it validates the shape, points the selection
// kernels at the static buffer below and launches them.
//
// The buffer is a file-scope __device__ array, so every GPU on which this
// library's device code is loaded holds LSA_NOALLOC_SCRATCH_BYTES of it until
// the process exits. All calls on a device share it: two calls whose kernels
// overlap on the GPU (different streams, no ordering between them) race on it
// and both results are undefined. The buffer keeps the last call's contents;
// the selection launch clears the parts that must start at zero (the per-row
// counters, release flags and histograms) on the caller's stream every call.
#include <cuda_runtime.h>

#include "internal.h"
#include "lsa.h"

namespace lsa {
namespace {

// Device scratch of the no-allocation selection. In host code this name is a
// host-side stand-in for the symbol, not a device address: never pass it to a
// kernel. The device address comes from cudaGetSymbolAddress (scratch_ptr).
static __device__ __align__(256) unsigned char g_noalloc_scratch[LSA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current device's context, looked
// up with that device current on the first call per device (and again if the
// context changes, e.g. after cudaDeviceReset); the lookup may load this
// library's device code onto the device, so the first call per device belongs
// before any stream capture. nullptr and *err set on failure.
void* scratch_ptr(cudaError_t* err) {
  static SymbolCache cache;
  return symbol_address_cached(&cache, &g_noalloc_scratch, err);
}

}  // namespace
}  // namespace lsa

extern "C" lsa_status_t lsa_select_streaming_noalloc(const float* scores, const int32_t* seq_len, int32_t B,
                                                     int32_t T, int32_t L_max, lsa_budget_t budget, int32_t* idx,
                                                     lsa_stream_t stream) {
  if (B < 1 || T < 1 || L_max < 1)
    return lsa::set_error(LSA_ERR_INVALID_ARG, "B, T and L_max must be >= 1");
  if (static_cast<long long>(B) * T > 65535)
    return lsa::set_error(LSA_ERR_UNSUPPORTED, "at most 65535 query rows per call");
  // scratch this shape needs, from the same plan the selection launch uses
  lsa_op_args_t q{};
  q.budget = budget;
  q.B = B;
  q.T = T;
  q.L_max = L_max;
  size_t need = 0;
  lsa_status_t s = lsa_workspace_size(LSA_OP_SELECT, &q, &need);
  if (s != LSA_OK) return s;
  if (need > LSA_NOALLOC_SCRATCH_BYTES)
    return lsa::set_error(LSA_ERR_WORKSPACE,
                          "lsa_select_streaming_noalloc: B=%d T=%d L_max=%d k=%d needs %zu bytes of scratch; "
                          "the static scratch holds %zu (use lsa_select_streaming with a workspace)",
                          B, T, L_max, budget.k, need, static_cast<size_t>(LSA_NOALLOC_SCRATCH_BYTES));
  cudaError_t e = cudaSuccess;
  void* ws = lsa::scratch_ptr(&e);
  if (!ws)
    return lsa::set_error(LSA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
  return lsa_select_streaming(scores, seq_len, B, T, L_max, budget, idx, ws, LSA_NOALLOC_SCRATCH_BYTES, stream);
}
