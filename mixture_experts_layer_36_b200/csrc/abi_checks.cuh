// Host-side argument checks shared by the C-ABI entry points (capi.cu and
// permute_noalloc.cu), so that every entry point applies the same limits and
// maps failures to the same status codes.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {
namespace abi {

constexpr int64_t kMaxE = 256;
constexpr int64_t kMaxK = 8;
constexpr int64_t kTileMultiple = 64;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Token / expert / top-k shape: 1 <= E <= kMaxE, 1 <= k <= min(E, kMaxK),
// T >= 0, T*k < 2^31.
inline int check_routing_shape(int64_t T, int64_t E, int64_t k) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E) return MOE_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// A row width (d or f): positive, a multiple of the kernels' tile width.
inline int check_width(int64_t w) {
  if (w < 1) return MOE_ERR_INVALID_ARG;
  if (w % kTileMultiple != 0 || w > (int64_t(1) << 20)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Everything moe_permute checks except its scratch argument, in the same
// order: shape, width, capacity, then (for T > 0) pointers and alignment.
// *C receives the capacity.  Returns MOE_OK, or the code the call returns;
// `done` is set when the call has nothing to do (T == 0).
inline int check_permute_args(const void* x, const int32_t* topk_idx, int64_t T, int64_t d,
                              int64_t E, int64_t k, double cf, const int32_t* counts,
                              const int32_t* offsets, const int32_t* slot,
                              const int32_t* row_src, const void* x_perm,
                              const int32_t* n_dropped, int64_t* C, bool* done) {
  *done = false;
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  *C = moe_capacity(T, E, k, cf);
  if (*C < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) {
    *done = true;
    return MOE_OK;
  }
  if (!x || !topk_idx || !counts || !offsets || !slot || !row_src || !x_perm || !n_dropped)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace abi
}  // namespace moe
