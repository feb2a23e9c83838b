// moe_permute_noalloc: the capacity-limited permutation for callers that
// cannot hand the library any scratch memory.
//
// Some callers hold nothing but their input and output buffers: a plugin or
// operator interface that passes only the tensors it declared, or a serving
// runtime that plans every device byte at start-up and fails (or stalls the
// device) on any later cudaMalloc.  They cannot call cudaMalloc themselves and
// cannot give moe_permute its `ws` argument.  This entry point runs the same
// permutation kernels as moe_permute, but their per-chunk bucket counters
// live in a fixed array compiled into the library, so nothing is allocated at
// call time.
//
// Costs and limits of that choice:
//   * the array (kNoAllocScratchInts int32, 257 KiB) is resident on every GPU
//     that loads the library, until the process exits;
//   * it holds (ceil(T/256) + 1) * E counters, so a call needing more is
//     rejected with MOE_ERR_WORKSPACE (E = 256 allows T <= 65536);
//   * every call uses the same array: two calls whose kernels overlap on the
//     GPU (different streams, or different host threads on one device) race
//     and corrupt each other's result.  Serialise them, e.g. on one stream;
//   * the array keeps the previous call's counters.  Nothing needs clearing:
//     the first kernel writes every counter the later ones read.
//   * the first call on each device looks the array's device address up
//     (cudaGetSymbolAddress, with that device current) and caches it; make
//     that first call before any stream capture begins.
#include <mutex>

#include "abi_checks.cuh"
#include "common.cuh"

namespace moe {
cudaError_t launch_permute(const __nv_bfloat16* x, const int32_t* topk_idx, int T, int d, int E,
                           int k, int64_t C, int32_t* counts, int32_t* offsets, int32_t* slot,
                           int32_t* row_src, __nv_bfloat16* x_perm, int32_t* n_dropped,
                           int32_t* chunk_hist, cudaStream_t s, int32_t* status);
size_t permute_scratch_bytes(int64_t T, int64_t E);
}  // namespace moe

namespace {

// 256 rows of 256 experts' chunk counters plus the row of totals
constexpr int64_t kNoAllocScratchInts = 65536 + 256;

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_permute_scratch on the current device (looked up once
// per device).  In host code the symbol itself is only a host-side handle, so
// the kernels must be given this address instead.
cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int moe_permute_noalloc(const void* x, const int32_t* topk_idx, int64_t T, int64_t d,
                                   int64_t E, int64_t k, double cf, int32_t* counts,
                                   int32_t* offsets, int32_t* slot, int32_t* row_src,
                                   void* x_perm, int32_t* n_dropped, int32_t* dev_status,
                                   void* stream) {
  int64_t C = 0;
  bool done = false;
  const int st = moe::abi::check_permute_args(x, topk_idx, T, d, E, k, cf, counts, offsets, slot,
                                              row_src, x_perm, n_dropped, &C, &done);
  if (st != MOE_OK || done) return st;
  if (moe::permute_scratch_bytes(T, E) > size_t(kNoAllocScratchInts) * sizeof(int32_t))
    return MOE_ERR_WORKSPACE;
  int32_t* scratch = nullptr;
  cudaError_t err = scratch_address(&scratch);
  if (err != cudaSuccess) return moe::abi::cuda_status(err);
  return moe::abi::cuda_status(moe::launch_permute(
      static_cast<const __nv_bfloat16*>(x), topk_idx, (int)T, (int)d, (int)E, (int)k, C, counts,
      offsets, slot, row_src, static_cast<__nv_bfloat16*>(x_perm), n_dropped, scratch,
      reinterpret_cast<cudaStream_t>(stream), dev_status));
}
