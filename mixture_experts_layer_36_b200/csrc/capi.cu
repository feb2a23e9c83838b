// libmoe C ABI: argument validation, capacity and workspace arithmetic, and
// the stage launches.  Every compute step runs in the kernels of router.cu,
// permute.cu, grouped_gemm.cu and combine.cu.
#include <math.h>
#include <nvtx3/nvToolsExt.h>

#include "abi_checks.cuh"
#include "common.cuh"

namespace moe {
cudaError_t launch_route(const __nv_bfloat16* x, const float* wr, const float* bias, int T,
                         int d, int E, int k, float* logits, int32_t* idx, float* w,
                         void* scratch, int32_t* status, cudaStream_t s, bool* map_failed);
size_t route_scratch_bytes(int64_t T, int64_t d, int64_t E);
size_t permute_scratch_bytes(int64_t T, int64_t E);
cudaError_t launch_permute(const __nv_bfloat16* x, const int32_t* topk_idx, int T, int d, int E,
                           int k, int64_t C, int32_t* counts, int32_t* offsets, int32_t* slot,
                           int32_t* row_src, __nv_bfloat16* x_perm, int32_t* n_dropped,
                           int32_t* chunk_hist, cudaStream_t s, int32_t* status);
cudaError_t launch_gate_up(const __nv_bfloat16* a_rows, const int32_t* offsets, int E, int d,
                           int f, int max_rows, const __nv_bfloat16* w_gate,
                           const __nv_bfloat16* w_up, __nv_bfloat16* h, int32_t* status,
                           cudaStream_t s, bool* map_failed, const FuseArgs& fz);
cudaError_t launch_down(const __nv_bfloat16* h, const int32_t* offsets, int E, int d, int f,
                        int max_rows, const __nv_bfloat16* w_down, float* y_perm,
                        int32_t* status, cudaStream_t s, bool* map_failed, const FuseArgs& fz);
cudaError_t launch_finalize(const float* y32, const __nv_bfloat16* x, const int32_t* slot, int T,
                            int d, int k, __nv_bfloat16* y, cudaStream_t s);
cudaError_t launch_combine(const float* y_perm, const __nv_bfloat16* x,
                           const int32_t* topk_idx, const float* topk_w, const int32_t* slot,
                           const int32_t* offsets, int T, int d, int k, __nv_bfloat16* y,
                           cudaStream_t s);
cudaError_t launch_combine_bf16rows(const __nv_bfloat16* y_rows, const __nv_bfloat16* x,
                                    const int32_t* topk_idx, const float* topk_w,
                                    const int32_t* slot, const int32_t* offsets, int T, int d,
                                    int k, __nv_bfloat16* y, cudaStream_t s);
cudaError_t launch_rows_to_bf16(const float* src, __nv_bfloat16* dst, long long n,
                                cudaStream_t s);
cudaError_t launch_permute_rows(const uint8_t* x, int row_bytes, const float* x_scale,
                                const int32_t* topk_idx, int T, int E, int k, int64_t C,
                                int32_t* counts, int32_t* offsets, int32_t* slot,
                                int32_t* row_src, uint8_t* x_perm, float* perm_scale,
                                int32_t* n_dropped, int32_t* chunk_hist, cudaStream_t s,
                                int32_t* row_pair, float* zero_rows, int zero_cols,
                                int32_t* status);
cudaError_t launch_permute_padded(const __nv_bfloat16* x, const int32_t* topk_idx, int T, int d,
                                  int E, int k, int64_t C, int32_t* counts, int32_t* offsets,
                                  int32_t* slot, int32_t* row_src, __nv_bfloat16* x_pad,
                                  int32_t* n_dropped, int32_t* chunk_hist, cudaStream_t s,
                                  int32_t* status);
cudaError_t launch_quantize_weights(const __nv_bfloat16* w, int E, int K, int N, uint8_t* q,
                                    float* scale, cudaStream_t s);
cudaError_t launch_quantize_rows(const __nv_bfloat16* x, int R, int K, const int32_t* n_rows,
                                 uint8_t* q, float* scale, cudaStream_t s);
cudaError_t launch_gate_up_e4m3(const uint8_t* xq, const float* sx, const int32_t* offsets,
                                int E, int d, int f, int max_rows, const uint8_t* wq_gate,
                                const float* s_gate, const uint8_t* wq_up, const float* s_up,
                                __nv_bfloat16* h, int32_t* status, cudaStream_t s,
                                bool* map_failed, const FuseArgs& fz);
cudaError_t launch_down_e4m3(const uint8_t* hq, const float* sh_rows, const int32_t* offsets,
                             int E, int d, int f, int max_rows, const uint8_t* wq_down,
                             const float* s_down, float* y_perm, int32_t* status, cudaStream_t s,
                             bool* map_failed, const FuseArgs& fz);
}  // namespace moe

namespace moe {
// One CTA waits, with the kernels' time-limited wait, on an mbarrier that
// nothing arrives at; on expiry it reports like the GEMM kernels do.
__global__ void selftest_wait_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit_ns))
    report(status, kDevErrWaitTimeout);
}
}  // namespace moe

using moe::launch_combine;
using moe::launch_down;
using moe::launch_gate_up;
using moe::launch_permute;
using moe::launch_route;
using moe::FuseArgs;

namespace {

using moe::abi::aligned16;
using moe::abi::check_routing_shape;
using moe::abi::check_width;
using moe::abi::cuda_status;
using moe::abi::kMaxE;
using moe::abi::kMaxK;

// An NVTX range around one stage of a one-shot layer call (host-side enqueue;
// a profiler attached to the process shows it on the timeline).
struct StageRange {
  explicit StageRange(const char* name) { nvtxRangePushA(name); }
  ~StageRange() { nvtxRangePop(); }
};

template <class F>
int staged(const char* name, F call) {
  StageRange range(name);
  return call();
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }


size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Byte sizes of the moe_layer_forward workspace fields, in field order.
bool field_sizes(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf,
                 size_t out[MOE_WS_NUM_FIELDS]) {
  const int64_t rows = moe_max_rows(T, E, k, cf);
  if (rows < 0 || d < 1 || f < 1) return false;
  out[MOE_WS_STATUS] = sizeof(int32_t);
  out[MOE_WS_LOGITS] = size_t(T * E) * sizeof(float);
  out[MOE_WS_TOPK_IDX] = size_t(T * k) * sizeof(int32_t);
  out[MOE_WS_TOPK_W] = size_t(T * k) * sizeof(float);
  out[MOE_WS_SLOT] = size_t(T * k) * sizeof(int32_t);
  out[MOE_WS_COUNTS] = size_t(E) * sizeof(int32_t);
  out[MOE_WS_OFFSETS] = size_t(E + 1) * sizeof(int32_t);
  out[MOE_WS_N_DROPPED] = sizeof(int32_t);
  out[MOE_WS_ROW_SRC] = size_t(rows) * sizeof(int32_t);
  out[MOE_WS_PERMUTE] = moe_permute_workspace_size(T, E, k);
  out[MOE_WS_X_PERM] = size_t(rows * d) * 2;
  out[MOE_WS_H] = size_t(rows * f) * 2;
  out[MOE_WS_Y_PERM] = size_t(rows * d) * sizeof(float);
  out[MOE_WS_ROUTE] = moe_route_workspace_size(T, d, E, k);
  return true;
}

// Byte sizes of the FP8 layer's extra fields (after the standard ones).
bool fp8_field_sizes(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf,
                     size_t out[MOE_WS_FP8_NUM_FIELDS - MOE_WS_NUM_FIELDS]) {
  const int64_t rows = moe_max_rows(T, E, k, cf);
  if (rows < 0 || d < 1 || f < 1) return false;
  out[MOE_WS_XQ - MOE_WS_NUM_FIELDS] = size_t(rows * d);
  out[MOE_WS_SX - MOE_WS_NUM_FIELDS] = size_t(rows) * sizeof(float);
  out[MOE_WS_HQ - MOE_WS_NUM_FIELDS] = size_t(rows * f);
  out[MOE_WS_SH - MOE_WS_NUM_FIELDS] = size_t(rows) * sizeof(float);
  out[MOE_WS_XQ_TOK - MOE_WS_NUM_FIELDS] = size_t(T * d);
  out[MOE_WS_SX_TOK - MOE_WS_NUM_FIELDS] = size_t(T) * sizeof(float);
  return true;
}

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    default: return "MOE_ERR_UNKNOWN";
  }
}

int moe_version(void) { return (1 << 16) | 0; }

int moe_selftest_bounded_wait(int32_t* dev_status, int64_t limit_ns, void* stream) {
  if (!dev_status || limit_ns < 0 || limit_ns > 10000000000LL) return MOE_ERR_INVALID_ARG;
  moe::selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(dev_status, (uint64_t)limit_ns);
  return cuda_status(cudaGetLastError());
}

int64_t moe_capacity(int64_t T, int64_t E, int64_t k, double cf) {
  if (T < 0 || E < 1 || k < 1 || !(cf >= 0.0) || isinf(cf)) return -1;
  if (cf == 0.0) return T;
  const double c = ceil(((cf * (double)k) * (double)T) / (double)E);
  if (c > 9.0e15) return -1;
  return (int64_t)c;
}

int64_t moe_max_rows(int64_t T, int64_t E, int64_t k, double cf) {
  const int64_t C = moe_capacity(T, E, k, cf);
  if (C < 0) return -1;
  const int64_t pairs = T * k;
  // E * C may exceed int64 only for absurd cf; the min keeps it bounded
  if (C >= pairs) return pairs;
  const int64_t cap_rows = E * C;
  return cap_rows < pairs ? cap_rows : pairs;
}

size_t moe_route_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k) {
  (void)k;
  if (T < 0 || d < 1 || E < 1 || E > kMaxE) return 0;
  if (T == 0) return 0;
  return moe::route_scratch_bytes(T, d, E);
}

size_t moe_permute_workspace_size(int64_t T, int64_t E, int64_t k) {
  (void)k;
  if (T < 0 || E < 1) return 0;
  return moe::permute_scratch_bytes(T, E);
}

int64_t moe_workspace_field_offset(int field, int64_t T, int64_t d, int64_t E, int64_t k,
                                   int64_t f, double cf) {
  size_t sz[MOE_WS_NUM_FIELDS];
  size_t sz8[MOE_WS_FP8_NUM_FIELDS - MOE_WS_NUM_FIELDS];
  if (field == MOE_WS_ROW_PAIR || field == MOE_WS_Y32) {
    // the fused layer's extra fields follow the standard ones
    const size_t base = moe_workspace_size(T, d, E, k, f, cf);
    const int64_t rows = moe_max_rows(T, E, k, cf);
    if (base == 0 || rows < 0) return -1;
    return (int64_t)(field == MOE_WS_ROW_PAIR
                         ? base
                         : base + align256(size_t(rows) * sizeof(int32_t)));
  }
  if (field < 0 || field >= MOE_WS_FP8_NUM_FIELDS) return -1;
  if (!field_sizes(T, d, E, k, f, cf, sz) || !fp8_field_sizes(T, d, E, k, f, cf, sz8)) return -1;
  size_t off = 0;
  for (int i = 0; i < field; ++i)
    off += align256(i < MOE_WS_NUM_FIELDS ? sz[i] : sz8[i - MOE_WS_NUM_FIELDS]);
  return (int64_t)off;
}

size_t moe_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf) {
  size_t sz[MOE_WS_NUM_FIELDS];
  if (!field_sizes(T, d, E, k, f, cf, sz)) return 0;
  size_t off = 0;
  for (int i = 0; i < MOE_WS_NUM_FIELDS; ++i) off += align256(sz[i]);
  return off;
}

size_t moe_workspace_size_fp8(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf) {
  const size_t base = moe_workspace_size(T, d, E, k, f, cf);
  size_t sz8[MOE_WS_FP8_NUM_FIELDS - MOE_WS_NUM_FIELDS];
  if (base == 0 || !fp8_field_sizes(T, d, E, k, f, cf, sz8)) return 0;
  size_t off = base;
  for (int i = 0; i < MOE_WS_FP8_NUM_FIELDS - MOE_WS_NUM_FIELDS; ++i) off += align256(sz8[i]);
  return off;
}

int moe_route(const void* x, const float* w_router, const float* bias, int64_t T, int64_t d,
              int64_t E, int64_t k, float* logits, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, int32_t* dev_status, void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !logits || !topk_idx || !topk_w || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_route_workspace_size(T, d, E, k)) return MOE_ERR_WORKSPACE;
  bool map_failed = false;
  cudaError_t err = launch_route(static_cast<const __nv_bfloat16*>(x), w_router, bias, (int)T,
                                 (int)d, (int)E, (int)k, logits, topk_idx, topk_w, ws,
                                 dev_status, as_stream(stream), &map_failed);
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_permute(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                int32_t* row_src, void* x_perm, int32_t* n_dropped, void* ws, size_t ws_bytes,
                int32_t* dev_status, void* stream) {
  int64_t C = 0;
  bool done = false;
  int st = moe::abi::check_permute_args(x, topk_idx, T, d, E, k, cf, counts, offsets, slot,
                                        row_src, x_perm, n_dropped, &C, &done);
  if (st != MOE_OK || done) return st;
  if (!ws || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_permute_workspace_size(T, E, k)) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_permute(static_cast<const __nv_bfloat16*>(x), topk_idx, (int)T,
                                    (int)d, (int)E, (int)k, C, counts, offsets, slot, row_src,
                                    static_cast<__nv_bfloat16*>(x_perm), n_dropped,
                                    static_cast<int32_t*>(ws), as_stream(stream), dev_status));
}

static int check_gemm_args(int64_t E, int64_t d, int64_t f, int64_t max_rows) {
  if (E < 1 || E > kMaxE || max_rows < 0 || max_rows >= (int64_t(1) << 31))
    return MOE_ERR_INVALID_ARG;
  int st = check_width(d);
  if (st != MOE_OK) return st;
  if ((st = check_width(f)) != MOE_OK) return st;
  // the kernels count tiles in 32-bit integers: (row tiles) x (column tiles)
  const int64_t row_tiles = max_rows / 64 + E;
  const int64_t col_tiles = (d > f ? d : f) / 64;
  if (row_tiles * col_tiles >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int moe_expert_gate_up(const void* x_perm, const int32_t* offsets, int64_t E, int64_t d,
                       int64_t f, int64_t max_rows, const void* w_gate, const void* w_up,
                       void* h, int32_t* dev_status, void* stream) {
  int st = check_gemm_args(E, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (max_rows == 0) return MOE_OK;
  if (!x_perm || !offsets || !w_gate || !w_up || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(h))
    return MOE_ERR_INVALID_ARG;
  bool map_failed = false;
  cudaError_t err = launch_gate_up(
      static_cast<const __nv_bfloat16*>(x_perm), offsets, (int)E, (int)d, (int)f, (int)max_rows,
      static_cast<const __nv_bfloat16*>(w_gate), static_cast<const __nv_bfloat16*>(w_up),
      static_cast<__nv_bfloat16*>(h), dev_status, as_stream(stream), &map_failed, FuseArgs{});
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_expert_down(const void* h, const int32_t* offsets, int64_t E, int64_t d, int64_t f,
                    int64_t max_rows, const void* w_down, float* y_perm, int32_t* dev_status,
                    void* stream) {
  int st = check_gemm_args(E, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (max_rows == 0) return MOE_OK;
  if (!h || !offsets || !w_down || !y_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_down) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  bool map_failed = false;
  cudaError_t err = launch_down(static_cast<const __nv_bfloat16*>(h), offsets, (int)E, (int)d,
                                (int)f, (int)max_rows, static_cast<const __nv_bfloat16*>(w_down),
                                y_perm, dev_status, as_stream(stream), &map_failed, FuseArgs{});
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_expert_mlp(const void* x_perm, const int32_t* offsets, int64_t E, int64_t d, int64_t f,
                   int64_t max_rows, const void* w_gate, const void* w_up, const void* w_down,
                   void* h, float* y_perm, int32_t* dev_status, void* stream) {
  int st = moe_expert_gate_up(x_perm, offsets, E, d, f, max_rows, w_gate, w_up, h, dev_status,
                              stream);
  if (st != MOE_OK) return st;
  return moe_expert_down(h, offsets, E, d, f, max_rows, w_down, y_perm, dev_status, stream);
}

int moe_combine(const float* y_perm, const void* x, const int32_t* topk_idx, const float* topk_w,
                const int32_t* slot, const int32_t* offsets, int64_t T, int64_t d, int64_t k,
                void* y, void* stream) {
  if (T < 0 || k < 1 || k > kMaxK || T * k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  int st = check_width(d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!y_perm || !x || !topk_idx || !topk_w || !slot || !offsets || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(y_perm, static_cast<const __nv_bfloat16*>(x), topk_idx,
                                    topk_w, slot,
                                    offsets, (int)T, (int)d, (int)k,
                                    static_cast<__nv_bfloat16*>(y), as_stream(stream)));
}

int moe_combine_bf16rows(const void* y_rows, const void* x, const int32_t* topk_idx,
                         const float* topk_w, const int32_t* slot, const int32_t* offsets,
                         int64_t T, int64_t d, int64_t k, void* y, void* stream) {
  if (T < 0 || k < 1 || k > kMaxK || T * k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  int st = check_width(d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!y_rows || !x || !topk_idx || !topk_w || !slot || !offsets || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_rows) || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_combine_bf16rows(
      static_cast<const __nv_bfloat16*>(y_rows), static_cast<const __nv_bfloat16*>(x), topk_idx,
      topk_w, slot, offsets, (int)T, (int)d, (int)k, static_cast<__nv_bfloat16*>(y),
      as_stream(stream)));
}

int moe_rows_to_bf16(const float* src, void* dst, int64_t rows, int64_t d, void* stream) {
  if (rows < 0 || rows >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  int st = check_width(d);
  if (st != MOE_OK) return st;
  if (rows == 0) return MOE_OK;
  if (!src || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_rows_to_bf16(src, static_cast<__nv_bfloat16*>(dst), rows * d,
                                              as_stream(stream)));
}

int64_t moe_padded_rows(int64_t T, int64_t E, int64_t k, double cf) {
  const int64_t C = moe_capacity(T, E, k, cf);
  if (C < 0) return -1;
  const int64_t rows = E * C;
  return rows >= (int64_t(1) << 31) ? -1 : rows;
}

int moe_permute_padded(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                       int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                       int32_t* row_src, void* x_pad, int32_t* n_dropped, void* ws,
                       size_t ws_bytes, int32_t* dev_status, void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  const int64_t C = moe_capacity(T, E, k, cf);
  if (C < 0 || moe_padded_rows(T, E, k, cf) < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !topk_idx || !counts || !offsets || !slot || !row_src || !x_pad || !n_dropped || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_pad) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_permute_workspace_size(T, E, k)) return MOE_ERR_WORKSPACE;
  return cuda_status(moe::launch_permute_padded(
      static_cast<const __nv_bfloat16*>(x), topk_idx, (int)T, (int)d, (int)E, (int)k, C, counts,
      offsets, slot, row_src, static_cast<__nv_bfloat16*>(x_pad), n_dropped,
      static_cast<int32_t*>(ws), as_stream(stream), dev_status));
}

int moe_quantize_weights_fp8(const void* w, int64_t E, int64_t K, int64_t N, uint8_t* w_q,
                             float* scale, void* stream) {
  if (E < 1 || K < 1 || N < 1 || E > 65535 || K > (1 << 30) || N > (1 << 30) ||
      E * K * N >= (int64_t(1) << 40))
    return MOE_ERR_INVALID_ARG;
  if (!w || !w_q || !scale) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_quantize_weights(static_cast<const __nv_bfloat16*>(w), (int)E,
                                                  (int)K, (int)N, w_q, scale, as_stream(stream)));
}

int moe_quantize_rows_fp8(const void* x, int64_t R, int64_t K, const int32_t* n_rows, uint8_t* q,
                          float* scale, void* stream) {
  if (R < 0 || K < 16 || K % 16 != 0 || R >= (int64_t(1) << 31) || K > (1 << 30))
    return MOE_ERR_INVALID_ARG;
  if (R == 0) return MOE_OK;
  if (!x || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_quantize_rows(static_cast<const __nv_bfloat16*>(x), (int)R,
                                               (int)K, n_rows, q, scale, as_stream(stream)));
}

int moe_permute_fp8(const uint8_t* xq, const float* sx, const int32_t* topk_idx, int64_t T,
                    int64_t d, int64_t E, int64_t k, double cf, int32_t* counts,
                    int32_t* offsets, int32_t* slot, int32_t* row_src, uint8_t* xq_perm,
                    float* sx_perm, int32_t* n_dropped, void* ws, size_t ws_bytes,
                    int32_t* dev_status, void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  const int64_t C = moe_capacity(T, E, k, cf);
  if (C < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!xq || !sx || !topk_idx || !counts || !offsets || !slot || !row_src || !xq_perm ||
      !sx_perm || !n_dropped || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(xq_perm) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_permute_workspace_size(T, E, k)) return MOE_ERR_WORKSPACE;
  return cuda_status(moe::launch_permute_rows(xq, (int)d, sx, topk_idx, (int)T, (int)E, (int)k, C,
                                              counts, offsets, slot, row_src, xq_perm, sx_perm,
                                              n_dropped, static_cast<int32_t*>(ws),
                                              as_stream(stream), nullptr, nullptr, 0,
                                              dev_status));
}

int moe_expert_gate_up_fp8(const uint8_t* xq, const float* sx, const int32_t* offsets, int64_t E,
                           int64_t d, int64_t f, int64_t max_rows, const uint8_t* wq_gate,
                           const float* s_gate, const uint8_t* wq_up, const float* s_up, void* h,
                           int32_t* dev_status, void* stream) {
  int st = check_gemm_args(E, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (max_rows == 0) return MOE_OK;
  if (!xq || !sx || !offsets || !wq_gate || !s_gate || !wq_up || !s_up || !h)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq_gate) || !aligned16(wq_up) || !aligned16(s_gate) ||
      !aligned16(s_up) || !aligned16(h))
    return MOE_ERR_INVALID_ARG;
  bool map_failed = false;
  cudaError_t err = moe::launch_gate_up_e4m3(
      xq, sx, offsets, (int)E, (int)d, (int)f, (int)max_rows, wq_gate, s_gate, wq_up, s_up,
      static_cast<__nv_bfloat16*>(h), dev_status, as_stream(stream), &map_failed, FuseArgs{});
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_expert_down_fp8(const uint8_t* hq, const float* sh, const int32_t* offsets, int64_t E,
                        int64_t d, int64_t f, int64_t max_rows, const uint8_t* wq_down,
                        const float* s_down, float* y_perm, int32_t* dev_status, void* stream) {
  int st = check_gemm_args(E, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (max_rows == 0) return MOE_OK;
  if (!hq || !sh || !offsets || !wq_down || !s_down || !y_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned16(hq) || !aligned16(wq_down) || !aligned16(s_down) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  bool map_failed = false;
  cudaError_t err = moe::launch_down_e4m3(hq, sh, offsets, (int)E, (int)d, (int)f, (int)max_rows,
                                          wq_down, s_down, y_perm, dev_status, as_stream(stream),
                                          &map_failed, FuseArgs{});
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_layer_forward_fp8(const void* x, const float* w_router, const float* bias,
                          const uint8_t* wq_gate, const float* s_gate, const uint8_t* wq_up,
                          const float* s_up, const uint8_t* wq_down, const float* s_down,
                          int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf,
                          void* y, void* ws, size_t ws_bytes, void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  if ((st = check_width(f)) != MOE_OK) return st;
  if (moe_capacity(T, E, k, cf) < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !wq_gate || !s_gate || !wq_up || !s_up || !wq_down || !s_down || !y ||
      !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size_fp8(T, d, E, k, f, cf)) return MOE_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  auto field = [&](int id) { return base + moe_workspace_field_offset(id, T, d, E, k, f, cf); };
  int32_t* status = reinterpret_cast<int32_t*>(field(MOE_WS_STATUS));
  float* logits = reinterpret_cast<float*>(field(MOE_WS_LOGITS));
  int32_t* topk_idx = reinterpret_cast<int32_t*>(field(MOE_WS_TOPK_IDX));
  float* topk_w = reinterpret_cast<float*>(field(MOE_WS_TOPK_W));
  int32_t* slot = reinterpret_cast<int32_t*>(field(MOE_WS_SLOT));
  int32_t* counts = reinterpret_cast<int32_t*>(field(MOE_WS_COUNTS));
  int32_t* offsets = reinterpret_cast<int32_t*>(field(MOE_WS_OFFSETS));
  int32_t* n_dropped = reinterpret_cast<int32_t*>(field(MOE_WS_N_DROPPED));
  int32_t* row_src = reinterpret_cast<int32_t*>(field(MOE_WS_ROW_SRC));
  void* h = field(MOE_WS_H);
  float* y_perm = reinterpret_cast<float*>(field(MOE_WS_Y_PERM));
  uint8_t* xq = reinterpret_cast<uint8_t*>(field(MOE_WS_XQ));
  float* sx = reinterpret_cast<float*>(field(MOE_WS_SX));
  uint8_t* hq = reinterpret_cast<uint8_t*>(field(MOE_WS_HQ));
  float* shr = reinterpret_cast<float*>(field(MOE_WS_SH));
  const int64_t max_rows = moe_max_rows(T, E, k, cf);
  const int32_t* n_rows = offsets + E;          // kept rows, written by the permutation
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  st = staged("moe_route", [&] {
    return moe_route(x, w_router, bias, T, d, E, k, logits, topk_idx, topk_w, field(MOE_WS_ROUTE),
                     moe_route_workspace_size(T, d, E, k), status, stream);
  });
  if (st != MOE_OK) return st;
  // each token is quantized once; the permutation moves its codes and scale
  uint8_t* xq_tok = reinterpret_cast<uint8_t*>(field(MOE_WS_XQ_TOK));
  float* sx_tok = reinterpret_cast<float*>(field(MOE_WS_SX_TOK));
  st = staged("moe_quantize_rows_fp8",
              [&] { return moe_quantize_rows_fp8(x, T, d, nullptr, xq_tok, sx_tok, stream); });
  if (st != MOE_OK) return st;
  st = staged("moe_permute_fp8", [&] {
    return moe_permute_fp8(xq_tok, sx_tok, topk_idx, T, d, E, k, cf, counts, offsets, slot,
                           row_src, xq, sx, n_dropped, field(MOE_WS_PERMUTE),
                           moe_permute_workspace_size(T, E, k), status, stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_expert_gate_up_fp8", [&] {
    return moe_expert_gate_up_fp8(xq, sx, offsets, E, d, f, max_rows, wq_gate, s_gate, wq_up,
                                  s_up, h, status, stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_quantize_rows_fp8",
              [&] { return moe_quantize_rows_fp8(h, max_rows, f, n_rows, hq, shr, stream); });
  if (st != MOE_OK) return st;
  st = staged("moe_expert_down_fp8", [&] {
    return moe_expert_down_fp8(hq, shr, offsets, E, d, f, max_rows, wq_down, s_down, y_perm,
                               status, stream);
  });
  if (st != MOE_OK) return st;
  return staged("moe_combine", [&] {
    return moe_combine(y_perm, x, topk_idx, topk_w, slot, offsets, T, d, k, y, stream);
  });
}

// ---------------------------------------------------------------- buckets (expert parallelism)
int moe_expert_mlp_buckets(const void* x_rows, const int32_t* offsets, const int32_t* bucket_rows,
                           int64_t B, int64_t E_w, int64_t d, int64_t f, int64_t max_rows,
                           const void* w_gate, const void* w_up, const void* w_down, void* h,
                           float* y_rows, int32_t* dev_status, void* stream) {
  if (E_w < 1 || B % E_w != 0) return MOE_ERR_INVALID_ARG;
  int st = check_gemm_args(B, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (max_rows == 0) return MOE_OK;
  if (!x_rows || !offsets || !w_gate || !w_up || !w_down || !h || !y_rows)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(h) || !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  FuseArgs fz{};
  fz.bucket_rows = bucket_rows;
  fz.n_weights = (int)E_w;
  bool map_failed = false;
  cudaError_t err = launch_gate_up(
      static_cast<const __nv_bfloat16*>(x_rows), offsets, (int)B, (int)d, (int)f, (int)max_rows,
      static_cast<const __nv_bfloat16*>(w_gate), static_cast<const __nv_bfloat16*>(w_up),
      static_cast<__nv_bfloat16*>(h), dev_status, as_stream(stream), &map_failed, fz);
  if (map_failed) return MOE_ERR_CUDA;
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  err = launch_down(static_cast<const __nv_bfloat16*>(h), offsets, (int)B, (int)d, (int)f,
                    (int)max_rows, static_cast<const __nv_bfloat16*>(w_down), y_rows, dev_status,
                    as_stream(stream), &map_failed, fz);
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

// ---------------------------------------------------------------- fused path
int moe_permute_fused(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                      int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                      int32_t* row_src, int32_t* row_pair, void* x_perm, int32_t* n_dropped,
                      float* y32, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  const int64_t C = moe_capacity(T, E, k, cf);
  if (C < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!topk_idx || !counts || !offsets || !slot || !row_src || !row_pair || !n_dropped || !ws)
    return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws) || (y32 && !aligned16(y32)) || (x && (!aligned16(x) || !aligned16(x_perm))))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_permute_workspace_size(T, E, k)) return MOE_ERR_WORKSPACE;
  return cuda_status(moe::launch_permute_rows(
      static_cast<const uint8_t*>(x), (int)d * 2, nullptr, topk_idx, (int)T, (int)E, (int)k, C,
      counts, offsets, slot, row_src, static_cast<uint8_t*>(x_perm), nullptr, n_dropped,
      static_cast<int32_t*>(ws), as_stream(stream), row_pair, y32, y32 ? (int)d : 0, dev_status));
}

int moe_expert_gate_up_gather(const void* x, int64_t T, const int32_t* row_src,
                              const int32_t* offsets, int64_t E, int64_t d, int64_t f,
                              int64_t max_rows, const void* w_gate, const void* w_up, void* h,
                              int32_t* dev_status, void* stream) {
  int st = check_gemm_args(E, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (T < 1 || T >= (int64_t(1) << 31) - 1) return MOE_ERR_INVALID_ARG;
  if (max_rows == 0) return MOE_OK;
  if (!x || !row_src || !offsets || !w_gate || !w_up || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(h))
    return MOE_ERR_INVALID_ARG;
  FuseArgs fz{};
  fz.row_src = row_src;
  fz.n_tok = (int)T;
  bool map_failed = false;
  cudaError_t err = launch_gate_up(
      static_cast<const __nv_bfloat16*>(x), offsets, (int)E, (int)d, (int)f, (int)max_rows,
      static_cast<const __nv_bfloat16*>(w_gate), static_cast<const __nv_bfloat16*>(w_up),
      static_cast<__nv_bfloat16*>(h), dev_status, as_stream(stream), &map_failed, fz);
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_expert_down_scatter(const void* h, const int32_t* offsets, int64_t E, int64_t d,
                            int64_t f, int64_t max_rows, const void* w_down,
                            const int32_t* row_pair, const float* topk_w, int64_t k, float* y32,
                            int32_t* dev_status, void* stream) {
  int st = check_gemm_args(E, d, f, max_rows);
  if (st != MOE_OK) return st;
  if (k < 1 || k > kMaxK) return MOE_ERR_INVALID_ARG;
  if (max_rows == 0) return MOE_OK;
  if (!h || !offsets || !w_down || !row_pair || !topk_w || !y32) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_down) || !aligned16(y32)) return MOE_ERR_INVALID_ARG;
  FuseArgs fz{};
  fz.row_pair = row_pair;
  fz.topk_w = topk_w;
  fz.k = (int)k;
  fz.y32 = y32;
  bool map_failed = false;
  cudaError_t err = launch_down(static_cast<const __nv_bfloat16*>(h), offsets, (int)E, (int)d,
                                (int)f, (int)max_rows, static_cast<const __nv_bfloat16*>(w_down),
                                nullptr, dev_status, as_stream(stream), &map_failed, fz);
  if (map_failed) return MOE_ERR_CUDA;
  return cuda_status(err);
}

int moe_combine_finalize(const float* y32, const void* x, const int32_t* slot, int64_t T,
                         int64_t d, int64_t k, void* y, void* stream) {
  if (T < 0 || k < 1 || k > kMaxK || T * k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  int st = check_width(d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!y32 || !x || !slot || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y32) || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_finalize(y32, static_cast<const __nv_bfloat16*>(x), slot,
                                          (int)T, (int)d, (int)k,
                                          static_cast<__nv_bfloat16*>(y), as_stream(stream)));
}

size_t moe_workspace_size_fused(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                                double cf) {
  const size_t base = moe_workspace_size(T, d, E, k, f, cf);
  const int64_t rows = moe_max_rows(T, E, k, cf);
  if (base == 0 || rows < 0) return 0;
  return base + align256(size_t(rows) * sizeof(int32_t)) + align256(size_t(T * d) * sizeof(float));
}

int moe_layer_forward_fused(const void* x, const float* w_router, const float* bias,
                            const void* w_gate, const void* w_up, const void* w_down, int64_t T,
                            int64_t d, int64_t E, int64_t k, int64_t f, double cf, void* y,
                            void* ws, size_t ws_bytes, void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  if ((st = check_width(f)) != MOE_OK) return st;
  if (moe_capacity(T, E, k, cf) < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !w_gate || !w_up || !w_down || !y || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size_fused(T, d, E, k, f, cf)) return MOE_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  auto field = [&](int id) { return base + moe_workspace_field_offset(id, T, d, E, k, f, cf); };
  int32_t* status = reinterpret_cast<int32_t*>(field(MOE_WS_STATUS));
  float* logits = reinterpret_cast<float*>(field(MOE_WS_LOGITS));
  int32_t* topk_idx = reinterpret_cast<int32_t*>(field(MOE_WS_TOPK_IDX));
  float* topk_w = reinterpret_cast<float*>(field(MOE_WS_TOPK_W));
  int32_t* slot = reinterpret_cast<int32_t*>(field(MOE_WS_SLOT));
  int32_t* counts = reinterpret_cast<int32_t*>(field(MOE_WS_COUNTS));
  int32_t* offsets = reinterpret_cast<int32_t*>(field(MOE_WS_OFFSETS));
  int32_t* n_dropped = reinterpret_cast<int32_t*>(field(MOE_WS_N_DROPPED));
  int32_t* row_src = reinterpret_cast<int32_t*>(field(MOE_WS_ROW_SRC));
  void* x_perm = field(MOE_WS_X_PERM);
  void* h = field(MOE_WS_H);
  int32_t* row_pair = reinterpret_cast<int32_t*>(field(MOE_WS_ROW_PAIR));
  float* y32 = reinterpret_cast<float*>(field(MOE_WS_Y32));
  const int64_t max_rows = moe_max_rows(T, E, k, cf);
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  st = staged("moe_route", [&] {
    return moe_route(x, w_router, bias, T, d, E, k, logits, topk_idx, topk_w, field(MOE_WS_ROUTE),
                     moe_route_workspace_size(T, d, E, k), status, stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_permute_fused", [&] {
    return moe_permute_fused(x, topk_idx, T, d, E, k, cf, counts, offsets, slot, row_src,
                             row_pair, x_perm, n_dropped, y32, field(MOE_WS_PERMUTE),
                             moe_permute_workspace_size(T, E, k), status, stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_expert_gate_up", [&] {
    return moe_expert_gate_up(x_perm, offsets, E, d, f, max_rows, w_gate, w_up, h, status,
                              stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_expert_down_scatter", [&] {
    return moe_expert_down_scatter(h, offsets, E, d, f, max_rows, w_down, row_pair, topk_w, k,
                                   y32, status, stream);
  });
  if (st != MOE_OK) return st;
  return staged("moe_combine_finalize",
                [&] { return moe_combine_finalize(y32, x, slot, T, d, k, y, stream); });
}

int moe_layer_forward(const void* x, const float* w_router, const float* bias, const void* w_gate,
                      const void* w_up, const void* w_down, int64_t T, int64_t d, int64_t E,
                      int64_t k, int64_t f, double cf, void* y, void* ws, size_t ws_bytes,
                      void* stream) {
  return moe_layer_forward_ex(x, w_router, bias, w_gate, w_up, w_down, T, d, E, k, f, cf, y,
                              nullptr, nullptr, nullptr, nullptr, nullptr, ws, ws_bytes, stream);
}

int moe_layer_forward_ex(const void* x, const float* w_router, const float* bias,
                         const void* w_gate, const void* w_up, const void* w_down, int64_t T,
                         int64_t d, int64_t E, int64_t k, int64_t f, double cf, void* y,
                         float* logits_out, int32_t* topk_idx_out, float* topk_w_out,
                         int32_t* slot_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                         void* stream) {
  int st = check_routing_shape(T, E, k);
  if (st != MOE_OK) return st;
  if ((st = check_width(d)) != MOE_OK) return st;
  if ((st = check_width(f)) != MOE_OK) return st;
  if (moe_capacity(T, E, k, cf) < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !w_gate || !w_up || !w_down || !y || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size(T, d, E, k, f, cf)) return MOE_ERR_WORKSPACE;

  char* base = static_cast<char*>(ws);
  auto field = [&](int id) {
    return base + moe_workspace_field_offset(id, T, d, E, k, f, cf);
  };
  // a caller's output pointer replaces the workspace field it names
  auto pick = [](auto* out, char* fld) {
    return out ? out : reinterpret_cast<decltype(out)>(fld);
  };
  int32_t* status = reinterpret_cast<int32_t*>(field(MOE_WS_STATUS));
  float* logits = pick(logits_out, field(MOE_WS_LOGITS));
  int32_t* topk_idx = pick(topk_idx_out, field(MOE_WS_TOPK_IDX));
  float* topk_w = pick(topk_w_out, field(MOE_WS_TOPK_W));
  int32_t* slot = pick(slot_out, field(MOE_WS_SLOT));
  int32_t* counts = pick(counts_out, field(MOE_WS_COUNTS));
  int32_t* offsets = reinterpret_cast<int32_t*>(field(MOE_WS_OFFSETS));
  int32_t* n_dropped = reinterpret_cast<int32_t*>(field(MOE_WS_N_DROPPED));
  int32_t* row_src = reinterpret_cast<int32_t*>(field(MOE_WS_ROW_SRC));
  void* pscratch = field(MOE_WS_PERMUTE);
  void* x_perm = field(MOE_WS_X_PERM);
  void* h = field(MOE_WS_H);
  float* y_perm = reinterpret_cast<float*>(field(MOE_WS_Y_PERM));
  void* rscratch = field(MOE_WS_ROUTE);
  const int64_t max_rows = moe_max_rows(T, E, k, cf);
  cudaStream_t s = as_stream(stream);

  if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  st = staged("moe_route", [&] {
    return moe_route(x, w_router, bias, T, d, E, k, logits, topk_idx, topk_w, rscratch,
                     moe_route_workspace_size(T, d, E, k), status, stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_permute", [&] {
    return moe_permute(x, topk_idx, T, d, E, k, cf, counts, offsets, slot, row_src, x_perm,
                       n_dropped, pscratch, moe_permute_workspace_size(T, E, k), status, stream);
  });
  if (st != MOE_OK) return st;
  st = staged("moe_expert_mlp", [&] {
    return moe_expert_mlp(x_perm, offsets, E, d, f, max_rows, w_gate, w_up, w_down, h, y_perm,
                          status, stream);
  });
  if (st != MOE_OK) return st;
  return staged("moe_combine", [&] {
    return moe_combine(y_perm, x, topk_idx, topk_w, slot, offsets, T, d, k, y, stream);
  });
}

}  // extern "C"
