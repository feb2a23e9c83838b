// Combine: inverse permutation plus gate-weighted sum.
//
// The combine undoes the dispatch permutation and sums each token's k expert
// outputs scaled by their gate weights ("Expert Parallelism & All-to-All"
// (neelmishra.github.io), section "All-to-all: the distributed transpose";
// last step of the infra.bea.ai guide's section 2 diagram).  A token whose
// pairs were all dropped leaves the layer unchanged (inferensys.com glossary,
// Dropped Tokens entry).
//
// One warp per (token, 512-column segment): lanes 0..k-1 resolve the k source
// rows and weights, broadcast them, then the warp streams its segment of the
// expert-output rows (fp32, or bf16 where an expert-parallel exchange sent
// them back at half the bytes) in 16-byte vectors, accumulating in fp32 in
// top-k order and rounding once to bf16.
#include "common.cuh"

namespace moe {

constexpr int kCombThreads = 256;
constexpr int kSegVec = 64;        // 16-byte output vectors per warp work unit (512 elements)

// values 8v .. 8v+7 of an expert-output row, as fp32
__device__ __forceinline__ void load8(const float* row, int v, float (&o)[8]) {
  const float4* src = reinterpret_cast<const float4*>(row);
  const float4 a = __ldg(src + 2 * v), b = __ldg(src + 2 * v + 1);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* row, int v, float (&o)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + v);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {      // bf16 -> fp32 is exact: the bits in the upper half
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One warp per (token, 512-column segment), so that a handful of tokens still
// spreads over many SMs.
template <typename RowT>
__global__ void __launch_bounds__(kCombThreads)
    combine_kernel(const RowT* __restrict__ y_perm, const __nv_bfloat16* __restrict__ x,
                   const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ slot, const int32_t* __restrict__ offsets, int T,
                   int d, int k, int nseg, __nv_bfloat16* __restrict__ y) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long unit = (long long)blockIdx.x * (kCombThreads / 32) + warp;
  if (unit >= (long long)T * nseg) return;
  const int t = (int)(unit / nseg), seg = (int)(unit % nseg);
  int my_row = -1;
  float my_w = 0.f;
  if (lane < k) {
    const size_t p = (size_t)t * k + lane;
    const int s = slot[p];
    if (s >= 0) {
      my_row = offsets[topk_idx[p]] + s;
      my_w = topk_w[p];
    }
  }
  int rows[8];
  float w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    w[j] = __shfl_sync(0xffffffffu, my_w, j);
  }
  const bool any_kept = __any_sync(0xffffffffu, my_row >= 0);
  const int nvec = d / 8;
  const int v_begin = seg * kSegVec;
  const int v_end = min(nvec, v_begin + kSegVec);
  uint4* dst = reinterpret_cast<uint4*>(y + (size_t)t * d);
  if (!any_kept) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    for (int v = v_begin + lane; v < v_end; v += 32) dst[v] = __ldg(src + v);
    return;
  }
  float acc[2][8];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[u][q] = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    if (rows[j] < 0) continue;
    const RowT* src = y_perm + (size_t)rows[j] * d;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = v_begin + lane + u * 32;
      if (v >= v_end) continue;
      float a[8];
      load8(src, v, a);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[u][q] = fmaf(w[j], a[q], acc[u][q]);
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int v = v_begin + lane + u * 32;
    if (v >= v_end) continue;
    uint4 o;
    o.x = pack_bf16x2(acc[u][0], acc[u][1]);
    o.y = pack_bf16x2(acc[u][2], acc[u][3]);
    o.z = pack_bf16x2(acc[u][4], acc[u][5]);
    o.w = pack_bf16x2(acc[u][6], acc[u][7]);
    dst[v] = o;
  }
}

template <typename RowT>
static cudaError_t launch_combine_t(const RowT* y_perm, const __nv_bfloat16* x,
                                   const int32_t* topk_idx, const float* topk_w,
                                   const int32_t* slot, const int32_t* offsets, int T, int d,
                                   int k, __nv_bfloat16* y, cudaStream_t s) {
  const int nseg = (d / 8 + kSegVec - 1) / kSegVec;
  const long long units = (long long)T * nseg;
  const int per_cta = kCombThreads / 32;
  combine_kernel<RowT><<<(unsigned)((units + per_cta - 1) / per_cta), kCombThreads, 0, s>>>(
      y_perm, x, topk_idx, topk_w, slot, offsets, T, d, k, nseg, y);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y_perm, const __nv_bfloat16* x,
                           const int32_t* topk_idx, const float* topk_w, const int32_t* slot,
                           const int32_t* offsets, int T, int d, int k, __nv_bfloat16* y,
                           cudaStream_t s) {
  return launch_combine_t(y_perm, x, topk_idx, topk_w, slot, offsets, T, d, k, y, s);
}

cudaError_t launch_combine_bf16rows(const __nv_bfloat16* y_rows, const __nv_bfloat16* x,
                                    const int32_t* topk_idx, const float* topk_w,
                                    const int32_t* slot, const int32_t* offsets, int T, int d,
                                    int k, __nv_bfloat16* y, cudaStream_t s) {
  return launch_combine_t(y_rows, x, topk_idx, topk_w, slot, offsets, T, d, k, y, s);
}

// fp32 rows -> bf16 (round to nearest even), 8 values per thread step: the
// expert outputs an expert-parallel rank sends back at half the bytes.
__global__ void __launch_bounds__(256)
    rows_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                        long long nvec) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < nvec;
       v += (long long)gridDim.x * blockDim.x) {
    const float4 a = __ldg(s4 + 2 * v), b = __ldg(s4 + 2 * v + 1);
    d4[v] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                       pack_bf16x2(b.z, b.w));
  }
}

cudaError_t launch_rows_to_bf16(const float* src, __nv_bfloat16* dst, long long n,
                                cudaStream_t s) {
  const long long nvec = n / 8;
  long long blocks = (nvec + 255) / 256;
  if (blocks > 4096) blocks = 4096;      // a grid-stride loop covers the rest
  if (blocks < 1) blocks = 1;
  rows_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, dst, nvec);
  return cudaGetLastError();
}

// Fused-combine finish: the down GEMM has added w * (expert output) of every
// kept pair into y32[t] (fp32); y[t] = bf16(y32[t]), or x[t] when all of the
// token's pairs were dropped.  One warp per token, 16-byte vectors.
__global__ void __launch_bounds__(256)
    finalize_kernel(const float* __restrict__ y32, const __nv_bfloat16* __restrict__ x,
                    const int32_t* __restrict__ slot, int T, int d, int k,
                    __nv_bfloat16* __restrict__ y) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const int kept = __any_sync(0xffffffffu, lane < k && slot[(size_t)t * k + lane] >= 0);
  uint4* dst = reinterpret_cast<uint4*>(y + (size_t)t * d);
  const int nvec = d / 8;
  if (!kept) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
    return;
  }
  const float4* src = reinterpret_cast<const float4*>(y32 + (size_t)t * d);
  for (int v = lane; v < nvec; v += 32) {
    const float4 a = __ldg(src + 2 * v), b = __ldg(src + 2 * v + 1);
    dst[v] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                        pack_bf16x2(b.z, b.w));
  }
}

cudaError_t launch_finalize(const float* y32, const __nv_bfloat16* x, const int32_t* slot, int T,
                            int d, int k, __nv_bfloat16* y, cudaStream_t s) {
  finalize_kernel<<<(T + 7) / 8, 256, 0, s>>>(y32, x, slot, T, d, k, y);
  return cudaGetLastError();
}

}  // namespace moe
