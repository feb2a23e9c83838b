// FP8 (e4m3) quantization for the FP8 expert variant (inferensys.com "Expert
// Parallelism" glossary, quantization entry: post-training FP8 experts).
//
// One rule for weights and activations: a group of values (a weight column
// over K, an activation row over K) shares one fp32 scale s = max |v| / 448
// (1 for an all-zero group; 448 is the largest finite e4m3 value) and each
// value becomes the e4m3 code of v / s, rounded to nearest even and saturated
// to +-448.  Row scales times column scales are constant along the
// contraction, so the GEMMs run on the codes and scale the fp32 accumulators.
//
// Weights [E, K, N] (N contiguous) are written K-major, codes [E, N, K], so
// that both GEMM operands are K-major e4m3 tiles.
#include "common.cuh"

namespace moe {

// e4m3 code of an fp32 value, nearest even, saturating (hardware conversion)
__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(pair) : "f"(v));
  return pair & 0xFFu;
}

// two codes packed as bytes (lo, hi) of a 16-bit value
__device__ __forceinline__ uint32_t e4m3_pair(float lo, float hi) {
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(hi), "f"(lo));
  return pair;
}

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? amax / 448.0f : 1.0f; }

// ---------------------------------------------------------------- weights
// 1. column scales: one thread per (expert, column), walking K (coalesced
//    across the threads of a warp)
__global__ void __launch_bounds__(256)
    weight_scale_kernel(const __nv_bfloat16* __restrict__ w, int K, int N,
                        float* __restrict__ scale) {
  const int e = blockIdx.y;
  const int n = blockIdx.x * 256 + threadIdx.x;
  if (n >= N) return;
  const __nv_bfloat16* col = w + (size_t)e * K * N + n;
  float mx = 0.f;
  for (int k = 0; k < K; ++k) mx = fmaxf(mx, fabsf(__bfloat162float(col[(size_t)k * N])));
  scale[(size_t)e * N + n] = scale_of(mx);
}

// 2. codes, transposed: a CTA stages a 64 (K) x 64 (N) tile in shared memory
//    and writes, for each of its 64 columns, 64 consecutive K codes
constexpr int kQT = 64;
__global__ void __launch_bounds__(256)
    weight_quant_kernel(const __nv_bfloat16* __restrict__ w, int K, int N,
                        const float* __restrict__ scale, uint8_t* __restrict__ q) {
  __shared__ float tile[kQT][kQT + 1];
  const int e = blockIdx.z;
  const int k0 = blockIdx.y * kQT, n0 = blockIdx.x * kQT;
  const __nv_bfloat16* src = w + (size_t)e * K * N;
  for (int i = threadIdx.x; i < kQT * kQT; i += 256) {
    const int kk = i / kQT, nn = i % kQT;
    const int k = k0 + kk, n = n0 + nn;
    tile[kk][nn] = (k < K && n < N) ? __bfloat162float(src[(size_t)k * N + n]) : 0.f;
  }
  __syncthreads();
  // thread -> (column nn, 16 consecutive K rows starting at kq)
  const int nn = threadIdx.x / 4, kq = (threadIdx.x % 4) * 16;
  const int n = n0 + nn;
  if (n >= N) return;
  const float s = scale[(size_t)e * N + n];
  uint32_t b[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) b[j] = e4m3_code(tile[kq + j][nn] / s);
  uint8_t* dst = q + ((size_t)e * N + n) * K + k0 + kq;
  if (k0 + kq + 16 <= K && (K % 16) == 0) {
    uint4 v;
    v.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    v.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
    v.z = b[8] | (b[9] << 8) | (b[10] << 16) | (b[11] << 24);
    v.w = b[12] | (b[13] << 8) | (b[14] << 16) | (b[15] << 24);
    *reinterpret_cast<uint4*>(dst) = v;
  } else {
    for (int j = 0; j < 16 && k0 + kq + j < K; ++j) dst[j] = static_cast<uint8_t>(b[j]);
  }
}

cudaError_t launch_quantize_weights(const __nv_bfloat16* w, int E, int K, int N, uint8_t* q,
                                    float* scale, cudaStream_t s) {
  weight_scale_kernel<<<dim3((N + 255) / 256, E), 256, 0, s>>>(w, K, N, scale);
  weight_quant_kernel<<<dim3((N + kQT - 1) / kQT, (K + kQT - 1) / kQT, E), 256, 0, s>>>(
      w, K, N, scale, q);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- activation rows
// Long rows (K > 16384): one warp per row, the row's max magnitude (16-byte
// loads), then its codes (the row is read again, now from cache).  Rows at or beyond *n_rows (a
// device count, e.g. offsets[E] of the permutation) are skipped.
constexpr int kRowWarps = 8;
__global__ void __launch_bounds__(32 * kRowWarps)
    quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int R, int K,
                         const int32_t* __restrict__ n_rows, uint8_t* __restrict__ q,
                         float* __restrict__ scale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int r = blockIdx.x * kRowWarps + warp;
  int limit = R;
  if (n_rows) limit = min(limit, *n_rows);
  if (r >= limit) return;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)r * K);
  const int nvec = K / 8;
  float mx = 0.f;
  for (int v = lane; v < nvec; v += 32) {
    const uint4 u = __ldg(row + v);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const float s = scale_of(mx);
  if (lane == 0) scale[r] = s;
  uint2* out = reinterpret_cast<uint2*>(q + (size_t)r * K);
  for (int v = lane; v < nvec; v += 32) {
    const uint4 u = __ldg(row + v);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      p[i] = e4m3_pair(__uint_as_float(w[i] << 16) / s, __uint_as_float(w[i] & 0xFFFF0000u) / s);
    out[v] = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
  }
}

// Short rows (K <= 2048): one warp per row holds the whole row in registers
// (at most 8 16-byte vectors per lane), so each value is read once.
constexpr int kShortVecs = 8;
__global__ void __launch_bounds__(32 * kRowWarps)
    quantize_rows_short_kernel(const __nv_bfloat16* __restrict__ x, int R, int K,
                               const int32_t* __restrict__ n_rows, uint8_t* __restrict__ q,
                               float* __restrict__ scale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int r = blockIdx.x * kRowWarps + warp;
  int limit = R;
  if (n_rows) limit = min(limit, *n_rows);
  if (r >= limit) return;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)r * K);
  const int nvec = K / 8;
  uint4 v[kShortVecs];
#pragma unroll
  for (int j = 0; j < kShortVecs; ++j) {
    const int i = lane + 32 * j;
    v[j] = i < nvec ? __ldg(row + i) : make_uint4(0, 0, 0, 0);
  }
  float mx = 0.f;
#pragma unroll
  for (int j = 0; j < kShortVecs; ++j) {
    const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const float s = scale_of(mx);
  if (lane == 0) scale[r] = s;
  uint2* out = reinterpret_cast<uint2*>(q + (size_t)r * K);
#pragma unroll
  for (int j = 0; j < kShortVecs; ++j) {
    const int i = lane + 32 * j;
    if (i < nvec) {
      const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      uint32_t p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        p[e] = e4m3_pair(__uint_as_float(w[e] << 16) / s, __uint_as_float(w[e] & 0xFFFF0000u) / s);
      out[i] = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
    }
  }
}

// Wide rows (2048 < K <= 16384): one CTA of THREADS threads per row holds the whole row
// in registers (at most kWideVecs 16-byte vectors per thread), so each value
// is read from memory once; the max magnitude is reduced across the CTA.
constexpr int kWideVecs = 8;             // K <= THREADS * 8 * 8
template <int kWideThreads>
__global__ void __launch_bounds__(kWideThreads)
    quantize_rows_wide_kernel(const __nv_bfloat16* __restrict__ x, int R, int K,
                              const int32_t* __restrict__ n_rows, uint8_t* __restrict__ q,
                              float* __restrict__ scale) {
  __shared__ float warp_max[kWideThreads / 32];
  const int r = blockIdx.x;
  int limit = R;
  if (n_rows) limit = min(limit, *n_rows);
  if (r >= limit) return;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)r * K);
  const int nvec = K / 8;
  uint4 v[kWideVecs];
  float mx = 0.f;
#pragma unroll
  for (int j = 0; j < kWideVecs; ++j) {
    const int i = threadIdx.x + j * kWideThreads;
    v[j] = i < nvec ? __ldg(row + i) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int j = 0; j < kWideVecs; ++j) {
    const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (threadIdx.x % 32 == 0) warp_max[threadIdx.x / 32] = mx;
  __syncthreads();
  mx = warp_max[0];
#pragma unroll
  for (int w = 1; w < kWideThreads / 32; ++w) mx = fmaxf(mx, warp_max[w]);
  const float s = scale_of(mx);
  if (threadIdx.x == 0) scale[r] = s;
  uint2* out = reinterpret_cast<uint2*>(q + (size_t)r * K);
#pragma unroll
  for (int j = 0; j < kWideVecs; ++j) {
    const int i = threadIdx.x + j * kWideThreads;
    if (i < nvec) {
      const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      uint32_t p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        p[e] = e4m3_pair(__uint_as_float(w[e] << 16) / s, __uint_as_float(w[e] & 0xFFFF0000u) / s);
      out[i] = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
    }
  }
}

cudaError_t launch_quantize_rows(const __nv_bfloat16* x, int R, int K, const int32_t* n_rows,
                                 uint8_t* q, float* scale, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  const int rows_ctas = (R + kRowWarps - 1) / kRowWarps;
  if (K <= 32 * kShortVecs * 8)
    quantize_rows_short_kernel<<<rows_ctas, 32 * kRowWarps, 0, s>>>(x, R, K, n_rows, q, scale);
  else if (K <= 128 * kWideVecs * 8)
    quantize_rows_wide_kernel<128><<<R, 128, 0, s>>>(x, R, K, n_rows, q, scale);
  else if (K <= 256 * kWideVecs * 8)
    quantize_rows_wide_kernel<256><<<R, 256, 0, s>>>(x, R, K, n_rows, q, scale);
  else
    quantize_rows_kernel<<<rows_ctas, 32 * kRowWarps, 0, s>>>(x, R, K, n_rows, q, scale);
  return cudaGetLastError();
}

}  // namespace moe
