// Weight-only FP8 (e4m3) quantization of expert weights, one fp32 scale per
// (expert, output column): s[e,n] = max_k |w[e,k,n]| / 448 (1 for an all-zero
// column), q[e,k,n] = e4m3(w[e,k,n] / s[e,n]) rounded to nearest even with
// saturation to +-448.  A one-time preprocessing step: FP8 expert weights halve
// the bytes the decode-sized layer streams (inferensys.com "Expert
// Parallelism" glossary, quantization entry: post-training FP8 experts).
#include "common.cuh"

namespace moe {

constexpr int kQuantCols = 256;

// one thread per column, 256 columns per CTA, grid (column blocks, E)
__global__ void __launch_bounds__(kQuantCols)
    quantize_fp8_kernel(const __nv_bfloat16* __restrict__ w, int K, int N,
                        uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int e = blockIdx.y;
  const int n = blockIdx.x * kQuantCols + threadIdx.x;
  if (n >= N) return;
  const __nv_bfloat16* col = w + (size_t)e * K * N + n;
  float mx = 0.f;
  for (int k = 0; k < K; ++k) mx = fmaxf(mx, fabsf(__bfloat162float(col[(size_t)k * N])));
  const float s = mx > 0.f ? mx / 448.0f : 1.0f;
  scale[(size_t)e * N + n] = s;
  uint8_t* qc = q + (size_t)e * K * N + n;
  for (int k = 0; k < K; ++k) {
    const float v = __bfloat162float(col[(size_t)k * N]) / s;
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(pair) : "f"(v));
    qc[(size_t)k * N] = static_cast<uint8_t>(pair & 0xFFu);
  }
}

cudaError_t launch_quantize_fp8(const __nv_bfloat16* w, int E, int K, int N, uint8_t* q,
                                float* scale, cudaStream_t s) {
  dim3 grid((N + kQuantCols - 1) / kQuantCols, E);
  quantize_fp8_kernel<<<grid, kQuantCols, 0, s>>>(w, K, N, q, scale);
  return cudaGetLastError();
}

}  // namespace moe
