// Router logits and top-k softmax gating in one kernel.
//
// The router is a linear layer with one output score per expert; top-k gating
// keeps the k best-scoring experts and their scores become the mixing weights
// (inferensys.com "Expert Parallelism" glossary, gating-network and Top-k
// Gating entries; klaylearn.com glossary, third paragraph).
//
// logits = x (bf16, widened exactly) @ Wr (fp32) + bias, fp32 FMA on the CUDA
// cores.  A CTA owns BT tokens and all (padded) EP experts; K is walked in
// chunks of KC with the x chunk (transposed) and the Wr chunk staged in shared
// memory; each thread keeps a TPT x EPT register tile.  The logits tile is then
// parked in shared memory and one warp per token runs k rounds of a warp-wide
// arg-max (value descending, expert index ascending on equal values).
#include "common.cuh"

namespace moe {

constexpr int kRouterThreads = 256;
constexpr int kRouterKC = 32;

template <int EP, int EPT, int TPT>
struct RouterShape {
  static constexpr int TX = EP / EPT;                  // threads along experts
  static constexpr int TY = kRouterThreads / TX;       // threads along tokens
  static constexpr int BT = TY * TPT;                  // tokens per CTA
  static constexpr int kStageFloats = kRouterKC * EP + kRouterKC * BT;
  static constexpr int kLogitFloats = BT * EP;
  static constexpr int kSmemFloats = kStageFloats > kLogitFloats ? kStageFloats : kLogitFloats;
};

template <int EP, int EPT, int TPT>
__global__ void __launch_bounds__(kRouterThreads)
    router_topk_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr,
                       const float* __restrict__ bias, int T, int d, int E, int k,
                       float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                       float* __restrict__ topk_w) {
  using S = RouterShape<EP, EPT, TPT>;
  __shared__ __align__(16) float smem[S::kSmemFloats];
  float* ws = smem;                          // [KC][EP]
  float* xs = smem + kRouterKC * EP;         // [KC][BT]

  const int tid = threadIdx.x;
  const int tx = tid % S::TX, ty = tid / S::TX;
  const int t0 = blockIdx.x * S::BT;

  float acc[TPT][EPT];
#pragma unroll
  for (int i = 0; i < TPT; ++i)
#pragma unroll
    for (int j = 0; j < EPT; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < d; k0 += kRouterKC) {
    // x chunk: BT tokens x KC values, 8 bf16 (16 B) per load, stored transposed
    for (int v = tid; v < S::BT * (kRouterKC / 8); v += kRouterThreads) {
      const int tt = v / (kRouterKC / 8), part = v % (kRouterKC / 8);
      const int t = t0 + tt;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (t < T) raw = *reinterpret_cast<const uint4*>(x + (size_t)t * d + k0 + part * 8);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int q = 0; q < 8; ++q) xs[(part * 8 + q) * S::BT + tt] = __bfloat162float(b[q]);
    }
    // Wr chunk: KC rows x EP experts (experts >= E read as zero)
    for (int v = tid; v < kRouterKC * EP; v += kRouterThreads) {
      const int kk = v / EP, e = v % EP;
      ws[v] = (e < E) ? wr[(size_t)(k0 + kk) * E + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRouterKC; ++kk) {
      float xv[TPT], wv[EPT];
#pragma unroll
      for (int i = 0; i < TPT; ++i) xv[i] = xs[kk * S::BT + ty * TPT + i];
#pragma unroll
      for (int j = 0; j < EPT; ++j) wv[j] = ws[kk * EP + tx * EPT + j];
#pragma unroll
      for (int i = 0; i < TPT; ++i)
#pragma unroll
        for (int j = 0; j < EPT; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }

  // logits (+bias) to global memory and to the shared tile [BT][EP]
  float* ls = smem;
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int tt = ty * TPT + i, t = t0 + tt;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = tx * EPT + j;
      float v = acc[i][j];
      if (e < E) {
        if (bias) v += bias[e];
        if (t < T) logits[(size_t)t * E + e] = v;
      }
      ls[tt * EP + e] = v;
    }
  }
  __syncthreads();

  // top-k: one warp per token
  constexpr int kPerLane = EP >= 32 ? EP / 32 : 1;
  const int warp = tid / 32, lane = tid % 32;
  for (int tt = warp; tt < S::BT; tt += kRouterThreads / 32) {
    const int t = t0 + tt;
    if (t >= T) break;
    float val[kPerLane];
    bool live[kPerLane];
#pragma unroll
    for (int c = 0; c < kPerLane; ++c) {
      const int e = lane + 32 * c;
      live[c] = e < E;
      val[c] = live[c] ? ls[tt * EP + e] : 0.f;
    }
    float sel_v[8];
    int sel_e[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      // best live candidate of this lane
      float bv = 0.f;
      int be = INT32_MAX;
#pragma unroll
      for (int c = 0; c < kPerLane; ++c) {
        const int e = lane + 32 * c;
        if (live[c] && (be == INT32_MAX || val[c] > bv)) { bv = val[c]; be = e; }
      }
      // warp arg-max: larger value wins, equal values go to the lower index
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        const bool take = (oe != INT32_MAX) &&
                          (be == INT32_MAX || ov > bv || (ov == bv && oe < be));
        if (take) { bv = ov; be = oe; }
      }
      sel_v[j] = bv;
      sel_e[j] = be;
#pragma unroll
      for (int c = 0; c < kPerLane; ++c)
        if (lane + 32 * c == be) live[c] = false;
    }
    if (lane == 0) {
      const float m = sel_v[0];
      float p[8], s = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j >= k) break;
        p[j] = expf(sel_v[j] - m);
        s += p[j];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j >= k) break;
        topk_idx[(size_t)t * k + j] = sel_e[j];
        topk_w[(size_t)t * k + j] = p[j] / s;
      }
    }
  }
}

template <int EP, int EPT, int TPT>
static cudaError_t launch_router(const __nv_bfloat16* x, const float* wr, const float* bias,
                                 int T, int d, int E, int k, float* logits, int32_t* idx,
                                 float* w, cudaStream_t s) {
  using S = RouterShape<EP, EPT, TPT>;
  const int grid = (T + S::BT - 1) / S::BT;
  router_topk_kernel<EP, EPT, TPT><<<grid, kRouterThreads, 0, s>>>(x, wr, bias, T, d, E, k,
                                                                    logits, idx, w);
  return cudaGetLastError();
}

cudaError_t launch_route(const __nv_bfloat16* x, const float* wr, const float* bias, int T,
                         int d, int E, int k, float* logits, int32_t* idx, float* w,
                         cudaStream_t s) {
  if (E <= 8) return launch_router<8, 2, 1>(x, wr, bias, T, d, E, k, logits, idx, w, s);
  if (E <= 16) return launch_router<16, 2, 2>(x, wr, bias, T, d, E, k, logits, idx, w, s);
  if (E <= 32) return launch_router<32, 4, 2>(x, wr, bias, T, d, E, k, logits, idx, w, s);
  if (E <= 64) return launch_router<64, 8, 2>(x, wr, bias, T, d, E, k, logits, idx, w, s);
  if (E <= 128) return launch_router<128, 8, 4>(x, wr, bias, T, d, E, k, logits, idx, w, s);
  return launch_router<256, 8, 4>(x, wr, bias, T, d, E, k, logits, idx, w, s);
}

}  // namespace moe
