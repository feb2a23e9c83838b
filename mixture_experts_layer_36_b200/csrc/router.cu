// Router logits and top-k softmax gating.
//
// The router is a linear layer with one output score per expert; top-k gating
// keeps the k best-scoring experts and their scores become the mixing weights
// (inferensys.com "Expert Parallelism" glossary, gating-network and Top-k
// Gating entries; klaylearn.com glossary, third paragraph).
//
// logits = x Wr + bias is a dense contraction (T x d by d x E), so it runs on
// the tensor cores.  x is bf16 already; the fp32 router weight is split into
// two bf16 terms, Wr = hi + lo + r with hi = bf16(Wr), lo = bf16(Wr - hi) and
// |r| <= 2^-18 |Wr|, so x Wr = x hi + x lo up to that residual, with exact
// bf16 products and fp32 accumulation.  Three launches:
//   1. split:  Wr (fp32 [d,E]) -> W2 (bf16 [2d, Ep]), 64-row blocks of hi and
//              lo interleaved (hi block j at rows 128j.., lo block j at
//              rows 128j+64..), so the two k-blocks that share an x tile run
//              back to back; Ep = E rounded up to 64, padding zero;
//   2. GEMM:   persistent tcgen05 kernel over (row tile of 128 tokens, K split
//              s); each ring stage holds one 64-column x tile and both the hi
//              and the lo weight block for it (the x tile is loaded once for
//              the two terms); each tile accumulates x W2 in TMEM and writes
//              fp32 partial logits [S][T][E] (K is split so that small
//              batches still occupy every SM);
//   3. top-k:  per token, the S partials are summed in a fixed order, the bias
//              added, the fp32 logits written, and one warp runs k rounds of
//              a warp-wide arg-max (value descending, lower expert index on
//              equal values) on exactly those values; weights are the softmax
//              over the k selected logits.
// When K is not split (S = 1: batches of more row tiles than SMs), step 3 runs
// in the GEMM's epilogue instead: each thread owns one token's accumulator
// row, adds the bias, writes the logits and keeps the best experts by
// insertion in expert order (a strictly larger value moves ahead, so equal
// values keep the lower index first: the same selection), then the same
// softmax arithmetic.
#include "common.cuh"
#include "host_util.cuh"

namespace moe {

constexpr int kRBM = 128;
constexpr int kRBK = 64;
constexpr int kRThreads = 192;
constexpr int kRMaxSplitSMs = 256;     // upper bound on SMs, sizes the partials buffer

// ---------------------------------------------------------------- 1. split
// One thread per two adjacent columns of one weight row (d * Ep / 2 < 2^31:
// d <= 2^20 and Ep <= 256 are checked by the caller).
__global__ void __launch_bounds__(256)
    router_split_kernel(const float* __restrict__ wr, int d, int E, int Ep,
                        __nv_bfloat16* __restrict__ w2) {
  const int half = Ep / 2;
  const int n = d * half;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += gridDim.x * blockDim.x) {
    const int i = idx / half, e = 2 * (idx - i * half);
    const float w0 = e < E ? wr[(size_t)i * E + e] : 0.f;
    const float w1 = e + 1 < E ? wr[(size_t)i * E + e + 1] : 0.f;
    const __nv_bfloat162 hi = __floats2bfloat162_rn(w0, w1);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(w0 - __low2float(hi), w1 - __high2float(hi));
    const int blk = i / kRBK, r = i % kRBK;
    *reinterpret_cast<__nv_bfloat162*>(w2 + (size_t)(blk * 2 * kRBK + r) * Ep + e) = hi;
    *reinterpret_cast<__nv_bfloat162*>(w2 + (size_t)(blk * 2 * kRBK + kRBK + r) * Ep + e) = lo;
  }
}

// ---------------------------------------------------------------- 2. GEMM
template <int NCH>
struct RouterCfg {
  static constexpr int N = 64 * NCH;                      // MMA N = Ep
  static constexpr int kABytes = kRBM * kRBK * 2;         // x tile: 128 tokens x 64
  static constexpr int kChunkBytes = 2 * kRBK * 64 * 2;   // hi + lo rows of 64 columns
  static constexpr int kBBytes = NCH * kChunkBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStagesFit = (200 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kTmemCols = (2 * N <= 128) ? 128 : (2 * N <= 256 ? 256 : 512);
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kRBM, N, /*b_mn_major=*/true);
};

struct RouterShared {
  uint64_t full_bar[8];
  uint64_t empty_bar[8];
  uint64_t tfull_bar[2];
  uint64_t tempty_bar[2];
  uint64_t drain_bar;
  uint32_t tmem_base;
  int abort_flag;
  int never;
};

// Keeps the best 8 (value, expert) pairs in descending order; called in
// increasing expert order, a value enters ahead of a kept one only if it is
// strictly larger, so equal values stay ordered by expert index.  From the
// slot where it enters, the kept pairs behind it shift down one place each
// (a displaced pair stays ahead of every later pair of equal value).
__device__ __forceinline__ void topk_insert(float (&sv)[8], int (&se)[8], float v, int e) {
  if (se[7] >= 0 && !(v > sv[7])) return;
  bool shifting = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (shifting || se[i] < 0 || v > sv[i]) {
      const float tv = sv[i];
      const int te = se[i];
      sv[i] = v;
      se[i] = e;
      v = tv;
      e = te;
      shifting = true;
    }
  }
}

// TOPK (S = 1 only): the epilogue writes logits / topk_idx / topk_w itself.
template <int NCH, bool TOPK>
__global__ void __launch_bounds__(kRThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW, int T, int E, int S,
                       int kp_total, float* __restrict__ partial, int32_t* status,
                       const float* __restrict__ bias, int k, float* __restrict__ logits,
                       int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  using Cfg = RouterCfg<NCH>;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ RouterShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m_tiles = (T + kRBM - 1) / kRBM;
  const int total_tiles = m_tiles * S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&sh.full_bar[s], 1);
      mbar_init(&sh.empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh.tfull_bar[a], 1);
      mbar_init(&sh.tempty_bar[a], 4);
    }
    mbar_init(&sh.drain_bar, 1);
    sh.abort_flag = 0;
    sh.never = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh.tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  volatile int* abort_flag = &sh.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int it = 0;
      int last_it[8];
      for (int s = 0; s < Cfg::kStages; ++s) last_it[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const int sp = tile / m_tiles, m = tile - sp * m_tiles;
        const int kp0 = (int)((long long)sp * kp_total / S);
        const int kp1 = (int)((long long)(sp + 1) * kp_total / S);
        for (int kp = kp0; kp < kp1; ++kp, ++it) {
          const int st = it % Cfg::kStages;
          const uint32_t ph = (it / Cfg::kStages) & 1;
          if (!mbar_wait(&sh.empty_bar[st], ph ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + st * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          mbar_arrive_expect_tx(&sh.full_bar[st], Cfg::kStageBytes);
          tma_load_2d(sa, &tmX, &sh.full_bar[st], kp * kRBK, m * kRBM);
          // W2 rows 128 kp .. 128 kp + 127: the hi block, then the lo block
#pragma unroll
          for (int c = 0; c < NCH; ++c)
            tma_load_2d(sb + c * Cfg::kChunkBytes, &tmW, &sh.full_bar[st], c * 64, kp * 2 * kRBK);
          last_it[st] = it;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        report(status, kDevErrWaitTimeout);
      }
      for (int st = 0; st < Cfg::kStages; ++st)
        if (last_it[st] >= 0)
          mbar_wait(&sh.full_bar[st], (last_it[st] / Cfg::kStages) & 1, &sh.never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++lt) {
        const int sp = tile / m_tiles;
        const int kp0 = (int)((long long)sp * kp_total / S);
        const int kp1 = (int)((long long)(sp + 1) * kp_total / S);
        const int a = lt & 1;
        const uint32_t aph = (lt >> 1) & 1;
        if (!mbar_wait(&sh.tempty_bar[a], aph ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * Cfg::N);
        for (int kp = kp0; kp < kp1; ++kp, ++it) {
          const int st = it % Cfg::kStages;
          const uint32_t ph = (it / Cfg::kStages) & 1;
          if (!mbar_wait(&sh.full_bar[st], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + st * Cfg::kStageBytes);
          const uint32_t b_addr = a_addr + Cfg::kABytes;
          // B MN-major: 64-column groups kChunkBytes apart, 8-row K groups 1 KB
          // apart; the lo block starts 64 K-rows (8 KB) into each group
#pragma unroll
          for (int ks = 0; ks < kRBK / 16; ++ks) {
            const uint64_t adesc = smem_desc_sw128(a_addr + ks * 32, 16, 1024);
            const uint64_t bhi = smem_desc_sw128(b_addr + ks * 2048, Cfg::kChunkBytes, 1024);
            const uint64_t blo = smem_desc_sw128(b_addr + 8192 + ks * 2048, Cfg::kChunkBytes, 1024);
            umma_bf16(d_tmem, adesc, bhi, Cfg::kIdesc, (kp != kp0 || ks != 0) ? 1u : 0u);
            umma_bf16(d_tmem, adesc, blo, Cfg::kIdesc, 1u);
          }
          umma_commit(&sh.empty_bar[st]);
        }
        if (!ok) break;
        umma_commit(&sh.tfull_bar[a]);
      }
      if (!ok) {
        *abort_flag = 1;
        report(status, kDevErrWaitTimeout);
      }
      umma_commit(&sh.drain_bar);
      mbar_wait(&sh.drain_bar, 0, &sh.never);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    int lt = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++lt) {
      const int sp = tile / m_tiles, m = tile - sp * m_tiles;
      const int a = lt & 1;
      const uint32_t aph = (lt >> 1) & 1;
      if (!mbar_wait(&sh.tfull_bar[a], aph, abort_flag)) {
        *abort_flag = 1;
        report(status, kDevErrWaitTimeout);
        break;
      }
      tc_fence_after();
      const int row = m * kRBM + q * 32 + lane;
      const bool valid = row < T;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * Cfg::N);
      if constexpr (TOPK) {
        float sv[8];
        int se[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          sv[j] = 0.f;
          se[j] = -1;
        }
        float* lrow = logits + (size_t)row * E;
#pragma unroll 1
        for (int c = 0; c < Cfg::N / 32; ++c) {
          if (c * 32 >= E) break;                   // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c * 32, v);
          tmem_ld_wait();
          float l[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = c * 32 + i;
            l[i] = 0.f;                             // the same sum as the split-K path
            l[i] += __uint_as_float(v[i]);
            if (bias && e < E) l[i] += __ldg(bias + e);
          }
          if (valid) {
            if ((E & 31) == 0) {
              float4* dst = reinterpret_cast<float4*>(lrow + c * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(l[4 * i], l[4 * i + 1], l[4 * i + 2], l[4 * i + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c * 32 + i < E) lrow[c * 32 + i] = l[i];
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i < E) topk_insert(sv, se, l[i], c * 32 + i);
          }
        }
        if (valid) {
          const float mx = sv[0];
          float p[8], sum = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j >= k) break;
            p[j] = expf(sv[j] - mx);
            sum += p[j];
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j >= k) break;
            topk_idx[(size_t)row * k + j] = se[j];
            topk_w[(size_t)row * k + j] = p[j] / sum;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.tempty_bar[a]);
        continue;
      }
      float* prow = partial + ((size_t)sp * T + row) * E;
#pragma unroll 1
      for (int c = 0; c < Cfg::N / 32; ++c) {
        if (c * 32 >= E) break;                     // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c * 32, v);
        tmem_ld_wait();
        if (valid) {
          if ((E & 31) == 0) {
            uint4* dst = reinterpret_cast<uint4*>(prow + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i < E) prow[c * 32 + i] = __uint_as_float(v[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tempty_bar[a]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------- 3. top-k
// 256 threads.  tpc tokens per CTA (8 when S < 8: one warp per token; 1 when
// S >= 8: the 8 warps split the partial sums of one token, combined in warp
// order through shared memory).
template <int EP>
__global__ void __launch_bounds__(256)
    router_topk_kernel(const float* __restrict__ partial, int S, const float* __restrict__ bias,
                       int T, int E, int k, int tpc, float* __restrict__ logits,
                       int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  constexpr int kPerLane = EP / 32;
  __shared__ float red[8][EP];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int wpt = 8 / tpc;
  const int tok = warp / wpt, part = warp % wpt;
  const int t = blockIdx.x * tpc + tok;
  float v[kPerLane];
#pragma unroll
  for (int c = 0; c < kPerLane; ++c) v[c] = 0.f;
  if (t < T) {
    for (int s = part; s < S; s += wpt) {
      const float* p = partial + ((size_t)s * T + t) * E;
#pragma unroll
      for (int c = 0; c < kPerLane; ++c) {
        const int e = lane + 32 * c;
        if (e < E) v[c] += p[e];
      }
    }
  }
  if (wpt > 1) {
#pragma unroll
    for (int c = 0; c < kPerLane; ++c) red[warp][lane + 32 * c] = v[c];
    __syncthreads();
    if (part == 0) {
      for (int w = 1; w < wpt; ++w)
#pragma unroll
        for (int c = 0; c < kPerLane; ++c) v[c] += red[warp + w][lane + 32 * c];
    }
  }
  if (part != 0 || t >= T) return;

  bool live[kPerLane];
#pragma unroll
  for (int c = 0; c < kPerLane; ++c) {
    const int e = lane + 32 * c;
    live[c] = e < E;
    if (live[c]) {
      if (bias) v[c] += bias[e];
      logits[(size_t)t * E + e] = v[c];
    }
  }
  float sel_v[8];
  int sel_e[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    float bv = 0.f;
    int be = INT32_MAX;
#pragma unroll
    for (int c = 0; c < kPerLane; ++c) {
      const int e = lane + 32 * c;
      if (live[c] && (be == INT32_MAX || v[c] > bv)) { bv = v[c]; be = e; }
    }
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
    const float mx = sel_v[0];
    float p[8], sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      p[j] = expf(sel_v[j] - mx);
      sum += p[j];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      topk_idx[(size_t)t * k + j] = sel_e[j];
      topk_w[(size_t)t * k + j] = p[j] / sum;
    }
  }
}

// ---------------------------------------------------------------- host side

static int round_up(int v, int m) { return (v + m - 1) / m * m; }

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// K splits for a batch: enough (row tile, split) tiles to occupy `sms` SMs,
// at most one split per 64-column x block.
static int route_splits(int T, int d, int sms) {
  const int m_tiles = (T + kRBM - 1) / kRBM;
  const int kp_total = d / kRBK;
  int S = sms / m_tiles;
  if (S < 1) S = 1;
  if (S > kp_total) S = kp_total;
  return S;
}

size_t route_scratch_bytes(int64_t T, int64_t d, int64_t E) {
  const int Ep = round_up((int)E, 64);
  const size_t w2 = align256((size_t)2 * d * Ep * 2);
  const int S = route_splits((int)T, (int)d, kRMaxSplitSMs);
  return w2 + align256((size_t)S * T * E * sizeof(float));
}

template <int NCH, bool TOPK>
static cudaError_t launch_router_gemm(DeviceInfo* di, const CUtensorMap& tx,
                                      const CUtensorMap& tw, int T, int E, int S, int kp_total,
                                      float* partial, int32_t* status, const float* bias, int k,
                                      float* logits, int32_t* idx, float* w, cudaStream_t s) {
  using Cfg = RouterCfg<NCH>;
  auto kern = router_gemm_kernel<NCH, TOPK>;
  const int slot = TOPK ? 18 + NCH : 2 + NCH;    // attribute slots 3..6, 19..22
  if (!di->attr_set[slot]) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           Cfg::kSmemBytes);
    if (err != cudaSuccess) return err;
    di->attr_set[slot] = true;
  }
  const int tiles = ((T + kRBM - 1) / kRBM) * S;
  const int grid = tiles < di->sms ? tiles : di->sms;
  kern<<<grid, kRThreads, Cfg::kSmemBytes, s>>>(tx, tw, T, E, S, kp_total, partial, status,
                                                bias, k, logits, idx, w);
  return cudaGetLastError();
}

template <int NCH>
static cudaError_t launch_router_gemm_s(DeviceInfo* di, const CUtensorMap& tx,
                                        const CUtensorMap& tw, int T, int E, int S, int kp_total,
                                        float* partial, int32_t* status, const float* bias,
                                        int k, float* logits, int32_t* idx, float* w,
                                        cudaStream_t s) {
  if (S == 1)
    return launch_router_gemm<NCH, true>(di, tx, tw, T, E, S, kp_total, partial, status, bias,
                                         k, logits, idx, w, s);
  return launch_router_gemm<NCH, false>(di, tx, tw, T, E, S, kp_total, partial, status, bias, k,
                                        logits, idx, w, s);
}

template <int EP>
static cudaError_t launch_topk(const float* partial, int S, const float* bias, int T, int E,
                               int k, float* logits, int32_t* idx, float* w, cudaStream_t s) {
  const int tpc = S >= 8 ? 1 : 8;
  router_topk_kernel<EP><<<(T + tpc - 1) / tpc, 256, 0, s>>>(partial, S, bias, T, E, k, tpc,
                                                              logits, idx, w);
  return cudaGetLastError();
}

cudaError_t launch_route(const __nv_bfloat16* x, const float* wr, const float* bias, int T,
                         int d, int E, int k, float* logits, int32_t* idx, float* w,
                         void* scratch, int32_t* status, cudaStream_t s, bool* map_failed) {
  *map_failed = false;
  DeviceInfo* di = nullptr;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int Ep = round_up(E, 64);
  const int NCH = Ep / 64;
  __nv_bfloat16* w2 = static_cast<__nv_bfloat16*>(scratch);
  float* partial = reinterpret_cast<float*>(static_cast<char*>(scratch) +
                                            align256((size_t)2 * d * Ep * 2));
  int S = route_splits(T, d, di->sms < kRMaxSplitSMs ? di->sms : kRMaxSplitSMs);
  const int kp_total = d / kRBK;

  const int n = d * (Ep / 2);
  int blocks = (n + 255) / 256;
  if (blocks > 8 * di->sms) blocks = 8 * di->sms;
  router_split_kernel<<<blocks, 256, 0, s>>>(wr, d, E, Ep, w2);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;

  CUtensorMap tx, tw;
  if (!map_rows(&tx, x, d, T, kRBM) || !map_rows(&tw, w2, Ep, 2 * (uint64_t)d, 2 * kRBK)) {
    *map_failed = true;
    return cudaSuccess;
  }
  switch (NCH) {
    case 1:
      err = launch_router_gemm_s<1>(di, tx, tw, T, E, S, kp_total, partial, status, bias, k,
                                    logits, idx, w, s);
      break;
    case 2:
      err = launch_router_gemm_s<2>(di, tx, tw, T, E, S, kp_total, partial, status, bias, k,
                                    logits, idx, w, s);
      break;
    case 3:
      err = launch_router_gemm_s<3>(di, tx, tw, T, E, S, kp_total, partial, status, bias, k,
                                    logits, idx, w, s);
      break;
    default:
      err = launch_router_gemm_s<4>(di, tx, tw, T, E, S, kp_total, partial, status, bias, k,
                                    logits, idx, w, s);
      break;
  }
  if (err != cudaSuccess || S == 1) return err;
  if (E <= 32) return launch_topk<32>(partial, S, bias, T, E, k, logits, idx, w, s);
  if (E <= 64) return launch_topk<64>(partial, S, bias, T, E, k, logits, idx, w, s);
  if (E <= 128) return launch_topk<128>(partial, S, bias, T, E, k, logits, idx, w, s);
  return launch_topk<256>(partial, S, bias, T, E, k, logits, idx, w, s);
}

}  // namespace moe
