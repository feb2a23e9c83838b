// Capacity-limited permutation of (token, expert) pairs into per-expert
// buckets, deterministic and in token order.
//
// Pairs are grouped by expert; an expert holds at most C pairs and the rest
// are dropped (inferensys.com "Expert Parallelism" glossary, Expert Capacity
// and Dropped Tokens entries); the token rows are permuted into that order
// before the experts run (klaylearn.com glossary, third paragraph).
//
// slot(t, j) = number of tokens t' < t that also chose expert e = topk_idx[t,j]
// (each expert appears at most once per token).  This is a stable counting
// sort keyed by expert, done in three launches:
//   1. rank:    per chunk of 256 tokens, the rank of each pair among the
//               chunk's pairs of the same expert (token order), plus the
//               chunk's per-expert histogram;
//   2. scan:    per expert, exclusive prefix of the histograms over chunks
//               (chunk bases), demand, kept = min(demand, C), offsets,
//               dropped-pair count;
//   3. scatter: slot = chunk base + rank; kept pairs copy their token row into
//               x_perm[offsets[e] + slot] with 16-byte vector loads/stores.
#include "common.cuh"

namespace moe {

constexpr int kChunk = 256;          // tokens per rank/histogram chunk
constexpr int kPermThreads = 256;    // 8 warps, 32 tokens each

__global__ void __launch_bounds__(kPermThreads)
    permute_rank_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                        int32_t* __restrict__ rank, int32_t* __restrict__ chunk_hist) {
  __shared__ int32_t cnt[kPermThreads / 32][256];
  __shared__ int32_t pairs[kChunk * 8];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int chunk_t0 = blockIdx.x * kChunk;
  const int nt = min(kChunk, T - chunk_t0);

  for (int i = tid; i < (kPermThreads / 32) * 256; i += kPermThreads) (&cnt[0][0])[i] = 0;
  for (int i = tid; i < nt * k; i += kPermThreads) pairs[i] = topk_idx[(size_t)chunk_t0 * k + i];
  __syncthreads();

  // each warp walks its 32 tokens in order; lane j handles pair j
  const int w_t0 = warp * 32;
  for (int i = 0; i < 32; ++i) {
    const int tt = w_t0 + i;
    if (tt < nt && lane < k) {
      const int e = pairs[tt * k + lane];
      const int r = cnt[warp][e];
      cnt[warp][e] = r + 1;        // experts are distinct within a token
      rank[(size_t)(chunk_t0 + tt) * k + lane] = r;
    }
    __syncwarp();
  }
  __syncthreads();

  // per expert: exclusive prefix over the warps, chunk total to global
  for (int e = tid; e < E; e += kPermThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kPermThreads / 32; ++w) {
      const int c = cnt[w][e];
      cnt[w][e] = run;
      run += c;
    }
    chunk_hist[(size_t)blockIdx.x * E + e] = run;
  }
  __syncthreads();

  // shift each pair's in-warp rank by its warp's base
  for (int i = tid; i < nt * k; i += kPermThreads) {
    const int tt = i / k;
    const int e = pairs[i];
    rank[(size_t)chunk_t0 * k + i] += cnt[tt / 32][e];
  }
}

// One CTA of 256 threads, thread e owns expert e.
__global__ void __launch_bounds__(256)
    permute_scan_kernel(int32_t* __restrict__ chunk_hist, int nchunks, int E, int64_t C,
                        int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                        int32_t* __restrict__ n_dropped) {
  __shared__ int32_t warp_sum[8];
  __shared__ int32_t warp_drop[8];
  const int e = threadIdx.x, lane = e % 32, warp = e / 32;
  int kept = 0, drop = 0;
  if (e < E) {
    int run = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int v = chunk_hist[(size_t)c * E + e];
      chunk_hist[(size_t)c * E + e] = run;
      run += v;
    }
    kept = (int64_t)run < C ? run : (int)C;
    drop = run - kept;
  }
  // block exclusive scan of kept, block sum of drop
  int incl = kept;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  int dsum = drop;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
  if (lane == 31) warp_sum[warp] = incl;
  if (lane == 0) warp_drop[warp] = dsum;
  __syncthreads();
  int base = 0, total = 0, dtotal = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    if (w < warp) base += warp_sum[w];
    total += warp_sum[w];
    dtotal += warp_drop[w];
  }
  if (e < E) {
    counts[e] = kept;
    offsets[e] = base + incl - kept;
  }
  if (e == 0) {
    offsets[E] = total;
    *n_dropped = dtotal;
  }
}

// One warp per token.
__global__ void __launch_bounds__(kPermThreads)
    permute_scatter_kernel(const __nv_bfloat16* __restrict__ x,
                           const int32_t* __restrict__ topk_idx, int32_t* __restrict__ slot,
                           const int32_t* __restrict__ chunk_base,
                           const int32_t* __restrict__ offsets, int T, int d, int E, int k,
                           int64_t C, int32_t* __restrict__ row_src,
                           __nv_bfloat16* __restrict__ x_perm) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * (kPermThreads / 32) + warp;
  if (t >= T) return;
  int my_row = -1;
  if (lane < k) {
    const size_t p = (size_t)t * k + lane;
    const int e = topk_idx[p];
    const int s = chunk_base[(size_t)(t / kChunk) * E + e] + slot[p];   // slot holds the rank
    const bool keep = (int64_t)s < C;
    slot[p] = keep ? s : -1;
    if (keep) {
      my_row = offsets[e] + s;
      row_src[my_row] = t;
    }
  }
  int rows[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);

  const int nvec = d / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
    uint4 val[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * 32;
      if (v < nvec) val[u] = __ldg(src + v);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      if (rows[j] < 0) continue;
      uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)rows[j] * d);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 32;
        if (v < nvec) dst[v] = val[u];
      }
    }
  }
}

size_t permute_scratch_bytes(int64_t T, int64_t E) {
  const int64_t nchunks = (T + kChunk - 1) / kChunk;
  return (size_t)(nchunks * E * (int64_t)sizeof(int32_t));
}

cudaError_t launch_permute(const __nv_bfloat16* x, const int32_t* topk_idx, int T, int d, int E,
                           int k, int64_t C, int32_t* counts, int32_t* offsets, int32_t* slot,
                           int32_t* row_src, __nv_bfloat16* x_perm, int32_t* n_dropped,
                           int32_t* chunk_hist, cudaStream_t s) {
  const int nchunks = (T + kChunk - 1) / kChunk;
  permute_rank_kernel<<<nchunks, kPermThreads, 0, s>>>(topk_idx, T, E, k, slot, chunk_hist);
  permute_scan_kernel<<<1, 256, 0, s>>>(chunk_hist, nchunks, E, C, counts, offsets, n_dropped);
  const int tokens_per_cta = kPermThreads / 32;
  permute_scatter_kernel<<<(T + tokens_per_cta - 1) / tokens_per_cta, kPermThreads, 0, s>>>(
      x, topk_idx, slot, chunk_hist, offsets, T, d, E, k, C, row_src, x_perm);
  return cudaGetLastError();
}

}  // namespace moe
