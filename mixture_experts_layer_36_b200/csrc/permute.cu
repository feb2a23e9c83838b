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
// sort keyed by expert, in three launches:
//   1. rank:    per chunk of 256 tokens, the rank of each pair among the
//               chunk's pairs of the same expert (token order), plus the
//               chunk's per-expert histogram;
//   2. scan:    per expert, the exclusive prefix of the histograms over the
//               chunks (each chunk's base, written over its histogram) and
//               the total demand (one extra row) — one pass, linear in T;
//               skipped when there are at most kDirectSum histogram counters:
//               each scatter CTA then sums them itself, which costs less than
//               one more launch in the chain;
//   3. scatter: per CTA of 8 tokens, kept = min(demand, C), offsets
//               (exclusive scan over experts) and slot = chunk base + rank;
//               kept pairs copy their token row into x_perm[offsets[e] + slot]
//               with 16-byte vector loads and stores.
// The launches are chained with programmatic dependent launch: the scatter
// CTAs start while the rank and scan kernels run and pull their token rows
// into L2 (bulk prefetch), so the row reads overlap the index work.
// Rows are moved as bytes: bf16 rows, or e4m3 rows with their fp32 scale
// (the FP8 layer quantizes each token once, before the permutation).
#include "common.cuh"
#include "host_util.cuh"

namespace moe {

constexpr int kChunk = 256;            // tokens per rank/histogram chunk
constexpr int kRankThreads = 1024;     // 32 warps x 8 tokens per chunk
constexpr int kRankWarps = kRankThreads / 32;
constexpr int kTokPerWarp = kChunk / kRankWarps;
constexpr int kScanThreads = 1024;     // 32 warps; lane = one expert of a group of 32
constexpr int kScatThreads = 256;      // 8 warps: thread e derives expert e's offsets
// tokens per scatter CTA, one per warp (divides kChunk): 4 keeps the staged
// rows of a CTA at 4 x row bytes, so that 8 KB rows still let 7 CTAs share
// an SM and a 4096-token batch runs in one wave
constexpr int kScatTokens = 4;
constexpr int kDirectSum = 4096;       // histogram counters a scatter CTA sums without the scan
constexpr int kBulkRowBytes = 16384;   // rows up to this size move through shared memory

// 1. rank: per chunk, the rank of each pair among the chunk's pairs of the
//    same expert (token order), and the chunk's per-expert histogram.
__global__ void __launch_bounds__(kRankThreads)
    permute_rank_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                        int32_t* __restrict__ rank, int32_t* __restrict__ chunk_hist,
                        int32_t* status) {
  __shared__ int32_t cnt[kRankWarps][256];
  __shared__ int32_t pairs[kChunk * 8];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int chunk_t0 = blockIdx.x * kChunk;
  const int nt = min(kChunk, T - chunk_t0);

  for (int i = tid; i < kRankWarps * 256; i += kRankThreads) (&cnt[0][0])[i] = 0;
  grid_dep_wait();          // topk_idx (and x) may come from the kernel before
  // only now may the scan and scatter start: the scatter reads x before it
  // waits, so every kernel before this permutation must have completed
  grid_dep_launch();
  for (int i = tid; i < nt * k; i += kRankThreads) pairs[i] = topk_idx[(size_t)chunk_t0 * k + i];
  __syncthreads();

  // each warp walks its 8 tokens in order; lane j handles pair j.  An expert
  // id outside [0, E) (only possible for caller-given top-k tables) takes no
  // bucket place: the scatter marks the pair dropped.
  const int w_t0 = warp * kTokPerWarp;
#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i) {
    const int tt = w_t0 + i;
    if (tt < nt && lane < k) {
      const int e = pairs[tt * k + lane];
      int r = -1;
      if (e >= 0 && e < E) {
        r = cnt[warp][e];
        cnt[warp][e] = r + 1;      // experts are distinct within a token
      } else {
        report(status, kDevErrBadRouting);
      }
#ifdef MOE_CHECKS
      // checked builds: an expert listed twice for one token is reported
      for (int j = 0; j < lane; ++j)
        if (pairs[tt * k + j] == e) report(status, kDevErrBadRouting);
#endif
      rank[(size_t)(chunk_t0 + tt) * k + lane] = r;
    }
    __syncwarp();
  }
  __syncthreads();

  // per expert: exclusive prefix over the warps, chunk total to global
  for (int e = tid; e < E; e += kRankThreads) {
    int run = 0;
#pragma unroll 8
    for (int w = 0; w < kRankWarps; ++w) {
      const int c = cnt[w][e];
      cnt[w][e] = run;
      run += c;
    }
    chunk_hist[(size_t)blockIdx.x * E + e] = run;
  }
  __syncthreads();

  for (int i = tid; i < nt * k; i += kRankThreads) {
    const int tt = i / k;
    const int e = pairs[i];
    if (e >= 0 && e < E) rank[(size_t)chunk_t0 * k + i] += cnt[tt / kTokPerWarp][e];
  }
}

// 2. scan: per expert e (lane of a warp; 32 experts per CTA), the exclusive
//    prefix of chunk_hist[., e] over the chunks, written in place, and the
//    total demand in row nchunks.  Warp w takes a contiguous range of chunks:
//    range sums, a prefix over the warps in shared memory, then the range is
//    rewritten with its running prefix.
__global__ void __launch_bounds__(kScanThreads)
    permute_scan_kernel(int32_t* __restrict__ chunk_hist, int nchunks, int E) {
  __shared__ int32_t part[32][33];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int e = blockIdx.x * 32 + lane;
  const int per = (nchunks + 31) / 32;
  const int c0 = min(nchunks, warp * per), c1 = min(nchunks, c0 + per);
  grid_dep_launch();
  grid_dep_wait();          // the rank kernel's histograms
  int sum = 0;
  if (e < E)
    for (int c = c0; c < c1; ++c) sum += chunk_hist[(size_t)c * E + e];
  part[warp][lane] = sum;
  __syncthreads();
  int run = 0;
  for (int w = 0; w < warp; ++w) run += part[w][lane];
  if (e < E) {
    for (int c = c0; c < c1; ++c) {
      const size_t i = (size_t)c * E + e;
      const int v = chunk_hist[i];
      chunk_hist[i] = run;
      run += v;
    }
    if (warp == 31) chunk_hist[(size_t)nchunks * E + e] = run;
  }
}

// 3. scatter: every CTA (8 tokens of one chunk) reads the per-expert demand
//    and its chunk's base, derives kept counts and offsets (exclusive scan
//    over experts); CTA 0 also writes counts / offsets / n_dropped.  Then one
//    warp per token (the first kScatTokens warps) turns ranks into slots,
//    drops pairs at slot >= C, and copies the token row to its kept rows.  Rows of up to kBulkRowBytes go
//    through shared memory by bulk copy: each warp's lane 0 loads its token's
//    row before waiting for the rank kernel (the read overlaps it), then
//    stores it to the k destination rows; longer rows are copied with
//    16-byte vector loads and stores.
__global__ void __launch_bounds__(kScatThreads)
    permute_scatter_kernel(const uint8_t* __restrict__ x, int row_bytes, bool bulk,
                           const float* __restrict__ x_scale,
                           const int32_t* __restrict__ topk_idx, int32_t* __restrict__ slot,
                           const int32_t* __restrict__ chunk_base, bool scanned,
                           int nchunks, int T, int E, int k, int64_t C,
                           int32_t* __restrict__ counts,
                           int32_t* __restrict__ offsets, int32_t* __restrict__ n_dropped,
                           int32_t* __restrict__ row_src, uint8_t* __restrict__ x_perm,
                           float* __restrict__ perm_scale, bool padded,
                           int32_t* __restrict__ row_pair, float* __restrict__ zero_rows,
                           int zero_cols, int32_t* status) {
  extern __shared__ __align__(128) uint8_t s_rows[];   // bulk: one row per warp
  __shared__ int32_t s_off[256];
  __shared__ int32_t s_base[256];
  __shared__ int32_t warp_sum[8];
  __shared__ int32_t warp_drop[8];
  __shared__ uint64_t row_bar[kScatTokens];
  __shared__ int never;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t0 = blockIdx.x * kScatTokens;
  const int my_chunk = t0 / kChunk;
  // the token this warp copies (warps past kScatTokens only help with the offsets)
  const int t_own = warp < kScatTokens ? t0 + warp : T;
  uint8_t* my_row_sh = s_rows + (size_t)(warp < kScatTokens ? warp : 0) * row_bytes;

  // this CTA's token rows (inputs, not produced by the kernels before) start
  // moving while the rank and scan kernels finish
  if (x && lane == 0 && t_own < T) {
    if (bulk) {
      never = 0;
      mbar_init(&row_bar[warp], 1);
      fence_barrier_init();
      mbar_arrive_expect_tx(&row_bar[warp], (uint32_t)row_bytes);
      bulk_load(my_row_sh, x + (size_t)t_own * row_bytes, (uint32_t)row_bytes, &row_bar[warp]);
    } else {
      prefetch_l2_bulk(x + (size_t)t_own * row_bytes, row_bytes);
    }
  }
  grid_dep_launch();
  grid_dep_wait();          // ranks in slot, chunk bases and totals

  // ---- per-expert totals, kept, chunk base (thread e owns expert e): from
  //      the scan's rows, or summed here over the (few) chunk histograms
  int kept = 0, drop = 0;
  if (tid < E) {
    int total = 0, base = 0;
    if (scanned) {
      total = chunk_base[(size_t)nchunks * E + tid];
      base = chunk_base[(size_t)my_chunk * E + tid];
    } else {
      for (int c = 0; c < nchunks; ++c) {
        const int v = chunk_base[(size_t)c * E + tid];
        if (c < my_chunk) base += v;
        total += v;
      }
    }
    s_base[tid] = base;
    kept = (int64_t)total < C ? total : (int)C;
    drop = total - kept;
  }
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
  int wbase = 0, total_rows = 0, dtotal = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    if (w < warp) wbase += warp_sum[w];
    total_rows += warp_sum[w];
    dtotal += warp_drop[w];
  }
  // ragged: buckets packed back to back; padded: bucket e starts at row e*C
  const int my_off = padded ? (int)((int64_t)tid * C) : wbase + incl - kept;
  if (tid < E) s_off[tid] = my_off;
  if (blockIdx.x == 0) {
    if (tid < E) {
      counts[tid] = kept;
      offsets[tid] = my_off;
    }
    if (tid == 0) {
      offsets[E] = padded ? (int)((int64_t)E * C) : total_rows;
      *n_dropped = dtotal;
    }
  }
  __syncthreads();

  // ---- one warp per token
  static_assert(kScatTokens <= kScatThreads / 32, "one token per warp");
  const int nvec = row_bytes / 16;
  {
    const int t = t_own;
    if (t >= T) return;
    int my_row = -1;
    if (lane < k) {
      const size_t p = (size_t)t * k + lane;
      const int e = topk_idx[p];
      const bool valid = e >= 0 && e < E;          // else dropped (rank kernel: -1)
      const int sl = valid ? s_base[e] + slot[p] : 0;   // slot holds the in-chunk rank
      const bool keep = valid && (int64_t)sl < C;
      slot[p] = keep ? sl : -1;
      if (keep) {
        my_row = s_off[e] + sl;
        row_src[my_row] = t;
        if (row_pair) row_pair[my_row] = t * k + lane;
        if (x_scale) perm_scale[my_row] = x_scale[t];
      }
    }
    if (zero_rows) {          // the fused combine's fp32 accumulator row of t
      float4* z = reinterpret_cast<float4*>(zero_rows + (size_t)t * zero_cols);
      for (int v = lane; v < zero_cols / 4; v += 32) z[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (!x) return;           // index-only: the GEMM gathers the rows itself
    int rows[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);

    if (bulk) {
      if (lane == 0) {
        // the row landed in shared memory: store it to each kept row
        if (!mbar_wait(&row_bar[warp], 0, &never)) {
          report(status, kDevErrWaitTimeout);
          mbar_wait(&row_bar[warp], 0, &never);     // the copy in flight must land
          return;
        }
        fence_proxy_async_smem();
        for (int j = 0; j < k; ++j)
          if (rows[j] >= 0)
            bulk_store(x_perm + (size_t)rows[j] * row_bytes, my_row_sh, (uint32_t)row_bytes);
        bulk_commit();
        bulk_wait_all();      // shared memory is read before the CTA exits
      }
      return;
    }

    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * row_bytes);
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
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)rows[j] * row_bytes);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * 32;
          if (v < nvec) dst[v] = val[u];
        }
      }
    }
  }
}

// Scratch: the per-chunk histograms (then bases) and one row of totals.
size_t permute_scratch_bytes(int64_t T, int64_t E) {
  const int64_t nchunks = (T + kChunk - 1) / kChunk;
  return (size_t)((nchunks + 1) * E * (int64_t)sizeof(int32_t));
}

// 3. padded layout only: rows of each bucket past its kept count are zeroed
//    (row_src = -1), one warp per padded row.
__global__ void __launch_bounds__(256)
    permute_pad_fill_kernel(const int32_t* __restrict__ counts, int E, int64_t C, int row_bytes,
                            int32_t* __restrict__ row_src, uint8_t* __restrict__ x_pad) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t r = (int64_t)blockIdx.x * 8 + warp;
  grid_dep_wait();          // the scatter's counts
  if (r >= (int64_t)E * C) return;
  const int e = (int)(r / C);
  if (r - (int64_t)e * C < counts[e]) return;
  if (lane == 0) row_src[r] = -1;
  uint4* dst = reinterpret_cast<uint4*>(x_pad + r * row_bytes);
  for (int v = lane; v < row_bytes / 16; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
}

// Rows of row_bytes bytes (a multiple of 16); x_scale / perm_scale (one fp32
// per row, moved with it) may be null; x null: no row copy (index-only), with
// row_pair (t*k + j of each kept row) and zeroed fp32 rows zero_rows[T,
// zero_cols] for the fused combine when those are non-null.
// The rank kernel, and the scan kernel when the histograms are many;
// *scanned tells the scatter which it gets.
static cudaError_t launch_rank_scan(const int32_t* topk_idx, int T, int E, int k, int32_t* slot,
                                    int32_t* chunk_hist, cudaStream_t s, int32_t* status,
                                    bool* scanned) {
  const int nchunks = (T + kChunk - 1) / kChunk;
  cudaError_t err = launch_dependent(permute_rank_kernel, dim3(nchunks), dim3(kRankThreads), 0, s,
                                     topk_idx, T, E, k, slot, chunk_hist, status);
  *scanned = (int64_t)nchunks * E > kDirectSum;
  if (err != cudaSuccess || !*scanned) return err;
  return launch_dependent(permute_scan_kernel, dim3((E + 31) / 32), dim3(kScanThreads), 0, s,
                          chunk_hist, nchunks, E);
}

// The scatter launch: rows staged through shared memory (bulk copies) when
// they fit kBulkRowBytes, one row per warp.
static cudaError_t launch_scatter(const uint8_t* x, int row_bytes, const float* x_scale,
                                  const int32_t* topk_idx, int32_t* slot,
                                  const int32_t* chunk_hist, bool scanned, int T, int E, int k,
                                  int64_t C, int32_t* counts, int32_t* offsets,
                                  int32_t* n_dropped, int32_t* row_src, uint8_t* x_perm,
                                  float* perm_scale, bool padded, int32_t* row_pair,
                                  float* zero_rows, int zero_cols, int32_t* status,
                                  cudaStream_t s) {
  DeviceInfo* di = nullptr;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  constexpr int kSlot = 24;                 // attribute slot of the scatter kernel
  const bool bulk = x != nullptr && row_bytes <= kBulkRowBytes;
  const size_t smem = bulk ? (size_t)kScatTokens * row_bytes : 0;
  if (bulk && !di->attr_set[kSlot]) {
    err = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kScatTokens * kBulkRowBytes);
    if (err != cudaSuccess) return err;
    di->attr_set[kSlot] = true;
  }
  const int nchunks = (T + kChunk - 1) / kChunk;
  return launch_dependent(permute_scatter_kernel, dim3((T + kScatTokens - 1) / kScatTokens),
                          dim3(kScatThreads), smem, s, x, row_bytes, bulk, x_scale, topk_idx,
                          slot, chunk_hist, scanned, nchunks, T, E, k, C, counts, offsets,
                          n_dropped, row_src, x_perm, perm_scale, padded, row_pair, zero_rows,
                          zero_cols, status);
}

cudaError_t launch_permute_rows(const uint8_t* x, int row_bytes, const float* x_scale,
                                const int32_t* topk_idx, int T, int E, int k, int64_t C,
                                int32_t* counts, int32_t* offsets, int32_t* slot,
                                int32_t* row_src, uint8_t* x_perm, float* perm_scale,
                                int32_t* n_dropped, int32_t* chunk_hist, cudaStream_t s,
                                int32_t* row_pair, float* zero_rows, int zero_cols,
                                int32_t* status) {
  bool scanned = false;
  cudaError_t err = launch_rank_scan(topk_idx, T, E, k, slot, chunk_hist, s, status, &scanned);
  if (err != cudaSuccess) return err;
  return launch_scatter(x, row_bytes, x_scale, topk_idx, slot, chunk_hist, scanned, T, E, k, C,
                        counts, offsets, n_dropped, row_src, x_perm, perm_scale, false, row_pair,
                        zero_rows, zero_cols, status, s);
}

// The padded [E, C, d] layout: bucket e holds rows e*C .. e*C + C - 1, its
// kept pairs first (in slot order), the rest zero.
cudaError_t launch_permute_padded(const __nv_bfloat16* x, const int32_t* topk_idx, int T, int d,
                                  int E, int k, int64_t C, int32_t* counts, int32_t* offsets,
                                  int32_t* slot, int32_t* row_src, __nv_bfloat16* x_pad,
                                  int32_t* n_dropped, int32_t* chunk_hist, cudaStream_t s,
                                  int32_t* status) {
  bool scanned = false;
  cudaError_t err = launch_rank_scan(topk_idx, T, E, k, slot, chunk_hist, s, status, &scanned);
  if (err != cudaSuccess) return err;
  uint8_t* xp = reinterpret_cast<uint8_t*>(x_pad);
  err = launch_scatter(reinterpret_cast<const uint8_t*>(x), d * 2, nullptr, topk_idx, slot,
                       chunk_hist, scanned, T, E, k, C, counts, offsets, n_dropped, row_src, xp,
                       nullptr, true, nullptr, nullptr, 0, status, s);
  if (err != cudaSuccess) return err;
  const int64_t rows = (int64_t)E * C;
  return launch_dependent(permute_pad_fill_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0,
                          s, counts, E, C, d * 2, row_src, xp);
}

cudaError_t launch_permute(const __nv_bfloat16* x, const int32_t* topk_idx, int T, int d, int E,
                           int k, int64_t C, int32_t* counts, int32_t* offsets, int32_t* slot,
                           int32_t* row_src, __nv_bfloat16* x_perm, int32_t* n_dropped,
                           int32_t* chunk_hist, cudaStream_t s, int32_t* status) {
  return launch_permute_rows(reinterpret_cast<const uint8_t*>(x), d * 2, nullptr, topk_idx, T, E,
                             k, C, counts, offsets, slot, row_src,
                             reinterpret_cast<uint8_t*>(x_perm), nullptr, n_dropped, chunk_hist,
                             s, nullptr, nullptr, 0, status);
}

}  // namespace moe
