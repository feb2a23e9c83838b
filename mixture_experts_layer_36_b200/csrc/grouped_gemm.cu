// Grouped expert GEMMs over ragged per-expert buckets on the sm_100a tensor
// cores (tcgen05.mma, accumulators in TMEM, operands staged by TMA).
//
// Experts are gate/up/down MLPs ("Expert Parallelism & All-to-All"
// (neelmishra.github.io), section "Tensor parallelism for experts"); the
// per-expert matmuls over the token buckets are grouped GEMMs (klaylearn.com
// "Expert Parallelism" glossary, fourth paragraph).
//
//   GEMM 1 (SWIGLU = true):  h[r, :]      = silu(x_perm[r] Wg[e]) * (x_perm[r] Wu[e])
//   GEMM 2 (SWIGLU = false): y_perm[r, :] = h[r] Wd[e]      (stored fp32)
// for every row r of bucket e (offsets[e] <= r < offsets[e+1]).
//
// Tiling.  A tile is 128 bucket rows x BN accumulator columns.  GEMM 1 puts the
// gate and the up projection of the same 128 h-columns side by side in one
// N = 256 MMA (accumulator columns [0,128) = gate, [128,256) = up), so the
// SwiGLU is an epilogue over one TMEM tile.  A (rows, K-contiguous) is loaded
// K-major; B is the weight [K, N] with N contiguous, loaded and consumed
// MN-major, so the weights are used in the layout they are given.
//
// Schedule.  Persistent CTAs (one per SM) walk a tile list built on the device
// from `offsets` (no host sync): per-expert tile counts ceil(n_e/128) x
// n_tiles are prefix-summed in shared memory and tile i is decoded by binary
// search.  Inside an expert the row tile varies fastest, so CTAs running at
// the same time share each weight tile through L2.
//
// Roles (320 threads): warp 0 lane 0 issues TMA into a ring of smem stages,
// warp 1 lane 0 issues tcgen05.mma into one of two TMEM accumulators, warps
// 2..9 drain the other accumulator (tcgen05.ld -> SwiGLU -> bf16 stores), so
// the epilogue of tile i overlaps the main loop of tile i+1.
//
// FP8 experts (grouped_gemm_e4m3_kernel): the same tiles and roles on e4m3
// activations and weights (tcgen05.mma.kind::f8f6f4), the per-row and
// per-column fp32 quantization scales applied to the accumulators.
//
// Every mbarrier wait is time-limited: a role that gives up sets the CTA's
// abort flag and the caller's status bit, the others notice and stop, the
// producer waits for its copies in flight, the MMA issuer waits for its MMAs,
// and TMEM is freed before the CTA exits.
#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "host_util.cuh"

namespace moe {

constexpr int kBM = 128;
constexpr int kBK = 64;                 // one 128-byte swizzle atom of bf16 along K
// Threads: warp 0 producer, warp 1 MMA issuer, then the epilogue warps.
// Each accumulator is drained by 8 epilogue warps, two per TMEM lane quarter
// on alternate 32-column chunks, so that short-K shapes are not bound by the
// epilogue.  The fp32 (down GEMM) epilogue stages rows through one padded
// 16-row shared tile per warp.
constexpr int kEpiWarps = 8;
__host__ __device__ constexpr int epi_warps(bool) { return kEpiWarps; }
__host__ __device__ constexpr int gemm_threads(bool swiglu) { return 64 + 32 * epi_warps(swiglu); }
constexpr int kChunkBytes = 64 * kBK * 2;   // one B chunk: 64 N x 64 K bf16 = 8 KB

// ---------------------------------------------------------------- epilogue stores
// Each epilogue thread owns one accumulator row; a warp owns 32 rows.  fp32
// rows are written through a padded ROWS x 32 staging tile in shared memory
// (one per warp; ROWS = 16 takes the warp's rows in two halves, for kernels
// whose operand ring leaves less room) so that each store instruction covers a
// whole 128-byte row segment instead of 16 B in each of 32 rows.
__host__ __device__ constexpr int stage_words(int rows) { return rows * 33; }   // per warp

// fp32: row `lane` holds v[0..31]; rows [0, nvalid) of the warp are stored
// to out_row0 + r * ld (columns [0, 32)).
template <int ROWS>
__device__ __forceinline__ void store_chunk_f32(const uint32_t (&v)[32], uint32_t* stage,
                                                float* out_row0, size_t ld, int nvalid,
                                                int lane) {
#pragma unroll
  for (int part = 0; part < 32 / ROWS; ++part) {
    const int r0 = part * ROWS;
    if (r0 >= nvalid) break;
    if (lane / ROWS == part) {
#pragma unroll
      for (int j = 0; j < 32; ++j) stage[(lane % ROWS) * 33 + j] = v[j];
    }
    __syncwarp();
    const int r1 = min(nvalid, r0 + ROWS);
    for (int r = r0; r < r1; ++r)
      out_row0[(size_t)r * ld + lane] = __uint_as_float(stage[(r - r0) * 33 + lane]);
    __syncwarp();
  }
}

// fp32 scatter-add (the fused combine): row `lane` holds v[0..31] of a
// permuted row whose token is my_t and gate weight my_w; for the warp's valid
// rows, y32_col0[t * ld + c] += w * v[c].  Staged through the padded tile so
// that each instruction covers four rows with one 16-byte vector add per lane
// (8 lanes per row, 32 consecutive columns).
template <int ROWS>
__device__ __forceinline__ void scatter_chunk_f32(const uint32_t (&v)[32], uint32_t* stage,
                                                  float* y32_col0, size_t ld, int my_t,
                                                  float my_w, int nvalid, int lane) {
  const int c = (lane % 8) * 4;
#pragma unroll
  for (int part = 0; part < 32 / ROWS; ++part) {
    const int h0 = part * ROWS;
    if (h0 >= nvalid) break;
    if (lane / ROWS == part) {
#pragma unroll
      for (int j = 0; j < 32; ++j) stage[(lane % ROWS) * 33 + j] = v[j];
    }
    __syncwarp();
    const int h1 = min(nvalid, h0 + ROWS);
    for (int r0 = h0; r0 < h1; r0 += 4) {
      const int r = r0 + lane / 8;                     // < 32: a lane of this warp
      const int t = __shfl_sync(0xffffffffu, my_t, r);
      const float w = __shfl_sync(0xffffffffu, my_w, r);
      if (r < h1) {
        const uint32_t* src = stage + (r - h0) * 33 + c;
        const float4 add = make_float4(w * __uint_as_float(src[0]), w * __uint_as_float(src[1]),
                                       w * __uint_as_float(src[2]), w * __uint_as_float(src[3]));
        atomicAdd(reinterpret_cast<float4*>(y32_col0 + (size_t)t * ld + c), add);
      }
    }
    __syncwarp();
  }
}

// bf16: row `lane` holds pk[0..15] (32 bf16), stored directly as four
// 16-byte vectors (the SwiGLU tile is a quarter of the fp32 one's bytes and
// measured faster without staging).
__device__ __forceinline__ void store_chunk_bf16(const uint32_t (&pk)[16],
                                                 __nv_bfloat16* out_row0, size_t ld, int nvalid,
                                                 int lane) {
  if (lane >= nvalid) return;
  uint4* dst = reinterpret_cast<uint4*>(out_row0 + (size_t)lane * ld);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

__device__ __forceinline__ void swiglu_pack(const uint32_t (&g)[32], const uint32_t (&u)[32],
                                            uint32_t (&pk)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
    const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
    pk[i] = pack_bf16x2(silu(g0) * u0, silu(g1) * u1);
  }
}

__device__ __forceinline__ int clamp_rows(int v) { return v < 0 ? 0 : (v > 32 ? 32 : v); }

// v[i] *= row_scale * col_scale[i] for the 32 accumulator columns of a chunk
// (fp32 bits): the e4m3 GEMMs' per-row and per-column quantization scales
__device__ __forceinline__ void apply_scales(uint32_t (&v)[32], const float* __restrict__ col_scale,
                                             float row_scale) {
  const float4* s4 = reinterpret_cast<const float4*>(col_scale);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 sc = __ldg(s4 + i);
    v[4 * i + 0] = __float_as_uint(__uint_as_float(v[4 * i + 0]) * row_scale * sc.x);
    v[4 * i + 1] = __float_as_uint(__uint_as_float(v[4 * i + 1]) * row_scale * sc.y);
    v[4 * i + 2] = __float_as_uint(__uint_as_float(v[4 * i + 2]) * row_scale * sc.z);
    v[4 * i + 3] = __float_as_uint(__uint_as_float(v[4 * i + 3]) * row_scale * sc.w);
  }
}

template <int BN, bool SWIGLU>
struct GemmCfg {
  static constexpr int kOutCols = SWIGLU ? BN / 2 : BN;  // output columns per tile
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kStagingOff = kStages * kStageBytes;
  static constexpr int kSmemBytes =
      kStagingOff + (SWIGLU ? 0 : kEpiWarps * stage_words(16) * 4) + 1024;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, BN, /*b_mn_major=*/true);
  static constexpr uint32_t kIdesc64 = idesc_bf16_f32(kBM / 2, BN, /*b_mn_major=*/true);
};

struct GemmShared {
  uint64_t full_bar[8];
  uint64_t empty_bar[8];
  uint64_t tfull_bar[2];
  uint64_t tempty_bar[2];
  uint64_t drain_bar;
  uint32_t tmem_base;
  int abort_flag;
  int never;                       // stays 0: wait with a time limit only
  int tile_prefix[257];
  int row_off[256];
  int row_cnt[256];
};

__device__ __forceinline__ void decode_tile(const GemmShared& sh, int tile, int E, int n_tiles,
                                            int& e, int& m, int& n) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sh.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int local = tile - sh.tile_prefix[e];
  const int mt = (sh.tile_prefix[e + 1] - sh.tile_prefix[e]) / n_tiles;
  n = local / mt;
  m = local - n * mt;
}

// ---------------------------------------------------------------- roles
// The pieces below are shared by the bf16 kernel and the e4m3-weight kernel.

// Barriers, TMEM, and the device-side tile list (warp 2: per-expert tile
// counts -> exclusive prefix, bucket offsets to smem).
__device__ __forceinline__ void gemm_setup(GemmShared& sh, int stages, int full_count,
                                           int tmem_cols, const int32_t* offsets, int E,
                                           int n_tiles, int max_rows, int32_t* status, int warp,
                                           int lane, const FuseArgs& fz, int epi_count) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&sh.full_bar[s], full_count);
      mbar_init(&sh.empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh.tfull_bar[a], 1);
      mbar_init(&sh.tempty_bar[a], epi_count);
    }
    mbar_init(&sh.drain_bar, 1);
    sh.abort_flag = 0;
    sh.never = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh.tmem_base, tmem_cols);
    tmem_relinquish();
  }
  if (warp == 2) {
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int tiles = 0;
      if (e < E) {
        const int o0 = offsets[e], o1 = offsets[e + 1];
        int cnt = o1 - o0;
        if (o0 < 0 || cnt < 0 || o1 > max_rows) {
          report(status, kDevErrBadOffsets);
          cnt = 0;
        }
        if (fz.bucket_rows) cnt = min(cnt, max(0, fz.bucket_rows[e]));
        sh.row_off[e] = o0;
        sh.row_cnt[e] = cnt;
        tiles = cnt > 0 ? ((cnt + kBM - 1) / kBM) * n_tiles : 0;
      }
      int incl = tiles;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (e < E) sh.tile_prefix[e] = carry + incl - tiles;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sh.tile_prefix[E] = carry;
  }
}

// Gathering TMA producer (all 32 lanes of warp 0): lane L copies rows
// 4L .. 4L+3 of each A tile from the token rows with one tile::gather4 per
// k-block; rows past the bucket read the zero row n_tok.  Lane 0 waits, arms
// the stage barrier and loads B.
template <int STAGES, int STAGE_BYTES, int A_BYTES, int B_BYTES, class LoadB>
__device__ __forceinline__ void producer_role_gather(GemmShared& sh, uint8_t* smem,
                                                     const CUtensorMap* tmX, const FuseArgs& fz,
                                                     int E, int n_tiles, int nkb, int32_t* status,
                                                     LoadB load_b, int kb_elems, int lane) {
  volatile int* abort_flag = &sh.abort_flag;
  const int total_tiles = sh.tile_prefix[E];
  int it = 0;
  int last_it[8];
  for (int s = 0; s < STAGES; ++s) last_it[s] = -1;
  bool ok = true;
  for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
    int e, m, n;
    decode_tile(sh, tile, E, n_tiles, e, m, n);
    const int left = sh.row_cnt[e] - m * kBM;
    const bool small = left <= kBM / 2;   // M = 64 tile
    const int nrows = small ? kBM / 2 : kBM;
    int idx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 4 * lane + i;
      idx[i] = (rr < nrows && rr < left) ? fz.row_src[sh.row_off[e] + m * kBM + rr] : fz.n_tok;
    }
    for (int kb = 0; kb < nkb; ++kb, ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      bool good = true;
      if (lane == 0) good = mbar_wait(&sh.empty_bar[s], ph ^ 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
      uint8_t* sa = smem + s * STAGE_BYTES;
      const uint32_t a_bytes = small ? A_BYTES / 2 : A_BYTES;
      if (lane == 0) mbar_arrive_expect_tx(&sh.full_bar[s], a_bytes + B_BYTES);
      __syncwarp();
      if (4 * lane < nrows)
        tma_gather4(sa + 4 * lane * 128, tmX, &sh.full_bar[s], kb * kb_elems, idx[0], idx[1],
                    idx[2], idx[3]);
      if (lane == 0) load_b(sa + A_BYTES, &sh.full_bar[s], weight_index(fz, e), n, kb);
      last_it[s] = it;
    }
  }
  if (lane == 0) {
    if (!ok) {
      *abort_flag = 1;
      report(status, kDevErrWaitTimeout);
    }
    // never leave with copies in flight: every stage's last fill must land
    for (int s = 0; s < STAGES; ++s)
      if (last_it[s] >= 0) mbar_wait(&sh.full_bar[s], (last_it[s] / STAGES) & 1, &sh.never);
  }
}

// TMA producer (one thread): per k-block the A tile (128 or, for a bucket's
// last <= 64 rows, 64 rows) and, through load_b(stage B buffer, bar, e, n,
// kb), the weight tile.
template <int STAGES, int STAGE_BYTES, int A_BYTES, int B_BYTES, class LoadB>
__device__ __forceinline__ void producer_role(GemmShared& sh, uint8_t* smem,
                                              const CUtensorMap* tmA, const CUtensorMap* tmA64,
                                              int E, int n_tiles, int nkb, int32_t* status,
                                              LoadB load_b, const FuseArgs& fz,
                                              int kb_elems = kBK) {
  volatile int* abort_flag = &sh.abort_flag;
  const int total_tiles = sh.tile_prefix[E];
  int it = 0;
  int last_it[8];
  for (int s = 0; s < STAGES; ++s) last_it[s] = -1;
  bool ok = true;
  for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
    int e, m, n;
    decode_tile(sh, tile, E, n_tiles, e, m, n);
    const int row0 = sh.row_off[e] + m * kBM;
    const bool small = sh.row_cnt[e] - m * kBM <= kBM / 2;   // M = 64 tile
    for (int kb = 0; kb < nkb; ++kb, ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      if (!mbar_wait(&sh.empty_bar[s], ph ^ 1, abort_flag)) { ok = false; break; }
      uint8_t* sa = smem + s * STAGE_BYTES;
      const uint32_t a_bytes = small ? A_BYTES / 2 : A_BYTES;
      mbar_arrive_expect_tx(&sh.full_bar[s], a_bytes + B_BYTES);
      if (small)
        tma_load_2d(sa, tmA64, &sh.full_bar[s], kb * kb_elems, row0);
      else
        tma_load_2d(sa, tmA, &sh.full_bar[s], kb * kb_elems, row0);
      load_b(sa + A_BYTES, &sh.full_bar[s], weight_index(fz, e), n, kb);
      last_it[s] = it;
    }
  }
  if (!ok) {
    *abort_flag = 1;
    report(status, kDevErrWaitTimeout);
  }
  // never leave with copies in flight: every stage's last fill must land
  for (int s = 0; s < STAGES; ++s)
    if (last_it[s] >= 0) mbar_wait(&sh.full_bar[s], (last_it[s] / STAGES) & 1, &sh.never);
}

// MMA issuer (one thread): per k-block, four K = 16 MMAs from the stage into
// accumulator buffer lt & 1; commits free the stage / hand the tile over.
template <int BN, int STAGES, int STAGE_BYTES, int A_BYTES, bool E4M3 = false>
__device__ __forceinline__ void mma_role(GemmShared& sh, uint8_t* smem, int E, int n_tiles,
                                         int nkb, uint32_t idesc, uint32_t idesc64,
                                         int32_t* status) {
  volatile int* abort_flag = &sh.abort_flag;
  const int total_tiles = sh.tile_prefix[E];
  const uint32_t tmem_base = sh.tmem_base;
  int it = 0, lt = 0;
  bool ok = true;
  for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++lt) {
    int e, m, n;
    decode_tile(sh, tile, E, n_tiles, e, m, n);
    const uint32_t id = (sh.row_cnt[e] - m * kBM <= kBM / 2) ? idesc64 : idesc;
    const int a = lt & 1;
    const uint32_t aph = (lt >> 1) & 1;
    if (!mbar_wait(&sh.tempty_bar[a], aph ^ 1, abort_flag)) { ok = false; break; }
    tc_fence_after();
    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * BN);
    for (int kb = 0; kb < nkb; ++kb, ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      if (!mbar_wait(&sh.full_bar[s], ph, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
      const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        // A: K-major rows of 128 B, 8-row atoms 1024 B apart; +32 B per K step
        // (16 bf16 or 32 e4m3 values)
        const uint64_t adesc = smem_desc_sw128(a_addr + ks * 32, 16, 1024);
        if (E4M3) {
          // B: K-major like A (e4m3 weights are stored [E, N, K])
          const uint64_t bdesc = smem_desc_sw128(b_addr + ks * 32, 16, 1024);
          umma_e4m3(d_tmem, adesc, bdesc, id, (kb | ks) != 0 ? 1u : 0u);
        } else {
          // B: MN-major; 64-wide N chunks 8 KB apart (LBO), 8-row K groups
          // 1024 B apart (SBO); +16 K rows = +2048 B per K step
          const uint64_t bdesc = smem_desc_sw128(b_addr + ks * 2048, kChunkBytes, 1024);
          umma_bf16(d_tmem, adesc, bdesc, id, (kb | ks) != 0 ? 1u : 0u);
        }
      }
      umma_commit(&sh.empty_bar[s]);
    }
    if (!ok) break;
    umma_commit(&sh.tfull_bar[a]);
  }
  if (!ok) {
    *abort_flag = 1;
    report(status, kDevErrWaitTimeout);
  }
  // wait until every MMA issued by this thread has finished
  umma_commit(&sh.drain_bar);
  mbar_wait(&sh.drain_bar, 0, &sh.never);
}

// Epilogue (warps 2..9): drain accumulator buffer lt & 1 of each tile
// (tcgen05.ld -> [column scales] -> SwiGLU + bf16 stores, or fp32 stores).
// Fusion compiled into a kernel instance: none, gather (GEMM 1's producer
// fetches token rows by row_src), scatter (GEMM 2's epilogue adds weighted rows
// into y32).  Kept out of the plain instances' code entirely.
constexpr int kFuseNone = 0, kFuseGather = 1, kFuseScatter = 2;

template <int BN, bool SWIGLU, bool SCALED, int FUSE = kFuseNone>
__device__ __forceinline__ void epilogue_role(GemmShared& sh, uint8_t* staging, int warp,
                                              int lane, int E, int n_tiles, int n_out,
                                              void* out_raw, const float* row_scale,
                                              const float* sc0, const float* sc1,
                                              const FuseArgs& fz, int32_t* status) {
  constexpr int kOutCols = SWIGLU ? BN / 2 : BN;
  volatile int* abort_flag = &sh.abort_flag;
  const int total_tiles = sh.tile_prefix[E];
  const uint32_t tmem_base = sh.tmem_base;
  const int q = warp & 3;                 // TMEM lane quarter this warp may read
  // with 8 epilogue warps, group 0 (warps 2..5) and group 1 (6..9) take
  // alternate 32-column chunks
  constexpr int kGroups = epi_warps(SWIGLU) / 4;
  const int grp = (warp - 2) / 4;
  int lt = 0;
  for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++lt) {
    int e, m, n;
    decode_tile(sh, tile, E, n_tiles, e, m, n);
    const int a = lt & 1;
    const uint32_t aph = (lt >> 1) & 1;
    if (!mbar_wait(&sh.tfull_bar[a], aph, abort_flag)) {
      *abort_flag = 1;
      report(status, kDevErrWaitTimeout);
      break;
    }
    tc_fence_after();
    // M = 64 tiles put rows 16q..16q+15 in TMEM lanes 32q..32q+15
    const bool small = sh.row_cnt[e] - m * kBM <= kBM / 2;
    const int rows_per_warp = small ? 16 : 32;
    const int first = m * kBM + q * rows_per_warp;
    int nvalid = clamp_rows(sh.row_cnt[e] - first);
    if (nvalid > rows_per_warp) nvalid = rows_per_warp;
    const size_t row0 = (size_t)sh.row_off[e] + first;
    const size_t sc_off = (size_t)weight_index(fz, e) * n_out + (size_t)n * kOutCols;
    const float sr = (SCALED && lane < nvalid) ? row_scale[row0 + lane] : 0.f;
    uint32_t* stage = reinterpret_cast<uint32_t*>(staging) + (warp - 2) * stage_words(16);
    const uint32_t tbase =
        tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * BN);
    if (SWIGLU) {
      __nv_bfloat16* o =
          static_cast<__nv_bfloat16*>(out_raw) + row0 * n_out + (size_t)n * kOutCols;
#pragma unroll 1
      for (int c = grp; c < BN / 2 / 32 && n * kOutCols + c * 32 < n_out; c += kGroups) {
        uint32_t g[32], u[32], pk[16];
        tmem_ld_32x32b_x32(tbase + c * 32, g);
        tmem_ld_32x32b_x32(tbase + BN / 2 + c * 32, u);
        tmem_ld_wait();
        if (SCALED) {
          apply_scales(g, sc0 + sc_off + c * 32, sr);
          apply_scales(u, sc1 + sc_off + c * 32, sr);
        }
        swiglu_pack(g, u, pk);
        store_chunk_bf16(pk, o + c * 32, n_out, nvalid, lane);
      }
    } else if (FUSE == kFuseScatter) {
      // fused combine: weighted rows added into the token accumulator
      int my_t = 0;
      float my_w = 0.f;
      if (lane < nvalid) {
        const int p = fz.row_pair[row0 + lane];
        my_t = p / fz.k;
        my_w = fz.topk_w[p];
      }
      float* o = fz.y32 + (size_t)n * kOutCols;
#pragma unroll 1
      for (int c = grp; c < BN / 32 && n * kOutCols + c * 32 < n_out; c += kGroups) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c * 32, v);
        tmem_ld_wait();
        if (SCALED) apply_scales(v, sc0 + sc_off + c * 32, sr);
        scatter_chunk_f32<16>(v, stage, o + c * 32, n_out, my_t, my_w, nvalid, lane);
      }
    } else {
      float* o = static_cast<float*>(out_raw) + row0 * n_out + (size_t)n * kOutCols;
#pragma unroll 1
      for (int c = grp; c < BN / 32 && n * kOutCols + c * 32 < n_out; c += kGroups) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c * 32, v);
        tmem_ld_wait();
        if (SCALED) apply_scales(v, sc0 + sc_off + c * 32, sr);
        store_chunk_f32<16>(v, stage, o + c * 32, n_out, nvalid, lane);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.tempty_bar[a]);
  }
}

// ---------------------------------------------------------------- bf16 weights
template <int BN, bool SWIGLU, int FUSE>
__global__ void __launch_bounds__(gemm_threads(SWIGLU), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmA64,   // 64-row boxes
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1,
                        const int32_t* __restrict__ offsets, int E, int K, int n_out,
                        int max_rows, void* __restrict__ out_raw, int32_t* status,
                        const FuseArgs fz) {
  using Cfg = GemmCfg<BN, SWIGLU>;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ GemmShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tiles = (n_out + Cfg::kOutCols - 1) / Cfg::kOutCols;
  const int nkb = K / kBK;

  gemm_setup(sh, Cfg::kStages, 1, Cfg::kTmemCols, offsets, E, n_tiles, max_rows, status, warp,
             lane, fz, epi_warps(SWIGLU));
  if (warp == 1 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmA64);
    prefetch_tensormap(&tmB0);
    if (SWIGLU) prefetch_tensormap(&tmB1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    auto load_b = [&](uint8_t* sb, uint64_t* bar, int e, int n, int kb) {
      const int col0 = n * Cfg::kOutCols;
      if (SWIGLU) {
#pragma unroll
        for (int c = 0; c < BN / 128; ++c)
          tma_load_3d(sb + c * kChunkBytes, &tmB0, bar, col0 + c * 64, kb * kBK, e);
#pragma unroll
        for (int c = 0; c < BN / 128; ++c)
          tma_load_3d(sb + (BN / 128 + c) * kChunkBytes, &tmB1, bar, col0 + c * 64, kb * kBK, e);
      } else {
#pragma unroll
        for (int c = 0; c < BN / 64; ++c)
          tma_load_3d(sb + c * kChunkBytes, &tmB0, bar, col0 + c * 64, kb * kBK, e);
      }
    };
    if constexpr (FUSE == kFuseGather)   // A rows gathered from the token rows (tmA maps those)
      producer_role_gather<Cfg::kStages, Cfg::kStageBytes, Cfg::kABytes, Cfg::kBBytes>(
          sh, smem, &tmA, fz, E, n_tiles, nkb, status, load_b, kBK, lane);
    else if (lane == 0)
      producer_role<Cfg::kStages, Cfg::kStageBytes, Cfg::kABytes, Cfg::kBBytes>(
          sh, smem, &tmA, &tmA64, E, n_tiles, nkb, status, load_b, fz);
  } else if (warp == 1) {
    if (lane == 0)
      mma_role<BN, Cfg::kStages, Cfg::kStageBytes, Cfg::kABytes>(sh, smem, E, n_tiles, nkb,
                                                                 Cfg::kIdesc, Cfg::kIdesc64,
                                                                 status);
  } else {
    epilogue_role<BN, SWIGLU, false, FUSE>(sh, smem + Cfg::kStagingOff, warp, lane, E, n_tiles,
                                           n_out,
                                     out_raw, nullptr, nullptr, nullptr, fz, status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(sh.tmem_base, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------- e4m3 operands
// FP8 experts: activations and weights both e4m3, the activations with one
// fp32 scale per row, the weights with one per (expert, output column); both
// operands K-major (weights stored [E, N, K]).  The same tiles and roles as
// the bf16 kernel, a 128-deep K block per stage (one 128-byte swizzle row of
// e4m3) and tcgen05.mma.kind::f8f6f4 (K = 32 per instruction); the epilogue
// multiplies each accumulator by its row and column scales.
template <int BN, bool SWIGLU>
struct E4m3Cfg {
  static constexpr int kBKe = 128;                    // e4m3 values per k-block
  static constexpr int kOutCols = SWIGLU ? BN / 2 : BN;
  static constexpr int kABytes = kBM * kBKe;
  static constexpr int kBBytes = BN * kBKe;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kStagingOff = kStages * kStageBytes;
  static constexpr int kSmemBytes =
      kStagingOff + (SWIGLU ? 0 : kEpiWarps * stage_words(16) * 4) + 1024;
  static constexpr uint32_t kIdesc = idesc_e4m3_f32(kBM, BN);
  static constexpr uint32_t kIdesc64 = idesc_e4m3_f32(kBM / 2, BN);
};

template <int BN, bool SWIGLU, int FUSE>
__global__ void __launch_bounds__(gemm_threads(SWIGLU), 1)
    grouped_gemm_e4m3_kernel(const __grid_constant__ CUtensorMap tmA,     // codes [rows, K]
                             const __grid_constant__ CUtensorMap tmA64,
                             const __grid_constant__ CUtensorMap tmB0,    // codes [E, N, K]
                             const __grid_constant__ CUtensorMap tmB1,    // (SwiGLU: up)
                             const float* __restrict__ row_scale,
                             const float* __restrict__ col_scale0,
                             const float* __restrict__ col_scale1,
                             const int32_t* __restrict__ offsets, int E, int K, int n_out,
                             int max_rows, void* __restrict__ out_raw, int32_t* status,
                             const FuseArgs fz) {
  using Cfg = E4m3Cfg<BN, SWIGLU>;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ GemmShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tiles = (n_out + Cfg::kOutCols - 1) / Cfg::kOutCols;
  const int nkb = (K + Cfg::kBKe - 1) / Cfg::kBKe;   // a last half k-block reads zeros past K

  gemm_setup(sh, Cfg::kStages, 1, Cfg::kTmemCols, offsets, E, n_tiles, max_rows, status, warp,
             lane, fz, epi_warps(SWIGLU));
  if (warp == 1 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmA64);
    prefetch_tensormap(&tmB0);
    if (SWIGLU) prefetch_tensormap(&tmB1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // B: 128 weight rows (output columns) x 128 K per copy
    auto load_b = [&](uint8_t* sb, uint64_t* bar, int e, int n, int kb) {
      const int col0 = n * Cfg::kOutCols;
      if (SWIGLU) {
        tma_load_3d(sb, &tmB0, bar, kb * Cfg::kBKe, col0, e);
        tma_load_3d(sb + 128 * Cfg::kBKe, &tmB1, bar, kb * Cfg::kBKe, col0, e);
      } else {
#pragma unroll
        for (int c = 0; c < BN / 128; ++c)
          tma_load_3d(sb + c * 128 * Cfg::kBKe, &tmB0, bar, kb * Cfg::kBKe, col0 + c * 128, e);
      }
    };
    if constexpr (FUSE == kFuseGather)
      producer_role_gather<Cfg::kStages, Cfg::kStageBytes, Cfg::kABytes, Cfg::kBBytes>(
          sh, smem, &tmA, fz, E, n_tiles, nkb, status, load_b, Cfg::kBKe, lane);
    else if (lane == 0)
      producer_role<Cfg::kStages, Cfg::kStageBytes, Cfg::kABytes, Cfg::kBBytes>(
          sh, smem, &tmA, &tmA64, E, n_tiles, nkb, status, load_b, fz, Cfg::kBKe);
  } else if (warp == 1) {
    if (lane == 0)
      mma_role<BN, Cfg::kStages, Cfg::kStageBytes, Cfg::kABytes, true>(
          sh, smem, E, n_tiles, nkb, Cfg::kIdesc, Cfg::kIdesc64, status);
  } else {
    epilogue_role<BN, SWIGLU, true, FUSE>(sh, smem + Cfg::kStagingOff, warp, lane, E, n_tiles,
                                          n_out,
                                    out_raw, row_scale, col_scale0, col_scale1, fz, status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(sh.tmem_base, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------- CTA-pair variant
// Two CTAs of a cluster share one tcgen05.mma.cta_group::2 of M = 256, N = 256:
// each CTA stages its own 128 bucket rows of A and half of the B columns
// (GEMM 1: CTA 0 the gate columns, CTA 1 the up columns of the same 128
// h-columns; GEMM 2: 128 of the 256 output columns each), so each SM receives
// 32 KB of operands per 64-deep k-block instead of 48 KB.  Both CTAs' TMA
// loads complete on the leader CTA's stage barrier (armed by the leader for
// the bytes of both); the leader issues the MMAs and multicasts "stage free"
// and "accumulator ready" to both CTAs; both epilogues (each on its own 128
// accumulator rows, all 256 columns) report back to the leader.  Used when
// buckets are large (the pair tile is 256 rows).
//
// Half tiles.  When the last tile of an expert has at most 128 rows, the pair
// runs the M = 128 form of the MMA instead (64 rows per CTA).  Its accumulator
// puts columns [0,128) in TMEM lanes 0-63 and [128,256) in lanes 64-127, so
// epilogue warps 0-1 and 2-3 take the two column halves of the same 64 rows.
// For GEMM 1 each CTA then stages 64 gate + 64 up columns (CTA r: h-columns
// [64r, 64r+64) of the tile), so every thread still holds g and u of the same
// h-column.  This halves the rows computed in vain at each expert's tail.
// Epilogue pieces of the pair kernel: 32 accumulator columns of 32 rows.
// SCALED (e4m3 operands): the accumulators are multiplied by the row's scale
// sr and the 32 columns' scales first.
template <bool SCALED>
__device__ __forceinline__ void swiglu_chunk_store(uint32_t tg, uint32_t tu,
                                                   __nv_bfloat16* out_row0, size_t ld, int nvalid,
                                                   int lane, const float* sg, const float* su,
                                                   float sr) {
  uint32_t g[32], u[32], pk[16];
  tmem_ld_32x32b_x32(tg, g);
  tmem_ld_32x32b_x32(tu, u);
  tmem_ld_wait();
  if (SCALED) {
    apply_scales(g, sg, sr);
    apply_scales(u, su, sr);
  }
  swiglu_pack(g, u, pk);
  store_chunk_bf16(pk, out_row0, ld, nvalid, lane);
}

template <bool SCALED, int ROWS = 32>
__device__ __forceinline__ void f32_chunk_store(uint32_t t, uint32_t* stage, float* out_row0,
                                                size_t ld, int nvalid, int lane,
                                                const float* sc, float sr) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(t, v);
  tmem_ld_wait();
  if (SCALED) apply_scales(v, sc, sr);
  store_chunk_f32<ROWS>(v, stage, out_row0, ld, nvalid, lane);
}

template <bool SCALED, int ROWS = 32>
__device__ __forceinline__ void f32_chunk_scatter(uint32_t t, uint32_t* stage, float* y32_col0,
                                                  size_t ld, int nvalid, int lane,
                                                  const float* sc, float sr, int my_t,
                                                  float my_w) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(t, v);
  tmem_ld_wait();
  if (SCALED) apply_scales(v, sc, sr);
  scatter_chunk_f32<ROWS>(v, stage, y32_col0, ld, my_t, my_w, nvalid, lane);
}

constexpr int kPairStages = 6;
constexpr int kPairStageBytes = 2 * kBM * kBK * 2;      // A 16 KB + half of B 16 KB
// the fp32 kernel gives one ring slot to the epilogue warps' staging tiles
__host__ __device__ constexpr int pair_stages(bool swiglu) { return swiglu ? kPairStages : kPairStages - 1; }
__host__ __device__ constexpr int pair_staging_off(bool swiglu) {
  return pair_stages(swiglu) * kPairStageBytes;
}
__host__ __device__ constexpr int pair_smem_bytes(bool swiglu) {
  return pair_staging_off(swiglu) + (swiglu ? 0 : kEpiWarps * stage_words(32) * 4) + 1024;
}

struct PairShared {
  uint64_t full_bar[kPairStages];
  uint64_t empty_bar[kPairStages];
  uint64_t tfull_bar[2];
  uint64_t tempty_bar[2];
  uint64_t drain_bar;
  uint32_t tmem_base;
  int abort_flag;
  int never;
  int tile_prefix[257];
  int row_off[256];
  int row_cnt[256];
};

__device__ __forceinline__ void decode_pair_tile(const PairShared& sh, int tile, int E,
                                                 int n_tiles, int& e, int& m, int& n) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sh.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int local = tile - sh.tile_prefix[e];
  const int mt = (sh.tile_prefix[e + 1] - sh.tile_prefix[e]) / n_tiles;
  n = local / mt;
  m = local - n * mt;
}

// E4M3: e4m3 operands, both K-major (weights [E, N, K]), 128-deep k-blocks,
// kind::f8f6f4; tmB0h / tmB1h are 64-row weight boxes for the half tiles'
// 64 + 64 column split; the epilogue applies the row and column scales.
template <bool SWIGLU, bool E4M3, int FUSE>
__global__ void __launch_bounds__(gemm_threads(SWIGLU), 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmA64,   // 64-row boxes
                             const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1,
                             const __grid_constant__ CUtensorMap tmB0h,
                             const __grid_constant__ CUtensorMap tmB1h,
                             const float* __restrict__ row_scale,
                             const float* __restrict__ col_scale0,
                             const float* __restrict__ col_scale1,
                             const int32_t* __restrict__ offsets, int E, int K, int n_out,
                             int max_rows, void* __restrict__ out_raw, int32_t* status,
                             const FuseArgs fz) {
  constexpr int kOutCols = SWIGLU ? 128 : 256;        // output columns per pair tile
  constexpr int kPairM = 2 * kBM;
  constexpr int kKb = E4M3 ? 128 : kBK;               // K values per k-block (128 bytes)
  constexpr uint32_t kIdesc = E4M3 ? idesc_e4m3_f32(kPairM, 256)
                                   : idesc_bf16_f32(kPairM, 256, /*b_mn_major=*/true);
  constexpr uint32_t kIdescHalf = E4M3 ? idesc_e4m3_f32(kBM, 256)
                                       : idesc_bf16_f32(kBM, 256, /*b_mn_major=*/true);
  constexpr int kTmemCols = 512;
  constexpr int kStagesP = pair_stages(SWIGLU);
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ PairShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int n_tiles = (n_out + kOutCols - 1) / kOutCols;
  const int nkb = (K + kKb - 1) / kKb;   // e4m3: a last half k-block reads zeros past K

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesP; ++s) {
      mbar_init(&sh.full_bar[s], 1);
      mbar_init(&sh.empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh.tfull_bar[a], 1);
      mbar_init(&sh.tempty_bar[a], 2 * epi_warps(SWIGLU));   // the epilogue warps of both CTAs
    }
    mbar_init(&sh.drain_bar, 1);
    sh.abort_flag = 0;
    sh.never = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&sh.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmA64);
    prefetch_tensormap(&tmB0);
    if (SWIGLU) prefetch_tensormap(&tmB1);
    if (E4M3) prefetch_tensormap(&tmB0h);
    if (E4M3 && SWIGLU) prefetch_tensormap(&tmB1h);
  }
  if (warp == 2) {
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int tiles = 0;
      if (e < E) {
        const int o0 = offsets[e], o1 = offsets[e + 1];
        int cnt = o1 - o0;
        if (o0 < 0 || cnt < 0 || o1 > max_rows) {
          report(status, kDevErrBadOffsets);
          cnt = 0;
        }
        if (fz.bucket_rows) cnt = min(cnt, max(0, fz.bucket_rows[e]));
        sh.row_off[e] = o0;
        sh.row_cnt[e] = cnt;
        tiles = cnt > 0 ? ((cnt + kPairM - 1) / kPairM) * n_tiles : 0;
      }
      int incl = tiles;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (e < E) sh.tile_prefix[e] = carry + incl - tiles;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sh.tile_prefix[E] = carry;
  }
  tc_fence_before();
  cluster_sync();            // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();

  const uint32_t tmem_base = sh.tmem_base;
  const int total_tiles = sh.tile_prefix[E];
  volatile int* abort_flag = &sh.abort_flag;
  const uint32_t peer_abort = mapa_shared(&sh.abort_flag, rank ^ 1u);
  auto give_up = [&]() {
    *abort_flag = 1;
    st_shared_cluster_u32(peer_abort, 1u);
    report(status, kDevErrWaitTimeout);
  };

  if (warp == 0) {
    // A rows gathered from the token rows (all 32 lanes issue tile::gather4),
    // else one thread loads the permuted rows' tile
    constexpr bool gather = FUSE == kFuseGather;
    if (gather || lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int it = 0;
      int last_it[kStagesP];
      for (int s = 0; s < kStagesP; ++s) last_it[s] = -1;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += npairs) {
        int e, m, n;
        decode_pair_tile(sh, tile, E, n_tiles, e, m, n);
        const bool half = sh.row_cnt[e] - m * kPairM <= kBM;
        const int ew = weight_index(fz, e);
        const int mrow = m * kPairM + (int)rank * (half ? kBM / 2 : kBM);  // in the bucket
        const int row0 = sh.row_off[e] + mrow;
        const int col0 = n * kOutCols;
        const int nrows = half ? kBM / 2 : kBM;
        int idx[4] = {0, 0, 0, 0};
        if (gather) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = 4 * lane + i;
            idx[i] = (rr < nrows && mrow + rr < sh.row_cnt[e]) ? fz.row_src[row0 + rr] : fz.n_tok;
          }
        }
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kStagesP;
          const uint32_t ph = (it / kStagesP) & 1;
          bool good = true;
          if (lane == 0) good = mbar_wait(&sh.empty_bar[s], ph ^ 1, abort_flag);
          if (gather) good = __shfl_sync(0xffffffffu, good, 0);
          if (!good) { ok = false; break; }
          uint8_t* sa = smem + s * kPairStageBytes;
          uint8_t* sb = sa + kBM * kBK * 2;
          const uint32_t full_lead = mapa_shared(&sh.full_bar[s], 0);
          // a half tile reads 64 rows of A per CTA (8 KB instead of 16 KB)
          if (leader && lane == 0)
            mbar_arrive_expect_tx(&sh.full_bar[s],
                                  half ? 2 * (kPairStageBytes - kBM * kBK) : 2 * kPairStageBytes);
          if (gather) {
            __syncwarp();
            if (4 * lane < nrows)
              tma_gather4_pair(sa + 4 * lane * 128, &tmA, full_lead, kb * kKb, idx[0], idx[1],
                               idx[2], idx[3]);
          } else if (half) {
            tma_load_2d_pair(sa, &tmA64, full_lead, kb * kKb, row0);
          } else {
            tma_load_2d_pair(sa, &tmA, full_lead, kb * kKb, row0);
          }
          if (lane == 0) {
            if (E4M3) {
              // K-major weights: 128 rows (output columns) of 128 K bytes per CTA
              const int k0 = kb * kKb;
              if (SWIGLU && half) {
                tma_load_3d_pair(sb, &tmB0h, full_lead, k0, col0 + (int)rank * 64, ew);
                tma_load_3d_pair(sb + 64 * 128, &tmB1h, full_lead, k0, col0 + (int)rank * 64, ew);
              } else if (SWIGLU) {
                tma_load_3d_pair(sb, leader ? &tmB0 : &tmB1, full_lead, k0, col0, ew);
              } else {
                tma_load_3d_pair(sb, &tmB0, full_lead, k0, col0 + (int)rank * 128, ew);
              }
            } else if (SWIGLU && half) {
              tma_load_3d_pair(sb, &tmB0, full_lead, col0 + (int)rank * 64, kb * kBK, ew);
              tma_load_3d_pair(sb + kChunkBytes, &tmB1, full_lead, col0 + (int)rank * 64,
                               kb * kBK, ew);
            } else if (SWIGLU) {
              const CUtensorMap* mb = leader ? &tmB0 : &tmB1;
#pragma unroll
              for (int c = 0; c < 2; ++c)
                tma_load_3d_pair(sb + c * kChunkBytes, mb, full_lead, col0 + c * 64, kb * kBK, ew);
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c)
                tma_load_3d_pair(sb + c * kChunkBytes, &tmB0, full_lead,
                                 col0 + (int)rank * 128 + c * 64, kb * kBK, ew);
            }
          }
          last_it[s] = it;
        }
      }
      if (lane == 0) {
        if (!ok) give_up();
        if (leader) {
          // both CTAs' copies of every issued phase count on the leader's barriers
          for (int s = 0; s < kStagesP; ++s)
            if (last_it[s] >= 0)
              mbar_wait(&sh.full_bar[s], (last_it[s] / kStagesP) & 1, &sh.never);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader CTA)
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += npairs, ++lt) {
        int e, m, n;
        decode_pair_tile(sh, tile, E, n_tiles, e, m, n);
        const bool half = sh.row_cnt[e] - m * kPairM <= kBM;
        const uint32_t idesc = half ? kIdescHalf : kIdesc;
        const int a = lt & 1;
        const uint32_t aph = (lt >> 1) & 1;
        if (!mbar_wait(&sh.tempty_bar[a], aph ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * 256);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kStagesP;
          const uint32_t ph = (it / kStagesP) & 1;
          if (!mbar_wait(&sh.full_bar[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kPairStageBytes);
          const uint32_t b_addr = a_addr + kBM * kBK * 2;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t adesc = smem_desc_sw128(a_addr + ks * 32, 16, 1024);
            if (E4M3) {
              const uint64_t bdesc = smem_desc_sw128(b_addr + ks * 32, 16, 1024);
              umma_e4m3_pair(d_tmem, adesc, bdesc, idesc, (kb | ks) != 0 ? 1u : 0u);
            } else {
              const uint64_t bdesc = smem_desc_sw128(b_addr + ks * 2048, kChunkBytes, 1024);
              umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | ks) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair_mc(&sh.empty_bar[s], 0x3);
        }
        if (!ok) break;
        umma_commit_pair_mc(&sh.tfull_bar[a], 0x3);
      }
      if (!ok) give_up();
      umma_commit_pair_mc(&sh.drain_bar, 0x1);
      mbar_wait(&sh.drain_bar, 0, &sh.never);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2.., both CTAs)
    const int q = warp & 3;
    constexpr int kGroups = epi_warps(SWIGLU) / 4;     // warp groups splitting the chunks
    const int grp = (warp - 2) / 4;
    int lt = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs, ++lt) {
      int e, m, n;
      decode_pair_tile(sh, tile, E, n_tiles, e, m, n);
      const int a = lt & 1;
      const uint32_t aph = (lt >> 1) & 1;
      if (!mbar_wait(&sh.tfull_bar[a], aph, abort_flag)) {
        give_up();
        break;
      }
      tc_fence_after();
      const bool half = sh.row_cnt[e] - m * kPairM <= kBM;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * 256);
      uint32_t* stage = reinterpret_cast<uint32_t*>(smem + pair_staging_off(SWIGLU)) + (warp - 2) * stage_words(32);
      // E4M3: column scales from (e, column), the row's scale per thread
      const int ew = weight_index(fz, e);
      const float* cs0 = E4M3 ? col_scale0 + (size_t)ew * n_out : nullptr;
      const float* cs1 = (E4M3 && SWIGLU) ? col_scale1 + (size_t)ew * n_out : nullptr;
      if (!half) {
        const int first = m * kPairM + (int)rank * kBM + q * 32;   // first row of this warp
        const int nvalid = clamp_rows(sh.row_cnt[e] - first);
        const size_t row0 = (size_t)(sh.row_off[e] + first);
        const float sr = (E4M3 && lane < nvalid) ? row_scale[row0 + lane] : 0.f;
        if (SWIGLU) {
          const int c0 = n * kOutCols;
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out_raw) + row0 * n_out + c0;
#pragma unroll 1
          for (int c = grp; c < 4 && c0 + c * 32 < n_out; c += kGroups)
            swiglu_chunk_store<E4M3>(tbase + c * 32, tbase + 128 + c * 32, o + c * 32, n_out,
                                     nvalid, lane, cs0 + c0 + c * 32, cs1 + c0 + c * 32, sr);
        } else if (FUSE == kFuseScatter) {
          const int c0 = n * kOutCols;
          int my_t = 0;
          float my_w = 0.f;
          if (lane < nvalid) {
            const int p = fz.row_pair[row0 + lane];
            my_t = p / fz.k;
            my_w = fz.topk_w[p];
          }
#pragma unroll 1
          for (int c = grp; c < 8 && c0 + c * 32 < n_out; c += kGroups)
            f32_chunk_scatter<E4M3>(tbase + c * 32, stage, fz.y32 + c0 + c * 32, n_out, nvalid,
                                    lane, cs0 + c0 + c * 32, sr, my_t, my_w);
        } else {
          const int c0 = n * kOutCols;
          float* o = static_cast<float*>(out_raw) + row0 * n_out + c0;
#pragma unroll 1
          for (int c = grp; c < 8 && c0 + c * 32 < n_out; c += kGroups)
            f32_chunk_store<E4M3>(tbase + c * 32, stage, o + c * 32, n_out, nvalid, lane,
                                  cs0 + c0 + c * 32, sr);
        }
      } else {
        // lanes 0-63: accumulator columns [0,128); lanes 64-127: [128,256)
        const int hh = q >> 1;
        const int first = m * kPairM + (int)rank * (kBM / 2) + (q & 1) * 32;
        const int nvalid = clamp_rows(sh.row_cnt[e] - first);
        const size_t row0 = (size_t)(sh.row_off[e] + first);
        const float sr = (E4M3 && lane < nvalid) ? row_scale[row0 + lane] : 0.f;
        if (SWIGLU) {
          // this CTA's h-columns [64*rank ... ) of the tile: gate in TMEM
          // columns [0,64), up in [64,128); lanes 64-127 hold the next 64
          // columns of the tile (staged by the other half of B)
          const int c0 = n * kOutCols + hh * 64;
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out_raw) + row0 * n_out + c0;
#pragma unroll 1
          for (int c = grp; c < 2 && c0 + c * 32 < n_out; c += kGroups)
            swiglu_chunk_store<E4M3>(tbase + c * 32, tbase + 64 + c * 32, o + c * 32, n_out,
                                     nvalid, lane, cs0 + c0 + c * 32, cs1 + c0 + c * 32, sr);
        } else if (FUSE == kFuseScatter) {
          const int c0 = n * kOutCols + hh * 128;
          int my_t = 0;
          float my_w = 0.f;
          if (lane < nvalid) {
            const int p = fz.row_pair[row0 + lane];
            my_t = p / fz.k;
            my_w = fz.topk_w[p];
          }
#pragma unroll 1
          for (int c = grp; c < 4 && c0 + c * 32 < n_out; c += kGroups)
            f32_chunk_scatter<E4M3>(tbase + c * 32, stage, fz.y32 + c0 + c * 32, n_out, nvalid,
                                    lane, cs0 + c0 + c * 32, sr, my_t, my_w);
        } else {
          const int c0 = n * kOutCols + hh * 128;
          float* o = static_cast<float*>(out_raw) + row0 * n_out + c0;
#pragma unroll 1
          for (int c = grp; c < 4 && c0 + c * 32 < n_out; c += kGroups)
            f32_chunk_store<E4M3>(tbase + c * 32, stage, o + c * 32, n_out, nvalid, lane,
                                  cs0 + c0 + c * 32, sr);
        }
      }
      // the warp's tensor-memory loads have completed; the signal does not
      // wait for its global stores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(&sh.tempty_bar[a], 0));
    }
  }

  if (*abort_flag) spin_ns(200000);      // let copies still in flight land
  tc_fence_before();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- CTA pairs with expert tails
// The CTA-pair tiles of the kernel above for buckets of 256 to 511 rows per
// expert (bf16 operands), where an expert's rows rarely fill whole 256-row
// tiles: buckets of 256 +- a few dozen rows would otherwise need a second,
// mostly empty tile per column block.
//
// Expert tails.  The last r <= 128 rows of an expert that has at least one
// full 256-row tile are computed inside the k-loop of its last full tile, with
// swapped operands: the weights staged for that tile are the M = 256 side of a
// second MMA per K step (each CTA's 128 weight columns, MN-major) and the tail
// rows its N side, rounded up to N = 32, 64, 96 or 128 (N/2 rows staged by
// each CTA, K-major, in a third region of the stage).  The tail costs MMA time
// in proportion to its rows and adds only its own rows to the operand
// traffic: the weights are not fetched again.  Its accumulator is transposed
// (TMEM lane = weight column, TMEM column = row) and takes the upper 128
// columns of the other accumulator buffer: the epilogue drains those columns
// of every tile first and reports them free on a barrier of their own, so a
// tile with a tail waits for half of the previous tile's epilogue only; it
// drains its own tail first in turn.  GEMM 1's epilogue hands the up values
// (lanes 64-127) to the warps holding the gate values of the same h-columns
// (lanes 0-63) through shared memory.  An expert of at most 128 rows runs the
// swapped MMA alone.  GEMM 1 stages, per CTA r, the gate and the up columns of
// h-columns [64r, 64r + 64) of the tile, so that both MMAs of a K step use
// the same weight tile (accumulator columns [128r, 128r + 64) gate,
// [128r + 64, 128r + 128) up).
//
// Dynamic tile order.  Tiles of one bucket have different lengths (with or
// without a tail), and with a fixed round-robin assignment the pairs drift
// apart until tiles that share a weight tile or a bucket's rows no longer run
// at the same time and read them from HBM again.  Here the pairs take tiles
// from a global counter in list order: the leader's producer draws the next
// index 8 k-blocks before its current tile ends and publishes it 2 k-blocks
// later to its MMA issuer and epilogue warps and to the other CTA, through a
// small ring of slots in shared memory.  The tiles running at any moment are
// then a contiguous window of the list.
constexpr int kPairRows = 2 * kBM;                     // rows of a full pair tile
// A stage: the CTA's rows of A (16 KB), its half of the weight tile (16 KB)
// and up to 64 tail rows (8 KB).
constexpr int kTailStages = 5;
constexpr int kTailWOff = kBM * kBK * 2;
constexpr int kTailTOff = 2 * kBM * kBK * 2;
constexpr int kTailStageBytes = kTailTOff + 64 * 128;
constexpr int kTailStagingOff = kTailStages * kTailStageBytes;
constexpr int kTailStageRows = 16;                     // fp32 epilogue staging rows per warp
// GEMM 1's tails pass up values between epilogue warps through one padded
// 32 x 32 tile per (warp group, lane half)
constexpr int kSwapXchgBytes = 4 * stage_words(32) * 4;
__host__ __device__ constexpr int tail_smem_bytes(bool swiglu) {
  return kTailStagingOff + (swiglu ? kSwapXchgBytes : kEpiWarps * stage_words(kTailStageRows) * 4) +
         1024;
}
// N of a swapped MMA over `rows` tail rows (1..128): a multiple of 32, so
// that each CTA stages a multiple of 16 rows
__host__ __device__ constexpr int swap_n(int rows) { return (rows + 31) & ~31; }

// Tiles per column block of an expert with cnt > 0 rows: one per 256 rows,
// except that a last r <= 128 rows after a full tile ride along with it.
__host__ __device__ constexpr int tail_tiles_per_block(int cnt) {
  return (cnt > kPairRows && cnt % kPairRows != 0 && cnt % kPairRows <= kBM)
             ? cnt / kPairRows
             : (cnt + kPairRows - 1) / kPairRows;
}

// Rows of tile m (of mt per column block) of a bucket of cnt rows: main =
// rows of its 256-row MMA (0: none), tail = rows of its swapped MMA (0: none),
// which start at bucket row m * 256 + (main ? 256 : 0).
__device__ __forceinline__ void tail_tile_rows(int cnt, int m, int mt, int& main_rows,
                                               int& tail_rows) {
  const int left = cnt - m * kPairRows;
  if (cnt <= kBM) {
    main_rows = 0;
    tail_rows = cnt;
  } else {
    main_rows = min(kPairRows, left);
    tail_rows = (m == mt - 1 && left > kPairRows) ? left - kPairRows : 0;
  }
}

// tile indices in flight between the leader's producer and the consumers:
// the leader's MMA issuer and epilogue warps, the other CTA's producer and
// epilogue warps
constexpr int kSchedDepth = 4;
constexpr int kSchedConsumers = 2 + 2 * kEpiWarps;

struct PairTailShared {
  uint64_t full_bar[kTailStages];
  uint64_t empty_bar[kTailStages];
  uint64_t tfull_bar[2];
  uint64_t tempty_bar[2];             // accumulator buffer drained
  uint64_t thalf_bar[2];              // its upper 128 columns drained
  uint64_t drain_bar;
  uint64_t xchg_full[4];              // GEMM 1 tails: up values written
  uint64_t xchg_empty[4];             // ... and read
  uint64_t sched_full[kSchedDepth];   // a tile index published in the slot
  uint64_t sched_empty[kSchedDepth];  // (leader) every consumer has read it
  int sched_tile[kSchedDepth];        // -1: no more tiles
  uint32_t tmem_base;
  int abort_flag;
  int never;
  int tile_prefix[257];
  int row_off[256];
  int row_cnt[256];
};

// tile -> expert e, row tile m, column block n (mt row tiles per block)
__device__ __forceinline__ void decode_tail_tile(const PairTailShared& sh, int tile, int E,
                                                 int n_tiles, int& e, int& m, int& n, int& mt) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sh.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int local = tile - sh.tile_prefix[e];
  mt = (sh.tile_prefix[e + 1] - sh.tile_prefix[e]) / n_tiles;
  n = local / mt;
  m = local - n * mt;
}

template <bool SWIGLU, int FUSE>
__global__ void __launch_bounds__(gemm_threads(SWIGLU), 1)
    grouped_gemm_pair_tail_kernel(const __grid_constant__ CUtensorMap tmA,
                                  const __grid_constant__ CUtensorMap tmA16,   // 16-row boxes
                                  const __grid_constant__ CUtensorMap tmB0,
                                  const __grid_constant__ CUtensorMap tmB1,
                                  const int32_t* __restrict__ offsets, int E, int K, int n_out,
                                  int max_rows, void* __restrict__ out_raw, int32_t* status,
                                  int* __restrict__ sched,   // [next tile, finished pairs], zero
                                  const FuseArgs fz) {
  constexpr int kOutCols = SWIGLU ? 128 : 256;        // output columns per pair tile
  constexpr uint32_t kIdesc = idesc_bf16_f32(kPairRows, 256, /*b_mn_major=*/true);
  constexpr int kTmemCols = 512;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ PairTailShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int npairs = gridDim.x >> 1;
  const int n_tiles = (n_out + kOutCols - 1) / kOutCols;
  const int nkb = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTailStages; ++s) {
      mbar_init(&sh.full_bar[s], 1);
      mbar_init(&sh.empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh.tfull_bar[a], 1);
      mbar_init(&sh.tempty_bar[a], 2 * kEpiWarps);   // the epilogue warps of both CTAs
      mbar_init(&sh.thalf_bar[a], 2 * kEpiWarps);
    }
    mbar_init(&sh.drain_bar, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&sh.xchg_full[i], 1);
      mbar_init(&sh.xchg_empty[i], 1);
    }
    for (int i = 0; i < kSchedDepth; ++i) {
      mbar_init(&sh.sched_full[i], 1);
      mbar_init(&sh.sched_empty[i], kSchedConsumers);
    }
    sh.abort_flag = 0;
    sh.never = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&sh.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmA16);
    prefetch_tensormap(&tmB0);
    if (SWIGLU) prefetch_tensormap(&tmB1);
  }
  if (warp == 2) {
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int tiles = 0;
      if (e < E) {
        const int o0 = offsets[e], o1 = offsets[e + 1];
        int cnt = o1 - o0;
        if (o0 < 0 || cnt < 0 || o1 > max_rows) {
          report(status, kDevErrBadOffsets);
          cnt = 0;
        }
        if (fz.bucket_rows) cnt = min(cnt, max(0, fz.bucket_rows[e]));
        sh.row_off[e] = o0;
        sh.row_cnt[e] = cnt;
        tiles = cnt > 0 ? tail_tiles_per_block(cnt) * n_tiles : 0;
      }
      int incl = tiles;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (e < E) sh.tile_prefix[e] = carry + incl - tiles;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sh.tile_prefix[E] = carry;
  }
  tc_fence_before();
  cluster_sync();            // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();

  const uint32_t tmem_base = sh.tmem_base;
  const int total_tiles = sh.tile_prefix[E];
  volatile int* abort_flag = &sh.abort_flag;
  const uint32_t peer_abort = mapa_shared(&sh.abort_flag, rank ^ 1u);
  auto give_up = [&]() {
    *abort_flag = 1;
    st_shared_cluster_u32(peer_abort, 1u);
    report(status, kDevErrWaitTimeout);
  };
  // the i-th tile of this pair (-1: none left); false if the wait gave up
  auto sched_take = [&](int i, int& tile) -> bool {
    const int slot = i % kSchedDepth;
    if (!mbar_wait_cluster(&sh.sched_full[slot], (i / kSchedDepth) & 1, abort_flag)) return false;
    tile = *reinterpret_cast<volatile int*>(&sh.sched_tile[slot]);
    return true;
  };
  // one consumer has read slot i (an arrive on the leader's barrier)
  auto sched_release = [&](int i) {
    const int slot = i % kSchedDepth;
    if (leader)
      mbar_arrive(&sh.sched_empty[slot]);
    else
      mbar_arrive_cluster(mapa_shared(&sh.sched_empty[slot], 0));
  };

  if (warp == 0) {
    // A rows gathered from the token rows (all 32 lanes issue tile::gather4),
    // else one thread loads the permuted rows' tiles
    constexpr bool gather = FUSE == kFuseGather;
    if (gather || lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int it = 0;
      int last_it[kTailStages];
      for (int s = 0; s < kTailStages; ++s) last_it[s] = -1;
      bool ok = true;
      // leader: the next tile is drawn 8 k-blocks before the current one
      // ends and published 2 k-blocks later, which hides the atomic's latency
      // and the hand-over to the other CTA behind the current tile
      const int claim_kb = nkb > 8 ? nkb - 8 : 0;
      const int publish_kb = claim_kb + 2 < nkb ? claim_kb + 2 : nkb - 1;
      auto sched_publish = [&](int i, int t) -> bool {
        const int slot = i % kSchedDepth;
        if (!mbar_wait_cluster(&sh.sched_empty[slot], ((i / kSchedDepth) & 1) ^ 1, abort_flag))
          return false;
        sh.sched_tile[slot] = t;
        st_shared_cluster_u32(mapa_shared(&sh.sched_tile[slot], 1), static_cast<uint32_t>(t));
        mbar_arrive(&sh.sched_full[slot]);
        mbar_arrive_cluster(mapa_shared(&sh.sched_full[slot], 1));
        return true;
      };
      int next = -1, drawn = -1;
      if (leader && lane == 0) {
        drawn = atomicAdd(sched, 1);
        next = drawn < total_tiles ? drawn : -1;
        ok = sched_publish(0, next);
      }
      if (gather) ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int i = 0; ok; ++i) {
        int tile = -1;
        if (lane == 0) {
          if (leader) {
            tile = next;                       // published during the previous tile
          } else {
            ok = sched_take(i, tile);
            if (ok) sched_release(i);
          }
        }
        if (gather) {
          ok = __shfl_sync(0xffffffffu, ok, 0);
          tile = __shfl_sync(0xffffffffu, tile, 0);
        }
        if (!ok || tile < 0) break;
        int e, m, n, mt;
        decode_tail_tile(sh, tile, E, n_tiles, e, m, n, mt);
        const int cnt = sh.row_cnt[e];
        int main_rows, tail_rows;
        tail_tile_rows(cnt, m, mt, main_rows, tail_rows);
        // rows this CTA stages: 128 of A, N/2 of the tail
        const int arows = main_rows > 0 ? kBM : 0;
        const int trows = tail_rows > 0 ? swap_n(tail_rows) / 2 : 0;
        const int ew = weight_index(fz, e);
        const int amrow = m * kPairRows + (int)rank * arows;                  // in the bucket
        const int tmrow = m * kPairRows + (main_rows > 0 ? kPairRows : 0) + (int)rank * trows;
        const int arow0 = sh.row_off[e] + amrow, trow0 = sh.row_off[e] + tmrow;
        const int col0 = n * kOutCols;
        const uint32_t cta_bytes = (uint32_t)(arows + trows) * 128u + kBM * kBK * 2;
        int aidx[4] = {0, 0, 0, 0}, tidx[4] = {0, 0, 0, 0};
        if (gather) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int rr = 4 * lane + j;
            aidx[j] = (rr < arows && amrow + rr < cnt) ? fz.row_src[arow0 + rr] : fz.n_tok;
            tidx[j] = (rr < trows && tmrow + rr < cnt) ? fz.row_src[trow0 + rr] : fz.n_tok;
          }
        }
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kTailStages;
          const uint32_t ph = (it / kTailStages) & 1;
          bool good = true;
          if (lane == 0) good = mbar_wait(&sh.empty_bar[s], ph ^ 1, abort_flag);
          if (gather) good = __shfl_sync(0xffffffffu, good, 0);
          if (!good) { ok = false; break; }
          uint8_t* sa = smem + s * kTailStageBytes;
          uint8_t* sb = sa + kTailWOff;
          uint8_t* st = sa + kTailTOff;
          const uint32_t full_lead = mapa_shared(&sh.full_bar[s], 0);
          if (leader && lane == 0) mbar_arrive_expect_tx(&sh.full_bar[s], 2 * cta_bytes);
          if (gather) {
            __syncwarp();
            if (4 * lane < arows)
              tma_gather4_pair(sa + 4 * lane * 128, &tmA, full_lead, kb * kBK, aidx[0], aidx[1],
                               aidx[2], aidx[3]);
            if (4 * lane < trows)
              tma_gather4_pair(st + 4 * lane * 128, &tmA, full_lead, kb * kBK, tidx[0], tidx[1],
                               tidx[2], tidx[3]);
          } else {
            if (arows > 0) tma_load_2d_pair(sa, &tmA, full_lead, kb * kBK, arow0);
            for (int j = 0; j < trows; j += 16)
              tma_load_2d_pair(st + j * 128, &tmA16, full_lead, kb * kBK, trow0 + j);
          }
          if (lane == 0) {
            if (SWIGLU) {
              // gate then up columns of h-columns [col0 + 64 rank, + 64)
              tma_load_3d_pair(sb, &tmB0, full_lead, col0 + (int)rank * 64, kb * kBK, ew);
              tma_load_3d_pair(sb + kChunkBytes, &tmB1, full_lead, col0 + (int)rank * 64,
                               kb * kBK, ew);
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c)
                tma_load_3d_pair(sb + c * kChunkBytes, &tmB0, full_lead,
                                 col0 + (int)rank * 128 + c * 64, kb * kBK, ew);
            }
          }
          last_it[s] = it;
          if (leader && lane == 0) {
            if (kb == claim_kb) drawn = atomicAdd(sched, 1);
            if (kb == publish_kb) {
              next = drawn < total_tiles ? drawn : -1;
              if (!sched_publish(i + 1, next)) ok = false;
            }
          }
        }
        if (gather) ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      if (lane == 0) {
        if (!ok) give_up();
        if (leader) {
          // this pair draws no more tiles: the last pair to get here leaves
          // the counters at zero for the next launch
          __threadfence();
          if (atomicAdd(sched + 1, 1) == npairs - 1) {
            atomicExch(sched, 0);
            atomicExch(sched + 1, 0);
          }
          // both CTAs' copies of every issued phase count on the leader's barriers
          for (int s = 0; s < kTailStages; ++s)
            if (last_it[s] >= 0)
              mbar_wait(&sh.full_bar[s], (last_it[s] / kTailStages) & 1, &sh.never);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader CTA)
      int it = 0;
      // uses so far of each accumulator buffer: whole (a main MMA) and of its
      // upper 128 columns (a main MMA, or a tail)
      int mains0 = 0, mains1 = 0, halves0 = 0, halves1 = 0;
      bool ok = true;
      for (int lt = 0; ok; ++lt) {
        int tile = -1;
        if (!sched_take(lt, tile)) { ok = false; break; }
        sched_release(lt);
        if (tile < 0) break;
        int e, m, n, mt;
        decode_tail_tile(sh, tile, E, n_tiles, e, m, n, mt);
        int main_rows, tail_rows;
        tail_tile_rows(sh.row_cnt[e], m, mt, main_rows, tail_rows);
        const int b = lt & 1;
        // the main accumulator takes buffer b; a tail the upper 128 columns of
        // the other buffer (of b when the tile has no main MMA): wait until
        // their previous uses are drained
        const int x = main_rows > 0 ? b ^ 1 : b;
        int& mains_b = b ? mains1 : mains0;
        int& halves_b = b ? halves1 : halves0;
        int& halves_x = x ? halves1 : halves0;
        if (main_rows > 0) {
          if (!mbar_wait(&sh.tempty_bar[b], (mains_b & 1) ^ 1, abort_flag) ||
              !mbar_wait(&sh.thalf_bar[b], (halves_b & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          ++mains_b;
          ++halves_b;
        }
        if (tail_rows > 0) {
          if (!mbar_wait(&sh.thalf_bar[x], (halves_x & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          ++halves_x;
        }
        tc_fence_after();
        const uint32_t d_main = tmem_base + static_cast<uint32_t>(b * 256);
        const uint32_t d_tail = tmem_base + static_cast<uint32_t>(x * 256 + 128);
        // swapped: M = 256 weight columns (MN-major), N = the tail rows (K-major)
        const uint32_t idesc_tail =
            idesc_bf16_f32(kPairRows, swap_n(tail_rows > 0 ? tail_rows : 1), false, true);
        auto kloop = [&](auto main_c, auto tail_c) {
          constexpr bool kMain = decltype(main_c)::value, kTail = decltype(tail_c)::value;
          static_assert(kMain || kTail, "a tile has a main or a tail MMA");
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % kTailStages;
            const uint32_t ph = (it / kTailStages) & 1;
            if (!mbar_wait(&sh.full_bar[s], ph, abort_flag)) { ok = false; return; }
            tc_fence_after();
            const uint32_t st_addr = smem_u32(smem + s * kTailStageBytes);
            // K step: +32 B in the K-major rows (+2 in the descriptor),
            // +16 K rows = +2 KB in the MN-major weights (+128)
            const uint64_t dw = smem_desc_sw128(st_addr + kTailWOff, kChunkBytes, 1024);
            if constexpr (kMain) {
              const uint64_t da = smem_desc_sw128(st_addr, 16, 1024);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_bf16_pair(d_main, da + 2 * ks, dw + 128 * ks, kIdesc,
                               (kb | ks) != 0 ? 1u : 0u);
            }
            if constexpr (kTail) {
              const uint64_t dt = smem_desc_sw128(st_addr + kTailTOff, 16, 1024);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_bf16_pair(d_tail, dw + 128 * ks, dt + 2 * ks, idesc_tail,
                               (kb | ks) != 0 ? 1u : 0u);
            }
            umma_commit_pair_mc(&sh.empty_bar[s], 0x3);
          }
        };
        using T_ = std::integral_constant<bool, true>;
        using F_ = std::integral_constant<bool, false>;
        if (tail_rows == 0)
          kloop(T_{}, F_{});
        else if (main_rows == 0)
          kloop(F_{}, T_{});
        else
          kloop(T_{}, T_{});
        if (!ok) break;
        umma_commit_pair_mc(&sh.tfull_bar[b], 0x3);
      }
      if (!ok) give_up();
      umma_commit_pair_mc(&sh.drain_bar, 0x1);
      mbar_wait(&sh.drain_bar, 0, &sh.never);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2.., both CTAs)
    const int q = warp & 3;
    constexpr int kGroups = kEpiWarps / 4;              // warp groups splitting the chunks
    const int grp = (warp - 2) / 4;
    int xc = 0;                  // up-value hand-overs so far (GEMM 1 tails)
    bool xok = true;
    uint32_t* stage = reinterpret_cast<uint32_t*>(smem + kTailStagingOff) +
                      (warp - 2) * stage_words(kTailStageRows);
    // this warp is done with accumulator buffer `buf` (whole) / its upper
    // half: its tensor-memory loads have completed (tcgen05.wait::ld), and the
    // signal does not wait for the warp's global stores
    auto release = [&](int buf) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(&sh.tempty_bar[buf], 0));
    };
    auto release_half = [&](int buf) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(&sh.thalf_bar[buf], 0));
    };
    for (int lt = 0;; ++lt) {
      int tile = -1;
      bool good = true;
      if (lane == 0) good = sched_take(lt, tile);
      good = __shfl_sync(0xffffffffu, good, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      // the slot has been read (its value is in every lane's register)
      if (good && lane == 0)
        mbar_arrive_cluster_relaxed(mapa_shared(&sh.sched_empty[lt % kSchedDepth], 0));
      if (!good) {
        give_up();
        break;
      }
      if (tile < 0) break;
      int e, m, n, mt;
      decode_tail_tile(sh, tile, E, n_tiles, e, m, n, mt);
      int main_rows, tail_rows;
      tail_tile_rows(sh.row_cnt[e], m, mt, main_rows, tail_rows);
      const int b = lt & 1;
      const int x = main_rows > 0 ? b ^ 1 : b;        // buffer of a tail
      if (!mbar_wait(&sh.tfull_bar[b], (lt >> 1) & 1, abort_flag)) {
        give_up();
        break;
      }
      tc_fence_after();
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      if (tail_rows > 0) {
        // swapped tail: TMEM lane = weight column of this CTA, TMEM column j =
        // bucket row rowb + j (j < tail_rows are real)
        const int left = tail_rows;
        const uint32_t tbase = lane_base + static_cast<uint32_t>(x * 256 + 128);
        const size_t rowb =
            (size_t)sh.row_off[e] + (size_t)m * kPairRows + (main_rows > 0 ? kPairRows : 0);
        if constexpr (SWIGLU) {
          // lanes 0-63: gate, lanes 64-127: up of h-columns col0 + 64 * rank + [0, 64)
          const int hc = n * kOutCols + 64 * (int)rank + 32 * (q & 1) + lane;
          const int xi = grp * 2 + (q & 1);            // the gate warp and its up warp
          uint32_t* xu = reinterpret_cast<uint32_t*>(smem + kTailStagingOff) + xi * stage_words(32);
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out_raw);
#pragma unroll 1
          for (int c = grp; c * 32 < left; c += kGroups, ++xc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + c * 32, v);
            tmem_ld_wait();
            const uint32_t par = xc & 1;
            bool gw = true;
            if (q >= 2) {
              if (lane == 0) gw = mbar_wait(&sh.xchg_empty[xi], par ^ 1, abort_flag);
              if (!__shfl_sync(0xffffffffu, gw, 0)) { xok = false; break; }
#pragma unroll
              for (int j = 0; j < 32; ++j) xu[lane * 33 + j] = v[j];
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.xchg_full[xi]);
            } else {
              if (lane == 0) gw = mbar_wait(&sh.xchg_full[xi], par, abort_flag);
              if (!__shfl_sync(0xffffffffu, gw, 0)) { xok = false; break; }
              if (hc < n_out) {
                const int nv = min(32, left - c * 32);
                __nv_bfloat16* oc = o + (rowb + (size_t)c * 32) * n_out + hc;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (j < nv) {
                    const float g = __uint_as_float(v[j]);
                    const float u = __uint_as_float(xu[lane * 33 + j]);
                    oc[(size_t)j * n_out] = __float2bfloat16_rn(silu(g) * u);
                  }
                }
              }
              __syncwarp();
              // the up values were read (used by the stores above)
              if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(&sh.xchg_empty[xi], rank));
            }
          }
          if (!xok) {
            give_up();
            break;
          }
        } else {
          // 128 output columns per CTA, one per lane
          const int oc = n * kOutCols + 128 * (int)rank + 32 * q + lane;
#pragma unroll 1
          for (int c = grp; c * 32 < left; c += kGroups) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + c * 32, v);
            tmem_ld_wait();
            const int nv = min(32, left - c * 32);
            const size_t r0 = rowb + (size_t)c * 32;
            if (oc < n_out) {
              float* o = static_cast<float*>(out_raw) + r0 * n_out + oc;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nv) o[(size_t)j * n_out] = __uint_as_float(v[j]);
            }
          }
        }
        release_half(x);
      }
      if (main_rows > 0) {
        const uint32_t tbase = lane_base + static_cast<uint32_t>(b * 256);
        const int first = m * kPairRows + (int)rank * kBM + q * 32;   // first row of this warp
        const int nvalid = clamp_rows(sh.row_cnt[e] - first);
        const size_t row0 = (size_t)(sh.row_off[e] + first);
        const int c0 = n * kOutCols;
        // 32-column chunks [c_lo, c_hi) of the tile's output columns
        auto chunks = [&](int c_lo, int c_hi) {
#pragma unroll 1
          for (int c = c_lo + grp; c < c_hi && c0 + c * 32 < n_out; c += kGroups) {
            if (SWIGLU) {
              // h-column chunk c: gate column (c / 2) * 128 + (c % 2) * 32, up 64 further
              const int gcol = (c >> 1) * 128 + (c & 1) * 32;
              swiglu_chunk_store<false>(tbase + gcol, tbase + gcol + 64,
                                        static_cast<__nv_bfloat16*>(out_raw) + row0 * n_out +
                                            c0 + c * 32,
                                        n_out, nvalid, lane, nullptr, nullptr, 0.f);
            } else {
              f32_chunk_store<false, kTailStageRows>(
                  tbase + c * 32, stage, static_cast<float*>(out_raw) + row0 * n_out + c0 + c * 32,
                  n_out, nvalid, lane, nullptr, 0.f);
            }
          }
        };
        // the upper 128 accumulator columns first: a tail of the next tile may
        // go there as soon as they are drained
        constexpr int kChunks = SWIGLU ? 4 : 8;
        chunks(kChunks / 2, kChunks);
        release_half(b);
        chunks(0, kChunks / 2);
        release(b);
      }
    }
  }

  if (*abort_flag) spin_ns(200000);      // let copies still in flight land
  tc_fence_before();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

// Counters of the CTA-pair kernels' dynamic tile order, [next tile, finished
// pairs] per launch, zero between launches (the kernel's last pair resets
// its own).  Each launch takes the next of kSchedPool entries in turn, so
// launches that run at the same time on different streams use different
// counters unless kSchedPool of them run at once (a device runs at most 128
// kernels at a time).
constexpr int kSchedPool = 256;
static __device__ int g_pair_sched[kSchedPool][2];
static std::atomic<unsigned> g_sched_seq{0};
static std::mutex g_sched_mutex;
static int* g_sched_base[64] = {nullptr};

// a counter pair for one launch on the current device (the pool's device
// address is looked up once per device)
static cudaError_t take_sched_counter(int** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(g_sched_mutex);
    if (!g_sched_base[dev]) {
      void* p = nullptr;
      err = cudaGetSymbolAddress(&p, g_pair_sched);
      if (err != cudaSuccess) return err;
      g_sched_base[dev] = static_cast<int*>(p);
    }
  }
  *out = g_sched_base[dev] + 2 * (g_sched_seq.fetch_add(1, std::memory_order_relaxed) % kSchedPool);
  return cudaSuccess;
}

template <int BN, bool SWIGLU, int FUSE>
static cudaError_t launch_gemm_t(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                               const CUtensorMap& b0, const CUtensorMap& b1,
                               const int32_t* offsets, int E, int K,
                               int n_out, int max_rows, void* out, int32_t* status,
                               cudaStream_t s, const FuseArgs& fz) {
  using Cfg = GemmCfg<BN, SWIGLU>;
  DeviceInfo* di = nullptr;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  auto kern = grouped_gemm_kernel<BN, SWIGLU, FUSE>;
  if (!di->attr_set[slot]) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes);
    if (err != cudaSuccess) return err;
    di->attr_set[slot] = true;
  }
  const int n_tiles = (n_out + Cfg::kOutCols - 1) / Cfg::kOutCols;
  const long long row_tiles = (long long)max_rows / kBM + (E < max_rows ? E : max_rows);
  long long ub = row_tiles * n_tiles;
  int grid = (int)(ub < di->sms ? ub : di->sms);
  if (grid < 1) grid = 1;
  kern<<<grid, gemm_threads(SWIGLU), Cfg::kSmemBytes, s>>>(a, a64, b0, b1, offsets, E, K, n_out,
                                                     max_rows, out, status, fz);
  return cudaGetLastError();
}

template <bool SWIGLU, bool E4M3, int FUSE>
static cudaError_t launch_gemm_pair_t(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                                      const CUtensorMap& b0, const CUtensorMap& b1,
                                      const int32_t* offsets, int E, int K, int n_out,
                                      int max_rows, void* out, int32_t* status, cudaStream_t s,
                                      const FuseArgs& fz, const CUtensorMap* b0h,
                                      const CUtensorMap* b1h, const float* row_scale,
                                      const float* cs0, const float* cs1) {
  constexpr int kSmem = pair_smem_bytes(SWIGLU);
  DeviceInfo* di = nullptr;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  auto kern = grouped_gemm_pair_kernel<SWIGLU, E4M3, FUSE>;
  if (!di->attr_set[slot]) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (err != cudaSuccess) return err;
    di->attr_set[slot] = true;
  }
  const int n_tiles = (n_out + (SWIGLU ? 127 : 255)) / (SWIGLU ? 128 : 256);
  const long long pair_rows = (long long)max_rows / (2 * kBM) + (E < max_rows ? E : max_rows);
  long long pairs = pair_rows * n_tiles;
  const int max_pairs = di->sms / 2;
  if (pairs > max_pairs) pairs = max_pairs;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(gemm_threads(SWIGLU), 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, a64, b0, b1, b0h ? *b0h : b0, b1h ? *b1h : b1,
                            row_scale, cs0, cs1, offsets, E, K, n_out, max_rows, out, status, fz);
}


template <bool SWIGLU, int FUSE>
static cudaError_t launch_gemm_pair_tail_t(int slot, const CUtensorMap& a, const CUtensorMap& a16,
                                           const CUtensorMap& b0, const CUtensorMap& b1,
                                           const int32_t* offsets, int E, int K, int n_out,
                                           int max_rows, void* out, int32_t* status,
                                           cudaStream_t s, const FuseArgs& fz) {
  constexpr int kSmem = tail_smem_bytes(SWIGLU);
  DeviceInfo* di = nullptr;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  int* sched = nullptr;
  err = take_sched_counter(&sched);
  if (err != cudaSuccess) return err;
  auto kern = grouped_gemm_pair_tail_kernel<SWIGLU, FUSE>;
  if (!di->attr_set[slot]) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (err != cudaSuccess) return err;
    di->attr_set[slot] = true;
  }
  const int n_tiles = (n_out + (SWIGLU ? 127 : 255)) / (SWIGLU ? 128 : 256);
  const long long pair_rows = (long long)max_rows / (2 * kBM) + (E < max_rows ? E : max_rows);
  long long pairs = pair_rows * n_tiles;
  const int max_pairs = di->sms / 2;
  if (pairs > max_pairs) pairs = max_pairs;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(gemm_threads(SWIGLU), 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, a16, b0, b1, offsets, E, K, n_out, max_rows, out,
                            status, sched, fz);
}

// The fusion an instance is compiled for, from the arguments.
static int fuse_kind(const FuseArgs& fz) {
  return fz.row_src ? kFuseGather : (fz.y32 ? kFuseScatter : kFuseNone);
}

// attribute slots: each (kernel, fusion) instance sets its smem limit once
template <int BN, bool SWIGLU>
static cudaError_t launch_gemm(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                               const CUtensorMap& b0, const CUtensorMap& b1,
                               const int32_t* offsets, int E, int K, int n_out, int max_rows,
                               void* out, int32_t* status, cudaStream_t s, const FuseArgs& fz) {
  const int kind = fuse_kind(fz);
  if constexpr (SWIGLU) {
    if (kind == kFuseGather)
      return launch_gemm_t<BN, SWIGLU, kFuseGather>(slot + 16, a, a64, b0, b1, offsets, E, K,
                                                    n_out, max_rows, out, status, s, fz);
  } else {
    if (kind == kFuseScatter)
      return launch_gemm_t<BN, SWIGLU, kFuseScatter>(slot + 32, a, a64, b0, b1, offsets, E, K,
                                                     n_out, max_rows, out, status, s, fz);
  }
  if (kind != kFuseNone) return cudaErrorInvalidValue;
  return launch_gemm_t<BN, SWIGLU, kFuseNone>(slot, a, a64, b0, b1, offsets, E, K, n_out,
                                              max_rows, out, status, s, fz);
}

template <bool SWIGLU, bool E4M3 = false>
static cudaError_t launch_gemm_pair(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                                    const CUtensorMap& b0, const CUtensorMap& b1,
                                    const int32_t* offsets, int E, int K, int n_out, int max_rows,
                                    void* out, int32_t* status, cudaStream_t s,
                                    const FuseArgs& fz, const CUtensorMap* b0h = nullptr,
                                    const CUtensorMap* b1h = nullptr,
                                    const float* row_scale = nullptr,
                                    const float* cs0 = nullptr, const float* cs1 = nullptr) {
  const int kind = fuse_kind(fz);
  if constexpr (!E4M3 && SWIGLU) {
    if (kind == kFuseGather)
      return launch_gemm_pair_t<SWIGLU, E4M3, kFuseGather>(slot + 16, a, a64, b0, b1, offsets, E,
                                                           K, n_out, max_rows, out, status, s,
                                                           fz, b0h, b1h, row_scale, cs0, cs1);
  } else if constexpr (!E4M3 && !SWIGLU) {
    if (kind == kFuseScatter)
      return launch_gemm_pair_t<SWIGLU, E4M3, kFuseScatter>(slot + 32, a, a64, b0, b1, offsets,
                                                            E, K, n_out, max_rows, out, status,
                                                            s, fz, b0h, b1h, row_scale, cs0, cs1);
  }
  if (kind != kFuseNone) return cudaErrorInvalidValue;
  return launch_gemm_pair_t<SWIGLU, E4M3, kFuseNone>(slot, a, a64, b0, b1, offsets, E, K, n_out,
                                                     max_rows, out, status, s, fz, b0h, b1h,
                                                     row_scale, cs0, cs1);
}

// slot: the plain instance's attribute slot (+16 gathering)
template <bool SWIGLU>
static cudaError_t launch_gemm_pair_tail(int slot, const CUtensorMap& a, const CUtensorMap& a16,
                                         const CUtensorMap& b0, const CUtensorMap& b1,
                                         const int32_t* offsets, int E, int K, int n_out,
                                         int max_rows, void* out, int32_t* status,
                                         cudaStream_t s, const FuseArgs& fz) {
  const int kind = fuse_kind(fz);
  if constexpr (SWIGLU) {
    if (kind == kFuseGather)
      return launch_gemm_pair_tail_t<SWIGLU, kFuseGather>(slot + 16, a, a16, b0, b1, offsets, E,
                                                          K, n_out, max_rows, out, status, s, fz);
  }
  if (kind != kFuseNone) return cudaErrorInvalidValue;   // no scattering form
  return launch_gemm_pair_tail_t<SWIGLU, kFuseNone>(slot, a, a16, b0, b1, offsets, E, K, n_out,
                                                    max_rows, out, status, s, fz);
}

template <int BN, bool SWIGLU, int FUSE>
static cudaError_t launch_gemm_e4m3_t(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                                      const CUtensorMap& b0, const CUtensorMap& b1,
                                      const float* row_scale, const float* s0, const float* s1,
                                      const int32_t* offsets, int E, int K, int n_out,
                                      int max_rows, void* out, int32_t* status, cudaStream_t s,
                                      const FuseArgs& fz);

template <int BN, bool SWIGLU>
static cudaError_t launch_gemm_e4m3(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                                    const CUtensorMap& b0, const CUtensorMap& b1,
                                    const float* row_scale, const float* s0, const float* s1,
                                    const int32_t* offsets, int E, int K, int n_out, int max_rows,
                                    void* out, int32_t* status, cudaStream_t s,
                                    const FuseArgs& fz) {
  if (fuse_kind(fz) != kFuseNone) return cudaErrorInvalidValue;   // not built for e4m3
  return launch_gemm_e4m3_t<BN, SWIGLU, kFuseNone>(slot, a, a64, b0, b1, row_scale, s0, s1,
                                                   offsets, E, K, n_out, max_rows, out, status,
                                                   s, fz);
}

// Tile shapes by the buffer's rows per expert, an upper bound on the average
// bucket: CTA pairs (256-row tiles) from 512; with bf16 operands, CTA pairs
// that compute an expert's last <= 128 rows inside its last full tile from
// 256 (buckets of a few hundred rows, which whole tiles fit badly); else
// single-CTA 128-row tiles.
enum class Tiles { kSingle, kPairTails, kPair };
static Tiles gemm_tiles(int E, int max_rows, bool e4m3) {
  if (max_rows >= 512LL * E) return Tiles::kPair;
  if (!e4m3 && max_rows >= 256LL * E) return Tiles::kPairTails;
  return Tiles::kSingle;
}

// The A operand: the permuted rows [max_rows, K] (128- and 64-row boxes), or,
// when gathering, the token rows [fz.n_tok, K] (one-row boxes for gather4).
static bool map_a(CUtensorMap* a, CUtensorMap* a64, const void* rows, int K, int max_rows,
                  bool e4m3, const FuseArgs& fz) {
  if (fz.row_src) {
    *a64 = {};
    return map_rows_gather(a, rows, K, fz.n_tok, e4m3);
  }
  if (e4m3)
    return map_rows_e4m3(a, rows, K, max_rows, kBM) && map_rows_e4m3(a64, rows, K, max_rows, kBM / 2);
  return map_rows(a, rows, K, max_rows, kBM) && map_rows(a64, rows, K, max_rows, kBM / 2);
}

// experts whose weights the tensor maps cover (buckets may outnumber them)
static int weight_count(const FuseArgs& fz, int E) { return fz.n_weights > 0 ? fz.n_weights : E; }

// GEMM 1: h = silu(A Wg) * (A Wu), A = x_perm or (gathering) the token rows
cudaError_t launch_gate_up(const __nv_bfloat16* a_rows, const int32_t* offsets, int E, int d,
                           int f, int max_rows, const __nv_bfloat16* w_gate,
                           const __nv_bfloat16* w_up, __nv_bfloat16* h, int32_t* status,
                           cudaStream_t s, bool* map_failed, const FuseArgs& fz) {
  CUtensorMap ta, ta64, tg, tu;
  *map_failed = !(map_a(&ta, &ta64, a_rows, d, max_rows, false, fz) &&
                  map_weights(&tg, w_gate, weight_count(fz, E), d, f) &&
                  map_weights(&tu, w_up, weight_count(fz, E), d, f));
  if (*map_failed) return cudaSuccess;
  const Tiles tiles = gemm_tiles(E, max_rows, false);
  if (tiles == Tiles::kPair)
    return launch_gemm_pair<true>(7, ta, ta64, tg, tu, offsets, E, d, f, max_rows, h, status, s,
                                  fz);
  if (tiles == Tiles::kPairTails) {
    // the tails are read in 16-row boxes of the permuted rows (the gathering
    // form reads token rows by tile::gather4 and needs none)
    CUtensorMap ta16 = ta;
    *map_failed = !fz.row_src && !map_rows(&ta16, a_rows, d, max_rows, 16);
    if (*map_failed) return cudaSuccess;
    return launch_gemm_pair_tail<true>(14, ta, ta16, tg, tu, offsets, E, d, f, max_rows, h, status,
                                       s, fz);
  }
  return launch_gemm<256, true>(0, ta, ta64, tg, tu, offsets, E, d, f, max_rows, h, status, s,
                                fz);
}

// GEMM 2: y_perm = h Wd, or (scattering) y32[t] += w * (h Wd)
cudaError_t launch_down(const __nv_bfloat16* h, const int32_t* offsets, int E, int d, int f,
                        int max_rows, const __nv_bfloat16* w_down, float* y_perm,
                        int32_t* status, cudaStream_t s, bool* map_failed, const FuseArgs& fz) {
  CUtensorMap ta, ta64, ta16, td;
  *map_failed = !(map_rows(&ta, h, f, max_rows, kBM) && map_rows(&ta64, h, f, max_rows, kBM / 2) &&
                  map_rows(&ta16, h, f, max_rows, 16) &&
                  map_weights(&td, w_down, weight_count(fz, E), f, d));
  if (*map_failed) return cudaSuccess;
  const Tiles tiles = gemm_tiles(E, max_rows, false);
  if (d % 256 == 0 && tiles == Tiles::kPair)
    return launch_gemm_pair<false>(8, ta, ta64, td, td, offsets, E, f, d, max_rows, y_perm, status,
                                   s, fz);
  // (the weighted scatter keeps the single-CTA tiles: the tails' transposed
  // accumulators can only add one value per lane and row, four times the
  // atomic instructions of the staged four-wide adds)
  if (d % 256 == 0 && tiles == Tiles::kPairTails && !fz.y32)
    return launch_gemm_pair_tail<false>(15, ta, ta16, td, td, offsets, E, f, d, max_rows, y_perm,
                                        status, s, fz);
  if (d % 256 == 0)
    return launch_gemm<256, false>(1, ta, ta64, td, td, offsets, E, f, d, max_rows, y_perm, status,
                                   s, fz);
  return launch_gemm<128, false>(2, ta, ta64, td, td, offsets, E, f, d, max_rows, y_perm, status,
                                 s, fz);
}

template <int BN, bool SWIGLU, int FUSE>
static cudaError_t launch_gemm_e4m3_t(int slot, const CUtensorMap& a, const CUtensorMap& a64,
                                    const CUtensorMap& b0, const CUtensorMap& b1,
                                    const float* row_scale, const float* s0, const float* s1,
                                    const int32_t* offsets, int E, int K, int n_out, int max_rows,
                                    void* out, int32_t* status, cudaStream_t s,
                                    const FuseArgs& fz) {
  using Cfg = E4m3Cfg<BN, SWIGLU>;
  DeviceInfo* di = nullptr;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  auto kern = grouped_gemm_e4m3_kernel<BN, SWIGLU, FUSE>;
  if (!di->attr_set[slot]) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes);
    if (err != cudaSuccess) return err;
    di->attr_set[slot] = true;
  }
  const int n_tiles = (n_out + Cfg::kOutCols - 1) / Cfg::kOutCols;
  const long long row_tiles = (long long)max_rows / kBM + (E < max_rows ? E : max_rows);
  long long ub = row_tiles * n_tiles;
  int grid = (int)(ub < di->sms ? ub : di->sms);
  if (grid < 1) grid = 1;
  kern<<<grid, gemm_threads(SWIGLU), Cfg::kSmemBytes, s>>>(a, a64, b0, b1, row_scale, s0, s1,
                                                           offsets, E,
                                                   K, n_out, max_rows, out, status, fz);
  return cudaGetLastError();
}

// GEMM 1 / GEMM 2 on e4m3 rows (per-row scales, indexed by permuted row) and
// e4m3 weights stored [E, N, K] (per-column scales)
cudaError_t launch_gate_up_e4m3(const uint8_t* xq, const float* sx, const int32_t* offsets,
                                int E, int d, int f, int max_rows, const uint8_t* wq_gate,
                                const float* s_gate, const uint8_t* wq_up, const float* s_up,
                                __nv_bfloat16* h, int32_t* status, cudaStream_t s,
                                bool* map_failed, const FuseArgs& fz) {
  CUtensorMap ta, ta64, tg, tu;
  *map_failed = !(map_a(&ta, &ta64, xq, d, max_rows, true, fz) &&
                  map_weights_e4m3(&tg, wq_gate, weight_count(fz, E), f, d) &&
                  map_weights_e4m3(&tu, wq_up, weight_count(fz, E), f, d));
  if (*map_failed) return cudaSuccess;
  if (gemm_tiles(E, max_rows, true) == Tiles::kPair) {
    CUtensorMap tgh, tuh;
    *map_failed = !(map_weights_e4m3(&tgh, wq_gate, weight_count(fz, E), f, d, 64) &&
                    map_weights_e4m3(&tuh, wq_up, weight_count(fz, E), f, d, 64));
    if (*map_failed) return cudaSuccess;
    return launch_gemm_pair<true, true>(9, ta, ta64, tg, tu, offsets, E, d, f, max_rows, h,
                                        status, s, fz, &tgh, &tuh, sx, s_gate, s_up);
  }
  return launch_gemm_e4m3<256, true>(11, ta, ta64, tg, tu, sx, s_gate, s_up, offsets, E, d, f,
                                     max_rows, h, status, s, fz);
}

cudaError_t launch_down_e4m3(const uint8_t* hq, const float* sh_rows, const int32_t* offsets,
                             int E, int d, int f, int max_rows, const uint8_t* wq_down,
                             const float* s_down, float* y_perm, int32_t* status, cudaStream_t s,
                             bool* map_failed, const FuseArgs& fz) {
  CUtensorMap ta, ta64, td;
  *map_failed = !(map_rows_e4m3(&ta, hq, f, max_rows, kBM) &&
                  map_rows_e4m3(&ta64, hq, f, max_rows, kBM / 2) &&
                  map_weights_e4m3(&td, wq_down, weight_count(fz, E), d, f));
  if (*map_failed) return cudaSuccess;
  if (d % 256 == 0 && gemm_tiles(E, max_rows, true) == Tiles::kPair)
    return launch_gemm_pair<false, true>(10, ta, ta64, td, td, offsets, E, f, d, max_rows, y_perm,
                                         status, s, fz, &td, &td, sh_rows, s_down, nullptr);
  if (d % 256 == 0)
    return launch_gemm_e4m3<256, false>(12, ta, ta64, td, td, sh_rows, s_down, nullptr, offsets,
                                        E, f, d, max_rows, y_perm, status, s, fz);
  return launch_gemm_e4m3<128, false>(13, ta, ta64, td, td, sh_rows, s_down, nullptr, offsets, E,
                                      f, d, max_rows, y_perm, status, s, fz);
}

int device_sm_count() {
  DeviceInfo* di = nullptr;
  if (device_info(&di) != cudaSuccess) return 0;
  return di->sms;
}

}  // namespace moe
