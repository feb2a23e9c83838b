/*
 * libmoe — forward pass of a sparse Mixture-of-Experts layer on one B200
 * (sm_100a).  C ABI: plain pointers and sizes, no framework types.
 *
 * The layer (the local part of the expert-parallel pipeline that all the
 * source pages describe: "Expert Parallelism" guide (infra.bea.ai), section 2
 * "The Dispatch Pattern"; "Expert Parallelism" glossary (klaylearn.com), third
 * paragraph):
 *   route    l = x Wr (+ bias); top-k experts per token; gate weights =
 *            softmax renormalised over the k selected logits
 *   permute  pairs (token, expert) into per-expert buckets of capacity
 *            C = ceil(cf*k*T/E) (dropless when cf == 0), slots in token order,
 *            overflow dropped
 *   experts  per expert e: h = silu(x_perm Wg[e]) * (x_perm Wu[e]),
 *            y_perm = h Wd[e]  (SwiGLU; h stored bf16, y_perm kept fp32 so the
 *            layer output is rounded to bf16 only once, in the combine)
 *   combine  y[t] = sum over kept pairs j of w[t,j] * y_perm[row(t,j)], in
 *            top-k order; a token whose k pairs were all dropped gets x[t]
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *     library never allocates or frees device memory and keeps no state
 *     beyond a per-device cache of attributes.  Outputs must not alias inputs.
 *   - Tensors are dense row-major.  bf16 = IEEE bfloat16 (__nv_bfloat16),
 *     passed as void*.  Base pointers must be 16-byte aligned.
 *   - Work is enqueued asynchronously on `stream` (cudaStream_t passed as
 *     void*; NULL = legacy default stream).  No entry point synchronises.
 *   - Return codes report host-side validation and launch errors only.  A
 *     kernel that detects a problem on the device (a bounded wait that gave
 *     up, inconsistent bucket offsets) ORs a bit into the caller's int32
 *     device status word `dev_status` (nullable: then nothing is reported);
 *     read it after synchronising.  Bits: 1 = wait timeout, 2 = bad offsets,
 *     4 = a top-k expert id outside [0, E) (such a pair is treated as
 *     dropped; builds with MOE_CHECKS also report an expert listed twice for
 *     one token).
 *   - Limits: 1 <= E <= 256, 1 <= k <= min(E, 8), T*k < 2^31, d and f
 *     multiples of 64 (else MOE_ERR_UNSUPPORTED).  T == 0 is a no-op.
 */
#ifndef LIBMOE_MOE_H_
#define LIBMOE_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer  */
  MOE_ERR_WORKSPACE = 2,     /* workspace smaller than the size query says  */
  MOE_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed          */
  MOE_ERR_UNSUPPORTED = 4,   /* shape outside the kernels' tiling limits     */
  MOE_ERR_DEVICE_CHECK = 5   /* reserved: device status word was non-zero    */
} moe_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(int status);

/* Library ABI version, (major << 16) | minor. */
int moe_version(void);

/* Self-test of the kernels' time-limited waits (no counterpart on the pages):
 * launches one CTA that waits, with the same bounded mbarrier wait the GEMM
 * kernels use, on a barrier nothing arrives at, for at most limit_ns
 * (0 .. 10 s), then ORs the wait-timeout bit (1) into *dev_status (device
 * int32).  A caller can check that a wait that cannot complete ends with a
 * status word instead of a hang, and that the context stays usable. */
int moe_selftest_bounded_wait(int32_t* dev_status, int64_t limit_ns, void* stream);

/* Expert capacity, step "capacity" above: ceil(((cf*k)*T)/E) evaluated in
 * fp64; cf == 0 selects the dropless layer and returns T.  Source: the
 * capacity-factor entry of the inferensys.com glossary and section "Why
 * fixed-size buffers matter here" of "Expert Parallelism & All-to-All"
 * (neelmishra.github.io); the infra.bea.ai guide's section 4 states the same
 * rule without k, read here as the k = 1 case.  Returns -1 on bad args. */
int64_t moe_capacity(int64_t T, int64_t E, int64_t k, double cf);

/* Rows of the permuted buffers: min(T*k, E*C), the most pairs that can be
 * kept.  Returns -1 on bad args. */
int64_t moe_max_rows(int64_t T, int64_t E, int64_t k, double cf);

/* Device scratch bytes moe_route needs: the two-term bf16 split of the router
 * weight (2*d*round_up(E,64) bf16) and the split-K partial logits. */
size_t moe_route_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k);

/* Device scratch bytes moe_permute needs (per-chunk bucket histograms). */
size_t moe_permute_workspace_size(int64_t T, int64_t E, int64_t k);

/* Device workspace bytes moe_layer_forward needs: every intermediate
 * (status word, logits, routing, slots, buckets, x_perm, h, y_perm). */
size_t moe_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf);

/* Fields of the moe_layer_forward workspace, for callers that want to read
 * an intermediate after the call. */
typedef enum {
  MOE_WS_STATUS = 0,     /* int32[1]  device status word (zeroed by the call) */
  MOE_WS_LOGITS = 1,     /* f32 [T,E] */
  MOE_WS_TOPK_IDX = 2,   /* i32 [T,k] */
  MOE_WS_TOPK_W = 3,     /* f32 [T,k] */
  MOE_WS_SLOT = 4,       /* i32 [T,k] */
  MOE_WS_COUNTS = 5,     /* i32 [E]   */
  MOE_WS_OFFSETS = 6,    /* i32 [E+1] */
  MOE_WS_N_DROPPED = 7,  /* i32 [1]   */
  MOE_WS_ROW_SRC = 8,    /* i32 [max_rows] */
  MOE_WS_PERMUTE = 9,    /* moe_permute scratch */
  MOE_WS_X_PERM = 10,    /* bf16 [max_rows, d] */
  MOE_WS_H = 11,         /* bf16 [max_rows, f] */
  MOE_WS_Y_PERM = 12,    /* f32  [max_rows, d] */
  MOE_WS_ROUTE = 13,     /* moe_route scratch */
  MOE_WS_NUM_FIELDS = 14,
  /* moe_layer_forward_fp8 only (after the fields above) */
  MOE_WS_XQ = 14,        /* u8  [max_rows, d] e4m3 codes of x_perm */
  MOE_WS_SX = 15,        /* f32 [max_rows]    their row scales */
  MOE_WS_HQ = 16,        /* u8  [max_rows, f] e4m3 codes of h */
  MOE_WS_SH = 17,        /* f32 [max_rows]    their row scales */
  MOE_WS_XQ_TOK = 18,    /* u8  [T, d]        e4m3 codes of x (before the permutation) */
  MOE_WS_SX_TOK = 19,    /* f32 [T]           their row scales */
  MOE_WS_FP8_NUM_FIELDS = 20,
  /* moe_layer_forward_fused only (right after the first MOE_WS_NUM_FIELDS) */
  MOE_WS_ROW_PAIR = 20,  /* i32 [max_rows]    t*k + j of each kept row */
  MOE_WS_Y32 = 21        /* f32 [T, d]        gate-weighted sum of the expert outputs */
} moe_ws_field;

/* Byte offset of a field inside the moe_layer_forward workspace (each field
 * 256-byte aligned; fields MOE_WS_XQ .. MOE_WS_SX_TOK exist only in a
 * moe_layer_forward_fp8 workspace, MOE_WS_ROW_PAIR and MOE_WS_Y32 only in a
 * moe_layer_forward_fused one); -1 on bad args. */
int64_t moe_workspace_field_offset(int field, int64_t T, int64_t d, int64_t E, int64_t k,
                                   int64_t f, double cf);

/* Router and top-k gating.  The router is a linear layer giving one score per
 * expert (inferensys.com glossary, gating-network and router-latency entries);
 * top-k gating keeps the k highest (same glossary, Top-k Gating); the router
 * also supplies the weights that mix the chosen experts' outputs
 * (klaylearn.com glossary, third paragraph).
 *   x        bf16 [T,d]     tokens
 *   w_router f32  [d,E]     router weight
 *   bias     f32  [E]       nullable; added to every token's logits
 *   logits   f32  [T,E]     out: sum_i x[t,i]*w_router[i,e] + bias[e], fp32
 *   topk_idx i32  [T,k]     out: the k largest logits, descending; equal
 *                           logits rank the lower expert index first
 *   topk_w   f32  [T,k]     out: exp(l_j - l_max) / sum over the k selected
 *   ws, ws_bytes            device scratch, >= moe_route_workspace_size
 *   dev_status              nullable device status word (see conventions)
 * The selection is taken on the fp32 values written to `logits`.  The logits
 * are computed on the tensor cores from a two-term bf16 split of w_router
 * (hi = bf16(w), lo = bf16(w - hi); x is bf16 already), with fp32
 * accumulation; the split's residual is below 2^-18 |w| per weight. */
int moe_route(const void* x, const float* w_router, const float* bias, int64_t T, int64_t d,
              int64_t E, int64_t k, float* logits, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, int32_t* dev_status, void* stream);

/* Capacity-limited permutation into per-expert buckets (pairs are bucketed by
 * expert, overflow beyond the capacity is dropped: inferensys.com glossary,
 * Expert Capacity and Dropped Tokens entries; the tokens are permuted before
 * the experts run: klaylearn.com glossary, third paragraph).
 *   x         bf16 [T,d]        tokens
 *   topk_idx  i32  [T,k]        experts per token (distinct within a token)
 *   cf                          capacity factor, C = moe_capacity(T,E,k,cf)
 *   counts    i32  [E]          out: pairs kept by each expert (<= C)
 *   offsets   i32  [E+1]        out: exclusive prefix sum of counts
 *   slot      i32  [T,k]        out: bucket slot of pair (t,j) = number of
 *                               tokens t' < t that chose the same expert;
 *                               -1 when that slot is >= C (dropped)
 *   row_src   i32  [max_rows]   out: token of permuted row r (rows < offsets[E])
 *   x_perm    bf16 [max_rows,d] out: row offsets[e]+slot holds x[t]
 *   n_dropped i32  [1]          out: number of dropped pairs
 *   ws, ws_bytes                device scratch, >= moe_permute_workspace_size
 *   dev_status                  nullable device status word: bit 4 when a
 *                               topk_idx entry lies outside [0, E) (that pair
 *                               is treated as dropped, slot -1, takes no
 *                               bucket place and is not counted in n_dropped,
 *                               which counts capacity overflow)
 * Rows at and beyond offsets[E] of row_src / x_perm are left untouched. */
int moe_permute(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                int32_t* row_src, void* x_perm, int32_t* n_dropped, void* ws, size_t ws_bytes,
                int32_t* dev_status, void* stream);

/* moe_permute without the scratch argument, for callers that cannot allocate
 * device memory or pass the library any: e.g. an operator plugin that only
 * receives its declared input and output tensors, or a runtime that plans all
 * device memory at start-up and forbids later allocations.  The pages have no
 * counterpart to this entry point; it is a deployment convenience.
 * Arguments, results and return codes are those of moe_permute (same checks,
 * same kernels, same outputs, including the bit-4 report into the nullable
 * dev_status for a topk_idx entry outside [0, E)), minus ws / ws_bytes.  The
 * per-chunk bucket counters live in a 257 KiB array compiled into the library
 * and held by every GPU that loads it until the process exits; nothing is
 * allocated per call.  Limits and rules:
 *   - (ceil(T/256) + 1) * E must be <= 65792, else MOE_ERR_WORKSPACE (E = 256
 *     allows T <= 65536);
 *   - all calls share that array: calls whose work overlaps on the GPU (other
 *     streams, other host threads on the same device) race; serialise them;
 *   - nothing in the array needs to start at zero (each call writes every
 *     counter before it is read);
 *   - the first call on a device resolves the array's device address (with
 *     that device current) and caches it; make it before any stream capture. */
int moe_permute_noalloc(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                        int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                        int32_t* row_src, void* x_perm, int32_t* n_dropped, int32_t* dev_status,
                        void* stream);

/* Grouped expert GEMM 1 with the SwiGLU fused into its epilogue: for every
 * expert e and every row r of its bucket (offsets[e] <= r < offsets[e+1]),
 *   h[r,:] = silu(x_perm[r,:] Wg[e]) * (x_perm[r,:] Wu[e]),  silu(z) = z*sigmoid(z)
 * (experts are gate/up/down MLPs: neelmishra.github.io, section "Tensor
 * parallelism for experts"; grouped GEMMs over the buckets: klaylearn.com
 * glossary, fourth paragraph).  bf16 operands, fp32 accumulation, bf16 h.
 *   x_perm bf16 [max_rows,d], offsets i32 [E+1] (device), w_gate / w_up bf16
 *   [E,d,f], h bf16 [max_rows,f] out (rows of no bucket are left untouched). */
int moe_expert_gate_up(const void* x_perm, const int32_t* offsets, int64_t E, int64_t d,
                       int64_t f, int64_t max_rows, const void* w_gate, const void* w_up,
                       void* h, int32_t* dev_status, void* stream);

/* Grouped expert GEMM 2 (down projection): y_perm[r,:] = h[r,:] Wd[e] for the
 * rows of bucket e.  h bf16 [max_rows,f], w_down bf16 [E,f,d], y_perm f32
 * [max_rows,d] out (fp32 accumulation, stored unrounded; rows of no bucket
 * are left untouched).  Same source passages as moe_expert_gate_up. */
int moe_expert_down(const void* h, const int32_t* offsets, int64_t E, int64_t d, int64_t f,
                    int64_t max_rows, const void* w_down, float* y_perm, int32_t* dev_status,
                    void* stream);

/* Both expert GEMMs: moe_expert_gate_up then moe_expert_down, with h as the
 * caller's buffer in between. */
int moe_expert_mlp(const void* x_perm, const int32_t* offsets, int64_t E, int64_t d, int64_t f,
                   int64_t max_rows, const void* w_gate, const void* w_up, const void* w_down,
                   void* h, float* y_perm, int32_t* dev_status, void* stream);

/* Inverse permutation and gate-weighted sum (the combine undoes the dispatch
 * permutation and adds each token's k expert outputs scaled by their gate
 * weights: neelmishra.github.io, section "All-to-all: the distributed
 * transpose"; the weighted sum closes the infra.bea.ai guide's section 2
 * diagram; a dropped token goes through the layer untouched: inferensys.com
 * glossary, Dropped Tokens entry).
 *   y[t,:] = sum_{j: slot[t,j] >= 0} topk_w[t,j] * y_perm[offsets[topk_idx[t,j]] + slot[t,j], :]
 * summed in fp32 in j order and rounded once to bf16; if no pair of t was
 * kept, y[t,:] = x[t,:] exactly.  y_perm f32 [>= offsets[E], d], x bf16
 * [T,d], y bf16 [T,d] out. */
int moe_combine(const float* y_perm, const void* x, const int32_t* topk_idx, const float* topk_w,
                const int32_t* slot, const int32_t* offsets, int64_t T, int64_t d, int64_t k,
                void* y, void* stream);

/* moe_combine on expert-output rows held in bf16 (y_rows bf16 [>= offsets[E],
 * d]): the same sum, each row value widened exactly to fp32.  For expert
 * parallelism, where the rows come back from the ranks that ran the experts
 * (the combine all-to-all of "Expert Parallelism & All-to-All"
 * (neelmishra.github.io), section "All-to-all: the distributed transpose")
 * and bf16 rows halve the bytes that cross the links.  Arguments, layout and
 * errors as moe_combine. */
int moe_combine_bf16rows(const void* y_rows, const void* x, const int32_t* topk_idx,
                         const float* topk_w, const int32_t* slot, const int32_t* offsets,
                         int64_t T, int64_t d, int64_t k, void* y, void* stream);

/* dst bf16 [rows, d] = src f32 [rows, d] rounded to nearest (ties to even):
 * expert-output rows made ready for the bf16 return exchange above.  d a
 * multiple of 64 (MOE_ERR_UNSUPPORTED otherwise), rows < 2^31, both pointers
 * device memory, 16-byte aligned (MOE_ERR_INVALID_ARG otherwise); rows = 0 is
 * a no-op.  Caller owns both buffers. */
int moe_rows_to_bf16(const float* src, void* dst, int64_t rows, int64_t d, void* stream);

/* ---- Padded-capacity layout (an optional variant of moe_permute) ----
 * The static [E, C, d] buffer the neelmishra page contrasts with ragged
 * buckets ("Expert Parallelism & All-to-All", section "Why fixed-size buffers
 * matter here": fixed-shape buffers cost padded compute when an expert is
 * under-filled).  Bucket e occupies rows e*C .. e*C + C - 1 whatever its
 * count. */

/* E*C rows of the padded buffer; -1 on bad args or E*C >= 2^31. */
int64_t moe_padded_rows(int64_t T, int64_t E, int64_t k, double cf);

/* moe_permute into the padded layout: counts, slot and n_dropped as
 * moe_permute; offsets[e] = e*C (offsets[E] = E*C), so the grouped GEMM and
 * combine entry points run on it unchanged and compute every row of every
 * bucket; x_pad bf16 [E*C, d] holds bucket e's kept rows at e*C + slot and
 * zeros after them; row_src i32 [E*C] the source token, -1 on padding rows. */
int moe_permute_padded(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                       int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                       int32_t* row_src, void* x_pad, int32_t* n_dropped, void* ws,
                       size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---- Buckets that are not experts (expert parallelism) ----
 * With the experts spread over P ranks ("Expert Parallelism & All-to-All"
 * (neelmishra), sections on dispatch and combine; "Expert Parallelism" guide
 * (infra.bea.ai), section 2), a rank receives from every source rank q a
 * fixed-size slot per local expert; bucket b = q * E_w + e holds the rows q
 * sent to local expert e, of which only the first bucket_rows[b] are real. */

/* moe_expert_mlp over B buckets: bucket b = rows offsets[b] .. offsets[b+1]-1
 * of x_rows (only the first bucket_rows[b] of them when bucket_rows is
 * non-null) through expert b % E_w of w_gate/w_up [E_w,d,f], w_down [E_w,f,d];
 * h bf16 [max_rows,f] and y_rows f32 [max_rows,d] out (rows past
 * bucket_rows[b] are not written).  B <= 256, B a multiple of E_w. */
int moe_expert_mlp_buckets(const void* x_rows, const int32_t* offsets, const int32_t* bucket_rows,
                           int64_t B, int64_t E_w, int64_t d, int64_t f, int64_t max_rows,
                           const void* w_gate, const void* w_up, const void* w_down, void* h,
                           float* y_rows, int32_t* dev_status, void* stream);

/* ---- Fused path (an optional variant) ----
 * The combine folded into the down GEMM ("Expert Parallelism" guide
 * (infra.bea.ai), section 5: fuse the gather into the expert GEMM and the
 * weighted scatter into its epilogue): GEMM 2 adds each gate-weighted output
 * row into an fp32 token accumulator y32 (red.add) instead of storing y_perm,
 * and a last pass rounds y32 to bf16.  The summation order of a token's k
 * terms then follows the GEMM tiles' completion, not j: results agree with
 * moe_layer_forward to fp32 rounding but are not bit-reproducible run to run.
 * The gather side (GEMM 1 reading x by row_src with TMA tile::gather4, no
 * x_perm) is available as moe_expert_gate_up_gather; it saves the x_perm
 * buffer but costs one 4-row copy per 512 bytes of A, which on B200 made the
 * gate/up GEMM ~3x slower than the permuted copy plus a tile load, so the
 * fused layer keeps the copy. */

/* The permutation for the fused path: moe_permute (counts, offsets, slot,
 * row_src, n_dropped; x_perm when x and x_perm are non-null, else no row
 * copy) plus row_pair i32 [max_rows] (t*k + j of each kept row) and, when
 * y32 is non-null, y32 f32 [T,d] zeroed. */
int moe_permute_fused(const void* x, const int32_t* topk_idx, int64_t T, int64_t d, int64_t E,
                      int64_t k, double cf, int32_t* counts, int32_t* offsets, int32_t* slot,
                      int32_t* row_src, int32_t* row_pair, void* x_perm, int32_t* n_dropped,
                      float* y32, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* moe_expert_gate_up with A row r of bucket storage = x[row_src[r]] (x bf16
 * [T,d], row_src from the permutation; no x_perm). */
int moe_expert_gate_up_gather(const void* x, int64_t T, const int32_t* row_src,
                              const int32_t* offsets, int64_t E, int64_t d, int64_t f,
                              int64_t max_rows, const void* w_gate, const void* w_up, void* h,
                              int32_t* dev_status, void* stream);

/* moe_expert_down with the combine's weighted sum in its epilogue:
 * y32[t, :] += topk_w[p] * (h[r] Wd[e]) for each kept row r, p = row_pair[r],
 * t = p / k.  y32 f32 [T,d] must hold zeros (or a sum to add to). */
int moe_expert_down_scatter(const void* h, const int32_t* offsets, int64_t E, int64_t d,
                            int64_t f, int64_t max_rows, const void* w_down,
                            const int32_t* row_pair, const float* topk_w, int64_t k, float* y32,
                            int32_t* dev_status, void* stream);

/* y[t] = bf16(y32[t]), or x[t] when every pair of t was dropped (slot < 0). */
int moe_combine_finalize(const float* y32, const void* x, const int32_t* slot, int64_t T,
                         int64_t d, int64_t k, void* y, void* stream);

/* Workspace of moe_layer_forward_fused: the moe_layer_forward fields followed
 * by MOE_WS_ROW_PAIR and MOE_WS_Y32 (0 on invalid shapes). */
size_t moe_workspace_size_fused(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                                double cf);

/* The layer on the fused path: moe_route, moe_permute_fused (with x_perm),
 * moe_expert_gate_up, moe_expert_down_scatter, moe_combine_finalize.
 * Arguments as moe_layer_forward. */
int moe_layer_forward_fused(const void* x, const float* w_router, const float* bias,
                            const void* w_gate, const void* w_up, const void* w_down, int64_t T,
                            int64_t d, int64_t E, int64_t k, int64_t f, double cf, void* y,
                            void* ws, size_t ws_bytes, void* stream);

/* ---- FP8 experts (e4m3 activations and weights; an optional variant) ----
 * Post-training FP8 quantization of the experts (inferensys.com "Expert
 * Parallelism" glossary, quantization entry).  One rule for every group of
 * values that shares a scale (a weight column over K, an activation row over
 * K): s = max |v| / 448 in fp32 (1 for an all-zero group), code = e4m3 of
 * v / s rounded to nearest even, saturating at +-448.  A row scale times a
 * column scale is constant along the contraction, so the expert GEMMs run on
 * the codes (tcgen05.mma.kind::f8f6f4, fp32 accumulation) and multiply each
 * accumulator by its row and column scales.  Routing, the permutation, h as
 * stored (bf16), y_perm (f32) and the combine are those of the bf16 path. */

/* Quantize bf16 weights w [E,K,N] (N contiguous; gate/up: K=d, N=f; down:
 * K=f, N=d) per (expert, column n): scale [E,N] f32 out, codes w_q out
 * stored K-major as u8 [E,N,K] (the transpose of w's layout).  Any K, N >= 1,
 * E <= 65535.  A one-time preprocessing step. */
int moe_quantize_weights_fp8(const void* w, int64_t E, int64_t K, int64_t N, uint8_t* w_q,
                             float* scale, void* stream);

/* Quantize bf16 rows x [R,K] per row: codes q u8 [R,K], scale [R] f32.  Rows
 * r >= *n_rows are skipped when n_rows (a device int32, e.g. offsets[E] of a
 * permutation) is non-null.  K a multiple of 16; x and q 16-byte aligned. */
int moe_quantize_rows_fp8(const void* x, int64_t R, int64_t K, const int32_t* n_rows, uint8_t* q,
                          float* scale, void* stream);

/* moe_permute on e4m3 token rows: the same counts, offsets, slots, row_src
 * and n_dropped, with the codes xq u8 [T,d] and row scales sx f32 [T] (from
 * moe_quantize_rows_fp8 on x) moved to xq_perm u8 [max_rows,d] and sx_perm
 * f32 [max_rows].  Per-row quantization commutes with the row copy, so this
 * equals quantizing moe_permute's x_perm. */
int moe_permute_fp8(const uint8_t* xq, const float* sx, const int32_t* topk_idx, int64_t T,
                    int64_t d, int64_t E, int64_t k, double cf, int32_t* counts,
                    int32_t* offsets, int32_t* slot, int32_t* row_src, uint8_t* xq_perm,
                    float* sx_perm, int32_t* n_dropped, void* ws, size_t ws_bytes,
                    int32_t* dev_status, void* stream);

/* GEMM 1 + SwiGLU on e4m3 operands: h[r,:] = silu(g) * u with
 * g[r,n] = sx[r] * s_gate[e,n] * sum_k xq[r,k] wq_gate[e,n,k] (u likewise) for
 * rows r of bucket e.  xq u8 [max_rows,d], sx f32 [max_rows], wq_* u8 [E,f,d]
 * (from moe_quantize_weights_fp8), s_* f32 [E,f]; h bf16 [max_rows,f] out.
 * Shapes and errors as moe_expert_gate_up. */
int moe_expert_gate_up_fp8(const uint8_t* xq, const float* sx, const int32_t* offsets, int64_t E,
                           int64_t d, int64_t f, int64_t max_rows, const uint8_t* wq_gate,
                           const float* s_gate, const uint8_t* wq_up, const float* s_up, void* h,
                           int32_t* dev_status, void* stream);

/* GEMM 2 on e4m3 operands: y_perm[r,n] = sh[r] * s_down[e,n] * sum_k
 * hq[r,k] wq_down[e,n,k].  hq u8 [max_rows,f], sh f32 [max_rows], wq_down u8
 * [E,d,f], s_down f32 [E,d]; y_perm f32 [max_rows,d] out. */
int moe_expert_down_fp8(const uint8_t* hq, const float* sh, const int32_t* offsets, int64_t E,
                        int64_t d, int64_t f, int64_t max_rows, const uint8_t* wq_down,
                        const float* s_down, float* y_perm, int32_t* dev_status, void* stream);

/* Workspace of moe_layer_forward_fp8: the moe_layer_forward fields followed by
 * MOE_WS_XQ .. MOE_WS_SX_TOK (0 on invalid shapes). */
size_t moe_workspace_size_fp8(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf);

/* The layer with FP8 experts: moe_route, moe_quantize_rows_fp8 (x),
 * moe_permute_fp8, moe_expert_gate_up_fp8, moe_quantize_rows_fp8 (h),
 * moe_expert_down_fp8, moe_combine on `stream` (the bf16 x_perm field of the
 * workspace is not used).  Weights and scales from
 * moe_quantize_weights_fp8; other arguments as moe_layer_forward. */
int moe_layer_forward_fp8(const void* x, const float* w_router, const float* bias,
                          const uint8_t* wq_gate, const float* s_gate, const uint8_t* wq_up,
                          const float* s_up, const uint8_t* wq_down, const float* s_down,
                          int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, double cf,
                          void* y, void* ws, size_t ws_bytes, void* stream);

/* The whole layer: moe_route, moe_permute, moe_expert_mlp, moe_combine on
 * one stream, every intermediate in `ws` (>= moe_workspace_size bytes; field
 * layout from moe_workspace_field_offset).  No host synchronisation: bucket
 * sizes stay on the device.  y bf16 [T,d] out. */
int moe_layer_forward(const void* x, const float* w_router, const float* bias, const void* w_gate,
                      const void* w_up, const void* w_down, int64_t T, int64_t d, int64_t E,
                      int64_t k, int64_t f, double cf, void* y, void* ws, size_t ws_bytes,
                      void* stream);

/* moe_layer_forward with the routing results written where the caller wants
 * them: each non-null output pointer (device memory the caller owns) takes
 * the place of the workspace field of the same name, so the stages write it
 * there directly and no copy is made; a null pointer leaves that result in
 * the workspace as moe_layer_forward does.
 *   logits_out   f32 [T,E]   router logits (MOE_WS_LOGITS)
 *   topk_idx_out i32 [T,k]   selected experts (MOE_WS_TOPK_IDX)
 *   topk_w_out   f32 [T,k]   gate weights (MOE_WS_TOPK_W)
 *   slot_out     i32 [T,k]   bucket slots, -1 = dropped (MOE_WS_SLOT)
 *   counts_out   i32 [E]     pairs kept per expert (MOE_WS_COUNTS)
 * ws is still required (>= moe_workspace_size bytes; the replaced fields are
 * left unused).  Same sources, shapes and errors as moe_layer_forward. */
int moe_layer_forward_ex(const void* x, const float* w_router, const float* bias,
                         const void* w_gate, const void* w_up, const void* w_down, int64_t T,
                         int64_t d, int64_t E, int64_t k, int64_t f, double cf, void* y,
                         float* logits_out, int32_t* topk_idx_out, float* topk_w_out,
                         int32_t* slot_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBMOE_MOE_H_ */
