/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * The layer (sources, by page title and section):
 *   [report-walkthrough] "DeepSeek-V3 technical report" walkthrough (2kiu.com),
 *       section 3.2 (sigmoid affinities, bias-ranked top-K, gates from s,
 *       batch-level bias update), section 3.4 (node-limited routing),
 *       section 4.3 (FP8 block scaling, high-precision accumulation);
 *   [repro-guide] "From technical report to a runnable config" (lpnh.cn),
 *       section 3 (num_experts 256, 1 shared, top-8, moe_intermediate 2048,
 *       norm_topk_prob, routed_scaling_factor 2.5, e4m3, 1x128 input tiles,
 *       128x128 weight blocks, moe_gating kept in high precision);
 *   [infra-answer] Zhihu answer on DeepSeek-V3's infrastructure: E4M3
 *       throughout, per-tile/per-group scales, partial-sum promotion.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates or frees memory.  Row-major everywhere;
 *     weights are [N, K] with K contiguous ("K-major").
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous and stream-ordered, keep no state
 *     between calls, and are safe to call from several host threads.
 *   - Host-side argument checks run before any launch and return
 *     MOE_ERR_INVALID_ARG (bad sizes, NULL or misaligned pointers) or
 *     MOE_ERR_UNSUPPORTED (valid but outside what the kernels implement).
 *     A launch failure returns MOE_ERR_CUDA.  Zero-size work returns MOE_OK
 *     without launching.
 *   - `status`, where present, is an optional device int32 that kernels
 *     OR MOE_FLAG_* bits into (never cleared by the library); NULL skips it.
 *   - Pointers to packed 16-byte vectors (bf16 rows, e4m3 rows, scales)
 *     must be 16-byte aligned.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem statement of one layer, as the pages state it: T tokens, hidden
 * size H, E routed experts, top-K, n_group expert groups of which
 * topk_group are kept per token (the node limit of [report-walkthrough]
 * section 3.4), expert intermediate size I and routed_scaling_factor
 * ([repro-guide] section 3). */
typedef struct moe_dims {
    int32_t T, H, E, K, n_group, topk_group, I;
    float routed_scaling_factor;
} moe_dims;

enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_TOO_LARGE = 5
};

/* Bits kernels OR into the optional device status word. */
enum moe_flag {
    MOE_FLAG_NONFINITE = 1,  /* a quantised tile held NaN/Inf: codes 0x7F, scale NaN */
    MOE_FLAG_BAD_INDEX = 2,  /* an expert index outside [0, E): entry skipped          */
    MOE_FLAG_TIMEOUT = 4,    /* a bounded on-device wait gave up; outputs undefined     */
    MOE_FLAG_BAD_OFFSETS = 8 /* group offsets not monotone or beyond m_capacity         */
};

/* GEMM epilogues. */
enum moe_epilogue {
    MOE_EPI_BF16 = 0,          /* C bf16 [M, N]                                      */
    MOE_EPI_F32 = 1,           /* C fp32 [M, N]                                      */
    MOE_EPI_SWIGLU_REQUANT = 2, /* N = 2I: C e4m3 [M, I] codes, sC fp32 [M, I/128]     */
    MOE_EPI_COMBINE_F32 = 3,   /* fp8_grouped_gemm_blockscaled_combine only              */
    /* OR-ed into `epilogue`: the tile mode.  Default (neither bit) and
     * MOE_GEMM_SINGLE_CTA: one-SM tiles of 128 rows.  MOE_GEMM_PAIR_CTA: tiles
     * of 256 rows on a cluster of two SMs (tcgen05 cta_group::2), each SM
     * staging half of the weight tile.  Same results either way. */
    MOE_GEMM_SINGLE_CTA = 0x100,
    MOE_GEMM_PAIR_CTA = 0x200
};

/* Human-readable name of a moe_status value.  Static string, never NULL. */
const char *moe_status_string(int status);

/* Library ABI version (increments on any signature change). */
int moe_abi_version(void);

/* Bytes of scratch `ws` that moe_route and moe_permute need for `dims`
 * (the larger of the two).  ws must be 256-byte aligned. */
size_t moe_workspace_size(const moe_dims *dims);

/* Activation quantisation, one scale per 1x128 tile ([report-walkthrough]
 * section 4.3; [repro-guide] section 3 input_quant_granularity
 * tile_wise_1x128, format e4m3).  For each row r and tile j:
 *   amax = max |x[r, 128j .. 128j+127]|
 *   scales[r, j] = amax == 0 ? 1 : fp32(amax / 448)
 *   q[r, c] = e4m3_rne_satfinite(fp32(x[r, c] / scales[r, j]))
 * A tile holding NaN/Inf gets codes 0x7F, scale NaN and MOE_FLAG_NONFINITE.
 *   x      bf16 [rows, cols], cols % 128 == 0
 *   q      e4m3 codes uint8 [rows, cols]
 *   scales fp32 [rows, cols/128]                                              */
int fp8_quant_1x128(const void *x, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                    int32_t *status, void *stream);

/* Weight quantisation, one scale per 128x128 block ([repro-guide] section 3
 * weight_quant_granularity block_wise_128x128; [infra-answer]).  Same rule
 * as fp8_quant_1x128 with the block in place of the tile.  A setup step.
 *   w      bf16 [batch, rows, cols], rows % 128 == 0, cols % 128 == 0
 *   q      uint8 [batch, rows, cols]
 *   scales fp32 [batch, rows/128, cols/128]                                   */
int fp8_quant_128x128(const void *w, int64_t batch, int64_t rows, int64_t cols, uint8_t *q,
                      float *scales, int32_t *status, void *stream);

/* Router ([report-walkthrough] sections 3.2 and 3.4; gating kept in fp32 per
 * [repro-guide] section 3 keep_bf16 moe_gating):
 *   s = sigmoid(x W_r^T + router_offset)      fp32 accumulation
 *   r = s + e_bias (one fp32 add); group score = fp32 sum of the top
 *   min(2, E/n_group) r in each of n_group groups; keep the topk_group best
 *   groups; topk_idx = top-K of r over the kept experts, in descending r,
 *   ties to the lower index (groups and experts alike);
 *   topk_w[t,k] = fp32((rho * s_k) / sum_j s_j) evaluated in float64.
 *   x             bf16 [T, H]
 *   w_router      fp32 [E, H]
 *   e_bias        fp32 [E]
 *   router_offset fp32 [E] additive logit offset, or NULL
 *   topk_idx      int32 [T, K];  topk_w fp32 [T, K]
 *   scores        fp32 [T, E] output of s, or NULL (then ws holds it)
 * Limits: E <= 1024, E % n_group == 0, n_group <= 32, K <= 32,
 * topk_group * E / n_group >= K, H % 128 == 0.                                 */
int moe_route(const moe_dims *dims, const void *x, const float *w_router, const float *e_bias,
              const float *router_offset, int32_t *topk_idx, float *topk_w, float *scores,
              void *ws, size_t ws_bytes, int32_t *status, void *stream);

/* The router weights split once, for callers that route many batches with the
 * same W_r: moe_router_split writes the three exact bf16 pieces of W_r
 * (W_r = P0 + P1 + P2 element by element: P0 = bf16(W_r), P1 = bf16(W_r - P0),
 * P2 = W_r - P0 - P1, which has at most 8 significant bits), the operand of
 * moe_route's tensor-core logits; moe_route_pieces is moe_route with those
 * pieces in place of w_router and gives the same bits.  The pieces stay valid
 * until W_r changes.
 *   w_router fp32 [E, H];  w_pieces bf16 [3, E, H] (moe_router_pieces_bytes)
 *   moe_route_pieces takes the workspace of moe_route (moe_workspace_size). */
size_t moe_router_pieces_bytes(int32_t E, int32_t H);
int moe_router_split(const float *w_router, int32_t E, int32_t H, void *w_pieces, void *stream);
int moe_route_pieces(const moe_dims *dims, const void *x, const void *w_pieces, const float *e_bias,
                     const float *router_offset, int32_t *topk_idx, float *topk_w, float *scores,
                     void *ws, size_t ws_bytes, int32_t *status, void *stream);

/* The selection half of moe_route alone, on given affinities s fp32 [T, E]. */
int moe_route_select(const moe_dims *dims, const float *scores, const float *e_bias,
                     int32_t *topk_idx, float *topk_w, void *stream);

/* Dispatch into per-expert segments (the token-to-expert step of
 * [report-walkthrough] sections 3.2 and 4.1; no token is dropped, section
 * 3.4).  A stable counting sort of the T*K (token, slot) pairs by expert:
 *   expert_load[e]    = #pairs routed to e                     int32 [E]
 *   expert_offsets[e] = exclusive prefix of expert_load        int32 [E+1]
 *   rows offsets[e] .. offsets[e+1]-1 hold expert e's pairs in ascending
 *   token order; tok_of[row] = token, row_of[t*K + k] = row    int32 [T*K]
 *   aq[row, :] = xq[tok_of[row], :]  (e4m3 [T*K, H]),
 *   as[row, :] = xs[tok_of[row], :]  (fp32 [T*K, H/128]);
 * xq/xs/aq/as may all be NULL to build the maps only.  An index outside
 * [0, E) raises MOE_FLAG_BAD_INDEX and that pair gets row_of = -1.         */
int moe_permute(const moe_dims *dims, const int32_t *topk_idx, const uint8_t *xq, const float *xs,
                int32_t *expert_load, int32_t *expert_offsets, int32_t *tok_of, int32_t *row_of,
                uint8_t *aq, float *as, void *ws, size_t ws_bytes, int32_t *status, void *stream);

/* moe_permute for callers that cannot allocate device memory.  The pages have
 * no counterpart to this call; it exists for the host side.  Some callers may
 * not call cudaMalloc at all: code that runs inside a host framework which owns
 * every device buffer and forbids allocations in its kernels' call path, fixed
 * memory budgets planned ahead of time (real-time or embedded deployments), and
 * paths that must not synchronise the device, as cudaMalloc/cudaFree can.  This
 * call takes no workspace: its scratch (the per-chunk expert counts) is a
 * static device array of moe_permute_noalloc_max_scratch() bytes (1 MiB) that
 * is part of the library's device image, so every GPU that loads the library
 * holds it until the process exits.  The caller still passes every input and
 * output, with the meaning, layout and limits of moe_permute.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - Problems whose counts exceed the scratch (ceil(T/32) * E * 4 bytes >
 *     1 MiB, e.g. T > 32768 at E = 256) return MOE_ERR_TOO_LARGE.
 *   - All calls share the one array and it keeps the last call's contents;
 *     each call writes every count it reads before reading it, so nothing
 *     needs clearing.  Calls whose work overlaps on the GPU (different
 *     streams, or different host threads without ordering) race on the
 *     array and give undefined results: order them on one stream.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.      */
int moe_permute_noalloc(const moe_dims *dims, const int32_t *topk_idx, const uint8_t *xq, const float *xs,
                        int32_t *expert_load, int32_t *expert_offsets, int32_t *tok_of, int32_t *row_of,
                        uint8_t *aq, float *as, int32_t *status, void *stream);

/* Size in bytes of moe_permute_noalloc's static scratch array. */
size_t moe_permute_noalloc_max_scratch(void);

/* Grouped FP8 GEMM with block scales, promoted every 128 of K
 * ([report-walkthrough] section 4.3; [infra-answer]: the tile/block scales
 * have no hardware support, so partial sums are promoted).  For group g,
 * rows m in [group_offsets[g], group_offsets[g+1]):
 *   C[m, n] = sum_kb sA[m, kb] * sB[g, n/128, kb] *
 *             sum_{k in kb} e4m3(A[m, k]) * e4m3(B[g, n, k])
 * with fp32 accumulation of each 128-wide partial and of the promotion.
 *   group_offsets  device int32 [G+1], non-decreasing, last <= m_capacity
 *   A   e4m3 [m_capacity, K];  sA fp32 [m_capacity, K/128]
 *   B   e4m3 [G, N, K];        sB fp32 [G, N/128, K/128]
 *   MOE_EPI_BF16 / MOE_EPI_F32: C [m_capacity, N] (rows outside every
 *   group are not written).
 *   MOE_EPI_SWIGLU_REQUANT: B rows 0..I-1 are the gate and I..2I-1 the up
 *   projection (N = 2I); act = silu(g) * u in fp32, then the 1x128 rule of
 *   fp8_quant_1x128: C e4m3 [m_capacity, I], sC fp32 [m_capacity, I/128].
 * Limits: K % 128 == 0, N % 128 == 0 (SwiGLU: I % 128 == 0), G <= 4000.    */
int fp8_grouped_gemm_blockscaled(int32_t G, const int32_t *group_offsets, int64_t m_capacity,
                                 int64_t N, int64_t K, const uint8_t *A, const float *sA,
                                 const uint8_t *B, const float *sB, int32_t epilogue, void *C,
                                 float *sC, int32_t *status, void *stream);

/* fp8_grouped_gemm_blockscaled with the A rows gathered through a row map
 * instead of stored in group order ([report-walkthrough] sections 3.2 and 4.1:
 * the routed rows are dispatched to their experts; gathering them inside the
 * GEMM leaves the result unchanged and never writes the permuted copy):
 *   row m of group g reads A row a_map[m] and its scales sA[a_map[m], :],
 *   i.e. C[m, n] = sum_kb sA[a_map[m], kb] * sB[g, n/128, kb] *
 *                  sum_{k in kb} e4m3(A[a_map[m], k]) * e4m3(B[g, n, k])
 *   A  e4m3 [a_rows, K] (16-byte aligned);  sA fp32 [a_rows, K/128]
 *   a_map device int32 [m_capacity]; entries of rows outside every group are
 *   not read.  An entry outside [0, a_rows) raises MOE_FLAG_BAD_INDEX and that
 *   output row is unspecified (nothing is read outside A).  a_rows >= 1.
 * Everything else (groups, B, epilogues, C, limits) as fp8_grouped_gemm_blockscaled;
 * the call always runs one-SM tiles (MOE_GEMM_PAIR_CTA is ignored).  In the
 * layer, A is the T quantised token rows and a_map the permutation's tok_of
 * followed by 0..T-1 for the shared expert's group.                         */
int fp8_grouped_gemm_blockscaled_gather(int32_t G, const int32_t *group_offsets, int64_t m_capacity,
                                        int64_t N, int64_t K, const uint8_t *A, const float *sA,
                                        int64_t a_rows, const int32_t *a_map, const uint8_t *B,
                                        const float *sB, int32_t epilogue, void *C, float *sC,
                                        int32_t *status, void *stream);

/* fp8_grouped_gemm_blockscaled with the gated combine in its epilogue
 * ([report-walkthrough] section 3.2: y = sum_j gate_j * ffn_j(h), plus the
 * shared expert; section 4.1: combine after the expert MLP).  Row m of group g
 * is not stored: its bf16-rounded value, times row_gate[m], is added into the
 * fp32 row row_token[m] of out_f32:
 *   out_f32[row_token[m], n] += row_gate[m] * bf16(C[m, n])
 * (C[m, n] as fp8_grouped_gemm_blockscaled defines it).  In the layer,
 * row_token is tok_of followed by 0..T-1 and row_gate the gates in row order
 * followed by 1 for the shared expert's rows, so out_f32 (zeroed before)
 * receives the layer's output before its bf16 rounding; moe_combine_finish
 * rounds it and re-zeroes the accumulator.
 *   row_token int32 [m_capacity] (entries outside [0, out_rows) of rows in a
 *   group raise MOE_FLAG_BAD_INDEX and that row is skipped), row_gate fp32
 *   [m_capacity], out_f32 fp32 [out_rows, N] (16-byte aligned).
 * The additions are fp32 reductions at the L2 in no fixed order: results agree
 * with a fixed-order fp32 sum within its rounding bound, not bit for bit.
 * Single tiles; other arguments and limits as fp8_grouped_gemm_blockscaled.  */
int fp8_grouped_gemm_blockscaled_combine(int32_t G, const int32_t *group_offsets, int64_t m_capacity,
                                         int64_t N, int64_t K, const uint8_t *A, const float *sA,
                                         const uint8_t *B, const float *sB, const int32_t *row_token,
                                         const float *row_gate, int64_t out_rows, float *out_f32,
                                         int32_t *status, void *stream);

/* out_bf16[i] = bf16(acc[i]) (round to nearest even) for n fp32 values (n % 8
 * == 0, 16-byte aligned buffers); out_f32 (or NULL) receives a copy of acc;
 * with zero != 0 acc is then set to 0 (ready for the next accumulation).    */
int moe_combine_finish(float *acc, int64_t n, void *out_bf16, float *out_f32, int32_t zero, void *stream);

/* Backward pass, weight gradient of the grouped expert GEMMs in FP8 ([repro-guide]
 * section 3: gemm_wgrad in e4m3 with 1x128 input tiles; [infra-answer]: E4M3
 * in the forward and the backward pass).  For group g (rows m in
 * [group_offsets[g], group_offsets[g+1]) of dY [M, N] and X [M, K]):
 *   dW[g, n, k] = sum_t sdy[t, n] * sx[t, k] * sum_{m in tile t} e4m3(dY[m, n]) e4m3(X[m, k])
 * The contraction runs over the group's rows, so the 1x128 tiling is taken
 * along it: tiles of 128 consecutive rows of one column (128x1) that never
 * cross the group's row range (the last tile of a ragged group is shorter).
 *
 * fp8_quant_128x1_grouped quantises x bf16 [M, C] (C % 128 == 0) that way,
 * with the scale rule of fp8_quant_1x128, and writes the codes TRANSPOSED and
 * padded: q_t[c, 128 t + r] = code of row r of tile t in column c (tiles
 * numbered in group order, codes 0 beyond a short tile), uint8 [C, p_capacity];
 * scales[t, c] fp32 [t_capacity, C].  Capacities: t_capacity >= the number of
 * tiles (at most ceil(M/128) + G), p_capacity >= 128 * t_capacity and a
 * multiple of 16.  Offsets that decrease, exceed M or need more tiles than the
 * capacities raise MOE_FLAG_BAD_OFFSETS and nothing is written.
 *
 * fp8_grouped_gemm_wgrad takes two such operands quantised with the same
 * offsets -- dy_t/sdy from dY (C = N) and x_t/sx from X (C = K) -- and writes
 * dW fp32 [G, N, K] (an empty group gets zeros); N % 128 == 0, K % 128 == 0,
 * G <= 2048; fp32 accumulation of each 128-row partial and of the promotion. */
int fp8_quant_128x1_grouped(const void *x, int64_t M, int64_t C, int32_t G, const int32_t *group_offsets,
                            uint8_t *q_t, int64_t p_capacity, float *scales, int64_t t_capacity,
                            int32_t *status, void *stream);
int fp8_grouped_gemm_wgrad(int32_t G, const int32_t *group_offsets, int64_t M, int64_t N, int64_t K,
                           const uint8_t *dy_t, const float *sdy, const uint8_t *x_t, const float *sx,
                           int64_t p_capacity, int64_t t_capacity, float *dW, int32_t *status, void *stream);

/* SwiGLU and 1x128 requantisation of a given fp32 [M, 2I] gate|up matrix
 * (the GEMM epilogue's arithmetic as a stand-alone call; SwiGLU named in
 * [infra-answer], expert intermediate I per [arch-overview]
 * "DeepSeek-V3 MoE architecture and FP8 training" (0539edu.com)):
 *   act = (g / (1 + exp(-g))) * u   in fp32;  q, s as in fp8_quant_1x128.
 *   q uint8 [M, I];  s fp32 [M, I/128]                                        */
int swiglu_requant(const float *gu, int64_t M, int64_t I, uint8_t *q, float *s, int32_t *status,
                   void *stream);

/* Gated combine ([report-walkthrough] section 3.2: y = sum_j gate_j *
 * ffn_{idx_j}(h)) plus the shared expert:
 *   out[t] = sum_k topk_w[t,k] * yperm[row_of[t*K+k]] + yshared[t]
 * summed in fp32 in k order (shared last), stored as bf16 and optionally fp32.
 *   yperm bf16 [T*K, H]; yshared bf16 [T, H] or NULL; out bf16 [T, H];
 *   out_f32 fp32 [T, H] or NULL.  Pairs with row_of < 0 are skipped.          */
int moe_combine(const moe_dims *dims, const void *yperm, const int32_t *row_of,
                const float *topk_w, const void *yshared, void *out, float *out_f32, void *stream);

/* Expert-parallel placement ([report-walkthrough] section 4.1: experts spread
 * over devices; tokens dispatched to the devices of their experts and combined
 * back).  Routed expert e lives on rank e % world as local expert e / world.
 *   moe_ep_split:   dest_rank[i] = topk_idx[i] % world, local_idx[i] = topk_idx[i] / world
 *                   for n entries; an index outside [0, E) gets -1 in both and
 *                   raises MOE_FLAG_BAD_INDEX.
 *   moe_ep_scatter: out[row_of[i]] = values[i] for the n entries with row_of[i] >= 0
 *                   (per-pair values into the order of a moe_permute result).
 * With these, dispatch is moe_permute with the destination ranks as its groups
 * (rows grouped by rank, (token, slot) order inside each), and the combine of
 * the returned rows is moe_combine with that permutation's row_of.              */
int moe_ep_split(const int32_t *topk_idx, int64_t n, int32_t E, int32_t world, int32_t *dest_rank,
                 int32_t *local_idx, int32_t *status, void *stream);
int moe_ep_scatter(const int32_t *row_of, const int32_t *values, int64_t n, int32_t *out, void *stream);

/* Node-limited dispatch: each token sent at most once to each rank
 * ([report-walkthrough] section 3.4: a token reaches at most M nodes, picked by
 * group; section 4.1: it crosses to a node once and is forwarded there to the
 * experts it selected on that node; [infra-answer]: grouped routing caps the
 * nodes per token at 4, halving cross-node traffic).  Placement:
 *   MOE_EP_CYCLIC  expert e on rank e % world as local expert e / world
 *   MOE_EP_BLOCK   expert e on rank e / (E/world) as local expert e % (E/world)
 *                  (with world = n_group, rank = group: topk_group ranks at most)
 * moe_ep_plan, for T tokens x K slots (K <= 32, E % world == 0):
 *   dest_rank[t*K+k] = rank of slot k's expert if no earlier slot of token t has
 *                      that rank, else -1 (not dispatched)
 *   for a dispatched slot i = t*K+k, row i of meta_ids / meta_w [T*K, K]:
 *     meta_ids[i, j] = local expert id of slot j if slot j's expert is on
 *                      dest_rank[i], else -1;  meta_w[i, j] = topk_w[t, j] or 0
 *   (rows of slots that are not dispatched hold -1 / 0).
 * An expert index outside [0, E) raises MOE_FLAG_BAD_INDEX; that slot is not
 * dispatched.  Dispatch is then moe_permute with dest_rank as its indices and
 * the ranks as groups (status NULL: the -1 slots are skipped, not errors), the
 * metadata moved into its order with moe_ep_scatter_rows; on the receiver the
 * rows' meta_ids are the indices of a moe_permute over the local experts, and
 * moe_combine with meta_w sums each row's experts.
 * moe_ep_scatter_rows: out[row_of[i], :] = values[i, :] for rows of `width`
 *                      int32 (fp32 bit patterns move unchanged) with row_of[i] >= 0. */
#define MOE_EP_CYCLIC 0
#define MOE_EP_BLOCK 1
int moe_ep_plan(const int32_t *topk_idx, const float *topk_w, int64_t T, int32_t K, int32_t E, int32_t world,
                int32_t placement, int32_t *dest_rank, int32_t *meta_ids, float *meta_w, int32_t *status,
                void *stream);
int moe_ep_scatter_rows(const int32_t *row_of, const int32_t *values, int64_t n, int32_t width, int32_t *out,
                        void *stream);

/* The whole layer forward in one call ([report-walkthrough] sections 3.2 and
 * 4.1: route -> dispatch -> expert MLP -> combine; section 4.3: FP8 steps):
 * moe_route_pieces, fp8_quant_1x128, moe_permute, the two grouped GEMMs (the
 * shared expert as group E) and moe_combine, then optionally moe_bias_update.
 * Every buffer is the caller's (device memory, the sizes of the single calls):
 *   w13, s13, w2, s2     the E+1 experts' E4M3 weights and scales (shared last)
 *   w_pieces             moe_router_split's pieces of W_r; e_bias [E];
 *                        router_offset [E] or NULL
 *   topk_idx, topk_w [T,K], scores [T,E]
 *   aq [T*K+T, H], as [T*K+T, H/128]  A of the first GEMM; its last T rows
 *                        receive the quantised tokens
 *   load [E]; offsets [E+2] with offsets[E+1] = T*K+T set by the caller once
 *                        (moe_permute writes entries 0..E)
 *   tok_of, row_of [T*K]; actq [T*K+T, I], acts [T*K+T, I/128]
 *   yperm bf16 [T*K+T, H] (its last T rows: the shared expert's output)
 *   ws, ws_bytes >= moe_workspace_size(dims); status (may be NULL)
 *   bias_out [E] or NULL: when set, bias_out += gamma * sign(T*K/E - load)
 *                        after the forward (the routing bias, or a copy of it)
 * moe_layer_forward: x bf16 [T,H] -> out bf16 [T,H] (device), on `stream`.
 * moe_layer_run_host: n batches from host memory: batch i's x_host[i] (pinned
 * bf16 [T,H]) is uploaded on a stream of its own into x_dev[i % 2], the forward
 * runs on `stream` into out_dev[i % 2], and out_host[i] (pinned) is downloaded
 * on a third stream, so the copies of batches i+1 and i-1 overlap batch i's
 * forward.  One cudaMemcpyAsync per copy; the copies start after the work
 * already enqueued on `stream`.  Returns once everything is enqueued; `stream`
 * completes after the last download.                                          */
typedef struct {
    moe_dims dims;
    const uint8_t *w13;
    const float *s13;
    const uint8_t *w2;
    const float *s2;
    const void *w_pieces;
    const float *e_bias;
    const float *router_offset;
    int32_t *topk_idx;
    float *topk_w;
    float *scores;
    uint8_t *aq;
    float *as;
    int32_t *load;
    int32_t *offsets;
    int32_t *tok_of;
    int32_t *row_of;
    uint8_t *actq;
    float *acts;
    void *yperm;
    void *ws;
    size_t ws_bytes;
    int32_t *status;
    float *bias_out;
    float gamma;
} moe_layer;
int moe_layer_forward(const moe_layer *layer, const void *x, void *out, void *stream);
int moe_layer_run_host(const moe_layer *layer, const void *const *x_host, void *const *out_host, int32_t n,
                       void *const *x_dev, void *const *out_dev, void *stream);

/* Sequence-wise balance loss and expert-load entropy ([report-walkthrough]
 * section 3.3: a complementary per-sequence balance loss with a very small
 * coefficient; aux_loss_alpha 0.001 in [repro-guide] section 3).  For each
 * sequence q of seq_len tokens (T % seq_len == 0):
 *   f_i = (#slots of the sequence routed to i) / (seq_len * K)
 *   P_i = mean over the sequence's tokens of scores[t, i]
 *   seq_loss[q] = alpha * sum_i f_i * P_i                    float64 [T/seq_len]
 *   *entropy = -sum_i p_i ln p_i, p_i = expert_load[i] / sum(expert_load)
 * Sums are float64 in a fixed order (deterministic).  seq_loss or entropy may
 * be NULL to skip that output.
 *   scores fp32 [T, E] (moe_route's affinities), topk_idx int32 [T, K],
 *   expert_load int32 [E] (moe_permute's load).                                */
int moe_balance_stats(const moe_dims *dims, const float *scores, const int32_t *topk_idx,
                      const int32_t *expert_load, int32_t seq_len, double alpha, double *seq_loss,
                      double *entropy, void *stream);

/* Auxiliary-loss-free bias update ([report-walkthrough] section 3.2; rate
 * expert_bias_update_rate 0.001 in [repro-guide] section 3):
 *   e_bias[e] += gamma * sign(T*K/E - expert_load[e]),  sign(0) = 0,
 * one fp32 addition per expert; the comparison is exact (T*K vs E*load).   */
int moe_bias_update(int32_t E, int64_t T, int32_t K, float gamma, const int32_t *expert_load,
                    float *e_bias, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
