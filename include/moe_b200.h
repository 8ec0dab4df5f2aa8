/*
 * moe_b200.h — C ABI of the single-GPU MoE FFN layer hot path for B200 (sm_100a):
 *
 *   route (router projection + softmax top-K)
 *   -> dispatch (per-expert histogram, prefix scan, capacity drop, scatter into an
 *      expert-contiguous buffer and a per-EP-rank packed buffer)
 *   -> expert GEMMs (ragged grouped GEMM, SwiGLU experts, tcgen05 tensor cores)
 *   -> combine (weighted un-permute back to token order)
 *
 * The dataflow is the one of "MoE 专家并行的 All-to-All 通信瓶颈：专家越多推理延迟为何
 * 反而上升", §All-to-All 分发与回收的机制 (its flowchart: route Top-K, pack by
 * destination card, exchange, group by expert, grouped GEMM, pack by source, exchange,
 * weighted merge into the original token order), with the two exchanges replaced by an
 * emulation of W virtual expert-parallel ranks inside one GPU's memory.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller, except where a comment
 *    says HOST. bf16 arrays are passed as uint16_t bit patterns. Row-major layouts.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream). The library never allocates or frees device memory; scratch comes from a
 *    caller workspace of at least the size the matching *_workspace_size function returns.
 *  - Argument errors are detected on the host and returned before anything is launched.
 *    Errors found by kernels (non-finite logits, out-of-range expert ids, a bounded wait
 *    that ran out) are recorded in a sticky per-device error word that
 *    moe_get_device_error() reads. No call throws; none synchronises unless it says so.
 *  - Pointers to bf16 or fp32 arrays must be 16-byte aligned (MOE_ERR_MISALIGNED).
 *
 * Notation (kept from the pages): N tokens, d hidden size, f expert FFN width, E experts,
 * K experts per token, W virtual EP ranks, cf capacity factor, C = ceil(cf*N*K/E) the
 * per-expert capacity, R the number of kept (token, slot) assignments (rows).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *moe_stream_t; /* identical to cudaStream_t */

#define MOE_ABI_VERSION 3

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,         /* null pointer, K > E, E % W != 0, N % W != 0, ... */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* a size outside the limits listed at moe_shape_t */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace_size() value */
    MOE_ERR_MISALIGNED = 4,          /* a pointer not 16-byte aligned */
    MOE_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 6,      /* a bounded device-side wait gave up */
    MOE_ERR_NONFINITE = 7,           /* a router logit was NaN or infinite */
    MOE_ERR_DEVICE_BOUNDS = 8,       /* an expert id outside [0, E) reached a kernel */
    MOE_ERR_F16_RANGE = 9            /* a value of h (or of a weight converted to fp16) beyond
                                        fp16's largest finite value 65504, or not finite */
} moe_status_t;

/* Problem description. Limits: 0 <= N, N*K < 2^31; d % 8 == 0 (d % 128 == 0 for
 * moe_expert_gemm / moe_layer); f % 128 == 0 for the GEMMs; 1 <= E <= 256;
 * 1 <= K <= min(E, 32); 1 <= W <= 64, E % W == 0, N % W == 0.
 * capacity_factor <= 0 selects dropless routing.
 * N = 0 (an empty batch) is valid everywhere: nothing is launched, the token-indexed
 * arguments may be NULL, and the outputs indexed by expert or rank (counts, kept, offsets,
 * rank_matrix, packed_offsets, stats) are set to zero. */
typedef struct moe_shape {
    int32_t N, d, f, E, K, W;
    float capacity_factor;
    uint32_t flags; /* MOE_FLAG_* bits below; other bits must be 0 */
} moe_shape_t;

/* moe_combine / moe_layer write `out` as bf16 (one rounding of the fp32 sum) instead of the
 * default fp32. Meant for a stack of layers whose next input is bf16. */
#define MOE_FLAG_OUT_BF16 1u

/* Which assignments claim an expert's capacity first ("MoE 推理服务工程真相 2026", §2.2:
 * assignments beyond the capacity are dropped; the page leaves the order open).
 * Default (flag clear): token-major, assignment a = t*K + k in increasing a, so an earlier
 * token's second choice beats a later token's first choice. With MOE_FLAG_SLOT_MAJOR:
 * slot-major, every token's slot 0 (tokens ascending), then every token's slot 1, ..., so
 * first choices are served before any second choice. Positions, row_of, the expert-sorted
 * rows and the packed buffer follow the chosen order (inside a packed block (i, j): expert
 * by expert, each expert's rows in their expert-sorted order). Slot-major dispatch scans
 * K times as many blocks. */
#define MOE_FLAG_SLOT_MAJOR 2u

/* Re-route overflowed assignments instead of dropping them ("MoE 推理服务工程真相 2026",
 * §4.3, token drop: move the excess to the next-best expert; §2.3, the remapping of the
 * overflow mask). Reading, one round: an expert is full when the assignments routed to it
 * number at least C. Every assignment past capacity moves to its token's best-ranked expert
 * (larger logit first, ties to the lower index) that the token did not route to, that is not
 * full, and that no earlier overflowed slot of the same token (in k order) took; if there is
 * none it is dropped. The moved assignments then queue at their new experts behind all the
 * routed assignments there, in the same priority order (token- or slot-major), and the ones
 * still past C are dropped. A moved assignment keeps its gate weight. The candidates are
 * ranked by the router logits, so the flag is taken by moe_layer, moe_layer_shared and
 * moe_dispatch_reroute, and refused (MOE_ERR_INVALID_ARG) by moe_dispatch and
 * moe_dispatch_static. The dispatch then runs two passes plus a ranking kernel. */
#define MOE_FLAG_REROUTE 4u

/* FP8 return payload ("MoE 推理服务工程真相 2026", §6.3: the exchange's token data in FP8,
 * here the expert outputs y that travel back to the tokens' ranks). With this flag the `y`
 * buffer of moe_expert_down, moe_expert_down_fp8, moe_expert_gemm and moe_combine (and the
 * layer's internal y) holds, per row, d e4m3 codes, then one exponent byte per 32 columns,
 * zero-padded to a multiple of 16 bytes: row stride d + roundup16(d / 32) bytes,
 * moe_y_bytes(shape) bytes in all. Block b of row r (columns [32b, 32b + 32)) with exponent
 * byte j + 127 holds the values code * 2^j, where j is the smallest power of two with
 * max|block| * 2^-j <= 448 (j in [-126, 127]; 0 for a zero or non-finite block) and each code
 * is the value * 2^-j rounded to nearest-even e4m3, saturating: the dispatch payload's rule
 * with a 32-column block in place of a row (a row of y spans several GEMM tiles, a block
 * does not). The values quantised are the fp32 y the plain down GEMM writes; the combine
 * decodes them exactly and accumulates in fp32 as before. Needs d % 128 == 0. */
#define MOE_FLAG_FP8_RETURN 8u

/* Precision of the SwiGLU activation h, the down projection's tensor-core operand.
 * Default (flag clear): h is stored as fp16 and the down projection reads fp16 weights (W2 of
 * moe_expert_down / moe_expert_gemm / moe_layer / moe_layer_shared, Ws2 of moe_shared_expert
 * and moe_layer_shared), converted once from the bf16 weights by moe_convert_bf16_to_f16. One
 * tensor-core MMA takes A and B of one type, so h and W2 share it. Why fp16: h is rounded once
 * (after fp32 accumulation and the SwiGLU in fp32) and that rounding is the largest error of the
 * layer; fp16 keeps 11 significant bits, bf16 8, so the error is 8 times smaller (on the
 * 128-expert layer with drops, max |error| / RMS(output) 0.0045 instead of 0.031; the bound
 * asked of the layer is 0.02). fp16's range is handled exactly: the gate/up GEMM records the
 * largest |h|, and only when it exceeds 65504 a second gate/up pass (launched every time, it
 * does nothing otherwise) stores h * 2^-k instead, k the smallest exponent that brings it into
 * range, and the down GEMM multiplies its accumulators by 2^k (powers of two: no rounding). The
 * record travels in the first 4 bytes of h's last row (row rows_alloc - 1, never a kept row), so
 * moe_expert_down must get the h buffer moe_expert_up wrote (a caller that fills h by other
 * means sets those 4 bytes to 0). A non-finite activation sets MOE_ERR_F16_RANGE.
 * With MOE_FLAG_H_BF16: h is bf16 and W2 / Ws2 are the bf16 weights themselves.
 * The FP8 path (moe_expert_up_fp8, moe_layer_fp8) keeps its bf16 h before the e4m3
 * quantisation and ignores this flag. */
#define MOE_FLAG_H_BF16 16u

/* fp16 return payload: the expert outputs y as fp16 codes with one power-of-two exponent per
 * 32 columns, half the bytes of fp32 y between the down projection and the combine. With this
 * flag the `y` buffer of moe_expert_down, moe_expert_down_fp8, moe_expert_gemm and moe_combine
 * (and the layer's internal y) holds, per row, d fp16 codes (2d bytes), then one exponent byte
 * j + 127 per 32 columns, zero-padded to a multiple of 16 bytes: row stride 2d + roundup16(d/32)
 * bytes, moe_y_bytes(shape) in all. Block b of row r (columns [32b, 32b + 32)) holds the values
 * code * 2^j, where j is the smallest power of two with max|block| * 2^-j <= 65504 (fp16's
 * largest finite value; j in [-126, 127]; 0 for a zero or non-finite block) and each code is the
 * value * 2^-j rounded to nearest-even fp16: the FP8 payload's block rule with fp16 codes. Every
 * block is in range whatever the magnitudes, and each value keeps fp16's 11 significant bits
 * relative to its block's top binade. The values quantised are the fp32 y the plain down GEMM
 * writes; the combine decodes them exactly and accumulates in fp32. Needs d % 128 == 0; not
 * with MOE_FLAG_FP8_RETURN. */
#define MOE_FLAG_Y_F16 32u

/* Per-call dispatch counters, written (not accumulated) by moe_dispatch / moe_layer into
 * DEVICE memory when a non-null pointer is given. Observability signals of
 * "MoE 专家并行的 All-to-All 通信瓶颈", §可观测指标与故障定位, and
 * "MoE 推理服务工程真相 2026", §5.1 (token_drop_count, overflow). */
typedef struct moe_stats {
    int64_t rows;             /* R = kept assignments */
    int64_t dropped;          /* N*K - R (assignments over capacity) */
    int64_t cross_rows;       /* kept rows whose expert rank differs from the token's home rank */
    int64_t dedup_pairs;      /* distinct (token, destination rank != home) pairs over kept rows:
                                 what an exchange that sends a token once per rank would carry */
    int64_t nonfinite_tokens; /* tokens with a non-finite logit (moe_layer only; else 0) */
    int32_t capacity;         /* C (N*K when dropless) */
    int32_t active_experts;   /* experts with at least one kept row */
    int32_t max_kept;         /* max_e kept[e] */
    int32_t min_kept;         /* min_e kept[e] */
    int64_t rerouted;         /* rows held by an expert the token did not route to (moved there
                                 by MOE_FLAG_REROUTE); 0 without re-routing */
} moe_stats_t;

/* Host-side report derived from moe_stats_t, the traffic matrix D and kept[]. */
typedef struct moe_report {
    double drop_rate;                 /* dropped / (N*K) */
    double send_max_over_min;         /* per-rank send (row sums of D): max / min (inf if min 0) */
    double recv_max_over_min;         /* per-rank receive (column sums of D): max / min */
    double cross_rank_fraction;       /* cross_rows / rows */
    double load_std_over_mean;        /* population std / mean of per-rank receive */
    double capacity_factor_effective; /* max_e kept[e] / (N*K/E) */
    int64_t tau_min_tokens;           /* max(max off-diagonal row sum, max column sum) of D */
    int64_t dispatch_bytes;           /* rows * d * 2 (bf16 payload of one dispatch) */
    int64_t send_max, send_min, recv_max, recv_min;
} moe_report_t;

/* ---------------------------------------------------------------- sizes */

/* Capacity C = ceil(cf * N * K / E) computed in double; N*K when dropless. Returns -1 on a
 * null shape. [MoE 推理服务工程真相 2026, §2.2 Expert Capacity Factor] */
int64_t moe_capacity(const moe_shape_t *shape);

/* Rows to allocate for every row-indexed buffer (assign_of_row, x_sorted, x_packed, h, y):
 * min(N*K, E*C) + 128. The 128 spare rows let the GEMM read whole 128-row tiles past the
 * last expert. Returns -1 on an invalid shape. */
int64_t moe_rows_alloc(const moe_shape_t *shape);

/* Workspace bytes for moe_route (the router's scratch: the logits when logits == NULL, and the
 * router weights transposed, [d][E rounded up to 64, 128 or 256] fp32, when N >= 2048 and
 * E > 32) and moe_dispatch (block histograms, pack bases). 0 on an invalid shape. */
size_t moe_workspace_size(const moe_shape_t *shape);

/* Workspace bytes for moe_layer: every intermediate of the layer plus the scratch above. */
size_t moe_layer_workspace_size(const moe_shape_t *shape);

/* Bytes of the y buffer of moe_expert_down / moe_expert_gemm / moe_combine: rows_alloc * d * 4
 * (fp32 y), rows_alloc * (d + roundup16(d / 32)) with MOE_FLAG_FP8_RETURN, or
 * rows_alloc * (2d + roundup16(d / 32)) with MOE_FLAG_Y_F16. 0 on an invalid shape. */
size_t moe_y_bytes(const moe_shape_t *shape);

/* ---------------------------------------------------------------- stages */

/* Router projection and softmax top-K.
 * [MoE Inference Communication, §DeepSpeed-MoE › MoE 计算核优化: gate top-k fused in one
 *  kernel; §Aurora, gate term G_i of the per-layer time model]
 * x [N][d] bf16; w_router [E][d] fp32; bias [E] fp32 or NULL (added to every logit).
 * logits[t][e] = (sum over i ascending of one fp32 fused multiply-add x[t][i]*Wr[e][i],
 * starting from +0) + bias[e]: bit-identical to any IEEE implementation of that order.
 * topk_idx [N][K] int32: the K largest logits, larger first, equal logits to the lower
 * expert index. topk_w [N][K] fp32: softmax over the K selected logits.
 * logits [N][E] fp32 or NULL (then not returned; the workspace holds them only where the two
 * steps run as separate kernels: few tokens or E < 32). The workspace (moe_workspace_size
 * bytes, 16-byte aligned, device) is required when logits == NULL, and always when N >= 2048
 * and E > 32 (the transposed router weights); MOE_ERR_WORKSPACE_TOO_SMALL otherwise. A
 * non-finite logit sets MOE_ERR_NONFINITE in the device error word; that token's result is
 * unspecified. */
moe_status_t moe_route(const moe_shape_t *shape, const uint16_t *x, const float *w_router,
                       const float *bias, int32_t *topk_idx, float *topk_w, float *logits,
                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* Dispatch permutation.
 * [MoE 推理服务工程真相 2026, §2.3 moe_dispatch pseudo-code: bincount of expert ids,
 *  overflow beyond capacity; §2.2: overflow dropped; MoE Inference Communication,
 *  §MoE 计算核优化: cumsum + scatter through a dense mapping table;
 *  MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制: pack by destination]
 * Assignments a = t*K + k are taken in increasing a; an assignment is kept iff fewer than C
 * earlier assignments chose the same expert.
 *  counts [E]: assignments per expert; kept [E] = min(counts, C);
 *  offsets [E+1]: exclusive scan of kept (offsets[E] = R);
 *  row_of [N*K]: offsets[e] + position, or -1 when dropped;
 *  assign_of_row [rows_alloc]: inverse of row_of on its first R entries;
 *  x_sorted [rows_alloc][d] bf16: x_sorted[row_of[a]] = x[a / K] (rows of one expert in
 *  increasing token order);
 *  x_packed [rows_alloc][d] bf16 or NULL: the same rows in blocks (home rank i, expert
 *  rank j), blocks row-major, rows inside a block ordered by (expert, token); expert e is on
 *  rank e / (E/W), token t's home is t / (N/W);
 *  rank_matrix [W][W] int64 or NULL: D[i][j] = kept rows from home i to rank j;
 *  packed_offsets [W*W+1] int64 or NULL: exclusive scan of D (block starts in x_packed);
 *  stats: DEVICE moe_stats_t or NULL.
 * topk_idx entries outside [0, E) set MOE_ERR_DEVICE_BOUNDS and are treated as dropped. */
moe_status_t moe_dispatch(const moe_shape_t *shape, const uint16_t *x, const int32_t *topk_idx,
                          int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *row_of,
                          int32_t *assign_of_row, uint16_t *x_sorted, uint16_t *x_packed,
                          int64_t *rank_matrix, int64_t *packed_offsets, moe_stats_t *stats,
                          void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_dispatch with overflowed assignments re-routed (MOE_FLAG_REROUTE must be set in
 * shape->flags; see there for the rule). Extra arguments:
 *  logits    [N][E] fp32, DEVICE: the router logits the candidates are ranked by (as written
 *            by moe_route).
 *  expert_of [N*K] int32, DEVICE, nullable: the expert whose row each assignment uses, -1 if
 *            it was dropped (equal to topk_idx where it was not moved).
 * counts[e] stays the routed demand; kept, offsets, row_of, assign_of_row, the scatter, the
 * traffic matrix and the packed layout describe the rows after re-routing (a moved row is
 * packed by its new expert's rank). The workspace is moe_workspace_size(shape) with the flag
 * set. */
moe_status_t moe_dispatch_reroute(const moe_shape_t *shape, const uint16_t *x, const float *logits,
                                  const int32_t *topk_idx, int32_t *counts, int32_t *kept,
                                  int32_t *offsets, int32_t *row_of, int32_t *assign_of_row,
                                  int32_t *expert_of, uint16_t *x_sorted, uint16_t *x_packed,
                                  int64_t *rank_matrix, int64_t *packed_offsets,
                                  moe_stats_t *stats, void *ws, size_t ws_bytes,
                                  moe_stream_t stream);

/* ---- W real ranks, one process per GPU (the exchange the one-GPU path emulates).
 * [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制: route Top-K, pack by
 *  destination card, all-to-all, group by expert, grouped GEMM, pack by source, all-to-all,
 *  weighted merge into the original token order]
 * Rank r holds the tokens of home shard r (tokens [r N/W, (r+1) N/W)) and experts
 * [r E/W, (r+1) E/W). After routing its own tokens (moe_route), every rank gathers every rank's
 * topk_idx [N][K] and runs the whole batch's bookkeeping (cheap integer work over N*K), so the
 * W ranks keep exactly the assignments one dispatch of the whole batch keeps (the capacity is
 * per expert over all ranks' tokens, in the same priority order). */

/* Rank `rank`'s dispatch. shape: the whole batch (N tokens over W ranks; MOE_FLAG_SLOT_MAJOR
 * allowed, MOE_FLAG_REROUTE refused: its candidates are ranked by every token's logits).
 * x_local [N/W][d] bf16: this rank's tokens. topk_idx_all [N][K]: every rank's routing.
 * Outputs of the whole batch, the same on every rank: counts, kept, offsets, row_of,
 * assign_of_row (as moe_dispatch), packed_row_of [N*K] (each kept assignment's row in the
 * whole batch's packed layout, -1 if dropped), rank_matrix D [W][W] and packed_offsets
 * [W*W+1] (required: the exchange's split sizes are D's row and column of this rank).
 * Outputs of this rank: x_send [rows_alloc][d] bf16, the rows it sends, blocks (rank, j) for
 * j = 0 .. W-1 (D[rank][j] rows each, rows inside a block by (expert, token)); send_row_of
 * [N/W * K]: per slot of this rank's tokens, its row in x_send (and so in the buffer the
 * return exchange brings back), -1 if dropped: the row_of of moe_combine after the return.
 * Workspace: moe_workspace_size(shape). */
moe_status_t moe_dispatch_rank(const moe_shape_t *shape, int32_t rank, const uint16_t *x_local,
                               const int32_t *topk_idx_all, int32_t *counts, int32_t *kept,
                               int32_t *offsets, int32_t *row_of, int32_t *assign_of_row,
                               int32_t *packed_row_of, int32_t *send_row_of, uint16_t *x_send,
                               int64_t *rank_matrix, int64_t *packed_offsets, moe_stats_t *stats,
                               void *ws, size_t ws_bytes, moe_stream_t stream);

/* Rank `rank`'s rows between the exchange's order and its experts' order. The received
 * buffer holds the blocks (i, rank) of i = 0 .. W-1 one after another (D[i][rank] rows each,
 * as moe_dispatch_rank of rank i sent them); the sorted buffer holds this rank's experts' kept
 * rows in the whole batch's expert-sorted order (rows offsets[r E/W] .. offsets[(r+1) E/W] - 1 of
 * the one-GPU layout, shifted to 0). direction 0: src = received rows, dst = sorted rows (the
 * way to the experts); direction 1: src = sorted rows, dst = rows in the received order (the
 * way back, before the return exchange). row_bytes: bytes per row (a multiple of 16: d*2 for
 * bf16 x, d*4 for fp32 y, the FP8 return payload's stride). offsets_local [E/W + 1] (nullable):
 * this rank's experts' offsets into the sorted rows (the grouped GEMM's offsets). Inputs are
 * moe_dispatch_rank's outputs (DEVICE). */
moe_status_t moe_regroup_rows(const moe_shape_t *shape, int32_t rank, int32_t row_bytes,
                              int32_t direction, const void *src, void *dst,
                              const int32_t *assign_of_row, const int32_t *packed_row_of,
                              const int32_t *offsets, const int64_t *packed_offsets,
                              int32_t *offsets_local, moe_stream_t stream);

/* Size of the library's fixed device scratch array used by moe_dispatch_static. */
#define MOE_STATIC_SCRATCH_BYTES (1u << 20)

/* moe_dispatch for callers that cannot allocate device memory. The pages have no counterpart:
 * this is an interface convenience, not a step of the method.
 * Some callers cannot hand the library a workspace: a plugin whose host owns every device
 * allocation and grants none to plugins, a process whose device-memory budget is fixed when it
 * starts, or a latency-critical loop where a cudaMalloc (which can synchronise the device) is
 * not acceptable. This entry point takes the same arguments and writes the same outputs as
 * moe_dispatch, but its scratch (block histograms, pack bases, and the traffic matrix and pack
 * offsets when those are NULL) lives in one static device array of MOE_STATIC_SCRATCH_BYTES
 * inside the library. Every GPU that loads the library holds that array until the process
 * exits. The call allocates and frees nothing.
 *  - Shapes whose scratch does not fit (about 8 * E * B + 8 * E * W + 16 * W * W bytes with
 *    B = W * ceil(N / (64 W)) token blocks, the first two terms K times larger with
 *    MOE_FLAG_SLOT_MAJOR) return MOE_ERR_WORKSPACE_TOO_SMALL before any launch.
 *    MOE_FLAG_REROUTE is refused.
 *  - The first call on a device looks up the array's device address on that device (the
 *    device must be current); make that first call before any stream capture. The address is
 *    kept per device and per CUDA context: after cudaDeviceReset (which destroys the context
 *    and the array with it) the next call looks it up again, so that call, too, must come
 *    before any stream capture.
 *  - All calls share the one array, and it keeps the last call's contents; each call clears
 *    the control words it needs (one cudaMemsetAsync on `stream`, which allocates nothing) and
 *    writes every other scratch byte before reading it. Two calls that overlap on the GPU
 *    (other streams, other host threads) race on the array: serialise them. */
moe_status_t moe_dispatch_static(const moe_shape_t *shape, const uint16_t *x,
                                 const int32_t *topk_idx, int32_t *counts, int32_t *kept,
                                 int32_t *offsets, int32_t *row_of, int32_t *assign_of_row,
                                 uint16_t *x_sorted, uint16_t *x_packed, int64_t *rank_matrix,
                                 int64_t *packed_offsets, moe_stats_t *stats,
                                 moe_stream_t stream);

/* Ragged grouped GEMM of the SwiGLU experts, one persistent launch per GEMM.
 * [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制 (grouped GEMM over
 *  variable per-expert token counts) and §容量因子、专家复制与 dropless 的取舍 (dropless
 *  grouped GEMM in a single call)]
 * For every expert e and every row r in [offsets[e], offsets[e+1]):
 *   h[r] = silu(x_sorted[r] W1[e]^T) * (x_sorted[r] W3[e]^T)   (fp16 out, fp32 accumulate)
 *   y[r] = h[r] W2[e]^T                                         (fp32 out, fp32 accumulate)
 * x_sorted [rows_alloc][d], w1, w3 [E][f][d] bf16; w2 [E][d][f] and h [rows_alloc][f] fp16
 * (both bf16 with MOE_FLAG_H_BF16; see there); y [rows_alloc][d] fp32 (the FP8 return payload
 * with MOE_FLAG_FP8_RETURN, moe_y_bytes); offsets [E+1] device int32 (as written by
 * moe_dispatch). h is rounded once because it is the second GEMM's tensor-core operand; y
 * stays fp32 so the combine adds unrounded expert outputs (unless the flag asks for the FP8
 * payload).
 * Rows past offsets[E] are neither read for output nor written. Experts with no rows cost
 * nothing (their weights are not read). Needs d % 128 == 0, f % 128 == 0. */
moe_status_t moe_expert_gemm(const moe_shape_t *shape, const uint16_t *x_sorted,
                             const int32_t *offsets, const uint16_t *w1, const uint16_t *w3,
                             const uint16_t *w2, uint16_t *h, void *y, moe_stream_t stream);

/* The two halves of moe_expert_gemm as separate launches (same contracts as above):
 * moe_expert_up:   h = silu(x_sorted W1^T) * (x_sorted W3^T)   (gate/up GEMM, fp16 h)
 * moe_expert_down: y = h W2^T                     (down GEMM, fp32 y or the FP8 payload) */
moe_status_t moe_expert_up(const moe_shape_t *shape, const uint16_t *x_sorted,
                           const int32_t *offsets, const uint16_t *w1, const uint16_t *w3,
                           uint16_t *h, moe_stream_t stream);
moe_status_t moe_expert_down(const moe_shape_t *shape, const uint16_t *h, const int32_t *offsets,
                             const uint16_t *w2, void *y, moe_stream_t stream);

/* bf16 -> fp16 copy of a weight array for the down projection (W2 [E][d][f], Ws2 [d][f_shared]),
 * made once when the weights are loaded. src, dst: DEVICE, n elements each, 16-byte aligned,
 * n % 8 == 0; dst may not overlap src. Each value is converted to the nearest fp16 (ties to
 * even): exact for magnitudes in [2^-17, 65504] (all but ~0.03 % of N(0, 0.02) weights, the
 * rest move by less than 2^-25); a magnitude above 65504 becomes infinite and sets
 * MOE_ERR_F16_RANGE. changed (DEVICE int64, nullable): the number of elements whose value
 * changed is ADDED to it. Not a step of the pages' method: a storage format of the weights. */
moe_status_t moe_convert_bf16_to_f16(const uint16_t *src, int64_t n, uint16_t *dst,
                                     int64_t *changed, moe_stream_t stream);

/* ---- FP8 payload ("MoE 推理服务工程真相 2026", §6.3: send the token data of the all-to-all
 * as FP8 instead of BF16, half the bytes, at the cost of quantisation noise).
 * Format e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448, no
 * infinities). Readings: one power-of-two scale per row, the smallest 2^j (j in [-126, 127])
 * with max|row| * 2^-j <= 448 (j = 0 for a zero or non-finite row); each element is
 * x * 2^-j rounded to nearest-even e4m3, saturating; value = code * 2^j. Routing stays on
 * the bf16 x; the experts' gate/up projections consume the e4m3 rows of x together with
 * e4m3 rows of W1 and W3 (one scale per output channel) on tcgen05 kind::f8f6f4; h is
 * written as bf16, its kept rows are then quantised to e4m3 the same way (one scale per
 * row), and the down projection runs on them and on e4m3 rows of W2 (one scale per output
 * channel); y and the combine stay fp32 unless MOE_FLAG_FP8_RETURN is set. */

/* Row-wise e4m3 quantisation of a bf16 matrix src [rows][cols] (DEVICE): codes [rows][cols]
 * uint8 and scale [rows] fp32 (DEVICE, caller-owned). For the experts' W1, W3 pass rows = E*f,
 * cols = d; for W2 rows = E*d, cols = f; for the activations h of the FP8 down projection
 * rows = rows_alloc, cols = f and rows_dev = offsets + E (nullable, DEVICE int32: only the
 * first min(rows, *rows_dev) rows are quantised, a count known only on the device).
 * cols % 16 == 0; src, codes 16-byte aligned. */
moe_status_t moe_quantize_rows_e4m3(const uint16_t *src, int64_t rows, int32_t cols,
                                    uint8_t *codes, float *scale, const int32_t *rows_dev,
                                    moe_stream_t stream);

/* moe_dispatch with the FP8 payload: x_sorted and x_packed hold e4m3 rows ([rows_alloc][d]
 * uint8) and sorted_scale / packed_scale [rows_alloc] fp32 the scale of each row (packed_scale
 * is required with x_packed and ignored without it). The bookkeeping outputs are identical to
 * moe_dispatch's. d % 16 == 0. MOE_FLAG_REROUTE is refused (no logits here; moe_layer_fp8
 * takes it). Same workspace as moe_dispatch. */
moe_status_t moe_dispatch_fp8(const moe_shape_t *shape, const uint16_t *x, const int32_t *topk_idx,
                              int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *row_of,
                              int32_t *assign_of_row, uint8_t *x_sorted, float *sorted_scale,
                              uint8_t *x_packed, float *packed_scale, int64_t *rank_matrix,
                              int64_t *packed_offsets, moe_stats_t *stats, void *ws,
                              size_t ws_bytes, moe_stream_t stream);

/* Gate/up GEMM on the FP8 payload: h = silu(sx * s1 * (xq W1q^T)) * (sx * s3 * (xq W3q^T)),
 * bf16 h [rows_alloc][f]; x_sorted e4m3 [rows_alloc][d] with sorted_scale per row (from
 * moe_dispatch_fp8); w1q, w3q e4m3 [E][f][d] with w1_scale, w3_scale [E][f] (from
 * moe_quantize_rows_e4m3; 16-byte aligned). d % 128 == 0, f % 128 == 0. */
moe_status_t moe_expert_up_fp8(const moe_shape_t *shape, const uint8_t *x_sorted,
                               const float *sorted_scale, const int32_t *offsets,
                               const uint8_t *w1q, const float *w1_scale, const uint8_t *w3q,
                               const float *w3_scale, uint16_t *h, moe_stream_t stream);

/* Down projection on e4m3 rows: y = sh * s2 * (hq W2q^T), fp32 y [rows_alloc][d] (or the FP8
 * return payload with MOE_FLAG_FP8_RETURN); hq e4m3
 * [rows_alloc][f] with h_scale per row (moe_quantize_rows_e4m3 of the bf16 h, rows =
 * offsets[E]); w2q e4m3 [E][d][f] with w2_scale [E][d] (16-byte aligned). d % 128 == 0,
 * f % 128 == 0. */
moe_status_t moe_expert_down_fp8(const moe_shape_t *shape, const uint8_t *hq, const float *h_scale,
                                 const int32_t *offsets, const uint8_t *w2q, const float *w2_scale,
                                 void *y, moe_stream_t stream);

/* Weighted combine back to token order.
 * [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制 (weighted merge into the
 *  original token order, then on to the next layer); MoE 推理服务工程真相 2026, §2.2 (a
 *  dropped slot contributes 0)]
 * out[t] = (sum over k = 0..K-1 with row_of[t*K+k] >= 0 of topk_w[t][k] * y[row])
 *          + shared_y[t] + residual[t], accumulated in fp32 in k order, then the shared dense
 * MLP's output (nullable, fp32 [N][d], see moe_shared_expert), then the residual (nullable,
 * bf16 [N][d]). y [rows_alloc][d] fp32, or the FP8 return payload with MOE_FLAG_FP8_RETURN
 * (each value decoded exactly before it is accumulated). out [N][d] is fp32, or bf16
 * (rounded once) when shape->flags has MOE_FLAG_OUT_BF16; a bf16 out may alias residual. */
moe_status_t moe_combine(const moe_shape_t *shape, const void *y, const int32_t *row_of,
                         const float *topk_w, const float *shared_y, const uint16_t *residual,
                         void *out, moe_stream_t stream);

/* The shared dense MLP of a Residual-MoE layer, for every token, on the same tcgen05 grouped GEMM
 * (one "expert" that owns all N rows of x).
 * [MoE Inference Communication, §DeepSpeed-MoE › PR-MoE, 现象二 / Residual: a dense MLP every
 *  token passes through, added to the output of the routed expert(s)]
 * Same SwiGLU form as the experts: h_s = silu(x Ws1^T) * (x Ws3^T), y_s = h_s Ws2^T (fp32).
 * x [N][d], ws1, ws3 [f_shared][d] bf16; ws2 [d][f_shared] and h_s [N][f_shared] fp16 (bf16
 * with MOE_FLAG_H_BF16); y_s [N][d] fp32. The fp16 range record of h_s lives in ws.
 * f_shared % 128 == 0. ws: at least 256 bytes of device scratch. */
moe_status_t moe_shared_expert(const moe_shape_t *shape, int32_t f_shared, const uint16_t *x,
                               const uint16_t *ws1, const uint16_t *ws3, const uint16_t *ws2,
                               uint16_t *h_s, float *y_s, void *ws, size_t ws_bytes,
                               moe_stream_t stream);

/* Residual-MoE layer: moe_layer's routed path plus the shared dense MLP, the two outputs
 * added in the combine (then the optional residual). Workspace: moe_layer_shared_workspace_size.
 * w2 and ws2 fp16 (bf16 with MOE_FLAG_H_BF16), the other weights bf16.
 * [MoE Inference Communication, §DeepSpeed-MoE › PR-MoE, Residual-MoE] */
size_t moe_layer_shared_workspace_size(const moe_shape_t *shape, int32_t f_shared);
moe_status_t moe_layer_shared(const moe_shape_t *shape, int32_t f_shared, const uint16_t *x,
                              const float *w_router, const float *bias, const uint16_t *w1,
                              const uint16_t *w3, const uint16_t *w2, const uint16_t *ws1,
                              const uint16_t *ws3, const uint16_t *ws2, const uint16_t *residual,
                              void *out, int32_t *topk_idx_out, moe_stats_t *stats, void *ws,
                              size_t ws_bytes, moe_stream_t stream);

/* The whole layer: moe_route -> moe_dispatch (with the packed buffer) -> moe_expert_gemm ->
 * moe_combine, every intermediate in the workspace (moe_layer_workspace_size bytes).
 * [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制: its flowchart (route
 *  Top-K, pack by destination, group by expert, grouped GEMM, weighted merge into the original
 *  token order), the two exchanges emulated for W ranks inside this GPU's memory]
 * w1, w3 bf16 [E][f][d]; w2 fp16 [E][d][f] (bf16 with MOE_FLAG_H_BF16).
 * residual (nullable) is added in the combine (pass x for x + MoE(x)); out [N][d] is fp32,
 * or bf16 with MOE_FLAG_OUT_BF16, and must not alias x. topk_idx_out [N][K] (nullable)
 * receives the routing; stats (nullable, DEVICE) the counters. */
moe_status_t moe_layer(const moe_shape_t *shape, const uint16_t *x, const float *w_router,
                       const float *bias, const uint16_t *w1, const uint16_t *w3,
                       const uint16_t *w2, const uint16_t *residual, void *out,
                       int32_t *topk_idx_out, moe_stats_t *stats, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_layer with the FP8 payload and FP8 expert GEMMs: the dispatch writes e4m3 rows, the
 * gate/up GEMM runs on them with the e4m3 weights w1q, w3q [E][f][d] (scales w1_scale,
 * w3_scale [E][f]), h's kept rows are quantised to e4m3 and the down GEMM runs on them with
 * w2q [E][d][f] (scales w2_scale [E][d]); all weights from moe_quantize_rows_e4m3. Every
 * flag of moe_layer applies; the workspace is moe_layer_workspace_size(shape). */
moe_status_t moe_layer_fp8(const moe_shape_t *shape, const uint16_t *x, const float *w_router,
                           const float *bias, const uint8_t *w1q, const float *w1_scale,
                           const uint8_t *w3q, const float *w3_scale, const uint8_t *w2q,
                           const float *w2_scale, const uint16_t *residual, void *out,
                           int32_t *topk_idx_out, moe_stats_t *stats, void *ws, size_t ws_bytes,
                           moe_stream_t stream);

/* Inter-layer expert affinity counts, accumulated into counts [E][E] int64:
 * for every token t, i in topk_j[t], p in topk_j1[t]: counts[i][p] += 1.
 * P(E_p at layer j+1 | E_i at layer j) = counts[i][p] / (tokens with i in topk_j).
 * [MoE Inference Communication, §ExFlow 核心发现：跨层专家亲和性] */
moe_status_t moe_affinity_accumulate(int32_t N, int32_t E, int32_t K, const int32_t *topk_j,
                                     const int32_t *topk_j1, int64_t *counts,
                                     moe_stream_t stream);

/* ---------------------------------------------------------------- host-side helpers */

/* Derived observability report. HOST pointers: stats (a copy of the device struct),
 * rank_matrix [W][W], kept [E]. Pure host computation; needs no GPU.
 * [MoE 专家并行的 All-to-All 通信瓶颈, §可观测指标与故障定位; MoE 推理服务工程真相 2026,
 *  §5.1; MoE Inference Communication, §Aurora 定理 4.2 (tau_min = max row/column sum of
 *  the traffic matrix, here in tokens and without the local diagonal)] */
moe_status_t moe_derive_report(const moe_shape_t *shape, const moe_stats_t *stats,
                               const int64_t *rank_matrix, const int32_t *kept,
                               moe_report_t *out);

/* Receiver-contention-free transmission order of one exchange of the packed rows.
 * [MoE Inference Communication, §Aurora 场景 1: 定理 4.2 (the bound) and the scheduling rule
 *  that follows it (no receiver is fed by two senders at once)]
 * rank_matrix: HOST [W][W] int64, D[i][j] = rows rank i sends to rank j (moe_dispatch's
 *   rank_matrix); the diagonal stays on its rank and is not scheduled. Entries must be >= 0.
 * Output, HOST, caller-owned: phases s = 0 .. *n_phases - 1. During phase s, which lasts
 *   phase_len[s] rows (> 0), rank i sends to rank phase_dst[s*W + i], or nothing when that is
 *   -1; within a phase no receiver appears twice and no rank sends to itself. Summed over the
 *   phases, rank i sends D[i][j] rows to every j != i. *makespan = the sum of phase_len =
 *   max(max_i sum_{j!=i} D[i][j], max_j sum_{i!=j} D[i][j]) (tau_min of moe_derive_report):
 *   the order reaches the theorem's lower bound. Each phase is chosen so that its shortest
 *   transfer is as long as possible (few, long phases: an executor synchronises once per
 *   phase); phases with the same destinations follow each other only once merged. At most
 *   2*W*W phases (218 for a dense 64-rank matrix): max_phases >= 2*W*W always suffices;
 *   a smaller max_phases that the order does not fit returns MOE_ERR_INVALID_ARG.
 * phase_dst holds max_phases*W int32, phase_len max_phases int64. Pure host computation,
 * needs no GPU. Errors: null pointers, W outside [1, 64], a negative entry, max_phases < 0. */
moe_status_t moe_exchange_schedule(int32_t W, const int64_t *rank_matrix, int32_t max_phases,
                                   int32_t *phase_dst, int64_t *phase_len, int32_t *n_phases,
                                   int64_t *makespan);

/* Expert placement across GPUs from inter-layer expert affinity.
 * [MoE Inference Communication, §ExFlow 形式化：整数线性规划建模: minimise the token hops
 *  between consecutive layers whose experts sit on different GPUs, every GPU holding E/P
 *  experts of every layer and every expert on one GPU]
 * counts: HOST [L-1][E][E] int64, counts[j][i][p] = token hops from expert i of layer j to
 *   expert p of layer j+1 (moe_affinity_accumulate of layers j and j+1), entries >= 0.
 * gpu_of: HOST out [L][E] int32: the GPU (0 .. P-1) of expert e of layer l; each GPU gets
 *   exactly E/P experts per layer. Deploying it means storing layer l's experts GPU by GPU.
 * cost (nullable): sum over j, i, p of counts[j][i][p] where gpu_of[j][i] != gpu_of[j+1][p],
 *   for the returned placement; contiguous_cost (nullable): the same for the contiguous
 *   placement (expert e on GPU e / (E/P)), the default of moe_dispatch's rank emulation.
 * Method: a heuristic, not the pages' exact ILP. From `starts` initial placements (all layers
 *   contiguous; layer 0 contiguous, grouped by the similarity of its experts' affinity rows, or
 *   shuffled, with the later layers built one by one, each best given the one before; all
 *   layers shuffled), each layer in turn is re-placed optimally
 *   given its two neighbours (a transportation problem, solved exactly), forward and backward,
 *   until nothing improves (at most 64 sweeps); then, 4*L times, two pairs of experts of one layer
 *   are swapped and the descent repeated, keeping the result when it is cheaper. The cheapest
 *   placement over the starts is returned; start 0 makes it never worse than contiguous.
 *   Deterministic. Cost grows as starts * L^2 * E^2 * P (E = 64, L = 4, 16 starts: 0.05 s;
 *   E = 256: 0.5 s; 58 layers of 256 experts on 32 GPUs, one start: 20 s).
 * Errors: null counts (L > 1) or gpu_of; L < 1; E outside [1, 256]; P < 1 or E % P != 0;
 *   starts outside [1, 64]; a negative count. Pure host computation, needs no GPU. */
moe_status_t moe_place_experts(int32_t L, int32_t E, int32_t P, const int64_t *counts,
                               int32_t starts, int32_t *gpu_of, int64_t *cost,
                               int64_t *contiguous_cost);

/* Storage order that deploys a placement: gpu_of [L][E] (HOST, from moe_place_experts or
 * moe_place_experts_staged) -> order [L][E] (HOST, out): order[l][s] = the expert of layer l to
 * store at slot s, GPU by GPU and experts ascending within a GPU, so that slot s sits on GPU
 * s / (E / P), the contiguous rank layout of the dispatch. Permuting a layer's router rows and
 * expert weights by it deploys the placement. MOE_ERR_INVALID_ARG unless every GPU holds
 * exactly E / P experts of every layer. Pure host computation. */
moe_status_t moe_placement_order(int32_t L, int32_t E, int32_t P, const int32_t *gpu_of,
                                 int32_t *order);

/* Staged expert placement over nodes of GPUs.
 * [MoE Inference Communication, §ExFlow 形式化：整数线性规划建模, the staged expert affinity:
 *  first minimise the hops that cross nodes, then, inside each node, the hops that cross GPUs]
 * GPUs are numbered node by node (GPU g is on node g / gpus_per_node). Stage 1 places every
 * layer's experts on the nodes (E / nodes each) by the method of moe_place_experts; stage 2, for
 * each node, places that node's experts on its GPUs by the same method, on the affinity counts
 * restricted to the node's experts of consecutive layers. Each GPU gets E / (nodes *
 * gpus_per_node) experts per layer. Outputs (HOST): gpu_of [L][E]; node_hops / gpu_hops (nullable):
 * the hops between consecutive layers whose experts sit on different nodes / GPUs; and the same
 * two for the contiguous placement (expert e on GPU e / (E / (nodes * gpus_per_node))).
 * counts as for moe_place_experts. Errors: as moe_place_experts, with E % (nodes *
 * gpus_per_node) != 0. Pure host computation, needs no GPU. */
moe_status_t moe_place_experts_staged(int32_t L, int32_t E, int32_t nodes, int32_t gpus_per_node,
                                      const int64_t *counts, int32_t starts, int32_t *gpu_of,
                                      int64_t *node_hops, int64_t *gpu_hops,
                                      int64_t *contiguous_node_hops,
                                      int64_t *contiguous_gpu_hops);

/* Reads (and, if clear != 0, resets) the calling device's sticky error word. Synchronises
 * the device. Returns MOE_OK when no kernel has recorded an error. */
moe_status_t moe_get_device_error(int clear);

/* Copies the counters a dispatch or layer call wrote to DEVICE memory (stats_dev) into HOST
 * memory (out, caller-owned), in order on `stream`, and waits for that stream: the one call
 * here that synchronises on purpose, for observability outside the timed path. */
moe_status_t moe_read_stats(const moe_stats_t *stats_dev, moe_stats_t *out, moe_stream_t stream);

/* Launches one kernel whose only work is a bounded wait on a flag that nothing sets; it gives
 * up after timeout_ns nanoseconds and records MOE_ERR_DEVICE_TIMEOUT. Lets a test see the
 * bounded-wait path end with an error status while the context stays usable. */
moe_status_t moe_debug_bounded_wait(uint64_t timeout_ns, moe_stream_t stream);

/* Human-readable name of a status code. Never NULL. */
const char *moe_status_string(moe_status_t status);

/* MOE_ABI_VERSION of the built library. */
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
