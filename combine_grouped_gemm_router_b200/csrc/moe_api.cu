// C ABI of the MoE layer hot path (declarations and contracts: include/moe_b200.h).
// Host side: argument checks, workspace carving, tensor maps, launches.
#include <cudaTypedefs.h>
#include <math.h>

#include <functional>
#include <map>
#include <mutex>

#include "combine.cuh"
#include "common.cuh"
#include "dispatch.cuh"
#include "exchange_plan.cuh"
#include "grouped_gemm.cuh"
#include "route.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxE = 256;
constexpr int kMaxK = 32;
constexpr int kMaxW = 64;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s bound on any device-side wait
constexpr size_t kCbMaxSmem = 215040;  // the bulk-fed combine's shared memory, at most

inline size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

struct Geometry {
    int64_t C;           // capacity as used by the kernels (<= N*K)
    int64_t rows_alloc;  // min(N*K, E*C) + 128
    int S, bps, nblk;    // dispatch token blocks
    int slot_major;      // priority order of the positions
    int rounds;          // 2 when overflowed assignments are re-routed
    int nvb_round, nseg_round;  // virtual blocks and segments of one round
    int nvb, nseg;       // ... of all rounds
};

int64_t capacity_of(const moe_shape_t *s)
{
    const int64_t NK = (int64_t)s->N * s->K;
    if (!(s->capacity_factor > 0.0f))
        return NK;
    return (int64_t)ceil((double)s->capacity_factor * (double)s->N * (double)s->K / (double)s->E);
}

// Row stride in bytes of the y payload: d e4m3 codes (FP8 return) or 2d fp16 codes (fp16
// return), then d/32 exponent bytes padded to 16; 0 when y is fp32.
int y_payload_stride(const moe_shape_t *s)
{
    const int ex = (s->d / 32 + 15) & ~15;
    if (s->flags & MOE_FLAG_FP8_RETURN)
        return s->d + ex;
    if (s->flags & MOE_FLAG_Y_F16)
        return 2 * s->d + ex;
    return 0;
}

bool y_is_f16(const moe_shape_t *s) { return (s->flags & MOE_FLAG_Y_F16) != 0; }

moe_status_t check_shape(const moe_shape_t *s, bool gemm, Geometry *g)
{
    if (!s)
        return MOE_ERR_INVALID_ARG;
    if ((s->flags & ~(uint32_t)(MOE_FLAG_OUT_BF16 | MOE_FLAG_SLOT_MAJOR | MOE_FLAG_REROUTE |
                                MOE_FLAG_FP8_RETURN | MOE_FLAG_H_BF16 | MOE_FLAG_Y_F16)) != 0)
        return MOE_ERR_INVALID_ARG;
    if ((s->flags & MOE_FLAG_FP8_RETURN) && (s->flags & MOE_FLAG_Y_F16))
        return MOE_ERR_INVALID_ARG;
    if (s->N < 0 || s->d < 8 || s->E < 1 || s->K < 1 || s->W < 1 || s->f < 0)
        return MOE_ERR_INVALID_ARG;
    if (s->K > s->E || s->E % s->W != 0 || s->N % s->W != 0)
        return MOE_ERR_INVALID_ARG;
    if (s->E > kMaxE || s->K > kMaxK || s->W > kMaxW || s->d % 8 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)s->N * s->K >= (int64_t)1 << 31)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (gemm && (s->d % 128 != 0 || s->f < 128 || s->f % 128 != 0))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((s->flags & (MOE_FLAG_FP8_RETURN | MOE_FLAG_Y_F16)) && s->d % 128 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (g) {
        const int64_t NK = (int64_t)s->N * s->K;
        int64_t C = capacity_of(s);
        if (C > NK)
            C = NK;
        g->C = C;
        g->rows_alloc = (NK < (int64_t)s->E * C ? NK : (int64_t)s->E * C) + 128;
        g->S = s->N / s->W;
        g->bps = (g->S + kDispatchHB - 1) / kDispatchHB;
        g->nblk = s->W * g->bps;
        g->slot_major = (s->flags & MOE_FLAG_SLOT_MAJOR) ? 1 : 0;
        g->rounds = (s->flags & MOE_FLAG_REROUTE) ? 2 : 1;
        g->nvb_round = g->slot_major ? s->K * g->nblk : g->nblk;
        g->nseg_round = g->slot_major ? s->K * s->W : s->W;
        g->nvb = g->rounds * g->nvb_round;
        g->nseg = g->rounds * g->nseg_round;
    }
    return MOE_OK;
}

// Route/dispatch scratch, carved in this order from the workspace.
struct ScratchLayout {
    size_t logits, ctl, agg, incl, pk_base, moved, D, pk_off, pk_of, total;
};

constexpr size_t kNoScratch = ~(size_t)0;

// The dispatch's own scratch, from offset o: the pass's control words (ticket, finished
// blocks, one flag per virtual block), the blocks' histograms and inclusive prefixes
// [nvb][E], the pack bases [nseg][E], the moved-to expert of each assignment (re-routing),
// the traffic matrix and the pack offsets (when the caller does not want them), and (with_pk)
// each assignment's packed row for the one-kernel pass's copy by destination row.
template <typename Layout>
size_t dispatch_scratch(const moe_shape_t *s, const Geometry &g, size_t o, Layout &L,
                        bool with_pk = true)
{
    L.ctl = o;
    o = align_up(o + ((size_t)g.nvb + 2) * 4);
    L.agg = o;
    o = align_up(o + (size_t)s->E * g.nvb * 4);
    L.incl = o;
    o = align_up(o + (size_t)s->E * g.nvb * 4);
    L.pk_base = o;
    o = align_up(o + (size_t)s->E * g.nseg * 8);
    L.moved = o;
    if (g.rounds > 1)
        o = align_up(o + (size_t)s->N * s->K * 4);
    L.D = o;
    o = align_up(o + (size_t)s->W * s->W * 8);
    L.pk_off = o;
    o = align_up(o + ((size_t)s->W * s->W + 1) * 8);
    L.pk_of = with_pk ? o : kNoScratch;
    if (with_pk)
        o = align_up(o + (size_t)s->N * s->K * 4);
    return o;
}

// The router's one-kernel path: many tokens and E >= 32.
inline bool router_fused(const moe_shape_t *s) { return s->E >= 32 && s->N >= 2048; }

// Experts the split-warp router form covers (E rounded up to 64, 128 or 256), 0 where another
// form runs. That form reads the router weights transposed, [d][EC] fp32, from the scratch.
inline int router_split_ec(const moe_shape_t *s)
{
    if (!router_fused(s) || s->E <= 32)
        return 0;
    return s->E <= 64 ? 64 : s->E <= 128 ? 128 : 256;
}

ScratchLayout scratch_layout(const moe_shape_t *s, const Geometry &g)
{
    ScratchLayout L;
    size_t o = 0;
    // the router's scratch: the [N][E] logits of its two-kernel path, or the transposed
    // weights of the split-warp form
    L.logits = o;
    o = align_up(o + std::max((size_t)s->N * s->E, (size_t)router_split_ec(s) * s->d) * 4);
    L.total = dispatch_scratch(s, g, o, L);
    return L;
}

// moe_layer: every intermediate, after the scratch.
struct LayerLayout {
    size_t topk_idx, topk_w, counts, kept, offsets, row_of, assign, x_sorted, x_packed,
        sorted_scale, packed_scale, h, hq, h_scale, y, nonfinite, total;
};

LayerLayout layer_layout(const moe_shape_t *s, const Geometry &g, size_t base)
{
    LayerLayout L;
    const size_t NK = (size_t)s->N * s->K, RA = (size_t)g.rows_alloc;
    size_t o = align_up(base);
    L.topk_idx = o;
    o = align_up(o + NK * 4);
    L.topk_w = o;
    o = align_up(o + NK * 4);
    L.counts = o;
    o = align_up(o + (size_t)s->E * 4);
    L.kept = o;
    o = align_up(o + (size_t)s->E * 4);
    L.offsets = o;
    o = align_up(o + ((size_t)s->E + 1) * 4);
    L.row_of = o;
    o = align_up(o + NK * 4);
    L.assign = o;
    o = align_up(o + RA * 4);
    L.x_sorted = o;
    o = align_up(o + RA * s->d * 2);
    L.x_packed = o;
    o = align_up(o + RA * s->d * 2);
    L.sorted_scale = o;  // FP8 payload only
    o = align_up(o + RA * 4);
    L.packed_scale = o;
    o = align_up(o + RA * 4);
    L.h = o;
    o = align_up(o + RA * (size_t)s->f * 2);
    L.hq = o;  // FP8 path: e4m3 rows of h and their scales
    o = align_up(o + RA * (size_t)s->f);
    L.h_scale = o;
    o = align_up(o + RA * 4);
    L.y = o;
    o = align_up(o + RA * s->d * 4);
    L.nonfinite = o;
    o = align_up(o + 8);
    L.total = o;
    return L;
}

// Per-device, per-kernel one-time setup (function attributes belong to a device's context,
// so a process that drives several GPUs sets them on each). `init` runs once per
// (device, key) under a lock; its result is cached, as is the integer it returns in *value.
cudaError_t once_per_device(const void *key, const std::function<cudaError_t(int *)> &init,
                            int *value = nullptr)
{
    static std::recursive_mutex mu;  // an init may itself ask for a per-device value
    static std::map<std::pair<int, const void *>, std::pair<cudaError_t, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::recursive_mutex> lock(mu);
    auto it = done.find({dev, key});
    if (it == done.end()) {
        int v = 0;
        const cudaError_t e = init(&v);
        it = done.emplace(std::make_pair(dev, key), std::make_pair(e, v)).first;
    }
    if (value)
        *value = it->second.second;
    return it->second.first;
}

// Streaming multiprocessors of the current device (queried once per device).
int num_sms()
{
    static const char key = 0;
    int n = 0;
    const cudaError_t e = once_per_device(&key, [](int *v) {
        int dev = 0;
        cudaError_t r = cudaGetDevice(&dev);
        if (r == cudaSuccess)
            r = cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
        return r;
    }, &n);
    return (e == cudaSuccess && n > 0) ? n : 148;
}

template <typename Kernel>
cudaError_t smem_attr_once(Kernel kernel, int bytes)
{
    return once_per_device(reinterpret_cast<const void *>(kernel), [&](int *) {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    });
}

// Warp work items of the row kernels (combine, bf16 scatter): a whole token row each
// when there are enough tokens to fill the GPU, else slices of `slice` chunks, so that a
// decode batch of a few tokens still spreads over every SM.
int row_slice(int N, int nchunks, int slice)
{
    return N >= 8 * num_sms() ? nchunks : slice;
}

int row_blocks(int N, int nchunks, int seg)
{
    const int64_t items = (int64_t)N * ((nchunks + seg - 1) / seg);
    const int64_t blocks = (items + 7) / 8;
    return (int)(blocks < 64 * num_sms() ? blocks : 64 * num_sms());
}


inline moe_status_t launch_status()
{
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------- route

template <int TY, int TX, int TT, int TE, int KC, int S>
void launch_logits(const uint16_t *x, const float *wr, const float *bias, float *logits, int N,
                   int d, int E, cudaStream_t st)
{
    using L = LogitTile<TY, TX, TT, TE, KC, S>;
    smem_attr_once(router_logits_kernel<TY, TX, TT, TE, KC, S>, L::SMEM_BYTES);
    dim3 grid((N + L::BT - 1) / L::BT, (E + L::BE - 1) / L::BE);
    router_logits_kernel<TY, TX, TT, TE, KC, S>
        <<<grid, L::NT, L::SMEM_BYTES, st>>>(x, wr, bias, logits, N, d, E);
}

template <int TY, int TX, int TT, int TE, int KC, int S>
void launch_logits_pairs(const uint16_t *x, const float *wr, const float *bias, float *logits,
                         int N, int d, int E, cudaStream_t st)
{
    using L = LogitTile<TY, TX, TT, TE, KC, S>;
    smem_attr_once(router_logits_pairs_kernel<TY, TX, TT, TE, KC, S>, L::SMEM_BYTES);
    dim3 grid((N + L::BT - 1) / L::BT, (E + L::BE - 1) / L::BE);
    router_logits_pairs_kernel<TY, TX, TT, TE, KC, S>
        <<<grid, L::NT, L::SMEM_BYTES, st>>>(x, wr, bias, logits, N, d, E);
}

template <int NW, int TT>
void launch_router_topk(const moe_shape_t *s, const uint16_t *x, const float *wr, const float *bias,
                        int32_t *topk_idx, float *topk_w, float *logits,
                        unsigned long long *nonfinite, cudaStream_t st)
{
    using L = RouterTopkTile<NW, TT, 16>;
    smem_attr_once(router_topk_kernel<NW, TT, 16>, L::SMEM_BYTES);
    router_topk_kernel<NW, TT, 16><<<(s->N + L::TOK - 1) / L::TOK, L::NT, L::SMEM_BYTES, st>>>(
        x, wr, bias, s->N, s->d, s->E, s->K, topk_idx, topk_w, logits, nonfinite);
}

template <int NE, int TT, int KC, int ST>
void launch_router_split(const moe_shape_t *s, const uint16_t *x, const float *wt,
                         const float *bias, int32_t *topk_idx, float *topk_w, float *logits,
                         unsigned long long *nonfinite, cudaStream_t st)
{
    using L = RouterSplitTile<NE, TT, KC, ST>;
    smem_attr_once(router_split_kernel<NE, TT, KC, ST>, L::SMEM_BYTES);
    router_split_kernel<NE, TT, KC, ST><<<(s->N + kRsTok - 1) / kRsTok, L::NT, L::SMEM_BYTES, st>>>(
        x, wt, bias, s->N, s->d, s->E, s->K, topk_idx, topk_w, logits, nonfinite);
}

// The router projection and the top-K selection. logits_out (nullable) receives the [N][E]
// logits; scratch ([N][E] fp32) is used when the two steps run as separate kernels.
moe_status_t route_impl(const moe_shape_t *s, const uint16_t *x, const float *w_router,
                        const float *bias, int32_t *topk_idx, float *topk_w, float *logits_out,
                        float *scratch, unsigned long long *nonfinite, cudaStream_t st)
{
    const int N = s->N, d = s->d, E = s->E;
    // Many tokens and E >= 32: the projection and the selection in one kernel (64 tokens x
    // every expert per CTA; the logits reach HBM only when asked for). E > 32: the split-warp
    // form, on the router weights transposed into the scratch by one small kernel first.
    if (router_fused(s)) {
        if (const int EC = router_split_ec(s)) {
            if (!scratch)
                return MOE_ERR_WORKSPACE_TOO_SMALL;
            router_transpose_kernel<<<dim3((d + 31) / 32, EC / 32), 256, 0, st>>>(w_router, E, d,
                                                                                 EC, scratch);
#define MOE_RS(NE, TT, KC, ST)                                                                     \
    launch_router_split<NE, TT, KC, ST>(s, x, scratch, bias, topk_idx, topk_w, logits_out,         \
                                        nonfinite, st)
            // 4 tokens per lane, except E <= 64 with too few tokens for several CTAs per SM
            // (2 tokens per lane and twice the warps there); 64-element chunks except the stack
            // layer's shape (measured on the B200: N = 8192, d = 2048, E = 128: 152 -> 136 us
            // against the broadcast form; N = 32768, d = 4096, E = 64: 509 -> 477 us against
            // the register-tiled form; N = 8192, d = 2048, E = 256: 266 -> 237 us; N = 8192,
            // d = 2048, E = 64: 111 -> 85 us)
            const bool many = (long long)N >= 64LL * 3 * num_sms();
            if (EC == 64) {
                if (many)
                    MOE_RS(4, 4, 32, 3);
                else
                    MOE_RS(4, 2, 64, 3);
            } else if (EC == 128) {
                MOE_RS(8, 4, 64, 3);
            } else {
                MOE_RS(16, 4, 64, 2);
            }
#undef MOE_RS
            return launch_status();
        }
        launch_router_topk<2, 2>(s, x, w_router, bias, topk_idx, topk_w, logits_out, nonfinite,
                                 st);  // E == 32: the broadcast form
        return launch_status();
    }
    float *logits = logits_out ? logits_out : scratch;
    // Tile choice. Each output is one dependent chain of d fused multiply-adds, so
    // the floor is d x (fma latency). Few outputs (small N or small E): one chain per
    // thread and many warps per SM, so latency, not issue, is the limit. Many outputs
    // (E >= 32 with large N): the fp32 FMA pipe is the limit; a thread owns 4 tokens x
    // 8 experts so each bf16 -> fp32 conversion of x feeds 8 FMAs.
    const long long outputs = (long long)N * E;
    if (outputs < 148LL * 1024 || E <= 16) {
        if (N < 64)  // 16 tokens x 8 experts per CTA (decode, 16 x 256: 55 us, 72 with 2 x 32)
            launch_logits<16, 8, 1, 1, 64, 4>(x, w_router, bias, logits, N, d, E, st);
        else if (E <= 8)
            launch_logits<32, 8, 1, 1, 64, 4>(x, w_router, bias, logits, N, d, E, st);
        else
            launch_logits<16, 16, 1, 1, 64, 4>(x, w_router, bias, logits, N, d, E, st);
    } else if (E <= 32) {
        launch_logits<8, 16, 2, 2, 64, 4>(x, w_router, bias, logits, N, d, E, st);
    } else if (N >= 8192) {
        // 8 tokens x 8 experts per thread, tokens paired in packed FMAs (measured 3 % faster
        // at N = 8192, E = 128 and 15 % at N = 32768, E = 64, same bits)
        launch_logits_pairs<16, 8, 8, 8, 64, 2>(x, w_router, bias, logits, N, d, E, st);
    } else {
        launch_logits<16, 8, 4, 8, 64, 3>(x, w_router, bias, logits, N, d, E, st);
    }
    topk_softmax_kernel<<<(N + 7) / 8, 256, 0, st>>>(logits, N, E, s->K, topk_idx, topk_w,
                                                      nonfinite);
    return launch_status();
}

// ---------------------------------------------------------------- dispatch

// Row payload of the scatter: bf16 rows, or e4m3 rows with a scale per row.
struct Payload {
    void *x_sorted;
    void *x_packed;       // nullable
    bool e4m3;
    float *sorted_scale;  // e4m3 only
    float *packed_scale;  // e4m3 with x_packed only
};

// W real ranks: this process's rank and where its rows go (see PlaceArgs).
struct RankPack {
    int rank = -1;
    int x_row0 = 0;
    int32_t *packed_row_of = nullptr;
    int32_t *send_row_of = nullptr;
};

// The dispatch's scratch pointers (inside a workspace or the static array).
struct DispatchScratch {
    unsigned int *ctl;
    int32_t *agg, *incl;
    int64_t *pk_base;
    int32_t *moved;
    int32_t *pk_of;  // null: not available (the fused pass then copies by token block)
};

// Row pieces of a token block (an upper bound: the block's tokens times pieces per row).
int place_items(const moe_shape_t *s, const Geometry &g)
{
    const int tokens = g.S < kDispatchHB ? g.S : kDispatchHB;
    const int npc = (int)(((size_t)s->d * 2 + kPiece - 1) / kPiece);
    return tokens * npc;
}

// Parts per token block of the placement kernel. FP8 payload: token parts, enough CTAs for
// about eight per SM, at least one token per warp. bf16 rows (bulk copies of pieces): about
// four CTAs per SM, at least four pieces per part.
int place_parts(const moe_shape_t *s, const Geometry &g, bool e4m3)
{
    int want, cap;
    if (e4m3) {
        want = (8 * num_sms() + g.nblk - 1) / g.nblk;
        cap = (kDispatchHB + 7) / 8;
    } else {
        want = (4 * num_sms() + g.nblk - 1) / g.nblk;
        cap = (place_items(s, g) + 3) / 4;
    }
    const int parts = want < cap ? want : cap;
    return parts < 1 ? 1 : parts;
}

// Ring slots per warp of the bf16 bulk copy: the pieces a warp takes, 1 to 3.
int place_slots(const moe_shape_t *s, const Geometry &g, int parts)
{
    const int per_warp = (place_items(s, g) + 8 * parts - 1) / (8 * parts);
    return per_warp < 1 ? 1 : per_warp > 3 ? 3 : per_warp;
}

// One dispatch pass over `rounds` rounds of virtual blocks: the control words zeroed, the
// histogram / look-back / totals kernel, then the placement kernel (positions, the mapping
// table and, when `pay` is given, the copy of the rows).
// The one-kernel pass (dispatch_fused_kernel) when it applies: one round, bf16 rows or no
// copy, the layout within a CTA's shared memory, and every CTA of the grid resident at once
// (a cooperative launch: the grid barrier needs them all). Returns 1 when launched, 0 when the
// two-kernel pass must run instead, -1 on a CUDA error.
int dispatch_fused(const moe_shape_t *s, const Geometry &g, const VBlocks &vbm,
                   const int32_t *topk_idx, int32_t *counts, int32_t *kept, int32_t *offsets,
                   int32_t *row_of, int32_t *assign_of_row, int32_t *expert_of, const Payload *pay,
                   const uint16_t *x, int64_t *D, int64_t *pk_off, moe_stats_t *stats,
                   const DispatchScratch &sc, cudaStream_t st, const RankPack &rk)
{
    if (pay && pay->e4m3)
        return 0;
    const int nvb = g.nvb_round, nseg = g.nseg_round;
    const int nsub = g.slot_major ? s->K : 1;
    constexpr size_t kMaxSmem = 200 * 1024;  // dynamic; the kernel's static part stays below 1 KB
    const size_t big = fused_layout(s->E, s->K, s->W, nvb, nseg, nsub, 2).total;
    if (big > kMaxSmem)
        return 0;
    int per_sm = 0;
    if (smem_attr_once(dispatch_fused_kernel, (int)kMaxSmem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_fused_kernel, kPlaceThreads,
                                                      big) != cudaSuccess) {
        (void)cudaGetLastError();  // not available here: the two-kernel pass runs instead
        return 0;
    }
    const int capacity = per_sm * num_sms();
    if (capacity < g.nblk)
        return 0;
    int parts = 1, slots = 1;
    if (pay) {
        const int items = place_items(s, g);
        parts = capacity / g.nblk;
        const int cap = (items + 3) / 4;
        parts = parts < cap ? parts : cap;
        parts = parts < 1 ? 1 : parts;
        slots = 2;  // the copy by destination row deals the rows over every warp of the grid
    }
    const size_t smem = fused_layout(s->E, s->K, s->W, nvb, nseg, nsub, slots).total;
    if (cudaMemsetAsync(sc.ctl, 0, 4, st) != cudaSuccess)
        return -1;
    FusedArgs fa = {};
    fa.topk_idx = topk_idx;
    fa.vbm = vbm;
    fa.nvb = nvb;
    fa.bps = g.bps;
    fa.nseg = nseg;
    fa.N = s->N;
    fa.E = s->E;
    fa.K = s->K;
    fa.W = s->W;
    fa.C = (int)g.C;
    fa.ctl = sc.ctl;
    fa.agg = sc.agg;
    fa.counts = counts;
    fa.kept = kept;
    fa.offsets = offsets;
    fa.D = D;
    fa.pk_off = pk_off;
    fa.row_of = row_of;
    fa.assign_of_row = assign_of_row;
    fa.expert_of = expert_of;
    fa.packed_row_of = rk.packed_row_of;
    fa.rank = rk.rank;
    fa.x_row0 = rk.x_row0;
    fa.send_row_of = rk.send_row_of;
    fa.pk_of = sc.pk_of;
    fa.copy = pay ? 1 : 0;
    fa.x = x;
    fa.d = s->d;
    fa.x_sorted = pay ? pay->x_sorted : nullptr;
    fa.x_packed = pay ? pay->x_packed : nullptr;
    fa.stats = stats;
    fa.slots = slots;
    fa.timeout_ns = kWaitTimeoutNs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.nblk, parts);
    cfg.blockDim = dim3(kPlaceThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, dispatch_fused_kernel, fa) == cudaSuccess ? 1 : -1;
}

moe_status_t dispatch_pass(const moe_shape_t *s, const Geometry &g, int rounds,
                           const int32_t *moved, const int32_t *topk_idx, int32_t *counts,
                           int32_t *kept, int32_t *offsets, int32_t *row_of,
                           int32_t *assign_of_row, int32_t *expert_of, const Payload *pay,
                           const uint16_t *x, int64_t *D, int64_t *pk_off, moe_stats_t *stats,
                           const DispatchScratch &sc, cudaStream_t st,
                           const RankPack &rk = RankPack())
{
    VBlocks vbm;
    vbm.bm = BlockMap{g.S, g.bps, kDispatchHB};
    vbm.nblk_tok = g.nblk;
    vbm.slot_major = g.slot_major;
    vbm.K = s->K;
    vbm.nvb_round = g.nvb_round;
    vbm.moved = moved;
    const int nvb = rounds * g.nvb_round, nseg = rounds * g.nseg_round;
    if (rounds == 1) {
        const int f = dispatch_fused(s, g, vbm, topk_idx, counts, kept, offsets, row_of,
                                     assign_of_row, expert_of, pay, x, D, pk_off, stats, sc, st, rk);
        if (f != 0)
            return f > 0 ? launch_status() : MOE_ERR_CUDA;
    }
    if (cudaMemsetAsync(sc.ctl, 0, ((size_t)nvb + 2) * 4, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    HistArgs ha;
    ha.topk_idx = topk_idx;
    ha.vbm = vbm;
    ha.nvb = nvb;
    ha.bps = g.bps;
    ha.nseg = nseg;
    ha.nseg_round = g.nseg_round;
    ha.N = s->N;
    ha.E = s->E;
    ha.K = s->K;
    ha.W = s->W;
    ha.C = (int)g.C;
    ha.ctl = sc.ctl;
    ha.agg = sc.agg;
    ha.incl = sc.incl;
    ha.counts = counts;
    ha.kept = kept;
    ha.offsets = offsets;
    ha.D = D;
    ha.pk_off = pk_off;
    ha.pk_base = sc.pk_base;
    ha.stats = stats;
    ha.timeout_ns = kWaitTimeoutNs;
    const size_t hsm = hist_smem_bytes(s->E, s->W, nseg);
    if (smem_attr_once(dispatch_hist_kernel,
                       (int)(hist_smem_bytes(kMaxE, kMaxW, 0) + (size_t)kCumCacheInts * 4)) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    dispatch_hist_kernel<<<nvb, kHistThreads, hsm, st>>>(ha);

    PlaceArgs pa = {};
    pa.topk_idx = topk_idx;
    pa.vbm = vbm;
    pa.rounds = rounds;
    pa.bps = g.bps;
    pa.E = s->E;
    pa.K = s->K;
    pa.W = s->W;
    pa.C = (int)g.C;
    pa.agg = sc.agg;
    pa.incl = sc.incl;
    pa.offsets = offsets;
    pa.pk_base = sc.pk_base;
    pa.row_of = row_of;
    pa.assign_of_row = assign_of_row;
    pa.expert_of = expert_of;
    pa.packed_row_of = rk.packed_row_of;
    pa.rank = rk.rank;
    pa.x_row0 = rk.x_row0;
    pa.pk_off = pk_off;
    pa.send_row_of = rk.send_row_of;
    pa.stats = stats;
    pa.x = x;
    pa.d = s->d;
    pa.timeout_ns = kWaitTimeoutNs;
    int parts = 1;
    size_t psm = place_smem_bytes(s->E, s->K);
    if (pay) {
        pa.copy = 1;
        pa.e4m3 = pay->e4m3 ? 1 : 0;
        pa.x_sorted = pay->x_sorted;
        pa.x_packed = pay->x_packed;
        pa.sorted_scale = pay->sorted_scale;
        pa.packed_scale = pay->packed_scale;
        parts = place_parts(s, g, pay->e4m3);
        if (!pay->e4m3) {
            pa.slots = place_slots(s, g, parts);
            psm = place_smem_total(s->E, s->K, pa.slots);
        }
    }
    if (smem_attr_once(dispatch_place_kernel, (int)place_smem_total(kMaxE, kMaxK, 3)) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    dispatch_place_kernel<<<dim3(g.nblk, parts), kPlaceThreads, psm, st>>>(pa);
    return launch_status();
}

template <typename Layout>
DispatchScratch scratch_at(char *w, const Layout &L)
{
    return DispatchScratch{reinterpret_cast<unsigned int *>(w + L.ctl),
                           reinterpret_cast<int32_t *>(w + L.agg),
                           reinterpret_cast<int32_t *>(w + L.incl),
                           reinterpret_cast<int64_t *>(w + L.pk_base),
                           reinterpret_cast<int32_t *>(w + L.moved),
                           L.pk_of == kNoScratch ? nullptr
                                                 : reinterpret_cast<int32_t *>(w + L.pk_of)};
}

// logits: needed when g.rounds == 2 (re-routing); the moved-to experts then go to sc.moved.
moe_status_t dispatch_impl(const moe_shape_t *s, const Geometry &g, const uint16_t *x,
                           const float *logits, const int32_t *topk_idx, int32_t *counts,
                           int32_t *kept, int32_t *offsets, int32_t *row_of,
                           int32_t *assign_of_row, int32_t *expert_of, const Payload &pay,
                           int64_t *D, int64_t *pk_off, moe_stats_t *stats,
                           const DispatchScratch &sc, cudaStream_t st)
{
    const int32_t *round1 = nullptr;
    if (g.rounds > 1) {
        // round 0 alone: which assignments are past capacity (positions only, no copy)
        moe_status_t rc = dispatch_pass(s, g, 1, nullptr, topk_idx, counts, kept, offsets,
                                        row_of, assign_of_row, nullptr, nullptr, x, D, pk_off,
                                        nullptr, sc, st);
        if (rc != MOE_OK)
            return rc;
        RerouteArgs ra;
        ra.logits = logits;
        ra.topk_idx = topk_idx;
        ra.row_of = row_of;
        ra.counts = counts;
        ra.N = s->N;
        ra.E = s->E;
        ra.K = s->K;
        ra.C = (int)g.C;
        ra.moved = sc.moved;
        reroute_kernel<<<(s->N + 7) / 8, 256, 0, st>>>(ra);
        round1 = sc.moved;
    }
    return dispatch_pass(s, g, g.rounds, round1, topk_idx, counts, kept, offsets, row_of,
                         assign_of_row, expert_of, &pay, x, D, pk_off, stats, sc, st);
}

// ---------------------------------------------------------------- expert GEMMs

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D tensor [rows][inner] of bf16 (or fp16, or e4m3 bytes), box 128 rows x one 128-byte
// swizzle atom (64 bf16 / fp16 or 128 e4m3 elements), 128-byte swizzle.
bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t rows, bool e4m3 = false,
               bool f16 = false)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    const uint64_t esize = e4m3 ? 1 : 2;
    const CUtensorMapDataType dt = e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * esize};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esize), 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The down projection's output as a store target, box 32 rows x 32 columns: fp32 y
// [rows][inner] (128-byte rows, 128-byte swizzle), or the fp16 codes of the fp16 return
// payload (row_bytes apart; 64-byte rows, 64-byte swizzle) -- the epilogue's shared-memory
// tile layouts.
bool make_tmap_y(CUtensorMap *m, void *ptr, uint64_t inner, uint64_t rows, bool f16 = false,
                 uint64_t row_bytes = 0)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {f16 ? row_bytes : inner * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                     2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     f16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE, int BN>
moe_status_t launch_gemm(const CUtensorMap &a, const CUtensorMap &b0, const CUtensorMap &b1,
                         const gg::Args &args, cudaStream_t st)
{
    const int smem = gg::smem_bytes<MODE, BN>(kMaxE);
    if (smem_attr_once(gg::grouped_gemm_kernel<MODE, BN>, smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    gg::grouped_gemm_kernel<MODE, BN><<<num_sms(), gg::THREADS, smem, st>>>(a, b0, b1, args);
    return launch_status();
}

// Launches the CTA-pair kernel with a 2-CTA cluster, as many pairs as fit on the
// GPU at once (the tile schedule is static per pair, so every pair must be resident).
template <int MODE>
moe_status_t launch_gemm_pair(const CUtensorMap &a, const CUtensorMap &b0, const CUtensorMap &b1,
                              const gg::Args &args, cudaStream_t st)
{
    const int smem = gg::smem_bytes_pair<MODE>(kMaxE);
    const int sms = num_sms();
    int pairs = 0;
    const cudaError_t attr_err = once_per_device(
        reinterpret_cast<const void *>(gg::grouped_gemm_pair_kernel<MODE>), [&](int *n_pairs) {
        cudaError_t e = cudaFuncSetAttribute(gg::grouped_gemm_pair_kernel<MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
        cfg.blockDim = dim3(gg::THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaOccupancyMaxActiveClusters(n_pairs, gg::grouped_gemm_pair_kernel<MODE>, &cfg);
    }, &pairs);
    if (attr_err != cudaSuccess || pairs <= 0)
        return MOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(gg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gg::grouped_gemm_pair_kernel<MODE>, a, b0, b1, args) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

// Kernel choice. With many rows per expert on average (prefill of a few large experts) both
// kernels are launched and each expert goes to the one whose tiles waste less (on the device,
// prefer_pair_tiles: 256-row pair tiles unless 128-row tiles save more than 10 %). With fewer
// (decode, or many small experts where skewed routing leaves most experts a few hundred rows)
// only the single-CTA kernel runs: measured faster there, its 128-row tiles wasting less.
bool use_pair_tiles(const moe_shape_t *s, const Geometry &g)
{
    const int64_t mean_rows = ((int64_t)s->N * s->K) / s->E;
    const int64_t rows = mean_rows < g.C ? mean_rows : g.C;
    return rows >= 768;
}

// Grouped GEMM launches for E experts of width f over an A buffer of a_rows rows (the
// tensor map's extent: rows past it read as zeros). `pair` selects the CTA-pair kernel;
// `f16`: h is written (gate/up) or read together with fp16 W2 (down) as fp16, else bf16;
// h_amax (f16 only, DEVICE, one word): the largest |h| of the gate/up, which sizes the fp16
// range scale (a second gate/up pass runs only when it is beyond fp16's range).
moe_status_t gemm_up(int E, int d, int f, int64_t a_rows, bool pair, const uint16_t *a,
                     const int32_t *offsets, const uint16_t *w1, const uint16_t *w3, uint16_t *h,
                     bool f16, uint32_t *h_amax, cudaStream_t st)
{
    CUtensorMap tA, tW1, tW3;
    if (!make_tmap(&tA, a, d, (uint64_t)a_rows) || !make_tmap(&tW1, w1, d, (uint64_t)E * f) ||
        !make_tmap(&tW3, w3, d, (uint64_t)E * f))
        return MOE_ERR_CUDA;
    gg::Args args = {};
    args.offsets = offsets;
    args.E = E;
    args.n_tiles = f / 128;
    args.k_blocks = d / gg::BK;
    args.b_rows = f;
    args.rows_alloc = (int)a_rows;
    args.out = h;
    args.ldo = f;
    args.h_f16 = f16 ? 1 : 0;
    args.h_amax = h_amax;
    args.timeout_ns = kWaitTimeoutNs;
    args.select = 0;
    if (f16 && cudaMemsetAsync(h_amax, 0, sizeof(uint32_t), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (pair) {
        args.select = 1;
        moe_status_t rc = launch_gemm_pair<0>(tA, tW1, tW3, args, st);
        if (rc != MOE_OK)
            return rc;
        args.select = 2;
    }
    moe_status_t rc = launch_gemm<0, 256>(tA, tW1, tW3, args, st);
    if (rc != MOE_OK || !f16)
        return rc;
    // the fp16 range pass: every expert again with h scaled into range, only if it is needed
    args.select = 0;
    args.h_pass = 1;
    return launch_gemm<0, 256>(tA, tW1, tW3, args, st);
}

// y_stride > 0: y is the FP8 return payload with that row stride (written by plain stores;
// the y tensor map, unused then, is a copy of the W2 map).
moe_status_t gemm_down(int E, int d, int f, int64_t a_rows, bool pair, const uint16_t *h,
                       const int32_t *offsets, const uint16_t *w2, void *y, int y_stride, bool y_f16,
                       bool f16, uint32_t *h_amax, cudaStream_t st)
{
    CUtensorMap tA, tW2, tY;
    if (!make_tmap(&tA, h, f, (uint64_t)a_rows, false, f16) ||
        !make_tmap(&tW2, w2, f, (uint64_t)E * d, false, f16))
        return MOE_ERR_CUDA;
    if (y_stride > 0 && !y_f16)
        tY = tW2;
    else if (!make_tmap_y(&tY, y, d, (uint64_t)a_rows, y_f16, (uint64_t)y_stride))
        return MOE_ERR_CUDA;
    gg::Args args = {};
    args.offsets = offsets;
    args.E = E;
    args.k_blocks = f / gg::BK;
    args.b_rows = d;
    args.rows_alloc = (int)a_rows;
    args.out = y;
    args.ldo = d;
    args.y_stride = y_stride;
    args.y_f16 = y_f16 ? 1 : 0;
    args.h_f16 = f16 ? 1 : 0;
    args.h_amax = h_amax;
    args.timeout_ns = kWaitTimeoutNs;
    args.select = 0;
    if (d % 256 == 0) {
        args.n_tiles = d / 256;
        if (pair) {
            args.select = 1;
            moe_status_t rc = launch_gemm_pair<1>(tA, tW2, tY, args, st);
            if (rc != MOE_OK)
                return rc;
            args.select = 2;
        }
        return launch_gemm<1, 256>(tA, tW2, tY, args, st);
    }
    args.n_tiles = d / 128;
    return launch_gemm<1, 128>(tA, tW2, tY, args, st);
}

// Gate/up on the FP8 payload: e4m3 rows of x (scale per row) and e4m3 rows of W1, W3
// (scale per output channel). The pair kernel's stages hold two atoms, so it needs
// d % 256 == 0; otherwise every expert takes the single-CTA kernel.
moe_status_t gemm_up_e4m3(int E, int d, int f, int64_t a_rows, bool pair, const uint8_t *a,
                          const float *a_scale, const int32_t *offsets, const uint8_t *w1,
                          const float *s1, const uint8_t *w3, const float *s3, uint16_t *h,
                          cudaStream_t st)
{
    CUtensorMap tA, tW1, tW3;
    if (!make_tmap(&tA, a, d, (uint64_t)a_rows, true) ||
        !make_tmap(&tW1, w1, d, (uint64_t)E * f, true) ||
        !make_tmap(&tW3, w3, d, (uint64_t)E * f, true))
        return MOE_ERR_CUDA;
    gg::Args args = {};
    args.offsets = offsets;
    args.E = E;
    args.n_tiles = f / 128;
    args.k_blocks = d / gg::atom_k(2);
    args.b_rows = f;
    args.rows_alloc = (int)a_rows;
    args.out = h;
    args.ldo = f;
    args.row_scale = a_scale;
    args.b_scale0 = s1;
    args.b_scale1 = s3;
    args.timeout_ns = kWaitTimeoutNs;
    args.select = 0;
    if (pair && args.k_blocks % gg::KA2 == 0) {
        args.select = 1;
        moe_status_t rc = launch_gemm_pair<2>(tA, tW1, tW3, args, st);
        if (rc != MOE_OK)
            return rc;
        args.select = 2;
    }
    return launch_gemm<2, 256>(tA, tW1, tW3, args, st);
}

// Down projection on e4m3 rows of h (scale per row) and e4m3 rows of W2 (scale per output
// channel), fp32 y. The pair kernel needs f % 256 == 0 (two atoms per stage).
moe_status_t gemm_down_e4m3(int E, int d, int f, int64_t a_rows, bool pair, const uint8_t *hq,
                            const float *h_scale, const int32_t *offsets, const uint8_t *w2,
                            const float *s2, void *y, int y_stride, bool y_f16, cudaStream_t st)
{
    CUtensorMap tA, tW2, tY;
    if (!make_tmap(&tA, hq, f, (uint64_t)a_rows, true) ||
        !make_tmap(&tW2, w2, f, (uint64_t)E * d, true))
        return MOE_ERR_CUDA;
    if (y_stride > 0 && !y_f16)
        tY = tW2;
    else if (!make_tmap_y(&tY, y, d, (uint64_t)a_rows, y_f16, (uint64_t)y_stride))
        return MOE_ERR_CUDA;
    gg::Args args = {};
    args.offsets = offsets;
    args.E = E;
    args.k_blocks = f / gg::atom_k(3);
    args.b_rows = d;
    args.rows_alloc = (int)a_rows;
    args.out = y;
    args.ldo = d;
    args.y_stride = y_stride;
    args.y_f16 = y_f16 ? 1 : 0;
    args.row_scale = h_scale;
    args.b_scale0 = s2;
    args.timeout_ns = kWaitTimeoutNs;
    args.select = 0;
    if (d % 256 == 0) {
        args.n_tiles = d / 256;
        if (pair && args.k_blocks % gg::KA2 == 0) {
            args.select = 1;
            moe_status_t rc = launch_gemm_pair<3>(tA, tW2, tY, args, st);
            if (rc != MOE_OK)
                return rc;
            args.select = 2;
        }
        return launch_gemm<3, 256>(tA, tW2, tY, args, st);
    }
    args.n_tiles = d / 128;
    return launch_gemm<3, 128>(tA, tW2, tY, args, st);
}

// Row-wise e4m3 quantisation launch; rows_dev (nullable, device) caps the row count.
moe_status_t quantize_rows_launch(const uint16_t *src, int64_t rows, int cols, uint8_t *codes,
                                  float *scale, const int32_t *rows_dev, cudaStream_t st)
{
    const int64_t blocks64 = (rows + 7) / 8;
    const int blocks = (int)(blocks64 < 148 * 64 ? blocks64 : 148 * 64);
    quantize_rows_e4m3_kernel<<<blocks, 256, 0, st>>>(src, rows, cols, codes, scale, rows_dev);
    return launch_status();
}

// h and the down-projection weights are fp16 unless the shape asks for bf16.
inline bool h_is_f16(const moe_shape_t *s) { return !(s->flags & MOE_FLAG_H_BF16); }

// The fp16 range word of an expert GEMM's h [rows_alloc][f]: the first 4 bytes of its last row,
// which is never a kept row (rows_alloc >= R + 128).
inline uint32_t *h_range_word(const uint16_t *h, const Geometry &g, int f)
{
    return reinterpret_cast<uint32_t *>(const_cast<uint16_t *>(h) + (size_t)(g.rows_alloc - 1) * f);
}

moe_status_t expert_up_impl(const moe_shape_t *s, const Geometry &g, const uint16_t *x_sorted,
                            const int32_t *offsets, const uint16_t *w1, const uint16_t *w3,
                            uint16_t *h, cudaStream_t st)
{
    return gemm_up(s->E, s->d, s->f, g.rows_alloc, use_pair_tiles(s, g), x_sorted, offsets, w1,
                   w3, h, h_is_f16(s), h_range_word(h, g, s->f), st);
}

moe_status_t expert_down_impl(const moe_shape_t *s, const Geometry &g, const uint16_t *h,
                              const int32_t *offsets, const uint16_t *w2, void *y,
                              cudaStream_t st)
{
    return gemm_down(s->E, s->d, s->f, g.rows_alloc, use_pair_tiles(s, g), h, offsets, w2, y,
                     y_payload_stride(s), y_is_f16(s), h_is_f16(s), h_range_word(h, g, s->f), st);
}

moe_status_t expert_gemm_impl(const moe_shape_t *s, const Geometry &g, const uint16_t *x_sorted,
                              const int32_t *offsets, const uint16_t *w1, const uint16_t *w3,
                              const uint16_t *w2, uint16_t *h, void *y, cudaStream_t st)
{
    moe_status_t rc = expert_up_impl(s, g, x_sorted, offsets, w1, w3, h, st);
    if (rc != MOE_OK)
        return rc;
    return expert_down_impl(s, g, h, offsets, w2, y, st);
}

// The shared dense MLP of a Residual-MoE layer: one "expert" that owns all N rows of x.
__global__ void whole_range_offsets_kernel(int32_t *o, int n)
{
    o[0] = 0;
    o[1] = n;
}

moe_status_t shared_expert_impl(const moe_shape_t *s, int f_s, const uint16_t *x,
                                const uint16_t *ws1, const uint16_t *ws3, const uint16_t *ws2,
                                uint16_t *h_s, float *y_s, int32_t *offsets2, cudaStream_t st)
{
    whole_range_offsets_kernel<<<1, 1, 0, st>>>(offsets2, s->N);
    const bool pair = s->N >= 768;
    // the fp16 range word lives beside the offsets in the caller's scratch
    uint32_t *amax = reinterpret_cast<uint32_t *>(offsets2 + 4);
    moe_status_t rc = gemm_up(1, s->d, f_s, s->N, pair, x, offsets2, ws1, ws3, h_s, h_is_f16(s),
                              amax, st);
    if (rc != MOE_OK)
        return rc;
    return gemm_down(1, s->d, f_s, s->N, pair, h_s, offsets2, ws2, y_s, 0, false, h_is_f16(s), amax,
                     st);
}

moe_status_t combine_impl(const moe_shape_t *s, const void *y, const int32_t *row_of,
                          const float *topk_w, const float *shared_y, const uint16_t *residual,
                          void *out, cudaStream_t st)
{
    const int nvec = s->d / 8;
    const int seg = row_slice(s->N, nvec, 64);
    const int blocks = row_blocks(s->N, nvec, seg);
    const int ys = y_payload_stride(s);
    const bool ob = (s->flags & MOE_FLAG_OUT_BF16) != 0;
    const int yk = ys == 0 ? 0 : y_is_f16(s) ? 2 : 1;  // fp32 y, e4m3 payload, fp16 payload
    // the block payloads with many tokens (64 or more per SM: measured faster on the stack
    // layer, 388 -> 326 us; no faster with the 55 and 28 tokens per SM of the 128-expert and
    // Mixtral layers, slower with top-1 routing's 28): the bulk-fed combine, as many stages as
    // fit (two at least)
    if (yk != 0 && s->d % 512 == 0 && s->N >= 64 * num_sms()) {
        const size_t stage = cb_stage_bytes(s->K, ys, s->d, residual != nullptr, shared_y != nullptr);
        int S = kCbMaxStages;
        while (S >= 2 && cb_smem_bytes(stage, S) > kCbMaxSmem)
            --S;
        if (S >= 2) {
            const size_t smem = cb_smem_bytes(stage, S);
            auto bulk = [&](auto kern) {
                if (smem_attr_once(kern, (int)kCbMaxSmem) != cudaSuccess)
                    return false;
                kern<<<num_sms(), 32 * (kCbConsumers + 1), smem, st>>>(
                    y, ys, row_of, topk_w, shared_y, residual, s->N, s->d, s->K, S, out,
                    kWaitTimeoutNs);
                return true;
            };
            const bool ok = ob ? (yk == 1 ? bulk(combine_bulk_kernel<true, 1>)
                                          : bulk(combine_bulk_kernel<true, 2>))
                               : (yk == 1 ? bulk(combine_bulk_kernel<false, 1>)
                                          : bulk(combine_bulk_kernel<false, 2>));
            if (!ok)
                return MOE_ERR_CUDA;
            return launch_status();
        }
    }
    auto go = [&](auto kern) {
        kern<<<blocks, 256, 0, st>>>(y, ys, row_of, topk_w, shared_y, residual, s->N, s->d, s->K,
                                     seg, out);
    };
    if (ob)
        yk == 0 ? go(combine_kernel<true, 0>) : yk == 1 ? go(combine_kernel<true, 1>)
                                                        : go(combine_kernel<true, 2>);
    else
        yk == 0 ? go(combine_kernel<false, 0>) : yk == 1 ? go(combine_kernel<false, 1>)
                                                         : go(combine_kernel<false, 2>);
    return launch_status();
}

// An empty batch (N = 0) is a valid call: nothing is launched, and the outputs indexed by
// expert or rank (counts, kept, offsets, traffic matrix, pack offsets, counters) are zeroed.
moe_status_t empty_dispatch(const moe_shape_t *s, int32_t *counts, int32_t *kept,
                            int32_t *offsets, int64_t *D, int64_t *pk_off, moe_stats_t *stats,
                            cudaStream_t st)
{
    if (!counts || !kept || !offsets)
        return MOE_ERR_INVALID_ARG;
    const size_t E = (size_t)s->E, WW = (size_t)s->W * s->W;
    bool ok = cudaMemsetAsync(counts, 0, E * 4, st) == cudaSuccess &&
              cudaMemsetAsync(kept, 0, E * 4, st) == cudaSuccess &&
              cudaMemsetAsync(offsets, 0, (E + 1) * 4, st) == cudaSuccess;
    if (ok && D)
        ok = cudaMemsetAsync(D, 0, WW * 8, st) == cudaSuccess;
    if (ok && pk_off)
        ok = cudaMemsetAsync(pk_off, 0, (WW + 1) * 8, st) == cudaSuccess;
    if (ok && stats)
        ok = cudaMemsetAsync(stats, 0, sizeof(moe_stats_t), st) == cudaSuccess;
    return ok ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t empty_layer(moe_stats_t *stats, cudaStream_t st)
{
    if (stats && cudaMemsetAsync(stats, 0, sizeof(moe_stats_t), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace

// ================================================================ C ABI

extern "C" {

__attribute__((visibility("default"))) int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

__attribute__((visibility("default"))) const char *moe_status_string(moe_status_t st)
{
    switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_NONFINITE: return "MOE_ERR_NONFINITE";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS";
    case MOE_ERR_F16_RANGE: return "MOE_ERR_F16_RANGE";
    }
    return "MOE_ERR_UNKNOWN";
}

__attribute__((visibility("default"))) int64_t moe_capacity(const moe_shape_t *shape)
{
    if (!shape)
        return -1;
    return capacity_of(shape);
}

__attribute__((visibility("default"))) int64_t moe_rows_alloc(const moe_shape_t *shape)
{
    Geometry g;
    if (check_shape(shape, false, &g) != MOE_OK)
        return -1;
    return g.rows_alloc;
}

__attribute__((visibility("default"))) size_t moe_workspace_size(const moe_shape_t *shape)
{
    Geometry g;
    if (check_shape(shape, false, &g) != MOE_OK)
        return 0;
    return scratch_layout(shape, g).total;
}

__attribute__((visibility("default"))) size_t moe_layer_workspace_size(const moe_shape_t *shape)
{
    Geometry g;
    if (check_shape(shape, true, &g) != MOE_OK)
        return 0;
    return layer_layout(shape, g, scratch_layout(shape, g).total).total;
}

__attribute__((visibility("default"))) size_t moe_y_bytes(const moe_shape_t *shape)
{
    Geometry g;
    if (check_shape(shape, false, &g) != MOE_OK)
        return 0;
    const int ys = y_payload_stride(shape);
    return (size_t)g.rows_alloc * (ys > 0 ? (size_t)ys : (size_t)shape->d * 4);
}

__attribute__((visibility("default"))) moe_status_t
moe_route(const moe_shape_t *shape, const uint16_t *x, const float *w_router, const float *bias,
          int32_t *topk_idx, float *topk_w, float *logits, void *ws, size_t ws_bytes,
          moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, false, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!x || !w_router || !topk_idx || !topk_w)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || (bias && !aligned4(bias)) ||
        !aligned4(topk_idx) || !aligned4(topk_w) || (logits && !aligned4(logits)))
        return MOE_ERR_MISALIGNED;
    float *scratch = nullptr;
    if (!logits || router_split_ec(shape)) {
        const ScratchLayout L = scratch_layout(shape, g);
        if (!ws || ws_bytes < L.total)
            return MOE_ERR_WORKSPACE_TOO_SMALL;
        if (!aligned16(ws))
            return MOE_ERR_MISALIGNED;
        scratch = reinterpret_cast<float *>(static_cast<char *>(ws) + L.logits);
    }
    return route_impl(shape, x, w_router, bias, topk_idx, topk_w, logits, scratch, nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

namespace {

moe_status_t dispatch_entry(const moe_shape_t *shape, const uint16_t *x, const float *logits,
                            const int32_t *topk_idx, int32_t *counts, int32_t *kept,
                            int32_t *offsets, int32_t *row_of, int32_t *assign_of_row,
                            int32_t *expert_of, const Payload &pay, int64_t *rank_matrix,
                            int64_t *packed_offsets, moe_stats_t *stats, void *ws,
                            size_t ws_bytes, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, false, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return empty_dispatch(shape, counts, kept, offsets, rank_matrix, packed_offsets, stats,
                              reinterpret_cast<cudaStream_t>(stream));
    if (!x || !topk_idx || !counts || !kept || !offsets || !row_of || !assign_of_row ||
        !pay.x_sorted)
        return MOE_ERR_INVALID_ARG;
    if ((g.rounds > 1) != (logits != nullptr))
        return MOE_ERR_INVALID_ARG;
    if (pay.e4m3 && (shape->d % 16 != 0 || !pay.sorted_scale ||
                     (pay.x_packed != nullptr) != (pay.packed_scale != nullptr)))
        return pay.e4m3 && shape->d % 16 != 0 ? MOE_ERR_UNSUPPORTED_SHAPE : MOE_ERR_INVALID_ARG;
    if (pay.e4m3 && (!aligned4(pay.sorted_scale) ||
                     (pay.packed_scale && !aligned4(pay.packed_scale))))
        return MOE_ERR_MISALIGNED;
    if (!aligned16(x) || !aligned16(pay.x_sorted) || (pay.x_packed && !aligned16(pay.x_packed)) ||
        !aligned4(topk_idx) || !aligned4(counts) || !aligned4(kept) || !aligned4(offsets) ||
        !aligned4(row_of) || !aligned4(assign_of_row) || (logits && !aligned4(logits)) ||
        (expert_of && !aligned4(expert_of)) ||
        (rank_matrix && (reinterpret_cast<uintptr_t>(rank_matrix) & 7u)) ||
        (packed_offsets && (reinterpret_cast<uintptr_t>(packed_offsets) & 7u)) ||
        (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return MOE_ERR_MISALIGNED;
    const ScratchLayout L = scratch_layout(shape, g);
    if (!ws || ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return MOE_ERR_MISALIGNED;
    char *w = static_cast<char *>(ws);
    int64_t *D = rank_matrix ? rank_matrix : reinterpret_cast<int64_t *>(w + L.D);
    int64_t *pk = packed_offsets ? packed_offsets : reinterpret_cast<int64_t *>(w + L.pk_off);
    return dispatch_impl(shape, g, x, logits, topk_idx, counts, kept, offsets, row_of,
                         assign_of_row, expert_of, pay, D, pk, stats, scratch_at(w, L),
                         reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

__attribute__((visibility("default"))) moe_status_t
moe_dispatch(const moe_shape_t *shape, const uint16_t *x, const int32_t *topk_idx, int32_t *counts,
             int32_t *kept, int32_t *offsets, int32_t *row_of, int32_t *assign_of_row,
             uint16_t *x_sorted, uint16_t *x_packed, int64_t *rank_matrix,
             int64_t *packed_offsets, moe_stats_t *stats, void *ws, size_t ws_bytes,
             moe_stream_t stream)
{
    // re-routing ranks candidates by the logits, which this entry point does not take
    if (shape && (shape->flags & MOE_FLAG_REROUTE))
        return MOE_ERR_INVALID_ARG;
    return dispatch_entry(shape, x, nullptr, topk_idx, counts, kept, offsets, row_of,
                          assign_of_row, nullptr, Payload{x_sorted, x_packed, false, nullptr, nullptr},
                          rank_matrix, packed_offsets, stats, ws, ws_bytes, stream);
}

__attribute__((visibility("default"))) moe_status_t
moe_dispatch_rank(const moe_shape_t *shape, int32_t rank, const uint16_t *x_local,
                  const int32_t *topk_idx_all, int32_t *counts, int32_t *kept, int32_t *offsets,
                  int32_t *row_of, int32_t *assign_of_row, int32_t *packed_row_of,
                  int32_t *send_row_of, uint16_t *x_send, int64_t *rank_matrix,
                  int64_t *packed_offsets, moe_stats_t *stats, void *ws, size_t ws_bytes,
                  moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, false, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->flags & MOE_FLAG_REROUTE)
        return MOE_ERR_INVALID_ARG;  // candidates are ranked by every token's logits
    if (rank < 0 || rank >= shape->W)
        return MOE_ERR_INVALID_ARG;
    if (shape->N == 0)
        return empty_dispatch(shape, counts, kept, offsets, rank_matrix, packed_offsets, stats,
                              reinterpret_cast<cudaStream_t>(stream));
    if (!x_local || !topk_idx_all || !counts || !kept || !offsets || !row_of || !assign_of_row ||
        !packed_row_of || !send_row_of || !x_send || !rank_matrix || !packed_offsets)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_local) || !aligned16(x_send) || !aligned4(topk_idx_all) || !aligned4(counts) ||
        !aligned4(kept) || !aligned4(offsets) || !aligned4(row_of) || !aligned4(assign_of_row) ||
        !aligned4(packed_row_of) || !aligned4(send_row_of) ||
        (reinterpret_cast<uintptr_t>(rank_matrix) & 7u) ||
        (reinterpret_cast<uintptr_t>(packed_offsets) & 7u) ||
        (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return MOE_ERR_MISALIGNED;
    const ScratchLayout L = scratch_layout(shape, g);
    if (!ws || ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return MOE_ERR_MISALIGNED;
    RankPack rk;
    rk.rank = rank;
    rk.x_row0 = rank * g.S;
    rk.packed_row_of = packed_row_of;
    rk.send_row_of = send_row_of;
    const Payload pay{nullptr, x_send, false, nullptr, nullptr};
    return dispatch_pass(shape, g, 1, nullptr, topk_idx_all, counts, kept, offsets, row_of,
                         assign_of_row, nullptr, &pay, x_local, rank_matrix, packed_offsets, stats,
                         scratch_at(static_cast<char *>(ws), L),
                         reinterpret_cast<cudaStream_t>(stream), rk);
}

__attribute__((visibility("default"))) moe_status_t
moe_regroup_rows(const moe_shape_t *shape, int32_t rank, int32_t row_bytes, int32_t direction,
                 const void *src, void *dst, const int32_t *assign_of_row,
                 const int32_t *packed_row_of, const int32_t *offsets,
                 const int64_t *packed_offsets, int32_t *offsets_local, moe_stream_t stream)
{
    moe_status_t rc = check_shape(shape, false, nullptr);
    if (rc != MOE_OK)
        return rc;
    if (rank < 0 || rank >= shape->W || (direction != 0 && direction != 1) || row_bytes <= 0)
        return MOE_ERR_INVALID_ARG;
    if (row_bytes % 16 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (shape->N == 0)
        return MOE_OK;  // no rows
    if (!src || !dst || !assign_of_row || !packed_row_of || !offsets || !packed_offsets)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst) || !aligned4(assign_of_row) ||
        !aligned4(packed_row_of) || !aligned4(offsets) ||
        (reinterpret_cast<uintptr_t>(packed_offsets) & 7u) ||
        (offsets_local && !aligned4(offsets_local)))
        return MOE_ERR_MISALIGNED;
    RegroupArgs ra;
    ra.assign_of_row = assign_of_row;
    ra.packed_row_of = packed_row_of;
    ra.offsets = offsets;
    ra.pk_off = packed_offsets;
    ra.E = shape->E;
    ra.K = shape->K;
    ra.W = shape->W;
    ra.S = shape->N / shape->W;
    ra.rank = rank;
    ra.row_vec = row_bytes / 16;
    ra.src = static_cast<const uint4 *>(src);
    ra.dst = static_cast<uint4 *>(dst);
    ra.dir = direction;
    ra.offsets_local = offsets_local;
    regroup_rows_kernel<<<2 * num_sms(), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ra);
    return launch_status();
}

__attribute__((visibility("default"))) moe_status_t
moe_dispatch_reroute(const moe_shape_t *shape, const uint16_t *x, const float *logits,
                     const int32_t *topk_idx, int32_t *counts, int32_t *kept, int32_t *offsets,
                     int32_t *row_of, int32_t *assign_of_row, int32_t *expert_of,
                     uint16_t *x_sorted, uint16_t *x_packed, int64_t *rank_matrix,
                     int64_t *packed_offsets, moe_stats_t *stats, void *ws, size_t ws_bytes,
                     moe_stream_t stream)
{
    if (!shape || !(shape->flags & MOE_FLAG_REROUTE) || (!logits && shape->N != 0))
        return MOE_ERR_INVALID_ARG;
    return dispatch_entry(shape, x, logits, topk_idx, counts, kept, offsets, row_of,
                          assign_of_row, expert_of,
                          Payload{x_sorted, x_packed, false, nullptr, nullptr}, rank_matrix,
                          packed_offsets, stats, ws, ws_bytes, stream);
}

__attribute__((visibility("default"))) moe_status_t
moe_dispatch_fp8(const moe_shape_t *shape, const uint16_t *x, const int32_t *topk_idx,
                 int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *row_of,
                 int32_t *assign_of_row, uint8_t *x_sorted, float *sorted_scale,
                 uint8_t *x_packed, float *packed_scale, int64_t *rank_matrix,
                 int64_t *packed_offsets, moe_stats_t *stats, void *ws, size_t ws_bytes,
                 moe_stream_t stream)
{
    if (shape && (shape->flags & MOE_FLAG_REROUTE))
        return MOE_ERR_INVALID_ARG;
    return dispatch_entry(shape, x, nullptr, topk_idx, counts, kept, offsets, row_of,
                          assign_of_row, nullptr,
                          Payload{x_sorted, x_packed, true, sorted_scale, packed_scale},
                          rank_matrix, packed_offsets, stats, ws, ws_bytes, stream);
}

__attribute__((visibility("default"))) moe_status_t
moe_quantize_rows_e4m3(const uint16_t *src, int64_t rows, int32_t cols, uint8_t *codes,
                       float *scale, const int32_t *rows_dev, moe_stream_t stream)
{
    if (rows < 0 || cols < 16 || !src || !codes || !scale)
        return MOE_ERR_INVALID_ARG;
    if (cols % 16 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(src) || !aligned16(codes) || !aligned4(scale) ||
        (rows_dev && !aligned4(rows_dev)))
        return MOE_ERR_MISALIGNED;
    if (rows == 0)
        return MOE_OK;
    return quantize_rows_launch(src, rows, cols, codes, scale, rows_dev,
                                reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_convert_bf16_to_f16(const uint16_t *src, int64_t n, uint16_t *dst, int64_t *changed,
                        moe_stream_t stream)
{
    if (n < 0 || (n > 0 && (!src || !dst)))
        return MOE_ERR_INVALID_ARG;
    if (n % 8 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((n > 0 && (!aligned16(src) || !aligned16(dst))) ||
        (changed && (reinterpret_cast<uintptr_t>(changed) & 7u)))
        return MOE_ERR_MISALIGNED;
    if (n == 0)
        return MOE_OK;
    const int64_t vec = n / 8;
    const int64_t blocks64 = (vec + 255) / 256;
    const int blocks = (int)(blocks64 < 64LL * num_sms() ? blocks64 : 64LL * num_sms());
    convert_bf16_f16_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        src, n, dst, reinterpret_cast<unsigned long long *>(changed));
    return launch_status();
}

__attribute__((visibility("default"))) moe_status_t
moe_expert_up_fp8(const moe_shape_t *shape, const uint8_t *x_sorted, const float *sorted_scale,
                  const int32_t *offsets, const uint8_t *w1q, const float *w1_scale,
                  const uint8_t *w3q, const float *w3_scale, uint16_t *h, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!x_sorted || !sorted_scale || !offsets || !w1q || !w1_scale || !w3q || !w3_scale || !h)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_sorted) || !aligned16(w1q) || !aligned16(w3q) || !aligned16(w1_scale) ||
        !aligned16(w3_scale) || !aligned16(h) || !aligned4(offsets) || !aligned4(sorted_scale))
        return MOE_ERR_MISALIGNED;
    return gemm_up_e4m3(shape->E, shape->d, shape->f, g.rows_alloc, use_pair_tiles(shape, g),
                        x_sorted, sorted_scale, offsets, w1q, w1_scale, w3q, w3_scale, h,
                        reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_expert_down_fp8(const moe_shape_t *shape, const uint8_t *hq, const float *h_scale,
                    const int32_t *offsets, const uint8_t *w2q, const float *w2_scale, void *y,
                    moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!hq || !h_scale || !offsets || !w2q || !w2_scale || !y)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(hq) || !aligned16(w2q) || !aligned16(w2_scale) || !aligned16(y) ||
        !aligned4(offsets) || !aligned4(h_scale))
        return MOE_ERR_MISALIGNED;
    return gemm_down_e4m3(shape->E, shape->d, shape->f, g.rows_alloc, use_pair_tiles(shape, g),
                          hq, h_scale, offsets, w2q, w2_scale, y, y_payload_stride(shape), y_is_f16(shape),
                          reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_expert_gemm(const moe_shape_t *shape, const uint16_t *x_sorted, const int32_t *offsets,
                const uint16_t *w1, const uint16_t *w3, const uint16_t *w2, uint16_t *h,
                void *y, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!x_sorted || !offsets || !w1 || !w3 || !w2 || !h || !y)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_sorted) || !aligned16(w1) || !aligned16(w3) || !aligned16(w2) ||
        !aligned16(h) || !aligned16(y) || !aligned4(offsets))
        return MOE_ERR_MISALIGNED;
    return expert_gemm_impl(shape, g, x_sorted, offsets, w1, w3, w2, h, y,
                            reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_expert_up(const moe_shape_t *shape, const uint16_t *x_sorted, const int32_t *offsets,
              const uint16_t *w1, const uint16_t *w3, uint16_t *h, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!x_sorted || !offsets || !w1 || !w3 || !h)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_sorted) || !aligned16(w1) || !aligned16(w3) || !aligned16(h) ||
        !aligned4(offsets))
        return MOE_ERR_MISALIGNED;
    return expert_up_impl(shape, g, x_sorted, offsets, w1, w3, h,
                          reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_expert_down(const moe_shape_t *shape, const uint16_t *h, const int32_t *offsets,
                const uint16_t *w2, void *y, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!h || !offsets || !w2 || !y)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(w2) || !aligned16(y) || !aligned4(offsets))
        return MOE_ERR_MISALIGNED;
    return expert_down_impl(shape, g, h, offsets, w2, y, reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_combine(const moe_shape_t *shape, const void *y, const int32_t *row_of,
            const float *topk_w, const float *shared_y, const uint16_t *residual, void *out,
            moe_stream_t stream)
{
    moe_status_t rc = check_shape(shape, false, nullptr);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (!y || !row_of || !topk_w || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out) || !aligned4(row_of) || !aligned4(topk_w) ||
        (residual && !aligned16(residual)) || (shared_y && !aligned16(shared_y)))
        return MOE_ERR_MISALIGNED;
    return combine_impl(shape, y, row_of, topk_w, shared_y, residual, out,
                        reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Expert weights of a layer: bf16 W1, W3, W2, or their e4m3 rows with per-row scales
// (then the dispatch writes the FP8 payload and both expert GEMMs run on e4m3).
struct ExpertWeights {
    const uint16_t *w1, *w3, *w2;
    const uint8_t *w1q, *w3q, *w2q;
    const float *s1, *s3, *s2;
    bool e4m3() const { return w1q != nullptr; }
};

// The layer: route -> dispatch -> gate/up -> down -> (shared MLP) -> combine, every
// intermediate in the workspace. Arguments validated by the caller; f_shared == 0: no
// shared MLP.
moe_status_t layer_run(const moe_shape_t *shape, const Geometry &g, const uint16_t *x,
                       const float *w_router, const float *bias, const ExpertWeights &up,
                       int32_t f_shared, const uint16_t *ws1,
                       const uint16_t *ws3, const uint16_t *ws2, const uint16_t *residual,
                       void *out, int32_t *topk_idx_out, moe_stats_t *stats, char *w,
                       size_t ws_need, cudaStream_t st)
{
    const ScratchLayout S = scratch_layout(shape, g);
    const LayerLayout L = layer_layout(shape, g, S.total);
    int32_t *topk_idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t *>(w + L.topk_idx);
    float *topk_w = reinterpret_cast<float *>(w + L.topk_w);
    unsigned long long *nonfinite = nullptr;
    if (stats) {
        nonfinite = reinterpret_cast<unsigned long long *>(&stats->nonfinite_tokens);
        if (cudaMemsetAsync(nonfinite, 0, sizeof(unsigned long long), st) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // the logits are kept (in the workspace) only when re-routing ranks candidates by them
    float *lg = reinterpret_cast<float *>(w + S.logits);
    moe_status_t rc = route_impl(shape, x, w_router, bias, topk_idx, topk_w,
                                 g.rounds > 1 ? lg : nullptr, lg, nonfinite, st);
    if (rc != MOE_OK)
        return rc;
    int32_t *offsets = reinterpret_cast<int32_t *>(w + L.offsets);
    int32_t *row_of = reinterpret_cast<int32_t *>(w + L.row_of);
    uint16_t *h = reinterpret_cast<uint16_t *>(w + L.h);
    float *y = reinterpret_cast<float *>(w + L.y);
    Payload pay{w + L.x_sorted, w + L.x_packed, up.e4m3(),
                reinterpret_cast<float *>(w + L.sorted_scale),
                reinterpret_cast<float *>(w + L.packed_scale)};
    rc = dispatch_impl(shape, g, x, reinterpret_cast<const float *>(w + S.logits), topk_idx,
                       reinterpret_cast<int32_t *>(w + L.counts),
                       reinterpret_cast<int32_t *>(w + L.kept), offsets, row_of,
                       reinterpret_cast<int32_t *>(w + L.assign), nullptr, pay,
                       reinterpret_cast<int64_t *>(w + S.D), reinterpret_cast<int64_t *>(w + S.pk_off),
                       stats, scratch_at(w, S), st);
    if (rc != MOE_OK)
        return rc;
    if (up.e4m3())
        rc = gemm_up_e4m3(shape->E, shape->d, shape->f, g.rows_alloc, use_pair_tiles(shape, g),
                          static_cast<const uint8_t *>(pay.x_sorted), pay.sorted_scale, offsets,
                          up.w1q, up.s1, up.w3q, up.s3, h, st);
    else
        rc = expert_up_impl(shape, g, static_cast<const uint16_t *>(pay.x_sorted), offsets, up.w1,
                            up.w3, h, st);
    if (rc != MOE_OK)
        return rc;
    if (up.e4m3()) {
        // h -> e4m3 rows (only the offsets[E] kept rows), then the e4m3 down projection
        uint8_t *hq = reinterpret_cast<uint8_t *>(w + L.hq);
        float *hs = reinterpret_cast<float *>(w + L.h_scale);
        rc = quantize_rows_launch(h, g.rows_alloc, shape->f, hq, hs, offsets + shape->E, st);
        if (rc != MOE_OK)
            return rc;
        rc = gemm_down_e4m3(shape->E, shape->d, shape->f, g.rows_alloc,
                            use_pair_tiles(shape, g), hq, hs, offsets, up.w2q, up.s2, y,
                            y_payload_stride(shape), y_is_f16(shape), st);
    } else {
        rc = expert_down_impl(shape, g, h, offsets, up.w2, y, st);
    }
    if (rc != MOE_OK)
        return rc;
    float *y_s = nullptr;
    if (f_shared > 0) {
        uint16_t *h_s = reinterpret_cast<uint16_t *>(w + L.total);
        y_s = reinterpret_cast<float *>(w + L.total + align_up((size_t)shape->N * f_shared * 2));
        int32_t *off2 = reinterpret_cast<int32_t *>(w + ws_need - kAlign);
        rc = shared_expert_impl(shape, f_shared, x, ws1, ws3, ws2, h_s, y_s, off2, st);
        if (rc != MOE_OK)
            return rc;
    }
    return combine_impl(shape, y, row_of, topk_w, y_s, residual, out, st);
}

}  // namespace

__attribute__((visibility("default"))) moe_status_t
moe_layer(const moe_shape_t *shape, const uint16_t *x, const float *w_router, const float *bias,
          const uint16_t *w1, const uint16_t *w3, const uint16_t *w2, const uint16_t *residual,
          void *out, int32_t *topk_idx_out, moe_stats_t *stats, void *ws, size_t ws_bytes,
          moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return empty_layer(stats, reinterpret_cast<cudaStream_t>(stream));
    if (!x || !w_router || !w1 || !w3 || !w2 || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || (bias && !aligned4(bias)) || !aligned16(w1) ||
        !aligned16(w3) || !aligned16(w2) || !aligned16(out) ||
        (residual && !aligned16(residual)) || (topk_idx_out && !aligned4(topk_idx_out)) ||
        (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return MOE_ERR_MISALIGNED;
    const size_t need = moe_layer_workspace_size(shape);
    if (!ws || ws_bytes < need)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return MOE_ERR_MISALIGNED;
    return layer_run(shape, g, x, w_router, bias,
                     ExpertWeights{w1, w3, w2, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr},
                     0, nullptr, nullptr, nullptr, residual, out, topk_idx_out, stats,
                     static_cast<char *>(ws), need, reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_layer_fp8(const moe_shape_t *shape, const uint16_t *x, const float *w_router,
              const float *bias, const uint8_t *w1q, const float *w1_scale, const uint8_t *w3q,
              const float *w3_scale, const uint8_t *w2q, const float *w2_scale,
              const uint16_t *residual, void *out, int32_t *topk_idx_out, moe_stats_t *stats,
              void *ws, size_t ws_bytes, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return empty_layer(stats, reinterpret_cast<cudaStream_t>(stream));
    if (!x || !w_router || !w1q || !w1_scale || !w3q || !w3_scale || !w2q || !w2_scale || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || (bias && !aligned4(bias)) || !aligned16(w1q) ||
        !aligned16(w3q) || !aligned16(w1_scale) || !aligned16(w3_scale) || !aligned16(w2q) ||
        !aligned16(w2_scale) ||
        !aligned16(out) || (residual && !aligned16(residual)) ||
        (topk_idx_out && !aligned4(topk_idx_out)) ||
        (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return MOE_ERR_MISALIGNED;
    const size_t need = moe_layer_workspace_size(shape);
    if (!ws || ws_bytes < need)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return MOE_ERR_MISALIGNED;
    return layer_run(shape, g, x, w_router, bias,
                     ExpertWeights{nullptr, nullptr, nullptr, w1q, w3q, w2q, w1_scale, w3_scale,
                                   w2_scale},
                     0, nullptr, nullptr, nullptr, residual, out, topk_idx_out, stats,
                     static_cast<char *>(ws), need, reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_shared_expert(const moe_shape_t *shape, int32_t f_shared, const uint16_t *x,
                  const uint16_t *ws1, const uint16_t *ws3, const uint16_t *ws2, uint16_t *h_s,
                  float *y_s, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status_t rc = check_shape(shape, true, nullptr);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return MOE_OK;  // empty batch: nothing to do
    if (f_shared < 128 || f_shared % 128 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!x || !ws1 || !ws3 || !ws2 || !h_s || !y_s)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(ws1) || !aligned16(ws3) || !aligned16(ws2) ||
        !aligned16(h_s) || !aligned16(y_s))
        return MOE_ERR_MISALIGNED;
    if (!ws || ws_bytes < kAlign)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return MOE_ERR_MISALIGNED;
    return shared_expert_impl(shape, f_shared, x, ws1, ws3, ws2, h_s, y_s,
                              static_cast<int32_t *>(ws), reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) size_t
moe_layer_shared_workspace_size(const moe_shape_t *shape, int32_t f_shared)
{
    const size_t base = moe_layer_workspace_size(shape);
    if (base == 0 || f_shared < 128 || f_shared % 128 != 0)
        return 0;
    return base + align_up((size_t)shape->N * f_shared * 2) + align_up((size_t)shape->N * shape->d * 4) +
           kAlign;
}

__attribute__((visibility("default"))) moe_status_t
moe_layer_shared(const moe_shape_t *shape, int32_t f_shared, const uint16_t *x,
                 const float *w_router, const float *bias, const uint16_t *w1,
                 const uint16_t *w3, const uint16_t *w2, const uint16_t *ws1, const uint16_t *ws3,
                 const uint16_t *ws2, const uint16_t *residual, void *out, int32_t *topk_idx_out,
                 moe_stats_t *stats, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, true, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return empty_layer(stats, reinterpret_cast<cudaStream_t>(stream));
    if (f_shared < 128 || f_shared % 128 != 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!x || !w_router || !w1 || !w3 || !w2 || !ws1 || !ws3 || !ws2 || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || (bias && !aligned4(bias)) || !aligned16(w1) ||
        !aligned16(w3) || !aligned16(w2) || !aligned16(ws1) || !aligned16(ws3) ||
        !aligned16(ws2) || !aligned16(out) || (residual && !aligned16(residual)) ||
        (topk_idx_out && !aligned4(topk_idx_out)) ||
        (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return MOE_ERR_MISALIGNED;
    const size_t need = moe_layer_shared_workspace_size(shape, f_shared);
    if (!ws || ws_bytes < need)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return MOE_ERR_MISALIGNED;
    return layer_run(shape, g, x, w_router, bias,
                     ExpertWeights{w1, w3, w2, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr},
                     f_shared, ws1, ws3, ws2, residual, out, topk_idx_out, stats,
                     static_cast<char *>(ws), need, reinterpret_cast<cudaStream_t>(stream));
}

__attribute__((visibility("default"))) moe_status_t
moe_affinity_accumulate(int32_t N, int32_t E, int32_t K, const int32_t *topk_j,
                        const int32_t *topk_j1, int64_t *counts, moe_stream_t stream)
{
    if (N < 0 || E < 1 || K < 1 || K > E || !counts)
        return MOE_ERR_INVALID_ARG;
    if (N == 0)
        return MOE_OK;  // no tokens: nothing to count
    if (!topk_j || !topk_j1)
        return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || K > kMaxK)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned4(topk_j) || !aligned4(topk_j1) || (reinterpret_cast<uintptr_t>(counts) & 7u))
        return MOE_ERR_MISALIGNED;
    const int use_smem = E <= 64 ? 1 : 0;
    const int threads = 256;
    int blocks = (N + threads - 1) / threads;
    if (blocks > 4 * num_sms())
        blocks = 4 * num_sms();
    affinity_kernel<<<blocks, threads, use_smem ? (size_t)E * E * 4 : 0,
                      reinterpret_cast<cudaStream_t>(stream)>>>(
        topk_j, topk_j1, N, E, K, reinterpret_cast<unsigned long long *>(counts), use_smem);
    return launch_status();
}

__attribute__((visibility("default"))) moe_status_t
moe_derive_report(const moe_shape_t *shape, const moe_stats_t *st, const int64_t *D,
                  const int32_t *kept, moe_report_t *out)
{
    if (check_shape(shape, false, nullptr) != MOE_OK)
        return MOE_ERR_INVALID_ARG;
    if (!st || !D || !kept || !out)
        return MOE_ERR_INVALID_ARG;
    const int W = shape->W, E = shape->E;
    const double NK = (double)shape->N * shape->K;
    int64_t smax = 0, smin = INT64_MAX, rmax = 0, rmin = INT64_MAX, off_row = 0, off_col = 0;
    double mean = 0.0;
    for (int i = 0; i < W; ++i) {
        int64_t s = 0, r = 0, so = 0, ro = 0;
        for (int j = 0; j < W; ++j) {
            s += D[i * W + j];
            r += D[j * W + i];
            if (j != i) {
                so += D[i * W + j];
                ro += D[j * W + i];
            }
        }
        smax = s > smax ? s : smax;
        smin = s < smin ? s : smin;
        rmax = r > rmax ? r : rmax;
        rmin = r < rmin ? r : rmin;
        off_row = so > off_row ? so : off_row;
        off_col = ro > off_col ? ro : off_col;
        mean += (double)r;
    }
    mean /= W;
    double var = 0.0;
    for (int j = 0; j < W; ++j) {
        int64_t r = 0;
        for (int i = 0; i < W; ++i)
            r += D[i * W + j];
        var += ((double)r - mean) * ((double)r - mean);
    }
    var /= W;
    int32_t kmax = 0;
    for (int e = 0; e < E; ++e)
        kmax = kept[e] > kmax ? kept[e] : kmax;
    out->drop_rate = NK > 0 ? (double)st->dropped / NK : 0.0;
    out->send_max_over_min = smin > 0 ? (double)smax / (double)smin : INFINITY;
    out->recv_max_over_min = rmin > 0 ? (double)rmax / (double)rmin : INFINITY;
    out->cross_rank_fraction = st->rows > 0 ? (double)st->cross_rows / (double)st->rows : 0.0;
    out->load_std_over_mean = mean > 0 ? sqrt(var) / mean : 0.0;
    out->capacity_factor_effective = NK > 0 ? (double)kmax / (NK / (double)E) : 0.0;
    out->tau_min_tokens = off_row > off_col ? off_row : off_col;
    out->dispatch_bytes = st->rows * (int64_t)shape->d * 2;
    out->send_max = smax;
    out->send_min = smin;
    out->recv_max = rmax;
    out->recv_min = rmin;
    return MOE_OK;
}

__attribute__((visibility("default"))) moe_status_t
moe_read_stats(const moe_stats_t *stats_dev, moe_stats_t *out, moe_stream_t stream)
{
    if (!stats_dev || !out)
        return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(stats_dev) & 7u)
        return MOE_ERR_MISALIGNED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(out, stats_dev, sizeof(moe_stats_t), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

__attribute__((visibility("default"))) moe_status_t
moe_exchange_schedule(int32_t W, const int64_t *D, int32_t max_phases, int32_t *phase_dst,
                      int64_t *phase_len, int32_t *n_phases, int64_t *makespan)
{
    if (!D || !n_phases || !makespan || W < 1 || W > kMaxW || max_phases < 0)
        return MOE_ERR_INVALID_ARG;
    if (max_phases > 0 && (!phase_dst || !phase_len))
        return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < W * W; ++i)
        if (D[i] < 0)
            return MOE_ERR_INVALID_ARG;
    int np = 0;
    int64_t span = 0;
    if (!moe_plan::exchange_schedule(W, D, max_phases, phase_dst, phase_len, &np, &span))
        return MOE_ERR_INVALID_ARG;
    *n_phases = np;
    *makespan = span;
    return MOE_OK;
}

__attribute__((visibility("default"))) moe_status_t
moe_place_experts(int32_t L, int32_t E, int32_t P, const int64_t *counts, int32_t starts,
                  int32_t *gpu_of, int64_t *cost, int64_t *contiguous_cost)
{
    if (!gpu_of || (L > 1 && !counts) || L < 1 || E < 1 || E > kMaxE || P < 1 || E % P != 0 ||
        starts < 1 || starts > 64)
        return MOE_ERR_INVALID_ARG;
    if (L > 1)
        for (size_t i = 0; i < (size_t)(L - 1) * E * E; ++i)
            if (counts[i] < 0)
                return MOE_ERR_INVALID_ARG;
    moe_plan::place_experts(L, E, P, counts, starts, gpu_of, cost, contiguous_cost);
    return MOE_OK;
}

__attribute__((visibility("default"))) moe_status_t
moe_placement_order(int32_t L, int32_t E, int32_t P, const int32_t *gpu_of, int32_t *order)
{
    if (!gpu_of || !order || L < 1 || E < 1 || P < 1 || E % P != 0)
        return MOE_ERR_INVALID_ARG;
    const int share = E / P;
    std::vector<int> fill(P);
    for (int l = 0; l < L; ++l) {
        const int32_t *g = gpu_of + (size_t)l * E;
        std::fill(fill.begin(), fill.end(), 0);
        for (int e = 0; e < E; ++e) {
            if (g[e] < 0 || g[e] >= P || fill[g[e]] >= share)
                return MOE_ERR_INVALID_ARG;  // not a placement with E / P experts per GPU
            ++fill[g[e]];
        }
        std::fill(fill.begin(), fill.end(), 0);
        for (int e = 0; e < E; ++e)  // experts ascending within each GPU
            order[(size_t)l * E + (size_t)g[e] * share + fill[g[e]]++] = e;
    }
    return MOE_OK;
}

__attribute__((visibility("default"))) moe_status_t
moe_place_experts_staged(int32_t L, int32_t E, int32_t nodes, int32_t gpus_per_node,
                         const int64_t *counts, int32_t starts, int32_t *gpu_of,
                         int64_t *node_hops, int64_t *gpu_hops, int64_t *contiguous_node_hops,
                         int64_t *contiguous_gpu_hops)
{
    if (!gpu_of || (L > 1 && !counts) || L < 1 || E < 1 || E > kMaxE || nodes < 1 ||
        gpus_per_node < 1 || E % (nodes * gpus_per_node) != 0 || starts < 1 || starts > 64)
        return MOE_ERR_INVALID_ARG;
    if (L > 1)
        for (size_t i = 0; i < (size_t)(L - 1) * E * E; ++i)
            if (counts[i] < 0)
                return MOE_ERR_INVALID_ARG;
    moe_plan::place_experts_staged(L, E, nodes, gpus_per_node, counts, starts, gpu_of);
    std::vector<int32_t> contiguous((size_t)L * E);
    const int share = E / (nodes * gpus_per_node);
    for (int l = 0; l < L; ++l)
        for (int e = 0; e < E; ++e)
            contiguous[(size_t)l * E + e] = e / share;
    if (node_hops)
        *node_hops = moe_plan::crossing_hops(L, E, counts, gpu_of, gpus_per_node);
    if (gpu_hops)
        *gpu_hops = moe_plan::crossing_hops(L, E, counts, gpu_of, 1);
    if (contiguous_node_hops)
        *contiguous_node_hops =
            moe_plan::crossing_hops(L, E, counts, contiguous.data(), gpus_per_node);
    if (contiguous_gpu_hops)
        *contiguous_gpu_hops = moe_plan::crossing_hops(L, E, counts, contiguous.data(), 1);
    return MOE_OK;
}

__attribute__((visibility("default"))) moe_status_t moe_get_device_error(int clear)
{
    if (cudaDeviceSynchronize() != cudaSuccess)
        return MOE_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof v) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (clear) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(g_dev_error, &z, sizeof z) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    return (moe_status_t)v;
}

__attribute__((visibility("default"))) moe_status_t moe_debug_bounded_wait(uint64_t timeout_ns,
                                                                           moe_stream_t stream)
{
    if (timeout_ns == 0 || timeout_ns > 10ull * 1000000000ull)
        return MOE_ERR_INVALID_ARG;
    bounded_wait_probe_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return launch_status();
}

}  // extern "C"

// ================================================================ dispatch without a workspace
//
// Scratch of moe_dispatch_static: one fixed array per device. Host code never uses the
// symbol itself as an address (on the host it is only a stand-in); the device address is
// looked up with cudaGetSymbolAddress while that device is current, once per device and
// context: the cache is keyed on the current context's unique id, so after a
// cudaDeviceReset (which destroys the context and, with it, the module holding the array)
// the next call looks the address up again instead of using a stale one.

static __device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_addr[kMaxDevices];
unsigned long long g_static_ctx[kMaxDevices];  // context id the cached address belongs to

// Unique id of the calling thread's current CUDA context (0 when none is current or the
// driver does not provide ids).
unsigned long long current_context_id()
{
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
        get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}

moe_status_t static_scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_static_addr[dev] || ctx == 0 || ctx != g_static_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p)
            return MOE_ERR_CUDA;
        g_static_addr[dev] = p;
        // the lookup made the device's primary context current if none was
        g_static_ctx[dev] = current_context_id();
    }
    *out = g_static_addr[dev];
    return MOE_OK;
}

struct StaticLayout {
    size_t ctl, agg, incl, pk_base, moved, D, pk_off, pk_of, total;
};

StaticLayout static_layout(const moe_shape_t *s, const Geometry &g)
{
    StaticLayout L;
    L.total = dispatch_scratch(s, g, 0, L, false);
    return L;
}

}  // namespace

extern "C" __attribute__((visibility("default"))) moe_status_t
moe_dispatch_static(const moe_shape_t *shape, const uint16_t *x, const int32_t *topk_idx,
                    int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *row_of,
                    int32_t *assign_of_row, uint16_t *x_sorted, uint16_t *x_packed,
                    int64_t *rank_matrix, int64_t *packed_offsets, moe_stats_t *stats,
                    moe_stream_t stream)
{
    Geometry g;
    moe_status_t rc = check_shape(shape, false, &g);
    if (rc != MOE_OK)
        return rc;
    if (shape->N == 0)
        return empty_dispatch(shape, counts, kept, offsets, rank_matrix, packed_offsets, stats,
                              reinterpret_cast<cudaStream_t>(stream));
    if (g.rounds > 1)  // re-routing needs the logits
        return MOE_ERR_INVALID_ARG;
    if (!x || !topk_idx || !counts || !kept || !offsets || !row_of || !assign_of_row || !x_sorted)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_sorted) || (x_packed && !aligned16(x_packed)) ||
        !aligned4(topk_idx) || !aligned4(counts) || !aligned4(kept) || !aligned4(offsets) ||
        !aligned4(row_of) || !aligned4(assign_of_row) ||
        (rank_matrix && (reinterpret_cast<uintptr_t>(rank_matrix) & 7u)) ||
        (packed_offsets && (reinterpret_cast<uintptr_t>(packed_offsets) & 7u)) ||
        (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return MOE_ERR_MISALIGNED;
    const StaticLayout L = static_layout(shape, g);
    if (L.total > MOE_STATIC_SCRATCH_BYTES)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    void *base = nullptr;
    rc = static_scratch_address(&base);
    if (rc != MOE_OK)
        return rc;
    char *w = static_cast<char *>(base);
    int64_t *D = rank_matrix ? rank_matrix : reinterpret_cast<int64_t *>(w + L.D);
    int64_t *pk = packed_offsets ? packed_offsets : reinterpret_cast<int64_t *>(w + L.pk_off);
    return dispatch_impl(shape, g, x, nullptr, topk_idx, counts, kept, offsets, row_of,
                         assign_of_row, nullptr,
                         Payload{x_sorted, x_packed, false, nullptr, nullptr}, D, pk, stats,
                         scratch_at(w, L), reinterpret_cast<cudaStream_t>(stream));
}
