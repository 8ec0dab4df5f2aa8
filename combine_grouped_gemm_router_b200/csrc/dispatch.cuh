// Dispatch permutation: per-block expert histogram -> scan over blocks (with
// capacity, offsets, traffic matrix and pack bases) -> stable positions and the
// token<->row mapping table -> 16-byte row scatter.
//
// [MoE 推理服务工程真相 2026, §2.3 moe_dispatch pseudo-code] bincount of the expert
// ids and an overflow mask against the capacity; [§2.2] overflow is dropped.
// [MoE Inference Communication, §DeepSpeed-MoE › MoE 计算核优化] cumsum (a
// parallel scan) and scatter through a dense token->expert mapping table
// instead of a one-hot einsum. [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All
// 分发与回收的机制] rows are packed by destination card before the exchange.
//
// Positions follow a priority order over the N*K assignments: token-major
// ((t, k), a = t*K + k ascending) or slot-major ((k, t): every token's first
// choice before any second choice). The dispatch walks that order as "virtual
// blocks": token-major block b covers the K slots of HB tokens; slot-major block
// (k, b) covers slot k of the same HB tokens. Blocks never straddle a home shard,
// so the order is cut into segments (one per home shard, or one per (slot,
// shard)) whose starts are block boundaries. A block's base per expert comes
// from the scan over blocks, ranks inside a block from per-warp counts and
// __match_any_sync, so the result is deterministic and equal to the sequential
// definition, with no global atomics.
//
// Re-routing of overflowed assignments ([MoE 推理服务工程真相 2026, §4.3] token
// drop: move to the next-best expert; [§2.3] the remapping of the overflow mask)
// runs the dispatch twice. The first pass walks round 0 (the routed experts) and
// finds the assignments past capacity; reroute_kernel picks each one's next-best
// expert that is outside the token's top-K and not full; the second pass walks
// round 0 followed by round 1 (the moved assignments at their new experts) as one
// priority sequence, so a moved assignment queues behind every first-round
// assignment of its new expert.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kDispatchHB = 64;  // tokens per dispatch block

// The dispatch's priority order, cut into virtual blocks: rounds of nvb_round
// blocks each (round 1 only when re-routing), each round in priority order.
struct VBlocks {
    BlockMap bm;
    int nblk_tok;           // token blocks (W * bps)
    int slot_major;         // 0: token-major (nblk_tok blocks a round); 1: slot-major (K * nblk_tok)
    int K;
    int nvb_round;          // virtual blocks per round
    const int32_t *moved;   // round 1's expert per assignment (-1: not moved), or null
    // tokens [t0, t1), slot k (slot-major), round of virtual block vb
    __device__ __forceinline__ void range(int vb, int &t0, int &t1, int &k, int &round) const
    {
        round = vb / nvb_round;
        vb -= round * nvb_round;
        k = slot_major ? vb / nblk_tok : 0;
        bm.range(slot_major ? vb - k * nblk_tok : vb, t0, t1);
    }
    __device__ __forceinline__ int count(int t0, int t1) const
    {
        return slot_major ? t1 - t0 : (t1 - t0) * K;
    }
    // the i-th assignment of the block
    __device__ __forceinline__ int assign(int t0, int k, int i) const
    {
        return slot_major ? (t0 + i) * K + k : t0 * K + i;
    }
    __device__ __forceinline__ const int32_t *experts(const int32_t *topk_idx, int round) const
    {
        return round ? moved : topk_idx;
    }
};

// Control words of one dispatch pass, zeroed before the pass: the ticket that hands out
// virtual blocks in launch order, the count of blocks finished, then one status flag per
// virtual block (0: nothing published; kFlagAgg: its histogram; kFlagIncl: its inclusive
// prefix over every earlier block of the priority order).
constexpr unsigned int kFlagAgg = 1;
constexpr unsigned int kFlagIncl = 2;

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p)
{
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(unsigned int *p, unsigned int v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct HistArgs {
    const int32_t *topk_idx;
    VBlocks vbm;
    int nvb;         // virtual blocks of the pass (all its rounds)
    int bps;         // virtual blocks per segment (segment g = blocks [g*bps, (g+1)*bps))
    int nseg;        // segments of the pass
    int nseg_round;  // segments of one round
    int N, E, K, W, C;
    unsigned int *ctl;  // [2 + nvb]: ticket, done, flags
    int32_t *agg;       // [nvb][E] the blocks' histograms
    int32_t *incl;      // [nvb][E] inclusive prefixes over the priority order
    // the pass's totals, written by the block that finishes last:
    int32_t *counts, *kept, *offsets;
    int64_t *D;        // [W][W]
    int64_t *pk_off;   // [W*W+1]
    int64_t *pk_base;  // [nseg][E]
    moe_stats_t *stats;
    uint64_t timeout_ns;
};

// Assignments to expert e before segment g in priority order (g = nseg: the pass's total).
__device__ __forceinline__ int seg_cum(const HistArgs &p, int e, int g)
{
    if (g >= p.nseg)
        return __ldcg(p.incl + (size_t)(p.nvb - 1) * p.E + e);
    const size_t o = (size_t)g * p.bps * p.E + e;
    return __ldcg(p.incl + o) - __ldcg(p.agg + o);
}

// In-place exclusive scan of a[0..n) in shared memory by the whole block of NT threads;
// a[n] receives the total. s_warp needs 32 entries.
template <int NT>
__device__ void block_excl_scan_i64(int64_t *a, int n, int64_t *s_warp)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (n + NT - 1) / NT;
    const int beg = min(n, (int)threadIdx.x * per), end = min(n, beg + per);
    int64_t local = 0;
    for (int i = beg; i < end; ++i)
        local += a[i];
    const int64_t incl = warp_incl_scan(local);
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int64_t w = lane < NT / 32 ? s_warp[lane] : 0;
        const int64_t wi = warp_incl_scan(w);
        if (lane < NT / 32)
            s_warp[lane] = wi - w;
    }
    __syncthreads();
    int64_t run = s_warp[warp] + incl - local;
    for (int i = beg; i < end; ++i) {
        const int64_t v = a[i];
        a[i] = run;
        run += v;
    }
    if (n == 0 && threadIdx.x == 0)
        a[0] = 0;
    else if (beg < end && end == n)
        a[n] = run;
    __syncthreads();
}

constexpr int kHistThreads = 256;

// Shared memory of dispatch_hist_kernel: the block's histogram, then (for the block that
// finishes last) s_a [max(E, W*W) + 1] int64, s_D [W*W] int64, s_warp [32] int64, s_kh [E][W]
// int32 (kept rows of expert e from home shard i) and, when (G + 1) E <= kCumCacheInts, s_cum
// [G + 1][E] int32: every segment-start prefix the totals read, loaded once, all at a time.
constexpr int kCumCacheInts = 16384;

__host__ __device__ inline bool cum_cached(int E, int G) { return (size_t)(G + 1) * E <= kCumCacheInts; }

__host__ __device__ inline size_t hist_smem_bytes(int E, int W, int G)
{
    const size_t scan = ((size_t)(E > W * W ? E : W * W) + 1) * 8 + (size_t)W * W * 8 + 32 * 8 +
                        (size_t)E * W * 4 + (cum_cached(E, G) ? (size_t)(G + 1) * E * 4 : 0);
    const size_t hist = (size_t)E * 4;
    return scan > hist ? scan : hist;
}

// The pass's totals, from the prefixes every block published (the block that finished last
// runs this): counts (routed demand: round 0's total), kept = min(total, C), offsets (scan of
// kept), the traffic matrix D, the pack offsets and the pack base of every (segment, expert),
// and the counters. Segment g belongs to home shard g % W; within one home shard its
// segments come in priority order, so the kept rows of expert e from that shard are a prefix
// of the shard's own sequence of assignments to e.
__device__ void pass_totals(const HistArgs &p, unsigned char *smem)
{
    constexpr int NT = kHistThreads;
    const int E = p.E, W = p.W, G = p.nseg;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t C = p.C;
    const int scan_len = max(E, W * W) + 1;
    int64_t *s_a = reinterpret_cast<int64_t *>(smem);
    int64_t *s_D = s_a + scan_len;
    int64_t *s_warp = s_D + W * W;
    int32_t *s_kh = reinterpret_cast<int32_t *>(s_warp + 32);
    int32_t *s_cum = s_kh + E * W;
    const bool cached = cum_cached(E, G);
    if (cached) {
#pragma unroll 4
        for (int i = threadIdx.x; i < (G + 1) * E; i += NT)
            s_cum[i] = seg_cum(p, i % E, i / E);
        __syncthreads();
    }
    auto cum = [&](int e, int g) { return cached ? s_cum[g * E + e] : seg_cum(p, e, g); };

    for (int e = threadIdx.x; e < E; e += NT) {
        const int kp = (int)min((int64_t)cum(e, G), C);
        p.counts[e] = cum(e, p.nseg_round);
        p.kept[e] = kp;
        s_a[e] = kp;
    }
    for (int ei = threadIdx.x; ei < E * W; ei += NT) {
        const int e = ei / W, i = ei % W;
        int64_t s = 0;
        for (int g = i; g < G; g += W)
            s += min((int64_t)cum(e, g + 1), C) - min((int64_t)cum(e, g), C);
        s_kh[ei] = (int32_t)s;
    }
    __syncthreads();
    block_excl_scan_i64<NT>(s_a, E, s_warp);
    for (int e = threadIdx.x; e <= E; e += NT)
        p.offsets[e] = (int32_t)s_a[e];
    __syncthreads();

    // traffic matrix D[i][j] = kept rows of experts on rank j from shard i
    const int e_per = E / W;
    for (int ij = threadIdx.x; ij < W * W; ij += NT) {
        const int i = ij / W, j = ij % W;
        int64_t s = 0;
        for (int e = j * e_per; e < (j + 1) * e_per; ++e)
            s += s_kh[e * W + i];
        s_D[ij] = s;
        p.D[ij] = s;
    }
    __syncthreads();
    for (int ij = threadIdx.x; ij < W * W; ij += NT)
        s_a[ij] = s_D[ij];
    __syncthreads();
    block_excl_scan_i64<NT>(s_a, W * W, s_warp);
    for (int ij = threadIdx.x; ij <= W * W; ij += NT)
        p.pk_off[ij] = s_a[ij];

    // pack bases: a kept assignment to expert e at position pos (in e's rows) from segment g
    // lands on packed row pk_base[g][e] + pos. Block (i, j) holds its experts in order, each
    // expert's rows from shard i in the shard's own order: the earlier segments of shard i
    // come first.
    for (int ei = threadIdx.x; ei < E * W; ei += NT) {
        const int e = ei / W, i = ei % W;
        const int j = e / e_per;
        int64_t base = s_a[i * W + j];
        for (int e2 = j * e_per; e2 < e; ++e2)
            base += s_kh[e2 * W + i];
        int64_t run = 0;
        for (int g = i; g < G; g += W) {
            const int c0 = cum(e, g);
            p.pk_base[(size_t)g * E + e] = base + run - c0;
            run += cum(e, g + 1) - c0;
        }
    }

    // counters (dedup_pairs is added by the placement kernel)
    if (p.stats && warp == 0) {
        int mx = 0, mn = 0x7fffffff, act = 0;
        int64_t first = 0;  // rows from round 0
        for (int e = lane; e < E; e += 32) {
            const int kp = (int)min((int64_t)cum(e, G), C);
            mx = max(mx, kp);
            mn = min(mn, kp);
            act += kp > 0;
            first += min((int64_t)cum(e, p.nseg_round), C);
        }
        first = warp_sum(first);
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            act += __shfl_xor_sync(0xffffffffu, act, off);
        }
        int64_t diag = 0;
        for (int i = lane; i < W; i += 32)
            diag += s_D[i * W + i];
        diag = warp_sum(diag);
        if (lane == 0) {
            const int64_t R = s_a[W * W];  // total of D == R
            p.stats->rows = R;
            p.stats->dropped = (int64_t)p.N * p.K - R;
            p.stats->cross_rows = R - diag;
            p.stats->dedup_pairs = 0;
            p.stats->capacity = p.C;
            p.stats->active_experts = act;
            p.stats->max_kept = mx;
            p.stats->min_kept = mn;
            p.stats->rerouted = R - first;
        }
    }
}

// One CTA per virtual block, taken in launch order from a ticket: the block's expert
// histogram, published; its exclusive prefix over all earlier blocks of the priority order
// by a decoupled look-back (each thread walks back over its expert's column: a predecessor
// that published its inclusive prefix ends the walk, one that published only its histogram
// adds it and the walk goes on), published as the inclusive prefix; the block that finishes
// last then forms the pass's totals. A block only ever waits for blocks that took earlier
// tickets, which are resident or done, so the waits end; each is bounded all the same
// (MOE_ERR_DEVICE_TIMEOUT). The scan stays deterministic: positions are exact counts.
__global__ void __launch_bounds__(kHistThreads, 4) dispatch_hist_kernel(HistArgs p)
{
    extern __shared__ __align__(16) unsigned char hist_smem[];
    int *s_hist = reinterpret_cast<int *>(hist_smem);
    __shared__ int s_vb, s_last, s_stop;
    const int E = p.E;
    if (threadIdx.x == 0)
        s_vb = (int)atomicAdd(&p.ctl[0], 1u);
    for (int e = threadIdx.x; e < E; e += kHistThreads)
        s_hist[e] = 0;
    __syncthreads();
    const int vb = s_vb;
    int t0, t1, k, round;
    p.vbm.range(vb, t0, t1, k, round);
    const int32_t *src = p.vbm.experts(p.topk_idx, round);
    const int n = p.vbm.count(t0, t1);
    for (int i = threadIdx.x; i < n; i += kHistThreads) {
        const int e = src[p.vbm.assign(t0, k, i)];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&s_hist[e], 1);
        else if (round == 0)
            set_dev_error(MOE_ERR_DEVICE_BOUNDS);  // round 1 marks "not moved" with -1
    }
    __syncthreads();
    unsigned int *flags = p.ctl + 2;
    for (int e = threadIdx.x; e < E; e += kHistThreads)
        p.agg[(size_t)vb * E + e] = s_hist[e];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        st_release_u32(&flags[vb], kFlagAgg);
    // look-back in windows of 32 predecessors: warp 0 reads their flags at once (waiting, with
    // a bound, for any that has not published yet) and finds the nearest one whose inclusive
    // prefix is out; every thread then adds its expert's histograms of the blocks after that
    // one (and that prefix), or of the whole window and the walk goes on.
    int excl[(256 + kHistThreads - 1) / kHistThreads] = {};  // one per expert of this thread
    int cur = vb;
    while (cur > 0) {
        const int lo = max(0, cur - 32);
        if (threadIdx.x < 32) {
            const int q = cur - 1 - (int)threadIdx.x;
            unsigned int f = kFlagIncl;
            if (q >= lo) {
                f = ld_acquire_u32(&flags[q]);
                if (f == 0) {
                    const uint64_t w0 = global_timer_ns();
                    while ((f = ld_acquire_u32(&flags[q])) == 0) {
                        if (global_timer_ns() - w0 > p.timeout_ns) {
                            set_dev_error(MOE_ERR_DEVICE_TIMEOUT);
                            f = kFlagIncl;  // give up on it (the error is recorded)
                            break;
                        }
                    }
                }
            }
            const unsigned incl_mask = __ballot_sync(0xffffffffu, q >= lo && f == kFlagIncl);
            if (threadIdx.x == 0)
                s_stop = incl_mask ? cur - 1 - (__ffs(incl_mask) - 1) : -1;
        }
        __syncthreads();
        const int stop = s_stop;  // the nearest block with its inclusive prefix out, or -1
        const int from = stop >= 0 ? stop + 1 : lo;
        int j = 0;
        for (int e = threadIdx.x; e < E; e += kHistThreads, ++j) {
            // the window's (at most 32) histograms: every load issued before the first add
            int part[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                part[i] = from + i < cur ? __ldcg(p.agg + (size_t)(from + i) * E + e) : 0;
            int acc = stop >= 0 ? __ldcg(p.incl + (size_t)stop * E + e) : 0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                acc += part[i];
            excl[j] += acc;
        }
        __syncthreads();  // s_stop is read by every thread before it is written again
        if (stop >= 0)
            break;
        cur = lo;
    }
    {
        int j = 0;
        for (int e = threadIdx.x; e < E; e += kHistThreads, ++j)
            p.incl[(size_t)vb * E + e] = excl[j] + s_hist[e];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        st_release_u32(&flags[vb], kFlagIncl);
        __threadfence();
        s_last = atomicAdd(&p.ctl[1], 1u) == (unsigned int)(p.nvb - 1);
    }
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    pass_totals(p, hist_smem);
}

constexpr int kPlaceThreads = 256;

struct PlaceArgs {
    const int32_t *topk_idx;
    VBlocks vbm;
    int rounds;
    int bps;          // virtual blocks per segment (a token block's segment: vb / bps)
    int E, K, W, C;
    const int32_t *agg, *incl;  // [nvb][E]
    const int32_t *offsets;     // [E+1]
    const int64_t *pk_base;     // [nseg][E]
    int32_t *row_of, *assign_of_row;
    int32_t *expert_of;         // nullable: the expert whose row each assignment uses, or -1
    int32_t *packed_row_of;     // nullable: each assignment's packed row, or -1
    // W real ranks: this process is rank `rank` (home shard `rank`), -1 for the whole batch on
    // one GPU. Then only the home shard's rows are copied, x holds just those tokens (token t
    // at row t - x_row0), and packed row p goes to x_packed row p - pk_off[rank W] (the start of
    // its block row); send_row_of (nullable) receives, per slot of the home shard's tokens,
    // that same row or -1.
    int rank;
    int x_row0;
    const int64_t *pk_off;  // [W*W+1]: the pack offsets the totals kernel wrote
    int32_t *send_row_of;
    // the copy of the rows (copy != 0)
    int copy;
    int e4m3;
    const uint16_t *x;
    int d;
    void *x_sorted, *x_packed;          // bf16 rows, or e4m3 rows with the FP8 payload
    float *sorted_scale, *packed_scale;  // FP8 payload: one scale per row
    moe_stats_t *stats;                  // nullable: dedup_pairs is accumulated here
    int slots;                           // bf16 copy: ring slots per warp (1 to 3)
    uint64_t timeout_ns;                 // bound of every wait of the bulk copy
};

// Shared memory of dispatch_place_kernel: per-warp counts [8][E] and offsets [E+1] (int32),
// then the expert-sorted row, the packed row and the expert of each of the token block's
// HB * K slots (int32 each).
__host__ __device__ inline size_t place_smem_bytes(int E, int K)
{
    return ((size_t)9 * E + 1 + (size_t)3 * kDispatchHB * K) * 4;
}

// The bf16 rows move by bulk copies (cp.async.bulk) in pieces of at most kPiece bytes: global
// -> a shared-memory ring slot (one mbarrier per slot) -> every kept destination row. The ring
// follows the tables above (128-byte aligned): per warp `slots` pieces, then the mbarriers.
constexpr int kPiece = 4096;

__host__ __device__ inline size_t place_ring_offset(int E, int K)
{
    return (place_smem_bytes(E, K) + 127) & ~(size_t)127;
}

__host__ __device__ inline size_t place_smem_total(int E, int K, int slots)
{
    return place_ring_offset(E, K) + (size_t)8 * slots * kPiece + (size_t)8 * slots * 8;
}

__device__ __forceinline__ void bulk_store_s2g(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}

// Bulk copy of a token block's bf16 rows (the share of part `part` of `parts`): the block's
// items are (token, piece) pairs, q = lt * npc + piece; warp w takes q = part + parts * (w + 8 j)
// of the tokens that keep a slot. Per warp a pipeline over its items: the piece of item c + 1
// is loaded into its ring slot while item c's stores go out (lane k < K stores slot k's
// expert-sorted row and, when it has one, its packed row), with up to S - 1 items' stores in
// flight; a slot is reloaded only once the stores that read it have read it. xb: the block's
// first token row; s_rk / s_pk: each slot's sorted / packed row or -1 (shared memory); ring_smem:
// 8 warps x S slots of kPiece bytes, then 8 x S mbarriers. Every wait is bounded.
__device__ void copy_rows_bulk(const uint16_t *xb, int nt, int K, const int *s_rk, const int *s_pk,
                               void *x_sorted, void *x_packed, int d, int part, int parts,
                               unsigned char *ring_smem, int S, uint64_t timeout_ns)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t rb = (uint32_t)d * 2u;
    const int npc = (int)((rb + kPiece - 1) / kPiece);
    const int nq = nt * npc, qstep = parts * 8;
    const uint32_t ring = smem_u32(ring_smem) + warp * S * kPiece;
    const uint32_t bars = smem_u32(ring_smem) + 8 * S * kPiece + warp * S * 8;
    if (lane == 0) {
        for (int j = 0; j < S; ++j)
            mbar_init(bars + 8 * j, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    // the next item at or after q whose token keeps a slot (nq: none)
    auto next_item = [&](int q) {
        for (; q < nq; q += qstep) {
            const int lt = q / npc;
            if (__any_sync(0xffffffffu, lane < K && s_rk[lt * K + lane] >= 0))
                break;
        }
        return q < nq ? q : nq;
    };
    auto issue_load = [&](int q, int slot) {
        if (lane == 0) {
            const int lt = q / npc, pc = q - lt * npc;
            const uint32_t bytes = min((uint32_t)kPiece, rb - (uint32_t)pc * kPiece);
            const unsigned char *src = reinterpret_cast<const unsigned char *>(xb) +
                                       (size_t)lt * rb + (size_t)pc * kPiece;
            mbar_arrive_expect_tx(bars + 8 * slot, bytes);
            bulk_load_g2s(ring + slot * kPiece, src, bytes, bars + 8 * slot);
        }
    };
    auto wait_read = [&](int pending) {  // this lane's store groups beyond `pending` read
        if (pending <= 0)
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        else
            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
    };
    unsigned char *dst_s = reinterpret_cast<unsigned char *>(x_sorted);
    unsigned char *dst_p = reinterpret_cast<unsigned char *>(x_packed);
    int q_cur = next_item(part + parts * warp);
    int c = 0;          // items whose stores have been issued
    int loaded = -1;    // the last item index whose load was issued
    if (q_cur < nq) {
        issue_load(q_cur, 0);
        loaded = 0;
    }
    while (q_cur < nq) {
        const int q_nxt = next_item(q_cur + qstep);
        if (S > 1 && q_nxt < nq) {  // load item c + 1 (its slot's earlier stores read)
            wait_read(S - 2);
            __syncwarp();
            issue_load(q_nxt, (c + 1) % S);
            loaded = c + 1;
        }
        const int slot = c % S;
        if (!mbar_wait_bounded(bars + 8 * slot, (uint32_t)((c / S) & 1), timeout_ns))
            break;
        const int lt = q_cur / npc, pc = q_cur - lt * npc;
        const uint32_t bytes = min((uint32_t)kPiece, rb - (uint32_t)pc * kPiece);
        const size_t off = (size_t)pc * kPiece;
        if (lane < K) {  // x_sorted is null for a rank's dispatch (send rows only)
            const int rk = s_rk[lt * K + lane];
            if (rk >= 0) {
                if (dst_s)
                    bulk_store_s2g(dst_s + (size_t)rk * rb + off, ring + slot * kPiece, bytes);
                const int pk = s_pk[lt * K + lane];
                if (pk >= 0)
                    bulk_store_s2g(dst_p + (size_t)pk * rb + off, ring + slot * kPiece, bytes);
            }
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        ++c;
        if (S == 1 && q_nxt < nq) {  // one slot: reload it once this item's stores read it
            wait_read(0);
            __syncwarp();
            issue_load(q_nxt, 0);
            loaded = c;
        }
        q_cur = q_nxt;
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    // loads issued and not consumed (only after a wait that ran out): let them land first
    if (lane == 0)
        for (int j = c; j <= loaded; ++j)
            mbar_wait_bounded(bars + 8 * (j % S), (uint32_t)((j / S) & 1), timeout_ns);
    __syncwarp();
}

// Bulk copy by destination row, for a balanced split whatever the routing: warp gw of nw takes
// a contiguous range of the (row, piece) items of the R expert-sorted rows; row r copies token
// assign_of_row[r] / K's piece to x_sorted row r and, when there is a packed buffer, to packed
// row pk_of[assign_of_row[r]]. A token row is read once per kept slot (from L2 after the first).
// The items' rows are looked up 32 at a time (lane l the l-th item of a batch, the next batch
// loaded while this one is copied); the copy pipeline is copy_rows_bulk's. ring / bars: this
// warp's S slots of kPiece bytes and its S mbarriers (shared-memory addresses).
__device__ void copy_rows_by_row(const uint16_t *x, const int32_t *assign_of_row,
                                 const int32_t *pk_of, int R, int K, void *x_sorted, void *x_packed,
                                 int d, int gw, int nw, uint32_t ring, uint32_t bars, int S,
                                 uint64_t timeout_ns)
{
    const int lane = threadIdx.x & 31;
    const uint32_t rb = (uint32_t)d * 2u;
    const int npc = (int)((rb + kPiece - 1) / kPiece);
    const long long nq = (long long)R * npc;
    const long long per = (nq + nw - 1) / nw;
    const long long q0 = min(nq, (long long)gw * per), q1 = min(nq, q0 + per);
    const int n = (int)(q1 - q0);
    if (lane == 0) {
        for (int j = 0; j < S; ++j)
            mbar_init(bars + 8 * j, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (n <= 0)
        return;
    // item j of the range: lane j % 32 of batch j / 32 holds its token row and packed row
    auto fetch = [&](int batch, int &tok, int &pk) {
        const int j = batch * 32 + lane;
        tok = -1;
        pk = -1;
        if (j < n) {
            const int r = (int)((q0 + j) / npc);
            const int a = __ldcg(assign_of_row + r);
            tok = a / K;
            if (x_packed)
                pk = __ldcg(pk_of + a);
        }
    };
    int cur_t, cur_p, nxt_t, nxt_p;
    fetch(0, cur_t, cur_p);
    fetch(1, nxt_t, nxt_p);
    auto info = [&](int j, int &tok, int &pk) {  // j in the current or the next batch
        const bool in_next = (j >> 5) != 0;
        const int t_src = in_next ? nxt_t : cur_t, p_src = in_next ? nxt_p : cur_p;
        tok = __shfl_sync(0xffffffffu, t_src, j & 31);
        pk = __shfl_sync(0xffffffffu, p_src, j & 31);
    };
    auto piece = [&](int j, uint32_t &off, uint32_t &bytes) {
        const int pc = (int)((q0 + j) % npc);
        off = (uint32_t)pc * kPiece;
        bytes = min((uint32_t)kPiece, rb - off);
    };
    auto issue_load = [&](int j, int jb) {  // item j (index jb inside the held batches)
        int tok, pk;
        info(jb, tok, pk);
        uint32_t off, bytes;
        piece(j, off, bytes);
        const int slot = j % S;
        if (lane == 0) {
            mbar_arrive_expect_tx(bars + 8 * slot, bytes);
            bulk_load_g2s(ring + slot * kPiece,
                          reinterpret_cast<const unsigned char *>(x) + (size_t)tok * rb + off,
                          bytes, bars + 8 * slot);
        }
    };
    auto wait_read = [&](int pending) {
        if (pending <= 0)
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        else
            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
    };
    unsigned char *dst_s = reinterpret_cast<unsigned char *>(x_sorted);
    unsigned char *dst_p = reinterpret_cast<unsigned char *>(x_packed);
    int loaded = 0, c = 0;
    issue_load(0, 0);
    for (; c < n; ++c) {
        if ((c & 31) == 0 && c > 0) {  // the next batch becomes the current one
            cur_t = nxt_t;
            cur_p = nxt_p;
            fetch((c >> 5) + 1, nxt_t, nxt_p);
        }
        const int cb = c & 31;
        if (S > 1 && c + 1 < n) {
            wait_read(S - 2);
            __syncwarp();
            issue_load(c + 1, cb + 1);
            loaded = c + 1;
        }
        const int slot = c % S;
        if (!mbar_wait_bounded(bars + 8 * slot, (uint32_t)((c / S) & 1), timeout_ns))
            break;
        int tok, pk;
        info(cb, tok, pk);
        uint32_t off, bytes;
        piece(c, off, bytes);
        const long long r = (q0 + c) / npc;
        if (lane == 0)
            bulk_store_s2g(dst_s + (size_t)r * rb + off, ring + slot * kPiece, bytes);
        else if (lane == 1 && pk >= 0)
            bulk_store_s2g(dst_p + (size_t)pk * rb + off, ring + slot * kPiece, bytes);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        if (S == 1 && c + 1 < n) {
            wait_read(0);
            __syncwarp();
            issue_load(c + 1, cb + 1);
            loaded = c + 1;
        }
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    if (lane == 0)
        for (int j = c; j <= loaded; ++j)
            mbar_wait_bounded(bars + 8 * (j % S), (uint32_t)((j / S) & 1), timeout_ns);
    __syncwarp();
}

// ---------------------------------------------------------------------------
// The dispatch pass in one kernel (one round, bf16 rows or no copy), for grids that fit on the
// GPU at once (cooperative launch). CTA (token block tb, part):
//  1. the block's top-K slice into shared memory; per virtual block of the token block (one,
//     or K slot-major), per-warp expert counts and each assignment's rank among the block's
//     assignments to its expert (first come first placed: per-warp bases, then
//     __match_any_sync inside the warp), and part 0 publishes the block's histogram;
//  2. one grid barrier (an arrival count, bounded wait);
//  3. every CTA loads all the histograms (shared memory), scans each expert's column (in
//     parallel over segments of blocks, then a second pass), and so knows its own blocks'
//     prefixes, the prefix at every segment start and the totals; from these, like the
//     totals of the two-kernel pass: kept = min(total, C), offsets, the kept rows of every
//     (expert, home shard), D, the pack offsets and its own blocks' pack bases. CTA (0, 0)
//     writes them out;
//  4. positions = block prefix + rank: the mapping table (part 0) and the dedup counter;
//  5. the bulk copy of its share of the block's rows (copy_rows_bulk).
// No position needs a second walk over the top-K, and the histograms are read once per CTA
// from L2. The arithmetic is the two-kernel pass's, so the results are the same bits.
struct FusedArgs {
    const int32_t *topk_idx;
    VBlocks vbm;  // one round
    int nvb, bps, nseg;
    int N, E, K, W, C;
    unsigned int *ctl;  // [0]: arrivals at the grid barrier (zeroed before the launch)
    int32_t *agg;       // [nvb][E]
    int32_t *counts, *kept, *offsets;
    int64_t *D, *pk_off;
    int32_t *row_of, *assign_of_row, *expert_of, *packed_row_of;
    int32_t *pk_of;  // nullable scratch [N*K]: each slot's packed row (for the copy by row)
    int rank, x_row0;
    int32_t *send_row_of;
    int copy;
    const uint16_t *x;
    int d;
    void *x_sorted, *x_packed;
    moe_stats_t *stats;
    int slots;
    uint64_t timeout_ns;
};

// Shared-memory layout of dispatch_fused_kernel (bytes from the start).
struct FusedLayout {
    size_t wcnt, off, e, lr, rk, pk, ex, base, cum, kh, part, a64, warp64, D, pko, pkb, uni, total;
};

__host__ __device__ inline FusedLayout fused_layout(int E, int K, int W, int nvb, int nseg, int nsub,
                                                    int slots)
{
    FusedLayout L;
    size_t o = 0;
    auto take = [&](size_t bytes, size_t align) {
        o = (o + align - 1) / align * align;
        const size_t at = o;
        o += bytes;
        return at;
    };
    const size_t slots_b = (size_t)kDispatchHB * K * 4;
    L.wcnt = take((size_t)8 * E * 4, 16);
    L.off = take((size_t)(E + 1) * 4, 16);
    L.e = take(slots_b, 16);
    L.lr = take(slots_b, 16);
    L.rk = take(slots_b, 16);
    L.pk = take(slots_b, 16);
    L.ex = take(slots_b, 16);
    L.base = take((size_t)nsub * E * 4, 16);
    L.cum = take((size_t)(nseg + 1) * E * 4, 16);
    L.kh = take((size_t)E * W * 4, 16);
    L.part = take(256 * 4, 16);
    L.a64 = take((size_t)((E > W * W ? E : W * W) + 1) * 8, 16);
    L.warp64 = take(32 * 8, 16);
    L.D = take((size_t)W * W * 8, 16);
    L.pko = take((size_t)(W * W + 1) * 8, 16);
    L.pkb = take((size_t)nsub * E * 8, 16);
    // the histograms of every block (phase 3), then the copy ring (phase 5), in one region
    const size_t ring = (size_t)8 * slots * kPiece + (size_t)8 * slots * 8;
    const size_t aggs = (size_t)nvb * E * 4;
    L.uni = take(ring > aggs ? ring : aggs, 128);
    L.total = o;
    return L;
}

__global__ void __launch_bounds__(kPlaceThreads) dispatch_fused_kernel(FusedArgs p)
{
    extern __shared__ __align__(128) unsigned char fz[];
    constexpr int NT = kPlaceThreads;
    const int E = p.E, K = p.K, W = p.W;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tb = blockIdx.x, part = blockIdx.y, parts = gridDim.y;
    const bool lead = tb == 0 && part == 0;
    const int nsub = p.vbm.slot_major ? K : 1;
    const FusedLayout L = fused_layout(E, K, W, p.nvb, p.nseg, nsub, p.slots);
    int *wcnt = reinterpret_cast<int *>(fz + L.wcnt);
    int *s_off = reinterpret_cast<int *>(fz + L.off);
    int *s_e = reinterpret_cast<int *>(fz + L.e);
    int *s_lr = reinterpret_cast<int *>(fz + L.lr);
    int *s_rk = reinterpret_cast<int *>(fz + L.rk);
    int *s_pk = reinterpret_cast<int *>(fz + L.pk);
    int *s_ex = reinterpret_cast<int *>(fz + L.ex);
    int *s_base = reinterpret_cast<int *>(fz + L.base);
    int *s_cum = reinterpret_cast<int *>(fz + L.cum);
    int *s_kh = reinterpret_cast<int *>(fz + L.kh);
    int *s_part = reinterpret_cast<int *>(fz + L.part);
    int64_t *s_a = reinterpret_cast<int64_t *>(fz + L.a64);
    int64_t *s_warp = reinterpret_cast<int64_t *>(fz + L.warp64);
    int64_t *s_D = reinterpret_cast<int64_t *>(fz + L.D);
    int64_t *s_pko = reinterpret_cast<int64_t *>(fz + L.pko);
    int64_t *s_pkb = reinterpret_cast<int64_t *>(fz + L.pkb);
    int *s_agg = reinterpret_cast<int *>(fz + L.uni);
    __shared__ int s_ok, s_dropped;

    int t0, t1;
    p.vbm.bm.range(tb, t0, t1);
    const int nt = t1 - t0;
    unsigned lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));

    // 1. the block's experts, ranks inside each virtual block, histograms
    for (int i = tid; i < nt * K; i += NT) {
        const int e = p.topk_idx[(size_t)t0 * K + i];
        const bool ok = (unsigned)e < (unsigned)E;
        if (!ok && part == 0)
            set_dev_error(MOE_ERR_DEVICE_BOUNDS);
        s_e[i] = ok ? e : -1;
        s_rk[i] = -1;
        s_pk[i] = -1;
        s_ex[i] = -1;
    }
    if (lead && tid == 0 && p.stats)
        p.stats->dedup_pairs = 0;  // before the barrier: every CTA adds to it after
    for (int kk = 0; kk < nsub; ++kk) {
        const int vb = (p.vbm.slot_major ? kk * p.vbm.nblk_tok : 0) + tb;
        const int na = p.vbm.count(t0, t1);
        const int per = (na + 7) / 8;
        const int wb = min(na, warp * per), we = min(na, wb + per);
        for (int i = tid; i < 8 * E; i += NT)
            wcnt[i] = 0;
        __syncthreads();
        for (int i = wb + lane; i < we; i += 32) {
            const int e = s_e[p.vbm.assign(t0, kk, i) - t0 * K];
            if (e >= 0)
                atomicAdd(&wcnt[warp * E + e], 1);
        }
        __syncthreads();
        for (int e = tid; e < E; e += NT) {
            int run = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const int c = wcnt[w * E + e];
                wcnt[w * E + e] = run;
                run += c;
            }
            if (part == 0)
                p.agg[(size_t)vb * E + e] = run;
        }
        __syncthreads();
        for (int g0 = wb; g0 < we; g0 += 32) {
            const int i = g0 + lane;
            const bool act = i < we;
            const int ls = act ? p.vbm.assign(t0, kk, i) - t0 * K : 0;
            const int e = act ? s_e[ls] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rk = __popc(peers & lt_mask);
            const int base = e >= 0 ? wcnt[warp * E + e] : 0;
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1)
                wcnt[warp * E + e] = base + __popc(peers);
            __syncwarp();
            if (act)
                s_lr[ls] = base + rk;
        }
        __syncthreads();
    }

    // 2. grid barrier
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned int n_cta = gridDim.x * gridDim.y;
        atomicAdd(&p.ctl[0], 1u);
        int ok = 1;
        if (ld_acquire_u32(&p.ctl[0]) < n_cta) {
            const uint64_t w0 = global_timer_ns();
            while (ld_acquire_u32(&p.ctl[0]) < n_cta) {
                if (global_timer_ns() - w0 > p.timeout_ns) {
                    set_dev_error(MOE_ERR_DEVICE_TIMEOUT);
                    ok = 0;
                    break;
                }
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    if (!s_ok)
        return;  // the histograms are incomplete: write nothing (the error is recorded)
    __threadfence();

    // 3. every block's histogram; column scans; totals
    const int nvE = p.nvb * E;
    {
        const int n4 = nvE >> 2;  // 16-byte pieces, every load in flight before the first store
        const int4 *src4 = reinterpret_cast<const int4 *>(p.agg);
        int4 *dst4 = reinterpret_cast<int4 *>(s_agg);
#pragma unroll 16
        for (int i = tid; i < n4; i += NT)
            dst4[i] = __ldcg(src4 + i);
        for (int i = 4 * n4 + tid; i < nvE; i += NT)
            s_agg[i] = __ldcg(p.agg + i);
    }
    __syncthreads();
    const int S = NT / E > 0 ? NT / E : 1;  // segments of blocks per expert column
    const int Lb = (p.nvb + S - 1) / S;
    const int col_e = tid % E, col_s = tid / E;
    const bool col = tid < S * E;
    const int lo = col ? min(p.nvb, col_s * Lb) : 0, hi = col ? min(p.nvb, lo + Lb) : 0;
    if (col) {  // pass 1: the segment's sum (8 loads in flight, then their adds)
        int sum = 0;
        for (int v0 = lo; v0 < hi; v0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = v0 + u < hi ? s_agg[(v0 + u) * E + col_e] : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                sum += v[u];
        }
        s_part[col_s * E + col_e] = sum;
    }
    __syncthreads();
    for (int e = tid; e < E; e += NT) {
        int run = 0;
        for (int q = 0; q < S; ++q) {
            const int v = s_part[q * E + e];
            s_part[q * E + e] = run;
            run += v;
        }
        s_cum[p.nseg * E + e] = run;
    }
    __syncthreads();
    if (col) {  // pass 2: prefixes at segment starts and at this CTA's own blocks
        int run = s_part[col_s * E + col_e];
        const int nb = p.vbm.nblk_tok;
        int to_seg = lo % p.bps;  // blocks since the last segment start
        int seg = lo / p.bps;
        // this CTA's next own block at or after lo: tb (+ k nb slot-major)
        int mine = p.vbm.slot_major ? (lo <= tb ? tb : tb + ((lo - tb + nb - 1) / nb) * nb)
                                    : (lo <= tb ? tb : 0x7fffffff);
        for (int v0 = lo; v0 < hi; v0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = v0 + u < hi ? s_agg[(v0 + u) * E + col_e] : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int vb = v0 + u;
                if (vb < hi) {
                    if (to_seg == 0)
                        s_cum[seg * E + col_e] = run;
                    if (vb == mine) {
                        s_base[(p.vbm.slot_major ? vb / nb : 0) * E + col_e] = run;
                        mine = p.vbm.slot_major ? mine + nb : 0x7fffffff;
                    }
                    run += v[u];
                    if (++to_seg == p.bps) {
                        to_seg = 0;
                        ++seg;
                    }
                }
            }
        }
    }
    __syncthreads();
    const int64_t C = p.C;
    const int G = p.nseg;
    for (int e = tid; e < E; e += NT)
        s_a[e] = min((int64_t)s_cum[G * E + e], C);
    if (warp == 0) {  // drops? (without them every token block keeps all its slots)
        int over = 0;
        for (int e = lane; e < E; e += 32)
            over |= s_cum[G * E + e] > p.C;
        over = __any_sync(0xffffffffu, over);
        if (lane == 0)
            s_dropped = over;
    }
    for (int ei = tid; ei < E * W; ei += NT) {
        const int e = ei / W, i = ei % W;
        int64_t sk = 0;
        for (int g = i; g < G; g += W)
            sk += min((int64_t)s_cum[(g + 1) * E + e], C) - min((int64_t)s_cum[g * E + e], C);
        s_kh[ei] = (int32_t)sk;
    }
    __syncthreads();
    block_excl_scan_i64<NT>(s_a, E, s_warp);
    for (int e = tid; e <= E; e += NT)
        s_off[e] = (int)s_a[e];
    __syncthreads();
    const int e_per = E / W;
    for (int ij = tid; ij < W * W; ij += NT) {
        const int i = ij / W, j = ij % W;
        int64_t sd = 0;
        for (int e = j * e_per; e < (j + 1) * e_per; ++e)
            sd += s_kh[e * W + i];
        s_D[ij] = sd;
    }
    __syncthreads();
    for (int ij = tid; ij < W * W; ij += NT)
        s_pko[ij] = s_D[ij];
    __syncthreads();
    block_excl_scan_i64<NT>(s_pko, W * W, s_warp);
    __syncthreads();
    // pack bases of this CTA's virtual blocks: a kept assignment to expert e at position pos
    // from segment g lands on packed row pkb + pos (block (i, j) holds its experts in order,
    // each expert's rows from shard i in the shard's own order)
    for (int ke = tid; ke < nsub * E; ke += NT) {
        const int kk = ke / E, e = ke % E;
        const int vb = (p.vbm.slot_major ? kk * p.vbm.nblk_tok : 0) + tb;
        const int g = vb / p.bps, i = g % W, j = e / e_per;
        int64_t base = s_pko[i * W + j];
        for (int e2 = j * e_per; e2 < e; ++e2)
            base += s_kh[e2 * W + i];
        for (int g2 = i; g2 < g; g2 += W)
            base += s_cum[(g2 + 1) * E + e] - s_cum[g2 * E + e];
        s_pkb[ke] = base - s_cum[g * E + e];
    }
    if (lead) {
        for (int e = tid; e < E; e += NT) {
            p.counts[e] = s_cum[G * E + e];
            p.kept[e] = s_off[e + 1] - s_off[e];
        }
        for (int e = tid; e <= E; e += NT)
            p.offsets[e] = s_off[e];
        for (int ij = tid; ij < W * W; ij += NT)
            p.D[ij] = s_D[ij];
        for (int ij = tid; ij <= W * W; ij += NT)
            p.pk_off[ij] = s_pko[ij];
        if (p.stats && warp == 0) {
            int mx = 0, mn = 0x7fffffff, act = 0;
            for (int e = lane; e < E; e += 32) {
                const int kp = s_off[e + 1] - s_off[e];
                mx = max(mx, kp);
                mn = min(mn, kp);
                act += kp > 0;
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                act += __shfl_xor_sync(0xffffffffu, act, off);
            }
            int64_t diag = 0;
            for (int i = lane; i < W; i += 32)
                diag += s_D[i * W + i];
            diag = warp_sum(diag);
            if (lane == 0) {
                const int64_t R = s_pko[W * W];
                p.stats->rows = R;
                p.stats->dropped = (int64_t)p.N * p.K - R;
                p.stats->cross_rows = R - diag;
                p.stats->capacity = p.C;
                p.stats->active_experts = act;
                p.stats->max_kept = mx;
                p.stats->min_kept = mn;
                p.stats->rerouted = 0;
            }
        }
    }
    __syncthreads();

    // 4. positions -> rows, the mapping table
    for (int kk = 0; kk < nsub; ++kk) {
        const int na = p.vbm.count(t0, t1);
        for (int i = tid; i < na; i += NT) {
            const int a = p.vbm.assign(t0, kk, i);
            const int ls = a - t0 * K;
            const int e = s_e[ls];
            if (e < 0)
                continue;
            const int pos = s_base[kk * E + e] + s_lr[ls];
            const int row = (pos < p.C && s_off[e] + pos < s_off[e + 1]) ? s_off[e] + pos : -1;
            s_rk[ls] = row;
            s_ex[ls] = row >= 0 ? e : -1;
            const int64_t pk = s_pkb[kk * E + e] + pos;
            s_pk[ls] = (row >= 0 && pk >= 0 && pk < s_off[E]) ? (int)pk : -1;
            if (row >= 0 && part == 0)
                p.assign_of_row[row] = a;
        }
    }
    __syncthreads();
    const bool home_block = p.rank < 0 || tb / p.vbm.bm.bps == p.rank;
    const int64_t pack_row0 = p.rank < 0 ? 0 : s_pko[(size_t)p.rank * W];
    if (part == 0) {
        for (int i = tid; i < nt * K; i += NT) {
            p.row_of[(size_t)t0 * K + i] = s_rk[i];
            if (p.expert_of)
                p.expert_of[(size_t)t0 * K + i] = s_ex[i];
            if (p.packed_row_of)
                p.packed_row_of[(size_t)t0 * K + i] = s_pk[i];
            if (p.pk_of)
                p.pk_of[(size_t)t0 * K + i] = s_pk[i];
            if (p.send_row_of && home_block)
                p.send_row_of[(size_t)(t0 - p.x_row0) * K + i] =
                    s_pk[i] >= 0 ? (int)(s_pk[i] - pack_row0) : -1;
        }
        if (p.stats) {
            // distinct destination ranks other than the token's home over its kept slots
            const int home = tb / p.vbm.bm.bps;
            unsigned long long pairs = 0;
            for (int l2 = warp; l2 < nt; l2 += 8) {
                const int ex = lane < K ? s_ex[l2 * K + lane] : -1;
                const int dest = ex >= 0 ? ex / e_per : -1;
                const int key = (dest >= 0 && dest != home) ? dest : -1 - lane;
                const unsigned grp = __match_any_sync(0xffffffffu, key);
                pairs += __popc(__ballot_sync(0xffffffffu, key >= 0 && (grp & lt_mask) == 0));
            }
            if (lane == 0 && pairs)
                atomicAdd(reinterpret_cast<unsigned long long *>(&p.stats->dedup_pairs), pairs);
        }
    }
    if (!p.copy)
        return;

    // 5. the rows. The whole batch on one GPU with drops: by destination row, after a second
    // grid barrier (every CTA's mapping written), an even split whatever the routing (token
    // blocks keep very different numbers of rows under skew: early tokens claim the capacity).
    // Without drops (every block keeps all its slots) and for a rank's own send rows: by token
    // block.
    if (p.rank < 0 && (p.pk_of || !p.x_packed) && s_dropped) {
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const unsigned int target = 2u * gridDim.x * gridDim.y;
            atomicAdd(&p.ctl[0], 1u);
            int ok = 1;
            const uint64_t w0 = global_timer_ns();
            while (ld_acquire_u32(&p.ctl[0]) < target) {
                if (global_timer_ns() - w0 > p.timeout_ns) {
                    set_dev_error(MOE_ERR_DEVICE_TIMEOUT);
                    ok = 0;
                    break;
                }
            }
            s_ok = ok;
        }
        __syncthreads();
        if (!s_ok)
            return;
        __threadfence();
        const uint32_t ring = smem_u32(fz + L.uni);
        copy_rows_by_row(p.x, p.assign_of_row, p.pk_of, s_off[E], K, p.x_sorted, p.x_packed, p.d,
                         (blockIdx.y * gridDim.x + blockIdx.x) * 8 + warp,
                         gridDim.x * gridDim.y * 8, ring + warp * p.slots * kPiece,
                         ring + 8 * p.slots * kPiece + warp * p.slots * 8, p.slots, p.timeout_ns);
        return;
    }
    if (!home_block)
        return;
    const uint16_t *xb = p.x + (size_t)(t0 - p.x_row0) * p.d;
    for (int i = tid; i < nt * K; i += NT)
        s_pk[i] = (!p.x_packed || s_pk[i] < 0) ? -1 : (int)(s_pk[i] - pack_row0);
    __syncthreads();  // s_agg (in the ring's region) is no longer read
    copy_rows_bulk(xb, nt, K, s_rk, s_pk, p.x_sorted, p.x_packed, p.d, part, parts, fz + L.uni,
                   p.slots, p.timeout_ns);
}

// One CTA per (token block, part). Positions: for every virtual block of the token block (all
// rounds; each slot k in slot-major order), warps count their sub-ranges per expert, take
// their bases from the block's exclusive prefix (inclusive minus own), and rank equal experts
// with __match_any_sync, which gives the sequential first-come position exactly; the
// mapping table (row_of, assign_of_row, expert_of) is written by part 0. Each assignment's
// row is decided by exactly one virtual block: its round-0 block unless it was moved, then
// its round-1 block. Copy: part p of the token block's rows (a column slice of every bf16
// row; whole rows of a share of the tokens for the FP8 payload, whose scale needs the row)
// goes to every kept slot's expert-sorted row and, when requested, its packed row.
__global__ void __launch_bounds__(kPlaceThreads) dispatch_place_kernel(PlaceArgs p)
{
    extern __shared__ __align__(16) int place_smem[];
    const int E = p.E, K = p.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int *wcnt = place_smem;
    int *s_off = wcnt + 8 * E;
    int *s_rk = s_off + E + 1;
    int *s_pk = s_rk + kDispatchHB * K;
    int *s_ex = s_pk + kDispatchHB * K;
    const int tb = blockIdx.x, part = blockIdx.y, parts = gridDim.y;
    int t0, t1;
    p.vbm.bm.range(tb, t0, t1);
    const int nt = t1 - t0;
    for (int i = threadIdx.x; i < nt * K; i += kPlaceThreads) {
        s_rk[i] = -1;
        s_pk[i] = -1;
        s_ex[i] = -1;
    }
    for (int e = threadIdx.x; e <= E; e += kPlaceThreads)
        s_off[e] = p.offsets[e];
    unsigned lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));
    const int nsub = p.vbm.slot_major ? K : 1;
    for (int round = 0; round < p.rounds; ++round) {
        const int32_t *src = p.vbm.experts(p.topk_idx, round);
        for (int kk = 0; kk < nsub; ++kk) {
            const int vb = round * p.vbm.nvb_round + (p.vbm.slot_major ? kk * p.vbm.nblk_tok : 0) + tb;
            const int g = vb / p.bps;
            const int na = p.vbm.count(t0, t1);
            const int per = (na + 7) / 8;
            const int wb = min(na, warp * per), we = min(na, wb + per);
            for (int i = threadIdx.x; i < 8 * E; i += kPlaceThreads)
                wcnt[i] = 0;
            __syncthreads();
            for (int i = wb + lane; i < we; i += 32) {
                const int e = src[p.vbm.assign(t0, kk, i)];
                if ((unsigned)e < (unsigned)E)
                    atomicAdd(&wcnt[warp * E + e], 1);
            }
            __syncthreads();
            for (int e = threadIdx.x; e < E; e += kPlaceThreads) {
                const size_t o = (size_t)vb * E + e;
                int run = __ldcg(p.incl + o) - __ldcg(p.agg + o);
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    const int c = wcnt[w * E + e];
                    wcnt[w * E + e] = run;
                    run += c;
                }
            }
            __syncthreads();
            for (int g0 = wb; g0 < we; g0 += 32) {
                const int i = g0 + lane;
                const bool act = i < we;
                const int a = act ? p.vbm.assign(t0, kk, i) : 0;
                int e = act ? src[a] : -1;
                if ((unsigned)e >= (unsigned)E)
                    e = -1;
                const unsigned peers = __match_any_sync(0xffffffffu, e);
                const int rank = __popc(peers & lt_mask);
                const int base = e >= 0 ? wcnt[warp * E + e] : 0;
                __syncwarp();
                if (e >= 0 && lane == __ffs(peers) - 1)
                    wcnt[warp * E + e] = base + __popc(peers);
                __syncwarp();
                if (act) {
                    const int pos = base + rank;
                    // kept iff pos < C; a kept position is always below the expert's kept
                    // count, which the second test restates so that no row outside the
                    // expert's range is ever written, whatever the prefixes held
                    const int row = (e >= 0 && pos < p.C && s_off[e] + pos < s_off[e + 1])
                                        ? s_off[e] + pos : -1;
                    const bool owner = round ? e >= 0
                                             : (row >= 0 || p.vbm.moved == nullptr ||
                                                p.vbm.moved[a] < 0);
                    if (owner) {
                        const int ls = a - t0 * K;
                        s_rk[ls] = row;
                        s_ex[ls] = row >= 0 ? e : -1;
                        const int64_t pk = p.pk_base[(size_t)g * E + e] + pos;
                        s_pk[ls] = (row >= 0 && pk >= 0 && pk < s_off[E]) ? (int)pk : -1;
                        if (row >= 0 && part == 0)
                            p.assign_of_row[row] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    const bool home_block = p.rank < 0 || tb / p.vbm.bm.bps == p.rank;
    const int64_t pack_row0 = p.rank < 0 ? 0 : p.pk_off[(size_t)p.rank * p.W];
    if (part == 0) {
        for (int i = threadIdx.x; i < nt * K; i += kPlaceThreads) {
            p.row_of[t0 * K + i] = s_rk[i];
            if (p.expert_of)
                p.expert_of[t0 * K + i] = s_ex[i];
            if (p.packed_row_of)
                p.packed_row_of[t0 * K + i] = s_pk[i];
            if (p.send_row_of && home_block)
                p.send_row_of[(t0 - p.x_row0) * K + i] =
                    s_pk[i] >= 0 ? (int)(s_pk[i] - pack_row0) : -1;
        }
        if (p.stats) {
            // distinct destination ranks other than the token's home over its kept slots
            const int e_per = E / p.W;
            const int home = tb / p.vbm.bm.bps;
            unsigned long long pairs = 0;
            for (int lt = warp; lt < nt; lt += 8) {
                const int ex = lane < K ? s_ex[lt * K + lane] : -1;
                const int dest = ex >= 0 ? ex / e_per : -1;
                const int key = (dest >= 0 && dest != home) ? dest : -1 - lane;
                const unsigned grp = __match_any_sync(0xffffffffu, key);
                pairs += __popc(__ballot_sync(0xffffffffu, key >= 0 && (grp & lt_mask) == 0));
            }
            if (lane == 0 && pairs)
                atomicAdd(reinterpret_cast<unsigned long long *>(&p.stats->dedup_pairs), pairs);
        }
    }
    if (!p.copy || !home_block)
        return;
    // rows of this block's tokens: x holds token t at row t - x_row0; the packed rows of a rank
    // start at its block row (pack_row0); without a packed buffer no packed row is written
    const uint16_t *xb = p.x + (size_t)(t0 - p.x_row0) * p.d;  // the block's first token
    if (!p.x_packed)
        for (int i = threadIdx.x; i < nt * K; i += kPlaceThreads)
            s_pk[i] = -1;
    else if (pack_row0 != 0)
        for (int i = threadIdx.x; i < nt * K; i += kPlaceThreads)
            s_pk[i] = s_pk[i] >= 0 ? (int)(s_pk[i] - pack_row0) : -1;
    __syncthreads();

    if (!p.e4m3) {
        copy_rows_bulk(xb, nt, K, s_rk, s_pk, p.x_sorted, p.x_packed, p.d, part, parts,
                       reinterpret_cast<unsigned char *>(place_smem) + place_ring_offset(E, K),
                       p.slots, p.timeout_ns);
        return;
    }

    // FP8 payload ([MoE 推理服务工程真相 2026, §6.3]: the token rows that cross the
    // all-to-all travel as FP8): one warp per token reads its bf16 row twice (the second pass
    // hits L1/L2), first for the largest magnitude, then to write e4m3 codes (row scaled by
    // 2^-j, the row's power-of-two scale) to every kept slot's sorted and packed row, with the
    // scale 2^j beside each row. This part takes the tokens part, part + parts, ... of the block.
    const int n16 = p.d >> 4;  // 16-element chunks: two 16-byte loads, one 16-byte store
    uint4 *dst_s = reinterpret_cast<uint4 *>(p.x_sorted);
    uint4 *dst_p = reinterpret_cast<uint4 *>(p.x_packed);
    for (int lt = part + parts * warp; lt < nt; lt += parts * 8) {
        const uint4 *src = reinterpret_cast<const uint4 *>(xb + (size_t)lt * p.d);
        const int *rk_l = s_rk + lt * K;
        const int *pk_l = s_pk + lt * K;
        // pass 1: largest magnitude of the row (bf16 bits with the sign cleared order like the
        // magnitudes; a NaN marks the row non-finite)
        uint32_t mx = 0;
        for (int c = lane; c < 2 * n16; c += 32) {
            const uint4 v = src[c];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                mx = max(mx, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float amax = __uint_as_float(mx << 16);  // NaN bits sort above Inf
        const int j = e4m3_scale_exp(amax);
        const float inv = pow2f(-j), scale = pow2f(j);
        if (lane < K) {
            const int rk = rk_l[lane], pk = pk_l[lane];
            if (rk >= 0) {
                if (p.sorted_scale)
                    p.sorted_scale[rk] = scale;
                if (pk >= 0)
                    p.packed_scale[pk] = scale;
            }
        }
        // pass 2
        for (int c = lane; c < n16; c += 32) {
            const uint4 a = src[2 * c], b = src[2 * c + 1];
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t lo = pack_e4m3x2(bf16_lo(w[2 * i]) * inv, bf16_hi(w[2 * i]) * inv);
                const uint32_t hi =
                    pack_e4m3x2(bf16_lo(w[2 * i + 1]) * inv, bf16_hi(w[2 * i + 1]) * inv);
                o[i] = lo | (hi << 16);
            }
            const uint4 q = make_uint4(o[0], o[1], o[2], o[3]);
            for (int k = 0; k < K; ++k) {
                const int rk = rk_l[k];
                if (rk < 0)
                    continue;
                if (dst_s)
                    dst_s[(size_t)rk * n16 + c] = q;
                const int pk = pk_l[k];
                if (pk >= 0)
                    dst_p[(size_t)pk * n16 + c] = q;
            }
        }
    }
}

// W real ranks: the rows that rank j receives in one exchange (the blocks (i, j) of every home
// rank i, one after another, each in its (expert, token) order) <-> rank j's expert-sorted rows
// (its experts [j E/W, (j+1) E/W), their rows in the one-GPU order: rows [offsets[e0],
// offsets[e1]) of the whole batch's expert-sorted layout). Row r of that layout is assignment
// a = assign_of_row[r], of a token whose home shard is i = (a / K) / S, at packed row
// packed_row_of[a] inside block (i, j), which starts at pk_off[i W + j]; in the received buffer
// block (i, j) starts after the blocks (i', j) of i' < i. dir 0 gathers received rows into
// sorted order (the layer's way out to the experts), dir 1 scatters sorted rows back into the
// received order (the way back). Block 0 also writes the rank's expert offsets (E/W + 1).
struct RegroupArgs {
    const int32_t *assign_of_row, *packed_row_of, *offsets;
    const int64_t *pk_off;  // [W*W+1]
    int E, K, W, S, rank;
    int row_vec;            // 16-byte vectors per row
    const uint4 *src;
    uint4 *dst;
    int dir;
    int32_t *offsets_local;  // nullable
};

__global__ void __launch_bounds__(256) regroup_rows_kernel(RegroupArgs p)
{
    __shared__ int64_t s_base[64 + 1];  // per home rank i: received index - packed row
    const int W = p.W, j = p.rank, e_per = p.E / W;
    const int e0 = j * e_per;
    if (threadIdx.x == 0) {
        int64_t run = 0;
        for (int i = 0; i < W; ++i) {
            const int64_t b0 = p.pk_off[i * W + j], b1 = p.pk_off[i * W + j + 1];
            s_base[i] = run - b0;
            run += b1 - b0;
        }
    }
    if (blockIdx.x == 0 && p.offsets_local)
        for (int e = threadIdx.x; e <= e_per; e += blockDim.x)
            p.offsets_local[e] = p.offsets[e0 + e] - p.offsets[e0];
    __syncthreads();
    const int r0 = p.offsets[e0], r1 = p.offsets[e0 + e_per];
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    for (int r = r0 + blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < r1; r += nwarps) {
        const int a = p.assign_of_row[r];
        const int i = (a / p.K) / p.S;
        const int64_t recv = s_base[i] + p.packed_row_of[a];
        const size_t sorted = (size_t)(r - r0);
        const uint4 *from = p.src + (p.dir == 0 ? (size_t)recv : sorted) * p.row_vec;
        uint4 *to = p.dst + (p.dir == 0 ? sorted : (size_t)recv) * p.row_vec;
        for (int c = lane; c < p.row_vec; c += 32)
            to[c] = from[c];
    }
}

struct RerouteArgs {
    const float *logits;     // [N][E]
    const int32_t *topk_idx;
    const int32_t *row_of;   // after round 0: -1 = past capacity (or invalid expert)
    const int32_t *counts;   // round-0 demand per expert
    int N, E, K, C;
    int32_t *moved;          // [N*K] out: new expert of a moved assignment, else -1
};

// One warp per token. An expert is full when its demand reached C. The token's
// overflowed slots, in slot order, take its best remaining experts (larger logit
// first, ties to the lower index; NaN ranks as -inf) that are neither routed to by
// the token, nor full, nor taken by an earlier slot.
__global__ void __launch_bounds__(256) reroute_kernel(RerouteArgs p)
{
    constexpr int MAXJ = 8;  // E <= 256
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < p.N; t += nwarps) {
        int mine = -1;
        bool over = false;
        if (lane < p.K) {
            mine = p.topk_idx[t * p.K + lane];
            over = (unsigned)mine < (unsigned)p.E && p.row_of[t * p.K + lane] < 0;
        }
        unsigned om = __ballot_sync(0xffffffffu, over);
        int res = -1;
        if (om) {
            float v[MAXJ];
            bool avail[MAXJ];
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) {
                const int e = lane + 32 * j;
                avail[j] = false;
                v[j] = -INFINITY;
                if (e < p.E) {
                    const float l = p.logits[(size_t)t * p.E + e];
                    v[j] = isnan(l) ? -INFINITY : l;
                    avail[j] = p.counts[e] < p.C;
                }
            }
            for (int k = 0; k < p.K; ++k) {
                const int ek = __shfl_sync(0xffffffffu, mine, k);
#pragma unroll
                for (int j = 0; j < MAXJ; ++j)
                    if (ek == lane + 32 * j)
                        avail[j] = false;
            }
            while (om) {
                const int k = __ffs(om) - 1;
                om &= om - 1;
                float bv = -INFINITY;
                int be = -1;
#pragma unroll
                for (int j = 0; j < MAXJ; ++j)
                    if (avail[j] && (be < 0 || v[j] > bv)) {  // j ascending: ties keep the lower
                        bv = v[j];
                        be = lane + 32 * j;
                    }
#pragma unroll
                for (int off = 16; off; off >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                    if (oe >= 0 && (be < 0 || ov > bv || (ov == bv && oe < be))) {
                        bv = ov;
                        be = oe;
                    }
                }
                if (lane == k)
                    res = be;
#pragma unroll
                for (int j = 0; j < MAXJ; ++j)
                    if (be == lane + 32 * j)
                        avail[j] = false;
            }
        }
        if (lane < p.K)
            p.moved[t * p.K + lane] = res;
    }
}

// Row-wise e4m3 quantisation of a bf16 matrix (for the experts' W1 and W3): one
// warp per row, the same two passes and rounding as the FP8 scatter. cols % 16 == 0.
// rows_dev (nullable, device): rows beyond *rows_dev are skipped (the FP8 down projection
// quantises only the rows the dispatch kept).
__global__ void __launch_bounds__(256)
    quantize_rows_e4m3_kernel(const uint16_t *__restrict__ src, int64_t rows, int cols,
                              uint8_t *__restrict__ codes, float *__restrict__ scale,
                              const int32_t *__restrict__ rows_dev)
{
    if (rows_dev && *rows_dev < rows)
        rows = *rows_dev;
    const int lane = threadIdx.x & 31;
    const int n16 = cols >> 4;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
         row += nwarps) {
        const uint4 *s = reinterpret_cast<const uint4 *>(src + row * cols);
        uint32_t mx = 0;
        for (int c = lane; c < 2 * n16; c += 32) {
            const uint4 v = s[c];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                mx = max(mx, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const int j = e4m3_scale_exp(__uint_as_float(mx << 16));
        const float inv = pow2f(-j);
        if (lane == 0)
            scale[row] = pow2f(j);
        uint4 *d = reinterpret_cast<uint4 *>(codes + row * cols);
        for (int c = lane; c < n16; c += 32) {
            const uint4 a = s[2 * c], b = s[2 * c + 1];
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t lo = pack_e4m3x2(bf16_lo(w[2 * i]) * inv, bf16_hi(w[2 * i]) * inv);
                const uint32_t hi =
                    pack_e4m3x2(bf16_lo(w[2 * i + 1]) * inv, bf16_hi(w[2 * i + 1]) * inv);
                o[i] = lo | (hi << 16);
            }
            d[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// bf16 -> fp16 conversion of a weight matrix (the experts' W2 and the shared MLP's Ws2, which
// the down projection reads as fp16 beside the fp16 h), eight elements per 16-byte load. Every
// bf16 value whose magnitude lies in [2^-17, 65504] converts exactly (fp16 keeps 11
// significant bits and reaches down to 2^-24 in steps of 2^-24); smaller ones round to the
// nearest fp16 step, larger ones become infinite and record MOE_ERR_F16_RANGE. The number of
// elements whose value changed is added to *changed (nullable). n % 8 == 0.
__global__ void __launch_bounds__(256)
    convert_bf16_f16_kernel(const uint16_t *__restrict__ src, int64_t n, uint16_t *__restrict__ dst,
                            unsigned long long *__restrict__ changed)
{
    const int64_t nvec = n >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    unsigned long long cnt = 0;
    bool over = false;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
        const uint4 a = reinterpret_cast<const uint4 *>(src)[v];
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
            uint32_t r;
            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
            float blo, bhi;
            asm("cvt.f32.f16 %0, %1;" : "=f"(blo) : "h"((unsigned short)(r & 0xFFFFu)));
            asm("cvt.f32.f16 %0, %1;" : "=f"(bhi) : "h"((unsigned short)(r >> 16)));
            cnt += (blo != lo) + (bhi != hi);
            over |= (isinf(blo) && !isinf(lo)) || (isinf(bhi) && !isinf(hi));
            o[i] = r;
        }
        reinterpret_cast<uint4 *>(dst)[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (over)
        set_dev_error(MOE_ERR_F16_RANGE);
    if (changed) {
        cnt = warp_sum(cnt);
        if ((threadIdx.x & 31) == 0 && cnt)
            atomicAdd(changed, cnt);
    }
}

}  // namespace moe
