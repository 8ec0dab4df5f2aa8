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

// blk[e][vb] = number of assignments in virtual block vb routed to expert e.
__global__ void __launch_bounds__(256)
    block_hist_kernel(const int32_t *__restrict__ topk_idx, int E, VBlocks vbm, int nvb,
                      int32_t *__restrict__ blk)
{
    extern __shared__ int s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_hist[e] = 0;
    __syncthreads();
    int t0, t1, k, round;
    vbm.range(blockIdx.x, t0, t1, k, round);
    const int32_t *src = vbm.experts(topk_idx, round);
    const int n = vbm.count(t0, t1);
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int e = src[vbm.assign(t0, k, i)];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&s_hist[e], 1);
        else if (round == 0)
            set_dev_error(MOE_ERR_DEVICE_BOUNDS);  // round 1 marks "not moved" with -1
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        blk[(size_t)e * nvb + blockIdx.x] = s_hist[e];
}

// In-place exclusive scan of a[0..n) in shared memory by the whole block;
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

// Many blocks (slot-major priority, re-routing): one CTA per expert turns its row of
// block counts into exclusive bases and records the expert's count at every segment start
// (cum [E][nseg+1], cum[e][nseg] = total); dispatch_scan_kernel then skips that step.
__global__ void __launch_bounds__(256)
    expert_block_scan_kernel(int32_t *__restrict__ blk, int nvb, int bps, int nseg,
                             int32_t *__restrict__ cum)
{
    __shared__ int s_warp[8];
    const int e = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t *row = blk + (size_t)e * nvb;
    const int per = (nvb + 255) / 256;
    const int beg = min(nvb, (int)threadIdx.x * per), end = min(nvb, beg + per);
    int local = 0;
    for (int i = beg; i < end; ++i)
        local += row[i];
    const int incl = warp_incl_scan(local);
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < 8 ? s_warp[lane] : 0;
        const int vi = warp_incl_scan(v);
        if (lane < 8)
            s_warp[lane] = vi - v;
    }
    __syncthreads();
    int run = s_warp[warp] + incl - local;
    for (int i = beg; i < end; ++i) {
        const int v = row[i];
        row[i] = run;
        if (i % bps == 0)
            cum[(size_t)e * (nseg + 1) + i / bps] = run;
        run += v;
    }
    if (threadIdx.x == 255)
        cum[(size_t)e * (nseg + 1) + nseg] = run;  // the last thread ends at the total
}

struct ScanArgs {
    int32_t *blk;  // [E][nvb] counts in, exclusive bases out
    int nvb;
    int bps;       // virtual blocks per segment
    int nseg;      // segments in priority order: W (token-major) or K*W (slot-major) a round
    int nseg_round;
    int N, E, K, W;
    int C;
    int32_t *cum_global;  // [E][nseg+1] when it does not fit in shared memory, else null
    int prescanned;       // expert_block_scan_kernel has done step 1 into cum_global
    int32_t *counts, *kept, *offsets;
    int64_t *D;        // [W][W]
    int64_t *pk_off;   // [W*W+1]
    int64_t *pk_base;  // [E][nseg]
    moe_stats_t *stats;
};

// One CTA of 1024 threads.
// Shared: s_a [max(E, W*W) + 1] int64 scan buffer, s_D [W*W] int64, s_warp [32],
//         s_kh [E][W] int32 (kept rows of expert e from home shard i), then
//         cum [E][nseg+1] int32 unless it lives in global memory: cum[e][g] =
//         assignments to e before segment g in priority order, cum[e][nseg] = total.
// Segment g belongs to home shard g % W; within one home shard its segments
// come in priority order, so the kept rows of expert e from that shard are a
// prefix of the shard's own sequence of assignments to e.
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(ScanArgs p)
{
    constexpr int NT = 1024;
    extern __shared__ __align__(16) unsigned char scan_smem[];
    const int E = p.E, W = p.W, nvb = p.nvb, bps = p.bps, G = p.nseg;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t C = p.C;
    const int scan_len = max(E, W * W) + 1;
    int64_t *s_a = reinterpret_cast<int64_t *>(scan_smem);
    int64_t *s_D = s_a + scan_len;
    int64_t *s_warp = s_D + W * W;
    int32_t *s_kh = reinterpret_cast<int32_t *>(s_warp + 32);
    int32_t *cum = p.cum_global ? p.cum_global : s_kh + E * W;

    // 1. per expert: exclusive scan over virtual blocks; record segment starts
    for (int e = warp; e < E && !p.prescanned; e += NT / 32) {
        int32_t *row = p.blk + (size_t)e * nvb;
        int carry = 0;
        for (int base = 0; base < nvb; base += 128) {
            int v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = base + lane * 4 + q;
                v[q] = idx < nvb ? row[idx] : 0;
            }
            const int lsum = v[0] + v[1] + v[2] + v[3];
            const int incl = warp_incl_scan(lsum);
            int run = carry + incl - lsum;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = base + lane * 4 + q;
                if (idx < nvb) {
                    row[idx] = run;
                    if (idx % bps == 0)
                        cum[e * (G + 1) + idx / bps] = run;
                }
                run += v[q];
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0)
            cum[e * (G + 1) + G] = carry;
    }
    __syncthreads();

    // 2. counts (round 0: the routed demand), kept, offsets; kept rows per
    //    (expert, home shard)
    for (int e = threadIdx.x; e < E; e += NT) {
        const int c = cum[e * (G + 1) + p.nseg_round];
        const int kp = (int)min((int64_t)cum[e * (G + 1) + G], C);
        p.counts[e] = c;
        p.kept[e] = kp;
        s_a[e] = kp;
    }
    for (int ei = threadIdx.x; ei < E * W; ei += NT) {
        const int e = ei / W, i = ei % W;
        const int32_t *ce = cum + e * (G + 1);
        int64_t s = 0;
        for (int g = i; g < G; g += W)
            s += min((int64_t)ce[g + 1], C) - min((int64_t)ce[g], C);
        s_kh[ei] = (int32_t)s;
    }
    __syncthreads();
    block_excl_scan_i64<NT>(s_a, E, s_warp);
    for (int e = threadIdx.x; e <= E; e += NT)
        p.offsets[e] = (int32_t)s_a[e];
    __syncthreads();

    // 3. traffic matrix D[i][j] = kept rows of experts on rank j from shard i
    const int e_per = E / W;
    for (int ij = threadIdx.x; ij < W * W; ij += NT) {
        const int i = ij / W, j = ij % W;
        int64_t s = 0;
        for (int e = j * e_per; e < (j + 1) * e_per; ++e)
            s += s_kh[e * W + i];
        s_D[ij] = s;
        if (p.D)
            p.D[ij] = s;
    }
    __syncthreads();
    for (int ij = threadIdx.x; ij < W * W; ij += NT)
        s_a[ij] = s_D[ij];
    __syncthreads();
    block_excl_scan_i64<NT>(s_a, W * W, s_warp);
    if (p.pk_off)
        for (int ij = threadIdx.x; ij <= W * W; ij += NT)
            p.pk_off[ij] = s_a[ij];

    // 4. pack bases: a kept assignment to expert e at position pos (in e's rows)
    //    from segment g lands on packed row pk_base[e][g] + pos. Block (i, j)
    //    holds its experts in order, each expert's rows from shard i in the
    //    shard's own order: the earlier segments of shard i come first.
    for (int ei = threadIdx.x; ei < E * W; ei += NT) {
        const int e = ei / W, i = ei % W;
        const int j = e / e_per;
        int64_t base = s_a[i * W + j];
        for (int e2 = j * e_per; e2 < e; ++e2)
            base += s_kh[e2 * W + i];
        const int32_t *ce = cum + e * (G + 1);
        int64_t run = 0;
        for (int g = i; g < G; g += W) {
            p.pk_base[(size_t)e * G + g] = base + run - ce[g];
            run += ce[g + 1] - ce[g];
        }
    }

    // 5. counters (dedup_pairs is added by the scatter kernel)
    if (p.stats && warp == 0) {
        int mx = 0, mn = 0x7fffffff, act = 0;
        int64_t first = 0;  // rows from round 0
        for (int e = lane; e < E; e += 32) {
            const int kp = (int)min((int64_t)cum[e * (G + 1) + G], C);
            mx = max(mx, kp);
            mn = min(mn, kp);
            act += kp > 0;
            first += min((int64_t)cum[e * (G + 1) + p.nseg_round], C);
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

struct PosArgs {
    const int32_t *topk_idx;
    const int32_t *blk;  // [E][nvb] exclusive bases
    int nvb;
    VBlocks vbm;
    int E;
    int C;
    const int32_t *offsets;
    int32_t *row_of;
    int32_t *assign_of_row;
};

// One CTA (8 warps) per virtual block. Shared: wcnt [8][E] int32, s_off [E] int32.
// Each assignment's row_of is written by exactly one block: its round-0 block,
// unless it was moved, then its round-1 block.
__global__ void __launch_bounds__(256) dispatch_positions_kernel(PosArgs p)
{
    extern __shared__ __align__(16) int pos_smem[];
    const int E = p.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int *wcnt = pos_smem;
    int *s_off = wcnt + 8 * E;

    int t0, t1, k, round;
    p.vbm.range(blockIdx.x, t0, t1, k, round);
    const int32_t *src = p.vbm.experts(p.topk_idx, round);
    const int na = p.vbm.count(t0, t1);
    const int per = (na + 7) / 8;
    const int wb = min(na, warp * per), we = min(na, wb + per);

    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x)
        wcnt[i] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_off[e] = p.offsets[e];
    __syncthreads();
    for (int i = wb + lane; i < we; i += 32) {
        const int e = src[p.vbm.assign(t0, k, i)];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&wcnt[warp * E + e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = p.blk[(size_t)e * p.nvb + blockIdx.x];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const int c = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();

    unsigned lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));
    for (int g = wb; g < we; g += 32) {
        const int i = g + lane;
        const bool act = i < we;
        const int a = act ? p.vbm.assign(t0, k, i) : 0;
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
            const int row = (e >= 0 && pos < p.C) ? s_off[e] + pos : -1;
            const bool owner = round ? e >= 0
                                     : (row >= 0 || p.vbm.moved == nullptr || p.vbm.moved[a] < 0);
            if (owner)
                p.row_of[a] = row;
            if (row >= 0)
                p.assign_of_row[row] = a;
        }
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

struct ScatterArgs {
    const uint16_t *x;
    const int32_t *topk_idx;
    const int32_t *row_of;
    const int32_t *offsets;
    const int64_t *pk_base;  // [E][nseg]
    const int32_t *moved;    // round-1 expert per assignment, or null
    int N, d, K, W, E;
    int S;           // N / W
    int slot_major;  // segment of (t, k) in its round: k*W + t/S, else t/S
    int nseg;        // all rounds
    int nseg_round;
    int32_t *expert_of;  // nullable out: the expert whose row each assignment uses, or -1
    int seg;             // bf16 scatter: 16-byte chunks per work item (whole row for large N)
    void *x_sorted;      // bf16 rows, or e4m3 rows with fp8 payload
    void *x_packed;      // nullable, same element type
    float *sorted_scale;  // e4m3 payload: scale of each x_sorted row
    float *packed_scale;  // e4m3 payload: scale of each x_packed row (nullable)
    moe_stats_t *stats;  // nullable: dedup_pairs is accumulated here
};

// Targets of slot `lane` (lanes < K) of token t: its expert-sorted row r (-1 if
// dropped) and packed row pk (-1 if dropped or not packing). When `first` (the
// token's first work item): also writes expert_of and returns the number of
// distinct non-home destination ranks of the token (the same value in every lane),
// when counting.
__device__ __forceinline__ int slot_targets(const ScatterArgs &p, int t, int lane,
                                            unsigned lt_mask, int &r, long long &pk,
                                            bool first = true)
{
    const int e_per = p.E / p.W;
    const int home = t / p.S;
    int dest = -1;
    r = -1;
    pk = -1;
    if (lane < p.K) {
        const int a = t * p.K + lane;
        r = p.row_of[a];
        int ef = -1;
        if (r >= 0) {
            const int em = p.moved ? p.moved[a] : -1;
            const int e = em >= 0 ? em : p.topk_idx[a];
            ef = e;
            dest = e / e_per;
            if (p.x_packed) {
                const int g = (em >= 0 ? p.nseg_round : 0) +
                              (p.slot_major ? lane * p.W + home : home);
                pk = p.pk_base[(size_t)e * p.nseg + g] + (r - p.offsets[e]);
            }
        }
        if (p.expert_of && first)
            p.expert_of[a] = ef;
    }
    if (!p.stats || !first)
        return 0;
    // distinct non-home destinations: count the lowest lane of each group
    const int key = (dest >= 0 && dest != home) ? dest : -1 - lane;
    const unsigned grp = __match_any_sync(0xffffffffu, key);
    return __popc(__ballot_sync(0xffffffffu, key >= 0 && (grp & lt_mask) == 0));
}

// One warp per work item (a token and `seg` 16-byte chunks of its row: the whole
// row unless there are too few tokens to fill the GPU): read the token's row once
// (16-byte loads), write it to each kept slot's expert-sorted row and, when
// requested, to its packed row. The token's distinct destination ranks other than
// its home (over kept slots) are counted into stats->dedup_pairs.
__global__ void __launch_bounds__(256) scatter_rows_kernel(ScatterArgs p)
{
    constexpr int U = 4;
    const int lane = threadIdx.x & 31;
    const int nvec = p.d >> 3;
    const int nseg = (nvec + p.seg - 1) / p.seg;
    const int64_t items = (int64_t)p.N * nseg;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    unsigned lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));
    unsigned long long pairs = 0;
    for (int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
         item < items; item += nwarps) {
        const int t = (int)(item / nseg);
        const int sidx = (int)(item % nseg);
        const int cbeg = sidx * p.seg, cend = min(nvec, cbeg + p.seg);
        int r;
        long long pk;
        pairs += slot_targets(p, t, lane, lt_mask, r, pk, sidx == 0);
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (size_t)t * p.d);
        uint4 *dst_s = reinterpret_cast<uint4 *>(p.x_sorted);
        uint4 *dst_p = reinterpret_cast<uint4 *>(p.x_packed);
        // every lane runs every iteration: the shuffles below read lanes 0..K-1
        for (int c0 = cbeg; c0 < cend; c0 += 32 * U) {
            const int c = c0 + lane;
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c + 32 * u < cend)
                    v[u] = __ldcs(src + c + 32 * u);
            for (int k = 0; k < p.K; ++k) {
                const int rk = __shfl_sync(0xffffffffu, r, k);
                const long long pkk = __shfl_sync(0xffffffffu, pk, k);
                if (rk < 0)
                    continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c + 32 * u < cend) {
                        dst_s[(size_t)rk * nvec + c + 32 * u] = v[u];
                        if (pkk >= 0)
                            dst_p[(size_t)pkk * nvec + c + 32 * u] = v[u];
                    }
                }
            }
        }
    }
    if (p.stats && lane == 0 && pairs)
        atomicAdd(reinterpret_cast<unsigned long long *>(&p.stats->dedup_pairs), pairs);
}

// FP8 payload ([MoE 推理服务工程真相 2026, §6.3]: the token rows that cross the
// all-to-all travel as FP8): one warp per token reads its bf16 row twice (the
// second pass hits L1/L2), first for the largest magnitude, then to write e4m3
// codes (row scaled by 2^-j, the row's power-of-two scale) to every kept slot's
// sorted and packed row, with the scale 2^j beside each row. d % 16 == 0.
__global__ void __launch_bounds__(256) scatter_rows_e4m3_kernel(ScatterArgs p)
{
    const int lane = threadIdx.x & 31;
    const int n16 = p.d >> 4;  // 16-element chunks: two 16-byte loads, one 16-byte store
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    unsigned lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));
    unsigned long long pairs = 0;
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < p.N; t += nwarps) {
        int r;
        long long pk;
        pairs += slot_targets(p, t, lane, lt_mask, r, pk);
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (size_t)t * p.d);
        // pass 1: largest magnitude of the row (bf16 bits with the sign cleared
        // order like the magnitudes; a NaN marks the row non-finite)
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
        for (int k = 0; k < p.K; ++k) {
            const int rk = __shfl_sync(0xffffffffu, r, k);
            const long long pkk = __shfl_sync(0xffffffffu, pk, k);
            if (lane == 0 && rk >= 0) {
                p.sorted_scale[rk] = scale;
                if (pkk >= 0)
                    p.packed_scale[pkk] = scale;
            }
        }
        uint4 *dst_s = reinterpret_cast<uint4 *>(p.x_sorted);
        uint4 *dst_p = reinterpret_cast<uint4 *>(p.x_packed);
        // pass 2: every lane runs every iteration (the shuffles read lanes 0..K-1)
        for (int c0 = 0; c0 < n16; c0 += 32) {
            const int c = c0 + lane;
            uint4 q = make_uint4(0, 0, 0, 0);
            if (c < n16) {
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
                q = make_uint4(o[0], o[1], o[2], o[3]);
            }
            for (int k = 0; k < p.K; ++k) {
                const int rk = __shfl_sync(0xffffffffu, r, k);
                const long long pkk = __shfl_sync(0xffffffffu, pk, k);
                if (rk < 0 || c >= n16)
                    continue;
                dst_s[(size_t)rk * n16 + c] = q;
                if (pkk >= 0)
                    dst_p[(size_t)pkk * n16 + c] = q;
            }
        }
    }
    if (p.stats && lane == 0 && pairs)
        atomicAdd(reinterpret_cast<unsigned long long *>(&p.stats->dedup_pairs), pairs);
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
