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
// Positions are taken in token-major (t, k) order without global atomics: a
// block's base per expert comes from the scan over blocks, ranks inside a block
// from per-warp counts and __match_any_sync, so the result is deterministic and
// equal to the sequential definition.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kDispatchHB = 64;  // tokens per dispatch block

// blk[e][b] = number of assignments in block b routed to expert e.
__global__ void __launch_bounds__(256)
    block_hist_kernel(const int32_t *__restrict__ topk_idx, int K, int E, BlockMap bm, int nblk,
                      int32_t *__restrict__ blk)
{
    extern __shared__ int s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_hist[e] = 0;
    __syncthreads();
    int t0, t1;
    bm.range(blockIdx.x, t0, t1);
    for (int a = t0 * K + threadIdx.x; a < t1 * K; a += blockDim.x) {
        const int e = topk_idx[a];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&s_hist[e], 1);
        else
            set_dev_error(MOE_ERR_DEVICE_BOUNDS);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        blk[(size_t)e * nblk + blockIdx.x] = s_hist[e];
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

struct ScanArgs {
    int32_t *blk;  // [E][nblk] counts in, exclusive bases out
    int nblk;
    BlockMap bm;
    int N, E, K, W;
    int C;
    int32_t *counts, *kept, *offsets;
    int64_t *D;        // [W][W]
    int64_t *pk_off;   // [W*W+1]
    int64_t *pk_base;  // [E][W]
    moe_stats_t *stats;
};

// One CTA of 1024 threads.
// Shared: s_cum [E][W+1] int32 (assignments of e before shard i; [W] = total),
//         s_a   [max(E, W*W) + 1] int64 scan buffer, s_D [W*W] int64, s_warp[32].
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(ScanArgs p)
{
    constexpr int NT = 1024;
    extern __shared__ __align__(16) unsigned char scan_smem[];
    const int E = p.E, W = p.W, nblk = p.nblk, bps = p.bm.bps;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t C = p.C;
    const int scan_len = max(E, W * W) + 1;
    int64_t *s_a = reinterpret_cast<int64_t *>(scan_smem);
    int64_t *s_D = s_a + scan_len;
    int64_t *s_warp = s_D + W * W;
    int32_t *s_cum = reinterpret_cast<int32_t *>(s_warp + 32);

    // 1. per expert: exclusive scan over blocks; record shard starts
    for (int e = warp; e < E; e += NT / 32) {
        int32_t *row = p.blk + (size_t)e * nblk;
        int carry = 0;
        for (int base = 0; base < nblk; base += 128) {
            int v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = base + lane * 4 + q;
                v[q] = idx < nblk ? row[idx] : 0;
            }
            const int lsum = v[0] + v[1] + v[2] + v[3];
            const int incl = warp_incl_scan(lsum);
            int run = carry + incl - lsum;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = base + lane * 4 + q;
                if (idx < nblk) {
                    row[idx] = run;
                    if (idx % bps == 0)
                        s_cum[e * (W + 1) + idx / bps] = run;
                }
                run += v[q];
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0)
            s_cum[e * (W + 1) + W] = carry;
    }
    __syncthreads();

    // 2. counts, kept, offsets
    for (int e = threadIdx.x; e < E; e += NT) {
        const int c = s_cum[e * (W + 1) + W];
        const int kp = (int)min((int64_t)c, C);
        p.counts[e] = c;
        p.kept[e] = kp;
        s_a[e] = kp;
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
        for (int e = j * e_per; e < (j + 1) * e_per; ++e) {
            const int64_t lo = min((int64_t)s_cum[e * (W + 1) + i], C);
            const int64_t hi = min((int64_t)s_cum[e * (W + 1) + i + 1], C);
            s += hi - lo;
        }
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

    // 4. pack bases: packed row of expert e's row at position pos from shard i
    //    = pk_base[e][i] + pos
    for (int ei = threadIdx.x; ei < E * W; ei += NT) {
        const int e = ei / W, i = ei % W;
        const int j = e / e_per;
        int64_t base = s_a[i * W + j];
        for (int e2 = j * e_per; e2 < e; ++e2) {
            const int64_t lo = min((int64_t)s_cum[e2 * (W + 1) + i], C);
            const int64_t hi = min((int64_t)s_cum[e2 * (W + 1) + i + 1], C);
            base += hi - lo;
        }
        base -= min((int64_t)s_cum[e * (W + 1) + i], C);
        p.pk_base[ei] = base;
    }

    // 5. counters
    if (p.stats && warp == 0) {
        int mx = 0, mn = 0x7fffffff, act = 0;
        for (int e = lane; e < E; e += 32) {
            const int kp = (int)min((int64_t)s_cum[e * (W + 1) + W], C);
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
            const int64_t R = s_a[W * W];  // total of D == R
            p.stats->rows = R;
            p.stats->dropped = (int64_t)p.N * p.K - R;
            p.stats->cross_rows = R - diag;
            p.stats->dedup_pairs = 0;
            p.stats->capacity = p.C;
            p.stats->active_experts = act;
            p.stats->max_kept = mx;
            p.stats->min_kept = mn;
        }
    }
}

struct PosArgs {
    const int32_t *topk_idx;
    const int32_t *blk;  // [E][nblk] exclusive bases
    int nblk;
    BlockMap bm;
    int N, E, K, W;
    int C;
    const int32_t *offsets;
    int32_t *row_of;
    int32_t *assign_of_row;
    moe_stats_t *stats;
};

// One CTA (8 warps) per dispatch block. Shared: wcnt [8][E] int32,
// s_off [E] int32, krank [HB*K] int8 (destination rank of a kept slot, else -1).
__global__ void __launch_bounds__(256) dispatch_positions_kernel(PosArgs p)
{
    extern __shared__ __align__(16) int pos_smem[];
    const int E = p.E, K = p.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int *wcnt = pos_smem;
    int *s_off = wcnt + 8 * E;
    signed char *krank = reinterpret_cast<signed char *>(s_off + E);

    int t0, t1;
    p.bm.range(blockIdx.x, t0, t1);
    const int a0 = t0 * K, na = (t1 - t0) * K;
    const int per = (na + 7) / 8;
    const int wb = min(na, warp * per), we = min(na, wb + per);

    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x)
        wcnt[i] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_off[e] = p.offsets[e];
    __syncthreads();
    for (int i = wb + lane; i < we; i += 32) {
        const int e = p.topk_idx[a0 + i];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&wcnt[warp * E + e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = p.blk[(size_t)e * p.nblk + blockIdx.x];
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
    const int e_per = E / p.W;
    for (int g = wb; g < we; g += 32) {
        const int i = g + lane;
        const bool act = i < we;
        int e = act ? p.topk_idx[a0 + i] : -1;
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
            p.row_of[a0 + i] = row;
            if (row >= 0)
                p.assign_of_row[row] = a0 + i;
            krank[i] = row >= 0 ? (signed char)(e / e_per) : (signed char)-1;
        }
    }
    if (p.stats == nullptr)
        return;
    __syncthreads();
    const int S = p.bm.S;
    unsigned long long pairs = 0;
    for (int tt = threadIdx.x; tt < t1 - t0; tt += blockDim.x) {
        const int home = (t0 + tt) / S;
        unsigned long long m = 0;
        for (int k = 0; k < K; ++k) {
            const int j = krank[tt * K + k];
            if (j >= 0 && j != home)
                m |= 1ull << j;
        }
        pairs += __popcll(m);
    }
    pairs = warp_sum(pairs);
    if (lane == 0 && pairs)
        atomicAdd(reinterpret_cast<unsigned long long *>(&p.stats->dedup_pairs), pairs);
}

struct ScatterArgs {
    const uint16_t *x;
    const int32_t *topk_idx;
    const int32_t *row_of;
    const int32_t *offsets;
    const int64_t *pk_base;  // [E][W]
    int N, d, K, W, E;
    int S;  // N / W
    uint16_t *x_sorted;
    uint16_t *x_packed;  // nullable
};

// One warp per token: read the token's row once (16-byte loads), write it to
// each kept slot's expert-sorted row and, when requested, to its packed row.
__global__ void __launch_bounds__(256) scatter_rows_kernel(ScatterArgs p)
{
    constexpr int U = 4;
    const int lane = threadIdx.x & 31;
    const int nvec = p.d >> 3;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < p.N; t += nwarps) {
        int r = -1;
        long long pk = -1;
        if (lane < p.K) {
            const int a = t * p.K + lane;
            r = p.row_of[a];
            if (r >= 0 && p.x_packed) {
                const int e = p.topk_idx[a];
                pk = p.pk_base[(size_t)e * p.W + t / p.S] + (r - p.offsets[e]);
            }
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (size_t)t * p.d);
        uint4 *dst_s = reinterpret_cast<uint4 *>(p.x_sorted);
        uint4 *dst_p = reinterpret_cast<uint4 *>(p.x_packed);
        // every lane runs every iteration: the shuffles below read lanes 0..K-1
        for (int c0 = 0; c0 < nvec; c0 += 32 * U) {
            const int c = c0 + lane;
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c + 32 * u < nvec)
                    v[u] = __ldcs(src + c + 32 * u);
            for (int k = 0; k < p.K; ++k) {
                const int rk = __shfl_sync(0xffffffffu, r, k);
                const long long pkk = __shfl_sync(0xffffffffu, pk, k);
                if (rk < 0)
                    continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c + 32 * u < nvec) {
                        dst_s[(size_t)rk * nvec + c + 32 * u] = v[u];
                        if (pkk >= 0)
                            dst_p[(size_t)pkk * nvec + c + 32 * u] = v[u];
                    }
                }
            }
        }
    }
}

}  // namespace moe
