// Router projection and softmax top-K.
//
// [MoE Inference Communication, §DeepSpeed-MoE › MoE 计算核优化] fuses the gate's
// top-k with the cumsum/scatter that follow. Here, with many tokens and E >= 32, the
// projection and the selection are one kernel (router_topk_kernel for E = 32,
// router_split_kernel after router_transpose_kernel for E > 32); otherwise they are two
// (router_logits_kernel, then topk_softmax_kernel). The cumsum/scatter live in dispatch.cuh.
//
// Logits are defined as one fp32 fused multiply-add per input element in
// ascending i, from +0, then + bias. That order is kept exactly: the kernel is a
// SIMT fp32 tile in which each thread owns whole outputs and walks d in order,
// so logits are bit-identical to any IEEE implementation of the same chain and
// the integer top-K decision is reproducible.
#pragma once

#include "common.cuh"

namespace moe {

// CTA tile: BT = TY*TT tokens x BE = TX*TE experts, TY*TX threads; d walked in
// chunks of KC staged by cp.async into an S-deep shared-memory ring, so the
// global-memory latency of later chunks overlaps the FMAs of earlier ones.
// Thread (ty, tx) owns tokens ty*TT + i and experts tx + TX*j; per 8 elements of
// d it reads one 16-byte bf16 vector per token and two 16-byte fp32 vectors per
// expert, then runs the 8 fused multiply-adds of every owned output in i order.
template <int TY, int TX, int TT, int TE, int KC, int S>
struct LogitTile {
    static constexpr int NT = TY * TX;
    static constexpr int BT = TY * TT;
    static constexpr int BE = TX * TE;
    static constexpr int XROW = KC + 8;  // bf16 per staged x row (16-byte pad: no bank conflicts)
    static constexpr int WROW = KC + 4;  // fp32 per staged Wr row (16-byte pad)
    static constexpr int X_BYTES = BT * XROW * 2;
    static constexpr int W_BYTES = BE * WROW * 4;
    static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
    static constexpr int SMEM_BYTES = S * STAGE_BYTES;
};

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Stages chunk c of d (x rows of the CTA's tokens, Wr rows of its experts) into ring
// slot c % S with cp.async; always commits a group (possibly empty) so that every
// thread's group count stays uniform.
template <class L, int KC, int S>
__device__ __forceinline__ void stage_logit_chunk(unsigned char *smem, int c, int nchunks,
                                                  const uint16_t *__restrict__ x,
                                                  const float *__restrict__ wr, int t0, int e0,
                                                  int N, int d, int E)
{
    const int tid = threadIdx.x;
    if (c < nchunks) {
        unsigned char *st = smem + (c % S) * L::STAGE_BYTES;
        uint16_t *xs = reinterpret_cast<uint16_t *>(st);
        float *ws = reinterpret_cast<float *>(st + L::X_BYTES);
        const int k0 = c * KC;
        const int kc = min(KC, d - k0);  // a multiple of 8 (d % 8 == 0)
        for (int idx = tid; idx < L::BT * (KC / 8); idx += L::NT) {
            const int row = idx / (KC / 8), v = idx % (KC / 8);
            if (t0 + row < N && v * 8 < kc)
                cp_async16(xs + row * L::XROW + v * 8, x + (size_t)(t0 + row) * d + k0 + v * 8);
        }
        for (int idx = tid; idx < L::BE * (KC / 4); idx += L::NT) {
            const int row = idx / (KC / 4), v = idx % (KC / 4);
            if (e0 + row < E && v * 4 < kc)
                cp_async16(ws + row * L::WROW + v * 4, wr + (size_t)(e0 + row) * d + k0 + v * 4);
        }
    }
    cp_async_commit();
}

template <int TY, int TX, int TT, int TE, int KC, int S>
__global__ void __launch_bounds__(TY *TX)
    router_logits_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr,
                         const float *__restrict__ bias, float *__restrict__ logits, int N, int d,
                         int E)
{
    using L = LogitTile<TY, TX, TT, TE, KC, S>;
    static_assert(KC % 8 == 0, "chunk must hold whole 16-byte vectors");
    extern __shared__ __align__(16) unsigned char logit_smem[];
    const int tid = threadIdx.x;
    const int ty = tid / TX, tx = tid % TX;
    const int t0 = blockIdx.x * L::BT;
    const int e0 = blockIdx.y * L::BE;
    const int nchunks = (d + KC - 1) / KC;
    auto issue = [&](int c) {
        stage_logit_chunk<L, KC, S>(logit_smem, c, nchunks, x, wr, t0, e0, N, d, E);
    };

    float acc[TT][TE];
#pragma unroll
    for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j)
            acc[i][j] = 0.0f;

#pragma unroll
    for (int c = 0; c < S - 1; ++c)
        issue(c);
    for (int c = 0; c < nchunks; ++c) {
        cp_async_wait<S - 2>();
        __syncthreads();
        issue(c + S - 1);
        const unsigned char *st = logit_smem + (c % S) * L::STAGE_BYTES;
        const uint16_t *xs = reinterpret_cast<const uint16_t *>(st);
        const float *ws = reinterpret_cast<const float *>(st + L::X_BYTES);
        const int kc = min(KC, d - c * KC);
        for (int kk = 0; kk < kc; kk += 8) {
            float xv[TT][8];
#pragma unroll
            for (int i = 0; i < TT; ++i) {
                const uint4 q = *reinterpret_cast<const uint4 *>(xs + (ty * TT + i) * L::XROW + kk);
                xv[i][0] = bf16_lo(q.x);
                xv[i][1] = bf16_hi(q.x);
                xv[i][2] = bf16_lo(q.y);
                xv[i][3] = bf16_hi(q.y);
                xv[i][4] = bf16_lo(q.z);
                xv[i][5] = bf16_hi(q.z);
                xv[i][6] = bf16_lo(q.w);
                xv[i][7] = bf16_hi(q.w);
            }
#pragma unroll
            for (int j = 0; j < TE; ++j) {
                const float *wrow = ws + (tx + TX * j) * L::WROW + kk;
                const float4 a = *reinterpret_cast<const float4 *>(wrow);
                const float4 b = *reinterpret_cast<const float4 *>(wrow + 4);
                const float wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int q = 0; q < 8; ++q)
#pragma unroll
                    for (int i = 0; i < TT; ++i)
                        acc[i][j] = __fmaf_rn(xv[i][q], wv[q], acc[i][j]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < TT; ++i) {
        const int t = t0 + ty * TT + i;
#pragma unroll
        for (int j = 0; j < TE; ++j) {
            const int e = e0 + tx + TX * j;
            if (t < N && e < E) {
                float v = acc[i][j];
                if (bias)
                    v = __fadd_rn(v, bias[e]);
                logits[(size_t)t * E + e] = v;
            }
        }
    }
}

// The same tile with two tokens per instruction: the accumulators of tokens (2p, 2p+1)
// for one expert form a pair, updated by one packed fp32 FMA (`__ffma2_rn`). Each half of
// a packed FMA is rounded exactly like one fmaf, and every chain still walks d in order,
// so the logits are the same bits as router_logits_kernel's. Halving the FMA instructions
// frees issue slots where a thread owns many outputs (large N, E > 32).
template <int TY, int TX, int TT, int TE, int KC, int S>
__global__ void __launch_bounds__(TY *TX)
    router_logits_pairs_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr,
                               const float *__restrict__ bias, float *__restrict__ logits, int N,
                               int d, int E)
{
    using L = LogitTile<TY, TX, TT, TE, KC, S>;
    static_assert(KC % 8 == 0 && TT % 2 == 0, "whole 16-byte vectors, token pairs");
    extern __shared__ __align__(16) unsigned char logit_smem[];
    const int tid = threadIdx.x;
    const int ty = tid / TX, tx = tid % TX;
    const int t0 = blockIdx.x * L::BT;
    const int e0 = blockIdx.y * L::BE;
    const int nchunks = (d + KC - 1) / KC;

    float2 acc[TT / 2][TE];
#pragma unroll
    for (int i = 0; i < TT / 2; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j)
            acc[i][j] = make_float2(0.0f, 0.0f);

#pragma unroll
    for (int c = 0; c < S - 1; ++c)
        stage_logit_chunk<L, KC, S>(logit_smem, c, nchunks, x, wr, t0, e0, N, d, E);
    for (int c = 0; c < nchunks; ++c) {
        cp_async_wait<S - 2>();
        __syncthreads();
        stage_logit_chunk<L, KC, S>(logit_smem, c + S - 1, nchunks, x, wr, t0, e0, N, d, E);
        const unsigned char *st = logit_smem + (c % S) * L::STAGE_BYTES;
        const uint16_t *xs = reinterpret_cast<const uint16_t *>(st);
        const float *ws = reinterpret_cast<const float *>(st + L::X_BYTES);
        const int kc = min(KC, d - c * KC);
        for (int kk = 0; kk < kc; kk += 8) {
            float2 xv[TT / 2][8];
#pragma unroll
            for (int p = 0; p < TT / 2; ++p) {
                const uint4 a =
                    *reinterpret_cast<const uint4 *>(xs + (ty * TT + 2 * p) * L::XROW + kk);
                const uint4 b =
                    *reinterpret_cast<const uint4 *>(xs + (ty * TT + 2 * p + 1) * L::XROW + kk);
                xv[p][0] = make_float2(bf16_lo(a.x), bf16_lo(b.x));
                xv[p][1] = make_float2(bf16_hi(a.x), bf16_hi(b.x));
                xv[p][2] = make_float2(bf16_lo(a.y), bf16_lo(b.y));
                xv[p][3] = make_float2(bf16_hi(a.y), bf16_hi(b.y));
                xv[p][4] = make_float2(bf16_lo(a.z), bf16_lo(b.z));
                xv[p][5] = make_float2(bf16_hi(a.z), bf16_hi(b.z));
                xv[p][6] = make_float2(bf16_lo(a.w), bf16_lo(b.w));
                xv[p][7] = make_float2(bf16_hi(a.w), bf16_hi(b.w));
            }
#pragma unroll
            for (int j = 0; j < TE; ++j) {
                const float *wrow = ws + (tx + TX * j) * L::WROW + kk;
                const float4 a = *reinterpret_cast<const float4 *>(wrow);
                const float4 b = *reinterpret_cast<const float4 *>(wrow + 4);
                const float wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float2 w2 = make_float2(wv[q], wv[q]);
#pragma unroll
                    for (int p = 0; p < TT / 2; ++p)
                        acc[p][j] = __ffma2_rn(xv[p][q], w2, acc[p][j]);
                }
            }
        }
    }
#pragma unroll
    for (int p = 0; p < TT / 2; ++p)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int t = t0 + ty * TT + 2 * p + h;
#pragma unroll
            for (int j = 0; j < TE; ++j) {
                const int e = e0 + tx + TX * j;
                if (t < N && e < E) {
                    float v = h ? acc[p][j].y : acc[p][j].x;
                    if (bias)
                        v = __fadd_rn(v, bias[e]);
                    logits[(size_t)t * E + e] = v;
                }
            }
        }
}

// ---------------------------------------------------------------------------
// Top-K selection of one token by one warp: lane l holds the logits of experts l + 32 j
// (j < MAXJ, E <= 32 MAXJ). K rounds of a warp-wide argmax on (value desc, expert asc), then a
// softmax over the K picked logits. NaN counts as -inf for the choice; any non-finite logit
// flags MOE_ERR_NONFINITE (the token's result is then unspecified). lrow: the token's logits
// (shared or global memory); logits_out (nullable): where to copy them.
template <int MAXJ>
__device__ __forceinline__ void topk_select_warp(const float *lrow, int E, int K, size_t t,
                                                 float *logits_out, int32_t *__restrict__ topk_idx,
                                                 float *__restrict__ topk_w,
                                                 unsigned long long *nonfinite_count)
{
    const int lane = threadIdx.x & 31;
    float v[MAXJ];
    unsigned taken = 0;  // bit j: entry j unavailable (chosen or absent)
    bool bad = false;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int e = lane + 32 * j;
        if (e < E) {
            float l = lrow[e];
            if (logits_out)
                logits_out[t * E + e] = l;
            if (!isfinite(l)) {
                bad = true;
                if (isnan(l))
                    l = -INFINITY;
            }
            v[j] = l;
        } else {
            v[j] = -INFINITY;
            taken |= 1u << j;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) {
        set_dev_error(MOE_ERR_NONFINITE);
        if (nonfinite_count)
            atomicAdd(nonfinite_count, 1ull);
    }
    float my_v = 0.0f;
    int my_e = 0;
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
            const int e = lane + 32 * j;
            if (!((taken >> j) & 1u) && (v[j] > bv || (v[j] == bv && e < be))) {
                bv = v[j];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane)
            taken |= 1u << (be >> 5);
        if (lane == k) {
            my_v = bv;
            my_e = be;
        }
    }
    const float top = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = lane < K ? expf(my_v - top) : 0.0f;
    const float ssum = warp_sum(ex);
    if (lane < K) {
        topk_idx[t * K + lane] = my_e;
        topk_w[t * K + lane] = ex / ssum;
    }
}

// ---------------------------------------------------------------------------
// Router projection fused with the top-K selection, broadcast form (many tokens, E = 32).
//
// [MoE Inference Communication, §DeepSpeed-MoE › MoE 计算核优化] the gate's top-k runs
// in the same kernel as the projection: the [N][E] logits need not go to HBM.
//
// A CTA takes 32 TT tokens and every expert. Lane l of every warp owns tokens l, l + 32, ... of
// the tile, and warp w owns experts [16w, 16w + 16), so the W values a warp needs are the same
// for all its lanes (broadcast shared-memory loads) and each lane's x values are its own. The
// 8-element pieces of d are walked in order; per element i a lane forms (x_t[i], x_t[i]) and
// multiplies it by two neighbouring experts' (W_e[i], W_e+1[i]) in one packed fp32 FMA
// (`__ffma2_rn`: each half rounds like one fmaf), so every logit is still the single ascending
// fmaf chain, bit for bit. W is staged transposed ([i][e]) so that one 16-byte load gives four
// experts' weights of one element; the transposition happens on the way through registers,
// one chunk ahead of its use. After the chain, the tile's logits go to shared memory and each
// warp selects the top K of its tokens: K rounds of a warp-wide argmax on (value desc, expert
// asc), then a softmax over the K picked logits, as topk_softmax_kernel does.
constexpr int kRtKC = 32;      // elements of d per staged chunk
constexpr int kRtXRow = kRtKC + 8;  // bf16 per staged x row (16-byte pad)

template <int NW, int TT, int EW>
struct RouterTopkTile {
    static constexpr int NT = 32 * NW;
    static constexpr int TOK = 32 * TT;     // tokens per CTA
    static constexpr int EP = EW * NW + 4;  // fp32 per staged W^T row (16-byte pad)
    static constexpr int X_BYTES = TOK * kRtXRow * 2;
    static constexpr int W_BYTES = kRtKC * EP * 4;
    static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
    static constexpr int LOGIT_BYTES = TOK * (EW * NW + 1) * 4;  // epilogue tile
    static constexpr int SMEM_BYTES =
        2 * STAGE_BYTES > LOGIT_BYTES ? 2 * STAGE_BYTES : LOGIT_BYTES;
    // W elements each thread carries from global memory to the next stage: E_pad x KC / NT
    static constexpr int WV = (EW * NW * kRtKC) / (4 * NT);  // float4 per thread
};

template <int NW, int TT, int EW>
__global__ void __launch_bounds__(32 * NW)
    router_topk_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr,
                       const float *__restrict__ bias, int N, int d, int E, int K,
                       int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                       float *__restrict__ logits, unsigned long long *nonfinite_count)
{
    using L = RouterTopkTile<NW, TT, EW>;
    constexpr int kRtTokens = L::TOK;
    extern __shared__ __align__(16) unsigned char rt_smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * kRtTokens;
    const int nchunks = (d + kRtKC - 1) / kRtKC;
    const int EC = EW * NW;  // experts covered (E rounded up to EW per warp)

    // x chunk c -> stage s (cp.async, 16 bytes per copy; rows past N are left alone)
    auto stage_x = [&](int c, int s) {
        if (c < nchunks) {
            uint16_t *xs = reinterpret_cast<uint16_t *>(rt_smem + s * L::STAGE_BYTES);
            const int k0 = c * kRtKC, kc = min(kRtKC, d - k0);
            for (int idx = tid; idx < kRtTokens * (kRtKC / 8); idx += L::NT) {
                const int row = idx / (kRtKC / 8), v = idx % (kRtKC / 8);
                if (t0 + row < N && v * 8 < kc)
                    cp_async16(xs + row * kRtXRow + v * 8, x + (size_t)(t0 + row) * d + k0 + v * 8);
            }
        }
        cp_async_commit();
    };
    // W chunk c -> registers: thread holds float4 pieces (expert e, elements 4q .. 4q+3)
    float4 wreg[L::WV];
    auto load_w = [&](int c) {
        const int k0 = c * kRtKC, kc = c < nchunks ? min(kRtKC, d - k0) : 0;
#pragma unroll
        for (int j = 0; j < L::WV; ++j) {
            const int idx = tid + j * L::NT;  // over EC x (KC / 4), element quad fastest
            const int e = idx / (kRtKC / 4), q = idx % (kRtKC / 4);
            wreg[j] = (e < E && q * 4 < kc)
                          ? __ldg(reinterpret_cast<const float4 *>(wr + (size_t)e * d + k0) + q)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    // registers -> stage s, transposed to [i][e]
    auto store_w = [&](int s) {
        float *ws = reinterpret_cast<float *>(rt_smem + s * L::STAGE_BYTES + L::X_BYTES);
#pragma unroll
        for (int j = 0; j < L::WV; ++j) {
            const int idx = tid + j * L::NT;
            const int e = idx / (kRtKC / 4), q = idx % (kRtKC / 4);
            ws[(4 * q + 0) * L::EP + e] = wreg[j].x;
            ws[(4 * q + 1) * L::EP + e] = wreg[j].y;
            ws[(4 * q + 2) * L::EP + e] = wreg[j].z;
            ws[(4 * q + 3) * L::EP + e] = wreg[j].w;
        }
    };

    float2 acc[TT][EW / 2];  // [token of the lane][expert pair of the warp]
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int p = 0; p < EW / 2; ++p)
            acc[t][p] = make_float2(0.0f, 0.0f);

    stage_x(0, 0);
    load_w(0);
    store_w(0);
    load_w(1);
    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        cp_async_wait<0>();
        __syncthreads();  // stage s complete (x by cp.async, W by the stores); stage s^1 free
        stage_x(c + 1, s ^ 1);
        const uint16_t *xs = reinterpret_cast<const uint16_t *>(rt_smem + s * L::STAGE_BYTES);
        const float *ws = reinterpret_cast<const float *>(rt_smem + s * L::STAGE_BYTES + L::X_BYTES);
        const int kc = min(kRtKC, d - c * kRtKC);
        for (int kk = 0; kk < kc; kk += 8) {
            uint4 xq[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t)
                xq[t] = *reinterpret_cast<const uint4 *>(xs + (lane + 32 * t) * kRtXRow + kk);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float *wrow = ws + (kk + q) * L::EP + EW * warp;
                float2 wp[EW / 2];
#pragma unroll
                for (int h = 0; h < EW / 4; ++h) {
                    const float4 v = *reinterpret_cast<const float4 *>(wrow + 4 * h);
                    wp[2 * h] = make_float2(v.x, v.y);
                    wp[2 * h + 1] = make_float2(v.z, v.w);
                }
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    const uint32_t word = (q < 2) ? xq[t].x : (q < 4) ? xq[t].y : (q < 6) ? xq[t].z : xq[t].w;
                    const float2 xx = (q & 1) ? prmt_pair<0x3244>(word) : prmt_pair<0x1044>(word);
#pragma unroll
                    for (int p = 0; p < EW / 2; ++p)
                        acc[t][p] = __ffma2_rn(xx, wp[p], acc[t][p]);
                }
            }
        }
        store_w(s ^ 1);  // chunk c + 1 (loaded one iteration ago) into the free stage
        load_w(c + 2);
    }
    cp_async_wait<0>();
    __syncthreads();  // every warp is done with the stages: the logit tile may reuse them

    // logits of the tile -> shared memory [token][expert] (row of EC + 1 floats)
    float *lt = reinterpret_cast<float *>(rt_smem);
    const int LR = EC + 1;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        const int tok = lane + 32 * t;
#pragma unroll
        for (int p = 0; p < EW / 2; ++p) {
            const int e = EW * warp + 2 * p;
            float a = acc[t][p].x, b = acc[t][p].y;
            if (bias) {
                if (e < E)
                    a = __fadd_rn(a, bias[e]);
                if (e + 1 < E)
                    b = __fadd_rn(b, bias[e + 1]);
            }
            lt[tok * LR + e] = a;
            lt[tok * LR + e + 1] = b;
        }
    }
    __syncthreads();

    // top-K of each token: warp w takes tokens w, w + NW, ...
    for (int tok = warp; tok < kRtTokens; tok += NW) {
        const int t = t0 + tok;
        if (t >= N)
            break;
        topk_select_warp<(EW * NW + 31) / 32>(lt + tok * LR, E, K, (size_t)t, logits, topk_idx,
                                              topk_w, nonfinite_count);
    }
}

// ---------------------------------------------------------------------------
// The router weights transposed for the split-warp form: wt[i][e] = Wr[e][i] for e < E, 0 for
// E <= e < EC (a tile of 32 elements x 32 experts per 256-thread CTA, through shared memory).
__global__ void __launch_bounds__(256)
    router_transpose_kernel(const float *__restrict__ wr, int E, int d, int EC,
                            float *__restrict__ wt)
{
    __shared__ float tile[32][33];
    const int i0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) {  // r: expert, tx: element
        const int e = e0 + r, i = i0 + tx;
        tile[r][tx] = (e < E && i < d) ? wr[(size_t)e * d + i] : 0.0f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {  // r: element, tx: expert
        const int i = i0 + r, e = e0 + tx;
        if (i < d && e < EC)
            wt[(size_t)i * EC + e] = tile[tx][r];
    }
}

// Fused router, split-warp form (E > 32, many tokens). A CTA takes 64 tokens and EC = 16 NE
// experts; a warp owns 16 experts: lanes 0-15 the first 8 of them, lanes 16-31 the other 8, and
// lane j (lane mod 16) of either half owns TT tokens, 16 apart (TT = 4: one token group per
// expert group; TT = 2: two warps per expert group). A 128-bit shared-memory load is served per
// half-warp, so when the two halves read two different 16-byte words, one load gives each half
// four experts' weights of one element at the cost the whole warp pays to read one word: W costs
// 4 wavefronts per warp and element (a whole-warp broadcast of the same 16 experts pays 8). The
// arithmetic is that of the other forms: per element a lane forms (x_t[i], x_t[i]) and multiplies
// it by two neighbouring experts' (W_e[i], W_e+1[i]) in one packed FMA, so every logit is its
// single ascending fmaf chain from +0. W arrives transposed ([i][e], router_transpose_kernel), so
// both operands are staged by cp.async alone, STAGES chunks deep; the next element's W and the
// next 8 elements' x are loaded before the current element's FMAs.
constexpr int kRsTok = 64;    // tokens per CTA

// NE groups of 16 experts, TT tokens per lane, KC elements of d per staged chunk, ST chunks in
// flight.
template <int NE, int TT, int KC, int ST>
struct RouterSplitTile {
    static constexpr int TG = 4 / TT;       // token groups of 16 TT tokens
    static constexpr int NW = NE * TG;
    static constexpr int NT = 32 * NW;
    static constexpr int EC = 16 * NE;      // experts covered
    static constexpr int EP = EC + 4;       // fp32 per staged W^T row
    static constexpr int XR = KC + 8;       // bf16 per staged x row (16-byte pad: 16-byte loads
                                            // of 8 consecutive rows hit 8 different bank groups)
    static constexpr int X_BYTES = kRsTok * XR * 2;
    static constexpr int W_BYTES = KC * EP * 4;
    static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
    static constexpr int LR = EC + 1;       // fp32 per epilogue logit row
    static constexpr int LOGIT_BYTES = kRsTok * LR * 4;
    static constexpr int SMEM_BYTES =
        ST * STAGE_BYTES > LOGIT_BYTES ? ST * STAGE_BYTES : LOGIT_BYTES;
    static_assert(TG * TT == 4 && KC % 32 == 0 && ST >= 2, "tile");
};

// NB 8-element blocks of one staged chunk (NB known at compile time, so the loop is unrolled
// whole and the loads of the next element and block are scheduled across it).
template <int NB, int TT, int EP, int XR>
__device__ __forceinline__ void split_chunk(const uint16_t *xs, const float *ws, int tok0,
                                            float2 (&acc)[TT][4])
{
    uint4 xq[TT];
#pragma unroll
    for (int m = 0; m < TT; ++m)
        xq[m] = *reinterpret_cast<const uint4 *>(xs + (tok0 + 16 * m) * XR);
    float4 va = *reinterpret_cast<const float4 *>(ws);
    float4 vb = *reinterpret_cast<const float4 *>(ws + 4);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        uint4 xn[TT];
        if (b + 1 < NB) {
#pragma unroll
            for (int m = 0; m < TT; ++m)
                xn[m] = *reinterpret_cast<const uint4 *>(xs + (tok0 + 16 * m) * XR + 8 * (b + 1));
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int k = 8 * b + q;
            float4 na = va, nb = vb;
            if (k + 1 < 8 * NB) {
                na = *reinterpret_cast<const float4 *>(ws + (k + 1) * EP);
                nb = *reinterpret_cast<const float4 *>(ws + (k + 1) * EP + 4);
            }
            const float2 wp[4] = {make_float2(va.x, va.y), make_float2(va.z, va.w),
                                  make_float2(vb.x, vb.y), make_float2(vb.z, vb.w)};
#pragma unroll
            for (int m = 0; m < TT; ++m) {
                const uint32_t word = (q < 2)   ? xq[m].x
                                      : (q < 4) ? xq[m].y
                                      : (q < 6) ? xq[m].z
                                                : xq[m].w;
                const float2 xx = (q & 1) ? prmt_pair<0x3244>(word) : prmt_pair<0x1044>(word);
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    acc[m][p] = __ffma2_rn(xx, wp[p], acc[m][p]);
            }
            va = na;
            vb = nb;
        }
        if (b + 1 < NB) {
#pragma unroll
            for (int m = 0; m < TT; ++m)
                xq[m] = xn[m];
        }
    }
}

template <int NE, int TT, int KC, int ST>
__global__ void __launch_bounds__(32 * NE * (4 / TT))
    router_split_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wt,
                        const float *__restrict__ bias, int N, int d, int E, int K,
                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                        float *__restrict__ logits, unsigned long long *nonfinite_count)
{
    using L = RouterSplitTile<NE, TT, KC, ST>;
    extern __shared__ __align__(16) unsigned char rs_smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, j16 = lane & 15;
    const int t0 = blockIdx.x * kRsTok;
    const int nchunks = (d + KC - 1) / KC;

    // chunk c -> stage c mod ST (cp.async, 16 bytes per copy; x rows past N are left
    // alone, their logits are never stored): x rows [64][kc] bf16 and W^T rows [kc][EC] fp32
    auto stage = [&](int c) {
        if (c < nchunks) {
            unsigned char *base = rs_smem + (c % ST) * L::STAGE_BYTES;
            uint16_t *xs = reinterpret_cast<uint16_t *>(base);
            float *ws = reinterpret_cast<float *>(base + L::X_BYTES);
            const int k0 = c * KC, kc = min(KC, d - k0);
            for (int idx = tid; idx < kRsTok * (KC / 8); idx += L::NT) {
                const int row = idx / (KC / 8), v = idx % (KC / 8);
                if (t0 + row < N && v * 8 < kc)
                    cp_async16(xs + row * L::XR + v * 8, x + (size_t)(t0 + row) * d + k0 + v * 8);
            }
            for (int idx = tid; idx < kc * (L::EC / 4); idx += L::NT) {
                const int r = idx / (L::EC / 4), v = idx % (L::EC / 4);
                cp_async16(ws + r * L::EP + 4 * v, wt + (size_t)(k0 + r) * L::EC + 4 * v);
            }
        }
        cp_async_commit();
    };

    float2 acc[TT][4];  // [token m: tok0 + 16 m][expert pair p of the half]
#pragma unroll
    for (int m = 0; m < TT; ++m)
#pragma unroll
        for (int p = 0; p < 4; ++p)
            acc[m][p] = make_float2(0.0f, 0.0f);

    const int ecol = 16 * (warp % NE) + 8 * half;      // this half's first expert
    const int tok0 = 16 * TT * (warp / NE) + j16;       // this lane's first token
#pragma unroll
    for (int c = 0; c < ST - 1; ++c)
        stage(c);
    for (int c = 0; c < nchunks; ++c) {
        cp_async_wait<ST - 2>();
        __syncthreads();  // chunk c has landed; the stage chunk c - 1 used is free
        stage(c + ST - 1);
        const unsigned char *base = rs_smem + (c % ST) * L::STAGE_BYTES;
        const uint16_t *xs = reinterpret_cast<const uint16_t *>(base);
        const float *ws = reinterpret_cast<const float *>(base + L::X_BYTES) + ecol;
        const int kc = min(KC, d - c * KC);  // a multiple of 8
        if (kc == KC) {
            split_chunk<KC / 8, TT, L::EP, L::XR>(xs, ws, tok0, acc);
        } else {  // the ragged last chunk, 8 elements at a time
            for (int k8 = 0; k8 < kc; k8 += 8)
                split_chunk<1, TT, L::EP, L::XR>(xs + k8, ws + k8 * L::EP, tok0, acc);
        }
    }
    cp_async_wait<0>();
    __syncthreads();  // every warp is done with the stages: the logit tile may reuse them

    // logits (+ bias) of the tile -> shared memory [token][expert]
    float *lt = reinterpret_cast<float *>(rs_smem);
#pragma unroll
    for (int m = 0; m < TT; ++m) {
        const int tok = tok0 + 16 * m;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int e = ecol + 2 * p;
            float a = acc[m][p].x, b = acc[m][p].y;
            if (bias) {
                if (e < E)
                    a = __fadd_rn(a, bias[e]);
                if (e + 1 < E)
                    b = __fadd_rn(b, bias[e + 1]);
            }
            lt[tok * L::LR + e] = a;
            lt[tok * L::LR + e + 1] = b;
        }
    }
    __syncthreads();

    // top-K of each token: warp w takes tokens w, w + NW, ...
    for (int tok = warp; tok < kRsTok; tok += L::NW) {
        const int t = t0 + tok;
        if (t >= N)
            break;
        topk_select_warp<(L::EC + 31) / 32>(lt + tok * L::LR, E, K, (size_t)t, logits, topk_idx,
                                            topk_w, nonfinite_count);
    }
}

// One warp per token (E <= 256): topk_select_warp on the token's row of the [N][E] logits.
__global__ void __launch_bounds__(256)
    topk_softmax_kernel(const float *__restrict__ logits, int N, int E, int K,
                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                        unsigned long long *nonfinite_count)
{
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= N)
        return;
    topk_select_warp<8>(logits + (size_t)t * E, E, K, (size_t)t, nullptr, topk_idx, topk_w,
                        nonfinite_count);
}

}  // namespace moe
