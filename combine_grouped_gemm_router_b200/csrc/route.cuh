// Router projection and softmax top-K.
//
// [MoE Inference Communication, §DeepSpeed-MoE › MoE 计算核优化] fuses the gate's
// top-k with the cumsum/scatter that follow; here the gate is two kernels
// (logits, then selection) and the cumsum/scatter live in dispatch.cuh.
//
// Logits are defined as one fp32 fused multiply-add per input element in
// ascending i, from +0, then + bias. That order is kept exactly: the kernel is a
// SIMT fp32 tile in which each thread owns whole outputs and walks d in order,
// so logits are bit-identical to any IEEE implementation of the same chain and
// the integer top-K decision is reproducible.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kLogitKC = 32;  // d-chunk staged in shared memory per step

// CTA tile: BT = TY*TT tokens x BE = TX*TE experts, TY*TX threads.
// Thread (ty, tx) owns tokens ty*TT + i (contiguous, float4 reads) and experts
// tx + TX*j (strided, conflict-free scalar reads).
template <int TY, int TX, int TT, int TE>
__global__ void __launch_bounds__(TY *TX)
    router_logits_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr,
                         const float *__restrict__ bias, float *__restrict__ logits, int N, int d,
                         int E)
{
    static_assert(TT % 4 == 0, "tokens per thread must be a multiple of 4");
    constexpr int NT = TY * TX;
    constexpr int BT = TY * TT;
    constexpr int BE = TX * TE;
    constexpr int KC = kLogitKC;
    constexpr int XS = BT + 4;  // keeps float4 alignment of every row
    __shared__ __align__(16) float xs[KC][XS];
    __shared__ float ws[KC][BE];

    const int tid = threadIdx.x;
    const int ty = tid / TX, tx = tid % TX;
    const int t0 = blockIdx.x * BT;
    const int e0 = blockIdx.y * BE;

    float acc[TT][TE];
#pragma unroll
    for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j)
            acc[i][j] = 0.0f;

    for (int k0 = 0; k0 < d; k0 += KC) {
        const int kc = min(KC, d - k0);  // a multiple of 8 (d % 8 == 0)
        for (int idx = tid; idx < BT * (KC / 8); idx += NT) {
            const int row = idx % BT, c8 = idx / BT;
            const int t = t0 + row;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < N && c8 * 8 < kc)
                v = *reinterpret_cast<const uint4 *>(x + (size_t)t * d + k0 + c8 * 8);
            xs[c8 * 8 + 0][row] = bf16_lo(v.x);
            xs[c8 * 8 + 1][row] = bf16_hi(v.x);
            xs[c8 * 8 + 2][row] = bf16_lo(v.y);
            xs[c8 * 8 + 3][row] = bf16_hi(v.y);
            xs[c8 * 8 + 4][row] = bf16_lo(v.z);
            xs[c8 * 8 + 5][row] = bf16_hi(v.z);
            xs[c8 * 8 + 6][row] = bf16_lo(v.w);
            xs[c8 * 8 + 7][row] = bf16_hi(v.w);
        }
        for (int idx = tid; idx < BE * (KC / 4); idx += NT) {
            const int col = idx % BE, c4 = idx / BE;
            const int e = e0 + col;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e < E && c4 * 4 < kc)
                v = *reinterpret_cast<const float4 *>(wr + (size_t)e * d + k0 + c4 * 4);
            ws[c4 * 4 + 0][col] = v.x;
            ws[c4 * 4 + 1][col] = v.y;
            ws[c4 * 4 + 2][col] = v.z;
            ws[c4 * 4 + 3][col] = v.w;
        }
        __syncthreads();
        for (int kk = 0; kk < kc; ++kk) {
            float a[TT], b[TE];
#pragma unroll
            for (int i = 0; i < TT; i += 4) {
                const float4 q = *reinterpret_cast<const float4 *>(&xs[kk][ty * TT + i]);
                a[i] = q.x;
                a[i + 1] = q.y;
                a[i + 2] = q.z;
                a[i + 3] = q.w;
            }
#pragma unroll
            for (int j = 0; j < TE; ++j)
                b[j] = ws[kk][tx + TX * j];
#pragma unroll
            for (int i = 0; i < TT; ++i)
#pragma unroll
                for (int j = 0; j < TE; ++j)
                    acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
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

// One warp per token. Lane l holds logits of experts l + 32*j (E <= 256).
// K rounds of a warp-wide argmax on (value desc, expert asc); then a softmax over
// the K picked logits. NaN is treated as -inf for the choice; any non-finite
// logit flags MOE_ERR_NONFINITE (the token's result is then unspecified).
__global__ void __launch_bounds__(256)
    topk_softmax_kernel(const float *__restrict__ logits, int N, int E, int K,
                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                        unsigned long long *nonfinite_count)
{
    constexpr int MAXJ = 8;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= N)
        return;
    const float *lrow = logits + (size_t)t * E;
    float v[MAXJ];
    unsigned taken = 0;  // bit j: entry j unavailable (chosen or absent)
    bool bad = false;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int e = lane + 32 * j;
        if (e < E) {
            float l = lrow[e];
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
    const float s = warp_sum(ex);
    if (lane < K) {
        topk_idx[(size_t)t * K + lane] = my_e;
        topk_w[(size_t)t * K + lane] = ex / s;
    }
}

}  // namespace moe
