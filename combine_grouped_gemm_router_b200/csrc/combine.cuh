// Weighted combine, inter-layer affinity counts, and the bounded-wait probe.
#pragma once

#include "common.cuh"

namespace moe {

// [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制, node I] weighted
// merge of the K expert outputs back into the original token order;
// [MoE 推理服务工程真相 2026, §2.2] a dropped slot's router output is zero.
// One warp per token; each lane owns 16-byte column chunks; the K rows are
// gathered (fp32 expert outputs) and accumulated in fp32 in slot order
// k = 0..K-1. Then, optionally and in this order, the fp32 output of a shared
// dense MLP is added ([MoE Inference Communication, §PR-MoE]: Residual-MoE adds
// the shared MLP's and the routed experts' outputs) and a bf16 residual row (the
// inter-layer step of a stack of MoE layers, x_{j+1} = x_j + MoE_j(x_j)). The
// result is stored as fp32, or rounded once to bf16 (OUT_BF16).
// A warp's work item is one token and `seg` 8-column chunks of its row (the whole
// row for large N; a slice when there are too few tokens to fill the GPU).
// YK: how the expert outputs arrive: 0 fp32 rows; 1 the FP8 return payload (rows of y_stride
// bytes: d e4m3 codes, then one exponent byte j + 127 per 32 columns); 2 the fp16 payload (2d
// bytes of fp16 codes, then the exponent bytes). A payload value is decoded exactly (code ->
// f32, times 2^j) before the same fp32 accumulation.
__device__ __forceinline__ float f16_to_f32(uint32_t h)
{
    float f;
    asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"((unsigned short)h));
    return f;
}

// Eight e4m3 codes (bytes of lo, then hi) -> eight floats scaled by sc (a power of two).
__device__ __forceinline__ void decode_e4m3x8(uint32_t lo, uint32_t hi, float sc, float o[8])
{
    const uint32_t w[2] = {lo, hi};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        uint32_t a, b;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(a) : "h"((unsigned short)(w[i] & 0xFFFFu)));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(b) : "h"((unsigned short)(w[i] >> 16)));
        o[4 * i] = f16_to_f32(a & 0xFFFFu) * sc;
        o[4 * i + 1] = f16_to_f32(a >> 16) * sc;
        o[4 * i + 2] = f16_to_f32(b & 0xFFFFu) * sc;
        o[4 * i + 3] = f16_to_f32(b >> 16) * sc;
    }
}

template <bool OUT_BF16, int YK>
__global__ void __launch_bounds__(256)
    combine_kernel(const void *__restrict__ y, int y_stride, const int32_t *__restrict__ row_of,
                   const float *__restrict__ topk_w, const float *__restrict__ shared_y,
                   const uint16_t *__restrict__ residual, int N, int d, int K, int seg,
                   void *__restrict__ out)
{
    constexpr int U = 2;
    const int lane = threadIdx.x & 31;
    const int nvec = d >> 3;  // 8-column chunks
    const int nseg = (nvec + seg - 1) / seg;
    const int64_t items = (int64_t)N * nseg;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const float4 *ysrc = reinterpret_cast<const float4 *>(y);
    for (int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
         item < items; item += nwarps) {
        const int t = (int)(item / nseg);
        const int cbeg = (int)(item % nseg) * seg, cend = min(nvec, cbeg + seg);
        int r = -1;
        float w = 0.0f;
        if (lane < K) {
            r = row_of[(size_t)t * K + lane];
            w = topk_w[(size_t)t * K + lane];
        }
        // every lane runs every iteration: the shuffles below read lanes 0..K-1
        for (int c0 = cbeg; c0 < cend; c0 += 32 * U) {
            const int c = c0 + lane;
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    acc[u][q] = 0.0f;
            for (int k = 0; k < K; ++k) {
                const int rk = __shfl_sync(0xffffffffu, r, k);
                const float wk = __shfl_sync(0xffffffffu, w, k);
                if (rk < 0)
                    continue;
                if constexpr (YK == 2) {
                    const uint8_t *prow = reinterpret_cast<const uint8_t *>(y) +
                                          (size_t)rk * y_stride;
                    uint4 v[U];
                    uint32_t ex[U];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c + 32 * u < cend) {
                            v[u] = reinterpret_cast<const uint4 *>(prow)[c + 32 * u];
                            ex[u] = prow[2 * d + (c + 32 * u) / 4];
                        }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        if (c + 32 * u < cend) {
                            const float sc = pow2f((int)ex[u] - 127);
                            const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                acc[u][2 * q] = __fmaf_rn(wk, f16_to_f32(w4[q] & 0xFFFFu) * sc,
                                                          acc[u][2 * q]);
                                acc[u][2 * q + 1] = __fmaf_rn(wk, f16_to_f32(w4[q] >> 16) * sc,
                                                              acc[u][2 * q + 1]);
                            }
                        }
                    }
                } else if constexpr (YK == 1) {
                    const uint8_t *prow = reinterpret_cast<const uint8_t *>(y) +
                                          (size_t)rk * y_stride;
                    uint2 v[U];
                    uint32_t ex[U];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c + 32 * u < cend) {
                            v[u] = reinterpret_cast<const uint2 *>(prow)[c + 32 * u];
                            ex[u] = prow[d + (c + 32 * u) / 4];
                        }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        if (c + 32 * u < cend) {
                            float f8[8];
                            decode_e4m3x8(v[u].x, v[u].y, pow2f((int)ex[u] - 127), f8);
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                acc[u][q] = __fmaf_rn(wk, f8[q], acc[u][q]);
                        }
                    }
                } else {
                    float4 v[U][2];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c + 32 * u < cend) {
                            v[u][0] = ysrc[((size_t)rk * nvec + c + 32 * u) * 2];
                            v[u][1] = ysrc[((size_t)rk * nvec + c + 32 * u) * 2 + 1];
                        }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        if (c + 32 * u < cend) {
                            const float f8[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                                                 v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                acc[u][q] = __fmaf_rn(wk, f8[q], acc[u][q]);
                        }
                    }
                }
            }
            if (shared_y) {
                const float4 *ssrc = reinterpret_cast<const float4 *>(shared_y);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c + 32 * u < cend) {
                        const size_t chunk = (size_t)t * nvec + c + 32 * u;
                        const float4 a = ssrc[chunk * 2], b = ssrc[chunk * 2 + 1];
                        const float f8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            acc[u][q] = __fadd_rn(acc[u][q], f8[q]);
                    }
                }
            }
            if (residual) {
                const uint4 *rsrc = reinterpret_cast<const uint4 *>(residual);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c + 32 * u < cend) {
                        const uint4 rv = rsrc[(size_t)t * nvec + c + 32 * u];
                        const uint32_t q4[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            acc[u][2 * q] = __fadd_rn(acc[u][2 * q], bf16_lo(q4[q]));
                            acc[u][2 * q + 1] = __fadd_rn(acc[u][2 * q + 1], bf16_hi(q4[q]));
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (c + 32 * u < cend) {
                    const size_t chunk = (size_t)t * nvec + c + 32 * u;
                    if (OUT_BF16) {
                        uint4 o;
                        o.x = pack_bf16x2(acc[u][0], acc[u][1]);
                        o.y = pack_bf16x2(acc[u][2], acc[u][3]);
                        o.z = pack_bf16x2(acc[u][4], acc[u][5]);
                        o.w = pack_bf16x2(acc[u][6], acc[u][7]);
                        reinterpret_cast<uint4 *>(out)[chunk] = o;
                    } else {
                        float4 *o = reinterpret_cast<float4 *>(out) + chunk * 2;
                        o[0] = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
                        o[1] = make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
                    }
                }
            }
        }
    }
}

// [MoE Inference Communication, §ExFlow 核心发现：跨层专家亲和性] counts of
// (expert i at layer j, expert p at layer j+1) over every token's top-K pairs.
// Block-private shared counters when E*E fits, else global atomics.
__global__ void __launch_bounds__(256)
    affinity_kernel(const int32_t *__restrict__ a, const int32_t *__restrict__ b, int N, int E,
                    int K, unsigned long long *__restrict__ cnt, int use_smem)
{
    extern __shared__ unsigned int s_cnt[];
    if (use_smem) {
        for (int i = threadIdx.x; i < E * E; i += blockDim.x)
            s_cnt[i] = 0;
        __syncthreads();
    }
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < N; t += gridDim.x * blockDim.x) {
        for (int k = 0; k < K; ++k) {
            const int i = a[(size_t)t * K + k];
            if ((unsigned)i >= (unsigned)E) {
                set_dev_error(MOE_ERR_DEVICE_BOUNDS);
                continue;
            }
            for (int q = 0; q < K; ++q) {
                const int pe = b[(size_t)t * K + q];
                if ((unsigned)pe >= (unsigned)E) {
                    set_dev_error(MOE_ERR_DEVICE_BOUNDS);
                    continue;
                }
                if (use_smem)
                    atomicAdd(&s_cnt[i * E + pe], 1u);
                else
                    atomicAdd(&cnt[(size_t)i * E + pe], 1ull);
            }
        }
    }
    if (use_smem) {
        __syncthreads();
        for (int i = threadIdx.x; i < E * E; i += blockDim.x)
            if (s_cnt[i])
                atomicAdd(&cnt[i], (unsigned long long)s_cnt[i]);
    }
}

// A flag that no code ever sets: the bounded-wait probe waits on it.
__device__ unsigned int g_never_set;

__global__ void bounded_wait_probe_kernel(uint64_t timeout_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (*reinterpret_cast<volatile unsigned int *>(&g_never_set) == 0u) {
        if (global_timer_ns() - t0 > timeout_ns) {
            set_dev_error(MOE_ERR_DEVICE_TIMEOUT);
            return;
        }
        __nanosleep(1000);
    }
}

}  // namespace moe
