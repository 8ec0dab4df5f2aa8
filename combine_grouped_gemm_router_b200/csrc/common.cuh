// Device helpers shared by the kernels of the MoE layer (one translation unit:
// moe_api.cu includes every .cuh).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

// Sticky per-device error word: the first kernel-side error code wins.
__device__ unsigned int g_dev_error;

__device__ __forceinline__ void set_dev_error(unsigned int code)
{
    atomicCAS(&g_dev_error, 0u, code);
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// (v, v) as the operand pair of a packed fp32 FMA, built by two byte permutes of one word with
// selector SEL (0x1044: the low bf16 of w as fp32; 0x3244: the high one; 0x3210: w itself).
// Both halves come from the integer pipe, so the pair costs no move on the FMA pipe, and one
// asm statement keeps the compiler from merging the two permutes into one register.
template <uint32_t SEL>
__device__ __forceinline__ float2 prmt_pair(uint32_t w)
{
    uint32_t a, b;
    asm("prmt.b32 %0, %2, 0, %3;\n\tprmt.b32 %1, %2, 0, %3;" : "=r"(a), "=r"(b) : "r"(w), "n"(SEL));
    return make_float2(__uint_as_float(a), __uint_as_float(b));
}

// Two fp32 -> one bf16x2 word (round to nearest even), one cvt instruction.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        T o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off)
            v += o;
    }
    return v;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v)
{
#pragma unroll
    for (int off = 16; off; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448):
// two fp32 values -> two codes, round to nearest even, saturating; lo in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Exponent j of a row's power-of-two scale: the smallest j with amax * 2^-j <= 448,
// clamped to [-126, 127]; 0 for a zero or non-finite amax. From the bits of amax
// (amax = m * 2^k, m in [1, 2)): j = k - 8 when m <= 1.75, else k - 7.
__device__ __forceinline__ int e4m3_scale_exp(float amax)
{
    if (!(amax > 0.0f) || !isfinite(amax))
        return 0;
    const uint32_t b = __float_as_uint(amax);
    int k;
    uint32_t frac;
    if (b >= 0x00800000u) {
        k = (int)(b >> 23) - 127;
        frac = b & 0x007FFFFFu;
    } else {  // subnormal: normalise the significand
        const int lz = __clz(b) - 8;
        k = -126 - lz;
        frac = (b << lz) & 0x007FFFFFu;
    }
    const int j = frac <= 0x00600000u ? k - 8 : k - 7;
    return max(-126, min(127, j));
}

// Exponent j of a block's power-of-two scale for fp16 codes: the smallest j with
// amax * 2^-j <= 65504 (fp16's largest finite value), clamped to [-126, 127]; 0 for a zero or
// non-finite amax. From the bits of amax (amax = m * 2^k, m in [1, 2)): 65504 = (2 - 2^-10) *
// 2^15, so j = k - 15 when m <= 2 - 2^-10 (fraction bits <= 0x7FE000), else k - 14.
__device__ __forceinline__ int f16_scale_exp(float amax)
{
    if (!(amax > 0.0f) || !isfinite(amax))
        return 0;
    const uint32_t b = __float_as_uint(amax);
    int k;
    uint32_t frac;
    if (b >= 0x00800000u) {
        k = (int)(b >> 23) - 127;
        frac = b & 0x007FFFFFu;
    } else {  // subnormal: normalise the significand
        const int lz = __clz(b) - 8;
        k = -126 - lz;
        frac = (b << lz) & 0x007FFFFFu;
    }
    const int j = frac <= 0x007FE000u ? k - 15 : k - 14;
    return max(-126, min(127, j));
}

// 2^j for j in [-126, 127] (a normal float).
__device__ __forceinline__ float pow2f(int j) { return __uint_as_float((uint32_t)(j + 127) << 23); }

// ---------------------------------------------------------------- mbarriers (shared::cta)

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bulk copy global -> shared memory, completing on the mbarrier at `bar` (bytes: a multiple of
// 16, both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_load_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Bounded wait on an mbarrier phase; false (and MOE_ERR_DEVICE_TIMEOUT) when it runs out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t timeout_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > timeout_ns) {
            set_dev_error(MOE_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}


// Token block b of the dispatch: blocks never straddle a home-rank shard, so
// per-shard prefix counts are available at block boundaries.
// shard = b / bps, tokens [shard*S + (b%bps)*HB, min(... + HB, (shard+1)*S)).
struct BlockMap {
    int S;    // tokens per shard (N / W)
    int bps;  // blocks per shard
    int HB;   // tokens per block
    __device__ __forceinline__ void range(int b, int &t0, int &t1) const
    {
        const int shard = b / bps;
        const int j = b - shard * bps;
        t0 = shard * S + j * HB;
        t1 = min(t0 + HB, (shard + 1) * S);
    }
};

}  // namespace moe
