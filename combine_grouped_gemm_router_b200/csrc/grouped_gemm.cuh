// Ragged grouped GEMM of the SwiGLU experts on 5th-generation tensor cores.
//
// [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制] each card groups
// its tokens by expert and runs a grouped GEMM over variable per-expert token
// counts; [§容量因子、专家复制与 dropless 的取舍] dropless routing handles the
// ragged counts directly with a grouped GEMM in a single call.
//
// Design (sm_100a):
//  - persistent kernel, one CTA per SM, 6 warps: warp 0 issues TMA loads,
//    warp 1 owns TMEM and issues tcgen05.mma, warps 2-5 are the epilogue
//    (one TMEM lane quadrant each);
//  - tile = 128 rows of one expert x BN output columns, K-steps of 64 bf16
//    (one 128-byte swizzle atom), 4-stage shared-memory ring fed by TMA;
//  - the fp32 accumulator lives in TMEM, double-buffered (2 x BN columns), so
//    the epilogue of one tile overlaps the MMAs of the next;
//  - the tile list is derived on device from the expert offsets: experts with
//    no rows have no tiles, so their weights are never read;
//  - tiles are ordered expert by expert (visiting the experts alternately from
//    both ends of the range, see visit_expert), then N-slab, then M (fastest):
//    CTAs that run at the same time share one weight slab and one expert's rows
//    in L2;
//  - rows of a tile past the expert's end are computed (they are the next
//    expert's rows or zero fill) but never stored.
// Mode 0 (gate/up): the B tile stacks 128 rows of W1 and 128 rows of W3, one
// N=256 MMA per K-step; the epilogue reads gate column c and up column 128+c
// and writes h = silu(g) * u, the next GEMM's operand, as fp16 (or bf16 when
// Args::h_f16 is 0): fp16's 11 significant bits against bf16's 8 make h's one
// rounding 8x smaller, and every value the epilogue produces is checked
// against fp16's range (65504). Mode 1 (down): h times W2 with both operands
// fp16 (or both bf16), fp32 output straight from TMEM, so the combine sums
// unrounded expert outputs (or the FP8 return payload: e4m3 codes with one
// exponent per 32 columns).
// Modes 2 and 3 (the FP8 path, [MoE 推理服务工程真相 2026, §6.3]): modes 0 and 1
// with e4m3 A and B (tcgen05 kind::f8f6f4). A 128-byte swizzle atom then holds
// 128 K elements instead of 64, so tiles, stages and descriptors keep their byte
// layout; the epilogue multiplies the accumulator by the row's scale and the
// output channel's scale (both powers of two, so the products are exact).
//
// Every mbarrier wait is bounded (globaltimer); a wait that runs out records
// MOE_ERR_DEVICE_TIMEOUT, raises a CTA-wide abort flag, and every role drains
// what it has in flight before TMEM is released.
#pragma once

#include "common.cuh"

namespace moe {
namespace gg {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int B_HALF_BYTES = 128 * BK * 2;  // 16 KB per 128-row B box
constexpr uint32_t TMEM_COLS = 512;
constexpr int THREADS = 192;

// K elements in one 128-byte swizzle atom: 64 bf16 or 128 e4m3.
__host__ __device__ constexpr bool is_e4m3(int MODE) { return MODE >= 2; }
__host__ __device__ constexpr bool is_gate(int MODE) { return MODE == 0 || MODE == 2; }
__host__ __device__ constexpr int atom_k(int MODE) { return is_e4m3(MODE) ? 128 : 64; }

struct Args {
    const int32_t *offsets;  // [E+1]
    int E;
    int n_tiles;         // N-slabs per expert
    int k_blocks;        // K / atom_k(MODE)
    int b_rows;          // rows of one expert's B matrix (f for mode 0, d for mode 1)
    int rows_alloc;      // rows of the A buffer
    int select;          // which experts this launch takes: 0 all, 1 pair-tile experts, 2 the rest
    void *out;           // modes 0, 2: bf16 h [rows_alloc][ldo]; 1, 3: fp32 y [rows_alloc][ldo],
                         // or the FP8 return payload when y_stride > 0
    int ldo;
    int y_stride;        // modes 1, 3: 0, or the payload's row stride in bytes (ldo e4m3 codes,
                         // or 2 ldo bytes of fp16 codes with y_f16, then ldo / 32 exponent
                         // bytes, padded to 16 bytes)
    int y_f16;           // the payload's codes are fp16 (else e4m3)
    const float *row_scale;  // modes 2, 3: scale of each A row [rows_alloc]
    const float *b_scale0;   // mode 2: scale of each W1 row; mode 3: of each W2 row [E * b_rows]
    const float *b_scale1;   // mode 2: scale of each W3 row [E * b_rows]
    int h_f16;               // modes 0, 1: h (mode 0's output, mode 1's A) and W2 are fp16,
                             // else bf16
    // fp16 h's range (h_f16 only): *h_amax holds the largest |h| of the launch's first pass
    // (fp32 bits; atomicMax). A second gate/up pass (h_pass 1) runs only when that exceeds
    // fp16's largest finite value: it recomputes every tile with h scaled by 2^-k, k the
    // smallest exponent that brings the largest |h| into range, and the down projection
    // multiplies its accumulators by 2^k (powers of two: both exact).
    uint32_t *h_amax;
    int h_pass;
    uint64_t timeout_ns;
};

// fp16's largest finite value.
constexpr float kF16Max = 65504.0f;

// Exponent k of the scale 2^-k that brings a largest |h| (fp32 bits) into fp16's range: 0 when
// it already is; -1 when it is not finite (nothing brings it into range).
__device__ __forceinline__ int f16_range_exp(uint32_t amax_bits)
{
    if (amax_bits >= 0x7F800000u)
        return -1;
    float t = __uint_as_float(amax_bits);
    int k = 0;
    while (t > kF16Max) {  // halving a normal fp32 value is exact
        t *= 0.5f;
        ++k;
    }
    return k;
}

// Bounded wait for the phase of parity `parity` to complete. Gives up when the
// CTA abort flag is raised (if honor_abort) or after timeout_ns, raising it.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint64_t timeout_ns, bool honor_abort = true)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (honor_abort && *abort_flag)
            return false;
        if (global_timer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            set_dev_error(MOE_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 2-D tiled bulk store shared -> global (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// This thread's bulk stores have finished reading shared memory / have completed.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// All but this thread's most recent bulk store have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// Shared-memory matrix descriptor: K-major operand in 128-byte swizzled atoms
// (8 rows x 128 bytes, atoms 1024 bytes apart), tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    uint64_t desc = 0;
    desc |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address, 16-byte units
    desc |= (uint64_t)1u << 16;                    // leading byte offset (unused: swizzled K-major)
    desc |= (uint64_t)(1024u >> 4) << 32;          // stride byte offset: 8-row group pitch
    desc |= (uint64_t)1u << 46;                    // descriptor version for sm_100
    desc |= (uint64_t)2u << 61;                    // 128-byte swizzle
    return desc;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t instr_desc_bf16(int M, int N)
{
    return (1u << 4)                          // D format: f32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Instruction descriptor, kind::f16: fp16 A and B (format code 0), fp32 accumulate.
__host__ __device__ constexpr uint32_t instr_desc_f16(int M, int N)
{
    return (1u << 4)                          // D format: f32
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format code 0), fp32 accumulate.
__host__ __device__ constexpr uint32_t instr_desc_e4m3(int M, int N)
{
    return (1u << 4)                          // D format: f32
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

template <int MODE>
__host__ __device__ constexpr uint32_t instr_desc(int M, int N)
{
    return is_e4m3(MODE) ? instr_desc_e4m3(M, N) : instr_desc_bf16(M, N);
}

// The descriptor a launch uses: the down projection (mode 1) reads fp16 h and W2 when the
// launch says so; every other case is fixed by the mode.
template <int MODE>
__device__ __forceinline__ uint32_t launch_idesc(const Args &args, int M, int N)
{
    return (MODE == 1 && args.h_f16) ? instr_desc_f16(M, N) : instr_desc<MODE>(M, N);
}

// Two fp32 -> one f16x2 word (round to nearest even; beyond 65504 becomes infinity).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Nonzero when either half of an f16x2 word is infinite or NaN (all exponent bits set).
__device__ __forceinline__ uint32_t f16x2_nonfinite(uint32_t p)
{
    return ((p & 0x7C00u) == 0x7C00u) | ((p & 0x7C000000u) == 0x7C000000u);
}

// One MMA of 32 bytes of K (16 bf16 or 32 e4m3 elements).
template <int MODE>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate)
{
    if constexpr (is_e4m3(MODE))
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// silu(g) * u = g * u / (1 + e^-g), with the fast exponential and division
// intrinsics (each within a few ulp; the result is rounded to bf16 next).
__device__ __forceinline__ float silu_mul(float g, float u)
{
    return __fdividef(g * u, 1.0f + __expf(-g));
}

// Which kernel computes an expert with `rows` rows: the pair kernel (256-row tiles,
// about 8 % cheaper per tile-row than the single-CTA kernel) unless 128-row tiles save
// more than 10 % of the padded work: 1.84 * ceil(r/256) <= 1.1 * ceil(r/128).
__host__ __device__ __forceinline__ bool prefer_pair_tiles(int rows)
{
    return rows > 0 && 460 * ((rows + 255) / 256) <= 275 * ((rows + 127) / 128);
}

__device__ __forceinline__ bool expert_selected(int select, int rows)
{
    return select == 0 || (select == 1) == prefer_pair_tiles(rows);
}

// The order in which experts take their tiles: alternately from the two ends of the expert
// range (0, E-1, 1, E-2, ...). With skewed routing the heavy experts crowd one end (a Zipf
// bias makes the low indices hot), and their tiles after the first of each N slab find the
// weight tile in L2 and run at tensor-core speed, while a light expert's tiles stream weights
// from DRAM; alternating the ends keeps both kinds in every wave of tiles, so DRAM stays busy
// throughout instead of idling through the heavy experts and then saturating. Uniform
// routing is unaffected. Position i of the order -> expert.
__device__ __forceinline__ int visit_expert(int i, int E)
{
    return (i & 1) ? E - 1 - (i >> 1) : (i >> 1);
}

// Tile index -> (expert, N-slab, M-tile). tile_start[i] = first tile of the expert at
// position i of the visit order, mtiles[i] its M-tile count.
__device__ __forceinline__ void decode_tile(int tile, const int *tile_start, const int *mtiles,
                                            int E, int n_tiles, int &e, int &n, int &m)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= tile)
            lo = mid;
        else
            hi = mid - 1;
    }
    e = visit_expert(lo, E);
    const int local = tile - tile_start[lo];
    const int mt = mtiles[lo];
    n = local / mt;
    m = local - n * mt;
}

// The four epilogue warps (threads 64..191) of the FP8 modes meet at named barrier 1 once
// per tile (after staging the tile's scales); every one of them passes it on every tile,
// and all of them learn whether all of them are to go on, so none is left waiting there.
__device__ __forceinline__ bool epilogue_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "barrier.cta.red.and.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Shared memory holding one tile's output-channel scales (FP8 modes), two tiles deep.
constexpr int SCALE_STAGE_FLOATS = 2 * 256;
constexpr int SCALE_STAGE_BYTES = SCALE_STAGE_FLOATS * 4 + 16;

// Before a tile's accumulator is ready: its channel scales into ss (FP8 modes; the 128
// epilogue threads copy them) and this thread's row scale into sx.
template <int MODE, int BN>
__device__ __forceinline__ void stage_scales(const Args &args, int e, int n, int row, bool valid,
                                             float *ss, float &sx)
{
    if constexpr (is_e4m3(MODE)) {
        const int t = (int)threadIdx.x - 64;
        if constexpr (is_gate(MODE)) {  // 128 W1 then 128 W3 channels
            const size_t base = (size_t)e * args.b_rows + n * 128;
            ss[t] = args.b_scale0[base + t];
            ss[128 + t] = args.b_scale1[base + t];
        } else {  // BN W2 channels
            const size_t base = (size_t)e * args.b_rows + n * BN;
            for (int c = t; c < BN; c += 128)
                ss[c] = args.b_scale0[base + c];
        }
        sx = valid ? args.row_scale[row] : 0.0f;
    }
}

// Columns per TMEM round trip of the epilogue: the FP8 modes' shorter K loop leaves
// the epilogue exposed, so they batch more loads per wait (measured: the bf16 modes are
// fastest with the smaller batches).
__host__ __device__ constexpr int epilogue_cols(int MODE)
{
    return MODE == 0 ? 16 : MODE == 1 ? 32 : MODE == 2 ? 32 : 64;
}

// Gate/up epilogue of one thread: accumulator row `row` (TMEM lane of this thread),
// gate columns [0, 128) and up columns [128, 256) of N-slab n -> 128 bf16 values of h.
// The FP8 mode first scales the accumulators by the row scale sx and the staged W1 / W3
// channel scales ss.
// hscale: the fp16 range scale 2^-k of a second pass (1 otherwise); hmax: the largest |h| bits
// this thread stored (fp16 path).
template <int MODE>
__device__ __forceinline__ void swiglu_epilogue(const Args &args, uint32_t taddr, int n, int row,
                                                bool store, float sx, const float *ss,
                                                float hscale, uint32_t &hmax)
{
    constexpr int CB = epilogue_cols(MODE);
    uint16_t *orow = reinterpret_cast<uint16_t *>(args.out) + (size_t)row * args.ldo;
    uint4 *dst = reinterpret_cast<uint4 *>(orow + n * 128);
#pragma unroll 1
    for (int c = 0; c < 128; c += CB) {
        uint32_t g[CB], u[CB];
#pragma unroll
        for (int q = 0; q < CB / 16; ++q) {
            tmem_ld16(taddr + c + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(g + 16 * q));
            tmem_ld16(taddr + 128 + c + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(u + 16 * q));
        }
        tmem_ld_wait();
        if (store) {
            float gf[CB], uf[CB];
#pragma unroll
            for (int j = 0; j < CB; ++j) {
                gf[j] = __uint_as_float(g[j]);
                uf[j] = __uint_as_float(u[j]);
            }
            if constexpr (MODE == 2) {
#pragma unroll
                for (int j = 0; j < CB; j += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(ss + c + j);
                    const float4 b = *reinterpret_cast<const float4 *>(ss + 128 + c + j);
                    gf[j] *= sx * a.x;
                    gf[j + 1] *= sx * a.y;
                    gf[j + 2] *= sx * a.z;
                    gf[j + 3] *= sx * a.w;
                    uf[j] *= sx * b.x;
                    uf[j + 1] *= sx * b.y;
                    uf[j + 2] *= sx * b.z;
                    uf[j + 3] *= sx * b.w;
                }
            }
            uint32_t p[CB / 2];
            if (MODE == 0 && args.h_f16) {
#pragma unroll
                for (int j = 0; j < CB / 2; ++j) {
                    const float h0 = silu_mul(gf[2 * j], uf[2 * j]) * hscale;
                    const float h1 = silu_mul(gf[2 * j + 1], uf[2 * j + 1]) * hscale;
                    hmax = max(hmax, max(__float_as_uint(h0) & 0x7FFFFFFFu,
                                         __float_as_uint(h1) & 0x7FFFFFFFu));
                    p[j] = pack_f16x2(h0, h1);
                }
            } else {
#pragma unroll
                for (int j = 0; j < CB / 2; ++j)
                    p[j] = pack_bf16x2(silu_mul(gf[2 * j], uf[2 * j]),
                                       silu_mul(gf[2 * j + 1], uf[2 * j + 1]));
            }
#pragma unroll
            for (int j = 0; j < CB / 8; ++j)
                dst[c / 8 + j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
        }
    }
}

// Per epilogue warp of the down-projection modes: a 32-row x 32-column fp32 tile in
// shared memory (4 KB, 128-byte swizzled as the y tensor map expects), stored by TMA.
constexpr int Y_STAGE_BYTES = 4 * 4096 + 1024;

// Down-projection epilogue of one thread: accumulator row `row`, columns [0, BN) of
// N-slab n -> fp32 y (not rounded before the combine). The FP8 mode scales by the row
// scale sx and the staged W2 channel scales ss. When all 32 rows of this warp belong to
// the expert (wfull), each 32-column piece goes through the warp's shared-memory tile
// (ystage) and one TMA store of 32 x 32 at (x = column, y = wrow0); otherwise every
// thread stores its own row's values directly (no row past the expert is written).
// FP8 return payload ("MoE 推理服务工程真相 2026", §6.3: the exchange's token data in FP8):
// every 32-column block of a y row becomes 32 e4m3 codes and one exponent j (stored as the
// byte j + 127), the smallest power of two with max|block| * 2^-j <= 448, as for the
// dispatch payload. Row `row` of the payload: codes at [0, ldo), exponents at
// [ldo, ldo + ldo / 32). The values quantised are the fp32 y values the plain mode stores.
template <int MODE, int BN>
__device__ __forceinline__ void down_epilogue_fp8_return(const Args &args, uint32_t taddr, int n,
                                                         int row, bool store, float sx,
                                                         const float *ss, float yscale)
{
    constexpr int CB = epilogue_cols(MODE);
    uint8_t *prow = reinterpret_cast<uint8_t *>(args.out) + (size_t)row * args.y_stride;
    uint64_t exps = 0;  // BN / 32 <= 8 exponent bytes of this tile's row piece
#pragma unroll 1
    for (int c = 0; c < BN; c += CB) {
        uint32_t v[CB];
#pragma unroll
        for (int q = 0; q < CB / 16; ++q)
            tmem_ld16(taddr + c + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(v + 16 * q));
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < CB / 32; ++h) {
            float f[32];
            uint32_t mx = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                float o = __uint_as_float(v[32 * h + k]);
                if constexpr (MODE == 3)
                    o *= sx * ss[c + 32 * h + k];
                else
                    o *= yscale;
                f[k] = o;
                mx = max(mx, __float_as_uint(o) & 0x7FFFFFFFu);
            }
            const int j = e4m3_scale_exp(__uint_as_float(mx));
            const float inv = pow2f(-j);
            uint32_t p[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                p[k] = pack_e4m3x2(f[4 * k] * inv, f[4 * k + 1] * inv) |
                       (pack_e4m3x2(f[4 * k + 2] * inv, f[4 * k + 3] * inv) << 16);
            const int col = c + 32 * h;
            if (store) {
                uint4 *dst = reinterpret_cast<uint4 *>(prow + n * BN + col);
                dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
                dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
            }
            exps |= (uint64_t)(uint32_t)(j + 127) << (8 * (col / 32));
        }
    }
    if (store) {
        uint8_t *eb = prow + args.ldo + n * (BN / 32);
        if constexpr (BN == 256)
            *reinterpret_cast<uint2 *>(eb) = make_uint2((uint32_t)exps, (uint32_t)(exps >> 32));
        else
            *reinterpret_cast<uint32_t *>(eb) = (uint32_t)exps;
    }
}

// The fp16 return payload: the same blocks with fp16 codes (2 bytes each, the exponent bytes
// after the 2 ldo code bytes), the block's exponent from f16_scale_exp. When all 32 rows of
// the warp belong to the expert (wfull), each 32-column piece of codes goes through one of two
// 2 KB halves of the warp's shared-memory tile (64-byte rows, 64-byte swizzle, as the codes'
// tensor map expects) and one TMA store of 32 x 32 codes; the pieces alternate halves, so a
// piece waits only for the store before the previous one. Otherwise (and for the exponent
// bytes) every thread stores its own row.
template <int MODE, int BN>
__device__ __forceinline__ void down_epilogue_f16_return(const Args &args, uint32_t taddr, int n,
                                                         int row, bool store, float sx,
                                                         const float *ss, float yscale,
                                                         const CUtensorMap *ymap, uint32_t ystage,
                                                         int wrow0, bool wfull)
{
    constexpr int CB = epilogue_cols(MODE);
    const int lane = threadIdx.x & 31;
    uint8_t *prow = reinterpret_cast<uint8_t *>(args.out) + (size_t)row * args.y_stride;
    uint64_t exps = 0;
#pragma unroll 1
    for (int c = 0; c < BN; c += CB) {
        uint32_t v[CB];
#pragma unroll
        for (int q = 0; q < CB / 16; ++q)
            tmem_ld16(taddr + c + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(v + 16 * q));
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < CB / 32; ++h) {
            float f[32];
            uint32_t mx = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                float o = __uint_as_float(v[32 * h + k]);
                if constexpr (MODE == 3)
                    o *= sx * ss[c + 32 * h + k];
                else
                    o *= yscale;
                f[k] = o;
                mx = max(mx, __float_as_uint(o) & 0x7FFFFFFFu);
            }
            const int j = f16_scale_exp(__uint_as_float(mx));
            const float inv = pow2f(-j);
            uint32_t p[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                p[k] = pack_f16x2(f[2 * k] * inv, f[2 * k + 1] * inv);
            const int col = c + 32 * h;
            if (wfull) {
                const uint32_t half = ystage + (uint32_t)((col / 32) & 1) * 2048u;
                if (lane == 0)
                    bulk_wait_read1();  // the store that last read this half has done so
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t addr = half + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(p[4 * k]), "r"(p[4 * k + 1]), "r"(p[4 * k + 2]),
                                 "r"(p[4 * k + 3])
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    tma_store_2d(ymap, half, n * BN + col, wrow0);
            } else if (store) {
                uint4 *dst = reinterpret_cast<uint4 *>(prow + 2 * (n * BN + col));
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    dst[k] = make_uint4(p[4 * k], p[4 * k + 1], p[4 * k + 2], p[4 * k + 3]);
            }
            exps |= (uint64_t)(uint32_t)(j + 127) << (8 * (col / 32));
        }
    }
    if (store) {
        uint8_t *eb = prow + 2 * args.ldo + n * (BN / 32);
        if constexpr (BN == 256)
            *reinterpret_cast<uint2 *>(eb) = make_uint2((uint32_t)exps, (uint32_t)(exps >> 32));
        else
            *reinterpret_cast<uint32_t *>(eb) = (uint32_t)exps;
    }
}

// yscale: 2^k when h was stored scaled by 2^-k to stay in fp16's range (1 otherwise).
template <int MODE, int BN>
__device__ __forceinline__ void down_epilogue(const Args &args, uint32_t taddr, int n, int row,
                                              bool store, float sx, const float *ss,
                                              const CUtensorMap *ymap, uint32_t ystage,
                                              int wrow0, bool wfull, float yscale)
{
    if (args.y_stride > 0) {
        if (args.y_f16)
            down_epilogue_f16_return<MODE, BN>(args, taddr, n, row, store, sx, ss, yscale, ymap,
                                               ystage, wrow0, wfull);
        else
            down_epilogue_fp8_return<MODE, BN>(args, taddr, n, row, store, sx, ss, yscale);
        return;
    }
    constexpr int CB = epilogue_cols(MODE);
    const int lane = threadIdx.x & 31;
    float *frow = reinterpret_cast<float *>(args.out) + (size_t)row * args.ldo;
    float4 *dst = reinterpret_cast<float4 *>(frow + n * BN);
#pragma unroll 1
    for (int c = 0; c < BN; c += CB) {
        uint32_t v[CB];
#pragma unroll
        for (int q = 0; q < CB / 16; ++q)
            tmem_ld16(taddr + c + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(v + 16 * q));
        tmem_ld_wait();
        if (wfull) {
#pragma unroll
            for (int h = 0; h < CB / 32; ++h) {
                if (lane == 0)
                    bulk_wait_read();  // the previous piece has left the tile
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int k = 32 * h + 4 * j;
                    float4 o = make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                                           __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
                    if constexpr (MODE == 3) {
                        const float4 sc = *reinterpret_cast<const float4 *>(ss + c + k);
                        o.x *= sx * sc.x;
                        o.y *= sx * sc.y;
                        o.z *= sx * sc.z;
                        o.w *= sx * sc.w;
                    } else {
                        o.x *= yscale;
                        o.y *= yscale;
                        o.z *= yscale;
                        o.w *= yscale;
                    }
                    const uint32_t addr = ystage + lane * 128 + ((j ^ (lane & 7)) << 4);
                    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(o.x),
                                 "f"(o.y), "f"(o.z), "f"(o.w)
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    tma_store_2d(ymap, ystage, n * BN + c + 32 * h, wrow0);
            }
        } else if (store) {
#pragma unroll
            for (int j = 0; j < CB; j += 4) {
                float4 o = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                       __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                if constexpr (MODE == 3) {
                    const float4 sc = *reinterpret_cast<const float4 *>(ss + c + j);
                    o.x *= sx * sc.x;
                    o.y *= sx * sc.y;
                    o.z *= sx * sc.z;
                    o.w *= sx * sc.w;
                } else {
                    o.x *= yscale;
                    o.y *= yscale;
                    o.z *= yscale;
                    o.w *= yscale;
                }
                dst[(c + j) / 4] = o;
            }
        }
    }
}

template <int MODE, int BN>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const Args args)
{
    static_assert(is_gate(MODE) ? BN == 256 : (BN == 128 || BN == 256), "tile shape");
    constexpr bool GATE = is_gate(MODE);  // gate/up: W1 and W3 halves, SwiGLU epilogue
    constexpr int KX = atom_k(MODE);
    constexpr int B_BYTES = BN * BK * 2;
    constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    const uint32_t IDESC = launch_idesc<MODE>(args, BM, BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *tile_start = reinterpret_cast<int *>(tmem_slot + 4);
    int *mtiles = tile_start + (args.E + 1);
    float *scale_stage = reinterpret_cast<float *>(
        (reinterpret_cast<uintptr_t>(mtiles + args.E) + 15) & ~uintptr_t(15));
    // down-projection modes: 4 warp tiles of 4 KB, 1024-byte aligned (128-byte swizzle)
    const uint32_t y_stage = (smem_u32(scale_stage + SCALE_STAGE_FLOATS) + 1023u) & ~1023u;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t bar_base = smem_u32(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + 2 + a); };
    const uint32_t done_bar = bar_base + 8u * (2 * STAGES + 4);
    const int E = args.E;
    // fp16 range: the second gate/up pass runs only if the first one's largest |h| is beyond
    // fp16's range; it stores h * 2^-k, and the down projection multiplies y by 2^k
    int hk = 0;
    if (args.h_f16 && (MODE == 1 || (MODE == 0 && args.h_pass == 1)))
        hk = f16_range_exp(*reinterpret_cast<volatile uint32_t *>(args.h_amax));
    const bool pass_needed = !(MODE == 0 && args.h_f16 && args.h_pass == 1) || hk > 0;
    if (MODE == 0 && args.h_pass == 1 && hk < 0 && blockIdx.x == 0 && threadIdx.x == 0)
        set_dev_error(MOE_ERR_F16_RANGE);  // a non-finite activation: no scale brings it in
    const float hscale = (MODE == 0 && args.h_pass == 1 && hk > 0) ? pow2f(-hk) : 1.0f;
    const float yscale = (MODE == 1 && hk > 0) ? pow2f(hk) : 1.0f;
    uint32_t hmax = 0;  // largest |h| this thread stored (first gate/up pass)

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 4);
        }
        mbar_init(done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort_flag = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 0) {
        // per-expert M-tile counts and their prefix (in tiles, times n_tiles)
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int i = base + lane;  // position in the visit order
            int mt = 0;
            if (i < E) {
                const int e = visit_expert(i, E);
                int rows = args.offsets[e + 1] - args.offsets[e];
                rows = max(0, min(rows, args.rows_alloc));
                mt = (expert_selected(args.select, rows) && pass_needed) ? (rows + BM - 1) / BM
                                                                         : 0;
                mtiles[i] = mt;
            }
            const int incl = warp_incl_scan(mt);
            if (i < E)
                tile_start[i] = (carry + incl - mt) * args.n_tiles;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0)
            tile_start[E] = carry * args.n_tiles;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[E];

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_parity[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s)
                issued[s] = false;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                int e, n, m;
                decode_tile(tile, tile_start, mtiles, E, args.n_tiles, e, n, m);
                const int row0 = args.offsets[e] + m * BM;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_base + stage * STAGE_BYTES;
                    const uint32_t b_dst = a_dst + A_BYTES;
                    mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
                    tma_load_2d(a_dst, &tmA, kb * KX, row0, full_bar(stage));
                    if (GATE) {
                        const int brow = e * args.b_rows + n * 128;
                        tma_load_2d(b_dst, &tmB0, kb * KX, brow, full_bar(stage));
                        tma_load_2d(b_dst + B_HALF_BYTES, &tmB1, kb * KX, brow, full_bar(stage));
                    } else {
#pragma unroll
                        for (int h = 0; h < BN / 128; ++h)
                            tma_load_2d(b_dst + h * B_HALF_BYTES, &tmB0, kb * KX,
                                        e * args.b_rows + n * BN + h * 128, full_bar(stage));
                    }
                    issued[stage] = true;
                    last_parity[stage] = phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: every issued copy has landed before the CTA may exit
            for (int s = 0; s < STAGES; ++s)
                if (issued[s])
                    mbar_wait(full_bar(s), last_parity[s], abort_flag, args.timeout_ns, false);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, args.timeout_ns))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_base + stage * STAGE_BYTES;
                    const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // four 32-byte K slices per atom
                        tc_mma<MODE>(d_tmem, smem_desc_sw128(a_addr + k * 32),
                                     smem_desc_sw128(b_addr + k * 32), IDESC,
                                     (kb > 0 || k > 0) ? 1u : 0u);
                    tc_commit(empty_bar(stage));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit(tfull_bar(acc));
                acc ^= 1;
                if (acc == 0)
                    acc_phase ^= 1u;
            }
            // every MMA issued so far has completed before TMEM is released
            tc_commit(done_bar);
            mbar_wait(done_bar, 0, abort_flag, args.timeout_ns, false);
        }
    } else {
        // ---------------- epilogue: warps 2..5, TMEM lane quadrant = warp % 4
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            int e, n, m;
            decode_tile(tile, tile_start, mtiles, E, args.n_tiles, e, n, m);
            const int rows_e = args.offsets[e + 1] - args.offsets[e];
            const int valid = min(BM, rows_e - m * BM);
            const int row0 = args.offsets[e] + m * BM;
            float *ss = scale_stage + (it & 1) * 256;
            float sx = 1.0f;
            stage_scales<MODE, BN>(args, e, n, row0 + r, r < valid, ss, sx);
            int ok = 0;
            if (lane == 0)
                ok = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if constexpr (is_e4m3(MODE)) {
                if (!epilogue_all(ok != 0))  // also publishes the staged scales
                    break;
            } else if (!ok) {
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            if (GATE) {
                swiglu_epilogue<MODE>(args, taddr, n, row0 + r, r < valid, sx, ss, hscale, hmax);
            } else {
                down_epilogue<MODE, BN>(args, taddr, n, row0 + r, r < valid, sx, ss, &tmB1,
                                        y_stage + q * 4096, row0 + q * 32, valid - q * 32 >= 32,
                                        yscale);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tempty_bar(acc));
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
        }
    }

    if (!is_gate(MODE) && warp >= 2 && lane == 0)
        bulk_wait_all();  // this warp's y stores are complete before its shared memory goes
    if (MODE == 0 && args.h_f16 && args.h_pass == 0 && warp >= 2) {
#pragma unroll
        for (int off = 16; off; off >>= 1)
            hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, off));
        if (lane == 0 && hmax)
            atomicMax(args.h_amax, hmax);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
}

// ---------------------------------------------------------------------------
// CTA-pair variant (tcgen05 cta_group::2). A cluster of 2 CTAs on 2 SMs computes
// a 256 x 256 tile: CTA r loads rows [128 r, 128 r + 128) of A and rows
// [128 r, 128 r + 128) of the 256-row B tile into its own shared memory at the
// same offsets; the first CTA of the pair issues one M=256, N=256 MMA per K step
// that reads A from each CTA and B from both, and each CTA's TMEM receives its 128
// rows of the accumulator. Per CTA and 64-element K step that is 32 KB of
// operands for the same MMA work that costs the single-CTA kernel 48 KB. A ring
// stage holds two K steps (128 elements, two swizzle atoms per operand, 64 KB per
// CTA, 3 stages): eight MMAs per barrier round trip instead of four, which the
// issue path of the pair needs to keep the tensor pipe busy.
// Barriers: full[s] lives in the first CTA and counts both CTAs' TMA bytes
// (the loads name it by its cluster address); empty[s] and tfull[a] live in each
// CTA and receive one tcgen05.commit each (two commits, one per CTA, to
// mapa-resolved addresses); tempty[a] lives in the first CTA and counts the 8
// epilogue warps of the pair.

constexpr int KA2 = 2;                                      // 64-element K atoms per stage
constexpr int STAGES2 = 3;
constexpr int STAGE2_BYTES = KA2 * (A_BYTES + B_HALF_BYTES);  // 64 KB per CTA

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_addr), "r"(rank));
    return out;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t bar_cluster_addr)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster_addr)
        : "memory");
}

__device__ __forceinline__ void tc_commit_pair(uint32_t bar_cluster_addr)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar_cluster_addr)
                 : "memory");
}

template <int MODE>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate)
{
    if constexpr (is_e4m3(MODE))
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                     bar_cluster_addr)
                 : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, const Args args)
{
    constexpr int BMP = 256;  // rows per pair tile
    constexpr int BN = 256;
    constexpr bool GATE = is_gate(MODE);
    constexpr int KX = atom_k(MODE);
    const uint32_t IDESC = launch_idesc<MODE>(args, BMP, BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES2 * STAGE2_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES2 + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *tile_start = reinterpret_cast<int *>(tmem_slot + 4);
    int *mtiles = tile_start + (args.E + 1);
    float *scale_stage = reinterpret_cast<float *>(
        (reinterpret_cast<uintptr_t>(mtiles + args.E) + 15) & ~uintptr_t(15));
    // down-projection modes: 4 warp tiles of 4 KB, 1024-byte aligned (128-byte swizzle)
    const uint32_t y_stage = (smem_u32(scale_stage + SCALE_STAGE_FLOATS) + 1023u) & ~1023u;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t bar_base = smem_u32(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES2 + s); };
    auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * STAGES2 + a); };
    auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * STAGES2 + 2 + a); };
    const uint32_t done_bar = bar_base + 8u * (2 * STAGES2 + 4);
    const int E = args.E;
    // fp16 range (see grouped_gemm_kernel); the pair kernel runs first passes only
    int hk = 0;
    if (args.h_f16 && MODE == 1)
        hk = f16_range_exp(*reinterpret_cast<volatile uint32_t *>(args.h_amax));
    const bool pass_needed = true;
    const float hscale = 1.0f;
    const float yscale = (MODE == 1 && hk > 0) ? pow2f(hk) : 1.0f;
    uint32_t hmax = 0;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES2; ++st) {
            mbar_init(full_bar(st), 1);
            mbar_init(empty_bar(st), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 8);
        }
        mbar_init(done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort_flag = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int i = base + lane;  // position in the visit order
            int mt = 0;
            if (i < E) {
                const int e = visit_expert(i, E);
                int rows = args.offsets[e + 1] - args.offsets[e];
                rows = max(0, min(rows, args.rows_alloc));
                mt = (expert_selected(args.select, rows) && pass_needed) ? (rows + BMP - 1) / BMP
                                                                         : 0;
                mtiles[i] = mt;
            }
            const int incl = warp_incl_scan(mt);
            if (i < E)
                tile_start[i] = (carry + incl - mt) * args.n_tiles;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0)
            tile_start[E] = carry * args.n_tiles;
    }
    tc_fence_before();
    cluster_sync_all();  // barriers initialised in both CTAs before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[E];

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs)
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_parity[STAGES2];
            bool issued[STAGES2];
            for (int st = 0; st < STAGES2; ++st)
                issued[st] = false;
            bool ok = true;
            const CUtensorMap *bmap = (GATE && rank == 1) ? &tmB1 : &tmB0;
            for (int tile = pair; tile < total && ok; tile += npairs) {
                int e, n, m;
                decode_tile(tile, tile_start, mtiles, E, args.n_tiles, e, n, m);
                const int row0 = args.offsets[e] + m * BMP + (int)rank * 128;
                const int brow = GATE ? e * args.b_rows + n * 128
                                      : e * args.b_rows + n * BN + (int)rank * 128;
                for (int kb = 0; kb < args.k_blocks / KA2; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_base + stage * STAGE2_BYTES;
                    const uint32_t full_leader = map_to_rank(full_bar(stage), 0);
                    if (leader)
                        mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE2_BYTES);
#pragma unroll
                    for (int at = 0; at < KA2; ++at) {
                        const int kx = (kb * KA2 + at) * KX;
                        tma_load_2d_pair(a_dst + at * A_BYTES, &tmA, kx, row0, full_leader);
                        tma_load_2d_pair(a_dst + KA2 * A_BYTES + at * B_HALF_BYTES, bmap, kx, brow,
                                         full_leader);
                    }
                    issued[stage] = true;
                    last_parity[stage] = phase;
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain (first CTA: its full barriers count both CTAs' copies)
            if (leader)
                for (int st = 0; st < STAGES2; ++st)
                    if (issued[st])
                        mbar_wait(full_bar(st), last_parity[st], abort_flag, args.timeout_ns, false);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (first CTA of the pair)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < total && ok; tile += npairs) {
                if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, args.timeout_ns))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < args.k_blocks / KA2; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_base + stage * STAGE2_BYTES;
                    const uint32_t b_addr = a_addr + KA2 * A_BYTES;
#pragma unroll
                    for (int k = 0; k < KA2 * 4; ++k) {  // four 32-byte K slices per atom
                        const uint32_t off = (uint32_t)((k / 4) * A_BYTES + (k % 4) * 32);
                        tc_mma_pair<MODE>(d_tmem, smem_desc_sw128(a_addr + off),
                                          smem_desc_sw128(b_addr + off), IDESC,
                                          (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(map_to_rank(empty_bar(stage), 0));
                    tc_commit_pair(map_to_rank(empty_bar(stage), 1));
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit_pair(map_to_rank(tfull_bar(acc), 0));
                tc_commit_pair(map_to_rank(tfull_bar(acc), 1));
                acc ^= 1;
                if (acc == 0)
                    acc_phase ^= 1u;
            }
            tc_commit_pair(map_to_rank(done_bar, 0));
            mbar_wait(done_bar, 0, abort_flag, args.timeout_ns, false);
        }
    } else {
        // ---------------- epilogue: warps 2..5 of both CTAs
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        int it = 0;
        for (int tile = pair; tile < total; tile += npairs, ++it) {
            int e, n, m;
            decode_tile(tile, tile_start, mtiles, E, args.n_tiles, e, n, m);
            const int rows_e = args.offsets[e + 1] - args.offsets[e];
            const int valid = min(128, rows_e - m * BMP - (int)rank * 128);
            const int row0 = args.offsets[e] + m * BMP + (int)rank * 128;
            float *ss = scale_stage + (it & 1) * 256;
            float sx = 1.0f;
            stage_scales<MODE, BN>(args, e, n, row0 + r, r < valid, ss, sx);
            int ok = 0;
            if (lane == 0)
                ok = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, args.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if constexpr (is_e4m3(MODE)) {
                if (!epilogue_all(ok != 0))  // also publishes the staged scales
                    break;
            } else if (!ok) {
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            if (GATE) {
                swiglu_epilogue<MODE>(args, taddr, n, row0 + r, r < valid, sx, ss, hscale, hmax);
            } else {
                down_epilogue<MODE, BN>(args, taddr, n, row0 + r, r < valid, sx, ss, &tmB1,
                                        y_stage + q * 4096, row0 + q * 32, valid - q * 32 >= 32,
                                        yscale);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(map_to_rank(tempty_bar(acc), 0));
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
        }
    }

    if (!is_gate(MODE) && warp >= 2 && lane == 0)
        bulk_wait_all();  // this warp's y stores are complete before its shared memory goes
    if (MODE == 0 && args.h_f16 && warp >= 2) {
#pragma unroll
        for (int off = 16; off; off >>= 1)
            hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, off));
        if (lane == 0 && hmax)
            atomicMax(args.h_amax, hmax);
    }
    __syncwarp();
    tc_fence_before();
    if (*abort_flag) {
        // after a timeout, give copies already in flight time to land before the pair
        // leaves (a CTA's shared memory must outlive the copies and MMAs that use it)
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
    }
    cluster_sync_all();  // neither CTA leaves while its partner may still use its memory
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
}

template <int MODE>
constexpr int smem_bytes_pair(int E)
{
    return STAGES2 * STAGE2_BYTES + 1024 + 8 * (2 * STAGES2 + 5) + 16 + 8 * (E + 1) + 64 +
           SCALE_STAGE_BYTES + (is_gate(MODE) ? 0 : Y_STAGE_BYTES);
}

template <int MODE, int BN>
constexpr int smem_bytes(int E)
{
    return STAGES * (A_BYTES + BN * BK * 2) + 1024 /* alignment */ + 8 * (2 * STAGES + 5) +
           16 + 8 * (E + 1) + 64 + SCALE_STAGE_BYTES + (is_gate(MODE) ? 0 : Y_STAGE_BYTES);
}

}  // namespace gg
}  // namespace moe
