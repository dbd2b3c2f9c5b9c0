// Shared device helpers of the W8A8 library (sm_100a only).
//
//  * a device error word that kernels set instead of trapping;
//  * bounded mbarrier waits (a wait that exceeds its time limit records
//    W8A8_ERR_TIMEOUT and returns false, so no kernel can spin forever);
//  * thin inline-PTX wrappers for mbarriers, TMA, tcgen05 and mma.sync.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "w8a8.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace w8a8 {

// ---------------------------------------------------------------------------
// Device error word.  0 = no error; otherwise the first W8A8_ERR_* a kernel
// recorded.  Read and cleared by w8a8_get_device_error().
__device__ int g_device_error = 0;
// Where the first bounded wait gave up: (kernel id << 16) | site.
__device__ int g_device_error_site = 0;

__device__ __forceinline__ void record_error(int code, int site) {
    if (atomicCAS(&g_device_error, 0, code) == 0) g_device_error_site = site;
}

// Time limit of every bounded wait, in nanoseconds of %globaltimer.
// Legitimate waits in these kernels last microseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of `parity` to complete.  Gives up when *abort becomes
// nonzero (another role of the CTA gave up) or after `limit_ns`; on a time-out
// it records W8A8_ERR_TIMEOUT with `site`, raises *abort and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  int site, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t polls = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++polls & 63u) == 0u) {
            if (abort != nullptr && *abort) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                record_error(W8A8_ERR_TIMEOUT, site);
                if (abort != nullptr) *abort = 1;
                return false;
            }
        }
    }
}

// Programmatic dependent launch: a kernel launched to overlap the one before
// it reads that kernel's results only after `griddepcontrol.wait`, and with
// ordinary loads (__ldca / ld.global.ca where the SM's warps share the data,
// __ldcg / ld.global.cg otherwise) or TMA: the compiler treats non-coherent
// loads (__ldg, ld.global.nc) as invariant and may hoist them above the wait.
// __ldg is kept for weights and for data written before the previous kernel
// started.

// ---------------------------------------------------------------------------
// TMA (tiled, no multicast)
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, s8 x s8 -> s32.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// lane (base + i), columns col .. col + 31.
// Every one of this thread's 32 consecutive TMEM columns (its lane) set to v,
// eight columns per store (a store takes its values from consecutive
// registers, so a wider one would hold that many copies of v).
__device__ __forceinline__ void tmem_st_32x32b_x32_fill(uint32_t taddr, uint32_t v) {
#pragma unroll
    for (int c = 0; c < 32; c += 8)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr + c),
                     "r"(v)
                     : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x8_fill(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr), "r"(v)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x16_fill(uint32_t taddr, uint32_t v) {
#pragma unroll
    for (int c = 0; c < 16; c += 8)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr + c),
                     "r"(v)
                     : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle
// layout that TMA's SWIZZLE_128B writes (rows of 128 bytes, 8-row groups
// 1024 bytes apart).  Start address must lie in a 1024-byte aligned atom
// (advancing along K inside the 128-byte row is a plain address offset).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);        // start address
    d |= (uint64_t)1u << 16;                          // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: next 8-row group
    d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                          // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor for tcgen05.mma kind::i8: s8 x s8 -> s32, both K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4)                      // D format: s32
           | (1u << 7)                    // A: signed 8-bit
           | (1u << 10)                   // B: signed 8-bit
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// ---------------------------------------------------------------------------
// Legacy warp MMA for the skinny (decode) shapes: D(16x8) += A(16x32) B(32x8).
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Streaming 16-byte load that bypasses L1 (weights are read once).
__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Project exponential, identical op for op to the oracle's: Cody & Waite
// reduction with a two-part ln 2, degree-7 Taylor polynomial of e^r with
// fused multiply-adds, scaling by 2^n via the exponent field; input clamped
// to [-87, 88].
__device__ __forceinline__ float exp_proj(float x) {
    x = fminf(fmaxf(x, -87.0f), 88.0f);
    const float t = __fmul_rn(x, 1.44269502162933349609375f);
    // n = rne(t) through the 1.5 * 2^23 bias (|t| <= 127): tb holds it in its
    // low mantissa bits, so both n and its integer come without a conversion
    const float tb = __fadd_rn(t, 12582912.0f);
    const float n = __fsub_rn(tb, 12582912.0f);
    float r = __fmaf_rn(-n, 0.693359375f, x);
    r = __fmaf_rn(-n, -2.12194440e-4f, r);
    float p = 1.0f / 5040.0f;
    p = __fmaf_rn(p, r, 1.0f / 720.0f);
    p = __fmaf_rn(p, r, 1.0f / 120.0f);
    p = __fmaf_rn(p, r, 1.0f / 24.0f);
    p = __fmaf_rn(p, r, 1.0f / 6.0f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int ni = (int)(__float_as_uint(tb) - 0x4B400000u);
    return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float silu_proj(float g) {
    const float e = exp_proj(-g);
    return __fdiv_rn(g, __fadd_rn(1.0f, e));
}

// Symmetric int8 code of v under scale s (s > 0): clamp(rne(v / s), +-127).
__device__ __forceinline__ int quant_code(float v, float s) {
    int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-127, min(127, q));
}

// The same code, with rcp = __frcp_rn(s) computed once per row: y = v * rcp
// (one rounding) differs from the correctly rounded v / s by less than
// 2.3e-5 for |v / s| <= 127.5, so rounding y to the nearest integer gives
// rne(v / s) unless y lies within 2^-14 of a half-integer; only then (about
// one element in 8000) is the exact division taken.
//
// Rounding y: t = y + 1.5 * 2^23 lies in [2^23, 2^24), where the spacing of
// floats is 1, so the addition itself rounds y to the nearest integer (ties
// to even, as 1.5 * 2^23 is even) and leaves it in the low mantissa bits:
// the code is bits(t) - bits(1.5 * 2^23).  r = t - 1.5 * 2^23 is that integer
// as a float and e = y - r is exact (Sterbenz), so |e| says how close y is to
// a tie.  A NaN y fails the test and takes the exact path as well.  Needs
// |v / s| < 2^22, which holds wherever s is the row maximum of |v| over 127
// (every caller: |v / s| <= 127.5 there).
__device__ __forceinline__ int quant_code_rcp(float v, float s, float rcp) {
    const float y = __fmul_rn(v, rcp);
    const float t = __fadd_rn(y, 12582912.0f);
    const float e = __fsub_rn(y, __fsub_rn(t, 12582912.0f));
    int q;
    if (!(fabsf(e) < 0.49993896484375f) || !(fabsf(rcp) < 1.0e38f))   // 0.5 - 2^-14
        q = __float2int_rn(__fdiv_rn(v, s));
    else
        q = (int)(__float_as_uint(t) - 0x4B400000u);
    return max(-127, min(127, q));
}

// Low bytes of four codes packed little-endian into one word.
__device__ __forceinline__ uint32_t pack4_s8(int q0, int q1, int q2, int q3) {
    const uint32_t lo = __byte_perm((uint32_t)q0, (uint32_t)q1, 0x0040);
    const uint32_t hi = __byte_perm((uint32_t)q2, (uint32_t)q3, 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

// ---- paired fp32 arithmetic: sm_100 adds, subtracts and multiplies the two
// fp32 halves of a 64-bit register pair in one instruction (each half
// rounded to nearest even, as the scalar operation would be).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ void f2_unpack(uint64_t d, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(d));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// max that returns NaN if either input is NaN
__device__ __forceinline__ float fmax_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

// Per-row quantizer: the scale s = amax / 127, its rounded reciprocal, and
// whether the reciprocal path applies (s normal enough that 1 / s is finite).
struct QuantRow {
    float s, rcp;
    uint64_t rcp2;
    bool zero, fast;
    __device__ __forceinline__ explicit QuantRow(float amax) {
        s = __fdiv_rn(amax, 127.0f);
        rcp = __frcp_rn(s);
        rcp2 = f2_pack(rcp, rcp);
        zero = s == 0.0f;
        fast = fabsf(s) < INFINITY && fabsf(rcp) < 1.0e38f;
    }
};

// Codes of 4W consecutive values v (|v| <= 127.25 s) under row quantizer r,
// four to a word, little-endian.  Fast path, two values per instruction:
// y = v * rcp; t = y + 1.5 * 2^23 rounds y to the nearest integer (ties to
// even) into the low mantissa bits of t, whose low byte is then the int8
// code itself (|rne(y)| <= 127 here); e = y - (t - 1.5 * 2^23) is exact and
// measures the distance from y to a tie.  y differs from v / s by < 2.3e-5,
// so unless some |e| of the group reaches 0.5 - 2^-14 (or is NaN) the codes
// equal clamp(rne(v / s)); otherwise the group is redone by exact division.
template <int W>
__device__ __forceinline__ void quant_codes(const float (&v)[4 * W], const QuantRow& r, uint32_t (&out)[W]) {
    if (r.zero) {
#pragma unroll
        for (int j = 0; j < W; ++j) out[j] = 0u;
        return;
    }
    bool ok = r.fast;
    if (ok) {
        const uint64_t magic2 = 0x4B4000004B400000ull;   // (1.5 * 2^23, 1.5 * 2^23)
        float emax = 0.0f;
        uint32_t tb[4 * W];
#pragma unroll
        for (int i = 0; i < 2 * W; ++i) {
            const uint64_t y = f2_mul(f2_pack(v[2 * i], v[2 * i + 1]), r.rcp2);
            const uint64_t t = f2_add(y, magic2);
            const uint64_t e = f2_sub(y, f2_sub(t, magic2));
            float e0, e1, t0, t1;
            f2_unpack(e, e0, e1);
            f2_unpack(t, t0, t1);
            emax = fmax_nan(emax, fmax_nan(fabsf(e0), fabsf(e1)));
            tb[2 * i] = __float_as_uint(t0);
            tb[2 * i + 1] = __float_as_uint(t1);
        }
        ok = emax < 0.49993896484375f;
        if (ok) {
#pragma unroll
            for (int j = 0; j < W; ++j)
                out[j] = __byte_perm(__byte_perm(tb[4 * j], tb[4 * j + 1], 0x0040),
                                     __byte_perm(tb[4 * j + 2], tb[4 * j + 3], 0x0040), 0x5410);
        }
    }
    if (!ok) {
#pragma unroll
        for (int j = 0; j < W; ++j)
            out[j] = pack4_s8(quant_code(v[4 * j], r.s), quant_code(v[4 * j + 1], r.s), quant_code(v[4 * j + 2], r.s),
                              quant_code(v[4 * j + 3], r.s));
    }
}

// running max of |bf16| over packed pairs: (bits & 0x7fff) orders like |value|
// for every non-NaN bf16, and a NaN shows up as a pattern above 0x7f80
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Four fp32 atomic adds in one vector reduction (16-byte aligned address).
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
}

}  // namespace w8a8
