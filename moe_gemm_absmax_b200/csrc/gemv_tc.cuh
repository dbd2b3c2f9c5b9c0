// Decode-sized W8A8 linear (a4: a2 + a3 at M <= 32 tokens) on the
// 5th-generation tensor cores -- "Online INT8 W8A8 ...", Precision split
// (int8 weights halve the bytes of the bandwidth-bound decode step) and
// Changes (gemm_a8w8 per-token path).
//
// Swap-AB: the weight matrix is the 128-row A operand of tcgen05.mma.kind::i8
// and the few tokens' codes are the narrow B operand (N = BN = 16 or 32), so
// each instruction reads a 128 x 32 weight slice at full tensor-core rate
// and the kernel is bound only by how fast TMA streams W from HBM:
//   D[n, m] = sum_k W[n, k] X[m, k]          (TMEM: lane = weight row, column = token)
//   y[m, n] = bf16_rne( (float(D) * sx[m]) * sw[n] )
//
// Work split (stream-K): units (128-row group, 128-byte k block), group-major,
// one contiguous range per CTA.  A CTA's range is cut into segments, one per
// group it meets; each segment accumulates in one of two TMEM buffers (the
// epilogue of a segment overlaps the MMAs of the next).  A segment that
// spans the group's whole K writes outputs; otherwise each epilogue warp
// stores its 32 rows' int32 partials in the CTA's slot for that group (slot
// 0: the CTA's first group, 1: its last) and bumps the (group, warp)
// counter; the warp completing the count adds all slots in CTA order --
// exact integer sums, so results are deterministic.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 2..5 epilogue (TMEM lane quarters).  All waits are bounded.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace w8a8 {

constexpr int kGcBM = 128;         // weight rows per group (MMA M)
constexpr int kGcBK = 128;         // bytes of K per stage
constexpr int kGcStages = 10;
constexpr int kGcThreads = 192;
constexpr int kKernelIdGemvTc = 3;

// S: 128-byte k slices per stage (one TMA op per operand covers all S slices
// through a 3-D view [K/128][rows][128]); STAGES: ring depth.
template <int BN, int S = 1, int STAGES = kGcStages>
struct GcSmem {
    static constexpr int kW = S * kGcBM * kGcBK;    // S x 16 KB
    static constexpr int kX = S * BN * kGcBK;       // S x 2 / 4 KB
    static constexpr int kStage = kW + kX;          // multiple of 1024
    static constexpr int kTiles = STAGES * kStage;
    static constexpr int kBars = (2 * STAGES + 4 + 1) * 8;
    static constexpr int kBytes = 1024 + kTiles + kBars + 16;
};

struct GemvTc {
    const float* sx;      // [M]
    const float* sw;      // [N]
    void* out;            // bf16 or int32 [M, N]
    int M, N, K;
    int ngroups;          // ceil(N / 128)
    int nkb;              // ceil(K / 128)
    int s32;
    int* part;            // [gridDim.x][2][128 rows][BN] int32
    int* counters;        // [ngroups][4], zero on entry, left zero on exit
    int prefetch_w;       // weight loads may start before the previous kernel ends
};

__device__ __forceinline__ int64_t gc_begin(int64_t total, int c, int grid) { return total * c / grid; }

// CTA whose unit range holds unit u.
__device__ __forceinline__ int gc_owner(int64_t u, int64_t total, int grid) {
    int c = (int)((u * grid) / total);
    while (c > 0 && gc_begin(total, c, grid) > u) --c;
    while (c + 1 < grid && gc_begin(total, c + 1, grid) <= u) ++c;
    return c;
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Stage load of S k slices starting at slice kb * S: a 2-D tile (S == 1) or a
// 3-D box over the view (byte, row, slice).
template <int S>
__device__ __forceinline__ void gc_load(void* dst, const CUtensorMap* map, uint64_t* bar, int kb, int row) {
    if (S == 1)
        tma_load_2d(dst, map, bar, kb * kGcBK, row);
    else
        tma_load_3d(dst, map, bar, 0, row, kb * S);
}

template <int BN>
__device__ __forceinline__ void gc_store_row(const GemvTc& a, int n, const int (&v)[BN]) {
    if (n >= a.N) return;
    const float swn = a.s32 ? 0.0f : __ldg(a.sw + n);
#pragma unroll
    for (int m = 0; m < BN; ++m) {
        if (m < a.M) {
            if (a.s32) {
                reinterpret_cast<int32_t*>(a.out)[(int64_t)m * a.N + n] = v[m];
            } else {
                const float r = __fmul_rn(__fmul_rn(__int2float_rn(v[m]), __ldcg(a.sx + m)), swn);
                reinterpret_cast<uint16_t*>(a.out)[(int64_t)m * a.N + n] = float_to_bf16_bits(r);
            }
        }
    }
}

// 32 lanes x 16 consecutive 32-bit columns.

template <int BN, int S = 1, int STAGES = kGcStages>
__global__ void __launch_bounds__(kGcThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, GemvTc a) {
    static_assert(BN == 16 || BN == 32, "BN");
    constexpr int kCols = 2 * BN >= 32 ? 2 * BN : 32;
    constexpr int kGcStages = STAGES;
    using SM = GcSmem<BN, S, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kTiles);
    uint64_t* empty = full + kGcStages;
    uint64_t* tfull = empty + kGcStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t total = (int64_t)a.ngroups * a.nkb;
    const int64_t u0 = gc_begin(total, blockIdx.x, gridDim.x);
    const int64_t u1 = gc_begin(total, blockIdx.x + 1, gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 128);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmX);
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_phase = 0;
            bool ok = true;
            // Weights never depend on the previous kernel: when allowed, arm the
            // first stages with their weight tiles before waiting for it.
            int64_t pre = 0;
            if (a.prefetch_w) {
                pre = (u1 - u0) < kGcStages ? (u1 - u0) : kGcStages;
                for (int64_t i = 0; i < pre; ++i) {
                    const int64_t u = u0 + i;
                    mbar_arrive_expect_tx(&full[i], (uint32_t)SM::kStage);
                    gc_load<S>(smem + i * SM::kStage, &tmW, &full[i], (int)(u % a.nkb), (int)(u / a.nkb) * kGcBM);
                }
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int64_t u = u0; u < u1; ++u) {
                const int grp = (int)(u / a.nkb), kb = (int)(u % a.nkb);
                if (u - u0 >= pre) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, (kKernelIdGemvTc << 16) | 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)SM::kStage);
                    gc_load<S>(smem + stage * SM::kStage, &tmW, &full[stage], kb, grp * kGcBM);
                }
                gc_load<S>(smem + stage * SM::kStage + SM::kW, &tmX, &full[stage], kb, 0);
                issued |= 1u << stage;
                last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == kGcStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                for (int s = 0; s < kGcStages; ++s)
                    if (issued & (1u << s))
                        mbar_wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, (kKernelIdGemvTc << 16) | 2,
                                          100000000ull);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kGcBM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            int64_t u = u0;
            while (ok && u < u1) {
                const int grp = (int)(u / a.nkb);
                const int64_t seg_end = ((int64_t)grp + 1) * a.nkb < u1 ? ((int64_t)grp + 1) * a.nkb : u1;
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, (kKernelIdGemvTc << 16) | 3)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int64_t v = u; v < seg_end; ++v) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdGemvTc << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t w0 = smem_u32(smem + stage * SM::kStage);
                    const uint32_t x0 = w0 + SM::kW;
#pragma unroll
                    for (int sl = 0; sl < S; ++sl)
#pragma unroll
                        for (int kk = 0; kk < kGcBK / 32; ++kk)
                            tc_mma_i8(d_tmem, smem_desc_k_sw128(w0 + sl * kGcBM * kGcBK + kk * 32),
                                      smem_desc_k_sw128(x0 + sl * BN * kGcBK + kk * 32), idesc,
                                      (v > u || sl > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    if (++stage == kGcStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
                u = seg_end;
            }
            tc_commit(mma_done);
            mbar_wait_bounded(mma_done, 0u, nullptr, (kKernelIdGemvTc << 16) | 5, 100000000ull);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int quarter = warp & 3;
        const int first_grp = (int)(u0 / a.nkb);
        int acc = 0;
        uint32_t acc_phase = 0;
        int64_t u = u0;
        while (u < u1) {
            const int grp = (int)(u / a.nkb);
            const int64_t gs = (int64_t)grp * a.nkb, ge = gs + a.nkb;
            const int64_t seg_end = ge < u1 ? ge : u1;
            const bool whole = (u == gs && seg_end == ge);
            if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdGemvTc << 16) | 6)) break;
            tc_fence_after();
            int v[BN];
            {
                uint32_t r[16];
                const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
                tmem_ld_32x32b_x16(taddr, r);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = (int)r[j];
                if (BN == 32) {
                    tmem_ld_32x32b_x16(taddr + 16, r);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[(16 + j) % BN] = (int)r[j];
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
            const int row_in = quarter * 32 + lane;
            const int n = grp * kGcBM + row_in;
            if (whole) {
                gc_store_row<BN>(a, n, v);
            } else {
                const int slot = (grp == first_grp) ? 0 : 1;
                int4* dst = reinterpret_cast<int4*>(a.part + ((((int64_t)blockIdx.x * 2 + slot) * kGcBM + row_in) * BN));
#pragma unroll
                for (int j = 0; j < BN / 4; ++j) dst[j] = make_int4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                __threadfence();
                __syncwarp();
                const int c0 = gc_owner(gs, total, gridDim.x), c1 = gc_owner(ge - 1, total, gridDim.x);
                int prev = 0;
                if (lane == 0) prev = atomicAdd(a.counters + grp * 4 + quarter, 1);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == c1 - c0) {
                    __threadfence();
                    int sum[BN];
#pragma unroll
                    for (int j = 0; j < BN; ++j) sum[j] = 0;
                    for (int c = c0; c <= c1; ++c) {
                        const int sl = (grp == (int)(gc_begin(total, c, gridDim.x) / a.nkb)) ? 0 : 1;
                        const int4* src =
                            reinterpret_cast<const int4*>(a.part + ((((int64_t)c * 2 + sl) * kGcBM + row_in) * BN));
#pragma unroll
                        for (int j = 0; j < BN / 4; ++j) {
                            const int4 q = __ldcg(src + j);
                            sum[4 * j] += q.x;
                            sum[4 * j + 1] += q.y;
                            sum[4 * j + 2] += q.z;
                            sum[4 * j + 3] += q.w;
                        }
                    }
                    gc_store_row<BN>(a, n, sum);
                    if (lane == 0) a.counters[grp * 4 + quarter] = 0;   // left zero for the next call
                }
            }
            u = seg_end;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kCols);
    }
}

}  // namespace w8a8
