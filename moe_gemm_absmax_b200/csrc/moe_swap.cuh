// Routed-expert GEMMs (a8 + a9 and a10 + a11) on the 5th-generation tensor
// cores, swap-AB -- "Online INT8 W8A8 ...", Changes (MoE pipeline: fused
// gated-SiLU via interleaved w13, per-token int8 quant before gemm2, gemm2
// with weighted scatter/combine).
//
// With a few to a few dozen rows per expert, the expert's weights are the
// 128-row A operand of tcgen05.mma.kind::i8 and its rows' codes the narrow B
// operand (N = BN = 16, 32 or 64 rows of one expert):
//   D[n, m] = sum_k W_e[n, k] X[r_m, k]     (TMEM: lane = weight row n, column = row m)
// so each MMA reads a 128 x 32 weight slice at full rate and the kernel runs
// at the speed TMA streams the touched experts' weights out of HBM.
//
// Work unit: (token block, 128-row weight group) with the whole K; token
// blocks are BN consecutive expert-sorted rows of one expert (the plan's
// tile_off counts them per expert).  Units are dealt round-robin to a
// persistent grid; unit u = block * ngroups + group, so the groups of one
// block run side by side and the blocks of one expert reuse its weights
// through L2.
//
// gemm1 epilogue (GATED): v = (float(acc) * sx[r]) * s13[e, n]; rows n = 2i
// (gate) and 2i + 1 (up) sit in neighbouring lanes; a[r, i] = SiLU(g) * u,
// fp32.  gemm2 epilogue: y2 = (float(acc) * sa[r]) * s2[e, n]; w_r * y2
// stored at (token, slot) for the slot-order combine.
//
// Launched with programmatic dependent launch: the routing plan is complete
// when a kernel of this chain starts (each kernel of the chain lets its
// successor start only after its own wait on its predecessor, and the plan
// comes two or more kernels back), so the producer reads the plan and starts
// the weight tiles of its first stages before it waits for the codes of the
// kernel just before.
//
// Roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2..9
// epilogue: in the per-token form two groups of four (one warp per TMEM lane
// quarter), each owning one of the two accumulators and taking every other
// unit; in the group-128 form lane quarter x half of the token block's
// columns.  All waits are bounded.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace w8a8 {

constexpr int kMsBM = 128;          // weight rows per group (MMA M)
constexpr int kMsBK = 128;          // bytes of K per k block (a ring stage holds one or two)
constexpr int kKernelIdMoeSwap = 5;
constexpr int kMsMaxGroups = 32;    // K / 128 of the group-128 form
constexpr int kMsSlots = 8;         // TMEM accumulators of the group-128 form: one per k block in flight

template <int BN, bool G128 = false>
struct MsSmem {
    // k blocks per stage: two in the per-token form (its MMAs of N = 16-64
    // take 262 cycles per k block, too few to cover the ring's per-stage
    // hand-off); one in the group-128 form (a TMEM slot per k block)
    static constexpr int kKB = G128 ? 1 : 2;
    static constexpr int kStages = G128 ? (BN <= 32 ? 10 : 8) : (BN <= 32 ? 5 : 4);
    static constexpr int kNAcc = G128 ? kMsSlots : 2;
    static constexpr int kW1 = kMsBM * kMsBK;       // one k block of weights: 16 KB
    static constexpr int kX1 = BN * kMsBK;          // one k block of codes: 2 / 4 / 8 KB
    static constexpr int kW = kKB * kW1;
    static constexpr int kX = kKB * kX1;
    static constexpr int kStage = kW + kX;          // multiple of 1024
    static constexpr int kTiles = kStages * kStage;
    static constexpr int kBars = (2 * kStages + 2 * kNAcc + 1) * 8;
    // the plan (tile_off, offsets, counts: 3 x 257 ints) and, per epilogue
    // buffer, the token block's row data (scale, destination, weight)
    static constexpr int kPlanOff = kTiles + kBars + 16;
    static constexpr int kPlanInts = 3 * 260;
    static constexpr int kRowOff = kPlanOff + kPlanInts * 4;
    static constexpr int kRowBytes = 2 * 2 * 3 * 64 * 4;   // [epilogue group][buffer][3][64]
    // group-128: the token block's scales, [2 buffers][group][row] fp32
    static constexpr int kSxOff = (kRowOff + kRowBytes + 15) / 16 * 16;   // read as float4
    static constexpr int kSxBytes = G128 ? 2 * kMsMaxGroups * BN * 4 : 0;
    static constexpr int kBytes = 1024 + kSxOff + kSxBytes;
    static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
};

struct MoeSwapArgs {
    const float* sw;          // [E, rows] weight-row scales
    const float* sx;          // [R] scales of the sorted rows (gemm1: x codes, gemm2: a codes)
    const int32_t* counts;    // [E]
    const int32_t* offsets;   // [E + 1]
    const int32_t* tile_off;  // [E + 1] prefix of ceil(counts / BN)
    int E, rows, K;           // rows: 2I (gemm1) or H (gemm2)
    int ngroups, nkb;         // rows / 128, K / 128
    // gemm1
    float* a_out;             // [R, I] fp32 gated intermediate
    // gemm2
    const int32_t* row_tok;   // [R]
    const int32_t* row_slot;  // [R]
    const float* row_w;       // [R]
    float* contrib;           // [T * topk, H] w * y2 at (token, slot)
    int topk;
    int early_plan;           // the plan comes two or more kernels back: read it before the wait
    // group-128 form (K / 128 groups, bf16 scales)
    const uint16_t* gsw;      // [E * rows, K / 128]
    const uint16_t* gsx;      // [R, K / 128] of the sorted rows
    const uint8_t* gsw_u8;    // two-level trunk format instead of gsw: [E * rows, K / 256] u8 ...
    const uint16_t* gsw_row;  // ... times a bf16 row scale [E * rows]
};

// Token block b (in tile_off numbering) -> expert, first sorted row, rows;
// the plan's arrays in shared memory (sp: tile_off [E + 1], offsets, counts).
struct MsBlock {
    int e, row0, valid;
};

__device__ __forceinline__ MsBlock ms_block(const int* sp, int E, int b, int BN) {
    const int* tile_off = sp;
    const int* offsets = sp + 260;
    const int* counts = sp + 520;
    int lo = 0, hi = E;   // largest e with tile_off[e] <= b (experts without rows own no block)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_off[mid] <= b) lo = mid;
        else hi = mid;
    }
    MsBlock k;
    k.e = lo;
    const int lb = b - tile_off[lo];
    k.row0 = offsets[lo] + lb * BN;
    k.valid = min(BN, counts[lo] - lb * BN);
    return k;
}

// Fetch into L2 without waiting (the next unit's weight scales, which come
// from HBM the first time an expert row is touched).
__device__ __forceinline__ void ms_prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

template <int NT>
__device__ __forceinline__ void ms_epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }

// Named barrier of one epilogue group of 4 warps (ids 1 and 2).
__device__ __forceinline__ void ms_group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// Threads: weight producer warp, MMA warp, 8 epilogue warps (two groups of
// four for the per-token form, lane quarter x column half for the group-128
// form), then the token-code producer warp.  Each k block takes one weight
// box and one code box; an issuing thread completes about one box per ~340
// cycles whatever its size, so with both on one thread a CTA would stream
// its 16 KB weight boxes at about half the rate one thread reaches alone.
constexpr int kMsXWarp = 10;
template <bool G128>
constexpr int ms_threads() { return 352; }

template <int BN, bool GATED, bool G128 = false>
__global__ void __launch_bounds__(ms_threads<G128>(), 1)
    moe_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, MoeSwapArgs a) {
    static_assert(BN == 16 || BN == 32 || BN == 64, "BN");
    using SM = MsSmem<BN, G128>;
    constexpr int STAGES = SM::kStages;
    constexpr int NACC = SM::kNAcc;
    constexpr int kCols = G128 ? kMsSlots * BN : (2 * BN >= 32 ? 2 * BN : 32);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kTiles);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + NACC;
    uint64_t* mma_done = tempty + NACC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // group-128 form with units of at most 4 groups (K <= 512): two epilogue
    // groups of four warps take alternate units, each with its own 4 TMEM
    // slots (see the epilogue)
    const bool alt = G128 && a.nkb <= 4;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], (G128 && !alt) ? 256 : 128);
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
    // The plan is complete (see above); the codes of the kernel just before may not be.
    if (!a.early_plan) asm volatile("griddepcontrol.wait;" ::: "memory");
    int* sp = reinterpret_cast<int*>(smem + SM::kPlanOff);
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
        sp[i] = __ldcg(a.tile_off + i);
        sp[260 + i] = __ldcg(a.offsets + i);
        sp[520 + i] = i < a.E ? __ldcg(a.counts + i) : 0;
    }
    __syncthreads();
    const int nunits = sp[a.E] * a.ngroups;
    const int my_units = nunits > (int)blockIdx.x ? (nunits - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int nst = (a.nkb + SM::kKB - 1) / SM::kKB;   // stages per unit
    const int64_t my_stages = (int64_t)my_units * nst;
    const int pre = my_stages < STAGES ? (int)my_stages : STAGES;   // stages armed before the wait
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmW);
        prefetch_tensormap(&tmX);
        for (int i = 0; i < pre; ++i) {   // unit blockIdx.x + (i / nst) * gridDim.x, k blocks from kKB (i % nst)
            const int u = blockIdx.x + (i / nst) * gridDim.x;
            const int b = u / a.ngroups, g = u - b * a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            mbar_arrive_expect_tx(&full[i], (uint32_t)SM::kStage);
#pragma unroll
            for (int j = 0; j < SM::kKB; ++j)   // a k block past K (odd count) reads as zeros
                tma_load_2d(smem + i * SM::kStage + j * SM::kW1, &tmW, &full[i], ((i % nst) * SM::kKB + j) * kMsBK,
                            k.e * a.rows + g * kMsBM);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 0 || warp == kMsXWarp) {
        // ---------------------------------------------------------- producers
        // warp 0: weight boxes (arming full[s] with the stage's bytes; the first
        // `pre` stages were armed and started before the wait above); warp
        // kMsXWarp: the token codes of the same stages.  A code box that lands
        // before its stage is armed only takes the barrier's transaction count
        // below zero while the arrival is still pending.
        if (lane == 0) {
            const bool codes = warp == kMsXWarp;
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_phase = 0;
            int64_t i = 0;   // stage count of this CTA
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const int b = u / a.ngroups, g = u - b * a.ngroups;
                const MsBlock k = ms_block(sp, a.E, b, BN);
                const int wrow = k.e * a.rows + g * kMsBM;
                for (int kb = 0; kb < a.nkb; kb += SM::kKB, ++i) {
                    if (i >= pre) {
                        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, (kKernelIdMoeSwap << 16) | 1)) {
                            ok = false;
                            break;
                        }
                        if (!codes) {
                            mbar_arrive_expect_tx(&full[stage], (uint32_t)SM::kStage);
#pragma unroll
                            for (int j = 0; j < SM::kKB; ++j)
                                tma_load_2d(smem + stage * SM::kStage + j * SM::kW1, &tmW, &full[stage],
                                            (kb + j) * kMsBK, wrow);
                        }
                    }
                    if (codes) {
#pragma unroll
                        for (int j = 0; j < SM::kKB; ++j)
                            tma_load_2d(smem + stage * SM::kStage + SM::kW + j * SM::kX1, &tmX, &full[stage],
                                        (kb + j) * kMsBK, k.row0);
                    }
                    issued |= 1u << stage;
                    last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // drain: every copy this thread started lands before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s))
                        mbar_wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, (kKernelIdMoeSwap << 16) | 2,
                                          100000000ull);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (G128 && lane == 0) {
            // one accumulator slot per k block (= group): every slot holds the
            // conversion bias when it is released, so the MMAs always accumulate
            // and a slot's first use waits for phase 0 like every later one
            // alternate-units mode (units of at most 4 groups): unit i of this
            // CTA uses slots 4 (i & 1) + kb, each slot once every other unit
            constexpr uint32_t idesc = idesc_i8(kMsBM, BN);
            int stage = 0, slot = 0, i = 0;
            uint32_t phase = 0, sphase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x, ++i) {
                if (alt) {
                    slot = 4 * (i & 1);
                    sphase = (uint32_t)(i >> 1) & 1u;
                }
                for (int kb = 0; kb < a.nkb; ++kb) {
                    if (!mbar_wait_bounded(&tempty[slot], sphase, abort_flag, (kKernelIdMoeSwap << 16) | 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdMoeSwap << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(slot * BN);
                    const uint32_t w0 = smem_u32(smem + stage * SM::kStage);
                    const uint32_t x0 = w0 + SM::kW;
#pragma unroll
                    for (int kk = 0; kk < kMsBK / 32; ++kk)
                        tc_mma_i8(d_tmem, smem_desc_k_sw128(w0 + kk * 32), smem_desc_k_sw128(x0 + kk * 32), idesc, 1u);
                    tc_commit(&empty[stage]);
                    tc_commit(&tfull[slot]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++slot == kMsSlots) {   // (never reached in the alternate-units mode)
                        slot = 0;
                        sphase ^= 1u;
                    }
                }
            }
            tc_commit(mma_done);
            mbar_wait_bounded(mma_done, 0u, nullptr, (kKernelIdMoeSwap << 16) | 5, 100000000ull);
        } else if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kMsBM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, (kKernelIdMoeSwap << 16) | 3)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < a.nkb; kb += SM::kKB) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdMoeSwap << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < SM::kKB; ++j) {
                        const uint32_t w0 = smem_u32(smem + stage * SM::kStage + j * SM::kW1);
                        const uint32_t x0 = smem_u32(smem + stage * SM::kStage + SM::kW + j * SM::kX1);
#pragma unroll
                        for (int kk = 0; kk < kMsBK / 32; ++kk)
                            tc_mma_i8(d_tmem, smem_desc_k_sw128(w0 + kk * 32), smem_desc_k_sw128(x0 + kk * 32),
                                      idesc, (kb > 0 || j > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) {
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
            }
            tc_commit(mma_done);
            mbar_wait_bounded(mma_done, 0u, nullptr, (kKernelIdMoeSwap << 16) | 5, 100000000ull);
        }
    } else if constexpr (G128) {
      if (alt) {
        // ---------------------------------------------------------- epilogue, group-128, alternate units
        // Units of at most 4 groups: two groups of four warps (one per TMEM
        // lane quarter, all BN columns each, read 32 at a time) take alternate
        // units; group j owns slots 4j .. 4j+3, one per k block of its unit.
        // The promotion is that of the column-split form below.
        const int grp = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int et = (threadIdx.x - 64) & 127;   // 0 .. 127 within the group
        float* s_row = reinterpret_cast<float*>(smem + SM::kRowOff) + grp * 2 * 3 * 64;   // [2][3][64]
        float* s_sxg = reinterpret_cast<float*>(smem + SM::kSxOff) + grp * 2 * 4 * BN;    // [2][4][BN]
        const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16);
        const int G = a.nkb;
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) {
#pragma unroll
            for (int c = 0; c < BN; c += 8) tmem_st_32x32b_x8_fill(tq + (uint32_t)((4 * grp + sl) * BN + c), 0x4B400000u);
        }
        tc_wait_st();
        tc_fence_before();
        for (int sl = 0; sl < 4; ++sl) mbar_arrive(&tempty[4 * grp + sl]);
        // the token block's group scales (thread et: row mm of groups g0, g0 + 128 / BN, ...),
        // loaded one unit ahead
        constexpr int JA = (4 * BN + 127) / 128;
        constexpr int kGStepA = 128 / BN;
        const int mm = et & (BN - 1), g0 = et / BN;
        float nx_g[JA];
        float nx_w = 0.0f;
        int nx_dst = 0;
        auto fetch = [&](int u) {
            const int b = u / a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            {   // this thread's weight-row scales of unit u
                const int64_t wr = (int64_t)k.e * a.rows + (u - b * a.ngroups) * kMsBM + quarter * 32 + lane;
                if (a.gsw_u8) {
                    ms_prefetch_l2(a.gsw_u8 + wr * (G / 2));
                    ms_prefetch_l2(a.gsw_row + wr);
                } else {
                    ms_prefetch_l2(a.gsw + wr * G);
                }
            }
#pragma unroll
            for (int j = 0; j < JA; ++j) {
                const int gg = g0 + kGStepA * j;
                nx_g[j] = (mm < k.valid && gg < G) ? bf16_bits_to_float(__ldcg(a.gsx + (int64_t)(k.row0 + mm) * G + gg)) : 0.0f;
            }
            if constexpr (!GATED) {
                if (et < k.valid) {
                    const int r = k.row0 + et;
                    nx_dst = __ldcg(a.row_tok + r) * a.topk + __ldcg(a.row_slot + r);
                    nx_w = __ldcg(a.row_w + r);
                }
            }
        };
        const int u0 = (int)blockIdx.x + grp * (int)gridDim.x;
        const int ustep = 2 * (int)gridDim.x;
        if (u0 < nunits) fetch(u0);
        int buf = 0;
        uint32_t kphase = 0;
        const uint64_t magic2 = 0x4B4000004B400000ull;
        const uint64_t inv2 = f2_pack(0.0078125f, 0.0078125f);
        for (int u = u0; u < nunits; u += ustep) {
            const int b = u / a.ngroups, g = u - b * a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            float* rs = s_row + buf * 3 * 64;
            float* sxs = s_sxg + buf * 4 * BN;
#pragma unroll
            for (int j = 0; j < JA; ++j) {
                const int gg = g0 + kGStepA * j;
                if (gg < G) sxs[gg * BN + mm] = nx_g[j];
            }
            if constexpr (!GATED) {
                if (et < BN) {
                    const bool have = et < k.valid;
                    rs[64 + et] = __int_as_float(have ? nx_dst : 0);
                    rs[128 + et] = have ? nx_w : 0.0f;
                }
            }
            if (u + ustep < nunits) fetch(u + ustep);
            ms_group_sync(1 + grp);   // also: the group is done with this buffer's use two units ago
            buf ^= 1;
            const int n = g * kMsBM + quarter * 32 + lane;   // weight row of expert e
            const int64_t wr = (int64_t)k.e * a.rows + n;
            const uint16_t* swrow = a.gsw + wr * G;
            const uint8_t* swu8 = a.gsw_u8 ? a.gsw_u8 + wr * (G / 2) : nullptr;
            const float swr = a.gsw_u8 ? bf16_bits_to_float(__ldg(a.gsw_row + wr)) : 0.0f;
            uint64_t y2[BN / 2];
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) y2[i] = 0ull;
            bool ok = true;
            for (int kb = 0; kb < G; ++kb) {
                const float swg = swu8 ? __fmul_rn((float)__ldg(swu8 + kb / 2), swr) : bf16_bits_to_float(__ldg(swrow + kb));
                const int slot = 4 * grp + kb;
                if (!mbar_wait_bounded(&tfull[slot], kphase, abort_flag, (kKernelIdMoeSwap << 16) | 6)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t sw2 = f2_pack(swg, swg);
                const float* sxk = sxs + kb * BN;
                const uint32_t ta = tq + (uint32_t)(slot * BN);
                constexpr int CW = BN < 32 ? BN : 32;   // columns per TMEM read
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += CW) {
                    uint32_t r[CW];
                    if constexpr (CW == 16) tmem_ld_32x32b_x16(ta + (uint32_t)c0, r);
                    else tmem_ld_32x32b_x32(ta + (uint32_t)c0, r);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < CW; c += 8) tmem_st_32x32b_x8_fill(ta + (uint32_t)(c0 + c), 0x4B400000u);
#pragma unroll
                    for (int q = 0; q < CW / 4; ++q) {
                        const float4 s4 = *reinterpret_cast<const float4*>(sxk + c0 + 4 * q);
                        const uint64_t sc01 = f2_mul(f2_pack(s4.x, s4.y), sw2);
                        const uint64_t sc23 = f2_mul(f2_pack(s4.z, s4.w), sw2);
                        const uint64_t p01 =
                            f2_sub(f2_pack(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])), magic2);
                        const uint64_t p23 =
                            f2_sub(f2_pack(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])), magic2);
                        y2[c0 / 2 + 2 * q] = f2_fma(p01, sc01, y2[c0 / 2 + 2 * q]);
                        y2[c0 / 2 + 2 * q + 1] = f2_fma(p23, sc23, y2[c0 / 2 + 2 * q + 1]);
                    }
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&tempty[slot]);   // the slot goes back to the MMA
            }
            if (!ok) break;
            kphase ^= 1u;
            float v[BN];
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) f2_unpack(f2_mul(y2[i], inv2), v[2 * i], v[2 * i + 1]);
            if constexpr (GATED) {
                const int I = a.rows >> 1;
                float* arow = a.a_out + (int64_t)k.row0 * I + (n >> 1);
                const bool odd = lane & 1;
#pragma unroll
                for (int j = 0; j < BN / 2; ++j) {
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? v[j] : v[j + BN / 2], 1);
                    const float gv = odd ? other : v[j];
                    const float uv = odd ? v[j + BN / 2] : other;
                    const int m = j + (odd ? BN / 2 : 0);
                    if (m < k.valid) arow[(int64_t)m * I] = __fmul_rn(silu_proj(gv), uv);
                }
            } else {
                const int H = a.rows;
#pragma unroll
                for (int m = 0; m < BN; ++m)
                    if (m < k.valid)
                        a.contrib[(int64_t)__float_as_int(rs[64 + m]) * H + n] = __fmul_rn(rs[128 + m], v[m]);
            }
        }
      } else {
        // ---------------------------------------------------------- epilogue, group-128
        // y[n, m] = sum over groups g ascending of fma(float(p_g), sx[m, g] * sw[n, g], y)
        // in fp32, then * 1/128: two token rows per instruction (f32x2).  Each
        // slot holds the bias 0x4B400000 (the bits of 1.5 * 2^23) before its
        // MMAs, so it ends holding the float bits of 1.5 * 2^23 + p_g exactly
        // (|p_g| <= 127^2 * 128 < 2^22) and float(p_g) is one subtraction.
        // Eight warps: TMEM lane quarter (warp % 4) x half of the block's columns.
        constexpr int HC = BN / 2;
        const int quarter = warp & 3;
        const int c0 = ((warp - 2) >> 2) * HC;
        const int et = threadIdx.x - 64;   // 0 .. 255
        float* s_row = reinterpret_cast<float*>(smem + SM::kRowOff);   // [2][3][64]
        float* s_sx = reinterpret_cast<float*>(smem + SM::kSxOff);     // [2][kMsMaxGroups][BN]
        const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0;
        const int G = a.nkb;
#pragma unroll 1
        for (int sl = 0; sl < kMsSlots; ++sl) {
#pragma unroll
            for (int c = 0; c < HC; c += 8) tmem_st_32x32b_x8_fill(tq + (uint32_t)(sl * BN + c), 0x4B400000u);
        }
        tc_wait_st();
        tc_fence_before();
        for (int sl = 0; sl < kMsSlots; ++sl) mbar_arrive(&tempty[sl]);
        // the token block's group scales: thread et holds row mm of groups
        // g0, g0 + 256 / BN, ...; loaded one unit ahead
        constexpr int J = BN * kMsMaxGroups / 256;
        constexpr int kGStep = 256 / BN;
        const int mm = et & (BN - 1), g0 = et / BN;
        float nx_g[J];
        float nx_w = 0.0f;
        int nx_dst = 0;
        auto fetch = [&](int u) {
            const int b = u / a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            {   // this thread's weight-row scales of unit u
                const int64_t wr = (int64_t)k.e * a.rows + (u - b * a.ngroups) * kMsBM + quarter * 32 + lane;
                if (a.gsw_u8) {
                    ms_prefetch_l2(a.gsw_u8 + wr * (G / 2));
                    ms_prefetch_l2(a.gsw_row + wr);
                } else {
                    ms_prefetch_l2(a.gsw + wr * G);
                }
            }
            const bool have = mm < k.valid;
            const uint16_t* src = a.gsx + (int64_t)(k.row0 + mm) * G;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int gg = g0 + kGStep * j;
                nx_g[j] = (have && gg < G) ? bf16_bits_to_float(__ldcg(src + gg)) : 0.0f;
            }
            if constexpr (!GATED) {
                if (et < k.valid) {
                    const int r = k.row0 + et;
                    nx_dst = __ldcg(a.row_tok + r) * a.topk + __ldcg(a.row_slot + r);
                    nx_w = __ldcg(a.row_w + r);
                }
            }
        };
        if ((int)blockIdx.x < nunits) fetch(blockIdx.x);
        int slot = 0, buf = 0;
        uint32_t sphase = 0;
        const uint64_t magic2 = 0x4B4000004B400000ull;
        const uint64_t inv2 = f2_pack(0.0078125f, 0.0078125f);
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
            const int b = u / a.ngroups, g = u - b * a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            float* rs = s_row + buf * 3 * 64;
            float* sxs = s_sx + buf * kMsMaxGroups * BN;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int gg = g0 + kGStep * j;
                if (gg < G) sxs[gg * BN + mm] = nx_g[j];
            }
            if constexpr (!GATED) {
                if (et < BN) {
                    const bool have = et < k.valid;
                    rs[64 + et] = __int_as_float(have ? nx_dst : 0);
                    rs[128 + et] = have ? nx_w : 0.0f;
                }
            }
            if (u + (int)gridDim.x < nunits) fetch(u + gridDim.x);
            ms_epi_sync<256>();   // also: every warp is done with this buffer's use two units ago
            buf ^= 1;
            const int n = g * kMsBM + quarter * 32 + lane;   // weight row of expert e
            const int64_t wr = (int64_t)k.e * a.rows + n;
            const uint16_t* swrow = a.gsw + wr * G;
            // weight scale of group kb: bf16, or (trunk format) u8 per 256 of K times a bf16 row scale
            const uint8_t* swu8 = a.gsw_u8 ? a.gsw_u8 + wr * (G / 2) : nullptr;
            const float swr = a.gsw_u8 ? bf16_bits_to_float(__ldg(a.gsw_row + wr)) : 0.0f;
            auto wscale = [&](int kb) -> float {
                return swu8 ? __fmul_rn((float)__ldg(swu8 + kb / 2), swr) : bf16_bits_to_float(__ldg(swrow + kb));
            };
            float sw_next = wscale(0);
            uint64_t y2[HC / 2];
#pragma unroll
            for (int i = 0; i < HC / 2; ++i) y2[i] = 0ull;
            bool ok = true;
            for (int kb = 0; kb < G; ++kb) {
                const float swg = sw_next;
                if (kb + 1 < G) sw_next = wscale(kb + 1);
                if (!mbar_wait_bounded(&tfull[slot], sphase, abort_flag, (kKernelIdMoeSwap << 16) | 6)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t sw2 = f2_pack(swg, swg);
                const float* sxk = sxs + kb * BN + c0;
                // this warp's columns into registers (one wait), the bias back
                // into TMEM, the promotion while those stores land, the release
                const uint32_t ta = tq + (uint32_t)(slot * BN);
                uint32_t r[HC];
                if constexpr (HC == 8) tmem_ld_32x32b_x8(ta, r);
                else if constexpr (HC == 16) tmem_ld_32x32b_x16(ta, r);
                else tmem_ld_32x32b_x32(ta, r);
                tc_wait_ld();
#pragma unroll
                for (int c = 0; c < HC; c += 8) tmem_st_32x32b_x8_fill(ta + (uint32_t)c, 0x4B400000u);
#pragma unroll
                for (int q = 0; q < HC / 4; ++q) {
                    const float4 s4 = *reinterpret_cast<const float4*>(sxk + 4 * q);
                    const uint64_t sc01 = f2_mul(f2_pack(s4.x, s4.y), sw2);
                    const uint64_t sc23 = f2_mul(f2_pack(s4.z, s4.w), sw2);
                    const uint64_t p01 = f2_sub(f2_pack(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])), magic2);
                    const uint64_t p23 =
                        f2_sub(f2_pack(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])), magic2);
                    y2[2 * q] = f2_fma(p01, sc01, y2[2 * q]);
                    y2[2 * q + 1] = f2_fma(p23, sc23, y2[2 * q + 1]);
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&tempty[slot]);   // the slot goes back to the MMA
                if (++slot == kMsSlots) {
                    slot = 0;
                    sphase ^= 1u;
                }
            }
            if (!ok) break;
            float v[HC];
#pragma unroll
            for (int i = 0; i < HC / 2; ++i) f2_unpack(f2_mul(y2[i], inv2), v[2 * i], v[2 * i + 1]);
            if constexpr (GATED) {
                // lanes 2i (gate_i) and 2i+1 (up_i) split the columns: the even
                // lane finishes the first half, the odd lane the second
                const int I = a.rows >> 1;
                float* arow = a.a_out + (int64_t)k.row0 * I + (n >> 1);
                const bool odd = lane & 1;
#pragma unroll
                for (int j = 0; j < HC / 2; ++j) {
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? v[j] : v[j + HC / 2], 1);
                    const float gv = odd ? other : v[j];
                    const float uv = odd ? v[j + HC / 2] : other;
                    const int m = c0 + j + (odd ? HC / 2 : 0);
                    if (m < k.valid) arow[(int64_t)m * I] = __fmul_rn(silu_proj(gv), uv);
                }
            } else {
                const int H = a.rows;
#pragma unroll
                for (int m = 0; m < HC; ++m)
                    if (c0 + m < k.valid)
                        a.contrib[(int64_t)__float_as_int(rs[64 + c0 + m]) * H + n] = __fmul_rn(rs[128 + c0 + m], v[m]);
            }
        }
      }
    } else {
        // ---------------------------------------------------------- epilogue
        // Two groups of four warps (one per TMEM lane quarter); group j owns
        // accumulator j and takes every other unit of this CTA, so that one
        // group's per-unit latency (row data, TMEM read, stores) overlaps the
        // other's.
        const int grp = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int et = (threadIdx.x - 64) & 127;   // 0 .. 127 within the group
        float* s_row = reinterpret_cast<float*>(smem + SM::kRowOff) + grp * 2 * 3 * 64;   // [2][3][64]
        const int acc = grp;
        const int ustep = 2 * (int)gridDim.x;
        int buf = 0;
        uint32_t acc_phase = 0;
        // row data of a token block, one row per thread (et < BN): loaded one
        // unit ahead so that its latency hides behind the current unit
        float nx_sx = 0.0f, nx_w = 0.0f;
        int nx_dst = 0;
        auto fetch = [&](int u) {
            const int b = u / a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            if (et < k.valid) {
                const int r = k.row0 + et;
                nx_sx = __ldcg(a.sx + r);
                if constexpr (!GATED) {
                    nx_dst = __ldcg(a.row_tok + r) * a.topk + __ldcg(a.row_slot + r);
                    nx_w = __ldcg(a.row_w + r);
                }
            }
        };
        // this thread's weight-row scale of unit u, into L2 one unit ahead
        auto prefetch_sw = [&](int u) {
            const int b = u / a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            ms_prefetch_l2(a.sw + (int64_t)k.e * a.rows + (u - b * a.ngroups) * kMsBM + quarter * 32 + lane);
        };
        const int u0 = (int)blockIdx.x + grp * (int)gridDim.x;
        if (et < BN && u0 < nunits) fetch(u0);
        if (u0 < nunits) prefetch_sw(u0);
        for (int u = u0; u < nunits; u += ustep) {
            const int b = u / a.ngroups, g = u - b * a.ngroups;
            const MsBlock k = ms_block(sp, a.E, b, BN);
            float* rs = s_row + buf * 3 * 64;
            if (et < BN) {
                const bool have = et < k.valid;
                rs[et] = have ? nx_sx : 0.0f;
                if constexpr (!GATED) {
                    rs[64 + et] = __int_as_float(have ? nx_dst : 0);
                    rs[128 + et] = have ? nx_w : 0.0f;
                }
                if (u + ustep < nunits) fetch(u + ustep);
            }
            if (u + ustep < nunits) prefetch_sw(u + ustep);
            ms_group_sync(1 + grp);   // also: the group is done with this buffer's use two units ago
            buf ^= 1;
            if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdMoeSwap << 16) | 6)) break;
            tc_fence_after();
            int v[BN];
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll
            for (int c = 0; c < BN; c += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(taddr + (uint32_t)c, r);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[c + j] = (int)r[j];
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc_phase ^= 1u;
            const int n = g * kMsBM + quarter * 32 + lane;   // weight row of expert e
            const float swn = __ldg(a.sw + (int64_t)k.e * a.rows + n);
            if constexpr (GATED) {
                // lanes 2i (gate_i) and 2i+1 (up_i) split the columns: the even
                // lane finishes the first half, the odd lane the second
                const int I = a.rows >> 1;
                float* arow = a.a_out + (int64_t)k.row0 * I + (n >> 1);
                const bool odd = lane & 1;
                float val[BN];
#pragma unroll
                for (int m = 0; m < BN; ++m) val[m] = __fmul_rn(__fmul_rn(__int2float_rn(v[m]), rs[m]), swn);
#pragma unroll
                for (int j = 0; j < BN / 2; ++j) {
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? val[j] : val[j + BN / 2], 1);
                    const float gv = odd ? other : val[j];
                    const float uv = odd ? val[j + BN / 2] : other;
                    const int m = j + (odd ? BN / 2 : 0);
                    if (m < k.valid) arow[(int64_t)m * I] = __fmul_rn(silu_proj(gv), uv);
                }
            } else {
                const int H = a.rows;
#pragma unroll
                for (int m = 0; m < BN; ++m) {
                    if (m < k.valid) {
                        const float y2 = __fmul_rn(__fmul_rn(__int2float_rn(v[m]), rs[m]), swn);
                        a.contrib[(int64_t)__float_as_int(rs[64 + m]) * H + n] = __fmul_rn(rs[128 + m], y2);
                    }
                }
            }
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
