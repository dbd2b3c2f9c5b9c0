// Prefill W8A8 GEMM (a2 + a3) on CTA pairs: tcgen05.mma.cta_group::2 with
// 256 x 256 output tiles -- "Online INT8 W8A8 ...", Changes (gemm_a8w8
// per-token path).
//
//   acc[m,n] = sum_k A[m,k] B[n,k];  y[m,n] = bf16_rne( (float(acc) * sx[m]) * sw[n] )
//
// A cluster of two CTAs (one per SM) owns a 256-row x 256-column tile: CTA
// r loads rows [128 r, 128 r + 128) of the A tile and rows [128 r, 128 r +
// 128) of the B tile (its half of N), both 128-byte-swizzled K-major, with
// plain (non-multicast) TMA loads whose completion is counted on the leader
// CTA's barrier.  The leader's single MMA thread issues M=256, N=256, K=32
// instructions that read both CTAs' shared memory; each CTA's TMEM holds
// its 128 rows x 256 columns of the accumulator (two buffers of 256
// columns, so the epilogue of one tile overlaps the MMAs of the next).
// Per SM and per 128-byte k block the pair moves 32 KB into shared memory
// instead of the 48 KB a one-CTA 128 x 256 tile needs.
//
// Barriers: full[s] lives in the leader (armed by the leader with both
// CTAs' bytes); empty[s] and tfull[b] in both CTAs, signalled by the
// leader's tcgen05.commit multicast to the pair; tempty[b] in the leader,
// one arrival per epilogue warp of either CTA.  All waits are bounded; a
// cluster barrier keeps both CTAs alive until the other is done with its
// shared memory.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace w8a8 {

constexpr int kTc2BM = 256;       // rows per pair tile (128 per CTA)
constexpr int kTc2Threads = 192;
constexpr int kKernelIdGemmTc2 = 4;

// BN columns per pair tile: each CTA holds BN / 2 rows of B (256 or 160).
// As many stages as fit: at a few hundred tokens every pair streams its own
// weight columns from HBM, and the bytes in flight per SM set the pace.
template <int BN>
struct Tc2Smem {
    static constexpr int kA = 128 * kTcBK;                   // 16 KB per stage
    static constexpr int kB = (BN / 2) * kTcBK;              // 16 / 10 KB per stage (multiples of 1 KB)
    static constexpr int kStages = BN == 256 ? 6 : 8;
    static constexpr int kTiles = kStages * (kA + kB);
    static constexpr int kBars = (2 * kStages + 2 + 2 + 1) * 8;
    static constexpr int kBytes = 1024 + kTiles + kBars + 16;
    static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared-memory address of the same variable in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA tile load into this CTA's shared memory, completion counted on the
// barrier at cluster address `mbar` (the leader CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t mbar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t mbar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void tc2_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at this smem offset in both CTAs of the pair
// when this thread's previously issued MMAs complete.
__device__ __forceinline__ void tc2_commit_pair(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

template <int EPI, int BN = 256>
__global__ void __launch_bounds__(kTc2Threads, 1)
    gemm_i8_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcParams p) {
    static_assert(EPI == kEpiBf16 || EPI == kEpiS32 || EPI == kEpiMoeGated, "dense epilogues");
    static_assert(BN % 32 == 0 && (BN / 2) % 8 == 0 && BN <= 256, "pair tile width");
    constexpr int kCols = 2 * BN <= 256 ? 256 : 512;   // two accumulators of BN columns (a power of two)
    using SM = Tc2Smem<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + SM::kStages * SM::kA;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kTiles);
    uint64_t* full = bars;                      // leader only
    uint64_t* empty = bars + SM::kStages;        // both
    uint64_t* tfull = empty + SM::kStages;       // both
    uint64_t* tempty = tfull + 2;               // leader only
    uint64_t* mma_done = tempty + 2;            // leader only
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SM::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);       // one arrival per epilogue warp of the pair
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_tiles = p.num_m_tiles * p.num_n_tiles;
    const int cluster_id = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += nclusters) {
                const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, (kKernelIdGemmTc2 << 16) | 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (SM::kA + SM::kB));
                    tma_load_2d_pair(sA + stage * SM::kA, &tmA, fb, kb * kTcBK, mt * kTc2BM + (int)rank * 128);
                    tma_load_2d_pair(sB + stage * SM::kB, &tmB, fb, kb * kTcBK, nt * BN + (int)rank * (BN / 2));
                    issued |= 1u << stage;
                    last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == SM::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {
                for (int s = 0; s < SM::kStages; ++s)
                    if (issued & (1u << s))
                        mbar_wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, (kKernelIdGemmTc2 << 16) | 2,
                                          100000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kTc2BM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += nclusters) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, (kKernelIdGemmTc2 << 16) | 3)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdGemmTc2 << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * SM::kA);
                    const uint32_t b0 = smem_u32(sB + stage * SM::kB);
#pragma unroll
                    for (int kk = 0; kk < kTcBK / 32; ++kk)
                        tc2_mma_i8(d_tmem, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
                    tc2_commit_pair(&empty[stage]);   // frees this stage in both CTAs
                    if (++stage == SM::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc2_commit_pair(&tfull[acc]);         // accumulator ready in both CTAs
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(mma_done))
                         : "memory");
            mbar_wait_bounded(mma_done, 0u, nullptr, (kKernelIdGemmTc2 << 16) | 5, 100000000ull);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters) {
            const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
            if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdGemmTc2 << 16) | 6)) break;
            tc_fence_after();
            const int row = mt * kTc2BM + (int)rank * 128 + quarter * 32 + lane;
            const bool row_ok = row < p.M;
            float sxr = 0.0f;
            if ((EPI == kEpiBf16 || EPI == kEpiMoeGated) && row_ok) sxr = __ldg(p.sx + row);
            const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tq + (uint32_t)c, r);
                tc_wait_ld();
                const int n0 = nt * BN + c;
                if (!row_ok || n0 >= p.N) continue;
                if (EPI == kEpiBf16) {
                    uint16_t* yrow = reinterpret_cast<uint16_t*>(p.out) + (int64_t)row * p.N;
                    const float4* swv = reinterpret_cast<const float4*>(p.sw + n0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (n0 + v * 8 < p.N) {
                            const float4 s0 = __ldg(swv + 2 * v);
                            const float4 s1 = __ldg(swv + 2 * v + 1);
                            const float sw8[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                            uint32_t pk[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float lo =
                                    __fmul_rn(__fmul_rn(__int2float_rn((int)r[v * 8 + 2 * j]), sxr), sw8[2 * j]);
                                const float hi = __fmul_rn(__fmul_rn(__int2float_rn((int)r[v * 8 + 2 * j + 1]), sxr),
                                                           sw8[2 * j + 1]);
                                pk[j] = pack_bf16x2(lo, hi);
                            }
                            *reinterpret_cast<uint4*>(yrow + n0 + v * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                } else if (EPI == kEpiMoeGated) {
                    // columns n0 .. n0+31: 16 (gate, up) pairs -> a[row, n0/2 .. n0/2+15] (N % 32 == 0)
                    const float* swc = p.sw + n0;
                    float* arow = p.a_out + (int64_t)row * (p.N / 2) + n0 / 2;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float av[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int j = 8 * q + 2 * i;
                            const float vg = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j]), sxr), __ldg(swc + j));
                            const float vu =
                                __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 1]), sxr), __ldg(swc + j + 1));
                            av[i] = __fmul_rn(silu_proj(vg), vu);
                        }
                        *reinterpret_cast<float4*>(arow + 4 * q) = make_float4(av[0], av[1], av[2], av[3]);
                    }
                } else {
                    int32_t* orow = reinterpret_cast<int32_t*>(p.out) + (int64_t)row * p.N;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (n0 + v * 4 < p.N)
                            *reinterpret_cast<uint4*>(orow + n0 + v * 4) =
                                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader0 + (uint32_t)(acc * 8));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // neither CTA leaves while its peer may touch its shared memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kCols) : "memory");
    }
}

}  // namespace w8a8
