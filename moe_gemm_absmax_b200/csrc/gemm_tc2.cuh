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
// instead of the 48 KB a one-CTA 128 x 256 tile needs.  Eight epilogue
// warps (TMEM lane quarter x alternate 32-column chunks) keep the next
// chunk's TMEM load in flight while they convert the current one, with the
// tile's column scales staged once in shared memory: with few k blocks per
// tile (K = 2048) or one tile per cluster (a few hundred tokens) the
// epilogue, not the MMA, would otherwise set the pace.
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
constexpr int kTc2Epi = 8;        // epilogue warps: TMEM lane quarter x alternate 32-column chunks
constexpr int kTc2Threads = 64 + 32 * kTc2Epi;
constexpr int kKernelIdGemmTc2 = 4;

// BN columns per pair tile: each CTA holds BN / 2 rows of B (256, 160 or 144).
// As many stages as fit.  A stage carries enough MMA work to cover the ring's
// per-stage hand-off (MMA completion -> empty -> producer -> full -> MMA
// thread): one k block for the 256 and 160 tiles (512 / 320 cycles of MMA),
// two for the 144 tile (2 x 288).
template <int BN>
struct Tc2Smem {
    // k blocks per stage: the 144 tile (a few hundred tokens, one tile per
    // cluster) takes two, halving the stage hand-offs per MMA
    static constexpr int kKB = BN == 144 ? 2 : 1;
    static constexpr int kA1 = 128 * kTcBK;                  // one k block of A: 16 KB
    static constexpr int kB1 = (BN / 2) * kTcBK;             // one k block of B: 16 / 10 / 9 KB (multiples of 1 KB)
    static constexpr int kA = kKB * kA1;
    static constexpr int kB = kKB * kB1;
    static constexpr int kStages = BN == 256 ? 6 : (BN == 144 ? 4 : 8);
    static constexpr int kTiles = kStages * (kA + kB);
    static constexpr int kBars = (2 * kStages + 2 + 2 + 1) * 8;
    // each epilogue warp's copy of the tile's column scales (fp32)
    static constexpr int kEpiOff = kTiles + (kBars + 16 + 15) / 16 * 16;
    static constexpr int kEpiBytes = kTc2Epi * BN * 4;
    static constexpr int kBytes = 1024 + kEpiOff + kEpiBytes;
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

// Two fp32 values to bf16 (round to nearest even each) packed lo | hi << 16, one instruction.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t mbar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// Arrive on a peer CTA's barrier with the default (CTA-scope release)
// semantics: for hand-offs that publish no memory of this CTA's, only that
// its tcgen05 loads are done (ordered by tcgen05.fence::before_thread_sync).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(mbar) : "memory");
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
    static_assert(BN % 16 == 0 && (BN / 2) % 8 == 0 && BN <= 256, "pair tile width");
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
    float* epi_scratch = reinterpret_cast<float*>(smem + SM::kEpiOff);

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
            mbar_init(&tempty[b], 2 * kTc2Epi);   // one arrival per epilogue warp of the pair
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
                for (int kb = 0; kb < p.num_k_blocks; kb += SM::kKB) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, (kKernelIdGemmTc2 << 16) | 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (SM::kA + SM::kB));
                    // a k block past K (odd count) reads as zeros and adds nothing
#pragma unroll
                    for (int j = 0; j < SM::kKB; ++j) {
                        tma_load_2d_pair(sA + stage * SM::kA + j * SM::kA1, &tmA, fb, (kb + j) * kTcBK,
                                         mt * kTc2BM + (int)rank * 128);
                        tma_load_2d_pair(sB + stage * SM::kB + j * SM::kB1, &tmB, fb, (kb + j) * kTcBK,
                                         nt * BN + (int)rank * (BN / 2));
                    }
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
                for (int kb = 0; kb < p.num_k_blocks; kb += SM::kKB) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdGemmTc2 << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < SM::kKB; ++j) {
                        const uint32_t a0 = smem_u32(sA + stage * SM::kA + j * SM::kA1);
                        const uint32_t b0 = smem_u32(sB + stage * SM::kB + j * SM::kB1);
#pragma unroll
                        for (int kk = 0; kk < kTcBK / 32; ++kk)
                            tc2_mma_i8(d_tmem, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32),
                                       idesc, (kb > 0 || j > 0 || kk > 0) ? 1u : 0u);
                    }
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
        const int quarter = warp & 3;              // TMEM lanes [32 q, 32 q + 32)
        const int chalf = (warp - 2) >> 2;         // chunks c = 32 chalf + 64 i
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
        float* sw_s = epi_scratch + (warp - 2) * BN;   // this warp's copy of the tile's column scales
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters) {
            const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
            const int row = mt * kTc2BM + (int)rank * 128 + quarter * 32 + lane;
            const bool row_ok = row < p.M;
            float sxr = 0.0f;
            if ((EPI == kEpiBf16 || EPI == kEpiMoeGated) && row_ok) sxr = __ldg(p.sx + row);
            if (EPI == kEpiBf16 || EPI == kEpiMoeGated) {
                // the tile's BN column scales (N % 8 == 0: a 4-column vector is all in or all out)
                __syncwarp();   // the previous tile's reads are done
                for (int v = lane; v < BN / 4; v += 32) {
                    const int n = nt * BN + 4 * v;
                    float4 sv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (n < p.N) sv = __ldg(reinterpret_cast<const float4*>(p.sw + n));
                    *reinterpret_cast<float4*>(sw_s + 4 * v) = sv;
                }
                __syncwarp();
            }
            if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdGemmTc2 << 16) | 6)) break;
            tc_fence_after();
            const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            // one 32-column chunk: convert and store (the next chunk's TMEM load is in flight)
            auto chunk = [&](const uint32_t (&r)[32], int c) {
                const int n0 = nt * BN + c;
                if (!row_ok || n0 >= p.N) return;
                // the tile's columns in this chunk (BN % 32 == 16: the last chunk holds
                // 16; its TMEM load reads 16 columns past the tile, which are ignored)
                const int ncol = BN - c < 32 ? BN - c : 32;
                if (EPI == kEpiBf16) {
                    uint16_t* yrow = reinterpret_cast<uint16_t*>(p.out) + (int64_t)row * p.N;
                    const uint64_t sx2 = f2_pack(sxr, sxr);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (v * 8 < ncol && n0 + v * 8 < p.N) {
                            const float4 s0 = *reinterpret_cast<const float4*>(sw_s + c + 8 * v);
                            const float4 s1 = *reinterpret_cast<const float4*>(sw_s + c + 8 * v + 4);
                            const float sw8[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                            uint32_t pk[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint64_t a2 = f2_pack(__int2float_rn((int)r[v * 8 + 2 * j]),
                                                            __int2float_rn((int)r[v * 8 + 2 * j + 1]));
                                float lo, hi;
                                f2_unpack(f2_mul(f2_mul(a2, sx2), f2_pack(sw8[2 * j], sw8[2 * j + 1])), lo, hi);
                                pk[j] = cvt_bf16x2(lo, hi);
                            }
                            *reinterpret_cast<uint4*>(yrow + n0 + v * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                } else if (EPI == kEpiMoeGated) {
                    // columns n0 .. n0+31: 16 (gate, up) pairs -> a[row, n0/2 .. n0/2+15]
                    // (N % 16 == 0 and n0 % 16 == 0: eight columns are all in or all out)
                    float* arow = p.a_out + (int64_t)row * (p.N / 2) + n0 / 2;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (8 * q >= ncol || n0 + 8 * q >= p.N) break;
                        float av[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int j = 8 * q + 2 * i;
                            const float vg = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j]), sxr), sw_s[c + j]);
                            const float vu = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 1]), sxr), sw_s[c + j + 1]);
                            av[i] = __fmul_rn(silu_proj(vg), vu);
                        }
                        *reinterpret_cast<float4*>(arow + 4 * q) = make_float4(av[0], av[1], av[2], av[3]);
                    }
                } else {
                    int32_t* orow = reinterpret_cast<int32_t*>(p.out) + (int64_t)row * p.N;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (v * 4 < ncol && n0 + v * 4 < p.N)
                            *reinterpret_cast<uint4*>(orow + n0 + v * 4) =
                                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                }
            };
            uint32_t ra[32], rb[32];
            int c = 32 * chalf;
            if (c < BN) tmem_ld_32x32b_x32(tq + (uint32_t)c, ra);
            while (c < BN) {
                tc_wait_ld();
                if (c + 64 < BN) tmem_ld_32x32b_x32(tq + (uint32_t)(c + 64), rb);
                chunk(ra, c);
                c += 64;
                if (c >= BN) break;
                tc_wait_ld();
                if (c + 64 < BN) tmem_ld_32x32b_x32(tq + (uint32_t)(c + 64), ra);
                chunk(rb, c);
                c += 64;
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

namespace w8a8 {

// ---------------------------------------------------------------------------
// Group-128 GEMM (a13; the head and trunk formats too) on CTA pairs:
//   p_g      = sum over the 128 k of group g of A[m,k] B[n,k]
//   y        = fma(float(p_g), float(sx[m,g]) * float(sw[n,g]), y), g ascending
//   out[m,n] = bf16_rne(y * post)
// A cluster of two CTAs owns a 256-row x 128-column tile: each CTA loads its
// 128 rows of A and 64 of the tile's 128 rows of B, and holds its 128 rows x
// 128 columns of the accumulator.  Every 128-wide k block is one group and
// gets its own TMEM accumulator (four of 128 columns, rotating), starting
// from zero; the leader's MMA thread hands each one to both CTAs' epilogues,
// which read their 32 columns into registers, release it at once (one
// arrival per warp on the leader's barrier) and promote it: float(p_g) is
// the float bits of p_g + 0x4B400000 less 1.5 * 2^23 (exact for
// |p_g| < 2^22), two columns per f32x2 instruction.  16 epilogue warps a
// CTA (TMEM lane quarter x 32-column quarter, 32 fp32 sums a thread): four
// of them on each scheduler, so that one warp's TMEM and shared-memory
// latencies hide behind the others' arithmetic.  A scale warp stages the group scales of the
// tile's rows and columns in shared memory as fp32, 16 groups at a time in
// two slots, ahead of the epilogue, so that no global load sits between two
// groups of the promotion.  Per SM and k block the pair moves 24 KB of
// operands into shared memory where the one-CTA 128 x 128 tile moves 32 KB.
constexpr int kKernelIdGemmTc2G = 8;
constexpr int kTc2gBN = 128;                      // columns per pair tile
constexpr int kTc2gEpi = 16;                      // epilogue warps
constexpr int kTc2gThreads = 64 + 32 * kTc2gEpi + 32;   // TMA warp, MMA warp, epilogue warps, scale warp
constexpr int kTc2gScaleWarp = 2 + kTc2gEpi;
constexpr int kTc2gAcc = 4;                       // TMEM accumulators of 128 columns
constexpr int kTc2gCG = 16;                       // groups per scale slot
constexpr int kTc2gSRow = 132;                    // fp32 per staged group row (128 + 4: fewer bank conflicts)

struct Tc2gSmem {
    static constexpr int kA = 128 * kTcBK;                 // 16 KB per stage
    static constexpr int kB = (kTc2gBN / 2) * kTcBK;       // 8 KB per stage
    static constexpr int kStages = 7;
    static constexpr int kTiles = kStages * (kA + kB);
    static constexpr int kBars = (2 * kStages + 2 * kTc2gAcc + 1 + 4) * 8;
    static constexpr int kScaleOff = kTiles + (kBars + 16 + 15) / 16 * 16;
    // per slot: column scales [16][132] then row scales [16][132], fp32
    static constexpr int kSlotFloats = 2 * kTc2gCG * kTc2gSRow;
    static constexpr int kBytes = 1024 + kScaleOff + 2 * kSlotFloats * 4;
    static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
};

__global__ void __launch_bounds__(kTc2gThreads, 1)
    gemm_i8_tc2_g128_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            TcParams p) {
    using SM = Tc2gSmem;
    constexpr int kCols = kTc2gAcc * kTc2gBN;   // 512
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + SM::kStages * SM::kA;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kTiles);
    uint64_t* full = bars;                            // leader only
    uint64_t* empty = bars + SM::kStages;              // both
    uint64_t* tfull = empty + SM::kStages;             // both
    uint64_t* tempty = tfull + kTc2gAcc;               // leader only
    uint64_t* sfull = tempty + kTc2gAcc;               // scale slots staged (both)
    uint64_t* sempty = sfull + 2;                      // scale slots consumed (both)
    uint64_t* mma_done = sempty + 2;                   // leader only
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* scales = reinterpret_cast<float*>(smem + SM::kScaleOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SM::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kTc2gAcc; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kTc2gEpi);   // one arrival per epilogue warp of the pair
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sfull[b], 32);       // every lane of the scale warp
            mbar_init(&sempty[b], kTc2gEpi);       // one arrival per epilogue warp of this CTA
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
    const int G = p.num_k_blocks;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, last_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += nclusters) {
                const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
                for (int kb = 0; kb < G; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, (kKernelIdGemmTc2G << 16) | 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (SM::kA + SM::kB));
                    tma_load_2d_pair(sA + stage * SM::kA, &tmA, fb, kb * kTcBK, mt * kTc2BM + (int)rank * 128);
                    tma_load_2d_pair(sB + stage * SM::kB, &tmB, fb, kb * kTcBK,
                                     nt * kTc2gBN + (int)rank * (kTc2gBN / 2));
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
                        mbar_wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, (kKernelIdGemmTc2G << 16) | 2,
                                          100000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kTc2BM, kTc2gBN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += nclusters) {
                for (int kb = 0; kb < G; ++kb) {
                    if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, (kKernelIdGemmTc2G << 16) | 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdGemmTc2G << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kTc2gBN);
                    const uint32_t a0 = smem_u32(sA + stage * SM::kA);
                    const uint32_t b0 = smem_u32(sB + stage * SM::kB);
#pragma unroll
                    for (int kk = 0; kk < kTcBK / 32; ++kk)
                        tc2_mma_i8(d_tmem, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                   kk > 0 ? 1u : 0u);
                    tc2_commit_pair(&empty[stage]);   // frees this stage in both CTAs
                    tc2_commit_pair(&tfull[acc]);     // group product ready in both CTAs
                    if (++stage == SM::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++acc == kTc2gAcc) {
                        acc = 0;
                        acc_phase ^= 1u;
                    }
                }
            }
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(mma_done))
                         : "memory");
            mbar_wait_bounded(mma_done, 0u, nullptr, (kKernelIdGemmTc2G << 16) | 5, 100000000ull);
        }
    } else if (warp == kTc2gScaleWarp) {
        // ------------------------------------------------------------ scale staging (both CTAs)
        // For each tile and each run of up to 16 groups: the column scales of
        // the tile's 128 columns and the row scales of this CTA's 128 rows, as
        // fp32, group-major ([g][col], [g][row]).  Lanes take consecutive
        // groups of one column (one 32-byte run of the [rows, G] scale array).
        int slot = 0;
        uint32_t sphase = 0;
        bool ok = true;
        // 16-byte loads of 16 bf16 scales (8 u8 of the trunk format) where the rows allow them
        const bool vec_ok = (G % 16) == 0 && (reinterpret_cast<uintptr_t>(p.gsx) & 15) == 0 &&
                            (p.gsw_u8 ? (reinterpret_cast<uintptr_t>(p.gsw_u8) & 7) == 0
                                      : (reinterpret_cast<uintptr_t>(p.gsw) & 15) == 0);
        for (int tile = cluster_id; ok && tile < num_tiles; tile += nclusters) {
            const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
            const int row0 = mt * kTc2BM + (int)rank * 128;
            const int col0 = nt * kTc2gBN;
            for (int c0 = 0; c0 < G; c0 += kTc2gCG) {
                const int ng = min(kTc2gCG, G - c0);
                if (!mbar_wait_bounded(&sempty[slot], sphase ^ 1u, abort_flag, (kKernelIdGemmTc2G << 16) | 7)) {
                    ok = false;
                    break;
                }
                float* sw_s = scales + slot * SM::kSlotFloats;
                float* sx_s = sw_s + kTc2gCG * kTc2gSRow;
                // lane l takes the tile columns / CTA rows l, l + 32, l + 64, l + 96;
                // every load of a run is issued before the first store
                if (vec_ok && ng == kTc2gCG) {
                    // 16 bf16 scales of a row or column: two 16-byte loads; two of
                    // the lane's four columns / rows at a time (register budget)
#pragma unroll 1
                    for (int jj = 0; jj < 4; jj += 2) {
                    uint4 wv[2][2], xv[2][2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int col = col0 + lane + 32 * (jj + j), row = row0 + lane + 32 * (jj + j);
                        wv[j][0] = wv[j][1] = xv[j][0] = xv[j][1] = make_uint4(0, 0, 0, 0);
                        if (col < p.N) {
                            if (p.gsw_u8) {
                                const uint2 u = __ldg(reinterpret_cast<const uint2*>(p.gsw_u8 + (int64_t)col * (G / 2) + c0 / 2));
                                wv[j][0] = make_uint4(u.x, u.y, __ldg(p.gsw_row + col), 0);
                            } else {
                                const uint4* src = reinterpret_cast<const uint4*>(p.gsw + (int64_t)col * G + c0);
                                wv[j][0] = __ldg(src);
                                wv[j][1] = __ldg(src + 1);
                            }
                        }
                        if (row < p.M) {
                            const uint4* src = reinterpret_cast<const uint4*>(p.gsx + (int64_t)row * G + c0);
                            xv[j][0] = __ldg(src);
                            xv[j][1] = __ldg(src + 1);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int c = lane + 32 * (jj + j);
#pragma unroll
                        for (int g = 0; g < kTc2gCG; ++g) {
                            const uint4& xq = xv[j][g >> 3];
                            const uint32_t xw = (g & 7) < 2 ? xq.x : (g & 7) < 4 ? xq.y : (g & 7) < 6 ? xq.z : xq.w;
                            sx_s[g * kTc2gSRow + c] = __uint_as_float((g & 1) ? (xw & 0xffff0000u) : (xw << 16));
                            float w;
                            if (p.gsw_u8) {
                                // the u8 of groups g and g ^ 1 (one per 256 of K), times the row's bf16 scale
                                const uint32_t uw = (g >> 1) < 4 ? wv[j][0].x : wv[j][0].y;
                                w = __fmul_rn((float)((uw >> (8 * ((g >> 1) & 3))) & 0xffu),
                                              __uint_as_float(wv[j][0].z << 16));
                            } else {
                                const uint4& wq = wv[j][g >> 3];
                                const uint32_t ww = (g & 7) < 2 ? wq.x : (g & 7) < 4 ? wq.y : (g & 7) < 6 ? wq.z : wq.w;
                                w = __uint_as_float((g & 1) ? (ww & 0xffff0000u) : (ww << 16));
                            }
                            sw_s[g * kTc2gSRow + c] = w;
                        }
                    }
                    }
                } else {
                    for (int g0 = 0; g0 < ng; g0 += 4) {
                        float wv[4][4], xv[4][4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int col = col0 + lane + 32 * j, row = row0 + lane + 32 * j;
#pragma unroll
                            for (int gg = 0; gg < 4; ++gg) {
                                const int g = c0 + g0 + gg;
                                wv[j][gg] = xv[j][gg] = 0.0f;
                                if (g0 + gg < ng && col < p.N) {
                                    if (p.gsw_u8)
                                        wv[j][gg] = __fmul_rn((float)__ldg(p.gsw_u8 + (int64_t)col * (G / 2) + g / 2),
                                                              bf16_bits_to_float(__ldg(p.gsw_row + col)));
                                    else
                                        wv[j][gg] = bf16_bits_to_float(__ldg(p.gsw + (int64_t)col * G + g));
                                }
                                if (g0 + gg < ng && row < p.M)
                                    xv[j][gg] = bf16_bits_to_float(__ldg(p.gsx + (int64_t)row * G + g));
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j)
#pragma unroll
                            for (int gg = 0; gg < 4; ++gg)
                                if (g0 + gg < ng) {
                                    sw_s[(g0 + gg) * kTc2gSRow + lane + 32 * j] = wv[j][gg];
                                    sx_s[(g0 + gg) * kTc2gSRow + lane + 32 * j] = xv[j][gg];
                                }
                    }
                }
                mbar_arrive(&sfull[slot]);   // every lane: its own stores are released
                if (++slot == 2) {
                    slot = 0;
                    sphase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;                 // TMEM lanes [32 q, 32 q + 32)
        const int cq = (warp - 2) >> 2;               // columns [32 cq, 32 cq + 32)
        const int rloc = quarter * 32 + lane;         // this thread's row within the CTA's 128
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
        const uint64_t magic2 = 0x4B4000004B400000ull;
        int acc = 0, slot = 0;
        uint32_t acc_phase = 0, sphase = 0;
        bool ok = true;
        for (int tile = cluster_id; ok && tile < num_tiles; tile += nclusters) {
            const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
            const int row = mt * kTc2BM + (int)rank * 128 + rloc;
            const bool row_ok = row < p.M;
            const int col0 = nt * kTc2gBN + 32 * cq;
            const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(32 * cq);
            uint64_t y2[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) y2[j] = 0ull;
            const float* sw_s = scales;
            const float* sx_s = scales;
            for (int kb = 0; kb < G; ++kb) {
                const int gi = kb % kTc2gCG;
                if (gi == 0) {
                    if (!mbar_wait_bounded(&sfull[slot], sphase, abort_flag, (kKernelIdGemmTc2G << 16) | 8)) {
                        ok = false;
                        break;
                    }
                    sw_s = scales + slot * SM::kSlotFloats + 32 * cq;
                    sx_s = scales + slot * SM::kSlotFloats + kTc2gCG * kTc2gSRow + rloc;
                }
                const float sxg = sx_s[gi * kTc2gSRow];
                if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdGemmTc2G << 16) | 6)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[32];
                tmem_ld_32x32b_x32(tq + (uint32_t)(acc * kTc2gBN), r);
                tc_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(tempty_leader0 + (uint32_t)(acc * 8));   // accumulator free
                if (++acc == kTc2gAcc) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
                const uint64_t sx2 = f2_pack(sxg, sxg);
                const float* swg = sw_s + gi * kTc2gSRow;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 s4 = *reinterpret_cast<const float4*>(swg + 4 * q);
                    const uint64_t sc01 = f2_mul(sx2, f2_pack(s4.x, s4.y));
                    const uint64_t sc23 = f2_mul(sx2, f2_pack(s4.z, s4.w));
                    const uint64_t p01 = f2_sub(f2_pack(__uint_as_float(r[4 * q] + 0x4B400000u),
                                                        __uint_as_float(r[4 * q + 1] + 0x4B400000u)), magic2);
                    const uint64_t p23 = f2_sub(f2_pack(__uint_as_float(r[4 * q + 2] + 0x4B400000u),
                                                        __uint_as_float(r[4 * q + 3] + 0x4B400000u)), magic2);
                    y2[2 * q] = f2_fma(p01, sc01, y2[2 * q]);
                    y2[2 * q + 1] = f2_fma(p23, sc23, y2[2 * q + 1]);
                }
                if (gi == kTc2gCG - 1 || kb == G - 1) {   // this slot's scales are no longer read
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sempty[slot]);
                    if (++slot == 2) {
                        slot = 0;
                        sphase ^= 1u;
                    }
                }
            }
            if (ok && row_ok) {
                uint16_t* yrow = reinterpret_cast<uint16_t*>(p.out) + (int64_t)row * p.N;
                const uint64_t post2 = f2_pack(p.gpost, p.gpost);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int n0 = col0 + v * 8;
                    if (n0 < p.N) {
                        uint32_t pk[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float a, b;
                            f2_unpack(f2_mul(y2[v * 4 + j], post2), a, b);
                            pk[j] = pack_bf16x2(a, b);
                        }
                        *reinterpret_cast<uint4*>(yrow + n0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
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
