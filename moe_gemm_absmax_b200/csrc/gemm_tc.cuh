// int8 x int8 -> int32 GEMMs on the 5th-generation tensor cores.
//
// (a2 + a3) dense W8A8 -- "Online INT8 W8A8 ...", Changes (gemm_a8w8
// per-token path); "Qwen3.6-27B-Quark-W8A8-INT8", Quantization Details:
//   acc[m,n] = sum_k A[m,k] B[n,k]                      A = codes [M,K], B = weights [N,K]
//   y[m,n]   = bf16_rne( (float(acc) * sx[m]) * sw[n] )  (or the raw int32 acc)
// (a13) group-128 scaled, rotated domain -- "Qwen3.6-35B-A3B IQ8R - radiance
// container", file table (one bf16 scale for each row and 128-wide slice of K):
//   p_g      = sum over the 128 k of group g of A[m,k] B[n,k]   (one TMEM tile per g)
//   acc      = fma(float(p_g), float(sx[m,g]) * float(sw[n,g]), acc), g ascending
//   y[m,n]   = bf16_rne(acc * (1/128))
//
// Persistent, warp-specialised CTA (one per SM, 192 threads):
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles of A (128 x 128)
//               and B (BN x 128) into a STAGES-deep shared-memory ring;
//   warp 1      TMEM allocator and single-thread tcgen05.mma.kind::i8 issuer
//               (M=128, N=BN, K=32 per instruction) into NACC rotating TMEM
//               accumulators, so the epilogue overlaps the next MMAs;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane TMEM quarter, dequant
//               (or per-group promotion), bf16 pack, 16-byte global stores.
// A dense tile hands its accumulator to the epilogue once, after the whole
// K loop; a group-128 tile hands over one accumulator per 128-wide k block.
// Every wait is bounded (mbar_wait_bounded); a CTA that gives up drains its
// own copies and MMAs, frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace w8a8 {

constexpr int kTcBM = 128;
constexpr int kTcBK = 128;          // int8 elements (= bytes) of K per stage: one swizzle atom
constexpr int kKernelIdGemmTc = 1;

// Epilogues: dense bf16, raw int32, group-128 promotion, and the two grouped
// MoE epilogues (gated SiLU over interleaved gate/up columns; the routing-
// weighted output of each sorted row, stored at its (token, slot)).
enum TcEpilogue : int {
    kEpiBf16 = 0,
    kEpiS32 = 1,
    kEpiG128 = 2,
    kEpiMoeGated = 3,
    kEpiMoeCombine = 4,        // w * y2 stored at (token, slot)
    kEpiMoeCombineAtomic = 5   // w * y2 added atomically into the token's row
};

struct TcParams {
    int M, N, K;
    int num_m_tiles, num_n_tiles, num_k_blocks;
    const float* sx;        // [M]        (kEpiBf16; grouped: scale of each sorted row)
    const float* sw;        // [N]        (kEpiBf16; grouped: [E, N] per-expert channel scales)
    const uint16_t* gsx;    // [M, G] bf16 (kEpiG128)
    const uint16_t* gsw;    // [N, G] bf16 (kEpiG128)
    float gpost;            // kEpiG128: final factor (1/128 in the rotated domain, 1 unrotated)
    const uint8_t* gsw_u8;  // kEpiG128, two-level trunk format: [N, G / 2] u8 ...
    const uint16_t* gsw_row;// ... times a bf16 row scale [N] (gsw unused)
    void* out;              // bf16 or int32 [M, N], row stride N
    // ---- grouped (MoE) mode: A = expert-sorted rows, B = per-expert weights [E * N, K]
    const int32_t* counts;  // [E] rows of each expert
    const int32_t* offsets; // [E + 1] first sorted row of each expert
    const int32_t* tile_off;// [E + 1] prefix sum of ceil(counts / 128)
    int E;
    float* a_out;           // kEpiMoeGated: fp32 [M, N / 2]
    const int32_t* row_tok; // kEpiMoeCombine: token of each sorted row
    const int32_t* row_slot;// kEpiMoeCombine: slot of each sorted row
    const float* row_w;     // kEpiMoeCombine: routing weight of each sorted row
    float* contrib;         // kEpiMoeCombine: fp32 [T * topk, N], row (token * topk + slot);
                            // kEpiMoeCombineAtomic: fp32 [T, N]
    int topk;
};

// Coordinates of one output tile.
struct TcTile {
    int a_row;      // first A row (TMA y coordinate)
    int b_row;      // first B row
    int valid;      // rows of the tile that belong to it (<= 128)
    int n0;         // first output column within the expert (or the matrix)
    int e;          // expert (grouped) / 0
};

template <bool GROUPED, int BN>
__device__ __forceinline__ TcTile tc_tile(const TcParams& p, int tile) {
    TcTile t;
    if (!GROUPED) {
        const int mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
        t.a_row = mt * kTcBM;
        t.b_row = nt * BN;
        t.valid = min(kTcBM, p.M - t.a_row);
        t.n0 = nt * BN;
        t.e = 0;
    } else {
        const int gm = tile / p.num_n_tiles, nt = tile % p.num_n_tiles;
        int lo = 0, hi = p.E - 1;          // expert e with tile_off[e] <= gm < tile_off[e + 1]
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(p.tile_off + mid) <= gm) lo = mid;
            else hi = mid - 1;
        }
        const int lm = gm - __ldg(p.tile_off + lo);
        t.e = lo;
        t.a_row = __ldg(p.offsets + lo) + lm * kTcBM;
        t.valid = min(kTcBM, __ldg(p.counts + lo) - lm * kTcBM);
        t.n0 = nt * BN;
        t.b_row = lo * p.N + nt * BN;
    }
    return t;
}

template <int BN, int STAGES>
struct TcSmem {
    static constexpr int kA = kTcBM * kTcBK;                 // bytes per A stage
    static constexpr int kB = BN * kTcBK;                    // bytes per B stage
    static constexpr int kTiles = STAGES * (kA + kB);
    static constexpr int kBars = (2 * STAGES + 2 * 4 + 1) * 8;
    // epilogue scratch: the group-128 column scales (8 warps x 64 fp32), or
    // each epilogue warp's copy of the tile's BN column scales
    static constexpr int kEpiOff = kTiles + (kBars + 16 + 15) / 16 * 16;
    static constexpr int kEpiBytes = 8 * (BN > 64 ? BN : 64) * 4;
    static constexpr int kBytes = 1024 /*alignment slack*/ + kEpiOff + kEpiBytes;
};

// NEPI epilogue warps: 4 (one per TMEM lane quarter) or 8 (two per quarter,
// each taking every other 32-column chunk) for epilogue-heavy tiles.
template <int NEPI>
constexpr int tc_threads() { return 64 + 32 * NEPI; }

template <int BN, int STAGES, int EPI, int NACC, bool GROUPED = false, int NEPI = 4>
__global__ void __launch_bounds__(tc_threads<NEPI>(), 1)
    gemm_i8_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcParams p) {
    static_assert(NEPI == 4 || NEPI == 8, "epilogue warps");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
    static_assert(NACC >= 2 && NACC <= 4, "NACC");
    constexpr int kCols = NACC * BN;
    static_assert(kCols == 64 || kCols == 128 || kCols == 256 || kCols == 512, "TMEM columns: power of two");
    static_assert(EPI != kEpiG128 || BN * 4 / NEPI <= 128, "group-128 epilogue keeps its columns' fp32 sums");
    using SM = TcSmem<BN, STAGES>;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * SM::kA;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kTiles);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 4;
    uint64_t* mma_done = tempty + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* epi_scratch = reinterpret_cast<float*>(smem + SM::kEpiOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 32 * NEPI);
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
        tmem_alloc(tmem_slot, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles =
        GROUPED ? __ldg(p.tile_off + p.E) * p.num_n_tiles : p.num_m_tiles * p.num_n_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;          // bit s: stage s was loaded at least once
            uint32_t last_phase = 0;      // bit s: phase of the last load into stage s
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const TcTile ti = tc_tile<GROUPED, BN>(p, tile);
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, (kKernelIdGemmTc << 16) | 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)(SM::kA + SM::kB));
                    tma_load_2d(sA + stage * SM::kA, &tmA, &full[stage], kb * kTcBK, ti.a_row);
                    tma_load_2d(sB + stage * SM::kB, &tmB, &full[stage], kb * kTcBK, ti.b_row);
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
                        mbar_wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, (kKernelIdGemmTc << 16) | 2,
                                          100000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kTcBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    const bool new_acc = (EPI == kEpiG128) || kb == 0;
                    if (new_acc) {
                        // group-128: the epilogue refills each buffer with the
                        // conversion bias and releases it once more at the start,
                        // so its first use waits for phase 0 as well
                        const uint32_t par = EPI == kEpiG128 ? acc_phase : (acc_phase ^ 1u);
                        if (!mbar_wait_bounded(&tempty[acc], par, abort_flag, (kKernelIdGemmTc << 16) | 3)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, (kKernelIdGemmTc << 16) | 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                    const uint32_t a0 = smem_u32(sA + stage * SM::kA);
                    const uint32_t b0 = smem_u32(sB + stage * SM::kB);
#pragma unroll
                    for (int kk = 0; kk < kTcBK / 32; ++kk) {
                        const bool accumulate = EPI == kEpiG128 || kk > 0 || kb > 0;
                        tc_mma_i8(d_tmem, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                  accumulate ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);       // frees the smem stage when these MMAs finish
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    const bool hand_over = (EPI == kEpiG128) || kb == p.num_k_blocks - 1;
                    if (hand_over) {
                        tc_commit(&tfull[acc]);     // accumulator ready for the epilogue
                        if (++acc == NACC) {
                            acc = 0;
                            acc_phase ^= 1u;
                        }
                    }
                }
            }
            // all MMAs issued by this thread complete before TMEM is released
            tc_commit(mma_done);
            mbar_wait_bounded(mma_done, 0u, nullptr, (kKernelIdGemmTc << 16) | 5, 100000000ull);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                 // TMEM lanes [32 q, 32 q + 32)
        const int chalf = (warp - 2) / 4;             // NEPI == 8: which alternate 32-column chunks
        const int row_in_tile = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        if constexpr (EPI == kEpiG128) {
            // every accumulator buffer starts from the conversion bias
            constexpr int kStep = NEPI == 8 ? 64 : 32;
            const uint32_t tq0 = tmem_base + ((uint32_t)(quarter * 32) << 16);
            for (int b = 0; b < NACC; ++b)
                for (int c = (NEPI == 8 ? 32 * chalf : 0); c < BN; c += kStep)
                    tmem_st_32x32b_x32_fill(tq0 + (uint32_t)(b * BN + c), 0x4B400000u);
            tc_wait_st();
            tc_fence_before();
            for (int b = 0; b < NACC; ++b) mbar_arrive(&tempty[b]);
        }
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            const TcTile ti = tc_tile<GROUPED, BN>(p, tile);
            const int nt = ti.n0 / BN;
            const int row = ti.a_row + row_in_tile;
            const bool row_ok = row_in_tile < ti.valid;
            const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16);
            if constexpr (EPI == kEpiG128) {
                // y[row, col] = sum over groups g ascending of
                //   fma(float(p_g), sx[row, g] * sw[col, g], y)   (fp32), then * 1/128.
                // Two columns per instruction (f32x2).  Each accumulator buffer
                // starts from the bias 0x4B400000 (the bits of 1.5 * 2^23)
                // instead of zero, so it ends holding the float bits of
                // 1.5 * 2^23 + p_g exactly (|p_g| <= 127^2 * 128 < 2^22) and
                // float(p_g) is one subtraction.  The 32 column scales of a chunk
                // go through this warp's shared scratch, read back as 4-wide
                // broadcasts.
                constexpr int kStep = NEPI == 8 ? 64 : 32;   // column distance between this warp's chunks
                constexpr int kChunks = BN / kStep;
                const int c0 = NEPI == 8 ? 32 * chalf : 0;
                const int G = p.num_k_blocks;
                const uint64_t magic2 = 0x4B4000004B400000ull;
                float* wsc = epi_scratch + (warp - 2) * 64;
                // column scale of group g: bf16, or (trunk format) u8 per 256 of K times a bf16 row scale
                auto col_scale = [&](int col, int g) -> float {
                    if (col >= p.N) return 0.0f;
                    if (p.gsw_u8)
                        return __fmul_rn((float)__ldg(p.gsw_u8 + (int64_t)col * (G / 2) + g / 2),
                                         bf16_bits_to_float(__ldg(p.gsw_row + col)));
                    return bf16_bits_to_float(__ldg(p.gsw + (int64_t)col * G + g));
                };
                uint64_t y2[kChunks * 16];
#pragma unroll
                for (int j = 0; j < kChunks * 16; ++j) y2[j] = 0ull;
                float sx_next = row_ok ? bf16_bits_to_float(__ldg(p.gsx + (int64_t)row * G)) : 0.0f;
                float sw_next[kChunks];
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    const int col = nt * BN + c0 + i * kStep + lane;
                    sw_next[i] = col_scale(col, 0);
                }
                for (int kb = 0; kb < G; ++kb) {
                    const float sxg = sx_next;
                    __syncwarp();   // the previous group's broadcast reads are done
#pragma unroll
                    for (int i = 0; i < kChunks; ++i) wsc[i * 32 + lane] = sw_next[i];
                    __syncwarp();
                    if (kb + 1 < G) {   // next group's scales, in flight during this group
                        sx_next = row_ok ? bf16_bits_to_float(__ldg(p.gsx + (int64_t)row * G + kb + 1)) : 0.0f;
#pragma unroll
                        for (int i = 0; i < kChunks; ++i) {
                            const int col = nt * BN + c0 + i * kStep + lane;
                            sw_next[i] = col_scale(col, kb + 1);
                        }
                    }
                    if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdGemmTc << 16) | 6)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // chunk by chunk: into registers, the bias back into TMEM, the
                    // promotion; the buffer goes back to the MMA after the last chunk
                    const uint64_t sx2 = f2_pack(sxg, sxg);
#pragma unroll
                    for (int i = 0; i < kChunks; ++i) {
                        const uint32_t ta = tq + (uint32_t)(acc * BN + c0 + i * kStep);
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(ta, r);
                        tc_wait_ld();
                        tmem_st_32x32b_x32_fill(ta, 0x4B400000u);
                        if (i == kChunks - 1) {
                            tc_wait_st();
                            tc_fence_before();
                            mbar_arrive(&tempty[acc]);
                        }
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 s4 = *reinterpret_cast<const float4*>(wsc + i * 32 + 4 * q);
                            const uint64_t sc01 = f2_mul(sx2, f2_pack(s4.x, s4.y));
                            const uint64_t sc23 = f2_mul(sx2, f2_pack(s4.z, s4.w));
                            const uint64_t p01 =
                                f2_sub(f2_pack(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])), magic2);
                            const uint64_t p23 =
                                f2_sub(f2_pack(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])), magic2);
                            y2[i * 16 + 2 * q] = f2_fma(p01, sc01, y2[i * 16 + 2 * q]);
                            y2[i * 16 + 2 * q + 1] = f2_fma(p23, sc23, y2[i * 16 + 2 * q + 1]);
                        }
                    }
                    if (++acc == NACC) {
                        acc = 0;
                        acc_phase ^= 1u;
                    }
                }
                if (ok && row_ok) {
                    uint16_t* yrow = reinterpret_cast<uint16_t*>(p.out) + (int64_t)row * p.N;
                    const uint64_t inv2 = f2_pack(p.gpost, p.gpost);
#pragma unroll
                    for (int i = 0; i < kChunks; ++i) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int n0 = nt * BN + c0 + i * kStep + v * 8;
                            if (n0 < p.N) {
                                uint32_t pk[4];
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    float a, b;
                                    f2_unpack(f2_mul(y2[i * 16 + v * 4 + j], inv2), a, b);
                                    pk[j] = pack_bf16x2(a, b);
                                }
                                *reinterpret_cast<uint4*>(yrow + n0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            }
                        }
                    }
                }
            } else {
                // the tile's column scales (per expert in the grouped modes) into this
                // warp's shared scratch, before the wait: N % 8 == 0, so a 4-column
                // vector is all in or all out
                constexpr bool kSw = EPI == kEpiBf16 || EPI == kEpiMoeGated || EPI == kEpiMoeCombine ||
                                     EPI == kEpiMoeCombineAtomic;
                float* sw_s = epi_scratch + (warp - 2) * BN;
                if (kSw) {
                    __syncwarp();   // the previous tile's reads are done
                    const float* swt = p.sw + (int64_t)ti.e * p.N;
                    for (int v = lane; v < BN / 4; v += 32) {
                        const int n = ti.n0 + 4 * v;
                        float4 sv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        if (n < p.N) sv = __ldg(reinterpret_cast<const float4*>(swt + n));
                        *reinterpret_cast<float4*>(sw_s + 4 * v) = sv;
                    }
                    __syncwarp();
                }
                if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, (kKernelIdGemmTc << 16) | 6)) break;
                tc_fence_after();
                float sxr = 0.0f;
                if ((EPI == kEpiBf16 || EPI == kEpiMoeGated || EPI == kEpiMoeCombine || EPI == kEpiMoeCombineAtomic) &&
                    row_ok)
                    sxr = __ldg(p.sx + row);
                int64_t orow_i = 0;
                float wr = 0.0f;
                if ((EPI == kEpiMoeCombine || EPI == kEpiMoeCombineAtomic) && row_ok) {
                    orow_i = EPI == kEpiMoeCombine ? (int64_t)__ldg(p.row_tok + row) * p.topk + __ldg(p.row_slot + row)
                                                   : (int64_t)__ldg(p.row_tok + row);
                    wr = __ldg(p.row_w + row);
                }
                // one 32-column chunk (the next one's TMEM load is in flight)
                auto chunk = [&](const uint32_t (&r)[32], int c) {
                    const int n0 = nt * BN + c;
                    if (!row_ok || n0 >= p.N) return;
                    if (EPI == kEpiMoeGated) {
                        // columns n0 .. n0+31 of expert e: 16 (gate, up) pairs
                        float* arow = p.a_out + (int64_t)row * (p.N / 2) + n0 / 2;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float av[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int j = 8 * q + 2 * i;
                                const float vg = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j]), sxr), sw_s[c + j]);
                                const float vu =
                                    __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 1]), sxr), sw_s[c + j + 1]);
                                av[i] = __fmul_rn(silu_proj(vg), vu);
                            }
                            *reinterpret_cast<float4*>(arow + 4 * q) = make_float4(av[0], av[1], av[2], av[3]);
                        }
                    } else if (EPI == kEpiMoeCombine || EPI == kEpiMoeCombineAtomic) {
                        float* orow = p.contrib + orow_i * p.N + n0;
                        const uint64_t sx2 = f2_pack(sxr, sxr), w2v = f2_pack(wr, wr);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 s4 = *reinterpret_cast<const float4*>(sw_s + c + 4 * q);
                            const uint64_t a01 = f2_pack(__int2float_rn((int)r[4 * q]), __int2float_rn((int)r[4 * q + 1]));
                            const uint64_t a23 =
                                f2_pack(__int2float_rn((int)r[4 * q + 2]), __int2float_rn((int)r[4 * q + 3]));
                            float c0, c1, c2, c3;
                            f2_unpack(f2_mul(w2v, f2_mul(f2_mul(a01, sx2), f2_pack(s4.x, s4.y))), c0, c1);
                            f2_unpack(f2_mul(w2v, f2_mul(f2_mul(a23, sx2), f2_pack(s4.z, s4.w))), c2, c3);
                            if constexpr (EPI == kEpiMoeCombine)
                                __stcs(reinterpret_cast<float4*>(orow + 4 * q), make_float4(c0, c1, c2, c3));
                            else
                                red_add_v4(orow + 4 * q, c0, c1, c2, c3);
                        }
                    } else if (EPI == kEpiBf16) {
                        uint16_t* yrow = reinterpret_cast<uint16_t*>(p.out) + (int64_t)row * p.N;
                        const uint64_t sx2 = f2_pack(sxr, sxr);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {           // 8 columns per 16-byte store
                            if (n0 + v * 8 < p.N) {
                                uint32_t pk[4];
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const uint64_t a2 = f2_pack(__int2float_rn((int)r[v * 8 + 2 * j]),
                                                                __int2float_rn((int)r[v * 8 + 2 * j + 1]));
                                    float lo, hi;
                                    f2_unpack(f2_mul(f2_mul(a2, sx2), f2_pack(sw_s[c + v * 8 + 2 * j],
                                                                              sw_s[c + v * 8 + 2 * j + 1])),
                                              lo, hi);
                                    pk[j] = pack_bf16x2(lo, hi);
                                }
                                *reinterpret_cast<uint4*>(yrow + n0 + v * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            }
                        }
                    } else {
                        int32_t* orow = reinterpret_cast<int32_t*>(p.out) + (int64_t)row * p.N;
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            if (n0 + v * 4 < p.N)
                                *reinterpret_cast<uint4*>(orow + n0 + v * 4) =
                                    make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                        }
                    }
                };
                constexpr int kStep = NEPI == 8 ? 64 : 32;
                uint32_t ra[32], rb[32];
                int c = NEPI == 8 ? 32 * chalf : 0;
                const uint32_t tqa = tq + (uint32_t)(acc * BN);
                if (c < BN) tmem_ld_32x32b_x32(tqa + (uint32_t)c, ra);
                while (c < BN) {
                    tc_wait_ld();
                    if (c + kStep < BN) tmem_ld_32x32b_x32(tqa + (uint32_t)(c + kStep), rb);
                    chunk(ra, c);
                    c += kStep;
                    if (c >= BN) break;
                    tc_wait_ld();
                    if (c + kStep < BN) tmem_ld_32x32b_x32(tqa + (uint32_t)(c + kStep), ra);
                    chunk(rb, c);
                    c += kStep;
                }
                tc_fence_before();
                mbar_arrive(&tempty[acc]);
                if (++acc == NACC) {
                    acc = 0;
                    acc_phase ^= 1u;
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
