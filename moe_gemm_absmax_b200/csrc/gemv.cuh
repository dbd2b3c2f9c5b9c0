// Weight-streaming int8 GEMV for decode-sized batches (a4: a2 + a3 at
// M <= 32 tokens) -- "Online INT8 W8A8 ...", Precision split (int8 weights
// halve the bytes of the bandwidth-bound decode step) and Changes
// (gemm_a8w8 per-token path).
//
// The weight matrix is read exactly once with 16-byte streaming loads; the
// few token rows ride along as the narrow operand of warp-level
// mma.m16n8k32 (weights are the 16-row A operand, tokens the 8-column B
// operand).  Because sum_k a_k b_k is unchanged by any permutation of k
// applied to both operands, each thread feeds the 16 contiguous weight
// bytes it loaded straight into its A fragment, and loads the 16 activation
// bytes of the same k range as its B fragment: no shuffles, no smem.
//
//   lane = 4 g + t  (g = 0..7, t = 0..3); for a 64-byte K chunk at k0:
//     W row (r0 + g)     bytes [k0 + 16t, +16) -> wa = {w0, w1, w2, w3}
//     W row (r0 + g + 8) bytes [k0 + 16t, +16) -> wb = {v0, v1, v2, v3}
//     x row (token g)    bytes [k0 + 16t, +16) -> xb = {x0, x1, x2, x3}
//     mma #1: A = {w0, v0, w1, v1}, B = {x0, x1};  mma #2: A = {w2, v2, w3, v3}, B = {x2, x3}
//   and C = {(r0+g, 2t), (r0+g, 2t+1), (r0+g+8, 2t), (r0+g+8, 2t+1)} (token columns).
//
// A CTA (8 warps) owns WN blocks of 16 weight rows (WN = 4, 2 or 1); WK =
// 8 / WN warps split each block's K range and meet in shared memory.  When
// gridDim.y > 1 the K range
// is also split over CTAs: each writes its int32 partial to the workspace
// and the last CTA to arrive (counter per row block) adds them in order and
// runs the epilogue -- integer sums, so the result is exact and
// deterministic.
#pragma once

#include "common.cuh"

namespace w8a8 {

constexpr int kGemvThreads = 256;
constexpr int kGemvUnroll = 4;

// The A rows a warp multiplies: dense blocks of 16 consecutive rows, or
// (for the MoE gate/up weights) 8 gate/up row pairs arranged so that MMA
// row g is gate row 2(8b + g) and MMA row g + 8 the matching up row.
struct RowMapDense {
    __device__ static int64_t row(int block, int r) { return (int64_t)block * 16 + r; }
};
struct RowMapPairs {
    __device__ static int64_t row(int block, int r) {
        return (int64_t)block * 16 + (r < 8 ? 2 * r : 2 * (r - 8) + 1);
    }
};

struct GemvShape {
    const int8_t* w;      // [rows, K] int8 weights (row stride K)
    const int8_t* x;      // [tokens, K] int8 codes (row stride K)
    int tokens;           // valid token rows (<= 8 * TG)
    int rows;             // weight rows (multiple of 16)
    int K;                // multiple of 16
    int nchunks;          // ceil(K / 64)
    int32_t* part;        // split-K partials [nkseg][row blocks][TG][32][4] (nkseg > 1)
    int* counters;        // arrival counters, one per CTA column, zero on entry (nkseg > 1)
    int trig;             // let the next kernel on the stream launch at once (programmatic launch)
};

// Computes this warp's int32 C fragments over its K range and reduces them
// across the WK warps (and CTAs).  Returns true in the threads that hold
// the final sums for their row block (warps with wk == 0 of the finishing CTA).
// kseg / nkseg: this CTA's share of a K range split over nkseg CTAs;
// ctr: this CTA's arrival counter slot (nkseg > 1).
template <int WN, int WK, int TG, class RowMap, int U = kGemvUnroll, bool PF = false>
__device__ __forceinline__ bool gemv_core(const GemvShape& a, int (&acc)[TG][4], int& block_out, int kseg = 0,
                                          int nkseg = 1, int ctr = 0) {
    static_assert(WN * WK == kGemvThreads / 32, "8 warps");
    __shared__ __align__(16) int red[WK > 1 ? WK - 1 : 1][WN][TG][32][4];   // read and written as int4
    __shared__ int is_last;
    // A kernel launched after this one with programmatic serialization may
    // start now: it waits for this grid's completion before it reads anything
    // (the library's quant kernels, which come next in a decode chain, also
    // hold their own dependents back until that wait returns).
    if (a.trig) asm volatile("griddepcontrol.launch_dependents;");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wn = warp % WN, wk = warp / WN;
    const int g = lane >> 2, t = lane & 3;
    const int block = blockIdx.x * WN + wn;
    block_out = block;
    const bool block_ok = block * 16 < a.rows;

    const int parts = nkseg * WK;
    const int part = kseg * WK + wk;
    const int c0 = (int)((int64_t)a.nchunks * part / parts);
    const int c1 = (int)((int64_t)a.nchunks * (part + 1) / parts);

#pragma unroll
    for (int i = 0; i < TG; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0;

    if (block_ok) {
        const int8_t* wr0 = a.w + RowMap::row(block, g) * a.K + 16 * t;
        const int8_t* wr1 = a.w + RowMap::row(block, g + 8) * a.K + 16 * t;
        uint4 wa[U], wb[U];
        auto load = [&](int c, uint4 (&xa)[U], uint4 (&xb)[U]) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = (c + u) * 64 + 16 * t;
                if (c + u < c1 && k < a.K) {
                    xa[u] = ld_stream_16(wr0 + (int64_t)(c + u) * 64);
                    xb[u] = ld_stream_16(wr1 + (int64_t)(c + u) * 64);
                } else {
                    xa[u] = make_uint4(0, 0, 0, 0);
                    xb[u] = make_uint4(0, 0, 0, 0);
                }
            }
        };
        if (PF) load(c0, wa, wb);
        bool waited = false;
        for (int c = c0; c < c1; c += U) {
            uint4 na[U], nb[U];
            if (PF) {
                // issue the next batch of weight loads before this batch's MMAs
                if (c + U < c1) load(c + U, na, nb);
            } else {
                load(c, wa, wb);
            }
            if (!waited) {
                // weights never depend on the previous kernel; the codes do
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = (c + u) * 64 + 16 * t;
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    const int tok = tg * 8 + g;
                    uint4 xb = make_uint4(0, 0, 0, 0);
                    if (tok < a.tokens && c + u < c1 && k < a.K)
                        xb = __ldca(reinterpret_cast<const uint4*>(a.x + (int64_t)tok * a.K + k));   // L1: shared by the SM's warps
                    const uint32_t A1[4] = {wa[u].x, wb[u].x, wa[u].y, wb[u].y};
                    const uint32_t B1[2] = {xb.x, xb.y};
                    const uint32_t A2[4] = {wa[u].z, wb[u].z, wa[u].w, wb[u].w};
                    const uint32_t B2[2] = {xb.z, xb.w};
                    mma_s8_16832(acc[tg], A1, B1);
                    mma_s8_16832(acc[tg], A2, B2);
                }
            }
            if (PF) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    wa[u] = na[u];
                    wb[u] = nb[u];
                }
            }
        }
        if (!waited) asm volatile("griddepcontrol.wait;" ::: "memory");
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");
    }

    if (WK > 1) {
        if (wk > 0) {
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
                *reinterpret_cast<int4*>(red[wk - 1][wn][tg][lane]) =
                    make_int4(acc[tg][0], acc[tg][1], acc[tg][2], acc[tg][3]);
        }
        __syncthreads();
        if (wk == 0) {
            for (int w = 0; w < WK - 1; ++w)
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    const int4 v = *reinterpret_cast<const int4*>(red[w][wn][tg][lane]);
                    acc[tg][0] += v.x;
                    acc[tg][1] += v.y;
                    acc[tg][2] += v.z;
                    acc[tg][3] += v.w;
                }
        }
    }
    if (nkseg == 1) return wk == 0 && block_ok;

    // ---- split K over CTAs: partials to the workspace, last CTA adds them.
    const int nblocks = (a.rows + 15) / 16;
    if (wk == 0 && block_ok) {
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) {
            int4* dst = reinterpret_cast<int4*>(a.part) +
                        (((int64_t)kseg * nblocks + block) * TG + tg) * 32 + lane;
            *dst = make_int4(acc[tg][0], acc[tg][1], acc[tg][2], acc[tg][3]);
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(a.counters + ctr, 1);
        is_last = (prev == nkseg - 1);
        if (is_last) a.counters[ctr] = 0;   // leave the counter zero for the next call
    }
    __syncthreads();
    if (!is_last) return false;
    __threadfence();
    if (wk == 0 && block_ok) {
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[tg][j] = 0;
        for (int s = 0; s < nkseg; ++s) {
#pragma unroll
            for (int tg = 0; tg < TG; ++tg) {
                const int4 v = __ldcg(reinterpret_cast<const int4*>(a.part) +
                                      (((int64_t)s * nblocks + block) * TG + tg) * 32 + lane);
                acc[tg][0] += v.x;
                acc[tg][1] += v.y;
                acc[tg][2] += v.z;
                acc[tg][3] += v.w;
            }
        }
    }
    return wk == 0 && block_ok;
}

// ---------------------------------------------------------------- dense
struct GemvEpiDense {
    const float* sx;   // [M]
    const float* sw;   // [N]
    void* out;         // bf16 [M,N] or int32 [M,N]
    int M, N;
    int s32;           // 1: raw int32
};

// MINB: resident CTAs per SM the register budget is sized for (4: 64
// registers a thread, 32 warps an SM) -- the decode weight stream needs many
// warps per SM with a few loads each, more than few warps with many loads.
template <int WN, int WK, int TG, int U, int MINB = 1>
__global__ void __launch_bounds__(kGemvThreads, MINB) gemv_dense_kernel(GemvShape a, GemvEpiDense e) {
    int acc[TG][4];
    int block;
    if (!gemv_core<WN, WK, TG, RowMapDense, U>(a, acc, block, blockIdx.y, gridDim.y, blockIdx.x)) return;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = tg * 8 + 2 * t + (j & 1);
            const int n = block * 16 + g + (j >> 1) * 8;
            if (m < e.M && n < e.N) {
                if (e.s32) {
                    reinterpret_cast<int32_t*>(e.out)[(int64_t)m * e.N + n] = acc[tg][j];
                } else {
                    const float v = __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][j]), __ldcg(e.sx + m)), __ldg(e.sw + n));
                    reinterpret_cast<uint16_t*>(e.out)[(int64_t)m * e.N + n] = float_to_bf16_bits(v);
                }
            }
        }
    }
}


// ---------------------------------------------------------------- gated
// The gate_up projection of a dense gated MLP: weight rows 2i (gate) and
// 2i + 1 (up) interleaved; RowMapPairs puts gate row 2(8b + g) in MMA row g
// and its up row in MMA row g + 8 of the same lane, so each thread holds
// (gate, up) of one pair for tokens 2t and 2t + 1:
//   v = (float(acc) * sx[m]) * sw[row];  a[m, i] = SiLU(v_gate) * v_up  (fp32)
struct GemvEpiGated {
    const float* sx;   // [M]
    const float* sw;   // [2I]
    float* a;          // [M, I]
    int M, I;
};

template <int WN, int WK, int TG, int U, int MINB = 1>
__global__ void __launch_bounds__(kGemvThreads, MINB) gemv_gated_kernel(GemvShape a, GemvEpiGated e) {
    int acc[TG][4];
    int block;
    if (!gemv_core<WN, WK, TG, RowMapPairs, U>(a, acc, block, blockIdx.y, gridDim.y, blockIdx.x)) return;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int pair = block * 8 + g;
    if (pair >= e.I) return;
    const float swg = __ldg(e.sw + 2 * pair), swu = __ldg(e.sw + 2 * pair + 1);
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
#pragma unroll
        for (int jt = 0; jt < 2; ++jt) {
            const int m = tg * 8 + 2 * t + jt;
            if (m < e.M) {
                const float sxm = __ldcg(e.sx + m);
                const float vg = __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][jt]), sxm), swg);
                const float vu = __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][2 + jt]), sxm), swu);
                e.a[(int64_t)m * e.I + pair] = __fmul_rn(silu_proj(vg), vu);
            }
        }
    }
}

}  // namespace w8a8


