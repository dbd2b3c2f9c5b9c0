// Routed W8A8 MoE expert layer (a5 .. a11) -- "Online INT8 W8A8 ...",
// Changes: Int8MoEMethod (int8 w13 / w2 with per-channel fp32 scales) and
// the forward routing -> per-token int8 quant -> gemm1 with fused gated SiLU
// via interleaved w13 -> per-token int8 quant -> gemm2 with scatter/combine;
// Precision split: the router gate stays bf16.
//
// Kernels, in launch order:
//   moe_route_kernel        one warp per token: fp32 softmax of the bf16
//                           logits (project exp), top-k by logit with ties to
//                           the lower expert index, weights renormalised
//   moe_plan_kernel         one CTA: expert histogram, exclusive offsets,
//                           list of touched experts, and the row of the
//                           expert-sorted order each (token, slot) lands in
//   moe_quant_scatter_kernel  one CTA per token: per-token int8 quant of x,
//                           codes written once per routed slot into the
//                           expert-sorted code matrix; clears the fp32 output
//   gemm1 (grouped GEMV)    per touched expert: codes x w13^T, dequant,
//                           SiLU(gate) * up -> fp32 intermediate
//   requant                 per-row absmax int8 quant of the intermediate
//   gemm2 (grouped GEMV)    codes x w2^T, dequant, times the routing weight,
//                           fp32 atomic add into the token's output row
//   moe_finalize_kernel     fp32 -> bf16
#pragma once

#include <type_traits>

#include "common.cuh"
#include "gemv.cuh"
#include "quant.cuh"

namespace w8a8 {

constexpr int kMoeMaxExperts = 1024;
constexpr int kMoeMaxTopk = 32;

// ---------------------------------------------------------------------------
// a5: routing.  E <= 32 * EPL; lane l holds experts l, l + 32, ...
template <int EPL>
__global__ void __launch_bounds__(256) moe_route_kernel(const uint16_t* __restrict__ logits, int64_t T, int E,
                                                        int topk, int32_t* __restrict__ ids,
                                                        float* __restrict__ wts) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    float l[EPL], ex[EPL];
    bool taken[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        l[i] = e < E ? bf16_bits_to_float(logits[t * E + e]) : -INFINITY;
        if (isnan(l[i])) l[i] = -INFINITY;   // out of domain; keeps the selection well defined
        taken[i] = e >= E;
        mx = fmaxf(mx, l[i]);
    }
    mx = warp_max(mx);
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        ex[i] = e < E ? exp_proj(__fsub_rn(l[i], mx)) : 0.0f;
        sum = __fadd_rn(sum, ex[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));

    float psel_j = 0.0f;   // lane j keeps the probability of slot j
    int id_j = 0;
    for (int j = 0; j < topk; ++j) {
        // best candidate of this lane: largest logit, then lowest index
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        float bex = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (!taken[i] && (l[i] > bv || (l[i] == bv && e < bi))) {
                bv = l[i];
                bi = e;
                bex = ex[i];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            const float oex = __shfl_xor_sync(0xffffffffu, bex, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
                bex = oex;
            }
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (lane + 32 * i == bi) taken[i] = true;
        if (lane == j) {
            id_j = bi;
            psel_j = __fdiv_rn(bex, sum);
        }
    }
    // renormalise over the k selected, summing in slot order
    float ssel = 0.0f;
    for (int j = 0; j < topk; ++j) ssel = __fadd_rn(ssel, __shfl_sync(0xffffffffu, psel_j, j));
    if (lane < topk) {
        ids[t * topk + lane] = id_j;
        wts[t * topk + lane] = __fdiv_rn(psel_j, ssel);
    }
}

// ---------------------------------------------------------------------------
// a6: plan.  One CTA of 1024 threads.
struct MoePlan {
    int32_t* counts;     // [E]
    int32_t* offsets;    // [E + 1]
    int32_t* active;     // [E] touched experts, ascending
    int32_t* n_active;   // [1]
    int32_t* tile_off;   // [E + 1] prefix sum of ceil(counts / 128): grouped-GEMM row tiles
    int32_t* row_of;     // [T * topk] expert-sorted row of (token, slot)
    int32_t* row_tok;    // [R] token of each sorted row
    int32_t* row_slot;   // [R] slot of each sorted row
    float* row_w;        // [R] routing weight of each sorted row
};

__global__ void __launch_bounds__(1024) moe_plan_kernel(const int32_t* __restrict__ ids,
                                                        const float* __restrict__ wts, int64_t n, int E,
                                                        int topk, MoePlan p) {
    __shared__ int cnt[kMoeMaxExperts];
    __shared__ int off[kMoeMaxExperts];
    __shared__ int warp_tot[32];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    // rank of each entry inside its expert (arrival order; any order is valid)
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int e = ids[i];
        p.row_of[i] = (e >= 0 && e < E) ? atomicAdd(&cnt[e], 1) : 0;   // ids come from moe_route_kernel: always < E
    }
    __syncthreads();
    // exclusive scan of cnt over E <= 1024 (one element per thread)
    const int e = threadIdx.x;
    const int c = e < E ? cnt[e] : 0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;   // exclusive prefix of warp totals
    }
    __syncthreads();
    const int excl = incl - c + warp_tot[warp];
    if (e < E) {
        off[e] = excl;
        p.counts[e] = c;
        p.offsets[e] = excl;
        if (e == E - 1) p.offsets[E] = excl + c;
    }
    // compact list of touched experts: rank among experts with c > 0
    const unsigned ball = __ballot_sync(0xffffffffu, c > 0);
    __syncthreads();
    if (lane == 0) warp_tot[warp] = __popc(ball);
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;
        if (lane == 31) p.n_active[0] = wi;
    }
    __syncthreads();
    if (e < E && c > 0) p.active[warp_tot[warp] + __popc(ball & ((1u << lane) - 1u))] = e;
    // exclusive scan of the 128-row tiles of each expert
    const int mt = (c + 127) / 128;
    int tincl = mt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, tincl, o);
        if (lane >= o) tincl += v;
    }
    __syncthreads();
    if (lane == 31) warp_tot[warp] = tincl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;
    }
    __syncthreads();
    if (e < E) {
        const int texcl = tincl - mt + warp_tot[warp];
        p.tile_off[e] = texcl;
        if (e == E - 1) p.tile_off[E] = texcl + mt;
    }
    // final rows and the per-row metadata of the sorted order
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int r = off[ids[i]] + p.row_of[i];
        p.row_of[i] = r;
        p.row_tok[r] = (int)(i / topk);
        p.row_slot[r] = (int)(i % topk);
        p.row_w[r] = wts[i];
    }
}

// ---------------------------------------------------------------------------
// a7: per-token quant of x, scattered to the token's sorted rows.  One CTA per
// token with one 16-byte vector (8 bf16) per thread; blockDim is H/8 rounded
// up to a whole number of warps (H <= 8 * 1024).
__global__ void __launch_bounds__(1024) moe_quant_scatter_kernel(const uint16_t* __restrict__ x, int H, int topk,
                                                                 const int32_t* __restrict__ row_of,
                                                                 int8_t* __restrict__ xq, float* __restrict__ sxr,
                                                                 float* __restrict__ out_f32,
                                                                 int8_t* __restrict__ dbg_qx,
                                                                 float* __restrict__ dbg_sx) {
    const int64_t t = blockIdx.x;
    const int v = threadIdx.x;          // vector index, 8 bf16
    const bool active = v < H / 8;
    float f[8];
    if (active) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + t * H) + v);
        VecTraits<uint16_t>::unpack(raw, f);
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    __shared__ float red[32];
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x < 32) {
        float m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        m = warp_max(m);
        if (threadIdx.x == 0) red[0] = m;
    }
    __syncthreads();
    const float s = __fdiv_rn(red[0], 127.0f);
    if (!active) return;
    uint32_t pk[2] = {0u, 0u};
    if (s != 0.0f) {
#pragma unroll
        for (int j = 0; j < 8; ++j) pk[j >> 2] |= (uint32_t)(uint8_t)(int8_t)quant_code(f[j], s) << (8 * (j & 3));
    }
    const uint2 codes = make_uint2(pk[0], pk[1]);
    for (int j = 0; j < topk; ++j) {
        const int r = row_of[t * topk + j];
        *reinterpret_cast<uint2*>(xq + (int64_t)r * H + v * 8) = codes;
        if (threadIdx.x == 0) sxr[r] = s;
    }
    if (dbg_qx) *reinterpret_cast<uint2*>(dbg_qx + t * H + v * 8) = codes;
    if (dbg_sx && threadIdx.x == 0) dbg_sx[t] = s;
    // clear this token's fp32 output row for the gemm2 combine
    float4* o = reinterpret_cast<float4*>(out_f32 + t * H) + 2 * v;
    o[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    o[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// a8 / a10: grouped GEMV over the touched experts.  blockIdx.y indexes the
// touched-expert list (CTAs past n_active return at once); each CTA walks its
// expert's rows in groups of 8 * TG tokens.
struct MoeGemmArgs {
    const int8_t* w;          // [E, rows, K]
    const float* sw;          // [E, rows]
    const int8_t* xq;         // [R, K] expert-sorted codes
    const float* sxr;         // [R] scale of each sorted row
    const int32_t* counts;    // [E]
    const int32_t* offsets;   // [E + 1]
    const int32_t* active;    // [E]
    const int32_t* n_active;  // [1]
    int rows, K;
    // gemm1: gated intermediate a [R, rows / 2] fp32
    float* a_out;
    // gemm2: combine into out_f32 [T, rows]
    const int32_t* row_tok;
    const float* row_w;
    float* out_f32;
};

template <int WN, int WK, int TG, bool GATED>
__global__ void __launch_bounds__(kGemvThreads) moe_gemm_kernel(MoeGemmArgs m) {
    if ((int)blockIdx.y >= __ldg(m.n_active)) return;
    const int e = __ldg(m.active + blockIdx.y);
    const int cnt = __ldg(m.counts + e);
    const int off = __ldg(m.offsets + e);
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    GemvShape a;
    a.w = m.w + (int64_t)e * m.rows * m.K;
    a.rows = m.rows;
    a.K = m.K;
    a.nchunks = (m.K + 63) / 64;
    a.part = nullptr;
    a.counters = nullptr;
    const float* swe = m.sw + (int64_t)e * m.rows;
    for (int tok0 = 0; tok0 < cnt; tok0 += 8 * TG) {
        a.x = m.xq + (int64_t)(off + tok0) * m.K;
        a.tokens = min(cnt - tok0, 8 * TG);
        int acc[TG][4];
        int block;
        const bool have = gemv_core<WN, WK, TG, typename std::conditional<GATED, RowMapPairs, RowMapDense>::type>(
            a, acc, block);
        if (have) {
#pragma unroll
            for (int tg = 0; tg < TG; ++tg) {
#pragma unroll
                for (int jt = 0; jt < 2; ++jt) {           // token column 2t + jt
                    const int mloc = tg * 8 + 2 * t + jt;
                    if (mloc >= a.tokens) continue;
                    const int r = off + tok0 + mloc;
                    const float sx = __ldg(m.sxr + r);
                    if (GATED) {
                        const int pair = block * 8 + g;
                        const float vg = __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][jt]), sx), __ldg(swe + 2 * pair));
                        const float vu =
                            __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][2 + jt]), sx), __ldg(swe + 2 * pair + 1));
                        m.a_out[(int64_t)r * (m.rows / 2) + pair] = __fmul_rn(silu_proj(vg), vu);
                    } else {
                        const float wr = __ldg(m.row_w + r);
                        float* orow = m.out_f32 + (int64_t)__ldg(m.row_tok + r) * m.rows;
#pragma unroll
                        for (int jr = 0; jr < 2; ++jr) {   // weight row g + 8 jr
                            const int n = block * 16 + g + 8 * jr;
                            const float y2 =
                                __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][2 * jr + jt]), sx), __ldg(swe + n));
                            atomicAdd(orow + n, __fmul_rn(wr, y2));
                        }
                    }
                }
            }
        }
        __syncthreads();   // the reduction scratch of gemv_core is reused by the next group
    }
}

// ---------------------------------------------------------------------------
// a11 tail: fp32 combine buffer -> bf16 output; optional debug gathers.
__global__ void moe_finalize_kernel(const float* __restrict__ out_f32, uint16_t* __restrict__ y, int64_t n) {
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i + 3 < n) {
        const float4 v = *reinterpret_cast<const float4*>(out_f32 + i);
        *reinterpret_cast<uint2*>(y + i) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    } else {
        for (int64_t j = i; j < n; ++j) y[j] = float_to_bf16_bits(out_f32[j]);
    }
}

__global__ void moe_debug_gather_kernel(const int8_t* __restrict__ qa, const float* __restrict__ sa,
                                        const int32_t* __restrict__ row_of, int64_t n, int I,
                                        int8_t* __restrict__ dqa, float* __restrict__ dsa) {
    const int64_t i = blockIdx.x;   // (token, slot) entry
    if (i >= n) return;
    const int r = row_of[i];
    for (int k = threadIdx.x; k < I; k += blockDim.x)
        if (dqa) dqa[i * I + k] = qa[(int64_t)r * I + k];
    if (threadIdx.x == 0 && dsa) dsa[i] = sa[r];
}

}  // namespace w8a8
