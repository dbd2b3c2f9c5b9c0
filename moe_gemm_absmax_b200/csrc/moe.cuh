// Routed W8A8 MoE expert layer (a5 .. a11) -- "Online INT8 W8A8 ...",
// Changes: Int8MoEMethod (int8 w13 / w2 with per-channel fp32 scales) and
// the forward routing -> per-token int8 quant -> gemm1 with fused gated SiLU
// via interleaved w13 -> per-token int8 quant -> gemm2 with scatter/combine;
// Precision split: the router gate stays bf16.
//
// Kernels, in launch order:
//   moe_route_plan_kernel   one warp per token: fp32 softmax of the bf16
//                           logits (project exp), top-k by logit with ties to
//                           the lower expert index, weights renormalised, rank
//                           of each (token, slot) inside its expert; the last
//                           CTA scans the histogram (offsets, tile offsets,
//                           touched experts)
//   moe_quant_scatter_kernel  one CTA per token: per-token int8 quant of x,
//                           codes written once per routed slot into the
//                           expert-sorted code matrix; row metadata; clears
//                           the token's fp32 output row
//   gemm1 (grouped GEMV)    per touched expert: codes x w13^T, dequant,
//                           SiLU(gate) * up -> fp32 intermediate
//   requant                 per-row absmax int8 quant of the intermediate
//   gemm2 (grouped)         codes x w2^T, dequant, times the routing weight,
//                           stored at (token, slot)
//   moe_finalize_kernel     sum of each token's k contributions in slot order,
//                           fp32, then bf16
#pragma once

#include <type_traits>

#include "common.cuh"
#include "gemv.cuh"
#include "quant.cuh"

namespace w8a8 {

constexpr int kMoeMaxExperts = 1024;
constexpr int kMoeMaxTopk = 32;

// ---------------------------------------------------------------------------
// a5 + a6: routing and the expert plan, one warp per token.
//   routing: lane l holds experts l, l + 32, ... (E <= 32 * EPL); fp32 softmax
//   with the project exponential, top-k by logit (ties to the lower expert
//   index), weights renormalised over the k in slot order;
//   plan: each selected (token, slot) takes its rank inside its expert from a
//   global atomic counter (any order is a valid expert-sorted order); the last
//   CTA to finish scans the counts into offsets, the 128-row tile offsets of
//   the grouped GEMMs and the list of touched experts.
// counts[E] and *done must be zero on entry.
struct MoePlan {
    int32_t* counts;     // [E]
    int32_t* offsets;    // [E + 1]
    int32_t* active;     // [E] touched experts, ascending
    int32_t* n_active;   // [1]
    int32_t* tile_off;   // [E + 1] prefix sum of ceil(counts / tile_rows): grouped-GEMM row tiles
    int32_t* rank;       // [T * topk] rank of (token, slot) inside its expert
    int32_t* done;       // [1] finished CTAs
    int tile_rows;       // rows per tile of the grouped GEMMs that follow
};

// Total order of bf16 logits as unsigned 16-bit keys (NaN taken as -inf,
// -0 as +0, so equal values get equal keys).
__device__ __forceinline__ uint32_t logit_key16(uint16_t b) {
    if ((b & 0x7fffu) > 0x7f80u) b = 0xff80u;   // NaN -> -inf
    if (b == 0x8000u) b = 0u;                   // -0 -> +0
    return (b & 0x8000u) ? (~(uint32_t)b & 0xffffu) : ((uint32_t)b | 0x8000u);
}

// a5 for one token, by one warp: lane l holds experts l, l + 32, ...
// (E <= 32 * EPL).  p = softmax(l) in fp32 with the project exponential and
// the denominator summed in expert-index order (staged in ex_s, this warp's
// 32 * EPL floats of shared memory, one lane folds them); top-k by logit,
// ties to the lower expert index: each expert's key is (ordered logit << 16)
// | (0xffff - e), so the largest key is the largest logit with the smallest
// index, and one warp max-reduction picks each slot.  Lane j < topk returns
// slot j's expert and its weight p_j / sum over the k of p (slot order).
template <int EPL>
__device__ __forceinline__ void route_token(const uint16_t* __restrict__ lrow, int E, int topk, float* ex_s,
                                            int& id_j, float& w_j) {
    const int lane = threadIdx.x & 31;
    float l[EPL];
    uint32_t key[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            const uint16_t b = __ldg(lrow + e);
            l[i] = bf16_bits_to_float(b);
            if (isnan(l[i])) l[i] = -INFINITY;   // out of domain; keeps the selection well defined
            key[i] = (logit_key16(b) << 16) | (0xffffu - (uint32_t)e);
        } else {
            l[i] = -INFINITY;
            key[i] = 0u;
        }
        mx = fmaxf(mx, l[i]);
    }
    mx = warp_max(mx);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        ex_s[lane + 32 * i] = e < E ? exp_proj(__fsub_rn(l[i], mx)) : 0.0f;
    }
    __syncwarp();
    float sum = 0.0f;
    if (lane == 0) {
#pragma unroll 8
        for (int e = 0; e < E; ++e) sum = __fadd_rn(sum, ex_s[e]);
    }
    sum = __shfl_sync(0xffffffffu, sum, 0);
    id_j = 0;
    for (int j = 0; j < topk; ++j) {
        uint32_t kl = key[0];
#pragma unroll
        for (int i = 1; i < EPL; ++i) kl = max(kl, key[i]);
        const uint32_t km = __reduce_max_sync(0xffffffffu, kl);
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (key[i] == km) key[i] = 0u;   // taken (keys are distinct: the index is in them)
        if (lane == j) id_j = (int)(0xffffu - (km & 0xffffu));
    }
    const float p_j = lane < topk ? __fdiv_rn(ex_s[id_j], sum) : 0.0f;
    float ssel = 0.0f;
    for (int j = 0; j < topk; ++j) ssel = __fadd_rn(ssel, __shfl_sync(0xffffffffu, p_j, j));
    w_j = lane < topk ? __fdiv_rn(p_j, ssel) : 0.0f;
}

// Exclusive scan of one int per thread over the whole CTA (at most 16
// warps); returns (exclusive prefix, total).  Every thread of the CTA calls it.
__device__ __forceinline__ int2 block_excl_scan(int v, int* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    __syncthreads();
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
        if (w < warp) before += warp_tot[w];
        total += warp_tot[w];
    }
    return make_int2(incl - v + before, total);
}

// a6: thread e (< E; one expert per thread, E <= blockDim.x) holds count c;
// writes offsets, tile offsets in tiles of tile_rows rows and the list of
// touched experts.  Returns the expert's offset.
__device__ __forceinline__ int moe_plan_write(int c, int E, const MoePlan& p, int* warp_tot) {
    const int e = threadIdx.x;
    const int2 off = block_excl_scan(c, warp_tot);
    if (e < E) p.offsets[e] = off.x;
    if (e == 0) p.offsets[E] = off.y;
    const int2 toff = block_excl_scan((c + p.tile_rows - 1) / p.tile_rows, warp_tot);
    if (e < E) p.tile_off[e] = toff.x;
    if (e == 0) p.tile_off[E] = toff.y;
    const int2 act = block_excl_scan(c > 0 ? 1 : 0, warp_tot);
    if (e < E && c > 0) p.active[act.x] = e;
    if (e == 0) p.n_active[0] = act.y;
    return off.x;
}

template <int EPL>
__global__ void __launch_bounds__(256) moe_route_plan_kernel(const uint16_t* __restrict__ logits, int64_t T, int E,
                                                             int topk, int32_t* __restrict__ ids,
                                                             float* __restrict__ wts, MoePlan p) {
    // the scatter that follows may start its launch now; it waits for this grid
    asm volatile("griddepcontrol.launch_dependents;");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
    __shared__ float ex_s[8][32 * EPL];
    if (t < T) {
        int id_j;
        float w_j;
        route_token<EPL>(logits + t * E, E, topk, ex_s[warp], id_j, w_j);
        if (lane < topk) {
            ids[t * topk + lane] = id_j;
            wts[t * topk + lane] = w_j;
            p.rank[t * topk + lane] = atomicAdd(p.counts + id_j, 1);
        }
    }

    // ---- the last CTA scans the histogram (E <= 256: one expert per thread)
    __shared__ int last;
    __shared__ int warp_tot[16];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = (atomicAdd(p.done, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int e = threadIdx.x;
    moe_plan_write(e < E ? __ldcg(p.counts + e) : 0, E, p, warp_tot);
}

// ---------------------------------------------------------------------------
// a7: per-token quant of x, scattered to the token's sorted rows.  One CTA per
// token with one 16-byte vector (8 bf16) per thread; blockDim is H/8 rounded
// up to a whole number of warps (H <= 8 * 1024).
struct MoeRows {
    const int32_t* ids;      // [T * topk]
    const float* wts;        // [T * topk]
    const int32_t* rank;     // [T * topk]
    const int32_t* offsets;  // [E + 1]
    int32_t* row_of;         // [T * topk] sorted row of (token, slot)
    int32_t* row_tok;        // [R]
    int32_t* row_slot;       // [R]
    float* row_w;            // [R]
};

__global__ void __launch_bounds__(1024) moe_quant_scatter_kernel(const uint16_t* __restrict__ x, int H, int topk,
                                                                 MoeRows rows,
                                                                 int8_t* __restrict__ xq, float* __restrict__ sxr,
                                                                 float* __restrict__ clear_rows,
                                                                 int8_t* __restrict__ dbg_qx,
                                                                 float* __restrict__ dbg_sx) {
    const int64_t t = blockIdx.x;
    // the plan comes from the kernel just before; the next kernel may launch
    // once every CTA is past this wait (so the plan is complete by then)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    // sorted rows of this token's slots (and their metadata)
    __shared__ int srow[kMoeMaxTopk];
    if (threadIdx.x < topk) {
        const int64_t i = t * topk + threadIdx.x;
        const int r = __ldcg(rows.offsets + __ldcg(rows.ids + i)) + __ldcg(rows.rank + i);
        srow[threadIdx.x] = r;
        rows.row_of[i] = r;
        rows.row_tok[r] = (int)t;
        rows.row_slot[r] = threadIdx.x;
        rows.row_w[r] = __ldcg(rows.wts + i);
    }
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
        const float rcp = __frcp_rn(s);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            pk[j >> 2] |= (uint32_t)(uint8_t)(int8_t)quant_code_rcp(f[j], s, rcp) << (8 * (j & 3));
    }
    const uint2 codes = make_uint2(pk[0], pk[1]);
    for (int j = 0; j < topk; ++j) {
        const int r = srow[j];
        *reinterpret_cast<uint2*>(xq + (int64_t)r * H + v * 8) = codes;
        if (threadIdx.x == 0) sxr[r] = s;
    }
    if (dbg_qx) *reinterpret_cast<uint2*>(dbg_qx + t * H + v * 8) = codes;
    if (dbg_sx && threadIdx.x == 0) dbg_sx[t] = s;
    if (clear_rows) {   // atomic combine: this token's fp32 output row starts at zero
        float4* o = reinterpret_cast<float4*>(clear_rows + t * H) + 2 * v;
        o[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        o[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------
// a5 + a6 + a7 for a few tokens (T <= 16) in one CTA of 16 warps, warp t
// handling token t: routing, ranks from a shared-memory histogram (so the
// plan needs no cleared global counters), the plan scan, then the token's
// int8 codes written once per routed slot into the expert-sorted rows.
constexpr int kMoeFrontMaxT = 16;

template <int EPL>
__global__ void __launch_bounds__(512) moe_front_small_kernel(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ logits, int T, int E,
                                                              int H, int topk, int32_t* __restrict__ ids,
                                                              float* __restrict__ wts, MoePlan p, MoeRows rows,
                                                              int8_t* __restrict__ xq, float* __restrict__ sxr,
                                                              int8_t* __restrict__ dbg_qx,
                                                              float* __restrict__ dbg_sx) {
    // the GEMM that follows reads nothing of ours before its own wait
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ int s_cnt[256];
    __shared__ int s_off[256];
    __shared__ int s_rows[kMoeFrontMaxT][kMoeMaxTopk];
    __shared__ float ex_s[kMoeFrontMaxT][32 * EPL];
    __shared__ int warp_tot[16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < 256; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    int id_j = 0, rank_j = 0;
    float w_j = 0.0f;
    if (warp < T) {
        route_token<EPL>(logits + (int64_t)warp * E, E, topk, ex_s[warp], id_j, w_j);
        if (lane < topk) {
            rank_j = atomicAdd(&s_cnt[id_j], 1);
            ids[warp * topk + lane] = id_j;
            wts[warp * topk + lane] = w_j;
            p.rank[warp * topk + lane] = rank_j;
        }
    }
    __syncthreads();
    const int e = threadIdx.x;
    const int c = e < E ? s_cnt[e] : 0;
    if (e < E) p.counts[e] = c;
    const int off = moe_plan_write(c, E, p, warp_tot);
    if (e < E) s_off[e] = off;
    __syncthreads();
    if (warp >= T) return;
    if (lane < topk) {
        const int r = s_off[id_j] + rank_j;
        s_rows[warp][lane] = r;
        rows.row_of[warp * topk + lane] = r;
        rows.row_tok[r] = warp;
        rows.row_slot[r] = lane;
        rows.row_w[r] = w_j;
    }
    __syncwarp();
    // a7: the token's codes (two passes over its row; the second hits L1)
    using VT = VecTraits<uint16_t>;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)warp * H);
    const int nvec = H / 8;
    VT::Acc acc = VT::acc_init();
    for (int v = lane; v < nvec; v += 32) VT::acc(acc, __ldg(xr + v));
    float amax;
    if (!VT::acc_final(acc, amax)) {   // NaN among this lane's values
        amax = 0.0f;
        for (int v = lane; v < nvec; v += 32) amax = fmaxf(amax, vec_absmax<uint16_t>(__ldg(xr + v)));
    }
    const QuantRow q(warp_max(amax));
    if (lane < topk) sxr[s_rows[warp][lane]] = q.s;
    if (dbg_sx && lane == 0) dbg_sx[warp] = q.s;
    for (int v = lane; v < nvec; v += 32) {
        float f[8];
        VT::unpack(__ldg(xr + v), f);
        uint32_t pk[2];
        quant_codes<2>(f, q, pk);
        const uint2 codes = make_uint2(pk[0], pk[1]);
        for (int j = 0; j < topk; ++j)
            *reinterpret_cast<uint2*>(xq + (int64_t)s_rows[warp][j] * H + v * 8) = codes;
        if (dbg_qx) *reinterpret_cast<uint2*>(dbg_qx + (int64_t)warp * H + v * 8) = codes;
    }
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
    // gemm2: w * y2 of each sorted row into contrib [T * topk, rows] at (token, slot),
    // or (topk == 0) added atomically into contrib [T, rows]
    const int32_t* row_tok;
    const int32_t* row_slot;
    const float* row_w;
    float* contrib;
    int topk;
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
    a.trig = 0;
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
                        // topk > 0: store at (token, slot); 0: atomic add into the token's row
                        const int64_t oi = m.topk > 0 ? (int64_t)__ldg(m.row_tok + r) * m.topk + __ldg(m.row_slot + r)
                                                      : (int64_t)__ldg(m.row_tok + r);
                        float* orow = m.contrib + oi * m.rows;
#pragma unroll
                        for (int jr = 0; jr < 2; ++jr) {   // weight row g + 8 jr
                            const int n = block * 16 + g + 8 * jr;
                            const float y2 =
                                __fmul_rn(__fmul_rn(__int2float_rn(acc[tg][2 * jr + jt]), sx), __ldg(swe + n));
                            if (m.topk > 0)
                                orow[n] = __fmul_rn(wr, y2);
                            else
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
// a11: out[t, n] = bf16( sum over slots j = 0 .. k-1 of contrib[t, j, n] ),
// summed in fp32 in slot order.  Four columns per thread (H % 4 == 0).
// With topk == 1 this is the plain fp32 -> bf16 conversion of an
// already-combined [T, H] buffer.
__global__ void moe_finalize_kernel(const float* __restrict__ contrib, uint16_t* __restrict__ y, int64_t T, int H,
                                    int topk) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // contrib comes from the kernel just before
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i >= T * H) return;
    const int64_t t = i / H, n = i % H;
    const float* src = contrib + t * topk * H + n;
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
    for (int j = 0; j < topk; ++j) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(src + (int64_t)j * H));
        a0 = __fadd_rn(a0, v.x);
        a1 = __fadd_rn(a1, v.y);
        a2 = __fadd_rn(a2, v.z);
        a3 = __fadd_rn(a3, v.w);
    }
    *reinterpret_cast<uint2*>(y + i) = make_uint2(pack_bf16x2(a0, a1), pack_bf16x2(a2, a3));
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
