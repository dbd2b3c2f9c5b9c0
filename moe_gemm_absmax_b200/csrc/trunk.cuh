// The trunk linears' two-level format -- "Qwen3.6-35B-A3B IQ8R - radiance
// container", file table (Trunk: int8 codes -127..127 with a u8 scale per
// row and 256 of K under a bf16 scale a row, each 128 of K rotated by the
// unnormalised Hadamard, round to nearest) and recipe (codes=i8 group=256
// scale=u8 scale2=bf16 block2=1x* transform=fwht128 clamp=sym rule=search).
//
// trunk_weight_quant_kernel: one CTA per weight row.  The row is rotated 128
// at a time (one warp per block, the butterflies of fwht128_warp) into shared
// memory in fp32; scale2 = bf16_rne(max |w'| / (127 * 255)); then one warp per
// 256-wide group searches u = 1 .. 255 for the scale s = u * scale2 with the
// smallest largest error max_k |w'_k - q_k s| (q_k = clamp(rne(w'_k / s), +-127),
// each step one fp32 rounding; the product q_k s is exact), ties to the
// smaller u, and writes the codes under the chosen scale.  A maximum is
// independent of the order it is taken in, so the choice is the same bit for
// bit wherever it is computed.  Set-up work (weights), not on the token path.
#pragma once

#include "common.cuh"
#include "fwht.cuh"

namespace w8a8 {

constexpr int kTrunkMaxK = 8192;

__global__ void __launch_bounds__(256) trunk_weight_quant_kernel(const uint16_t* __restrict__ w, int64_t K,
                                                                 int8_t* __restrict__ q, uint8_t* __restrict__ su8,
                                                                 uint16_t* __restrict__ s2) {
    __shared__ __align__(16) float v[kTrunkMaxK];
    __shared__ float wmax[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n = blockIdx.x;
    const uint16_t* row = w + n * K;
    const int nblk = (int)(K / 128);
    float m = 0.0f;
    for (int b = warp; b < nblk; b += 8) {
        float x[4];
        fwht128_load4(row + b * 128 + 4 * lane, x);
        fwht128_warp(x, lane);
        *reinterpret_cast<float4*>(v + b * 128 + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp] = m;
    __syncthreads();
    float rmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) rmax = fmaxf(rmax, wmax[i]);
    const uint16_t sb = float_to_bf16_bits(__fdiv_rn(rmax, 32385.0f));
    const float s2f = bf16_bits_to_float(sb);
    if (threadIdx.x == 0) s2[n] = sb;
    const int ngrp = (int)(K / 256);
    for (int j = warp; j < ngrp; j += 8) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = v[j * 256 + i * 32 + lane];   // conflict-free: lane-strided
        int best = 0;
        if (s2f != 0.0f) {
            float best_err = INFINITY;
            for (int u = 1; u <= 255; ++u) {
                const float s = __fmul_rn((float)u, s2f);
                float worst = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float c = (float)quant_code(x[i], s);
                    worst = fmaxf(worst, fabsf(__fsub_rn(x[i], __fmul_rn(c, s))));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xffffffffu, worst, o));
                if (worst < best_err) {
                    best_err = worst;
                    best = u;
                }
            }
        }
        const float s = __fmul_rn((float)best, s2f);
#pragma unroll
        for (int i = 0; i < 8; ++i) q[n * K + j * 256 + i * 32 + lane] = best ? (int8_t)quant_code(x[i], s) : (int8_t)0;
        if (lane == 0) su8[n * ngrp + j] = (uint8_t)best;
    }
}

// Identity plan of a single expert over M token rows (the shared expert
// through the expert GEMMs): every row is its token, slot 0, weight 1.
__global__ void shared_plan_kernel(int M, int bn, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                   int32_t* __restrict__ tile_off, int32_t* __restrict__ row_tok,
                                   int32_t* __restrict__ row_slot, float* __restrict__ row_w) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r == 0) {
        counts[0] = M;
        offsets[0] = 0;
        offsets[1] = M;
        tile_off[0] = 0;
        tile_off[1] = (M + bn - 1) / bn;
    }
    if (r < M) {
        row_tok[r] = r;
        row_slot[r] = 0;
        row_w[r] = 1.0f;
    }
}

}  // namespace w8a8
