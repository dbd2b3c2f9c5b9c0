// Routed experts on the FWHT128 grid -- "Qwen3.6-35B-A3B IQ8R - radiance
// container", file table (Experts row: int8 codes on the rotated grid with
// one bf16 scale per row and 128-wide slice of K; Activations row: the
// activations quantized after the same rotation, the routed experts taking
// the codes of the trunk's activation quantizer) and the
// recipe rows of the experts' gate_up and down weights (group=128 scale=bf16
// transform=fwht128).
//
// The chain is that of the per-token absmax MoE with each quantizer replaced
// by the FWHT128 group quantizer and each expert GEMM by its group-128 form:
//   route + plan -> moe_fwht_scatter (x rotated along H, group codes and bf16
//   scales written to the token's k expert-sorted rows) -> gemm1 (swap-AB,
//   group-128 promotion, SiLU(gate) * up, fp32) -> fwht128_quant<float> of
//   the intermediate (rotated along I) -> gemm2 (swap-AB, group-128, times
//   the routing weight at (token, slot)) -> slot-order combine.
#pragma once

#include "fwht.cuh"
#include "moe.cuh"

namespace w8a8 {

constexpr int kMoeG128MaxGroupsH = 32;   // H <= 4096: one warp per group in the scatter CTA

// One CTA per token, one warp per 128-wide group of x (blockDim = 32 * H / 128).
__global__ void __launch_bounds__(1024) moe_fwht_scatter_kernel(const uint16_t* __restrict__ x, int H, int topk,
                                                                MoeRows rows, int8_t* __restrict__ xq,
                                                                uint16_t* __restrict__ sxg,
                                                                int8_t* __restrict__ dbg_qx,
                                                                uint16_t* __restrict__ dbg_sx) {
    const int64_t t = blockIdx.x;
    // the plan comes from the kernel just before; the next kernel may launch
    // once every CTA is past this wait (so the plan is complete by then)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
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
    const int lane = threadIdx.x & 31, g = threadIdx.x >> 5, G = H / 128;
    float v[4];
    fwht128_load4(x + t * H + g * 128 + 4 * lane, v);
    fwht128_warp(v, lane);
    uint16_t sb;
    const uint32_t pk = fwht128_codes(v, sb);
    __syncthreads();   // srow
    for (int j = 0; j < topk; ++j) {
        const int r = srow[j];
        *reinterpret_cast<uint32_t*>(xq + (int64_t)r * H + g * 128 + 4 * lane) = pk;
        if (lane == 0) sxg[(int64_t)r * G + g] = sb;
    }
    if (dbg_qx) *reinterpret_cast<uint32_t*>(dbg_qx + t * H + g * 128 + 4 * lane) = pk;
    if (dbg_sx && lane == 0) dbg_sx[t * G + g] = sb;
}

// Parity outputs: the sorted rows' codes and group scales of the gated
// intermediate, gathered into (token, slot) order.
__global__ void moe_debug_gather_g128_kernel(const int8_t* __restrict__ qa, const uint16_t* __restrict__ sa,
                                             const int32_t* __restrict__ row_of, int64_t n, int I,
                                             int8_t* __restrict__ dqa, uint16_t* __restrict__ dsa) {
    const int64_t i = blockIdx.x;   // (token, slot) entry
    if (i >= n) return;
    const int r = row_of[i];
    const int G = I / 128;
    for (int k = threadIdx.x; k < I; k += blockDim.x)
        if (dqa) dqa[i * I + k] = qa[(int64_t)r * I + k];
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        if (dsa) dsa[i * G + g] = sa[(int64_t)r * G + g];
}

}  // namespace w8a8
