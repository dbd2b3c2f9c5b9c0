// FWHT128-domain W8A8 (a12, a13) -- "Qwen3.6-35B-A3B IQ8R - radiance
// container": file table (every 128-wide slice of K turned by the
// unnormalised Hadamard matrix; int8 codes in -127..127 with one bf16 scale
// for each row and slice; the activations quantized after the same
// rotation) and the recipe (transform=fwht128 group=128
// scale=bf16 clamp=sym).
//
// fwht128_warp / fwht128_quant_kernel: one warp per 128-wide block of a row.  Lane l holds
// elements 4l .. 4l+3 in fp32.  The textbook in-place butterflies run stage
// by stage, h = 1, 2, 4, ..., 64, each pair (a, b) at distance h becoming
// (a + b, a - b): stages 1 and 2 inside the lane, stages 4 .. 64 between
// lanes l and l ^ (h / 4) through shuffles.  The same pairs in the same
// order as the serial loop, so the fp32 result is the same bit for bit.
// Then s = bf16_rne(max |x'| / 127), q = clamp(rne(x' / float(s)), +-127).
//
// gemv_g128_kernel: decode-sized M (<= 8) group-scaled GEMV.  Warps split the
// K groups, keep each group's exact int32 partial p_g in shared memory, and
// one warp applies acc = fma(float(p_g), sx*sw, acc) in ascending g -- the
// same fp32 steps as the serial definition -- and y = acc * post (1/128 in the
// rotated domain, 1 on the unrotated grid).
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace w8a8 {

// The rotation of one 128-wide block by one warp: lane l holds elements
// 4l .. 4l+3 in fp32 (see above for the stage order).
__device__ __forceinline__ void fwht128_warp(float (&v)[4], int lane) {
    // h = 1: (0,1), (2,3)
    {
        const float a0 = v[0], b0 = v[1], a1 = v[2], b1 = v[3];
        v[0] = __fadd_rn(a0, b0);
        v[1] = __fsub_rn(a0, b0);
        v[2] = __fadd_rn(a1, b1);
        v[3] = __fsub_rn(a1, b1);
    }
    // h = 2: (0,2), (1,3)
    {
        const float a0 = v[0], b0 = v[2], a1 = v[1], b1 = v[3];
        v[0] = __fadd_rn(a0, b0);
        v[2] = __fsub_rn(a0, b0);
        v[1] = __fadd_rn(a1, b1);
        v[3] = __fsub_rn(a1, b1);
    }
    // h = 4 .. 64: partner lane l ^ (h / 4); the lane with the bit clear holds a
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const bool upper = (lane & d) != 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], d);
            v[j] = upper ? __fsub_rn(o, v[j]) : __fadd_rn(v[j], o);
        }
    }
}

// Group quantization of a rotated block held as above: the bf16 scale
// s = bf16_rne(max |x'| / 127) (returned in sb, every lane) and this lane's
// four codes clamp(rne(x' / float(s)), +-127), packed little-endian.
__device__ __forceinline__ uint32_t fwht128_codes(const float (&v)[4], uint16_t& sb) {
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    sb = float_to_bf16_bits(__fdiv_rn(amax, 127.0f));
    const float sf = bf16_bits_to_float(sb);
    uint32_t pk = 0u;
    if (sf != 0.0f) {
        const float rcp = __frcp_rn(sf);
#pragma unroll
        for (int j = 0; j < 4; ++j) pk |= (uint32_t)(uint8_t)(int8_t)quant_code_rcp(v[j], sf, rcp) << (8 * j);
    }
    return pk;
}

__device__ __forceinline__ void fwht128_load4(const uint16_t* src, float (&v)[4]) {
    const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(src));
    v[0] = __uint_as_float(raw.x << 16);
    v[1] = __uint_as_float(raw.x & 0xffff0000u);
    v[2] = __uint_as_float(raw.y << 16);
    v[3] = __uint_as_float(raw.y & 0xffff0000u);
}
__device__ __forceinline__ void fwht128_load4(const float* src, float (&v)[4]) {
    const float4 raw = __ldcg(reinterpret_cast<const float4*>(src));
    v[0] = raw.x;
    v[1] = raw.y;
    v[2] = raw.z;
    v[3] = raw.w;
}

// Each warp quantizes BPW consecutive 128-wide blocks (of one row or of
// consecutive rows), all of their loads issued before the first butterfly so
// that several are in flight (BPW = 4 for large inputs, 1 for a few rows,
// where spreading the blocks over more warps is shorter); bf16 rows (activations, weights) or
// fp32 rows (the routed experts' gated intermediate).  ROTATE = false is the
// same group quantizer on the unrotated grid (the head's format: a bf16 scale
// per row and 128 of K, no transform).  On a chain with programmatic
// dependent launch it waits for the kernel before it (a no-op otherwise) and
// reads its rows with coherent loads.
template <typename Tin, bool ROTATE = true, int BPW = 1>
__global__ void __launch_bounds__(256) fwht128_quant_kernel(const Tin* __restrict__ x, int64_t M, int64_t K,
                                                            int8_t* __restrict__ q, uint16_t* __restrict__ s) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int lane = threadIdx.x & 31;
    const int64_t G = K / 128, nblk = M * G;
    const int64_t blk0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * BPW;
    if (blk0 >= nblk) return;
    // block b of row m starts at m * K + g * 128 = b * 128: the blocks are contiguous
    float v[BPW][4];
#pragma unroll
    for (int i = 0; i < BPW; ++i)
        if (blk0 + i < nblk) fwht128_load4(x + (blk0 + i) * 128 + 4 * lane, v[i]);
#pragma unroll
    for (int i = 0; i < BPW; ++i) {
        if (blk0 + i >= nblk) break;
        if constexpr (ROTATE) fwht128_warp(v[i], lane);
        uint16_t sb;
        const uint32_t pk = fwht128_codes(v[i], sb);
        *reinterpret_cast<uint32_t*>(q + (blk0 + i) * 128 + 4 * lane) = pk;
        if (lane == 0) s[blk0 + i] = sb;
    }
}

// Blocks per warp for M rows of K, and the grid (8 warps per CTA).
inline int fwht128_quant_bpw(int64_t M, int64_t K) { return M * (K / 128) >= 148 * 8 * 8 ? 4 : 1; }
inline int64_t fwht128_quant_ctas(int64_t M, int64_t K) {
    const int bpw = fwht128_quant_bpw(M, K);
    const int64_t warps = (M * (K / 128) + bpw - 1) / bpw;
    return (warps + 7) / 8;
}

// Launches fwht128_quant_kernel (optionally chained with programmatic
// dependent launch) with the block count per warp chosen for the size.
template <typename Tin, bool ROTATE>
cudaError_t launch_fwht128_quant(const Tin* x, int64_t M, int64_t K, int8_t* q, uint16_t* s, cudaStream_t st,
                                 bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)fwht128_quant_ctas(M, K), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
    if (fwht128_quant_bpw(M, K) == 4)
        return cudaLaunchKernelEx(&cfg, fwht128_quant_kernel<Tin, ROTATE, 4>, x, M, K, q, s);
    return cudaLaunchKernelEx(&cfg, fwht128_quant_kernel<Tin, ROTATE, 1>, x, M, K, q, s);
}

constexpr int kG128MaxGroups = 64;

// Dynamic shared memory of gemv_g128_kernel for K / 128 = G groups (<= 39 KB).
inline size_t gemv_g128_smem(int G) { return (size_t)G * (32 * 16 + 16 * 4 + 8 * 4); }

// One CTA per 16 weight rows; 8 warps split the K groups; tokens <= 8.  The
// scales of the CTA's rows and tokens are staged in shared memory first, so
// that the serial per-group promotion of warp 0 reads no global memory.
// GATED: rows 2i / 2i+1 are gate_i / up_i (both in one CTA's 16 rows) and the
// output is a[m, i] = SiLU(v_2i) * v_2i+1 in fp32 (a_out [M, N/2]) instead of
// bf16 y.  Launched with programmatic dependent launch, a CTA only prefetches
// its weight rows into L2 before the dependency wait (L2 is coherent with
// whatever kernel before it may still be writing them) and reads everything
// after it, with coherent loads (the wait is a no-op otherwise).
template <bool GATED>
__global__ void __launch_bounds__(256) gemv_g128_kernel(const int8_t* __restrict__ qx,
                                                        const uint16_t* __restrict__ sx,
                                                        const int8_t* __restrict__ qw,
                                                        const uint16_t* __restrict__ sw, uint16_t* __restrict__ y,
                                                        int M, int N, int K, float post,
                                                        const uint8_t* __restrict__ sw_u8,
                                                        const uint16_t* __restrict__ sw_row,
                                                        float* __restrict__ a_out) {
    // shared memory sized by the group count (gemv_g128_smem), so that short
    // rows leave room for more CTAs per SM
    extern __shared__ int4 g128_smem[];
    const int G = K / 128;
    int4* pg = g128_smem;                                               // [G][32] int32 partials
    float* s_sw = reinterpret_cast<float*>(g128_smem + G * 32);         // [16][G] row scales
    float* s_sx = s_sw + 16 * G;                                        // [8][G] token scales
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t = lane & 3;
    const int block = blockIdx.x;
    {   // this CTA's 16 weight rows into L2, one 128-byte line per thread and pass
        const int64_t base = (int64_t)block * 16 * K, bytes = (int64_t)min(16, N - block * 16) * K;
        for (int64_t o = (int64_t)threadIdx.x * 128; o < bytes; o += (int64_t)blockDim.x * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(qw + base + o));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    for (int i = threadIdx.x; i < 16 * G; i += blockDim.x) {
        const int r = i / G, grp = i - r * G, n = block * 16 + r;
        float v = 0.0f;
        if (n < N)   // the two-level trunk format: u8 per 256 of K times a bf16 row scale (exact)
            v = sw_u8 ? __fmul_rn((float)__ldcg(sw_u8 + (int64_t)n * (G / 2) + grp / 2),
                                  bf16_bits_to_float(__ldcg(sw_row + n)))
                      : bf16_bits_to_float(__ldcg(sw + (int64_t)n * G + grp));
        s_sw[r * G + grp] = v;
    }
    for (int i = threadIdx.x; i < 8 * G; i += blockDim.x) {
        const int m = i / G, grp = i - m * G;
        s_sx[m * G + grp] = m < M ? bf16_bits_to_float(__ldcg(sx + (int64_t)m * G + grp)) : 0.0f;
    }
    const int8_t* w0 = qw + (int64_t)(block * 16 + g8) * K + 16 * t;
    const int8_t* w1 = w0 + 8 * (int64_t)K;
    const bool tok_ok = g8 < M;
    const int8_t* xr = qx + (int64_t)g8 * K + 16 * t;
    for (int grp = warp; grp < G; grp += 8) {
        int acc[4] = {0, 0, 0, 0};
        uint4 wa[2], wb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            wa[u] = ld_stream_16(w0 + grp * 128 + u * 64);
            wb[u] = ld_stream_16(w1 + grp * 128 + u * 64);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            uint4 xb = make_uint4(0, 0, 0, 0);
            if (tok_ok) xb = __ldca(reinterpret_cast<const uint4*>(xr + grp * 128 + u * 64));
            const uint32_t A1[4] = {wa[u].x, wb[u].x, wa[u].y, wb[u].y};
            const uint32_t B1[2] = {xb.x, xb.y};
            const uint32_t A2[4] = {wa[u].z, wb[u].z, wa[u].w, wb[u].w};
            const uint32_t B2[2] = {xb.z, xb.w};
            mma_s8_16832(acc, A1, B1);
            mma_s8_16832(acc, A2, B2);
        }
        pg[grp * 32 + lane] = make_int4(acc[0], acc[1], acc[2], acc[3]);
    }
    __syncthreads();
    if (warp != 0) return;
    float yv[4] = {0.f, 0.f, 0.f, 0.f};
    for (int grp = 0; grp < G; ++grp) {
        const int4 p = pg[grp * 32 + lane];
        const int pv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = 2 * t + (j & 1);
            const int r = g8 + 8 * (j >> 1);
            if (m < M) yv[j] = __fmaf_rn(__int2float_rn(pv[j]), __fmul_rn(s_sx[m * G + grp], s_sw[r * G + grp]), yv[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int m = 2 * t + (j & 1);
        const int n = block * 16 + g8 + 8 * (j >> 1);
        const float v = __fmul_rn(yv[j], post);
        if constexpr (GATED) {
            // rows 2i (even g8) and 2i+1 (odd g8) sit in lanes 4 apart
            const float up = __shfl_xor_sync(0xffffffffu, v, 4);
            if (m < M && n < N && !(g8 & 1)) a_out[(int64_t)m * (N / 2) + (n >> 1)] = __fmul_rn(silu_proj(v), up);
        } else {
            if (m < M && n < N) y[(int64_t)m * N + n] = float_to_bf16_bits(v);
        }
    }
}

}  // namespace w8a8
