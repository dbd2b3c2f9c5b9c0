// Per-row symmetric absmax int8 quantization (a0 weights, a1 activations,
// a9 MoE requant) -- "Qwen3.6-27B-Quark-W8A8-INT8", Quantization Scheme
// (per-channel / per-token symmetric); "Online INT8 W8A8 ...", Precision
// split (dynamic per-token int8 activation).
//
//   s = max_k |v_k| / 127           (fp32, IEEE division)
//   q = clamp(rne(v_k / s), -127, 127),  s == 0 -> q = 0
//
// One pass over HBM: each CTA keeps its slice of the row in registers
// (16-byte vector loads), reduces |v| with warp shuffles, and for short
// rows (decode: few tokens, long K) a thread-block cluster splits one row
// over up to 8 CTAs whose partial maxima meet through distributed shared
// memory.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace w8a8 {

namespace cg = cooperative_groups;

constexpr int kQuantMaxVec = 16;   // 16-byte vectors kept in registers per thread
constexpr int64_t kQuantSmemRowMax = 200 * 1024;   // largest row staged in shared memory

// Per input type: unpacking a 16-byte vector to fp32, and a running |v|
// maximum (Acc) whose final value equals the fp32 maximum that skips NaN;
// acc_final returns false when the fast accumulator cannot say (bf16 NaN
// seen), and the caller then takes the fp32 maximum of its vectors itself.
template <typename Tin>
struct VecTraits;
template <>
struct VecTraits<uint16_t> {   // bf16 bits: 8 per 16 bytes
    static constexpr int kElems = 8;
    using Acc = uint32_t;       // two 16-bit maxima of (bits & 0x7fff)
    __device__ static void unpack(const uint4& v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static Acc acc_init() { return 0u; }
    __device__ static void acc(Acc& a, const uint4& v) {
        a = max_u16x2(a, v.x & 0x7fff7fffu);
        a = max_u16x2(a, v.y & 0x7fff7fffu);
        a = max_u16x2(a, v.z & 0x7fff7fffu);
        a = max_u16x2(a, v.w & 0x7fff7fffu);
    }
    __device__ static bool acc_final(Acc a, float& amax) {
        const uint32_t m = max(a & 0xffffu, a >> 16);
        amax = __uint_as_float(m << 16);
        return m <= 0x7f80u;
    }
};
template <>
struct VecTraits<float> {      // fp32: 4 per 16 bytes
    static constexpr int kElems = 4;
    using Acc = float;
    __device__ static void unpack(const uint4& v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ static Acc acc_init() { return 0.0f; }
    __device__ static void acc(Acc& a, const uint4& v) {
        a = fmaxf(a, fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))));
        a = fmaxf(a, fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
    }
    __device__ static bool acc_final(Acc a, float& amax) {
        amax = a;
        return true;
    }
};

// fp32 maximum of |v| over one vector, NaN skipped (fmaxf returns the other operand)
template <typename Tin>
__device__ __forceinline__ float vec_absmax(const uint4& raw) {
    using VT = VecTraits<Tin>;
    float f[VT::kElems];
    VT::unpack(raw, f);
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < VT::kElems; ++j) m = fmaxf(m, fabsf(f[j]));
    return m;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int E>
__device__ __forceinline__ void store_codes(int8_t* dst, const uint32_t (&packed)[E / 4]) {
    if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
        *reinterpret_cast<uint32_t*>(dst) = packed[0];
    }
}

// unpack one vector and write its codes
template <typename Tin>
__device__ __forceinline__ void quant_vec_store(const uint4& raw, const QuantRow& r, int8_t* dst) {
    using VT = VecTraits<Tin>;
    constexpr int E = VT::kElems;
    float f[E];
    VT::unpack(raw, f);
    uint32_t packed[E / 4];
    quant_codes<E / 4>(f, r, packed);
    store_codes<E>(dst, packed);
}

// Start of every quant kernel.  It may be launched to overlap the kernel
// before it on the stream (programmatic dependent launch), so it touches no
// memory before griddepcontrol.wait: x may come from that kernel, and q / s
// may still be read by it.  Only after the wait does it let the kernel after
// it launch (that kernel streams weights before its own wait), so that
// everything before this quant kernel on the stream has completed by the
// time anything after it runs.
__device__ __forceinline__ void quant_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}

// Many rows: one CTA per row, the row staged in shared memory by 16-byte
// asynchronous copies (no registers held while the loads are in flight, so
// an SM keeps as many rows in flight as its shared memory holds).  Each
// thread reads back only the vectors it copied itself, so its own
// cp.async.wait_group is the only wait before the first pass.
template <typename Tin, int NT>
__global__ void __launch_bounds__(NT) quant_rows_smem_kernel(const Tin* __restrict__ x, int64_t K, int64_t ldx,
                                                             int8_t* __restrict__ q, int64_t ldq,
                                                             float* __restrict__ s, int* zero_buf, int zero_n) {
    using VT = VecTraits<Tin>;
    constexpr int E = VT::kElems;
    extern __shared__ __align__(16) uint4 row_s[];
    quant_dependency_wait();
    const int64_t row = blockIdx.x;
    const int nvec = (int)(K / E);
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
    for (int v = threadIdx.x; v < nvec; v += NT) cp_async_16(row_s + v, xr + v);
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int i = blockIdx.x * NT + threadIdx.x; i < zero_n; i += gridDim.x * NT) zero_buf[i] = 0;
    asm volatile("cp.async.wait_group 0;" ::: "memory");

    typename VT::Acc acc = VT::acc_init();
    for (int v = threadIdx.x; v < nvec; v += NT) VT::acc(acc, row_s[v]);
    float amax;
    if (!VT::acc_final(acc, amax)) {   // NaN among this thread's values
        amax = 0.0f;
        for (int v = threadIdx.x; v < nvec; v += NT) amax = fmaxf(amax, vec_absmax<Tin>(row_s[v]));
    }
    __shared__ float red[NT / 32];
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) amax = fmaxf(amax, red[w]);
    const QuantRow qrow(amax);
    if (threadIdx.x == 0) s[row] = qrow.s;

    int8_t* qr = q + row * ldq;
    for (int v = threadIdx.x; v < nvec; v += NT) quant_vec_store<Tin>(row_s[v], qrow, qr + (int64_t)v * E);
}

// grid = (CL * rows); cluster = (CL, 1, 1).  Cluster r handles row r; its
// CTA c handles vectors [c * vpc, (c + 1) * vpc) (vpc = vectors per CTA).
template <typename Tin, int NT, int MAXV = kQuantMaxVec>
__global__ void __launch_bounds__(NT) quant_rows_kernel(const Tin* __restrict__ x, int64_t K, int64_t ldx,
                                                        int8_t* __restrict__ q, int64_t ldq, float* __restrict__ s,
                                                        int vpc, int cl, int* zero_buf, int zero_n) {
    using VT = VecTraits<Tin>;
    quant_dependency_wait();
    // optional side job: clear a small int buffer that a later kernel on the
    // same stream expects to find zero (split-K arrival counters)
    for (int i = blockIdx.x * NT + threadIdx.x; i < zero_n; i += gridDim.x * NT) zero_buf[i] = 0;
    constexpr int E = VT::kElems;
    const int64_t row = blockIdx.x / cl;
    const int crank = blockIdx.x % cl;
    const int64_t nvec = K / E;
    const int64_t v0 = (int64_t)crank * vpc;
    const int64_t v1 = min(nvec, v0 + vpc);
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);

    uint4 regs[MAXV];
    typename VT::Acc acc = VT::acc_init();
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int64_t v = v0 + threadIdx.x + (int64_t)i * NT;
        if (v < v1) {
            regs[i] = __ldcg(xr + v);
            VT::acc(acc, regs[i]);
        }
    }
    float amax;
    if (!VT::acc_final(acc, amax)) {   // NaN among this thread's values
        amax = 0.0f;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (v0 + threadIdx.x + (int64_t)i * NT < v1) amax = fmaxf(amax, vec_absmax<Tin>(regs[i]));
    }
    __shared__ float red[NT / 32];
    __shared__ float cta_max;
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, red[w]);
        cta_max = m;
    }
    if (cl > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        if (threadIdx.x == 0) {
            float m = 0.0f;
            for (int r = 0; r < cl; ++r) m = fmaxf(m, *cluster.map_shared_rank(&cta_max, r));
            red[0] = m;
        }
        cluster.sync();   // no CTA leaves while a peer may still read its cta_max
    } else {
        __syncthreads();
        if (threadIdx.x == 0) red[0] = cta_max;
    }
    __syncthreads();
    const QuantRow qrow(red[0]);
    if (crank == 0 && threadIdx.x == 0) s[row] = qrow.s;

    int8_t* qr = q + row * ldq;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int64_t v = v0 + threadIdx.x + (int64_t)i * NT;
        if (v < v1) quant_vec_store<Tin>(regs[i], qrow, qr + v * E);
    }
}

// Short rows (K <= 32 lanes x 8 vectors): one warp per row, 8 rows per CTA.
template <typename Tin>
__global__ void __launch_bounds__(256) quant_rows_warp_kernel(const Tin* __restrict__ x, int64_t rows, int64_t K,
                                                              int8_t* __restrict__ q, float* __restrict__ s) {
    using VT = VecTraits<Tin>;
    constexpr int E = VT::kElems;
    constexpr int kMaxV = 8;
    quant_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int64_t nvec = K / E;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * K);
    uint4 regs[kMaxV];
    typename VT::Acc acc = VT::acc_init();
#pragma unroll
    for (int i = 0; i < kMaxV; ++i) {
        const int64_t v = lane + 32 * i;
        if (v < nvec) {
            regs[i] = __ldcg(xr + v);
            VT::acc(acc, regs[i]);
        }
    }
    float amax;
    if (!VT::acc_final(acc, amax)) {   // NaN among this lane's values
        amax = 0.0f;
#pragma unroll
        for (int i = 0; i < kMaxV; ++i)
            if (lane + 32 * i < nvec) amax = fmaxf(amax, vec_absmax<Tin>(regs[i]));
    }
    const QuantRow qrow(warp_max(amax));
    if (lane == 0) s[row] = qrow.s;
    int8_t* qr = q + row * K;
#pragma unroll
    for (int i = 0; i < kMaxV; ++i) {
        const int64_t v = lane + 32 * i;
        if (v < nvec) quant_vec_store<Tin>(regs[i], qrow, qr + v * E);
    }
}

// Picks the CTA size, the cluster width and the register slice, and launches.
// Requirements (checked by callers): K % (16 / sizeof(Tin)) == 0, ldx likewise,
// 16-byte aligned x, 8-byte aligned q rows.
//   many rows: one CTA per row (no cluster), 64..1024 threads so that each
//              thread holds at most 4 vectors where possible;
//   few rows (decode): a power-of-two cluster of up to 8 CTAs per row, so that
//              more SMs pull the row from HBM.
template <typename Tin>
cudaError_t launch_quant_rows(const Tin* x, int64_t rows, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* s,
                              cudaStream_t stream, int num_sms, int* zero_buf = nullptr, int zero_n = 0,
                              bool pdl = false) {
    cudaLaunchAttribute pdl_attr[1];
    pdl_attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr[0].val.programmaticStreamSerializationAllowed = 1;
    constexpr int E = VecTraits<Tin>::kElems;
    const int64_t nvec = K / E;
    if (nvec <= 256 && rows >= 4 * (int64_t)num_sms && zero_n == 0 && ldx == K && ldq == K) {
        // many short rows (the MoE requant): a warp per row
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((rows + 7) / 8), 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = stream;
        cfg.attrs = pdl_attr;
        cfg.numAttrs = pdl ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, quant_rows_warp_kernel<Tin>, x, rows, K, q, s);
    }
    if (rows >= 2 * (int64_t)num_sms && nvec * 16 <= kQuantSmemRowMax) {
        const size_t smem = (size_t)nvec * 16;
        int rows_per_sm = (int)((228 * 1024) / (smem + 1024));
        rows_per_sm = rows_per_sm < 1 ? 1 : (rows_per_sm > 32 ? 32 : rows_per_sm);
        // threads per CTA: fill the SM's 2048 threads so that the dependent ALU
        // chains of the quantization overlap across warps -- with 16 or more
        // rows resident 128 threads do (64 from 32 rows); with fewer, the
        // largest power of two that keeps every row that fits resident
        int nt = rows_per_sm >= 32 ? 64 : 128;
        while (rows_per_sm < 16 && nt < 512 && rows_per_sm * nt * 2 <= 2048) nt *= 2;
        auto kern = nt == 512 ? quant_rows_smem_kernel<Tin, 512>
                  : nt == 256 ? quant_rows_smem_kernel<Tin, 256>
                  : nt == 128 ? quant_rows_smem_kernel<Tin, 128> : quant_rows_smem_kernel<Tin, 64>;
        if (smem > 48 * 1024) {
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)rows, 1, 1);
        cfg.blockDim = dim3((unsigned)nt, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cfg.attrs = pdl_attr;
        cfg.numAttrs = pdl ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, kern, x, K, ldx, q, ldq, s, zero_buf, zero_n);
    }
    int NT, cl;
    if (rows >= 2 * (int64_t)num_sms && nvec <= 1024 * 6) {
        // (1024 threads leave 64 registers a thread: at most 6 vectors)
        cl = 1;
        NT = 64;
        while (NT < 1024 && nvec > (int64_t)NT * 4) NT *= 2;
    } else {
        NT = nvec <= 64 ? 64 : (nvec <= 128 ? 128 : 256);
        cl = 1;
        while (cl < 8 && nvec > (int64_t)NT * 4 * cl) cl *= 2;                       // fit in 4 / thread
        if (nvec > (int64_t)NT * kQuantMaxVec * cl) return cudaErrorInvalidValue;
        while (cl < 8 && rows * cl < 2 * num_sms && nvec / (cl * 2) >= (int64_t)NT) cl *= 2;   // spread
    }
    const int vpc = (int)((nvec + cl - 1) / cl);
    const int per_thread = (vpc + NT - 1) / NT;

    cudaLaunchConfig_t cfg = {};
    if (rows * cl > 0x7fffffffLL) return cudaErrorInvalidValue;
    cfg.gridDim = dim3((unsigned)(rows * cl), 1, 1);
    cfg.blockDim = dim3((unsigned)NT, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (cl > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)cl;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) attr[na++] = pdl_attr[0];
    cfg.attrs = attr;
    cfg.numAttrs = na;
#define W8A8_QUANT_LAUNCH(nt, mv) \
    return cudaLaunchKernelEx(&cfg, quant_rows_kernel<Tin, nt, mv>, x, K, ldx, q, ldq, s, vpc, cl, zero_buf, zero_n)
    switch (NT) {
        case 64:
            if (per_thread <= 4) W8A8_QUANT_LAUNCH(64, 4);
            W8A8_QUANT_LAUNCH(64, 16);
        case 128:
            if (per_thread <= 4) W8A8_QUANT_LAUNCH(128, 4);
            W8A8_QUANT_LAUNCH(128, 16);
        case 256:
            if (per_thread <= 4) W8A8_QUANT_LAUNCH(256, 4);
            if (per_thread <= 8) W8A8_QUANT_LAUNCH(256, 8);
            W8A8_QUANT_LAUNCH(256, 16);
        case 512:
            W8A8_QUANT_LAUNCH(512, 4);
        default:
            if (per_thread <= 4) W8A8_QUANT_LAUNCH(1024, 4);
            W8A8_QUANT_LAUNCH(1024, 6);
    }
#undef W8A8_QUANT_LAUNCH
}

}  // namespace w8a8
