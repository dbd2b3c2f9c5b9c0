// libw8a8.so: the C ABI declared in include/w8a8.h.
//
// Host side only: argument checks, workspace carving, kernel selection and
// launches.  Every entry point enqueues on the caller's stream, allocates
// nothing and never synchronizes (w8a8_get_device_error excepted, which is
// documented to synchronize).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "fwht.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "gemv.cuh"
#include "gemv_tc.cuh"
#include "moe.cuh"
#include "moe_g128.cuh"
#include "moe_swap.cuh"
#include "quant.cuh"
#include "trunk.cuh"
#include "w8a8.h"

using namespace w8a8;

namespace {

constexpr int kMaxDevices = 64;

int device_sms(int dev) {
    static int sms[kMaxDevices] = {0};
    if (dev < 0 || dev >= kMaxDevices) return 148;
    if (sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        sms[dev] = v;
    }
    return sms[dev];
}

int current_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return device_sms(dev);
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? W8A8_OK : W8A8_ERR_CUDA; }

inline int last_launch_status() { return cuda_status(cudaGetLastError()); }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ----------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// int8 matrix [rows, cols] (row stride cols bytes) read as box_rows x 128-byte tiles, 128-byte swizzle.
bool make_tmap_i8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols};
    cuuint32_t box[2] = {(cuuint32_t)kTcBK, box_rows};
    cuuint32_t estride[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- tcgen05 GEMM
template <int BN, int STAGES, int EPI, int NACC, int NEPI = 4>
int launch_tc(const int8_t* A, const int8_t* B, TcParams p, cudaStream_t st) {
    using SM = TcSmem<BN, STAGES>;
    auto kern = gemm_i8_tc_kernel<BN, STAGES, EPI, NACC, false, NEPI>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    static bool attr_done[kMaxDevices] = {false};
    if (dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes) != cudaSuccess)
            return W8A8_ERR_CUDA;
        attr_done[dev] = true;
    }
    CUtensorMap ta, tb;
    if (!make_tmap_i8(&ta, A, (uint64_t)p.M, (uint64_t)p.K, kTcBM)) return W8A8_ERR_CUDA;
    if (!make_tmap_i8(&tb, B, (uint64_t)p.N, (uint64_t)p.K, BN)) return W8A8_ERR_CUDA;
    p.num_m_tiles = (p.M + kTcBM - 1) / kTcBM;
    p.num_n_tiles = (p.N + BN - 1) / BN;
    p.num_k_blocks = (p.K + kTcBK - 1) / kTcBK;
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    const int grid = tiles < device_sms(dev) ? tiles : device_sms(dev);
    kern<<<grid, tc_threads<NEPI>(), SM::kBytes, st>>>(ta, tb, p);
    return last_launch_status();
}

// Pair-tile GEMM (cta_group::2, 256 x BN tiles over two SMs).
template <int EPI, int BN>
int launch_tc2_bn(const int8_t* A, const int8_t* B, TcParams p, cudaStream_t st) {
    using SM = Tc2Smem<BN>;
    auto kern = gemm_i8_tc2_kernel<EPI, BN>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    static int max_clusters[kMaxDevices] = {0};
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kTc2Threads, 1, 1);
    cfg.dynamicSmemBytes = SM::kBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (max_clusters[dev] == 0) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes) != cudaSuccess)
            return W8A8_ERR_CUDA;
        cfg.gridDim = dim3((unsigned)(2 * (device_sms(dev) / 2)), 1, 1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = device_sms(dev) / 2;
        max_clusters[dev] = n;
    }
    CUtensorMap ta, tb;
    if (!make_tmap_i8(&ta, A, (uint64_t)p.M, (uint64_t)p.K, 128)) return W8A8_ERR_CUDA;
    if (!make_tmap_i8(&tb, B, (uint64_t)p.N, (uint64_t)p.K, BN / 2)) return W8A8_ERR_CUDA;
    p.num_m_tiles = (p.M + kTc2BM - 1) / kTc2BM;
    p.num_n_tiles = (p.N + BN - 1) / BN;
    p.num_k_blocks = (p.K + kTcBK - 1) / kTcBK;
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    const int clusters = tiles < max_clusters[dev] ? tiles : max_clusters[dev];
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, p));
}

// Pair-tile width: 256 columns, or 160 / 144 where a narrower tile's better
// filled last wave outweighs its higher operand traffic per MAC.  Per 128-byte
// k block a CTA spends about max(2.78 cycles per column, (16 KB of A + 64 B
// per column of B) / 43 B per cycle): a fit to the pair kernel's measured
// rates.  The MMA alone needs 2.0 cycles per column; the 256-wide tile's
// ~712 cycles come from the SM's shared-memory port, which carries both the
// TMA writes and the MMA's operand reads.
int pick_tc2_bn(int64_t M, int64_t N, int clusters) {
    const int64_t mt = (M + kTc2BM - 1) / kTc2BM;
    auto cost = [&](int bn) {
        const int64_t tiles = mt * ((N + bn - 1) / bn);
        const int64_t waves = (tiles + clusters - 1) / clusters;
        const double kblock = std::max(2.78 * bn, (16384.0 + 64.0 * bn) / 43.0);
        return (double)waves * kblock;
    };
    int best = 256;
    for (int bn : {160, 144})
        if (cost(bn) < cost(best)) best = bn;
    return best;
}

// Group-128 GEMM on pair tiles (256 x 128).
int launch_tc2_g128(const int8_t* A, const int8_t* B, TcParams p, cudaStream_t st) {
    using SM = Tc2gSmem;
    auto kern = gemm_i8_tc2_g128_kernel;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    static int max_clusters[kMaxDevices] = {0};
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kTc2gThreads, 1, 1);
    cfg.dynamicSmemBytes = SM::kBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (max_clusters[dev] == 0) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes) != cudaSuccess)
            return W8A8_ERR_CUDA;
        cfg.gridDim = dim3((unsigned)(2 * (device_sms(dev) / 2)), 1, 1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = device_sms(dev) / 2;
        max_clusters[dev] = n;
    }
    CUtensorMap ta, tb;
    if (!make_tmap_i8(&ta, A, (uint64_t)p.M, (uint64_t)p.K, 128)) return W8A8_ERR_CUDA;
    if (!make_tmap_i8(&tb, B, (uint64_t)p.N, (uint64_t)p.K, kTc2gBN / 2)) return W8A8_ERR_CUDA;
    p.num_m_tiles = (p.M + kTc2BM - 1) / kTc2BM;
    p.num_n_tiles = (p.N + kTc2gBN - 1) / kTc2gBN;
    p.num_k_blocks = (p.K + kTcBK - 1) / kTcBK;
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    const int clusters = tiles < max_clusters[dev] ? tiles : max_clusters[dev];
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, p));
}

template <int EPI>
int launch_tc2(const int8_t* A, const int8_t* B, TcParams p, cudaStream_t st) {
    const int bn = pick_tc2_bn(p.M, p.N, current_sms() / 2);
    return bn == 160 ? launch_tc2_bn<EPI, 160>(A, B, p, st)
         : bn == 144 ? launch_tc2_bn<EPI, 144>(A, B, p, st)
                     : launch_tc2_bn<EPI, 256>(A, B, p, st);
}

// Tile width: the one with less work in its last wave (256 on ties).
int pick_bn(int64_t M, int64_t N, int sms) {
    const int64_t mt = (M + kTcBM - 1) / kTcBM;
    const int64_t w256 = (mt * ((N + 255) / 256) + sms - 1) / sms;
    const int64_t w128 = (mt * ((N + 127) / 128) + sms - 1) / sms;
    return (w128 * 128 < w256 * 256) ? 128 : 256;
}

// Token counts from which the pair-tile kernel is used.
constexpr int64_t kTc2MinM = 256;

int run_tc(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, void* out, int64_t M, int64_t N,
           int64_t K, int epi, cudaStream_t st) {
    TcParams p = {};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.sx = sx;
    p.sw = sw;
    p.out = out;
    if (M >= kTc2MinM) return epi == kEpiBf16 ? launch_tc2<kEpiBf16>(qx, qw, p, st) : launch_tc2<kEpiS32>(qx, qw, p, st);
    const int bn = pick_bn(M, N, current_sms());
    if (epi == kEpiBf16)
        return bn == 256 ? launch_tc<256, 4, kEpiBf16, 2>(qx, qw, p, st) : launch_tc<128, 6, kEpiBf16, 2>(qx, qw, p, st);
    return bn == 256 ? launch_tc<256, 4, kEpiS32, 2>(qx, qw, p, st) : launch_tc<128, 6, kEpiS32, 2>(qx, qw, p, st);
}

// ----------------------------------------------------------------- GEMV
// Decode GEMV.  M <= 8: the register-streaming mma.sync kernel
// (gemv_dense_kernel): WN row blocks of 16 rows x WK = 8 / WN K-slices per
// CTA, 4 chunks of weight loads in flight per thread, 64 registers so that
// 4 CTAs (32 warps) stay resident per SM.  WN is the largest of 4, 2, 1 that
// still gives at least half a wave of CTAs (296 on 148 SMs); only when even
// 16-row CTAs do not reach that is the K range also split over `nkseg` CTAs
// (partials in the workspace), until the CTAs fill about 70% of the slots.
// The GEMV lets the next kernel launch at once when its own CTAs fill most
// of the SM slots (the wide gate_up shapes); measured on the decode step of
// the dense MLP shapes with two weight sets alternating (gate_up 4 x 2
// warps, 544 CTAs, early launch; down 1 x 8 warps, 320 CTAs, no split, no
// early launch: 54.1 us a step against 61.8 us for a 5-way split of 4 x 2
// warps).  9 <= M <= 32: the swap-AB tcgen05 kernel (gemv_tc_kernel), whose
// token columns grow for free.  Plans are fixed per shape (independent of
// the device) so that workspace sizes are too.
struct GemvPlan {
    bool tc;           // tcgen05 swap-AB kernel
    // register kernel
    int tg;            // token groups of 8
    int wn;            // row blocks per CTA (4, 2 or 1; 8 / wn warps along K)
    int ctas_x;        // CTAs along the rows
    int nkseg;         // CTAs along K
    int trig;          // early launch of the next kernel
    // tcgen05 kernel
    int bn, grid, ngroups, nkb;
    size_t part_bytes;
    int counters;
};

constexpr int kGemvUnrollDecode = 4, kGemvMinBlocks = 4;
constexpr int kGemvGrid = 148;
constexpr int kGemvMaxM = 32;

GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K) {
    GemvPlan g = {};
    g.tc = M > 8;
    if (!g.tc) {
        g.tg = 1;
        const int64_t blocks = (N + 15) / 16;
        const int64_t slots = (int64_t)kGemvGrid * kGemvMinBlocks;
        int wn = 4;
        while (wn > 1 && (blocks + wn - 1) / wn * 2 < slots) wn /= 2;
        g.wn = wn;
        const int wk = 8 / wn;
        g.ctas_x = (int)((blocks + wn - 1) / wn);
        const int64_t nchunks = (K + 63) / 64;
        int s = 1;
        while ((int64_t)g.ctas_x * 2 < slots && s < 16 && (int64_t)g.ctas_x * (s + 1) * 10 <= slots * 7 &&
               nchunks / (wk * (s + 1)) >= 8)
            ++s;
        g.nkseg = s;
        g.trig = (int64_t)g.ctas_x * s * 4 >= slots * 3 ? 1 : 0;
        g.part_bytes = s > 1 ? align_up((size_t)s * blocks * g.tg * 32 * 16, 256) : 0;
        g.counters = s > 1 ? g.ctas_x : 0;
    } else {
        g.bn = M <= 16 ? 16 : 32;
        g.ngroups = (int)((N + kGcBM - 1) / kGcBM);
        g.nkb = (int)((K + kGcBK - 1) / kGcBK);
        const int64_t units = (int64_t)g.ngroups * g.nkb;
        g.grid = (int)(units < kGemvGrid ? units : kGemvGrid);
        g.part_bytes = align_up((size_t)g.grid * 2 * kGcBM * g.bn * 4, 256);
        g.counters = g.ngroups * 4;
    }
    return g;
}

int gemv_counter_count(const GemvPlan& g) { return g.counters; }

size_t gemv_ws_bytes(const GemvPlan& g) { return g.part_bytes + align_up((size_t)g.counters * 4, 256); }

int* gemv_counters(const GemvPlan& g, void* scratch) {
    return g.counters ? reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(scratch) + g.part_bytes) : nullptr;
}

// Launch attribute: right after this library's activation-quant kernel (whose
// inputs were complete before it started), the weight stream may begin while
// that kernel finishes; codes, scales and counters are read only after it.
// Otherwise plain stream order.
void pdl_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* at, bool after_quant) {
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = after_quant ? 1 : 0;
}

template <int BN>
int launch_gemv_tc(const int8_t* qx, const int8_t* qw, const GemvTc& a, const GemvPlan& g, bool after_quant,
                   cudaStream_t st) {
    using SM = GcSmem<BN>;
    auto kern = gemv_tc_kernel<BN>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    static bool attr_done[kMaxDevices] = {false};
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes) != cudaSuccess)
            return W8A8_ERR_CUDA;
        attr_done[dev] = true;
    }
    CUtensorMap tw, tx;
    if (!make_tmap_i8(&tw, qw, (uint64_t)a.N, (uint64_t)a.K, kGcBM)) return W8A8_ERR_CUDA;
    if (!make_tmap_i8(&tx, qx, (uint64_t)a.M, (uint64_t)a.K, BN)) return W8A8_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.grid, 1, 1);
    cfg.blockDim = dim3(kGcThreads, 1, 1);
    cfg.dynamicSmemBytes = SM::kBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    pdl_config(cfg, at, after_quant);
    GemvTc args = a;
    args.prefetch_w = after_quant ? 1 : 0;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, tw, tx, args));
}

template <int TG, int U>
int launch_gemv_reg(const GemvShape& a, const GemvEpiDense& e, const GemvPlan& g, bool after_quant, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.ctas_x, (unsigned)g.nkseg, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    pdl_config(cfg, at, after_quant);
    GemvShape args = a;
    args.trig = g.trig;
    auto kern = g.wn == 4 ? gemv_dense_kernel<4, 2, TG, U, kGemvMinBlocks>
              : g.wn == 2 ? gemv_dense_kernel<2, 4, TG, U, kGemvMinBlocks>
                          : gemv_dense_kernel<1, 8, TG, U, kGemvMinBlocks>;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, args, e));
}

// gate_up GEMV of the dense MLP block, gated epilogue (same plan as the dense GEMV).
int launch_gemv_gated(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, float* a_out, int64_t M,
                      int64_t I, int64_t K, const GemvPlan& g, void* scratch, bool after_quant, cudaStream_t st) {
    GemvShape a;
    a.w = qw;
    a.x = qx;
    a.tokens = (int)M;
    a.rows = (int)(2 * I);
    a.K = (int)K;
    a.nchunks = (int)((K + 63) / 64);
    a.part = reinterpret_cast<int32_t*>(scratch);
    a.counters = gemv_counters(g, scratch);
    a.trig = g.trig;
    GemvEpiGated e;
    e.sx = sx;
    e.sw = sw;
    e.a = a_out;
    e.M = (int)M;
    e.I = (int)I;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.ctas_x, (unsigned)g.nkseg, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    pdl_config(cfg, at, after_quant);
    auto kern = g.wn == 4 ? gemv_gated_kernel<4, 2, 1, kGemvUnrollDecode, kGemvMinBlocks>
              : g.wn == 2 ? gemv_gated_kernel<2, 4, 1, kGemvUnrollDecode, kGemvMinBlocks>
                          : gemv_gated_kernel<1, 8, 1, kGemvUnrollDecode, kGemvMinBlocks>;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, a, e));
}

// Runs the GEMV; `scratch` holds the partials and the counters (zero on entry).
int run_gemv(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, void* out, int64_t M, int64_t N,
             int64_t K, bool s32, const GemvPlan& g, void* scratch, bool after_quant, cudaStream_t st) {
    if (!g.tc) {
        GemvShape a;
        a.w = qw;
        a.x = qx;
        a.tokens = (int)M;
        a.rows = (int)N;
        a.K = (int)K;
        a.nchunks = (int)((K + 63) / 64);
        a.part = reinterpret_cast<int32_t*>(scratch);
        a.counters = gemv_counters(g, scratch);
        GemvEpiDense e;
        e.sx = sx;
        e.sw = sw;
        e.out = out;
        e.M = (int)M;
        e.N = (int)N;
        e.s32 = s32 ? 1 : 0;
        return launch_gemv_reg<1, kGemvUnrollDecode>(a, e, g, after_quant, st);
    }
    GemvTc a;
    a.sx = sx;
    a.sw = sw;
    a.out = out;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.ngroups = g.ngroups;
    a.nkb = g.nkb;
    a.s32 = s32 ? 1 : 0;
    a.part = reinterpret_cast<int*>(scratch);
    a.counters = gemv_counters(g, scratch);
    a.prefetch_w = 0;
    if (g.bn == 16) return launch_gemv_tc<16>(qx, qw, a, g, after_quant, st);
    return launch_gemv_tc<32>(qx, qw, a, g, after_quant, st);
}

bool gemm_shape_ok(int64_t M, int64_t N, int64_t K) {
    return M > 0 && N > 0 && K > 0 && K % 16 == 0 && N % 8 == 0 && M <= (1 << 30) && N <= (1 << 30) &&
           K <= (1 << 30);
}

// ----------------------------------------------------------------- misc kernels
__global__ void exp_proj_kernel(const float* x, float* y, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = exp_proj(x[i]);
}

constexpr int kKernelIdDebugWait = 9;

__global__ void debug_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);   // one arrival expected; nobody arrives
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait_bounded(&bar, 0u, &abort_flag, (kKernelIdDebugWait << 16) | 1, limit_ns);
}

}  // namespace

// ----------------------------------------------------------------- MoE
namespace {
struct MoeWs {
    int32_t* ids;
    float* wts;
    int32_t* counts;
    int32_t* offsets;
    int32_t* active;
    int32_t* n_active;
    int32_t* tile_off;
    int32_t* rank;
    int32_t* done;
    int32_t* row_of;
    int32_t* row_tok;
    int32_t* row_slot;
    float* row_w;
    int8_t* xq;
    float* sxr;
    float* a;
    int8_t* qa;
    float* sa;
    float* out;
    size_t bytes;
};

// The combine sums each token's k contributions in slot order -- the same
// fp32 steps as the definition -- while the [T * k, H] contribution buffer
// fits comfortably in L2; beyond that it accumulates with fp32 vector atomics
// into [T, H] (order unspecified).
constexpr size_t kMoeExactCombineBytes = (size_t)64 << 20;
std::atomic<int> g_moe_combine{W8A8_MOE_COMBINE_AUTO};
inline bool moe_exact_combine(int64_t R, int H) {
    return g_moe_combine.load(std::memory_order_relaxed) == W8A8_MOE_COMBINE_EXACT ||
           (size_t)R * H * 4 <= kMoeExactCombineBytes;
}

// Token blocks of the swap path: at most one partial block per touched expert.
inline int64_t moe_max_blocks(int64_t R, int E, int bn) { return R / bn + (R < E ? R : E) + 1; }

MoeWs moe_carve(void* base, int64_t T, int E, int H, int I, int topk) {
    MoeWs w;
    const int64_t R = T * topk;
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        uint8_t* r = p ? p + o : nullptr;
        o += align_up(bytes, 256);
        return r;
    };
    w.ids = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.wts = reinterpret_cast<float*>(take((size_t)R * 4));
    // counts and the plan's CTA counter are adjacent: one memset clears both
    w.counts = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
    w.done = w.counts + E;
    w.offsets = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
    w.active = reinterpret_cast<int32_t*>(take((size_t)E * 4));
    w.n_active = reinterpret_cast<int32_t*>(take(4));
    w.tile_off = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
    w.rank = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_of = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_tok = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_slot = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_w = reinterpret_cast<float*>(take((size_t)R * 4));
    w.xq = reinterpret_cast<int8_t*>(take((size_t)R * H));
    w.sxr = reinterpret_cast<float*>(take((size_t)R * 4));
    w.a = reinterpret_cast<float*>(take((size_t)R * I * 4));
    w.qa = reinterpret_cast<int8_t*>(take((size_t)R * I));
    w.sa = reinterpret_cast<float*>(take((size_t)R * 4));
    // w * y2 at (token, slot), or the atomically combined [T, H] for large T
    w.out = reinterpret_cast<float*>(take(moe_exact_combine(R, H) ? (size_t)R * H * 4 : (size_t)T * H * 4));
    w.bytes = o;
    return w;
}

// Dense gated MLP block workspace: x codes and scales, the fp32 gated
// intermediate, its codes and scales, and (decode) the two GEMVs' split-K
// partials and counters.
struct MlpWs {
    int8_t* qx;
    float* sx;
    float* a;
    int8_t* qa;
    float* sa;
    void* scratch1;
    void* scratch2;
    size_t bytes;
};

MlpWs mlp_carve(void* base, int64_t M, int64_t H, int64_t I) {
    MlpWs w;
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        uint8_t* r = p ? p + o : nullptr;
        o += align_up(bytes, 256);
        return r;
    };
    w.qx = reinterpret_cast<int8_t*>(take((size_t)(M * H)));
    w.sx = reinterpret_cast<float*>(take((size_t)M * 4));
    w.a = reinterpret_cast<float*>(take((size_t)(M * I) * 4));
    w.qa = reinterpret_cast<int8_t*>(take((size_t)(M * I)));
    w.sa = reinterpret_cast<float*>(take((size_t)M * 4));
    w.scratch1 = w.scratch2 = nullptr;
    if (M <= 8) {
        w.scratch1 = take(gemv_ws_bytes(gemv_plan(M, 2 * I, H)));
        w.scratch2 = take(gemv_ws_bytes(gemv_plan(M, H, I)));
    }
    w.bytes = o;
    return w;
}

// Grouped tcgen05 GEMM over the expert-sorted rows: A = sorted codes
// [R, K], B = the experts' weights viewed as [E * N, K].
template <int EPI>
int launch_tc_grouped(const int8_t* A, int64_t rowsA, const int8_t* B, int E, TcParams p, cudaStream_t st) {
    constexpr int BN = 256, STAGES = 4, NEPI = 8;
    using SM = TcSmem<BN, STAGES>;
    auto kern = gemm_i8_tc_kernel<BN, STAGES, EPI, 2, true, NEPI>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    static bool attr_done[kMaxDevices] = {false};
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes) != cudaSuccess)
            return W8A8_ERR_CUDA;
        attr_done[dev] = true;
    }
    CUtensorMap ta, tb;
    if (!make_tmap_i8(&ta, A, (uint64_t)rowsA, (uint64_t)p.K, kTcBM)) return W8A8_ERR_CUDA;
    if (!make_tmap_i8(&tb, B, (uint64_t)E * p.N, (uint64_t)p.K, BN)) return W8A8_ERR_CUDA;
    p.E = E;
    p.num_m_tiles = 0;
    p.num_n_tiles = (p.N + BN - 1) / BN;
    p.num_k_blocks = (p.K + kTcBK - 1) / kTcBK;
    kern<<<device_sms(dev), tc_threads<NEPI>(), SM::kBytes, st>>>(ta, tb, p);
    return last_launch_status();
}

// Swap-AB expert GEMM over token blocks of BN rows: W = an expert stack
// viewed as [E * rows, K], X = the sorted codes [R, K].
template <int BN, bool GATED, bool G128 = false>
int launch_moe_swap(const int8_t* W, const int8_t* X, int64_t R, MoeSwapArgs a, int64_t nb_max, cudaStream_t st) {
    using SM = MsSmem<BN, G128>;
    auto kern = moe_swap_kernel<BN, GATED, G128>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    static bool attr_done[kMaxDevices] = {false};
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes) != cudaSuccess)
            return W8A8_ERR_CUDA;
        attr_done[dev] = true;
    }
    CUtensorMap tw, tx;
    if (!make_tmap_i8(&tw, W, (uint64_t)a.E * a.rows, (uint64_t)a.K, kMsBM)) return W8A8_ERR_CUDA;
    if (!make_tmap_i8(&tx, X, (uint64_t)R, (uint64_t)a.K, BN)) return W8A8_ERR_CUDA;
    const int64_t units = nb_max * a.ngroups;
    const int sms = device_sms(dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units < sms ? units : sms), 1, 1);
    cfg.blockDim = dim3(ms_threads<G128>(), 1, 1);
    cfg.dynamicSmemBytes = SM::kBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    pdl_config(cfg, at, true);
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, tw, tx, a));
}

// A plain kernel launch on the MoE chain, with programmatic dependent launch.
template <typename... KArgs, typename... Args>
int launch_chained_smem(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                        Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    pdl_config(cfg, at, true);
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, args...));
}

template <typename... KArgs, typename... Args>
int launch_chained(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    pdl_config(cfg, at, true);
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, args...));
}

template <int WN, int WK, int TG, bool GATED>
int launch_moe_gemm(const MoeGemmArgs& m, int ctas_x, int max_active, cudaStream_t st) {
    dim3 grid((unsigned)ctas_x, (unsigned)max_active, 1);
    moe_gemm_kernel<WN, WK, TG, GATED><<<grid, kGemvThreads, 0, st>>>(m);
    return last_launch_status();
}
}  // namespace

// =====================================================================================
extern "C" {

const char* w8a8_version(void) { return "w8a8 sm_100a 0.1"; }

const char* w8a8_status_str(int status) {
    switch (status) {
        case W8A8_OK:
            return "ok";
        case W8A8_ERR_INVALID_ARG:
            return "invalid argument";
        case W8A8_ERR_WORKSPACE:
            return "workspace too small";
        case W8A8_ERR_UNSUPPORTED:
            return "unsupported shape";
        case W8A8_ERR_CUDA:
            return "CUDA error";
        case W8A8_ERR_TIMEOUT:
            return "device wait timed out";
        default:
            return "unknown status";
    }
}

int w8a8_quant_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s, void* stream) {
    if (!x || !q || !s || M <= 0 || K <= 0 || K % 16 != 0 || ldx < K || ldx % 8 != 0) return W8A8_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4)) return W8A8_ERR_INVALID_ARG;
    if (K / 8 > (int64_t)8 * 256 * kQuantMaxVec) return W8A8_ERR_UNSUPPORTED;
    cudaError_t e = launch_quant_rows<uint16_t>(x, M, K, ldx, q, K, s, (cudaStream_t)stream, current_sms());
    return cuda_status(e);
}

int w8a8_quant_rows_f32(const float* w, int64_t N, int64_t K, int8_t* q, float* s, void* stream) {
    if (!w || !q || !s || N <= 0 || K <= 0 || K % 16 != 0) return W8A8_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(q, 16) || !aligned(s, 4)) return W8A8_ERR_INVALID_ARG;
    if (K / 4 > (int64_t)8 * 256 * kQuantMaxVec) return W8A8_ERR_UNSUPPORTED;
    cudaError_t e = launch_quant_rows<float>(w, N, K, K, q, K, s, (cudaStream_t)stream, current_sms());
    return cuda_status(e);
}

size_t w8a8_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    size_t b = align_up((size_t)M * K, 256) + align_up((size_t)M * 4, 256);
    if (M <= 8) b += gemv_ws_bytes(gemv_plan(M, N, K));
    return b;
}

int w8a8_linear(const uint16_t* x, const int8_t* qw, const float* sw, uint16_t* y, int64_t M, int64_t N, int64_t K,
                void* ws, size_t ws_bytes, void* stream) {
    if (!x || !qw || !sw || !y || !ws) return W8A8_ERR_INVALID_ARG;
    if (!gemm_shape_ok(M, N, K)) return W8A8_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(qw, 16) || !aligned(sw, 16) || !aligned(y, 16) || !aligned(ws, 256))
        return W8A8_ERR_INVALID_ARG;
    if (ws_bytes < w8a8_linear_workspace_size(M, N, K)) return W8A8_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    int8_t* qx = reinterpret_cast<int8_t*>(ws);
    float* sx = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + align_up((size_t)M * K, 256));
    void* scratch = reinterpret_cast<uint8_t*>(sx) + align_up((size_t)M * 4, 256);
    const bool gemv = M <= 8;
    GemvPlan g = gemv_plan(M, N, K);
    int* ctr = gemv ? gemv_counters(g, scratch) : nullptr;
    if (K / 8 > (int64_t)8 * 256 * kQuantMaxVec) return W8A8_ERR_UNSUPPORTED;
    cudaError_t e =
        launch_quant_rows<uint16_t>(x, M, K, K, qx, K, sx, st, current_sms(), ctr, ctr ? gemv_counter_count(g) : 0,
                                    true);
    if (e != cudaSuccess) return W8A8_ERR_CUDA;
    if (gemv) return run_gemv(qx, sx, qw, sw, y, M, N, K, false, g, scratch, true, st);
    return run_tc(qx, sx, qw, sw, y, M, N, K, kEpiBf16, st);
}

// ----------------------------------------------------------------- linear without caller workspace
// Some callers cannot allocate device memory at the point where they run the
// layer (an allocator that is locked while a step runs, a plugin host that
// only hands over its input and output buffers, code that must not touch the
// allocator's state).  For them w8a8_linear_noalloc keeps w8a8_linear's
// scratch -- the activation codes and scales and the GEMV's split-K partials
// and arrival counters -- in this file-scope device array instead of a
// caller-provided workspace.  Every GPU that loads the library holds the array
// until the process exits.
static __device__ __align__(256) uint8_t g_linear_noalloc_scratch[W8A8_NOALLOC_SCRATCH_BYTES];

}  // extern "C"

namespace {
// Device address of g_linear_noalloc_scratch, looked up once per device with
// that device current (the host-side symbol is only a stand-in, never a
// device address).
uint8_t* noalloc_scratch_ptr(int dev) {
    static uint8_t* ptrs[kMaxDevices] = {nullptr};
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_linear_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
        ptrs[dev] = reinterpret_cast<uint8_t*>(p);
    }
    return ptrs[dev];
}
}  // namespace

extern "C" {

size_t w8a8_linear_noalloc_scratch_size(int64_t M, int64_t N, int64_t K) {
    return w8a8_linear_workspace_size(M, N, K);
}

int w8a8_linear_noalloc(const uint16_t* x, const int8_t* qw, const float* sw, uint16_t* y, int64_t M, int64_t N,
                        int64_t K, void* stream) {
    if (!x || !qw || !sw || !y) return W8A8_ERR_INVALID_ARG;
    if (!gemm_shape_ok(M, N, K)) return W8A8_ERR_INVALID_ARG;
    if (w8a8_linear_workspace_size(M, N, K) > (size_t)W8A8_NOALLOC_SCRATCH_BYTES) return W8A8_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED;
    uint8_t* scratch = noalloc_scratch_ptr(dev);
    if (scratch == nullptr) return W8A8_ERR_CUDA;
    // The same kernels as w8a8_linear, on the static scratch; the quant kernel
    // clears the split-K counters each call, so earlier contents do not matter.
    return w8a8_linear(x, qw, sw, y, M, N, K, scratch, (size_t)W8A8_NOALLOC_SCRATCH_BYTES, stream);
}

size_t w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int path) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    const bool gemv = (path == W8A8_PATH_GEMV) || (path == W8A8_PATH_AUTO && M <= 8);
    if (!gemv) return 0;
    return gemv_ws_bytes(gemv_plan(M, N, K));
}

static int gemm_common(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, void* out, int64_t M,
                       int64_t N, int64_t K, int path, void* ws, size_t ws_bytes, bool s32, cudaStream_t st) {
    if (!qx || !qw || !out) return W8A8_ERR_INVALID_ARG;
    if (!s32 && (!sx || !sw)) return W8A8_ERR_INVALID_ARG;
    if (!gemm_shape_ok(M, N, K)) return W8A8_ERR_INVALID_ARG;
    if (!aligned(qx, 16) || !aligned(qw, 16) || !aligned(out, 16)) return W8A8_ERR_INVALID_ARG;
    if (!s32 && (!aligned(sx, 4) || !aligned(sw, 16))) return W8A8_ERR_INVALID_ARG;
    if (path < W8A8_PATH_AUTO || path > W8A8_PATH_GEMV) return W8A8_ERR_INVALID_ARG;
    const bool gemv = (path == W8A8_PATH_GEMV) || (path == W8A8_PATH_AUTO && M <= 8);
    if (gemv) {
        if (M > kGemvMaxM) return W8A8_ERR_UNSUPPORTED;
        GemvPlan g = gemv_plan(M, N, K);
        const size_t need = gemv_ws_bytes(g);
        if (g.counters > 0) {
            if (!ws || !aligned(ws, 256)) return W8A8_ERR_INVALID_ARG;
            if (ws_bytes < need) return W8A8_ERR_WORKSPACE;
            if (cudaMemsetAsync(gemv_counters(g, ws), 0, (size_t)gemv_counter_count(g) * 4, st) != cudaSuccess)
                return W8A8_ERR_CUDA;
        }
        return run_gemv(qx, sx, qw, sw, out, M, N, K, s32, g, ws, false, st);
    }
    return run_tc(qx, sx, qw, sw, out, M, N, K, s32 ? kEpiS32 : kEpiBf16, st);
}

int w8a8_gemm_q(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, uint16_t* y, int64_t M,
                int64_t N, int64_t K, int path, void* ws, size_t ws_bytes, void* stream) {
    return gemm_common(qx, sx, qw, sw, y, M, N, K, path, ws, ws_bytes, false, (cudaStream_t)stream);
}

int w8a8_gemm_s32(const int8_t* qx, const int8_t* qw, int32_t* acc, int64_t M, int64_t N, int64_t K, int path,
                  void* ws, size_t ws_bytes, void* stream) {
    return gemm_common(qx, nullptr, qw, nullptr, acc, M, N, K, path, ws, ws_bytes, true, (cudaStream_t)stream);
}


}  // extern "C"

namespace {
// Optional parity outputs of the MoE forward (a debug struct given by the caller).
int moe_debug_copies(const MoeWs& w, const w8a8_moe_debug* dbg, int64_t R, int E, int I, cudaStream_t st) {
    if (!dbg) return W8A8_OK;
    if (dbg->topk_ids && cudaMemcpyAsync(dbg->topk_ids, w.ids, (size_t)R * 4, cudaMemcpyDeviceToDevice, st))
        return W8A8_ERR_CUDA;
    if (dbg->topk_w && cudaMemcpyAsync(dbg->topk_w, w.wts, (size_t)R * 4, cudaMemcpyDeviceToDevice, st))
        return W8A8_ERR_CUDA;
    if (dbg->counts && cudaMemcpyAsync(dbg->counts, w.counts, (size_t)E * 4, cudaMemcpyDeviceToDevice, st))
        return W8A8_ERR_CUDA;
    if (dbg->qa || dbg->sa) {
        moe_debug_gather_kernel<<<(unsigned)R, 128, 0, st>>>(w.qa, w.sa, w.row_of, R, I, dbg->qa, dbg->sa);
        return last_launch_status();
    }
    return W8A8_OK;
}
}  // namespace

extern "C" {

int w8a8_moe_set_combine(int mode) {
    if (mode != W8A8_MOE_COMBINE_AUTO && mode != W8A8_MOE_COMBINE_EXACT) return W8A8_ERR_INVALID_ARG;
    return g_moe_combine.exchange(mode);
}

size_t w8a8_moe_workspace_size(int64_t T, int E, int H, int I, int topk) {
    if (T <= 0 || E <= 0 || H <= 0 || I <= 0 || topk <= 0) return 0;
    return moe_carve(nullptr, T, E, H, I, topk).bytes;
}

int w8a8_moe_forward(const uint16_t* x, const uint16_t* logits, const int8_t* w13, const float* s13,
                     const int8_t* w2, const float* s2, uint16_t* y, int64_t T, int E, int H, int I, int topk,
                     void* ws, size_t ws_bytes, const w8a8_moe_debug* dbg, void* stream) {
    if (!x || !logits || !w13 || !s13 || !w2 || !s2 || !y || !ws) return W8A8_ERR_INVALID_ARG;
    if (T <= 0 || E <= 0 || H <= 0 || I <= 0 || topk <= 0 || topk > E || topk > kMoeMaxTopk) return W8A8_ERR_INVALID_ARG;
    if (E > 256) return W8A8_ERR_UNSUPPORTED;
    if (H % 64 != 0 || I % 64 != 0 || H > 8192 || I > 8192) return W8A8_ERR_UNSUPPORTED;
    if (T * topk > (int64_t)1 << 30 || T > 0x7fffffffLL) return W8A8_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(logits, 2) || !aligned(w13, 16) || !aligned(s13, 4) || !aligned(w2, 16) ||
        !aligned(s2, 4) || !aligned(y, 16) || !aligned(ws, 256))
        return W8A8_ERR_INVALID_ARG;
    if (ws_bytes < w8a8_moe_workspace_size(T, E, H, I, topk)) return W8A8_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    MoeWs w = moe_carve(ws, T, E, H, I, topk);
    const int64_t R = T * topk;
    int rc;

    const bool exact_combine = moe_exact_combine(R, H);
    // up to a few dozen rows per expert: swap-AB expert GEMMs with the requant
    // and the combine fused in (weights streamed once per token block)
    const int64_t avg_rows = (R + E - 1) / E;
    const bool swap = exact_combine && H % 128 == 0 && I % 128 == 0 && I <= 2048 && avg_rows <= 64;
    const int swap_bn = avg_rows <= 12 ? 16 : (avg_rows <= 24 ? 32 : 64);
    MoePlan plan = {w.counts, w.offsets, w.active, w.n_active, w.tile_off, w.rank, w.done, swap ? swap_bn : 128};
    MoeRows rows = {w.ids, w.wts, w.rank, w.offsets, w.row_of, w.row_tok, w.row_slot, w.row_w};
    const bool front_small = T <= kMoeFrontMaxT && exact_combine;
    if (front_small) {
        // routing, plan and x codes in one CTA
        moe_front_small_kernel<8><<<1, 512, 0, st>>>(x, logits, (int)T, E, H, topk, w.ids, w.wts, plan, rows, w.xq,
                                                     w.sxr, dbg ? dbg->qx : nullptr, dbg ? dbg->sx : nullptr);
        if ((rc = last_launch_status()) != W8A8_OK) return rc;
    } else {
        if (cudaMemsetAsync(w.counts, 0, (size_t)(E + 1) * 4, st) != cudaSuccess) return W8A8_ERR_CUDA;
        moe_route_plan_kernel<8><<<(unsigned)((T + 7) / 8), 256, 0, st>>>(logits, T, E, topk, w.ids, w.wts, plan);
        if ((rc = last_launch_status()) != W8A8_OK) return rc;
        rc = launch_chained(moe_quant_scatter_kernel, (unsigned)T, (unsigned)((H / 8 + 31) / 32 * 32), st, x, H,
                            topk, rows, w.xq, w.sxr, exact_combine ? (float*)nullptr : w.out,
                            dbg ? dbg->qx : (int8_t*)nullptr, dbg ? dbg->sx : (float*)nullptr);
        if (rc != W8A8_OK) return rc;
    }

    if (swap) {
        const int64_t nb_max = moe_max_blocks(R, E, swap_bn);
        MoeSwapArgs a1 = {};
        a1.sw = s13;
        a1.sx = w.sxr;
        a1.counts = w.counts;
        a1.offsets = w.offsets;
        a1.tile_off = w.tile_off;
        a1.E = E;
        a1.rows = 2 * I;
        a1.K = H;
        a1.ngroups = (2 * I) / 128;
        a1.nkb = H / 128;
        a1.a_out = w.a;
        a1.early_plan = front_small ? 0 : 1;   // after the front kernel the plan is one kernel back
        MoeSwapArgs a2 = a1;
        a2.early_plan = 1;
        a2.sw = s2;
        a2.sx = w.sa;
        a2.rows = H;
        a2.K = I;
        a2.ngroups = H / 128;
        a2.nkb = I / 128;
        a2.row_tok = w.row_tok;
        a2.row_slot = w.row_slot;
        a2.row_w = w.row_w;
        a2.contrib = w.out;
        a2.topk = topk;
        rc = swap_bn == 16 ? launch_moe_swap<16, true>(w13, w.xq, R, a1, nb_max, st)
           : swap_bn == 32 ? launch_moe_swap<32, true>(w13, w.xq, R, a1, nb_max, st)
                           : launch_moe_swap<64, true>(w13, w.xq, R, a1, nb_max, st);
        if (rc != W8A8_OK) return rc;
        if (launch_quant_rows<float>(w.a, R, I, I, w.qa, I, w.sa, st, current_sms(), nullptr, 0, true) != cudaSuccess)
            return W8A8_ERR_CUDA;
        rc = swap_bn == 16 ? launch_moe_swap<16, false>(w2, w.qa, R, a2, nb_max, st)
           : swap_bn == 32 ? launch_moe_swap<32, false>(w2, w.qa, R, a2, nb_max, st)
                           : launch_moe_swap<64, false>(w2, w.qa, R, a2, nb_max, st);
        if (rc != W8A8_OK) return rc;
        rc = launch_chained(moe_finalize_kernel, (unsigned)((T * H / 4 + 255) / 256), 256u, st, (const float*)w.out,
                            y, T, H, topk);
        if (rc != W8A8_OK) return rc;
        return moe_debug_copies(w, dbg, R, E, I, st);
    }
    const int max_active = (int)(R < E ? R : E);
    const bool wide = R > (int64_t)E * 8;   // more than 8 rows per expert on average
    // many rows per expert: grouped tcgen05 GEMMs over 128-row tiles of each expert's rows
    const bool tiled = R >= (int64_t)E * 16 && (2 * I) % 256 == 0 && H % 256 == 0;
    if (tiled) {
        TcParams p1 = {};
        p1.N = 2 * I;
        p1.K = H;
        p1.M = (int)R;
        p1.sx = w.sxr;
        p1.sw = s13;
        p1.counts = w.counts;
        p1.offsets = w.offsets;
        p1.tile_off = w.tile_off;
        p1.a_out = w.a;
        if ((rc = launch_tc_grouped<kEpiMoeGated>(w.xq, R, w13, E, p1, st)) != W8A8_OK) return rc;
        cudaError_t e2 = launch_quant_rows<float>(w.a, R, I, I, w.qa, I, w.sa, st, current_sms());
        if (e2 != cudaSuccess) return W8A8_ERR_CUDA;
        TcParams p2 = {};
        p2.N = H;
        p2.K = I;
        p2.M = (int)R;
        p2.sx = w.sa;
        p2.sw = s2;
        p2.counts = w.counts;
        p2.offsets = w.offsets;
        p2.tile_off = w.tile_off;
        p2.row_tok = w.row_tok;
        p2.row_slot = w.row_slot;
        p2.row_w = w.row_w;
        p2.contrib = w.out;
        p2.topk = topk;
        rc = exact_combine ? launch_tc_grouped<kEpiMoeCombine>(w.qa, R, w2, E, p2, st)
                           : launch_tc_grouped<kEpiMoeCombineAtomic>(w.qa, R, w2, E, p2, st);
        if (rc != W8A8_OK) return rc;
    }
    MoeGemmArgs g1 = {};
    g1.w = w13;
    g1.sw = s13;
    g1.xq = w.xq;
    g1.sxr = w.sxr;
    g1.counts = w.counts;
    g1.offsets = w.offsets;
    g1.active = w.active;
    g1.n_active = w.n_active;
    g1.rows = 2 * I;
    g1.K = H;
    g1.a_out = w.a;
    if (!tiled) {
    rc = wide ? launch_moe_gemm<2, 4, 4, true>(g1, (2 * I) / 32, max_active, st)
              : launch_moe_gemm<2, 4, 1, true>(g1, (2 * I) / 32, max_active, st);
    if (rc != W8A8_OK) return rc;

    cudaError_t e = launch_quant_rows<float>(w.a, R, I, I, w.qa, I, w.sa, st, current_sms());
    if (e != cudaSuccess) return W8A8_ERR_CUDA;

    MoeGemmArgs g2 = {};
    g2.w = w2;
    g2.sw = s2;
    g2.xq = w.qa;
    g2.sxr = w.sa;
    g2.counts = w.counts;
    g2.offsets = w.offsets;
    g2.active = w.active;
    g2.n_active = w.n_active;
    g2.rows = H;
    g2.K = I;
    g2.row_tok = w.row_tok;
    g2.row_slot = w.row_slot;
    g2.row_w = w.row_w;
    g2.contrib = w.out;
    g2.topk = exact_combine ? topk : 0;
    rc = wide ? launch_moe_gemm<8, 1, 4, false>(g2, H / 128, max_active, st)
              : launch_moe_gemm<8, 1, 1, false>(g2, H / 128, max_active, st);
    if (rc != W8A8_OK) return rc;
    }

    const int64_t n = T * H;
    moe_finalize_kernel<<<(unsigned)((n / 4 + 255) / 256), 256, 0, st>>>(w.out, y, T, H, exact_combine ? topk : 1);
    if ((rc = last_launch_status()) != W8A8_OK) return rc;

    return moe_debug_copies(w, dbg, R, E, I, st);
}

// ----------------------------------------------------------------- dense gated MLP block
size_t w8a8_mlp_workspace_size(int64_t M, int64_t H, int64_t I) {
    if (M <= 0 || H <= 0 || I <= 0) return 0;
    return mlp_carve(nullptr, M, H, I).bytes;
}

int w8a8_mlp_forward(const uint16_t* x, const int8_t* w13, const float* s13, const int8_t* w2, const float* s2,
                     uint16_t* y, int64_t M, int64_t H, int64_t I, void* ws, size_t ws_bytes,
                     const w8a8_mlp_debug* dbg, void* stream) {
    if (!x || !w13 || !s13 || !w2 || !s2 || !y || !ws) return W8A8_ERR_INVALID_ARG;
    if (M <= 0 || H <= 0 || I <= 0 || H % 16 != 0 || I % 16 != 0) return W8A8_ERR_INVALID_ARG;
    if (!gemm_shape_ok(M, 2 * I, H) || !gemm_shape_ok(M, H, I)) return W8A8_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w13, 16) || !aligned(s13, 16) || !aligned(w2, 16) || !aligned(s2, 16) ||
        !aligned(y, 16) || !aligned(ws, 256))
        return W8A8_ERR_INVALID_ARG;
    if (H / 8 > (int64_t)8 * 256 * kQuantMaxVec || I / 4 > (int64_t)8 * 256 * kQuantMaxVec) return W8A8_ERR_UNSUPPORTED;
    if (ws_bytes < w8a8_mlp_workspace_size(M, H, I)) return W8A8_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const MlpWs w = mlp_carve(ws, M, H, I);
    const bool gemv = M <= 8;
    const GemvPlan g1 = gemv_plan(M, 2 * I, H), g2 = gemv_plan(M, H, I);
    int* ctr1 = gemv ? gemv_counters(g1, w.scratch1) : nullptr;
    int* ctr2 = gemv ? gemv_counters(g2, w.scratch2) : nullptr;
    int rc;
    // a1 (it also clears the gate_up GEMV's counters)
    if (launch_quant_rows<uint16_t>(x, M, H, H, w.qx, H, w.sx, st, current_sms(), ctr1, ctr1 ? g1.counters : 0,
                                    true) != cudaSuccess)
        return W8A8_ERR_CUDA;
    // gate_up GEMM with SiLU(gate) * up -> fp32 a [M, I]
    if (gemv) {
        rc = launch_gemv_gated(w.qx, w.sx, w13, s13, w.a, M, I, H, g1, w.scratch1, true, st);
    } else {
        TcParams p = {};
        p.M = (int)M;
        p.N = (int)(2 * I);
        p.K = (int)H;
        p.sx = w.sx;
        p.sw = s13;
        p.a_out = w.a;
        rc = M >= kTc2MinM ? launch_tc2<kEpiMoeGated>(w.qx, w13, p, st)
                           : launch_tc<256, 4, kEpiMoeGated, 2, 8>(w.qx, w13, p, st);
    }
    if (rc != W8A8_OK) return rc;
    // a9 (it also clears the down GEMV's counters)
    if (launch_quant_rows<float>(w.a, M, I, I, w.qa, I, w.sa, st, current_sms(), ctr2, ctr2 ? g2.counters : 0,
                                 true) != cudaSuccess)
        return W8A8_ERR_CUDA;
    // down GEMM with the dense dequant
    rc = gemv ? run_gemv(w.qa, w.sa, w2, s2, y, M, H, I, false, g2, w.scratch2, true, st)
              : run_tc(w.qa, w.sa, w2, s2, y, M, H, I, kEpiBf16, st);
    if (rc != W8A8_OK) return rc;
    if (dbg) {
        if (dbg->qx && cudaMemcpyAsync(dbg->qx, w.qx, (size_t)(M * H), cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        if (dbg->sx && cudaMemcpyAsync(dbg->sx, w.sx, (size_t)M * 4, cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        if (dbg->qa && cudaMemcpyAsync(dbg->qa, w.qa, (size_t)(M * I), cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        if (dbg->sa && cudaMemcpyAsync(dbg->sa, w.sa, (size_t)M * 4, cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
    }
    return W8A8_OK;
}

}  // extern "C"

// ----------------------------------------------------------------- MoE, FWHT128 grid
namespace {
struct MoeG128Ws {
    int32_t* ids;
    float* wts;
    int32_t* counts;
    int32_t* offsets;
    int32_t* active;
    int32_t* n_active;
    int32_t* tile_off;
    int32_t* rank;
    int32_t* done;
    int32_t* row_of;
    int32_t* row_tok;
    int32_t* row_slot;
    float* row_w;
    int8_t* xq;       // [R, H] rotated codes of x, expert-sorted rows
    uint16_t* sxg;    // [R, H / 128]
    float* a;         // [R, I] fp32 gated intermediate
    int8_t* qa;       // [R, I] its rotated codes
    uint16_t* sag;    // [R, I / 128]
    float* out;       // [R, H] w * y2 at (token, slot)
    size_t bytes;
};

MoeG128Ws moe_g128_carve(void* base, int64_t T, int E, int H, int I, int topk) {
    MoeG128Ws w;
    const int64_t R = T * topk;
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        uint8_t* r = p ? p + o : nullptr;
        o += align_up(bytes, 256);
        return r;
    };
    w.ids = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.wts = reinterpret_cast<float*>(take((size_t)R * 4));
    w.counts = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));   // counts and the plan's CTA counter
    w.done = w.counts + E;
    w.offsets = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
    w.active = reinterpret_cast<int32_t*>(take((size_t)E * 4));
    w.n_active = reinterpret_cast<int32_t*>(take(4));
    w.tile_off = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
    w.rank = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_of = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_tok = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_slot = reinterpret_cast<int32_t*>(take((size_t)R * 4));
    w.row_w = reinterpret_cast<float*>(take((size_t)R * 4));
    w.xq = reinterpret_cast<int8_t*>(take((size_t)R * H));
    w.sxg = reinterpret_cast<uint16_t*>(take((size_t)R * (H / 128) * 2));
    w.a = reinterpret_cast<float*>(take((size_t)R * I * 4));
    w.qa = reinterpret_cast<int8_t*>(take((size_t)R * I));
    w.sag = reinterpret_cast<uint16_t*>(take((size_t)R * (I / 128) * 2));
    w.out = reinterpret_cast<float*>(take((size_t)R * H * 4));
    w.bytes = o;
    return w;
}
}  // namespace

extern "C" {

size_t w8a8_moe_g128_workspace_size(int64_t T, int E, int H, int I, int topk) {
    if (T <= 0 || E <= 0 || H < 128 || I < 128 || topk <= 0) return 0;
    return moe_g128_carve(nullptr, T, E, H, I, topk).bytes;
}

int w8a8_moe_g128_forward(const uint16_t* x, const uint16_t* logits, const int8_t* w13, const uint16_t* s13,
                          const int8_t* w2, const uint16_t* s2, uint16_t* y, int64_t T, int E, int H, int I, int topk,
                          void* ws, size_t ws_bytes, const w8a8_moe_g128_debug* dbg, void* stream) {
    if (!x || !logits || !w13 || !s13 || !w2 || !s2 || !y || !ws) return W8A8_ERR_INVALID_ARG;
    if (T <= 0 || E <= 0 || H <= 0 || I <= 0 || topk <= 0 || topk > E || topk > kMoeMaxTopk) return W8A8_ERR_INVALID_ARG;
    if (E > 256) return W8A8_ERR_UNSUPPORTED;
    if (H % 128 != 0 || I % 128 != 0 || H > 128 * kMoeG128MaxGroupsH || I > 2048) return W8A8_ERR_UNSUPPORTED;
    if (T * topk > (int64_t)1 << 30 || T > 0x7fffffffLL) return W8A8_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(logits, 2) || !aligned(w13, 16) || !aligned(s13, 2) || !aligned(w2, 16) ||
        !aligned(s2, 2) || !aligned(y, 16) || !aligned(ws, 256))
        return W8A8_ERR_INVALID_ARG;
    if (ws_bytes < w8a8_moe_g128_workspace_size(T, E, H, I, topk)) return W8A8_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    MoeG128Ws w = moe_g128_carve(ws, T, E, H, I, topk);
    const int64_t R = T * topk;
    int rc;

    // token blocks of 16 / 32 / 64 expert-sorted rows, by the average rows per expert
    const int64_t avg_rows = (R + E - 1) / E;
    const int bn = avg_rows <= 12 ? 16 : (avg_rows <= 24 ? 32 : 64);
    MoePlan plan = {w.counts, w.offsets, w.active, w.n_active, w.tile_off, w.rank, w.done, bn};
    MoeRows rows = {w.ids, w.wts, w.rank, w.offsets, w.row_of, w.row_tok, w.row_slot, w.row_w};
    if (cudaMemsetAsync(w.counts, 0, (size_t)(E + 1) * 4, st) != cudaSuccess) return W8A8_ERR_CUDA;
    moe_route_plan_kernel<8><<<(unsigned)((T + 7) / 8), 256, 0, st>>>(logits, T, E, topk, w.ids, w.wts, plan);
    if ((rc = last_launch_status()) != W8A8_OK) return rc;
    rc = launch_chained(moe_fwht_scatter_kernel, (unsigned)T, (unsigned)(32 * (H / 128)), st, x, H, topk, rows, w.xq,
                        w.sxg, dbg ? dbg->qx : (int8_t*)nullptr, dbg ? dbg->sx : (uint16_t*)nullptr);
    if (rc != W8A8_OK) return rc;

    const int64_t nb_max = moe_max_blocks(R, E, bn);
    MoeSwapArgs a1 = {};
    a1.counts = w.counts;
    a1.offsets = w.offsets;
    a1.tile_off = w.tile_off;
    a1.E = E;
    a1.rows = 2 * I;
    a1.K = H;
    a1.ngroups = (2 * I) / 128;
    a1.nkb = H / 128;
    a1.a_out = w.a;
    a1.early_plan = 1;   // the plan comes two kernels back
    a1.gsw = s13;
    a1.gsx = w.sxg;
    MoeSwapArgs a2 = a1;
    a2.rows = H;
    a2.K = I;
    a2.ngroups = H / 128;
    a2.nkb = I / 128;
    a2.gsw = s2;
    a2.gsx = w.sag;
    a2.row_tok = w.row_tok;
    a2.row_slot = w.row_slot;
    a2.row_w = w.row_w;
    a2.contrib = w.out;
    a2.topk = topk;
    rc = bn == 16 ? launch_moe_swap<16, true, true>(w13, w.xq, R, a1, nb_max, st)
       : bn == 32 ? launch_moe_swap<32, true, true>(w13, w.xq, R, a1, nb_max, st)
                  : launch_moe_swap<64, true, true>(w13, w.xq, R, a1, nb_max, st);
    if (rc != W8A8_OK) return rc;
    // the intermediate rotated along I and group-quantized
    rc = cuda_status(launch_fwht128_quant<float, true>(w.a, R, (int64_t)I, w.qa, w.sag, st, true));
    if (rc != W8A8_OK) return rc;
    rc = bn == 16 ? launch_moe_swap<16, false, true>(w2, w.qa, R, a2, nb_max, st)
       : bn == 32 ? launch_moe_swap<32, false, true>(w2, w.qa, R, a2, nb_max, st)
                  : launch_moe_swap<64, false, true>(w2, w.qa, R, a2, nb_max, st);
    if (rc != W8A8_OK) return rc;
    rc = launch_chained(moe_finalize_kernel, (unsigned)((T * H / 4 + 255) / 256), 256u, st, (const float*)w.out, y, T,
                        H, topk);
    if (rc != W8A8_OK) return rc;
    if (!dbg) return W8A8_OK;
    if (dbg->topk_ids && cudaMemcpyAsync(dbg->topk_ids, w.ids, (size_t)R * 4, cudaMemcpyDeviceToDevice, st))
        return W8A8_ERR_CUDA;
    if (dbg->topk_w && cudaMemcpyAsync(dbg->topk_w, w.wts, (size_t)R * 4, cudaMemcpyDeviceToDevice, st))
        return W8A8_ERR_CUDA;
    if (dbg->counts && cudaMemcpyAsync(dbg->counts, w.counts, (size_t)E * 4, cudaMemcpyDeviceToDevice, st))
        return W8A8_ERR_CUDA;
    if (dbg->qa || dbg->sa) {
        moe_debug_gather_g128_kernel<<<(unsigned)R, 128, 0, st>>>(w.qa, w.sag, w.row_of, R, I, dbg->qa, dbg->sa);
        return last_launch_status();
    }
    return W8A8_OK;
}

}  // extern "C"

// ----------------------------------------------------------------- FWHT128 and the unrotated group-128 grid
namespace {
// The group-128 GEMM of the rotated domain (post = 1/128) and of the
// unrotated grid (post = 1).
// The weight scales are bf16 per row and 128 of K (sw), or, for the trunk
// format, u8 per row and 256 of K times a bf16 row scale (sw_u8, sw_row).
int linear_group_scaled(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint16_t* sw, uint16_t* y,
                        int64_t M, int64_t N, int64_t K, float post, cudaStream_t st,
                        const uint8_t* sw_u8 = nullptr, const uint16_t* sw_row = nullptr) {
    if (!qx || !sx || !qw || !(sw || (sw_u8 && sw_row)) || !y) return W8A8_ERR_INVALID_ARG;
    if (!gemm_shape_ok(M, N, K) || K % (sw_u8 ? 256 : 128) != 0) return W8A8_ERR_INVALID_ARG;
    if (!aligned(qx, 16) || !aligned(qw, 16) || !aligned(y, 16) || !aligned(sx, 2) || !aligned(sw, 2) ||
        !aligned(sw_row, 2))
        return W8A8_ERR_INVALID_ARG;
    if (M <= 8) {
        if (K / 128 > kG128MaxGroups || N % 16 != 0) return W8A8_ERR_UNSUPPORTED;
        // chained: the weight rows go to L2 while the activation quant before it runs
        return launch_chained_smem(gemv_g128_kernel<false>, (unsigned)(N / 16), 256u, gemv_g128_smem((int)(K / 128)),
                                   st, qx, sx, qw, sw, y, (int)M, (int)N, (int)K, post, sw_u8, sw_row,
                                   (float*)nullptr);
    }
    TcParams p = {};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.gsx = sx;
    p.gsw = sw;
    p.gsw_u8 = sw_u8;
    p.gsw_row = sw_row;
    p.gpost = post;
    p.out = y;
    if (M >= kTc2MinM) return launch_tc2_g128(qx, qw, p, st);
    return launch_tc<128, 6, kEpiG128, 4, 8>(qx, qw, p, st);
}

int group_quant(const uint16_t* x, int64_t M, int64_t K, int8_t* q, uint16_t* s, bool rotate, cudaStream_t st) {
    if (!x || !q || !s || M <= 0 || K <= 0 || K % 128 != 0) return W8A8_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 2)) return W8A8_ERR_INVALID_ARG;
    const int64_t ctas = fwht128_quant_ctas(M, K);
    if (ctas > 0x7fffffffLL) return W8A8_ERR_UNSUPPORTED;
    return cuda_status(rotate ? launch_fwht128_quant<uint16_t, true>(x, M, K, q, s, st, false)
                              : launch_fwht128_quant<uint16_t, false>(x, M, K, q, s, st, false));
}
}  // namespace

extern "C" {

int w8a8_linear_g128(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint16_t* sw, uint16_t* y,
                     int64_t M, int64_t N, int64_t K, void* stream) {
    return linear_group_scaled(qx, sx, qw, sw, y, M, N, K, 0.0078125f, (cudaStream_t)stream);
}

int fwht128_quant(const uint16_t* x, int64_t M, int64_t K, int8_t* q, uint16_t* s, void* stream) {
    return group_quant(x, M, K, q, s, true, (cudaStream_t)stream);
}

int group128_quant(const uint16_t* x, int64_t M, int64_t K, int8_t* q, uint16_t* s, void* stream) {
    return group_quant(x, M, K, q, s, false, (cudaStream_t)stream);
}

int w8a8_linear_group128(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint16_t* sw, uint16_t* y,
                         int64_t M, int64_t N, int64_t K, void* stream) {
    return linear_group_scaled(qx, sx, qw, sw, y, M, N, K, 1.0f, (cudaStream_t)stream);
}

// ----------------------------------------------------------------- trunk format, shared expert
int w8a8_trunk_weight_quant(const uint16_t* w, int64_t N, int64_t K, int8_t* q, uint8_t* su8, uint16_t* s2,
                            void* stream) {
    if (!w || !q || !su8 || !s2 || N <= 0 || K <= 0 || K % 256 != 0) return W8A8_ERR_INVALID_ARG;
    if (K > kTrunkMaxK || N > 0x7fffffffLL) return W8A8_ERR_UNSUPPORTED;
    if (!aligned(w, 16) || !aligned(s2, 2)) return W8A8_ERR_INVALID_ARG;
    trunk_weight_quant_kernel<<<(unsigned)N, 256, 0, (cudaStream_t)stream>>>(w, K, q, su8, s2);
    return last_launch_status();
}

}  // extern "C"

namespace {
struct SharedWs {
    int32_t* counts;
    int32_t* offsets;
    int32_t* tile_off;
    int32_t* row_tok;
    int32_t* row_slot;
    float* row_w;
    int8_t* xq;       // [M, H] rotated codes of x
    uint16_t* sxg;    // [M, H / 128]
    float* a;         // [M, I] fp32 gated intermediate
    int8_t* qa;       // [M, I]
    uint16_t* sag;    // [M, I / 128]
    float* out;       // [M, H] fp32 before the bf16 rounding
    size_t bytes;
};

SharedWs shared_carve(void* base, int64_t M, int H, int I) {
    SharedWs w;
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        uint8_t* r = p ? p + o : nullptr;
        o += align_up(bytes, 256);
        return r;
    };
    w.counts = reinterpret_cast<int32_t*>(take(16));
    w.offsets = reinterpret_cast<int32_t*>(take(16));
    w.tile_off = reinterpret_cast<int32_t*>(take(16));
    w.row_tok = reinterpret_cast<int32_t*>(take((size_t)M * 4));
    w.row_slot = reinterpret_cast<int32_t*>(take((size_t)M * 4));
    w.row_w = reinterpret_cast<float*>(take((size_t)M * 4));
    w.xq = reinterpret_cast<int8_t*>(take((size_t)M * H));
    w.sxg = reinterpret_cast<uint16_t*>(take((size_t)M * (H / 128) * 2));
    w.a = reinterpret_cast<float*>(take((size_t)M * I * 4));
    w.qa = reinterpret_cast<int8_t*>(take((size_t)M * I));
    w.sag = reinterpret_cast<uint16_t*>(take((size_t)M * (I / 128) * 2));
    w.out = reinterpret_cast<float*>(take((size_t)M * H * 4));
    w.bytes = o;
    return w;
}
}  // namespace

extern "C" {

size_t w8a8_shared_expert_workspace_size(int64_t M, int H, int I) {
    if (M <= 0 || H < 256 || I < 128) return 0;
    return shared_carve(nullptr, M, H, I).bytes;
}

int w8a8_shared_expert_forward(const uint16_t* x, const int8_t* w13, const uint8_t* u13, const uint16_t* r13,
                               const int8_t* w2, const uint16_t* s2, uint16_t* y, int64_t M, int H, int I, void* ws,
                               size_t ws_bytes, const w8a8_shared_expert_debug* dbg, void* stream) {
    if (!x || !w13 || !u13 || !r13 || !w2 || !s2 || !y || !ws) return W8A8_ERR_INVALID_ARG;
    if (M <= 0 || H <= 0 || I <= 0) return W8A8_ERR_INVALID_ARG;
    if (H % 256 != 0 || H > 128 * kMoeG128MaxGroupsH || I % 128 != 0 || I > 2048) return W8A8_ERR_UNSUPPORTED;
    if (M > (int64_t)1 << 30) return W8A8_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(w13, 16) || !aligned(r13, 2) || !aligned(w2, 16) || !aligned(s2, 2) ||
        !aligned(y, 16) || !aligned(ws, 256))
        return W8A8_ERR_INVALID_ARG;
    if (ws_bytes < w8a8_shared_expert_workspace_size(M, H, I)) return W8A8_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    SharedWs w = shared_carve(ws, M, H, I);
    int rc;
    auto debug_copies = [&]() -> int {
        if (!dbg) return W8A8_OK;
        if (dbg->qx && cudaMemcpyAsync(dbg->qx, w.xq, (size_t)(M * H), cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        if (dbg->sx && cudaMemcpyAsync(dbg->sx, w.sxg, (size_t)M * (H / 128) * 2, cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        if (dbg->qa && cudaMemcpyAsync(dbg->qa, w.qa, (size_t)M * I, cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        if (dbg->sa && cudaMemcpyAsync(dbg->sa, w.sag, (size_t)M * (I / 128) * 2, cudaMemcpyDeviceToDevice, st))
            return W8A8_ERR_CUDA;
        return W8A8_OK;
    };
    if (M <= 8 && H / 128 <= kG128MaxGroups && I / 128 <= kG128MaxGroups) {
        // decode sizes: x quant, the gated group-128 GEMV over w13 (16 rows per
        // CTA), the intermediate's quant, the group-128 GEMV over w2 writing y
        rc = cuda_status(launch_fwht128_quant<uint16_t, true>(x, M, (int64_t)H, w.xq, w.sxg, st, false));
        if (rc != W8A8_OK) return rc;
        rc = launch_chained_smem(gemv_g128_kernel<true>, (unsigned)(2 * I / 16), 256u, gemv_g128_smem(H / 128), st,
                                 (const int8_t*)w.xq,
                            (const uint16_t*)w.sxg, w13, (const uint16_t*)nullptr, (uint16_t*)nullptr, (int)M, 2 * I, H,
                            0.0078125f, u13, r13, w.a);
        if (rc != W8A8_OK) return rc;
        rc = cuda_status(launch_fwht128_quant<float, true>(w.a, M, (int64_t)I, w.qa, w.sag, st, true));
        if (rc != W8A8_OK) return rc;
        rc = launch_chained_smem(gemv_g128_kernel<false>, (unsigned)(H / 16), 256u, gemv_g128_smem(I / 128), st,
                                 (const int8_t*)w.qa,
                            (const uint16_t*)w.sag, w2, s2, y, (int)M, H, I, 0.0078125f, (const uint8_t*)nullptr,
                            (const uint16_t*)nullptr, (float*)nullptr);
        if (rc != W8A8_OK) return rc;
        return debug_copies();
    }
    const int bn = M <= 12 ? 16 : (M <= 24 ? 32 : 64);
    shared_plan_kernel<<<(unsigned)((M + 255) / 256), 256, 0, st>>>((int)M, bn, w.counts, w.offsets, w.tile_off,
                                                                     w.row_tok, w.row_slot, w.row_w);
    if ((rc = last_launch_status()) != W8A8_OK) return rc;
    // x rotated along H and group-quantized: the sorted rows are the tokens
    rc = cuda_status(launch_fwht128_quant<uint16_t, true>(x, M, (int64_t)H, w.xq, w.sxg, st, true));
    if (rc != W8A8_OK) return rc;
    const int64_t nb = (M + bn - 1) / bn;
    MoeSwapArgs a1 = {};
    a1.counts = w.counts;
    a1.offsets = w.offsets;
    a1.tile_off = w.tile_off;
    a1.E = 1;
    a1.rows = 2 * I;
    a1.K = H;
    a1.ngroups = (2 * I) / 128;
    a1.nkb = H / 128;
    a1.a_out = w.a;
    a1.early_plan = 1;   // the plan comes two kernels back
    a1.gsx = w.sxg;
    a1.gsw_u8 = u13;     // gate_up in the trunk's two-level format
    a1.gsw_row = r13;
    MoeSwapArgs a2 = a1;
    a2.rows = H;
    a2.K = I;
    a2.ngroups = H / 128;
    a2.nkb = I / 128;
    a2.gsx = w.sag;
    a2.gsw = s2;         // down on the group-128 grid
    a2.gsw_u8 = nullptr;
    a2.gsw_row = nullptr;
    a2.row_tok = w.row_tok;
    a2.row_slot = w.row_slot;
    a2.row_w = w.row_w;
    a2.contrib = w.out;
    a2.topk = 1;
    rc = bn == 16 ? launch_moe_swap<16, true, true>(w13, w.xq, M, a1, nb, st)
       : bn == 32 ? launch_moe_swap<32, true, true>(w13, w.xq, M, a1, nb, st)
                  : launch_moe_swap<64, true, true>(w13, w.xq, M, a1, nb, st);
    if (rc != W8A8_OK) return rc;
    rc = cuda_status(launch_fwht128_quant<float, true>(w.a, M, (int64_t)I, w.qa, w.sag, st, true));
    if (rc != W8A8_OK) return rc;
    rc = bn == 16 ? launch_moe_swap<16, false, true>(w2, w.qa, M, a2, nb, st)
       : bn == 32 ? launch_moe_swap<32, false, true>(w2, w.qa, M, a2, nb, st)
                  : launch_moe_swap<64, false, true>(w2, w.qa, M, a2, nb, st);
    if (rc != W8A8_OK) return rc;
    rc = launch_chained(moe_finalize_kernel, (unsigned)((M * H / 4 + 255) / 256), 256u, st, (const float*)w.out, y,
                        M, H, 1);
    if (rc != W8A8_OK) return rc;
    return debug_copies();
}

int w8a8_linear_trunk(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint8_t* su8, const uint16_t* s2,
                      uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream) {
    if (!su8 || !s2) return W8A8_ERR_INVALID_ARG;
    return linear_group_scaled(qx, sx, qw, nullptr, y, M, N, K, 0.0078125f, (cudaStream_t)stream, su8, s2);
}

// ----------------------------------------------------------------- diagnostics
int w8a8_exp_proj(const float* x, float* y, int64_t n, void* stream) {
    if (!x || !y || n <= 0) return W8A8_ERR_INVALID_ARG;
    exp_proj_kernel<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(x, y, n);
    return last_launch_status();
}

int w8a8_get_device_error(void* stream, int* site) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return W8A8_ERR_CUDA;
    int err = 0, where = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&err, g_device_error, sizeof(int)) != cudaSuccess) return W8A8_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&where, g_device_error_site, sizeof(int)) != cudaSuccess) return W8A8_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return W8A8_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_device_error_site, &zero, sizeof(int)) != cudaSuccess) return W8A8_ERR_CUDA;
    if (site) *site = where;
    return err;
}

int w8a8_debug_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000LL) return W8A8_ERR_INVALID_ARG;
    debug_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_ns);
    return last_launch_status();
}

}  // extern "C"
