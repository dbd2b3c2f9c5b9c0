/*
 * w8a8.h -- C ABI of libw8a8.so: online INT8 W8A8 linear layers and the
 * routed W8A8 MoE expert layer for NVIDIA B200 (sm_100a).
 *
 * Sources (page title, section):
 *   [ATOM]  "[gfx1151] Online INT8 W8A8 for Qwen3.6 27B / 35B-A3B on RDNA3.5,
 *            with working MTP" -- "Precision split" (int8 weights with dynamic
 *            per-token int8 activations; router gate stays bf16) and "Changes"
 *            (gemm_a8w8 per-token path; Int8MoEMethod with int8 w13/w2 and
 *            per-channel fp32 scales; the MoE forward: routing -> per-token int8
 *            quant -> gemm1 with fused gated SiLU via interleaved w13 -> per-token
 *            int8 quant -> gemm2 with scatter/combine).
 *   [QUARK] "Qwen3.6-27B-Quark-W8A8-INT8" -- "Quantization Scheme" and
 *            "Quantization Details" (per-channel symmetric weights, per-token
 *            symmetric dynamic activations).
 *   [IQ8R]  "Qwen3.6-35B-A3B IQ8R - radiance container" -- file table (int8
 *            codes in -127..127 after every 128-wide slice of K is turned by
 *            the unnormalised Hadamard matrix, one bf16 scale for each row and
 *            each 128-wide slice; the activations quantized the same way) and
 *            the conversion recipe (transform=fwht128 group=128 scale=bf16
 *            clamp=sym).
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless stated otherwise; the caller owns
 *     every buffer.  The library allocates nothing, keeps no per-call state
 *     and never synchronizes: each call enqueues its kernels on `stream`
 *     (a cudaStream_t; NULL is the legacy default stream) and returns.
 *   - Matrices are dense and row-major.  bf16 values are passed as their
 *     16-bit patterns (uint16_t).  Weights are [N, K] with K contiguous.
 *   - Pointers must be 16-byte aligned; K must be a multiple of 16 (the
 *     tensor-memory-access unit); N a multiple of 8.
 *   - Return value: W8A8_OK (0) or a negative W8A8_ERR_* code.  Argument
 *     errors are detected on the host before anything is enqueued.  A kernel
 *     that had to give up (a bounded wait ran out) records
 *     W8A8_ERR_TIMEOUT in a device error word instead of trapping; read it
 *     with w8a8_get_device_error().
 */
#ifndef W8A8_H_
#define W8A8_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W8A8_API __attribute__((visibility("default")))
#else
#define W8A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define W8A8_OK 0
#define W8A8_ERR_INVALID_ARG (-1)  /* null pointer, bad size, misalignment */
#define W8A8_ERR_WORKSPACE (-2)    /* workspace smaller than the *_workspace_size query */
#define W8A8_ERR_UNSUPPORTED (-3)  /* shape outside what the kernels handle */
#define W8A8_ERR_CUDA (-4)         /* a CUDA launch or driver call failed */
#define W8A8_ERR_TIMEOUT (-5)      /* a device-side bounded wait gave up */

/* Selects the GEMM kernel in w8a8_gemm_q / w8a8_gemm_s32. */
#define W8A8_PATH_AUTO 0      /* decode GEMV for M <= 8, tiled tensor-core GEMM otherwise */
#define W8A8_PATH_TCGEN05 1   /* tiled tcgen05 kind::i8 GEMM (128-token tiles), any M */
#define W8A8_PATH_GEMV 2      /* weight-streaming swap-AB tcgen05 GEMV, M <= 32 */

/* ---------------------------------------------------------------------------
 * Per-token dynamic activation quantization (a1) -- [ATOM] "Precision split",
 * [QUARK] "Quantization Scheme" (activation: per-token, symmetric, dynamic).
 *   x  bf16 [M, K], row stride ldx elements (ldx >= K, ldx % 8 == 0)
 *   q  int8 [M, K] (row stride K): q = clamp(rne(x / s), -127, 127)
 *   s  fp32 [M]: s = max_k |x[m,k]| / 127 in fp32; a zero row gives s = 0, q = 0.
 * Division and rounding are IEEE fp32 round-to-nearest-even. */
W8A8_API int w8a8_quant_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s, void* stream);

/* Online per-output-channel weight quantization (a0) -- [ATOM] "Changes"
 * (FusedMoE._online_quant; no offline step), [QUARK] "Quantization Scheme"
 * (weight: per-channel, symmetric).  Same arithmetic as w8a8_quant_act on fp32
 * rows:  w fp32 [N, K] -> q int8 [N, K], s fp32 [N]. */
W8A8_API int w8a8_quant_rows_f32(const float* w, int64_t N, int64_t K, int8_t* q, float* s, void* stream);

/* Workspace bytes w8a8_linear needs for an M x K activation. */
W8A8_API size_t w8a8_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/* Dense W8A8 linear (a1 + a2 + a3, or a1 + a4 for M <= 8) -- [ATOM] "Changes"
 * (per-token int8 branch -> gemm_a8w8), [QUARK] "Quantization Details".
 *   x  bf16 [M, K];  qw int8 [N, K];  sw fp32 [N];  y bf16 [M, N]
 *   y[m,n] = bf16_rne( (float(sum_k qx[m,k] qw[n,k]) * sx[m]) * sw[n] )
 * with (qx, sx) = w8a8_quant_act(x) held in `ws` (ws_bytes >=
 * w8a8_linear_workspace_size(M, N, K)).  The int32 sum is exact. */
W8A8_API int w8a8_linear(const uint16_t* x, const int8_t* qw, const float* sw, uint16_t* y, int64_t M, int64_t N, int64_t K,
                void* ws, size_t ws_bytes, void* stream);

/* Dense W8A8 linear for callers that cannot allocate device memory.
 * No counterpart in the cited sources: an interface addition of this library.
 * Some callers cannot call cudaMalloc where they run the layer (an allocator
 * locked during a step, a plugin host that only passes its input and output
 * buffers).  This entry point computes exactly what w8a8_linear computes, with
 * the same kernels, but keeps the scratch (activation codes and scales, split-K
 * partials and counters) in a file-scope device array of
 * W8A8_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.  It allocates nothing.
 *   - Sizes: w8a8_linear_noalloc_scratch_size(M, N, K) must not exceed
 *     W8A8_NOALLOC_SCRATCH_BYTES (4 MiB: e.g. M <= 8 at K = 17408, or
 *     M * K up to about 4 million); larger calls return W8A8_ERR_UNSUPPORTED
 *     and enqueue nothing.
 *   - The first call on a device looks up the array's device address (with that
 *     device current); make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents (what
 *     must start at zero is cleared by each call): calls that overlap on the GPU
 *     (different streams, or different host threads on one device) race and
 *     must be serialized by the caller. */
#define W8A8_NOALLOC_SCRATCH_BYTES (4u << 20)
W8A8_API size_t w8a8_linear_noalloc_scratch_size(int64_t M, int64_t N, int64_t K);
W8A8_API int w8a8_linear_noalloc(const uint16_t* x, const int8_t* qw, const float* sw, uint16_t* y, int64_t M,
                                 int64_t N, int64_t K, void* stream);

/* GEMM on pre-quantized activations with the dequant epilogue (a2 + a3):
 *   qx int8 [M, K], sx fp32 [M], qw int8 [N, K], sw fp32 [N] -> y bf16 [M, N].
 * `path` is one of W8A8_PATH_*.  The GEMV path with M > 8 and K split over
 * several CTAs uses `ws` (bytes from w8a8_gemm_workspace_size); pass NULL/0
 * when w8a8_gemm_workspace_size returns 0. */
W8A8_API size_t w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int path);
W8A8_API int w8a8_gemm_q(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, uint16_t* y, int64_t M,
                int64_t N, int64_t K, int path, void* ws, size_t ws_bytes, void* stream);

/* Raw int32 accumulators (a2), for parity checks:
 *   acc[m,n] = sum_k qx[m,k] * qw[n,k]   (int32 [M, N], exact). */
W8A8_API int w8a8_gemm_s32(const int8_t* qx, const int8_t* qw, int32_t* acc, int64_t M, int64_t N, int64_t K, int path,
                  void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Routed W8A8 MoE expert layer (a5 .. a11) -- [ATOM] "Changes" (Int8MoEMethod,
 * triton_kernel_int8_moe_forward), "Precision split" (bf16 router).
 *   x       bf16 [T, H]             token activations
 *   logits  bf16 [T, E]             router logits (the bf16 gate GEMM is the caller's)
 *   w13     int8 [E, 2I, H]         row 2i = gate_i, row 2i+1 = up_i ("interleaved w13")
 *   s13     fp32 [E, 2I]            per-channel scales of w13
 *   w2      int8 [E, H, I]; s2 fp32 [E, H]
 *   y       bf16 [T, H]             output
 * Steps: top-k of softmax(logits) (ties -> lower expert index), weights
 * renormalised over the k; x quantized once per token (shared by its
 * experts); v = (float(qx . w13[e,r]) * sx) * s13[e,r];
 * a_i = SiLU(v_2i) * v_2i+1; (qa, sa) = per-row quant of a; y2_n =
 * (float(qa . w2[e,n]) * sa) * s2[e,n]; y = bf16( sum_j w_j * y2 ) with the k
 * contributions added in fp32 in slot order.
 * ws_bytes >= w8a8_moe_workspace_size(T, E, H, I, topk).  `dbg` may be NULL;
 * otherwise its non-NULL members receive intermediate values. */
typedef struct w8a8_moe_debug {
    int32_t* topk_ids;   /* [T, topk], descending logits */
    float* topk_w;       /* [T, topk] */
    int32_t* counts;     /* [E] rows routed to each expert */
    int8_t* qx;          /* [T, H] codes of x */
    float* sx;           /* [T] */
    int8_t* qa;          /* [T, topk, I] codes of the gated intermediate, by (token, slot) */
    float* sa;           /* [T, topk] */
} w8a8_moe_debug;

W8A8_API size_t w8a8_moe_workspace_size(int64_t T, int E, int H, int I, int topk);

/* How w8a8_moe_forward adds each token's k contributions (process-wide;
 * no counterpart on the pages, which fix only the sum itself):
 *   W8A8_MOE_COMBINE_AUTO (default)  in fp32 in slot order -- the definition's
 *       order, bit-exact and deterministic -- while T * topk * H * 4 bytes of
 *       contributions stay within 64 MiB; beyond that with fp32 atomics into
 *       the token's row (order unspecified: within one bf16 ulp plus the
 *       reordering bound of a k-term fp32 sum, not bit-exact, not
 *       run-to-run deterministic), which saves an HBM round trip of the
 *       [T * topk, H] contributions;
 *   W8A8_MOE_COMBINE_EXACT           in slot order at every T.
 * The mode also sizes the workspace (w8a8_moe_workspace_size): set it before
 * sizing, and do not change it between sizing and the forward call (a call
 * whose workspace is then too small returns W8A8_ERR_WORKSPACE).  Returns the
 * previous mode, or W8A8_ERR_INVALID_ARG for an unknown one. */
#define W8A8_MOE_COMBINE_AUTO 0
#define W8A8_MOE_COMBINE_EXACT 1
W8A8_API int w8a8_moe_set_combine(int mode);

W8A8_API int w8a8_moe_forward(const uint16_t* x, const uint16_t* logits, const int8_t* w13, const float* s13,
                     const int8_t* w2, const float* s2, uint16_t* y, int64_t T, int E, int H, int I, int topk,
                     void* ws, size_t ws_bytes, const w8a8_moe_debug* dbg, void* stream);

/* ---------------------------------------------------------------------------
 * Dense gated MLP block -- the dense analogue of a8 .. a10 ([ATOM] "Changes":
 * gemm1 with fused gated SiLU over interleaved w13, per-token int8 quant,
 * gemm2), one expert without routing:
 *   x    bf16 [M, H];  w13 int8 [2I, H] (row 2i = gate_i, 2i+1 = up_i), s13 fp32 [2I]
 *   w2   int8 [H, I];  s2 fp32 [H];   y bf16 [M, H]
 * Steps: (qx, sx) = per-token quant of x; v = (float(qx . w13[r]) * sx) *
 * s13[r]; a_i = SiLU(v_2i) * v_2i+1 (fp32, the project exponential);
 * (qa, sa) = per-row quant of a; y = bf16( (float(qa . w2[n]) * sa) * s2[n] ).
 * M <= 8 runs the weight-streaming GEMV path, larger M the tcgen05 GEMMs.
 * Requires H % 16 == 0 and I % 16 == 0; 16-byte aligned pointers.
 * ws_bytes >= w8a8_mlp_workspace_size(M, H, I).  `dbg` may be NULL;
 * otherwise its non-NULL members receive intermediate values. */
typedef struct w8a8_mlp_debug {
    int8_t* qx;          /* [M, H] codes of x */
    float* sx;           /* [M] */
    int8_t* qa;          /* [M, I] codes of the gated intermediate */
    float* sa;           /* [M] */
} w8a8_mlp_debug;

W8A8_API size_t w8a8_mlp_workspace_size(int64_t M, int64_t H, int64_t I);
W8A8_API int w8a8_mlp_forward(const uint16_t* x, const int8_t* w13, const float* s13, const int8_t* w2,
                              const float* s2, uint16_t* y, int64_t M, int64_t H, int64_t I, void* ws,
                              size_t ws_bytes, const w8a8_mlp_debug* dbg, void* stream);

/* ---------------------------------------------------------------------------
 * FWHT128-domain group quantization (a12) -- [IQ8R] file table ("each 128 of
 * K rotated by the unnormalised Hadamard"; codes -127..127; a bf16 scale per
 * row and 128 of K) and recipe (transform=fwht128 group=128 scale=bf16
 * clamp=sym).  For each 128-wide block of each row of x bf16 [M, K]
 * (K % 128 == 0): x' = H128 x_blk (unnormalised Sylvester Hadamard, fp32,
 * butterfly stages 1, 2, 4, ..., 64); s = bf16_rne(max|x'| / 127);
 * q = clamp(rne(x' / s), -127, 127).
 *   q int8 [M, K];  s bf16 [M, K/128].
 * Used for activations at run time and for weights at set-up. */
W8A8_API int fwht128_quant(const uint16_t* x, int64_t M, int64_t K, int8_t* q, uint16_t* s, void* stream);

/* Group-128 scaled GEMM in the rotated domain (a13):
 *   y[m,n] = bf16_rne( (1/128) * sum_g float(p_g) * (sx[m,g] * sw[n,g]) ),
 *   p_g = sum over the 128 k of group g of qx[m,k] qw[n,k] (int32, exact).
 * qx int8 [M, K], sx bf16 [M, K/128], qw int8 [N, K], sw bf16 [N, K/128],
 * y bf16 [M, N].  The groups are summed in ascending order, one fp32 fma
 * each: acc = fma(float(p_g), sx * sw, acc); y = bf16_rne(acc * (1/128)).
 * M <= 8 needs N % 16 == 0 and K <= 8192. */
W8A8_API int w8a8_linear_g128(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint16_t* sw, uint16_t* y,
                     int64_t M, int64_t N, int64_t K, void* stream);

/* ---------------------------------------------------------------------------
 * The group-128 grid without the rotation -- [IQ8R] file table (Head row:
 * the lm_head holds int8 codes with one bf16 scale per row and 128 elements
 * of K, and no rotation is listed for it) and recipe row
 * output.weight (codes=i8 group=128 scale=bf16 clamp=sym, no transform).
 * group128_quant: fwht128_quant without the butterflies: for each 128-wide
 * block of each row of x bf16 [M, K] (K % 128 == 0): s = bf16_rne(max|x| /
 * 127), q = clamp(rne(x / s), -127, 127); q int8 [M, K], s bf16 [M, K/128].
 * w8a8_linear_group128: y[m,n] = bf16_rne( sum_g float(p_g) * (sx[m,g] *
 * sw[n,g]) ) with one fp32 fma per group in ascending g -- the group-128
 * GEMM without the 1/128 (there is no rotation to undo).  Shapes, layouts
 * and the M <= 8 / M > 8 split as w8a8_linear_g128. */
W8A8_API int group128_quant(const uint16_t* x, int64_t M, int64_t K, int8_t* q, uint16_t* s, void* stream);
W8A8_API int w8a8_linear_group128(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint16_t* sw,
                                  uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream);

/* ---------------------------------------------------------------------------
 * The trunk linears' two-level format -- [IQ8R] file table (Trunk row:
 * int8 codes in -127..127; each 256-wide slice of a row has a u8 scale, and
 * the row as a whole a bf16 scale that multiplies it; the rows are turned
 * 128 elements at a time by the unnormalised Hadamard matrix; rounding to
 * nearest) and recipe (codes=i8 group=256 scale=u8 scale2=bf16 block2=1x*
 * transform=fwht128 clamp=sym rule=search).
 * w8a8_trunk_weight_quant (set-up): each row of w bf16 [N, K] (K % 256 == 0,
 * K <= 8192) rotated 128 at a time; scale2[n] = bf16_rne(max|w'| / (127*255));
 * for each 256-wide group j, su8[n, j] = the u in 1..255 whose scale
 * s = u * scale2 gives the smallest largest error max_k |w'_k - q_k s| with
 * q_k = clamp(rne(w'_k / s), +-127) (ties to the smaller u); codes under the
 * chosen s.  A zero row: scale2 = 0, su8 = 0, codes 0.
 *   q int8 [N, K];  su8 uint8 [N, K/256];  s2 bf16 [N].
 * w8a8_linear_trunk: x codes and bf16 group scales from fwht128_quant
 * (qx int8 [M, K], sx bf16 [M, K/128]) times W in that format:
 *   y[m,n] = bf16_rne( (1/128) * sum_g fma(float(p_g), sx[m,g] * sw_g, .) ),
 *   sw_g = float(su8[n, g/2]) * float(s2[n]) (exact), groups ascending.
 * M <= 8 runs the GEMV (N % 16 == 0), larger M the tcgen05 GEMM. */
W8A8_API int w8a8_trunk_weight_quant(const uint16_t* w, int64_t N, int64_t K, int8_t* q, uint8_t* su8, uint16_t* s2,
                                     void* stream);
W8A8_API int w8a8_linear_trunk(const int8_t* qx, const uint16_t* sx, const int8_t* qw, const uint8_t* su8,
                               const uint16_t* s2, uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream);


/* ---------------------------------------------------------------------------
 * The shared expert -- [IQ8R] file table (Experts row: the shared expert is
 * stored like the routed ones, except that its gate/up projection takes the
 * trunk linears' format) and recipe rows
 * ffn_gate_up_shexp (the trunk format above) and ffn_down_shexp (group=128
 * scale=bf16 transform=fwht128).  A dense gated MLP on the rotated grid:
 *   x    bf16 [M, H]
 *   w13  int8 [2I, H] + su8 [2I, H/256] + bf16 row scales [2I] (trunk format;
 *        row 2i = gate_i, 2i+1 = up_i)
 *   w2   int8 [H, I] + bf16 [H, I/128] (fwht128_quant of the bf16 rows)
 *   y    bf16 [M, H]
 * Steps: (qx, sx) = fwht128_quant(x); v = the trunk product of (qx, sx) with
 * w13 (fp32); a_i = SiLU(v_2i) * v_2i+1; (qa, sa) = FWHT128 group quant of the
 * fp32 row a (along I); y = bf16( the group-128 product of (qa, sa) with w2 ).
 * M <= 8 runs group-128 GEMVs (the gated one over w13 writes a), larger M the
 * swap-AB tcgen05 expert kernels.
 * Requires H % 256 == 0, H <= 4096, I % 128 == 0, I <= 2048; 16-byte aligned
 * x, w13, w2, y; 256-byte aligned ws; ws_bytes >=
 * w8a8_shared_expert_workspace_size(M, H, I).  `dbg` may be NULL. */
typedef struct w8a8_shared_expert_debug {
    int8_t* qx;          /* [M, H] rotated codes of x */
    uint16_t* sx;        /* [M, H/128] bf16 */
    int8_t* qa;          /* [M, I] rotated codes of the gated intermediate */
    uint16_t* sa;        /* [M, I/128] bf16 */
} w8a8_shared_expert_debug;

W8A8_API size_t w8a8_shared_expert_workspace_size(int64_t M, int H, int I);
W8A8_API int w8a8_shared_expert_forward(const uint16_t* x, const int8_t* w13, const uint8_t* u13, const uint16_t* r13,
                                        const int8_t* w2, const uint16_t* s2, uint16_t* y, int64_t M, int H, int I,
                                        void* ws, size_t ws_bytes, const w8a8_shared_expert_debug* dbg, void* stream);

/* ---------------------------------------------------------------------------
 * Routed experts on the FWHT128 grid -- [IQ8R] file table (Experts row: the
 * routed experts are int8 codes on the rotated grid, one bf16 scale for each
 * row and 128-wide slice of K; Activations row: the activations are
 * quantized after the same rotation, and the routed experts take the codes
 * that the trunk's activation quantizer produces) and recipe (ffn_gate_up_exps / ffn_down_exps:
 * group=128 scale=bf16 transform=fwht128).  The layer of w8a8_moe_forward
 * with each quantizer replaced by fwht128_quant and each expert GEMM by its
 * group-128 form:
 *   x       bf16 [T, H]             token activations (unrotated)
 *   logits  bf16 [T, E]             router logits
 *   w13     int8 [E, 2I, H]         rows rotated along H (fwht128_quant of the
 *                                   bf16 rows), row 2i = gate_i, 2i+1 = up_i
 *   s13     bf16 [E, 2I, H/128]
 *   w2      int8 [E, H, I]          rows rotated along I; s2 bf16 [E, H, I/128]
 *   y       bf16 [T, H]
 * Steps: routing as w8a8_moe_forward; (qx, sx) = fwht128_quant(x[t]);
 * v_r = (sum over g ascending of fma(float(p_g), sx[g] * s13[e,r,g], .)) / 128
 * (fp32, p_g the int32 dot product of group g); a_i = SiLU(v_2i) * v_2i+1;
 * (qa, sa) = FWHT128 group quant of the fp32 row a (rotated along I);
 * y2_n = the same group-128 product of (qa, sa) with (w2[e,n], s2[e,n]);
 * y = bf16( sum_j w_j * y2 ) with the k contributions added in fp32 in slot
 * order.  Requires H % 128 == 0, H <= 4096, I % 128 == 0, I <= 2048,
 * E <= 256, topk <= 32; 16-byte aligned x, w13, w2, y; 256-byte aligned ws.
 * ws_bytes >= w8a8_moe_g128_workspace_size(T, E, H, I, topk).  `dbg` may be
 * NULL; otherwise its non-NULL members receive intermediate values. */
typedef struct w8a8_moe_g128_debug {
    int32_t* topk_ids;   /* [T, topk], descending logits */
    float* topk_w;       /* [T, topk] */
    int32_t* counts;     /* [E] rows routed to each expert */
    int8_t* qx;          /* [T, H] rotated codes of x */
    uint16_t* sx;        /* [T, H/128] bf16 */
    int8_t* qa;          /* [T, topk, I] rotated codes of the gated intermediate, by (token, slot) */
    uint16_t* sa;        /* [T, topk, I/128] bf16 */
} w8a8_moe_g128_debug;

W8A8_API size_t w8a8_moe_g128_workspace_size(int64_t T, int E, int H, int I, int topk);
W8A8_API int w8a8_moe_g128_forward(const uint16_t* x, const uint16_t* logits, const int8_t* w13,
                                   const uint16_t* s13, const int8_t* w2, const uint16_t* s2, uint16_t* y, int64_t T,
                                   int E, int H, int I, int topk, void* ws, size_t ws_bytes,
                                   const w8a8_moe_g128_debug* dbg, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics. */

/* The library's fp32 exponential (Cody & Waite reduction, degree-7 Taylor),
 * applied elementwise: y[i] = exp_proj(x[i]).  Used by the router softmax and
 * by SiLU; exposed so tests can compare it bit for bit. */
W8A8_API int w8a8_exp_proj(const float* x, float* y, int64_t n, void* stream);

/* Synchronizes `stream`, then returns and clears the device error word:
 * W8A8_OK or the first W8A8_ERR_* a kernel recorded (W8A8_ERR_CUDA if the
 * synchronization itself failed).  When site != NULL it receives where the
 * error was recorded ((kernel id << 16) | site). */
W8A8_API int w8a8_get_device_error(void* stream, int* site);

/* Test hook for the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing will arrive at, with a limit of `limit_ns` nanoseconds
 * (1e3 <= limit_ns <= 1e9).  The wait gives up, records W8A8_ERR_TIMEOUT and
 * the kernel returns; no GPU fault is raised. */
W8A8_API int w8a8_debug_wait_timeout(int64_t limit_ns, void* stream);

/* Human-readable name of a status code (static string). */
W8A8_API const char* w8a8_status_str(int status);

/* Library version string (static). */
W8A8_API const char* w8a8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H_ */
