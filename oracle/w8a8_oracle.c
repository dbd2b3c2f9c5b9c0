/*
 * CPU oracle for the online INT8 W8A8 linear / routed-MoE hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * Plain scalar C, written for a reader to check against the sources below by eye.
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * OpenMP is used only to split independent output rows across threads;
 * the arithmetic of each row is unchanged by it.
 *
 * Sources (page title, section):
 *   [ATOM]  "[gfx1151] Online INT8 W8A8 for Qwen3.6 27B / 35B-A3B on RDNA3.5,
 *            with working MTP", sections "Precision split" and "Changes".
 *   [IQ8R]  "Qwen3.6-35B-A3B IQ8R - radiance container", the file table
 *            (Trunk / Experts / Activations rows) and the conversion recipe.
 *   [QUARK] "Qwen3.6-27B-Quark-W8A8-INT8", sections "Quantization Scheme"
 *            and "Quantization Details".
 *
 * Floating point: the sources fix fp32 scales, int32 accumulation and bf16
 * outputs, so the arithmetic below is fp32 with one IEEE round-to-nearest
 * operation per C operator (fp contraction is off); fp64 copies are kept
 * only where a test needs an error bound.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef uint16_t bf16_t;

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32                                                        */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
float oracle_bf16_to_f32(bf16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even, by its definition:
 * keep the upper 16 bits, add one unit when the dropped 16 bits exceed
 * half a unit, or equal half a unit and the kept part is odd. */
bf16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (bf16_t)((u >> 16) | 0x0040u);          /* NaN stays NaN */
    uint32_t hi = u >> 16;
    uint32_t rem = u & 0xffffu;
    if (rem > 0x8000u || (rem == 0x8000u && (hi & 1u)))
        hi += 1u;                                      /* carry may reach inf: correct */
    return (bf16_t)hi;
}

/* ------------------------------------------------------------------ */
/* Round to nearest integer, ties to even (the "round to nearest" of    */
/* [IQ8R] Trunk row; round-to-nearest-even for the per-token scheme).   */
/* ------------------------------------------------------------------ */
static int64_t rne_to_int(float y)
{
    double d = (double)y;          /* exact */
    double fl = floor(d);
    double frac = d - fl;          /* exact: both are doubles of a float */
    int64_t r = (int64_t)fl;
    if (frac > 0.5 || (frac == 0.5 && (r & 1)))
        r += 1;
    return r;
}

static int8_t clamp_sym127(int64_t r)
{
    if (r > 127) r = 127;
    if (r < -127) r = -127;        /* symmetric: -128 is never produced */
    return (int8_t)r;
}

/* ------------------------------------------------------------------ */
/* a0/a1/a9: symmetric absmax quantization of one row.                  */
/* [QUARK] "Quantization Scheme": weights per-channel symmetric,        */
/* activations per-token symmetric dynamic; [ATOM] "Precision split":   */
/* dynamic per-token int8 activation.  Scale s = absmax / 127 (fp32),   */
/* code q = clamp(rne(v / s), -127, 127).  A row whose scale is zero    */
/* (all-zero row) gets s = 0 and all codes 0.                           */
/* ------------------------------------------------------------------ */
void oracle_quant_row_f32(const float* v, int64_t K, int8_t* q, float* s_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(v[k]);
        if (a > amax) amax = a;
    }
    float s = amax / 127.0f;
    *s_out = s;
    if (s == 0.0f) {
        for (int64_t k = 0; k < K; ++k) q[k] = 0;
        return;
    }
    for (int64_t k = 0; k < K; ++k) {
        float y = v[k] / s;
        q[k] = clamp_sym127(rne_to_int(y));
    }
}

/* bf16 activations [M, K] with row stride ldx -> int8 [M, K], fp32 [M]. */
void oracle_quant_rows_bf16(const bf16_t* x, int64_t M, int64_t K, int64_t ldx,
                            int8_t* q, float* s)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float* row = (float*)malloc(sizeof(float) * (size_t)K);
        for (int64_t k = 0; k < K; ++k) row[k] = oracle_bf16_to_f32(x[m * ldx + k]);
        oracle_quant_row_f32(row, K, q + m * K, s + m);
        free(row);
    }
}

/* fp32 rows [N, K] -> int8 [N, K], fp32 [N]  (the online weight quant). */
void oracle_quant_rows_f32(const float* w, int64_t N, int64_t K, int8_t* q, float* s)
{
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        oracle_quant_row_f32(w + n * K, K, q + n * K, s + n);
}

/* ------------------------------------------------------------------ */
/* a2: int8 x int8 -> int32, acc[m,n] = sum_k qa[m,k] * qb[n,k]         */
/* ([ATOM] "Changes": gemm_a8w8).  Accumulated in int64 and checked     */
/* against the int32 range; returns the number of overflowing entries.  */
/* ------------------------------------------------------------------ */
int64_t oracle_gemm_s32(const int8_t* qa, const int8_t* qb, int64_t M, int64_t N, int64_t K,
                        int32_t* acc)
{
    int64_t bad = 0;
    #pragma omp parallel for schedule(static) reduction(+:bad)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0;
            const int8_t* a = qa + m * K;
            const int8_t* b = qb + n * K;
            for (int64_t k = 0; k < K; ++k) sum += (int64_t)a[k] * (int64_t)b[k];
            if (sum > INT32_MAX || sum < INT32_MIN) bad += 1;
            acc[m * N + n] = (int32_t)sum;
        }
    }
    return bad;
}

/* The same contraction evaluated only at listed (m, n) pairs. */
void oracle_gemm_s32_at(const int8_t* qa, const int8_t* qb, int64_t K,
                        const int64_t* ms, const int64_t* ns, int64_t count, int32_t* acc)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const int8_t* a = qa + ms[i] * K;
        const int8_t* b = qb + ns[i] * K;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) sum += (int64_t)a[k] * (int64_t)b[k];
        acc[i] = (int32_t)sum;
    }
}

/* ------------------------------------------------------------------ */
/* a3: dequant epilogue.  y = bf16_rne( (float(acc) * s_x[m]) * s_w[n] )*/
/* fp32, left to right.  Optional fp32 and fp64 copies for the tests.   */
/* ------------------------------------------------------------------ */
static float dequant_one(int32_t acc, float sx, float sw)
{
    float r = (float)acc;          /* int32 -> fp32, round to nearest */
    r = r * sx;
    r = r * sw;
    return r;
}

void oracle_dequant(const int32_t* acc, const float* sx, const float* sw, int64_t M, int64_t N,
                    bf16_t* y, float* y32, double* y64)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int32_t a = acc[m * N + n];
            float r = dequant_one(a, sx[m], sw[n]);
            if (y) y[m * N + n] = oracle_f32_to_bf16(r);
            if (y32) y32[m * N + n] = r;
            if (y64) y64[m * N + n] = (double)a * (double)sx[m] * (double)sw[n];
        }
    }
}

/* The whole dense W8A8 linear: a1 on x, then a2 + a3 against (qw, sw).  */
void oracle_linear(const bf16_t* x, const int8_t* qw, const float* sw, int64_t M, int64_t N,
                   int64_t K, int8_t* qx_out, float* sx_out, bf16_t* y, float* y32)
{
    oracle_quant_rows_bf16(x, M, K, K, qx_out, sx_out);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* a = qx_out + m * K;
            const int8_t* b = qw + n * K;
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k) sum += (int64_t)a[k] * (int64_t)b[k];
            float r = dequant_one((int32_t)sum, sx_out[m], sw[n]);
            y[m * N + n] = oracle_f32_to_bf16(r);
            if (y32) y32[m * N + n] = r;
        }
    }
}

/* ------------------------------------------------------------------ */
/* exp_proj: the project's own fp32 exponential, used by the softmax of */
/* the router and by SiLU, so that both sides of the parity check take  */
/* the same fp32 steps.  Method: Cody & Waite (1980) argument reduction */
/* with a two-part ln 2, then the degree-7 Taylor polynomial of e^r     */
/* (coefficients 1/j!) in Horner form with fused multiply-adds, then    */
/* scaling by 2^n through the exponent field.  Input clamped to         */
/* [-87, 88] so that 2^n stays a normal number.                         */
/* ------------------------------------------------------------------ */
static const float EXPP_LOG2E  = 1.44269502162933349609375f;     /* fp32(log2 e) */
static const float EXPP_LN2_HI = 0.693359375f;                   /* 355/512, 9 bits */
static const float EXPP_LN2_LO = -2.12194440e-4f;                /* ln2 - 355/512 */

float oracle_exp_proj(float x)
{
    if (x > 88.0f) x = 88.0f;
    if (x < -87.0f) x = -87.0f;
    float t = x * EXPP_LOG2E;
    float n = (float)rne_to_int(t);
    float r = fmaf(-n, EXPP_LN2_HI, x);
    r = fmaf(-n, EXPP_LN2_LO, r);
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int32_t ni = (int32_t)n;
    uint32_t bits = (uint32_t)(ni + 127) << 23;   /* 2^n, n in [-126, 127] */
    float scale;
    memcpy(&scale, &bits, 4);
    return p * scale;
}

/* SiLU(g) = g / (1 + e^-g) ([ATOM] "Changes": fused gated-SiLU). */
float oracle_silu(float g)
{
    float e = oracle_exp_proj(-g);
    float d = 1.0f + e;
    return g / d;
}

void oracle_exp_proj_array(const float* x, float* y, int64_t n)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_exp_proj(x[i]);
}

void oracle_silu_array(const float* x, float* y, int64_t n)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_silu(x[i]);
}

void oracle_f32_to_bf16_array(const float* x, bf16_t* y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_f32_to_bf16(x[i]);
}

/* ------------------------------------------------------------------ */
/* a5: routing.  Router logits stay bf16 ([ATOM] "Precision split":    */
/* the MoE router gate is not quantized).  p = softmax(logits) in fp32  */
/* (subtract the max, exponentiate, sum in index order, divide); the    */
/* top-k experts are those with the largest logits (softmax is         */
/* monotone), ties to the lower expert index, listed in descending      */
/* order; their weights are p renormalised over the k selected.         */
/* ------------------------------------------------------------------ */
void oracle_route(const bf16_t* logits, int64_t T, int E, int topk, int32_t* ids, float* wts)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float* l = (float*)malloc(sizeof(float) * (size_t)E);
        float* p = (float*)malloc(sizeof(float) * (size_t)E);
        char* taken = (char*)calloc((size_t)E, 1);
        for (int e = 0; e < E; ++e) l[e] = oracle_bf16_to_f32(logits[t * E + e]);
        float mx = l[0];
        for (int e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
        float sum = 0.0f;
        for (int e = 0; e < E; ++e) { p[e] = oracle_exp_proj(l[e] - mx); sum = sum + p[e]; }
        for (int e = 0; e < E; ++e) p[e] = p[e] / sum;
        for (int j = 0; j < topk; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep the lower index */
            }
            taken[best] = 1;
            ids[t * topk + j] = best;
        }
        float ssel = 0.0f;
        for (int j = 0; j < topk; ++j) ssel = ssel + p[ids[t * topk + j]];
        for (int j = 0; j < topk; ++j) wts[t * topk + j] = p[ids[t * topk + j]] / ssel;
        free(l); free(p); free(taken);
    }
}

/* a6: histogram of routed rows by expert. */
void oracle_moe_histogram(const int32_t* ids, int64_t n, int E, int32_t* counts)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n; ++i) counts[ids[i]] += 1;
}

/* ------------------------------------------------------------------ */
/* a5-a11: routed W8A8 MoE expert layer for a list of tokens            */
/* ([ATOM] "Changes": routing -> per-token int8 quant -> gemm1 with     */
/* fused gated-SiLU via interleaved w13 -> per-token int8 quant ->      */
/* gemm2 with scatter/combine).                                         */
/*   w13 int8 [E, 2I, H], row 2i = gate_i, row 2i+1 = up_i; s13 [E, 2I] */
/*   w2  int8 [E, H, I];  s2 [E, H]                                      */
/* Per token t and slot j (expert e = ids[t,j]):                         */
/*   v_r  = (float(sum_h qx[t,h] w13[e,r,h]) * sx[t]) * s13[e,r]          */
/*   a_i  = SiLU(v_2i) * v_2i+1,  (qa, sa) = quant_row(a)                 */
/*   y2_n = (float(sum_i qa_i w2[e,n,i]) * sa) * s2[e,n]                  */
/*   out_n = sum over j = 0..k-1 of  wts[t,j] * y2_n   (fp32, slot order)*/
/* Outputs for each listed token (index i in 0..ntok-1 of `toks`):       */
/*   y [ntok, H] bf16, y32 [ntok, H], yabs [ntok, H] = sum_j |w*y2|,      */
/*   and optionally ids/wts [ntok,k], qx [ntok,H], sx [ntok],             */
/*   qa [ntok,k,I], sa [ntok,k].                                          */
/* ------------------------------------------------------------------ */
void oracle_moe_forward(const bf16_t* x, const bf16_t* logits,
                        const int8_t* w13, const float* s13,
                        const int8_t* w2, const float* s2,
                        int64_t T, int E, int H, int I, int topk,
                        const int64_t* toks, int64_t ntok,
                        bf16_t* y, float* y32, float* yabs,
                        int32_t* ids_out, float* wts_out,
                        int8_t* qx_out, float* sx_out,
                        int8_t* qa_out, float* sa_out)
{
    (void)T;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < ntok; ++i) {
        int64_t t = toks[i];
        int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)topk);
        float* wts = (float*)malloc(sizeof(float) * (size_t)topk);
        float* xr = (float*)malloc(sizeof(float) * (size_t)H);
        int8_t* qx = (int8_t*)malloc((size_t)H);
        float* v = (float*)malloc(sizeof(float) * (size_t)(2 * I));
        float* a = (float*)malloc(sizeof(float) * (size_t)I);
        int8_t* qa = (int8_t*)malloc((size_t)I);
        float* out = (float*)calloc((size_t)H, sizeof(float));
        float* oabs = (float*)calloc((size_t)H, sizeof(float));
        float sx, sa;

        oracle_route(logits + t * E, 1, E, topk, ids, wts);
        for (int h = 0; h < H; ++h) xr[h] = oracle_bf16_to_f32(x[t * H + h]);
        oracle_quant_row_f32(xr, H, qx, &sx);

        for (int j = 0; j < topk; ++j) {
            int e = ids[j];
            const int8_t* we = w13 + (int64_t)e * 2 * I * H;
            for (int r = 0; r < 2 * I; ++r) {
                int64_t sum = 0;
                for (int h = 0; h < H; ++h) sum += (int64_t)qx[h] * (int64_t)we[(int64_t)r * H + h];
                float vr = (float)(int32_t)sum;
                vr = vr * sx;
                vr = vr * s13[(int64_t)e * 2 * I + r];
                v[r] = vr;
            }
            for (int ii = 0; ii < I; ++ii) {
                float g = v[2 * ii];
                float u = v[2 * ii + 1];
                a[ii] = oracle_silu(g) * u;
            }
            oracle_quant_row_f32(a, I, qa, &sa);
            if (qa_out) memcpy(qa_out + (i * topk + j) * I, qa, (size_t)I);
            if (sa_out) sa_out[i * topk + j] = sa;
            const int8_t* w2e = w2 + (int64_t)e * H * I;
            for (int n = 0; n < H; ++n) {
                int64_t sum = 0;
                for (int ii = 0; ii < I; ++ii) sum += (int64_t)qa[ii] * (int64_t)w2e[(int64_t)n * I + ii];
                float y2 = (float)(int32_t)sum;
                y2 = y2 * sa;
                y2 = y2 * s2[(int64_t)e * H + n];
                float c = wts[j] * y2;
                out[n] = out[n] + c;
                oabs[n] = oabs[n] + fabsf(c);
            }
        }
        for (int n = 0; n < H; ++n) {
            if (y) y[i * H + n] = oracle_f32_to_bf16(out[n]);
            if (y32) y32[i * H + n] = out[n];
            if (yabs) yabs[i * H + n] = oabs[n];
        }
        if (ids_out) memcpy(ids_out + i * topk, ids, sizeof(int32_t) * (size_t)topk);
        if (wts_out) memcpy(wts_out + i * topk, wts, sizeof(float) * (size_t)topk);
        if (qx_out) memcpy(qx_out + i * H, qx, (size_t)H);
        if (sx_out) sx_out[i] = sx;
        free(ids); free(wts); free(xr); free(qx); free(v); free(a); free(qa); free(out); free(oabs);
    }
}

/* ------------------------------------------------------------------ */
/* Dense gated MLP block (the dense analogue of a8-a10: [ATOM] "Changes": */
/* gemm1 with fused gated-SiLU via interleaved w13 -> per-token int8     */
/* quant -> gemm2).  For each token m:                                   */
/*   (qx, sx) = quant_row(x[m])                                          */
/*   v_r  = (float(sum_h qx[h] w13[r,h]) * sx) * s13[r],  r < 2I         */
/*   a_i  = SiLU(v_2i) * v_2i+1;  (qa, sa) = quant_row(a)                */
/*   y_n  = bf16( (float(sum_i qa[i] w2[n,i]) * sa) * s2[n] )            */
/* w13 int8 [2I, H] (row 2i gate_i, 2i+1 up_i), s13 [2I]; w2 [H, I], s2 [H]. */
void oracle_mlp_forward(const bf16_t* x, const int8_t* w13, const float* s13,
                        const int8_t* w2, const float* s2, int64_t M, int H, int I,
                        bf16_t* y, float* y32, int8_t* qx_out, float* sx_out,
                        int8_t* qa_out, float* sa_out)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        float* xr = (float*)malloc(sizeof(float) * (size_t)H);
        int8_t* qx = (int8_t*)malloc((size_t)H);
        float* v = (float*)malloc(sizeof(float) * (size_t)(2 * I));
        float* a = (float*)malloc(sizeof(float) * (size_t)I);
        int8_t* qa = (int8_t*)malloc((size_t)I);
        float sx, sa;
        for (int h = 0; h < H; ++h) xr[h] = oracle_bf16_to_f32(x[m * H + h]);
        oracle_quant_row_f32(xr, H, qx, &sx);
        for (int r = 0; r < 2 * I; ++r) {
            int64_t sum = 0;
            for (int h = 0; h < H; ++h) sum += (int64_t)qx[h] * (int64_t)w13[(int64_t)r * H + h];
            float vr = (float)(int32_t)sum;
            vr = vr * sx;
            vr = vr * s13[r];
            v[r] = vr;
        }
        for (int i = 0; i < I; ++i) a[i] = oracle_silu(v[2 * i]) * v[2 * i + 1];
        oracle_quant_row_f32(a, I, qa, &sa);
        for (int n = 0; n < H; ++n) {
            int64_t sum = 0;
            for (int i = 0; i < I; ++i) sum += (int64_t)qa[i] * (int64_t)w2[(int64_t)n * I + i];
            float y2 = (float)(int32_t)sum;
            y2 = y2 * sa;
            y2 = y2 * s2[n];
            if (y) y[m * H + n] = oracle_f32_to_bf16(y2);
            if (y32) y32[m * H + n] = y2;
        }
        if (qx_out) memcpy(qx_out + m * H, qx, (size_t)H);
        if (sx_out) sx_out[m] = sx;
        if (qa_out) memcpy(qa_out + m * I, qa, (size_t)I);
        if (sa_out) sa_out[m] = sa;
        free(xr); free(qx); free(v); free(a); free(qa);
    }
}

/* ------------------------------------------------------------------ */
/* a12: FWHT128 group quantization ([IQ8R] file table: "each 128 of K   */
/* rotated by the unnormalised Hadamard", codes -127..127, a bf16 scale */
/* per row and 128 of K; recipe: transform=fwht128 group=128 scale=bf16 */
/* clamp=sym).                                                          */
/* The rotation is the textbook in-place fast Walsh-Hadamard transform  */
/* in fp32: stages h = 1, 2, 4, ..., 64, each pair (a, b) at distance h */
/* becoming (a + b, a - b).  This is H_128 x for the Sylvester matrix.  */
/* Scale: s = bf16_rne(absmax / 127); codes from the stored bf16 scale. */
/* ------------------------------------------------------------------ */
void oracle_fwht128(float* v)
{
    for (int h = 1; h < 128; h *= 2) {
        for (int i = 0; i < 128; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = v[j];
                float b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
}

/* One 128-wide block already in fp32: rotate it in place, then the bf16  */
/* scale and the codes from that stored scale.                           */
static bf16_t fwht128_quant_block(float* v, int8_t* q)
{
    oracle_fwht128(v);
    float amax = 0.0f;
    for (int k = 0; k < 128; ++k) { float a = fabsf(v[k]); if (a > amax) amax = a; }
    bf16_t sb = oracle_f32_to_bf16(amax / 127.0f);
    float sf = oracle_bf16_to_f32(sb);
    for (int k = 0; k < 128; ++k) {
        int8_t code = 0;
        if (sf != 0.0f) code = clamp_sym127(rne_to_int(v[k] / sf));
        q[k] = code;
    }
    return sb;
}

void oracle_fwht128_quant(const bf16_t* x, int64_t M, int64_t K, int8_t* q, bf16_t* s,
                          float* xr_out)
{
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float v[128];
        for (int64_t g = 0; g < G; ++g) {
            for (int k = 0; k < 128; ++k) v[k] = oracle_bf16_to_f32(x[m * K + g * 128 + k]);
            s[m * G + g] = fwht128_quant_block(v, q + m * K + g * 128);
            if (xr_out) for (int k = 0; k < 128; ++k) xr_out[m * K + g * 128 + k] = v[k];
        }
    }
}

/* The same for fp32 rows (the routed experts' gated intermediate). */
void oracle_fwht128_quant_f32(const float* x, int64_t M, int64_t K, int8_t* q, bf16_t* s)
{
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float v[128];
        for (int64_t g = 0; g < G; ++g) {
            for (int k = 0; k < 128; ++k) v[k] = x[m * K + g * 128 + k];
            s[m * G + g] = fwht128_quant_block(v, q + m * K + g * 128);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Group-128 quantization without the rotation (f3: [IQ8R] file table,  */
/* Head row: int8 codes, one bf16 scale per row and 128 of K, no         */
/* rotation listed; recipe row output.weight: codes=i8 group=128 scale=bf16 clamp=sym, no        */
/* transform).  Each 128-wide block of each row: s = bf16_rne(absmax /  */
/* 127), codes from that stored scale -- the block quantizer above       */
/* without the butterflies.                                              */
/* ------------------------------------------------------------------ */
void oracle_group128_quant(const bf16_t* x, int64_t M, int64_t K, int8_t* q, bf16_t* s)
{
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            float v[128];
            for (int k = 0; k < 128; ++k) v[k] = oracle_bf16_to_f32(x[m * K + g * 128 + k]);
            float amax = 0.0f;
            for (int k = 0; k < 128; ++k) { float a = fabsf(v[k]); if (a > amax) amax = a; }
            bf16_t sb = oracle_f32_to_bf16(amax / 127.0f);
            float sf = oracle_bf16_to_f32(sb);
            s[m * G + g] = sb;
            for (int k = 0; k < 128; ++k) {
                int8_t code = 0;
                if (sf != 0.0f) code = clamp_sym127(rne_to_int(v[k] / sf));
                q[m * K + g * 128 + k] = code;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* a13: group-128 scaled GEMM.                                          */
/*   p_g = sum_{k in group g} qx[m,k] qw[n,k]            (int32, exact)   */
/*   acc = fma(float(p_g), float(sx[m,g]) * float(sw[n,g]), acc), g asc  */
/*   y = bf16_rne(acc * post)                                             */
/* post = 1/128 in the rotated domain (it undoes H H^T = 128 I of the    */
/* unnormalised rotation), 1 on the unrotated grid of the head (f3).     */
/* ------------------------------------------------------------------ */
static void gemm_group_scaled(const int8_t* qx, const bf16_t* sx, const int8_t* qw, const bf16_t* sw,
                              int64_t M, int64_t N, int64_t K, float post, bf16_t* y, float* y32)
{
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int64_t g = 0; g < G; ++g) {
                int32_t p = 0;
                for (int k = 0; k < 128; ++k)
                    p += (int32_t)qx[m * K + g * 128 + k] * (int32_t)qw[n * K + g * 128 + k];
                float sc = oracle_bf16_to_f32(sx[m * G + g]) * oracle_bf16_to_f32(sw[n * G + g]);
                acc = fmaf((float)p, sc, acc);
            }
            float r = acc * post;
            if (y) y[m * N + n] = oracle_f32_to_bf16(r);
            if (y32) y32[m * N + n] = r;
        }
    }
}

void oracle_gemm_g128(const int8_t* qx, const bf16_t* sx, const int8_t* qw, const bf16_t* sw,
                      int64_t M, int64_t N, int64_t K, bf16_t* y, float* y32)
{
    gemm_group_scaled(qx, sx, qw, sw, M, N, K, 0.0078125f, y, y32);
}

void oracle_gemm_group128(const int8_t* qx, const bf16_t* sx, const int8_t* qw, const bf16_t* sw,
                          int64_t M, int64_t N, int64_t K, bf16_t* y, float* y32)
{
    gemm_group_scaled(qx, sx, qw, sw, M, N, K, 1.0f, y, y32);
}

/* ------------------------------------------------------------------ */
/* f4: the trunk linears' two-level scales ([IQ8R] file table, Trunk     */
/* row: int8 codes in -127..127, a u8 scale for each row and 256-wide    */
/* slice of K times a bf16 scale for the row, rows turned 128 at a time  */
/* by the unnormalised Hadamard matrix, rounding to nearest; recipe: codes=i8 group=256 scale=u8      */
/* scale2=bf16 block2=1x* transform=fwht128 clamp=sym rule=search).      */
/* Per row n of W (bf16 [N, K], K % 256 == 0), after the rotation of     */
/* each 128 of K:                                                         */
/*   scale2 = bf16_rne(max |w'| / (127 * 255))                            */
/*   for each 256-wide group j, u8[j] = the u in 1..255 whose scale      */
/*   s = float(u) * float(scale2) gives the smallest largest error        */
/*   max_k |w'_k - q_k * s|, q_k = clamp(rne(w'_k / s), +-127) (fp32,     */
/*   one rounding per operation; ties to the smaller u)                   */
/*   codes from the chosen s.  A zero row: scale2 = 0, u8 = 0, codes 0.   */
/* ------------------------------------------------------------------ */
static float trunk_group_error(const float* v, float s)
{
    float worst = 0.0f;
    for (int k = 0; k < 256; ++k) {
        int8_t c = clamp_sym127(rne_to_int(v[k] / s));
        float e = fabsf(v[k] - (float)c * s);
        if (e > worst) worst = e;
    }
    return worst;
}

void oracle_trunk_weight_quant(const bf16_t* w, int64_t N, int64_t K, int8_t* q, uint8_t* su8, bf16_t* s2)
{
    const int64_t G2 = K / 256;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; ++n) {
        float* v = (float*)malloc(sizeof(float) * (size_t)K);
        for (int64_t k = 0; k < K; ++k) v[k] = oracle_bf16_to_f32(w[n * K + k]);
        for (int64_t g = 0; g < K / 128; ++g) oracle_fwht128(v + g * 128);
        float rmax = 0.0f;
        for (int64_t k = 0; k < K; ++k) { float a = fabsf(v[k]); if (a > rmax) rmax = a; }
        bf16_t sb = oracle_f32_to_bf16(rmax / 32385.0f);
        float s2f = oracle_bf16_to_f32(sb);
        s2[n] = sb;
        for (int64_t j = 0; j < G2; ++j) {
            const float* vg = v + j * 256;
            int best = 0;
            if (s2f != 0.0f) {
                float best_err = INFINITY;
                for (int u = 1; u <= 255; ++u) {
                    float e = trunk_group_error(vg, (float)u * s2f);
                    if (e < best_err) { best_err = e; best = u; }
                }
            }
            su8[n * G2 + j] = (uint8_t)best;
            float s = (float)best * s2f;
            for (int k = 0; k < 256; ++k)
                q[n * K + j * 256 + k] = best ? clamp_sym127(rne_to_int(vg[k] / s)) : 0;
        }
        free(v);
    }
}

/* The trunk GEMM: x on the rotated grid of a12 (bf16 scale per token and  */
/* 128 of K), W in the two-level format above:                             */
/*   sw_g = float(u8[n, g / 2]) * float(scale2[n])      (exact in fp32)      */
/*   acc  = fma(float(p_g), float(sx[m, g]) * sw_g, acc), g ascending        */
/*   y    = bf16_rne(acc * (1/128))                                          */
void oracle_gemm_trunk(const int8_t* qx, const bf16_t* sx, const int8_t* qw, const uint8_t* su8,
                       const bf16_t* s2, int64_t M, int64_t N, int64_t K, bf16_t* y, float* y32)
{
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int64_t g = 0; g < G; ++g) {
                int32_t p = 0;
                for (int k = 0; k < 128; ++k)
                    p += (int32_t)qx[m * K + g * 128 + k] * (int32_t)qw[n * K + g * 128 + k];
                float swg = (float)su8[n * (K / 256) + g / 2] * oracle_bf16_to_f32(s2[n]);
                float sc = oracle_bf16_to_f32(sx[m * G + g]) * swg;
                acc = fmaf((float)p, sc, acc);
            }
            float r = acc * 0.0078125f;
            if (y) y[m * N + n] = oracle_f32_to_bf16(r);
            if (y32) y32[m * N + n] = r;
        }
    }
}

/* ------------------------------------------------------------------ */
/* f1: routed experts on the rotated grid ([IQ8R] file table, Experts    */
/* row: int8 codes on the rotated grid with one bf16 scale per row and   */
/* 128-wide slice of K; Activations row: activations quantized after the */
/* same rotation, the routed experts taking the trunk quantizer's codes; */
/* recipe rows                                                            */
/* ffn_gate_up_exps / ffn_down_exps: group=128 scale=bf16                 */
/* transform=fwht128).  The pipeline is that of oracle_moe_forward with  */
/* each quantizer replaced by the FWHT128 group quantizer and each GEMM  */
/* by the group-128 GEMM of oracle_gemm_g128.  Per token t and slot j    */
/* (expert e = ids[t,j]):                                                 */
/*   (qx, sx[g]) = fwht128_quant(x[t])           (rotation along H)       */
/*   v_r  = g128(qx, sx; w13[e,r], s13[e,r])     (fp32, not rounded)      */
/*   a_i  = SiLU(v_2i) * v_2i+1                                           */
/*   (qa, sa[g]) = fwht128_quant(a)              (rotation along I, fp32) */
/*   y2_n = g128(qa, sa; w2[e,n], s2[e,n])                                */
/*   out_n = sum over j = 0..k-1 of wts[t,j] * y2_n   (fp32, slot order)  */
/* with g128(qa, sa; qw, sw) = (sum over g ascending of                   */
/*   fma(float(p_g), float(sa[g]) * float(sw[g]), acc)) * (1/128).        */
/* w13 int8 [E, 2I, H] + bf16 [E, 2I, H/128]; w2 int8 [E, H, I] + bf16    */
/* [E, H, I/128] (rows rotated along K and group-quantized).              */
/* Outputs per listed token as in oracle_moe_forward, with the scales    */
/* bf16: sx [ntok, H/128], sa [ntok, k, I/128].                           */
/* ------------------------------------------------------------------ */
static float g128_dot(const int8_t* qa, const bf16_t* sa, const int8_t* qw, const bf16_t* sw, int64_t K)
{
    float acc = 0.0f;
    for (int64_t g = 0; g < K / 128; ++g) {
        int32_t p = 0;
        for (int k = 0; k < 128; ++k) p += (int32_t)qa[g * 128 + k] * (int32_t)qw[g * 128 + k];
        float sc = oracle_bf16_to_f32(sa[g]) * oracle_bf16_to_f32(sw[g]);
        acc = fmaf((float)p, sc, acc);
    }
    return acc * 0.0078125f;
}

void oracle_moe_g128_forward(const bf16_t* x, const bf16_t* logits,
                             const int8_t* w13, const bf16_t* s13,
                             const int8_t* w2, const bf16_t* s2,
                             int64_t T, int E, int H, int I, int topk,
                             const int64_t* toks, int64_t ntok,
                             bf16_t* y, float* y32, float* yabs,
                             int32_t* ids_out, float* wts_out,
                             int8_t* qx_out, bf16_t* sx_out,
                             int8_t* qa_out, bf16_t* sa_out)
{
    (void)T;
    const int GH = H / 128, GI = I / 128;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < ntok; ++i) {
        int64_t t = toks[i];
        int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)topk);
        float* wts = (float*)malloc(sizeof(float) * (size_t)topk);
        int8_t* qx = (int8_t*)malloc((size_t)H);
        bf16_t* sx = (bf16_t*)malloc(sizeof(bf16_t) * (size_t)GH);
        float* v = (float*)malloc(sizeof(float) * (size_t)(2 * I));
        float* a = (float*)malloc(sizeof(float) * (size_t)I);
        int8_t* qa = (int8_t*)malloc((size_t)I);
        bf16_t* sa = (bf16_t*)malloc(sizeof(bf16_t) * (size_t)GI);
        float* out = (float*)calloc((size_t)H, sizeof(float));
        float* oabs = (float*)calloc((size_t)H, sizeof(float));

        oracle_route(logits + t * E, 1, E, topk, ids, wts);
        oracle_fwht128_quant(x + t * H, 1, H, qx, sx, NULL);

        for (int j = 0; j < topk; ++j) {
            int e = ids[j];
            for (int r = 0; r < 2 * I; ++r) {
                int64_t wr = (int64_t)e * 2 * I + r;
                v[r] = g128_dot(qx, sx, w13 + wr * H, s13 + wr * GH, H);
            }
            for (int ii = 0; ii < I; ++ii) a[ii] = oracle_silu(v[2 * ii]) * v[2 * ii + 1];
            oracle_fwht128_quant_f32(a, 1, I, qa, sa);
            if (qa_out) memcpy(qa_out + (i * topk + j) * I, qa, (size_t)I);
            if (sa_out) memcpy(sa_out + (i * topk + j) * GI, sa, sizeof(bf16_t) * (size_t)GI);
            for (int n = 0; n < H; ++n) {
                int64_t wr = (int64_t)e * H + n;
                float y2 = g128_dot(qa, sa, w2 + wr * I, s2 + wr * GI, I);
                float c = wts[j] * y2;
                out[n] = out[n] + c;
                oabs[n] = oabs[n] + fabsf(c);
            }
        }
        for (int n = 0; n < H; ++n) {
            if (y) y[i * H + n] = oracle_f32_to_bf16(out[n]);
            if (y32) y32[i * H + n] = out[n];
            if (yabs) yabs[i * H + n] = oabs[n];
        }
        if (ids_out) memcpy(ids_out + i * topk, ids, sizeof(int32_t) * (size_t)topk);
        if (wts_out) memcpy(wts_out + i * topk, wts, sizeof(float) * (size_t)topk);
        if (qx_out) memcpy(qx_out + i * H, qx, (size_t)H);
        if (sx_out) memcpy(sx_out + i * GH, sx, sizeof(bf16_t) * (size_t)GH);
        free(ids); free(wts); free(qx); free(sx); free(v); free(a); free(qa); free(sa); free(out); free(oabs);
    }
}

/* ------------------------------------------------------------------ */
/* f3: the shared expert ([IQ8R] file table, Experts row: stored like the */
/* routed experts, its gate/up projection in the trunk's format; recipe   */
/* rows                                                                   */
/* ffn_gate_up_shexp: the trunk's two-level format, ffn_down_shexp:       */
/* group=128 scale=bf16 transform=fwht128).  A dense gated MLP on the     */
/* rotated grid, for each token m:                                         */
/*   (qx, sx[g]) = fwht128_quant(x[m])                                     */
/*   v_r = the trunk product of (qx, sx) with (w13[r], u8[r], scale2[r])   */
/*   a_i = SiLU(v_2i) * v_2i+1                                             */
/*   (qa, sa[g]) = fwht128_quant(a)               (rotation along I, fp32) */
/*   y_n = bf16( g128(qa, sa; w2[n], s2[n]) )                              */
/* w13 int8 [2I, H] + u8 [2I, H/256] + bf16 [2I]; w2 int8 [H, I] + bf16   */
/* [H, I/128].                                                             */
/* ------------------------------------------------------------------ */
void oracle_shared_expert_forward(const bf16_t* x, const int8_t* w13, const uint8_t* u13, const bf16_t* r13,
                                  const int8_t* w2, const bf16_t* s2, int64_t M, int H, int I,
                                  bf16_t* y, float* y32, int8_t* qx_out, bf16_t* sx_out,
                                  int8_t* qa_out, bf16_t* sa_out)
{
    const int GH = H / 128, GI = I / 128;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        int8_t* qx = (int8_t*)malloc((size_t)H);
        bf16_t* sx = (bf16_t*)malloc(sizeof(bf16_t) * (size_t)GH);
        float* v = (float*)malloc(sizeof(float) * (size_t)(2 * I));
        float* a = (float*)malloc(sizeof(float) * (size_t)I);
        int8_t* qa = (int8_t*)malloc((size_t)I);
        bf16_t* sa = (bf16_t*)malloc(sizeof(bf16_t) * (size_t)GI);
        oracle_fwht128_quant(x + m * H, 1, H, qx, sx, NULL);
        for (int r = 0; r < 2 * I; ++r)
            oracle_gemm_trunk(qx, sx, w13 + (int64_t)r * H, u13 + (int64_t)r * (H / 256), r13 + r, 1, 1, H,
                              NULL, v + r);
        for (int i = 0; i < I; ++i) a[i] = oracle_silu(v[2 * i]) * v[2 * i + 1];
        oracle_fwht128_quant_f32(a, 1, I, qa, sa);
        for (int n = 0; n < H; ++n) {
            float yn = g128_dot(qa, sa, w2 + (int64_t)n * I, s2 + (int64_t)n * GI, I);
            if (y) y[m * H + n] = oracle_f32_to_bf16(yn);
            if (y32) y32[m * H + n] = yn;
        }
        if (qx_out) memcpy(qx_out + m * H, qx, (size_t)H);
        if (sx_out) memcpy(sx_out + m * GH, sx, sizeof(bf16_t) * (size_t)GH);
        if (qa_out) memcpy(qa_out + m * I, qa, (size_t)I);
        if (sa_out) memcpy(sa_out + m * GI, sa, sizeof(bf16_t) * (size_t)GI);
        free(qx); free(sx); free(v); free(a); free(qa); free(sa);
    }
}

/* ------------------------------------------------------------------ */
/* Thread control for timing. */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
