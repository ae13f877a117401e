/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for the tree-MTP
 * verification step.  TEST INFRASTRUCTURE ONLY: it is loaded by tests/,
 * by __graft_entry__.smoke() and by the cpu_baseline leg of bench.py, never
 * by the product path.  It shares no code, header, table or constant with
 * the CUDA library; it depends on libc, libm and OpenMP only.
 *
 * Sources of what is computed (cited by page title and section):
 *   [EDGE] "TensorRT Edge-LLM Completes the MLPerf Edge Agentic Benchmark 6.4x
 *          Faster on Jetson AGX Thor" (spbcomputers.ru, mechatronicstore.cl,
 *          ai4snews copies):
 *          - section "NVFP4 and FP8" (NVFP4 for weights AND activations,
 *            LM head included; FP8 KV cache; low-batch decode is DRAM bound);
 *          - section "KV-cache reuse between agent steps" (cached attention KV
 *            pages are restored);
 *          - section "Tree multi-token prediction" (16-node verification tree,
 *            8 draft steps, top-2 per depth, verified in one forward pass).
 *   [MX]   OCP Microscaling Formats (MX) v1.0, FP4 E2M1 element format.
 *   [OFP8] OCP 8-bit Floating Point Specification (OFP8), E4M3 ("fn": no
 *          infinities, S.1111.111 is NaN, max finite 448).
 * The pages name the formats but do not spell out the bit-level recipe; the
 * readings taken where they are silent are stated in the comments below.
 *
 * Arithmetic: fp64 throughout.  Where the quantisation recipe is defined as a
 * sequence of IEEE fp32 operations, each single fp32 operation is emulated by
 * computing it in fp64 and rounding once to fp32; for one +,-,*,/ this equals
 * the correctly rounded fp32 result (53 >= 2*24+2).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Codecs, decoded from the bit-field definitions                           */
/* ------------------------------------------------------------------------ */

/* [MX] E2M1: sign s, 2 exponent bits e (bias 1), 1 mantissa bit m.
 * e == 0 is subnormal: m * 2^(1-1) * 0.5; otherwise (1 + m/2) * 2^(e-1). */
EXPORT double oracle_e2m1_value(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
    return s ? -mag : mag;
}

/* [OFP8] E4M3: sign s, 4 exponent bits e (bias 7), 3 mantissa bits m.
 * e == 0 is subnormal: (m/8) * 2^-6.  e == 15 && m == 7 is NaN; there are no
 * infinities, so e == 15 with m < 7 are ordinary normals (max 448). */
EXPORT double oracle_e4m3_value(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? (m / 8.0) * ldexp(1.0, -6)
                          : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -mag : mag;
}

EXPORT void oracle_e2m1_table(double *out16)
{
    for (int c = 0; c < 16; ++c) out16[c] = oracle_e2m1_value(c);
}

EXPORT void oracle_e4m3_table(double *out256)
{
    for (int c = 0; c < 256; ++c) out256[c] = oracle_e4m3_value(c);
}

/* Round-to-nearest-even onto the non-negative codes 0..max_code of a format
 * whose magnitudes grow with the code; values at or above the largest finite
 * magnitude saturate to it ("satfinite").  Ties go to the even code, which is
 * the code whose mantissa LSB (bit 0) is 0. */
static int rne_code(double a, int max_code, double (*value)(int))
{
    if (a >= value(max_code)) return max_code;
    int lo = 0, hi = max_code;              /* value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (value(mid) <= a) lo = mid; else hi = mid;
    }
    double dlo = a - value(lo), dhi = value(hi) - a;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1) ? hi : lo;
}

/* E2M1 encode with RNE + satfinite; the sign bit is copied from the input,
 * so -0 and negative values that round to zero give code 0x8. */
EXPORT int oracle_e2m1_encode(double v)
{
    int s = signbit(v) ? 1 : 0;
    return (s << 3) | rne_code(fabs(v), 7, oracle_e2m1_value);
}

/* E4M3 encode with RNE + satfinite (|v| >= 448 -> 448); sign copied. */
EXPORT int oracle_e4m3_encode(double v)
{
    int s = signbit(v) ? 1 : 0;
    return (s << 7) | rne_code(fabs(v), 0x7E, oracle_e4m3_value);
}

/* Element-wise encode of a float array into one code per byte (diagnostics
 * for the exhaustive conversion check). */
EXPORT void oracle_encode_many(const float *x, int64_t n, uint8_t *e2m1, uint8_t *e4m3)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        if (e2m1) e2m1[i] = (uint8_t)oracle_e2m1_encode((double)x[i]);
        if (e4m3) e4m3[i] = (uint8_t)oracle_e4m3_encode((double)x[i]);
    }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantisation ([EDGE] "NVFP4 and FP8"; format per BASELINE configs:  */
/* E2M1 elements, one E4M3 scale per 16 contiguous K elements, fp32 tensor   */
/* scale amax / (6 * 448)).                                                  */
/* ------------------------------------------------------------------------ */

static float f32(double v) { return (float)v; }   /* one rounding to fp32 */

/* Tensor scale g = fp32(amax / 2688); reading: amax == 0 gives g = 1. */
EXPORT float oracle_nvfp4_tensor_scale(const float *x, int64_t n)
{
    double amax = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double a = fabs((double)x[i]);
        if (a > amax) amax = a;
    }
    return amax > 0.0 ? f32(amax / 2688.0) : 1.0f;
}

/* Quantise x[rows][K] (K % 16 == 0).  If g_in is non-NULL it is used as the
 * tensor scale, otherwise g = oracle_nvfp4_tensor_scale(x).  Per 16-block:
 *   r = fp32(amax_b / 6); t = fp32(r / g); scale = E4M3_rne_sat(t);
 *   s = fp32(value(scale) * g);
 *   code_k = s == 0 ? +0 : E2M1_rne_sat(fp32(x_k / s)).
 * Codes are packed two per byte, even K index in the low nibble.
 * Returns 0, or -1 if K is not a multiple of 16. */
EXPORT int oracle_nvfp4_quantize(const float *x, int64_t rows, int64_t K, const float *g_in,
                                 uint8_t *codes, uint8_t *scales, float *g_out)
{
    if (K % 16 != 0) return -1;
    float g = g_in ? *g_in : oracle_nvfp4_tensor_scale(x, rows * K);
    if (g_out) *g_out = g;
    int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float *xb = x + r * K + b * 16;
            double amax_b = 0.0;
            for (int k = 0; k < 16; ++k)
                if (fabs((double)xb[k]) > amax_b) amax_b = fabs((double)xb[k]);
            float rr = f32(amax_b / 6.0);
            float t = f32((double)rr / (double)g);
            int sc = oracle_e4m3_encode((double)t);
            scales[r * nb + b] = (uint8_t)sc;
            float s = f32(oracle_e4m3_value(sc) * (double)g);
            uint8_t c[16];
            for (int k = 0; k < 16; ++k) {
                if (s == 0.0f) c[k] = 0;
                else c[k] = (uint8_t)oracle_e2m1_encode((double)f32((double)xb[k] / (double)s));
            }
            for (int k = 0; k < 16; k += 2)
                codes[r * (K / 2) + b * 8 + k / 2] = (uint8_t)(c[k] | (c[k + 1] << 4));
        }
    }
    return 0;
}

static int nibble(const uint8_t *codes_row, int64_t k)
{
    uint8_t byte = codes_row[k / 2];
    return (k & 1) ? (byte >> 4) : (byte & 15);
}

/* Dequantised value of element (r, k): g * value(scale) * value(code). */
EXPORT void oracle_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, float g,
                                    int64_t rows, int64_t K, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = (double)g * oracle_e4m3_value(scales[r * (K / 16) + k / 16])
                             * oracle_e2m1_value(nibble(codes + r * (K / 2), k));
}

/* One output of the W4A4 linear layer, Y = A W^T:
 *   y[m,n] = g_a g_w sum_b s_a[m,b] s_w[n,b] sum_{k in b} a[m,k] w[n,k]
 * where a, w are E2M1 values and s are E4M3 block-scale values (fp64). */
static double linear_one(const uint8_t *a_codes, const uint8_t *a_scales, float g_a,
                         const uint8_t *w_codes, const uint8_t *w_scales, float g_w,
                         int64_t K, int64_t m, int64_t n)
{
    const uint8_t *ar = a_codes + m * (K / 2), *wr = w_codes + n * (K / 2);
    double acc = 0.0;
    for (int64_t b = 0; b < K / 16; ++b) {
        double blk = 0.0;
        for (int64_t k = b * 16; k < b * 16 + 16; ++k)
            blk += oracle_e2m1_value(nibble(ar, k)) * oracle_e2m1_value(nibble(wr, k));
        acc += oracle_e4m3_value(a_scales[m * (K / 16) + b])
             * oracle_e4m3_value(w_scales[n * (K / 16) + b]) * blk;
    }
    return (double)g_a * (double)g_w * acc;
}

/* Full Y[M][N] (fp64). */
EXPORT void oracle_nvfp4_linear(const uint8_t *a_codes, const uint8_t *a_scales, float g_a, int64_t M,
                                const uint8_t *w_codes, const uint8_t *w_scales, float g_w,
                                int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(dynamic, 64) collapse(2)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m)
            y[m * N + n] = linear_one(a_codes, a_scales, g_a, w_codes, w_scales, g_w, K, m, n);
}

/* Selected outputs y[idx_m[i], idx_n[i]] only (for full-size shapes). */
EXPORT void oracle_nvfp4_linear_sampled(const uint8_t *a_codes, const uint8_t *a_scales, float g_a,
                                        const uint8_t *w_codes, const uint8_t *w_scales, float g_w,
                                        int64_t K, const int64_t *idx_m, const int64_t *idx_n,
                                        int64_t n_samples, double *y)
{
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n_samples; ++i)
        y[i] = linear_one(a_codes, a_scales, g_a, w_codes, w_scales, g_w, K, idx_m[i], idx_n[i]);
}

/* ------------------------------------------------------------------------ */
/* Tree-masked attention over an FP8 paged KV cache ([EDGE] "Tree multi-     */
/* token prediction": candidates organised into a tree and verified in one   */
/* target forward; "NVFP4 and FP8": FP8 KV cache; "KV-cache reuse": pages).  */
/*                                                                           */
/* Cache layout (per layer): K pool uint8 [n_pages][Hkv][P][D] (token-major  */
/* page), V pool uint8 [n_pages][Hkv][D*P]: a (page, head) plane of V is cut */
/* into 8-dimension x 16-slot tiles of 128 bytes, tile (d/8, slot/16) at     */
/* tile index (d/8)*(P/16) + slot/16, rows d%8 of 16 slots inside (v_byte    */
/* below; needs D % 8 == 0 and P % 16 == 0).  Logical                        */
/* position p lives in physical page page_table[p / P], slot p % P.  The     */
/* tree nodes' own K/V sit at positions L .. L+T-1 (node i at L+i).          */
/* Node i sees every context position p < L and the tree positions of its    */
/* ancestors and itself: anc(i) = {i} u anc(parent(i)), anc(-1) = {}.        */
/* Query head hq uses KV head hq / (Hq / Hkv).                               */
/*   s_p = sm_scale * sum_d q[d] * k_scale[h] * value(K code)                */
/*   o   = sum_p softmax(s)_p * v_scale[h] * value(V code)   (fp64)          */
/* ------------------------------------------------------------------------ */

/* byte offset of (dimension d, slot) inside one V plane */
static int64_t v_byte(int d, int slot, int P)
{
    int64_t tile = (int64_t)(d / 8) * (P / 16) + slot / 16;
    return tile * 128 + (d % 8) * 16 + slot % 16;
}

static int is_ancestor(const int32_t *parent, int j, int i)
{
    for (int a = i; a >= 0; a = parent[a])
        if (a == j) return 1;
    return 0;
}

EXPORT int oracle_tree_attn(const float *q, int T, int Hq, int Hkv, int D,
                            const uint8_t *k_pool, const uint8_t *v_pool, int64_t n_pages, int P,
                            const int32_t *page_table, int64_t L, const int32_t *parent,
                            const float *k_scale, const float *v_scale, double sm_scale,
                            double *out)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || D % 8 != 0 || P % 16 != 0) return -1;
    int group = Hq / Hkv;
    int64_t total = L + T;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2) reduction(| : bad)
    for (int i = 0; i < T; ++i) {
        for (int hq = 0; hq < Hq; ++hq) {
            int h = hq / group;
            const float *qi = q + ((int64_t)i * Hq + hq) * D;
            double *o = out + ((int64_t)i * Hq + hq) * D;
            double *s = (double *)malloc(sizeof(double) * (size_t)total);
            char *vis = (char *)malloc((size_t)total);
            double smax = -INFINITY;
            for (int64_t p = 0; p < total; ++p) {
                vis[p] = (p < L) || is_ancestor(parent, (int)(p - L), i);
                if (!vis[p]) continue;
                int64_t pg = page_table[p / P];
                if (pg < 0 || pg >= n_pages) { bad = 1; vis[p] = 0; continue; }
                const uint8_t *kr = k_pool + ((pg * Hkv + h) * P + p % P) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += (double)qi[d] * ((double)k_scale[h] * oracle_e4m3_value(kr[d]));
                s[p] = sm_scale * dot;
                if (s[p] > smax) smax = s[p];
            }
            double den = 0.0;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t p = 0; p < total; ++p) {
                if (!vis[p]) continue;
                double w = exp(s[p] - smax);
                den += w;
                int64_t pg = page_table[p / P];
                const uint8_t *vb = v_pool + (pg * Hkv + h) * (int64_t)D * P;
                for (int d = 0; d < D; ++d)
                    o[d] += w * ((double)v_scale[h] * oracle_e4m3_value(vb[v_byte(d, (int)(p % P), P)]));
            }
            for (int d = 0; d < D; ++d) o[d] /= den;
            free(s);
            free(vis);
        }
    }
    return bad ? -7 : 0;
}

/* Write the T new tokens' K/V (fp32 values [T][Hkv][D]) into the cache at
 * positions L .. L+T-1 as E4M3 codes of fp32(x / scale[h]) (RNE, satfinite).
 * This is the FP8 KV cache write of [EDGE] "NVFP4 and FP8". */
EXPORT int oracle_kv_append(const float *k_new, const float *v_new, int T, int Hkv, int D,
                            uint8_t *k_pool, uint8_t *v_pool, int64_t n_pages, int P,
                            const int32_t *page_table, int64_t L,
                            const float *k_scale, const float *v_scale)
{
    if (D % 8 != 0 || P % 16 != 0) return -1;
    for (int i = 0; i < T; ++i) {
        int64_t p = L + i, pg = page_table[p / P], slot = p % P;
        if (pg < 0 || pg >= n_pages) return -7;
        for (int h = 0; h < Hkv; ++h)
            for (int d = 0; d < D; ++d) {
                double kx = f32((double)k_new[((int64_t)i * Hkv + h) * D + d] / (double)k_scale[h]);
                double vx = f32((double)v_new[((int64_t)i * Hkv + h) * D + d] / (double)v_scale[h]);
                k_pool[((pg * Hkv + h) * P + slot) * D + d] = (uint8_t)oracle_e4m3_encode(kx);
                v_pool[(pg * Hkv + h) * (int64_t)D * P + v_byte(d, (int)slot, P)] = (uint8_t)oracle_e4m3_encode(vx);
            }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Prefix-cache restore ([EDGE] "KV-cache reuse between agent steps": the    */
/* runtime restores the cached attention KV pages of a reused prefix):       */
/* dst page dst_ids[i] <- src page src_ids[i], page_bytes each.              */
/* ------------------------------------------------------------------------ */
EXPORT int oracle_kv_page_restore(const uint8_t *src_pool, const int32_t *src_ids,
                                  uint8_t *dst_pool, const int32_t *dst_ids, int64_t n,
                                  int64_t page_bytes, int64_t n_src_pages, int64_t n_dst_pages)
{
    for (int64_t i = 0; i < n; ++i) {
        if (src_ids[i] < 0 || src_ids[i] >= n_src_pages || dst_ids[i] < 0 || dst_ids[i] >= n_dst_pages)
            return -7;
        memcpy(dst_pool + (int64_t)dst_ids[i] * page_bytes, src_pool + (int64_t)src_ids[i] * page_bytes,
               (size_t)page_bytes);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Layer glue of the dense 27B-class verify step (not on the pages; the      */
/* readings are stated with each function): RMSNorm, SwiGLU.                 */
/* ------------------------------------------------------------------------ */

/* y = x / sqrt(mean(x^2) + eps) * w, per row of length n. */
EXPORT void oracle_rmsnorm(const float *x, int64_t rows, int64_t n, const float *w, double eps, double *out)
{
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int64_t j = 0; j < n; ++j) ss += (double)x[r * n + j] * (double)x[r * n + j];
        double inv = 1.0 / sqrt(ss / (double)n + eps);
        for (int64_t j = 0; j < n; ++j) out[r * n + j] = (double)x[r * n + j] * inv * (double)w[j];
    }
}

/* out[r][j] = silu(gu[r][j]) * gu[r][F + j], silu(x) = x / (1 + e^-x). */
EXPORT void oracle_swiglu(const float *gu, int64_t rows, int64_t F, double *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < F; ++j) {
            double gx = gu[r * 2 * F + j], ux = gu[r * 2 * F + F + j];
            out[r * F + j] = gx / (1.0 + exp(-gx)) * ux;
        }
}
