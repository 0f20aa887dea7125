/*
 * csa_oracle.c -- plain, slow, fp64 CPU oracle for C4 compressed sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path may link, load or call
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or constant generator with
 * the CUDA kernels: every number format, the Hadamard matrix and every step of
 * the method is written out here from its definition.
 *
 * Pages cited (by title and section):
 *   [T] "Token 的一生：DSV4 架构与 DSpark" (SGLang DSV4 internals article)
 *       §1 从 DSA 到 DSV4, §2.1 什么是 C4, §2.2 C4 KV Cache 的尺寸,
 *       §3.1 FP4 量化支持, §3.2 Top-512 变换, §4 Hadamard 旋转
 *   [H] "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）：將百萬標記長上下文變為可用資源"
 *       section "Compressed Sparse Attention（CSA）" and section
 *       "低精度與儲存策略的配合"
 *
 * Where the pages are silent the readings taken are listed beside each
 * function.  All accumulation is in double; where a floating-point value
 * decides an integer code (a quantised element), the decision is taken in
 * float, the precision the kernels use, so that both sides round the same
 * quantity.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no -ffast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* OCP FP8 E4M3 ("e4m3fn"): sign, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, S.1111.111 is NaN, largest finite magnitude 448.  Used for
 * the FP8 index keys/queries ([T] §3.1) and the FP8 KV latent ([H] "低精度與
 * 儲存策略的配合"). */
double oracle_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);          /* subnormal */
    else        v = ldexp(1.0 + (double)m / 8.0, e - 7);  /* normal    */
    return s ? -v : v;
}

/* FP4 E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  Code in the low 4 bits. ([T] §3.1) */
double oracle_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v;
    if (e == 0) v = 0.5 * m;
    else        v = ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* Unsigned E4M3 block scale (the E4M3 byte with its sign bit zero), the
 * block-16 scale format of the FP4 index cache. */
double oracle_ue4m3_value(uint8_t code) { return oracle_e4m3_value(code & 0x7F); }

/* Round |x| to the nearest entry of an increasing table of magnitudes
 * value(0) < value(1) < ... < value(n-1); ties go to the even code; values
 * beyond the last entry saturate to it.  Codes are consecutive integers whose
 * lowest bit is the lowest mantissa bit, so "even code" is "even mantissa". */
static int nearest_code(double ax, double (*value)(uint8_t), int n)
{
    int lo = 0, hi = n - 1;
    if (!(ax > 0.0)) return 0;
    if (ax >= value((uint8_t)(n - 1))) return n - 1;
    /* find lo with value(lo) <= ax < value(lo + 1) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (value((uint8_t)mid) <= ax) lo = mid; else hi = mid;
    }
    {
        double dlo = ax - value((uint8_t)lo), dhi = value((uint8_t)hi) - ax;
        if (dlo < dhi) return lo;
        if (dhi < dlo) return hi;
        return (lo & 1) ? hi : lo;
    }
}

static double e4m3_mag(uint8_t c) { return oracle_e4m3_value(c); }
static double e2m1_mag(uint8_t c) { return oracle_e2m1_value(c); }

/* Round-to-nearest-even, saturating at +-448; the sign of x (including -0)
 * is kept. */
uint8_t oracle_e4m3_encode(double x)
{
    uint8_t s = signbit(x) ? 0x80 : 0x00;
    return (uint8_t)(s | nearest_code(fabs(x), e4m3_mag, 0x7F));
}

/* Round-to-nearest-even, saturating at +-6; sign kept. */
uint8_t oracle_e2m1_encode(double x)
{
    uint8_t s = signbit(x) ? 0x8 : 0x0;
    return (uint8_t)(s | nearest_code(fabs(x), e2m1_mag, 8));
}

/* Unsigned E4M3 scale: round-to-nearest-even of a non-negative value,
 * saturating at 448. */
uint8_t oracle_ue4m3_encode(double x)
{
    return (uint8_t)nearest_code(x > 0.0 ? x : 0.0, e4m3_mag, 0x7F);
}

/* bfloat16: 8 significant bits, float's exponent range.  Round to nearest,
 * ties to even, from a double. */
uint16_t oracle_bf16_encode(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    int e;
    double f, r, v;
    float vf;
    uint32_t bits;
    if (isnan(x)) return 0x7FC0;
    if (ax == 0.0) return sign;
    f = frexp(ax, &e);                 /* ax = f * 2^e, f in [0.5, 1) */
    if (e < -125) {                    /* bf16 subnormal: fixed quantum 2^-133 */
        r = nearbyint(ldexp(ax, 133));
        v = ldexp(r, -133);
    } else {
        r = nearbyint(ldexp(f, 8));    /* 8 significant bits, ties to even */
        v = ldexp(r, e - 8);
    }
    if (v > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80); /* inf */
    vf = (float)v;                     /* exact: v has <= 8 significant bits */
    memcpy(&bits, &vf, 4);
    return (uint16_t)(sign | (bits >> 16));
}

void oracle_bf16_encode_array(const double *x, long n, uint16_t *out)
{
    long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; i++) out[i] = oracle_bf16_encode(x[i]);
}

double oracle_bf16_value(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Hadamard rotation ([T] §4 Hadamard 旋转)                                  */
/* ------------------------------------------------------------------------ */

/* Sylvester construction: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].
 * out is n*n int8, row-major.  n must be a power of two. */
void oracle_hadamard_matrix(int n, int8_t *out)
{
    int size;
    out[0] = 1;
    for (size = 1; size < n; size *= 2) {
        int i, j;
        /* the current H_size sits in the top-left size x size corner of an
         * n-wide row-major array; fill the other three quadrants of H_2size */
        for (i = 0; i < size; i++)
            for (j = 0; j < size; j++) {
                int8_t h = out[i * n + j];
                out[i * n + (j + size)] = h;
                out[(i + size) * n + j] = h;
                out[(i + size) * n + (j + size)] = (int8_t)-h;
            }
    }
}

/* y = (1/sqrt(n)) H_n x for each of `rows` rows, by an explicit
 * matrix-vector product (no fast transform). */
void oracle_hadamard_rotate(const double *x, long rows, int n, double *y)
{
    int8_t *h = (int8_t *)malloc((size_t)n * n);
    double inv = 1.0 / sqrt((double)n);
    long r;
    oracle_hadamard_matrix(n, h);
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        int i, j;
        for (i = 0; i < n; i++) {
            double acc = 0.0;
            for (j = 0; j < n; j++) acc += (double)h[i * n + j] * x[r * n + j];
            y[r * n + i] = acc * inv;
        }
    }
    free(h);
}

/* ------------------------------------------------------------------------ */
/* Quantisers for the index queries/keys ([T] §3.1, §4)                     */
/* ------------------------------------------------------------------------ */

/* FP8: one fp32 scale per row, s = amax/448 (s = 1 for an all-zero row);
 * code = RNE(x/s) saturated to +-448, decided in float. */
void oracle_quant_fp8_rows(const double *x, long rows, int n,
                           uint8_t *codes, float *scales)
{
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        float amax = 0.0f, s;
        int i;
        for (i = 0; i < n; i++) {
            float v = fabsf((float)x[r * n + i]);
            if (v > amax) amax = v;
        }
        s = amax > 0.0f ? amax / 448.0f : 1.0f;
        for (i = 0; i < n; i++) {
            float q = (float)x[r * n + i] / s;
            codes[r * n + i] = oracle_e4m3_encode((double)q);
        }
        scales[r] = s;
    }
}

/* FP4 with two-level scales (the NVFP4 layout): a per-row fp32 scale
 * s_t = amax/(6*448) (1 for an all-zero row), and per 16-element block an
 * unsigned-E4M3 scale sb = RN(amax_blk / (6*s_t)); code = RNE(x/(sb*s_t))
 * saturated to +-6 (code 0, sign kept, where sb decodes to zero).  All
 * decisions in float.  codes: one E2M1 code per byte (unpacked), n per row;
 * block_scales: n/16 per row. */
void oracle_quant_fp4_rows(const double *x, long rows, int n, uint8_t *codes,
                           uint8_t *block_scales, float *row_scales)
{
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        float amax = 0.0f, st;
        int i, b;
        for (i = 0; i < n; i++) {
            float v = fabsf((float)x[r * n + i]);
            if (v > amax) amax = v;
        }
        st = amax > 0.0f ? amax / 2688.0f : 1.0f;
        for (b = 0; b < n / 16; b++) {
            float ab = 0.0f, six_st = 6.0f * st, sbv, dq;
            uint8_t sb;
            for (i = 0; i < 16; i++) {
                float v = fabsf((float)x[r * n + b * 16 + i]);
                if (v > ab) ab = v;
            }
            sbv = ab / six_st;
            sb = oracle_ue4m3_encode((double)sbv);
            dq = (float)oracle_ue4m3_value(sb) * st;
            for (i = 0; i < 16; i++) {
                float xv = (float)x[r * n + b * 16 + i];
                if (dq > 0.0f)
                    codes[r * n + b * 16 + i] = oracle_e2m1_encode((double)(xv / dq));
                else
                    codes[r * n + b * 16 + i] = signbit(xv) ? 0x8 : 0x0;
            }
            block_scales[r * (n / 16) + b] = sb;
        }
        row_scales[r] = st;
    }
}

/* Dequantise FP8 rows: x = e4m3(code) * s. */
void oracle_dequant_fp8_rows(const uint8_t *codes, const float *scales,
                             long rows, int n, double *x)
{
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        int i;
        for (i = 0; i < n; i++)
            x[r * n + i] = oracle_e4m3_value(codes[r * n + i]) * (double)scales[r];
    }
}

/* Dequantise FP4 rows: x = e2m1(code) * ue4m3(sb) * s_t. */
void oracle_dequant_fp4_rows(const uint8_t *codes, const uint8_t *block_scales,
                             const float *row_scales, long rows, int n, double *x)
{
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        int i;
        for (i = 0; i < n; i++)
            x[r * n + i] = oracle_e2m1_value(codes[r * n + i]) *
                           oracle_ue4m3_value(block_scales[r * (n / 16) + i / 16]) *
                           (double)row_scales[r];
    }
}

/* ------------------------------------------------------------------------ */
/* KV row format ([H] "低精度與儲存策略的配合": FP8 for most entries, BF16 for */
/* the RoPE dimensions).                                                     */
/*   FP8 row, 656 bytes: 512 E4M3 latent codes | 4 fp32 scales, one per      */
/*   128-channel block (s = amax/448, 1 for an all-zero block) | 64 bf16     */
/*   RoPE values.                                                            */
/*   BF16 row, 1152 bytes: 576 bf16 values.                                  */
/* ------------------------------------------------------------------------ */

#define KV_DIM 576
#define KV_LATENT 512

void oracle_kv_encode_rows(const double *x, long rows, int fp8, uint8_t *out)
{
    long r;
    int row_bytes = fp8 ? 656 : 1152;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        const double *xr = x + r * KV_DIM;
        uint8_t *o = out + r * row_bytes;
        int i, b;
        if (!fp8) {
            for (i = 0; i < KV_DIM; i++) {
                uint16_t h = oracle_bf16_encode(xr[i]);
                memcpy(o + 2 * i, &h, 2);
            }
            continue;
        }
        for (b = 0; b < 4; b++) {
            float amax = 0.0f, s;
            for (i = 0; i < 128; i++) {
                float v = fabsf((float)xr[b * 128 + i]);
                if (v > amax) amax = v;
            }
            s = amax > 0.0f ? amax / 448.0f : 1.0f;
            for (i = 0; i < 128; i++)
                o[b * 128 + i] = oracle_e4m3_encode((double)((float)xr[b * 128 + i] / s));
            memcpy(o + 512 + 4 * b, &s, 4);
        }
        for (i = 0; i < 64; i++) {
            uint16_t h = oracle_bf16_encode(xr[KV_LATENT + i]);
            memcpy(o + 528 + 2 * i, &h, 2);
        }
    }
}

void oracle_kv_decode_rows(const uint8_t *in, long rows, int fp8, double *x)
{
    long r;
    int row_bytes = fp8 ? 656 : 1152;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        const uint8_t *o = in + r * row_bytes;
        double *xr = x + r * KV_DIM;
        int i;
        if (!fp8) {
            for (i = 0; i < KV_DIM; i++) {
                uint16_t h;
                memcpy(&h, o + 2 * i, 2);
                xr[i] = oracle_bf16_value(h);
            }
            continue;
        }
        for (i = 0; i < KV_LATENT; i++) {
            float s;
            memcpy(&s, o + 512 + 4 * (i / 128), 4);
            xr[i] = oracle_e4m3_value(o[i]) * (double)s;
        }
        for (i = 0; i < 64; i++) {
            uint16_t h;
            memcpy(&h, o + 528 + 2 * i, 2);
            xr[KV_LATENT + i] = oracle_bf16_value(h);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Step 1: C4 compressor ([T] §2.1; [H] "Compressed Sparse Attention（CSA）"). */
/* ------------------------------------------------------------------------ */

/* Softmax-gated pooling with a learned positional bias.  The raw rows of one
 * request start at a block boundary; block j pools rows 4j..4j+3 and is
 * produced only when all four are present (the trigger at raw position
 * 4j+3), so floor(T/4) rows come out.  Per channel c:
 *   alpha_i = softmax_i(g[4j+i][c] + bias[i][c]),  y[j][c] = sum_i alpha_i x[4j+i][c].
 * Reading: the gate is per channel (gate logits have the KV row's shape) and
 * the bias is indexed by the position inside the block. */
long oracle_c4_compress(const double *x, const double *gate, const double *bias,
                        long T, int D, double *y)
{
    long nblk = T / 4, j;
#pragma omp parallel for schedule(static)
    for (j = 0; j < nblk; j++) {
        int c, i;
        for (c = 0; c < D; c++) {
            double z[4], m, e[4], Z = 0.0, acc = 0.0;
            for (i = 0; i < 4; i++) z[i] = gate[(4 * j + i) * D + c] + bias[i * D + c];
            m = z[0];
            for (i = 1; i < 4; i++) if (z[i] > m) m = z[i];
            for (i = 0; i < 4; i++) { e[i] = exp(z[i] - m); Z += e[i]; }
            for (i = 0; i < 4; i++) acc += (e[i] / Z) * x[(4 * j + i) * D + c];
            y[j * D + c] = acc;
        }
    }
    return nblk;
}

/* HCA compressor ([H] "Heavily Compressed Attention（HCA）"): the same
 * softmax-gated pooling with a per-position bias over blocks of `ratio` raw
 * rows (about 128 for HCA).  Block j pools rows ratio*j .. ratio*j+ratio-1 and
 * is produced only once all are present, so floor(T/ratio) rows come out.
 * Per channel c:  alpha_i = softmax_i(g[ratio*j+i][c] + bias[i][c]),
 *                 y[j][c] = sum_i alpha_i x[ratio*j+i][c]. */
long oracle_pool_compress(const double *x, const double *gate, const double *bias,
                          long T, int D, int ratio, double *y)
{
    long nblk = T / ratio, j;
#pragma omp parallel for schedule(static)
    for (j = 0; j < nblk; j++) {
        int c, i;
        for (c = 0; c < D; c++) {
            double m = -INFINITY, Z = 0.0, acc = 0.0;
            for (i = 0; i < ratio; i++) {
                double z = gate[(ratio * j + i) * (long)D + c] + bias[(long)i * D + c];
                if (z > m) m = z;
            }
            for (i = 0; i < ratio; i++) {
                double e = exp(gate[(ratio * j + i) * (long)D + c] + bias[(long)i * D + c] - m);
                Z += e;
                acc += e * x[(ratio * j + i) * (long)D + c];
            }
            y[j * D + c] = acc / Z;
        }
    }
    return nblk;
}

/* ------------------------------------------------------------------------ */
/* Step 2: indexer scores ([T] §1, §3.1; [H] "Compressed Sparse Attention"). */
/* ------------------------------------------------------------------------ */

/* logits[t][s] = sum_h w[t][h] * max(0, sum_d q[t][h][d] * k[s][d]) for
 * s < n_vis[t]; other entries of the row are left untouched.  q and k are
 * the dequantised (real-valued) queries and keys after the rotation. */
void oracle_indexer_logits(const double *q, const double *w, long nq, int Hi, int Di,
                           const double *k, const long *n_vis, double *logits,
                           long logits_stride)
{
    long t;
    for (t = 0; t < nq; t++) {
        long s, nv = n_vis[t];
#pragma omp parallel for schedule(static)
        for (s = 0; s < nv; s++) {
            double acc = 0.0;
            int h, d;
            for (h = 0; h < Hi; h++) {
                double dot = 0.0;
                for (d = 0; d < Di; d++)
                    dot += q[(t * Hi + h) * Di + d] * k[s * Di + d];
                acc += w[t * Hi + h] * (dot > 0.0 ? dot : 0.0);
            }
            logits[t * logits_stride + s] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Step 3: fixed top-512 and the paged index transform ([T] §3.2, §2.2).    */
/* ------------------------------------------------------------------------ */

typedef struct { float v; long i; } scored_t;

/* Larger score first; equal scores keep the lower index first, so this
 * total order is exactly a stable descending sort. */
static int by_score_desc(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int by_index(const void *a, const void *b)
{
    long x = *(const long *)a, y = *(const long *)b;
    return (x > y) - (x < y);
}

/* Selects the min(K, n_vis) logical compressed indices with the largest
 * logits (ties: lower index), lists them in ascending logical order, pads
 * with -1 to K, and maps each through the page table:
 *   physical = page_table[s / c4_page_size] * c4_page_size + s % c4_page_size.
 * Scores are float (the logits' stored type); -0 and +0 compare equal.
 * Returns the number selected, or -1 if a page id is out of [0, num_slots). */
long oracle_topk_transform(const float *logits, long n_vis, int K,
                           const int *page_table, int c4_page_size, long num_slots,
                           int *phys_out, int *logical_out)
{
    scored_t *all = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n_vis > 0 ? n_vis : 1));
    long *sel = (long *)malloc(sizeof(long) * (size_t)K);
    long s, n_sel = n_vis < K ? n_vis : K, r, bad = 0;
    for (s = 0; s < n_vis; s++) { all[s].v = logits[s]; all[s].i = s; }
    qsort(all, (size_t)n_vis, sizeof(scored_t), by_score_desc);
    for (r = 0; r < n_sel; r++) sel[r] = all[r].i;
    qsort(sel, (size_t)n_sel, sizeof(long), by_index);
    for (r = 0; r < K; r++) {
        if (r < n_sel) {
            long lg = sel[r];
            long page = page_table[lg / c4_page_size];
            long phys = page * c4_page_size + lg % c4_page_size;
            if (page < 0 || phys >= num_slots) bad = 1;
            phys_out[r] = (int)phys;
            if (logical_out) logical_out[r] = (int)lg;
        } else {
            phys_out[r] = -1;
            if (logical_out) logical_out[r] = -1;
        }
    }
    free(all);
    free(sel);
    return bad ? -1 : n_sel;
}

/* ------------------------------------------------------------------------ */
/* Step 4: sparse attention over the selected compressed rows joined with   */
/* the sliding window of raw rows, one softmax over both ([T] §1;           */
/* [H] "Compressed Sparse Attention（CSA）").                                */
/* ------------------------------------------------------------------------ */

/* q: [H][576]; rows: [R][576] dequantised key rows (selected compressed rows
 * and window rows together); values are the first 512 dims of each row.
 *   z[h][r] = tau * q[h] . rows[r];  p = softmax_r(z);  o[h] = sum_r p[h][r] rows[r][0:512]
 * lse[h] = log(sum_r exp(z[h][r])).  R = 0 gives o = 0 and lse = -inf. */
void oracle_sparse_attention(const double *q, int H, const double *rows, long R,
                             double tau, double *out, double *lse)
{
    int h;
#pragma omp parallel for schedule(static)
    for (h = 0; h < H; h++) {
        double *z = (double *)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1));
        double m = -INFINITY, Z = 0.0;
        long r;
        int c;
        for (r = 0; r < R; r++) {
            double dot = 0.0;
            int d;
            for (d = 0; d < KV_DIM; d++) dot += q[h * KV_DIM + d] * rows[r * KV_DIM + d];
            z[r] = tau * dot;
            if (z[r] > m) m = z[r];
        }
        for (r = 0; r < R; r++) Z += exp(z[r] - m);
        for (c = 0; c < KV_LATENT; c++) {
            double acc = 0.0;
            for (r = 0; r < R; r++) acc += exp(z[r] - m) / Z * rows[r * KV_DIM + c];
            out[h * KV_LATENT + c] = R > 0 ? acc : 0.0;
        }
        lse[h] = R > 0 ? m + log(Z) : -INFINITY;
        free(z);
    }
}

/* Number of threads the oracle's parallel loops use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
