/*
 * oracle.c -- float64 CPU reference for causal grouped-query attention with
 * rotary position embedding, optional QK-RMSNorm, and the KV-cache decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load this file or
 * the library built from it: only the tests, the package entry's smoke check and
 * the benchmark's CPU-baseline leg do.  It shares no code with the CUDA library.
 *
 * Everything is written as the plain definition, in float64, with no blocking,
 * no fusion and no reordering beyond what the definition states:
 *
 *   RMSNorm (unit gain)  y = x / sqrt(mean_d(x_d^2) + eps)
 *       Page "训练3.8B LLM至0.384 CORE，成本998美元 – Hugo Vergnes", section
 *       "设置" (QK-norm in the final Llama-style model) and section "无效的方法"
 *       (the built-in F.rms_norm, whose eps sits inside the square root).
 *
 *   RoPE  rotate coordinate pairs of q and k by angle p * theta_i,
 *         theta_i = base^(-2i/D), i = 0 .. D/2-1, so that q_m . k_n depends on
 *         m - n only.
 *       Page "750美元从零训练3个LLM：一位开发者的实战复盘", section "V1：现代架构基线"
 *       (RoPE item); page "从零手训LLaMa：125M模型11小时训练全记录", section
 *       "核心架构：手动实现LLaMa的四个关键组件".
 *
 *   GQA   query head h reads key/value head floor(h / g), g = Hq / Hkv.
 *       Page "750美元从零训练3个LLM", section "V2：引入前沿技术" (GQA item:
 *       query heads are split into groups, each group shares one K/V projection).
 *
 *   Causal scaled-dot-product attention
 *         o = sum_{u visible} softmax_u(q . k_u * scale) v_u,
 *         visible = keys at positions 0 .. qpos (inclusive), scale = 1/sqrt(D).
 *       Page "训练3.8B LLM…", section "无效的方法" (attention returns to an
 *       unconditional causal scaled_dot_product_attention); page "Build a Large
 *       Language Model from Scratch" (nxbn.cn), section 3.1 (the causal mask is
 *       handled inside the library call, default scale).
 *
 *   KV cache: the new token computes its own q, k, v, the k/v are appended to
 *         the cache and q attends over the cache including itself.
 *       Page "750美元从零训练3个LLM", section "V3：扩容与推理优化".
 *
 * Layouts (all row-major, float64 unless noted):
 *   q [B, Tq, Hq, D]   k, v [B, Tk, Hkv, D]   qpos [B, Tq] (int64)
 *   o [B, Tq, Hq, D]   one output "row" = one (b, t, h) triple,
 *                      flat index r = (b * Tq + t) * Hq + h.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bfloat16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void oracle_bf16_to_f64(const uint16_t *src, double *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = bf16_bits_to_double(src[i]);
}

/* RMSNorm with unit gain over each row of D values. */
void oracle_rmsnorm(const double *x, double *y, int64_t rows, int D, double eps)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * D;
        double *yr = y + r * D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d)
            ss += xr[d] * xr[d];
        double inv = 1.0 / sqrt(ss / (double)D + eps);
        for (int d = 0; d < D; ++d)
            yr[d] = xr[d] * inv;
    }
}

/*
 * RoPE over x [N, H, D]: token n sits at position pos[n].  For pair i the two
 * rotated coordinates are (a, b) = (i, i + D/2) when interleaved == 0 (halves
 * pairing) or (2i, 2i + 1) when interleaved != 0; the rotation is
 *   x_a' = x_a cos(p th_i) - x_b sin(p th_i)
 *   x_b' = x_a sin(p th_i) + x_b cos(p th_i).
 * oracle_rope_theta takes the table th_i (the context-extension variants change
 * only the table); oracle_rope builds the plain one, th_i = base^(-2i/D).
 */
void oracle_rope_theta(const double *x, double *y, const int64_t *pos, int64_t N, int H,
                       int D, const double *theta, int interleaved)
{
    int half = D / 2;
    for (int64_t n = 0; n < N; ++n) {
        double p = (double)pos[n];
        for (int h = 0; h < H; ++h) {
            const double *xr = x + (n * H + h) * D;
            double *yr = y + (n * H + h) * D;
            for (int i = 0; i < half; ++i) {
                double ang = p * theta[i];
                double c = cos(ang), s = sin(ang);
                int ia = interleaved ? 2 * i : i;
                int ib = interleaved ? 2 * i + 1 : i + half;
                double xa = xr[ia], xb = xr[ib];
                yr[ia] = xa * c - xb * s;
                yr[ib] = xa * s + xb * c;
            }
        }
    }
}

/* Plain RoPE: the table theta_i = base^(-2i/D). */
void oracle_rope(const double *x, double *y, const int64_t *pos, int64_t N, int H,
                 int D, double base, int interleaved)
{
    int half = D / 2;
    double *theta = (double *)malloc(sizeof(double) * (size_t)(half > 0 ? half : 1));
    for (int i = 0; i < half; ++i)
        theta[i] = pow(base, -2.0 * (double)i / (double)D);
    oracle_rope_theta(x, y, pos, N, H, D, theta, interleaved);
    free(theta);
}

/*
 * One output row: softmax over visible keys, then the weighted sum of values.
 * With document ids (qdoc [B, Tq], kdoc [B, Tk]; NULL for none) a key is
 * visible only if it also belongs to the query's document -- page "训练3.8B
 * LLM…", section "无效的方法" (masking at document boundaries, flex attention).
 */
static void attend_row(const double *q, const double *k, const double *v,
                       const int64_t *qpos, const int64_t *qdoc, const int64_t *kdoc,
                       double *o, int Tq, int Tk, int Hq, int Hkv, int D, double scale,
                       int64_t r, double *scores)
{
    int64_t h = r % Hq;
    int64_t bt = r / Hq;
    int64_t b = bt / Tq;
    int g = Hq / Hkv;
    int64_t kvh = h / g;
    int64_t nvis = qpos[bt] + 1;
    if (nvis > Tk)
        nvis = Tk;
    const double *qr = q + r * D;
    double *orow = o + r * D;

    double m = -INFINITY;
    for (int64_t u = 0; u < nvis; ++u) {
        if (kdoc && kdoc[b * Tk + u] != qdoc[bt]) {
            scores[u] = -INFINITY;       /* another document: exp gives 0 */
            continue;
        }
        const double *kr = k + ((b * Tk + u) * Hkv + kvh) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += qr[d] * kr[d];
        s *= scale;
        scores[u] = s;
        if (s > m)
            m = s;
    }
    double l = 0.0;
    for (int64_t u = 0; u < nvis; ++u) {
        scores[u] = exp(scores[u] - m);
        l += scores[u];
    }
    for (int d = 0; d < D; ++d)
        orow[d] = 0.0;
    for (int64_t u = 0; u < nvis; ++u) {
        const double *vr = v + ((b * Tk + u) * Hkv + kvh) * D;
        double p = scores[u] / l;
        for (int d = 0; d < D; ++d)
            orow[d] += p * vr[d];
    }
}

/*
 * Causal GQA attention.  rows == NULL computes every (b, t, h) row; otherwise
 * only the nrows flat row indices listed.  nthreads <= 0 uses the OpenMP default.
 * qdoc / kdoc: document ids of queries and keys, or NULL (no document mask).
 * Returns 0, or -1 when Hq is not a multiple of Hkv or an allocation fails.
 */
int oracle_attention_docs(const double *q, const double *k, const double *v,
                          const int64_t *qpos, const int64_t *qdoc, const int64_t *kdoc,
                          double *o, int B, int Tq, int Tk, int Hq, int Hkv, int D,
                          double scale, const int64_t *rows, int64_t nrows, int nthreads)
{
    if (Hkv <= 0 || Hq % Hkv != 0)
        return -1;
    int64_t total = rows ? nrows : (int64_t)B * Tq * Hq;
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
    size_t per = (size_t)(Tk > 0 ? Tk : 1);
    double *scratch = (double *)malloc(sizeof(double) * per * (size_t)nt);
    if (!scratch)
        return -1;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 4)
    for (int64_t i = 0; i < total; ++i) {
        int64_t r = rows ? rows[i] : i;
        double *scores = scratch + per * (size_t)omp_get_thread_num();
        attend_row(q, k, v, qpos, qdoc, kdoc, o, Tq, Tk, Hq, Hkv, D, scale, r, scores);
    }
    free(scratch);
    return 0;
}

int oracle_attention(const double *q, const double *k, const double *v,
                     const int64_t *qpos, double *o, int B, int Tq, int Tk, int Hq,
                     int Hkv, int D, double scale, const int64_t *rows,
                     int64_t nrows, int nthreads)
{
    return oracle_attention_docs(q, k, v, qpos, NULL, NULL, o, B, Tq, Tk, Hq, Hkv, D, scale,
                                 rows, nrows, nthreads);
}
