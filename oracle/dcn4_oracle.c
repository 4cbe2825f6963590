/*
 * dcn4_oracle.c -- plain, slow CPU restatement of DCNv4 deformable spatial
 * aggregation, its backward pass and the FlowDCN groupwise multi-scale
 * (MSDCN) variant with its backward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no header, helper, table or
 * constant with the CUDA path.
 *
 * Sources (page title, section):
 *  [DIGEST]  "(论文速读）DCNv4：高效可变形卷积算子" (CSDN summary of the CVPR 2024
 *            DCNv4 paper): "移除Softmax归一化" (aggregation weights are
 *            unbounded, no softmax), "GPU效率的理论分析" (36HWC FLOPs, the
 *            factor 4 is the bilinear interpolation; ideal traffic
 *            2HWC + 27HWG; worst case 64HWC), "方法1. 消除冗余工作负载" (the D = C/G
 *            channels of a group share offsets and weights).
 *  [FLOWDCN] "NeurIPS'24 | FlowDCN：基于可变形卷积的任意分辨率图像生成模型":
 *            "2.2 DCN结构简介" (sample at p0 + p_k + delta p, aggregate with the
 *            dynamic weights, concatenate the groups), "3.1 组间多尺度可变形卷积"
 *            (delta p split into a per-group scale with prior s0_g and a
 *            per-tap direction; the maximum scale Smax).
 *  [CANN]    "CANN ops-nn 算子与 Stable Diffusion 的卷积实现", "2.1 标准卷积的数学
 *            表达" (conv indexing y*s + i used for the base sampling grid).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - offset_weight layout [N][Ho][Wo][G][kh*kw][3] holding (dx along W,
 *    dy along H, m); tap k = i*kw + j with i along H.
 *  - base point of tap (i, j) for output (ho, wo) is
 *    (ho*sh - ph + i*dh, wo*sw - pw + j*dw), as in conv indexing with padding
 *    and dilation; the sample is that point plus (dy, dx) * offset_scale.
 *  - positions are computed in fp32: the product d*offset_scale and the sum
 *    base + product are each rounded to nearest (this file must be built
 *    with -ffp-contract=off so no fused multiply-add merges them).
 *  - "zero outside the image" is per corner: a sample with x in (-1, W) and
 *    y in (-1, H) keeps its in-image corners; any other sample (including a
 *    NaN position) contributes nothing.
 *  - the corner indices are floor(x), floor(y) of the fp32 position; the
 *    fractional parts x - floor(x), y - floor(y) and the four bilinear
 *    weights are taken in fp64, where they are exact.
 *  - accumulation in fp64 from inputs widened exactly from their stored type.
 *  - MSDCN: s = s0_g * softplus(raw) in fp32 with
 *    softplus(r) = max(r, 0) + log1p(exp(-|r|)); s is clamped from above at
 *    Smax; delta = s * dir (fp32); the sample point is then formed exactly as
 *    in DCNv4 with delta in place of the offset.
 *  - MSDCN backward: the gradient reaches raw through
 *    ds/draw = s0 * sigmoid(raw) while s0 * softplus(raw) <= Smax and is 0
 *    once the clamp is active (and for a NaN raw).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

/* The oracle's own problem description (deliberately not the product's). */
typedef struct {
    int N, H, W, C, G;   /* input N x H x W x C, channel-last; G groups    */
    int kh, kw;          /* kernel taps along H and W                     */
    int sh, sw;          /* stride                                        */
    int ph, pw;          /* padding                                       */
    int dh, dw;          /* dilation                                      */
    float offset_scale;  /* multiplies every offset before it is added    */
    int softmax;         /* DCNv3 weights: softmax of m over the taps     */
    int msdcn_dilation;  /* MSDCN reading p0 + s * (p_k + dir)            */
} orc_problem;

/* Output size, standard convolution arithmetic ([CANN] 2.1). Returns 0 when
 * the problem is well formed, -1 otherwise. */
int orc_out_hw(const orc_problem *p, int *Ho, int *Wo)
{
    if (!p || p->N <= 0 || p->H <= 0 || p->W <= 0 || p->C <= 0 || p->G <= 0)
        return -1;
    if (p->C % p->G != 0 || p->kh <= 0 || p->kw <= 0 || p->sh <= 0 ||
        p->sw <= 0 || p->ph < 0 || p->pw < 0 || p->dh <= 0 || p->dw <= 0)
        return -1;
    int ho = (p->H + 2 * p->ph - p->dh * (p->kh - 1) - 1) / p->sh + 1;
    int wo = (p->W + 2 * p->pw - p->dw * (p->kw - 1) - 1) / p->sw + 1;
    if (ho <= 0 || wo <= 0)
        return -1;
    if (Ho) *Ho = ho;
    if (Wo) *Wo = wo;
    return 0;
}

/* The sampling position of one tap, in fp32 ([FLOWDCN] 2.2: p0 + p_k + dp). */
static void orc_position(const orc_problem *p, int ho, int wo, int i, int j,
                         float dx, float dy, float *x, float *y)
{
    float bx = (float)(wo * p->sw - p->pw + j * p->dw);
    float by = (float)(ho * p->sh - p->ph + i * p->dh);
    float tx = dx * p->offset_scale;
    float ty = dy * p->offset_scale;
    *x = bx + tx;
    *y = by + ty;
}

/* The aggregation weights of one (pixel, group): m as given ([DIGEST]
 * 移除Softmax归一化), or with p->softmax the DCNv3 normalisation the same
 * section describes, softmax over the kh*kw taps (in fp64, largest logit
 * subtracted first). t holds the (dx, dy, m) triples; w receives K weights. */
static void orc_tap_weights(const orc_problem *p, const float *t, double *w)
{
    const int K = p->kh * p->kw;
    if (!p->softmax) {
        for (int k = 0; k < K; ++k)
            w[k] = (double)t[3 * k + 2];
        return;
    }
    double mx = (double)t[2];
    for (int k = 1; k < K; ++k)
        if ((double)t[3 * k + 2] > mx)
            mx = (double)t[3 * k + 2];
    double sum = 0.0;
    for (int k = 0; k < K; ++k) {
        w[k] = exp((double)t[3 * k + 2] - mx);
        sum += w[k];
    }
    for (int k = 0; k < K; ++k)
        w[k] /= sum;
}

/* The MSDCN sample of tap (i, j) with scale s and direction (dirx, diry)
 * ([FLOWDCN] 3.1). Default reading: the offset is s * dir, then as
 * orc_position. With p->msdcn_dilation the scale stretches the kernel grid as
 * well: centre + s * (p_k + dir * offset_scale), centre the middle of the
 * kh x kw window and p_k the tap's grid offset from it; each product and sum
 * rounded to fp32. (tx, ty) receive the factor that multiplies s, i.e. the
 * derivative of the position with respect to s. */
static void orc_position_ms(const orc_problem *p, int ho, int wo, int i, int j, float s,
                            float dirx, float diry, float *x, float *y, double *tx,
                            double *ty)
{
    if (!p->msdcn_dilation) {
        float dx = s * dirx, dy = s * diry;
        orc_position(p, ho, wo, i, j, dx, dy, x, y);
        *tx = (double)dirx * (double)p->offset_scale;
        *ty = (double)diry * (double)p->offset_scale;
        return;
    }
    float cx = (float)(wo * p->sw - p->pw) + 0.5f * (float)((p->kw - 1) * p->dw);
    float cy = (float)(ho * p->sh - p->ph) + 0.5f * (float)((p->kh - 1) * p->dh);
    float kx = ((float)j - 0.5f * (float)(p->kw - 1)) * (float)p->dw;
    float ky = ((float)i - 0.5f * (float)(p->kh - 1)) * (float)p->dh;
    float ox = dirx * p->offset_scale, oy = diry * p->offset_scale;
    float ux = kx + ox, uy = ky + oy;
    float sx = s * ux, sy = s * uy;
    *x = cx + sx;
    *y = cy + sy;
    *tx = (double)ux;
    *ty = (double)uy;
}

/* Adds m * bilinear(img at (x, y))[c0 .. c0+D) into acc ([DIGEST]: 4 terms of
 * the bilinear interpolation per sample; out-of-image corners are zero). */
static void orc_splat_sample(const float *img, int H, int W, int C, int c0,
                             int D, float x, float y, double m, double *acc)
{
    if (!(x > -1.0f && x < (float)W && y > -1.0f && y < (float)H))
        return;
    float x0f = floorf(x), y0f = floorf(y);
    double lx = (double)x - (double)x0f, ly = (double)y - (double)y0f;
    int x0 = (int)x0f, y0 = (int)y0f;
    for (int a = 0; a < 2; ++a) {
        for (int b = 0; b < 2; ++b) {
            int yy = y0 + a, xx = x0 + b;
            if (yy < 0 || yy >= H || xx < 0 || xx >= W)
                continue;
            double wy = a ? ly : 1.0 - ly;
            double wx = b ? lx : 1.0 - lx;
            const float *v = img + ((size_t)yy * W + xx) * C + c0;
            for (int d = 0; d < D; ++d)
                acc[d] += m * (wy * wx) * (double)v[d];
        }
    }
}

/* DCNv4 forward ([FLOWDCN] 2.2; [DIGEST] 移除Softmax归一化: m is used as given).
 * input [N][H][W][C], offset_weight [N][Ho][Wo][G][kh*kw][3], out [N][Ho][Wo][C].
 * Returns 0 on success, -1 on a malformed problem. */
int orc_dcn4_forward(const orc_problem *p, const float *input,
                     const float *offset_weight, double *out)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo) || !input || !offset_weight || !out)
        return -1;
    const int K = p->kh * p->kw, D = p->C / p->G;
    const size_t img = (size_t)p->H * p->W * p->C;
#pragma omp parallel for collapse(2) schedule(static)
    for (int n = 0; n < p->N; ++n) {
        for (int ho = 0; ho < Ho; ++ho) {
            for (int wo = 0; wo < Wo; ++wo) {
                size_t pix = ((size_t)n * Ho + ho) * Wo + wo;
                for (int g = 0; g < p->G; ++g) {
                    double *o = out + pix * p->C + (size_t)g * D;
                    const float *t = offset_weight + (pix * p->G + g) * (size_t)K * 3;
                    double wk[K];
                    orc_tap_weights(p, t, wk);
                    for (int d = 0; d < D; ++d)
                        o[d] = 0.0;
                    for (int i = 0; i < p->kh; ++i) {
                        for (int j = 0; j < p->kw; ++j) {
                            int k = i * p->kw + j;
                            float x, y;
                            orc_position(p, ho, wo, i, j, t[3 * k], t[3 * k + 1], &x, &y);
                            orc_splat_sample(input + (size_t)n * img, p->H, p->W, p->C,
                                             g * D, D, x, y, wk[k], o);
                        }
                    }
                }
            }
        }
    }
    return 0;
}

/* DCNv4 backward: the derivative of the forward above, written out.
 * grad_out [N][Ho][Wo][C] (values as stored), grad_input [N][H][W][C] and
 * grad_offset_weight [N][Ho][Wo][G][kh*kw][3] are written (not accumulated).
 *   grad m      = sum_d go_d * bilinear_d
 *   grad dx     = offset_scale * m * sum_corners (+-wy) * <go, V_corner>
 *   grad dy     = offset_scale * m * sum_corners (+-wx) * <go, V_corner>
 *   grad in[c] += m * wy * wx * go        (for every in-image corner c)
 * At an integer position the derivative taken is the one of the cell that
 * floor() selects (the right-hand derivative). Samples outside
 * (-1, W) x (-1, H) have zero gradient. With p->softmax, m above is the
 * softmax weight w_k and the m-gradient is taken through the softmax. */
int orc_dcn4_backward(const orc_problem *p, const float *input,
                      const float *offset_weight, const float *grad_out,
                      double *grad_input, double *grad_offset_weight)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo) || !input || !offset_weight || !grad_out ||
        !grad_input || !grad_offset_weight)
        return -1;
    const int K = p->kh * p->kw, D = p->C / p->G;
    const size_t img = (size_t)p->H * p->W * p->C;
    memset(grad_input, 0, sizeof(double) * img * p->N);
    /* images are independent, so they may run in parallel */
#pragma omp parallel for schedule(static)
    for (int n = 0; n < p->N; ++n) {
        const float *in_n = input + (size_t)n * img;
        double *gin_n = grad_input + (size_t)n * img;
        for (int ho = 0; ho < Ho; ++ho) {
            for (int wo = 0; wo < Wo; ++wo) {
                size_t pix = ((size_t)n * Ho + ho) * Wo + wo;
                for (int g = 0; g < p->G; ++g) {
                    const float *t = offset_weight + (pix * p->G + g) * (size_t)K * 3;
                    double *gt = grad_offset_weight + (pix * p->G + g) * (size_t)K * 3;
                    const float *go = grad_out + pix * p->C + (size_t)g * D;
                    double wk[K], gwk[K];  /* tap weights; d loss / d weight */
                    orc_tap_weights(p, t, wk);
                    for (int i = 0; i < p->kh; ++i) {
                        for (int j = 0; j < p->kw; ++j) {
                            int k = i * p->kw + j;
                            float x, y;
                            orc_position(p, ho, wo, i, j, t[3 * k], t[3 * k + 1], &x, &y);
                            double m = wk[k];
                            double gx = 0.0, gy = 0.0, gm = 0.0;
                            if (x > -1.0f && x < (float)p->W && y > -1.0f && y < (float)p->H) {
                                float x0f = floorf(x), y0f = floorf(y);
                                double lx = (double)x - (double)x0f;
                                double ly = (double)y - (double)y0f;
                                int x0 = (int)x0f, y0 = (int)y0f;
                                for (int a = 0; a < 2; ++a) {
                                    for (int b = 0; b < 2; ++b) {
                                        int yy = y0 + a, xx = x0 + b;
                                        if (yy < 0 || yy >= p->H || xx < 0 || xx >= p->W)
                                            continue;
                                        double wy = a ? ly : 1.0 - ly;
                                        double wx = b ? lx : 1.0 - lx;
                                        size_t at = ((size_t)yy * p->W + xx) * p->C + (size_t)g * D;
                                        double dot = 0.0;
                                        for (int d = 0; d < D; ++d) {
                                            dot += (double)go[d] * (double)in_n[at + d];
                                            gin_n[at + d] += m * (wy * wx) * (double)go[d];
                                        }
                                        gm += wy * wx * dot;
                                        gx += (b ? wy : -wy) * dot;
                                        gy += (a ? wx : -wx) * dot;
                                    }
                                }
                            }
                            gt[3 * k] = (double)p->offset_scale * m * gx;
                            gt[3 * k + 1] = (double)p->offset_scale * m * gy;
                            gwk[k] = gm;
                        }
                    }
                    /* through the softmax: d/d m_k = w_k (gw_k - sum_j w_j gw_j) */
                    double dotw = 0.0;
                    if (p->softmax)
                        for (int k = 0; k < K; ++k)
                            dotw += wk[k] * gwk[k];
                    for (int k = 0; k < K; ++k)
                        gt[3 * k + 2] = p->softmax ? wk[k] * (gwk[k] - dotw) : gwk[k];
                }
            }
        }
    }
    return 0;
}

/* MSDCN per-group scale ([FLOWDCN] 3.1): s = min(s0 * softplus(raw), smax)
 * in fp32. A NaN raw gives a NaN scale (and hence no contribution). */
float orc_msdcn_scale(float raw, float s0, float smax)
{
    float sp = fmaxf(raw, 0.0f) + log1pf(expf(-fabsf(raw)));
    float s = s0 * sp;
    if (s > smax)
        s = smax;
    return s;
}

/* MSDCN forward ([FLOWDCN] 3.1): DCNv4 aggregation whose offset for group g
 * and tap k is s_g(p0) * dir_{g,k}(p0) (or, with p->msdcn_dilation, whose
 * kernel grid is scaled too, see orc_position_ms). m is used as given
 * (p->softmax does not apply to MSDCN).
 * dir_weight [N][Ho][Wo][G][kh*kw][3] holds (dir_x, dir_y, m);
 * scale_raw [N][Ho][Wo][G]; s0 [G]. */
int orc_msdcn_forward(const orc_problem *p, const float *input,
                      const float *dir_weight, const float *scale_raw,
                      const float *s0, float smax, double *out)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo) || !input || !dir_weight || !scale_raw || !s0 || !out)
        return -1;
    const int K = p->kh * p->kw, D = p->C / p->G;
    const size_t img = (size_t)p->H * p->W * p->C;
#pragma omp parallel for collapse(2) schedule(static)
    for (int n = 0; n < p->N; ++n) {
        for (int ho = 0; ho < Ho; ++ho) {
            for (int wo = 0; wo < Wo; ++wo) {
                size_t pix = ((size_t)n * Ho + ho) * Wo + wo;
                for (int g = 0; g < p->G; ++g) {
                    double *o = out + pix * p->C + (size_t)g * D;
                    const float *t = dir_weight + (pix * p->G + g) * (size_t)K * 3;
                    float s = orc_msdcn_scale(scale_raw[pix * p->G + g], s0[g], smax);
                    for (int d = 0; d < D; ++d)
                        o[d] = 0.0;
                    for (int i = 0; i < p->kh; ++i) {
                        for (int j = 0; j < p->kw; ++j) {
                            int k = i * p->kw + j;
                            float x, y;
                            double tx, ty;
                            orc_position_ms(p, ho, wo, i, j, s, t[3 * k], t[3 * k + 1], &x, &y,
                                            &tx, &ty);
                            orc_splat_sample(input + (size_t)n * img, p->H, p->W, p->C,
                                             g * D, D, x, y, (double)t[3 * k + 2], o);
                        }
                    }
                }
            }
        }
    }
    return 0;
}

/* Derivative of the MSDCN scale with respect to raw: s0 * sigmoid(raw) while
 * the clamp is inactive (s0 * softplus(raw) <= smax, the branch
 * orc_msdcn_scale keeps), 0 once it clamps, 0 for a NaN raw. sigmoid is the
 * derivative of softplus (read from [FLOWDCN] 3.1's softplus scale; the
 * page prints no gradient). */
static double orc_msdcn_scale_grad(float raw, float s0, float smax)
{
    float sp = fmaxf(raw, 0.0f) + log1pf(expf(-fabsf(raw)));
    float u = s0 * sp;
    if (!(u <= smax))
        return 0.0;
    return (double)s0 / (1.0 + exp(-(double)raw));
}

/* MSDCN backward: the gradients of orc_msdcn_forward's output, given
 * grad_out, with respect to the input, to dir_weight (dir_x, dir_y, m) and to
 * scale_raw. The sample of tap k is p0 + p_k + (s * dir_k) * offset_scale,
 * so with g_x = m * sum_d go . dv/dx (and g_y likewise) at the sample:
 *   d/d dir_x = s * os * g_x,   d/d dir_y = s * os * g_y,
 *   d/d m     = sum_d go . v  (as in DCNv4),
 *   d/d raw   = (ds/draw) * sum_k (g_x * dx/ds + g_y * dy/ds), where
 *               dx/ds = os * dir_x (or p_kx + os * dir_x with msdcn_dilation),
 *   grad_in[corner] += m * w_corner * go.
 * Outputs are fp64: grad_input [N][H][W][C], grad_dir_weight
 * [N][Ho][Wo][G][kh*kw][3], grad_scale_raw [N][Ho][Wo][G]. */
int orc_msdcn_backward(const orc_problem *p, const float *input,
                       const float *dir_weight, const float *scale_raw,
                       const float *s0, float smax, const float *grad_out,
                       double *grad_input, double *grad_dir_weight,
                       double *grad_scale_raw)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo) || !input || !dir_weight || !scale_raw || !s0 ||
        !grad_out || !grad_input || !grad_dir_weight || !grad_scale_raw)
        return -1;
    const int K = p->kh * p->kw, D = p->C / p->G;
    const size_t img = (size_t)p->H * p->W * p->C;
    const double os = (double)p->offset_scale;
    memset(grad_input, 0, sizeof(double) * img * p->N);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < p->N; ++n) {
        const float *in_n = input + (size_t)n * img;
        double *gin_n = grad_input + (size_t)n * img;
        for (int ho = 0; ho < Ho; ++ho) {
            for (int wo = 0; wo < Wo; ++wo) {
                size_t pix = ((size_t)n * Ho + ho) * Wo + wo;
                for (int g = 0; g < p->G; ++g) {
                    const float *t = dir_weight + (pix * p->G + g) * (size_t)K * 3;
                    double *gt = grad_dir_weight + (pix * p->G + g) * (size_t)K * 3;
                    const float *go = grad_out + pix * p->C + (size_t)g * D;
                    const float raw = scale_raw[pix * p->G + g];
                    const float s = orc_msdcn_scale(raw, s0[g], smax);
                    double gs = 0.0;  /* d loss / d s */
                    for (int i = 0; i < p->kh; ++i) {
                        for (int j = 0; j < p->kw; ++j) {
                            int k = i * p->kw + j;
                            float x, y;
                            double tx, ty;  /* d position / d s */
                            orc_position_ms(p, ho, wo, i, j, s, t[3 * k], t[3 * k + 1], &x, &y,
                                            &tx, &ty);
                            double m = (double)t[3 * k + 2];
                            double gx = 0.0, gy = 0.0, gm = 0.0;
                            if (x > -1.0f && x < (float)p->W && y > -1.0f && y < (float)p->H) {
                                float x0f = floorf(x), y0f = floorf(y);
                                double lx = (double)x - (double)x0f;
                                double ly = (double)y - (double)y0f;
                                int x0 = (int)x0f, y0 = (int)y0f;
                                for (int a = 0; a < 2; ++a) {
                                    for (int b = 0; b < 2; ++b) {
                                        int yy = y0 + a, xx = x0 + b;
                                        if (yy < 0 || yy >= p->H || xx < 0 || xx >= p->W)
                                            continue;
                                        double wy = a ? ly : 1.0 - ly;
                                        double wx = b ? lx : 1.0 - lx;
                                        size_t at = ((size_t)yy * p->W + xx) * p->C + (size_t)g * D;
                                        double dot = 0.0;
                                        for (int d = 0; d < D; ++d) {
                                            dot += (double)go[d] * (double)in_n[at + d];
                                            gin_n[at + d] += m * (wy * wx) * (double)go[d];
                                        }
                                        gm += wy * wx * dot;
                                        gx += (b ? wy : -wy) * dot;
                                        gy += (a ? wx : -wx) * dot;
                                    }
                                }
                            }
                            /* gx, gy: d(sum_d go . sample) / dx, dy of the position */
                            /* a sample that contributes nothing (outside, or a NaN
                             * scale) has zero gradient, not s * 0 */
                            const double gdx = os * m * gx, gdy = os * m * gy;
                            gt[3 * k] = gdx == 0.0 ? 0.0 : (double)s * gdx;
                            gt[3 * k + 1] = gdy == 0.0 ? 0.0 : (double)s * gdy;
                            gt[3 * k + 2] = gm;
                            gs += m * (gx * tx + gy * ty);
                        }
                    }
                    grad_scale_raw[pix * p->G + g] =
                        gs == 0.0 ? 0.0 : gs * orc_msdcn_scale_grad(raw, s0[g], smax);
                }
            }
        }
    }
    return 0;
}

/* --- cost model of [DIGEST] "GPU效率的理论分析" -------------------------- */

/* FLOPs: 4 (bilinear terms) per tap per output element, i.e. 36 HWC for a
 * 3x3 kernel with H, W the output size. */
/* Offset/weight producer of the DCNv4 module ([DIGEST] "方法3. DCN模块的微设计优化":
 * once softmax is gone, one linear layer emits both the offsets and the
 * aggregation weights, and the sub-network in front of it is a plain
 * separable convolution, a depthwise 3x3 then that linear layer, without the
 * DCNv3 LayerNorm and GELU).  For every pixel (n, y, x) of the H x W map:
 *   h[c]  = dw_b[c] + sum_{i,j in 0..2} dw_w[i][j][c] * x[n][y+i-1][x+j-1][c]
 *           (stride 1, zero outside the image),
 *   out[j] = lin_b[j] + sum_c lin_w[j][c] * h[c],   j in [0, G*kh*kw*3),
 * so out[n][y][x] is laid out exactly like offset_weight [G][kh*kw][3].
 * dw_w is [3][3][C] (tap-major), dw_b [C], lin_w [G*kh*kw*3][C] (output
 * row-major), lin_b [G*kh*kw*3]; all accumulation in fp64.  Returns 0, or
 * -1 for a malformed problem. */
int orc_offset_producer(const orc_problem *p, const float *x, const float *dw_w,
                        const float *dw_b, const float *lin_w, const float *lin_b,
                        double *out)
{
    if (orc_out_hw(p, NULL, NULL) != 0)
        return -1;
    const int H = p->H, W = p->W, C = p->C;
    const int J = p->G * p->kh * p->kw * 3;
    double *h = (double *)malloc(sizeof(double) * (size_t)C);
    if (!h)
        return -1;
    for (int n = 0; n < p->N; ++n)
        for (int y = 0; y < H; ++y)
            for (int xx = 0; xx < W; ++xx) {
                for (int c = 0; c < C; ++c) {
                    double acc = dw_b[c];
                    for (int i = 0; i < 3; ++i)
                        for (int j = 0; j < 3; ++j) {
                            const int yy = y + i - 1, xs = xx + j - 1;
                            if (yy < 0 || yy >= H || xs < 0 || xs >= W)
                                continue;
                            acc += (double)dw_w[(i * 3 + j) * C + c] *
                                   (double)x[(((size_t)n * H + yy) * W + xs) * C + c];
                        }
                    h[c] = acc;
                }
                double *o = out + (((size_t)n * H + y) * W + xx) * (size_t)J;
                for (int j = 0; j < J; ++j) {
                    double acc = lin_b[j];
                    for (int c = 0; c < C; ++c)
                        acc += (double)lin_w[(size_t)j * C + c] * h[c];
                    o[j] = acc;
                }
            }
    free(h);
    return 0;
}

double orc_flops(const orc_problem *p)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo))
        return -1.0;
    return 4.0 * p->kh * p->kw * (double)p->N * Ho * Wo * p->C;
}

/* Ideal traffic in bytes: input and output once, plus 3 values per tap per
 * group per output pixel (27 HWG for 3x3); elem_bytes per value. */
double orc_ideal_bytes(const orc_problem *p, int elem_bytes)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo))
        return -1.0;
    double in = (double)p->N * p->H * p->W * p->C;
    double out = (double)p->N * Ho * Wo * p->C;
    double ow = 3.0 * p->kh * p->kw * (double)p->N * Ho * Wo * p->G;
    return (in + out + ow) * elem_bytes;
}

/* Worst-case traffic with no cache: for every output element 4 reads per
 * tap, 3 offset/weight reads per tap and one write (64 HWC for 3x3). */
double orc_worst_bytes(const orc_problem *p, int elem_bytes)
{
    int Ho, Wo;
    if (orc_out_hw(p, &Ho, &Wo))
        return -1.0;
    double per = 4.0 * p->kh * p->kw + 3.0 * p->kh * p->kw + 1.0;
    return per * (double)p->N * Ho * Wo * p->C * elem_bytes;
}
