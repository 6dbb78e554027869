/*
 * Float64 CPU oracle for the modulated deformable convolution (DCNv2).
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py may load this library. The product (the CUDA library under
 * deformable_convolution_dcn_b200/) never calls it and shares no code with it.
 *
 * What is computed (all sums in float64, in the order written below):
 *
 *   y(p0) = bias + sum_{k in R} w(p_k) * m_k * x(p0 + p_k + dp_k)
 *
 *   - the plain convolution over the regular grid R and its deformable form with
 *     a learned offset dp_k per tap ("Deformable ConvNets" notes, section
 *     "可变形卷积", the two y(p0) equations);
 *   - the DCNv2 modulation scalar m_k that multiplies each sampled value
 *     ("DCNv2", section 3.2 "添加幅值参数"; the tutorial's mask argument, table in
 *     section 2.1, default all ones);
 *   - x(p) at a fractional p is bilinear interpolation over the four integer
 *     neighbours, each weighted by the area of the opposite sub-rectangle
 *     (notes, "双线性插值" equation S1..S4);
 *   - channels are split into G deformable groups, every channel of a group
 *     sharing one offset field (notes, "Deformable Group");
 *   - torchvision deform_conv2d conventions for layout and borders (tutorial,
 *     section 2 "解剖torchvision.ops.deform_conv2d"): offsets carry 2*G*K*K
 *     channels with channel g*2K^2 + 2k = dy (row) and +1 = dx (column); a
 *     neighbour that lies outside the map contributes zero (no clamping).
 *
 * Layouts (row-major, innermost last):
 *   x       [B, H, W, Cin]                  channel-contiguous (NHWC)
 *   offset  [B, 2*G*K*K, Ho, Wo]
 *   mask    [B, G*K*K, Ho, Wo]              NULL means m = 1 everywhere (DCNv1)
 *   weight  [Cout, K, K, Cin]
 *   bias    [Cout]                          NULL means no bias
 *   y       [B, Ho, Wo, Cout]
 *   Ho = (H + 2*pad - dil*(K-1) - 1) / stride + 1, likewise Wo.
 *
 * Tap k = i*K + j (i = kernel row, j = kernel column) samples at
 *   py = ho*stride - pad + i*dil + dy,   px = wo*stride - pad + j*dil + dx.
 *
 * Backward: the chain rule through the same expression. The offset gradient is
 * the page's d y(p0) / d dp_n = sum w(p_n) * sum_q dG(q, p)/d dp_n * x(q)
 * (notes, "计算梯度"), with dG taken through floor(p): at an exact integer
 * coordinate the derivative uses the neighbours floor(p) and floor(p)+1, i.e. the
 * right-hand derivative (the tutorial, section 3.2, notes the kink there).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, H, W, Cin, Cout, K, stride, pad, dil, G;
} dcn_oracle_shape;

int dcn_oracle_out_h(const dcn_oracle_shape* s) {
    return (s->H + 2 * s->pad - s->dil * (s->K - 1) - 1) / s->stride + 1;
}
int dcn_oracle_out_w(const dcn_oracle_shape* s) {
    return (s->W + 2 * s->pad - s->dil * (s->K - 1) - 1) / s->stride + 1;
}

void dcn_oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
int dcn_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- sampling -- */

/* Value of channel c of image b at integer (r, q); zero outside the map. */
static double pixel_or_zero(const double* x, const dcn_oracle_shape* s, int b, int r, int q, int c) {
    if (r < 0 || r >= s->H || q < 0 || q >= s->W) return 0.0;
    return x[(((size_t)b * s->H + r) * s->W + q) * s->Cin + c];
}

/* Bilinear interpolation at fractional (py, px): the four integer neighbours
 * (floor(py) + a, floor(px) + e), a, e in {0, 1}, weighted by
 * (1 - |py - row|) * (1 - |px - col|). */
static double bilinear(const double* x, const dcn_oracle_shape* s, int b, int c, double py, double px) {
    double y0 = floor(py), x0 = floor(px);
    double v = 0.0;
    for (int a = 0; a < 2; ++a)
        for (int e = 0; e < 2; ++e) {
            double r = y0 + a, q = x0 + e;
            double g = (1.0 - fabs(py - r)) * (1.0 - fabs(px - q));
            v += g * pixel_or_zero(x, s, b, (int)r, (int)q, c);
        }
    return v;
}

/* d bilinear / d py and d bilinear / d px, taken through floor(): the row
 * factor of neighbour row y0 is (1 - (py - y0)) with derivative -1, that of
 * row y0 + 1 is (py - y0) with derivative +1; likewise for columns. */
static void bilinear_grad(const double* x, const dcn_oracle_shape* s, int b, int c, double py, double px,
                          double* dpy, double* dpx) {
    double y0 = floor(py), x0 = floor(px);
    double ly = py - y0, lx = px - x0;
    double v00 = pixel_or_zero(x, s, b, (int)y0, (int)x0, c);
    double v01 = pixel_or_zero(x, s, b, (int)y0, (int)x0 + 1, c);
    double v10 = pixel_or_zero(x, s, b, (int)y0 + 1, (int)x0, c);
    double v11 = pixel_or_zero(x, s, b, (int)y0 + 1, (int)x0 + 1, c);
    *dpy = (1.0 - lx) * (v10 - v00) + lx * (v11 - v01);
    *dpx = (1.0 - ly) * (v01 - v00) + ly * (v11 - v10);
}

/* Sampling position, modulation scalar for tap k = i*K + j of group g at output
 * pixel (b, ho, wo). */
static void tap_position(const dcn_oracle_shape* s, const double* off, const double* mask, int b, int ho, int wo,
                         int g, int i, int j, double* py, double* px, double* m) {
    int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    int K2 = s->K * s->K, k = i * s->K + j;
    size_t plane = (size_t)Ho * Wo, pix = (size_t)ho * Wo + wo;
    double dy = off[((size_t)b * 2 * s->G * K2 + (size_t)g * 2 * K2 + 2 * k) * plane + pix];
    double dx = off[((size_t)b * 2 * s->G * K2 + (size_t)g * 2 * K2 + 2 * k + 1) * plane + pix];
    *py = (double)(ho * s->stride - s->pad + i * s->dil) + dy;
    *px = (double)(wo * s->stride - s->pad + j * s->dil) + dx;
    *m = mask ? mask[((size_t)b * s->G * K2 + (size_t)g * K2 + k) * plane + pix] : 1.0;
}

static size_t weight_index(const dcn_oracle_shape* s, int o, int i, int j, int c) {
    return (((size_t)o * s->K + i) * s->K + j) * s->Cin + c;
}

/* ----------------------------------------------------------------- forward -- */

/* y for one output pixel p (flat index into B*Ho*Wo), all Cout channels. */
static void forward_pixel(const dcn_oracle_shape* s, const double* x, const double* off, const double* mask,
                          const double* w, const double* bias, long p, double* yrow) {
    int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    int b = (int)(p / ((long)Ho * Wo)), ho = (int)((p / Wo) % Ho), wo = (int)(p % Wo);
    int Cg = s->Cin / s->G;
    for (int o = 0; o < s->Cout; ++o) yrow[o] = bias ? bias[o] : 0.0;
    for (int g = 0; g < s->G; ++g)
        for (int i = 0; i < s->K; ++i)
            for (int j = 0; j < s->K; ++j) {
                double py, px, m;
                tap_position(s, off, mask, b, ho, wo, g, i, j, &py, &px, &m);
                for (int c = g * Cg; c < (g + 1) * Cg; ++c) {
                    double v = m * bilinear(x, s, b, c, py, px);
                    for (int o = 0; o < s->Cout; ++o) yrow[o] += w[weight_index(s, o, i, j, c)] * v;
                }
            }
}

/* Forward at a list of output pixels (pix == NULL: every pixel in order).
 * y receives npix rows of Cout values. */
int dcn_oracle_forward_pixels(const dcn_oracle_shape* s, const double* x, const double* off, const double* mask,
                              const double* w, const double* bias, long npix, const long* pix, double* y) {
    if (s->G <= 0 || s->Cin % s->G) return -1;
    long n;
#pragma omp parallel for schedule(dynamic, 16)
    for (n = 0; n < npix; ++n) forward_pixel(s, x, off, mask, w, bias, pix ? pix[n] : n, y + (size_t)n * s->Cout);
    return 0;
}

int dcn_oracle_forward(const dcn_oracle_shape* s, const double* x, const double* off, const double* mask,
                       const double* w, const double* bias, double* y) {
    long P = (long)s->B * dcn_oracle_out_h(s) * dcn_oracle_out_w(s);
    return dcn_oracle_forward_pixels(s, x, off, mask, w, bias, P, NULL, y);
}

/* Single bilinear sample of a [H, W, C] image at (py, px), C values. */
void dcn_oracle_bilinear(int H, int W, int C, const double* img, double py, double px, double* out) {
    dcn_oracle_shape s = {1, H, W, C, 1, 1, 1, 0, 1, 1};
    for (int c = 0; c < C; ++c) out[c] = bilinear(img, &s, 0, c, py, px);
}

/* ---------------------------------------------------------------- backward -- */

/* Upstream gradient propagated to the sampled column: gcol = sum_o gy[o] * w[o, i, j, c]. */
static double column_grad(const dcn_oracle_shape* s, const double* w, const double* gyrow, int i, int j, int c) {
    double acc = 0.0;
    for (int o = 0; o < s->Cout; ++o) acc += gyrow[o] * w[weight_index(s, o, i, j, c)];
    return acc;
}

/* Full backward. Any output pointer may be NULL. Outputs are overwritten.
 *   gx [B,H,W,Cin], goff [B,2GK^2,Ho,Wo], gmask [B,GK^2,Ho,Wo] (needs mask),
 *   gw [Cout,K,K,Cin], gb [Cout].
 * Parallel over the batch: image b's pixels only touch gx[b]; gw and gb are
 * accumulated per image and summed over b in order afterwards. */
int dcn_oracle_backward(const dcn_oracle_shape* s, const double* x, const double* off, const double* mask,
                        const double* w, const double* gy, double* gx, double* goff, double* gmask, double* gw,
                        double* gb) {
    if (s->G <= 0 || s->Cin % s->G) return -1;
    int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    int K2 = s->K * s->K, Cg = s->Cin / s->G;
    size_t nw = (size_t)s->Cout * K2 * s->Cin, plane = (size_t)Ho * Wo;
    double* gw_b = (double*)calloc(nw * s->B, sizeof(double));
    double* gb_b = (double*)calloc((size_t)s->Cout * s->B, sizeof(double));
    if (!gw_b || !gb_b) {
        free(gw_b);
        free(gb_b);
        return -2;
    }
    if (gx) memset(gx, 0, sizeof(double) * (size_t)s->B * s->H * s->W * s->Cin);
    int b;
#pragma omp parallel for schedule(dynamic, 1)
    for (b = 0; b < s->B; ++b) {
        double* gwb = gw_b + nw * b;
        double* gbb = gb_b + (size_t)s->Cout * b;
        for (int ho = 0; ho < Ho; ++ho)
            for (int wo = 0; wo < Wo; ++wo) {
                size_t p = ((size_t)b * Ho + ho) * Wo + wo;
                const double* gyrow = gy + p * s->Cout;
                for (int o = 0; o < s->Cout; ++o) gbb[o] += gyrow[o];
                for (int g = 0; g < s->G; ++g)
                    for (int i = 0; i < s->K; ++i)
                        for (int j = 0; j < s->K; ++j) {
                            int k = i * s->K + j;
                            double py, px, m;
                            tap_position(s, off, mask, b, ho, wo, g, i, j, &py, &px, &m);
                            double y0 = floor(py), x0 = floor(px);
                            double gdy = 0.0, gdx = 0.0, gm = 0.0;
                            for (int c = g * Cg; c < (g + 1) * Cg; ++c) {
                                double gcol = column_grad(s, w, gyrow, i, j, c);
                                double v = bilinear(x, s, b, c, py, px);
                                double dpy, dpx;
                                bilinear_grad(x, s, b, c, py, px, &dpy, &dpx);
                                gm += gcol * v;
                                gdy += gcol * m * dpy;
                                gdx += gcol * m * dpx;
                                for (int o = 0; o < s->Cout; ++o) gwb[weight_index(s, o, i, j, c)] += gyrow[o] * m * v;
                                if (gx)
                                    for (int a = 0; a < 2; ++a)
                                        for (int e = 0; e < 2; ++e) {
                                            int r = (int)y0 + a, q = (int)x0 + e;
                                            if (r < 0 || r >= s->H || q < 0 || q >= s->W) continue;
                                            double gq = (1.0 - fabs(py - r)) * (1.0 - fabs(px - q));
                                            gx[(((size_t)b * s->H + r) * s->W + q) * s->Cin + c] += gcol * m * gq;
                                        }
                            }
                            size_t ob = (size_t)b * 2 * s->G * K2 + (size_t)g * 2 * K2 + 2 * k;
                            if (goff) {
                                goff[ob * plane + (size_t)ho * Wo + wo] = gdy;
                                goff[(ob + 1) * plane + (size_t)ho * Wo + wo] = gdx;
                            }
                            if (gmask && mask) gmask[((size_t)b * s->G * K2 + (size_t)g * K2 + k) * plane + (size_t)ho * Wo + wo] = gm;
                        }
            }
    }
    if (gw) {
        memset(gw, 0, sizeof(double) * nw);
        for (int bb = 0; bb < s->B; ++bb)
            for (size_t t = 0; t < nw; ++t) gw[t] += gw_b[nw * bb + t];
    }
    if (gb) {
        memset(gb, 0, sizeof(double) * s->Cout);
        for (int bb = 0; bb < s->B; ++bb)
            for (int o = 0; o < s->Cout; ++o) gb[o] += gb_b[(size_t)s->Cout * bb + o];
    }
    free(gw_b);
    free(gb_b);
    return 0;
}

/* --------------------------------------------- backward at sampled entries -- */
/* These compute single gradient entries straight from their definitions, so that
 * full-size problems can be checked at sampled positions. */

/* grad_offset (2GK^2 values) and grad_mask (GK^2 values) for listed output pixels. */
int dcn_oracle_grad_offset_mask_pixels(const dcn_oracle_shape* s, const double* x, const double* off,
                                       const double* mask, const double* w, const double* gy, long npix,
                                       const long* pix, double* goff, double* gmask) {
    if (s->G <= 0 || s->Cin % s->G) return -1;
    int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    int K2 = s->K * s->K, Cg = s->Cin / s->G;
    long n;
#pragma omp parallel for schedule(dynamic, 4)
    for (n = 0; n < npix; ++n) {
        long p = pix[n];
        int b = (int)(p / ((long)Ho * Wo)), ho = (int)((p / Wo) % Ho), wo = (int)(p % Wo);
        const double* gyrow = gy + (size_t)p * s->Cout;
        for (int g = 0; g < s->G; ++g)
            for (int i = 0; i < s->K; ++i)
                for (int j = 0; j < s->K; ++j) {
                    int k = i * s->K + j;
                    double py, px, m;
                    tap_position(s, off, mask, b, ho, wo, g, i, j, &py, &px, &m);
                    double gdy = 0.0, gdx = 0.0, gm = 0.0;
                    for (int c = g * Cg; c < (g + 1) * Cg; ++c) {
                        double gcol = column_grad(s, w, gyrow, i, j, c);
                        double dpy, dpx;
                        bilinear_grad(x, s, b, c, py, px, &dpy, &dpx);
                        gm += gcol * bilinear(x, s, b, c, py, px);
                        gdy += gcol * m * dpy;
                        gdx += gcol * m * dpx;
                    }
                    goff[(size_t)n * 2 * s->G * K2 + (size_t)g * 2 * K2 + 2 * k] = gdy;
                    goff[(size_t)n * 2 * s->G * K2 + (size_t)g * 2 * K2 + 2 * k + 1] = gdx;
                    if (gmask) gmask[(size_t)n * s->G * K2 + (size_t)g * K2 + k] = gm;
                }
    }
    return 0;
}

/* grad_weight at listed flat indices into [Cout, K, K, Cin]:
 * sum over every output pixel of gy[p, o] * m * x(sample). */
int dcn_oracle_grad_weight_entries(const dcn_oracle_shape* s, const double* x, const double* off, const double* mask,
                                   const double* gy, long n_ent, const long* idx, double* out) {
    if (s->G <= 0 || s->Cin % s->G) return -1;
    int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    int Cg = s->Cin / s->G;
    long n;
#pragma omp parallel for schedule(dynamic, 1)
    for (n = 0; n < n_ent; ++n) {
        long t = idx[n];
        int c = (int)(t % s->Cin), j = (int)((t / s->Cin) % s->K), i = (int)((t / ((long)s->Cin * s->K)) % s->K);
        int o = (int)(t / ((long)s->Cin * s->K * s->K));
        int g = c / Cg;
        double acc = 0.0;
        for (int b = 0; b < s->B; ++b)
            for (int ho = 0; ho < Ho; ++ho)
                for (int wo = 0; wo < Wo; ++wo) {
                    double py, px, m;
                    tap_position(s, off, mask, b, ho, wo, g, i, j, &py, &px, &m);
                    size_t p = ((size_t)b * Ho + ho) * Wo + wo;
                    acc += gy[p * s->Cout + o] * m * bilinear(x, s, b, c, py, px);
                }
        out[n] = acc;
    }
    return 0;
}

/* grad_x at listed flat indices into [B, H, W, Cin]: every (output pixel, tap)
 * of image b whose bilinear neighbourhood contains the input pixel adds
 * gcol * m * (its bilinear weight). */
int dcn_oracle_grad_x_entries(const dcn_oracle_shape* s, const double* off, const double* mask, const double* w,
                              const double* gy, long n_ent, const long* idx, double* out) {
    if (s->G <= 0 || s->Cin % s->G) return -1;
    int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    int Cg = s->Cin / s->G;
    long n;
#pragma omp parallel for schedule(dynamic, 1)
    for (n = 0; n < n_ent; ++n) {
        long t = idx[n];
        int c = (int)(t % s->Cin), q = (int)((t / s->Cin) % s->W), r = (int)((t / ((long)s->Cin * s->W)) % s->H);
        int b = (int)(t / ((long)s->Cin * s->W * s->H));
        int g = c / Cg;
        double acc = 0.0;
        for (int ho = 0; ho < Ho; ++ho)
            for (int wo = 0; wo < Wo; ++wo) {
                const double* gyrow = gy + (((size_t)b * Ho + ho) * Wo + wo) * s->Cout;
                for (int i = 0; i < s->K; ++i)
                    for (int j = 0; j < s->K; ++j) {
                        double py, px, m;
                        tap_position(s, off, mask, b, ho, wo, g, i, j, &py, &px, &m);
                        double y0 = floor(py), x0 = floor(px);
                        if (!(r == (int)y0 || r == (int)y0 + 1) || !(q == (int)x0 || q == (int)x0 + 1)) continue;
                        double gq = (1.0 - fabs(py - r)) * (1.0 - fabs(px - q));
                        acc += column_grad(s, w, gyrow, i, j, c) * m * gq;
                    }
            }
        out[n] = acc;
    }
    return 0;
}

/* --------------------------------------------------- offset/mask predictor -- */

/* The offsets and modulation scalars of a DCNv2 layer come from a separate
 * plain convolution over the same input, at the layer's own spatial resolution
 * (here: the layer's kernel size, stride, padding and dilation), with 3 output
 * channels per tap and group: the first 2*G*K*K outputs are the offsets, the
 * remaining G*K*K pass through a sigmoid and become the masks (notes, DCNv2
 * section 3.2, the paragraph after the modulated y(p0) equation).
 *   wp   [3*G*K*K, K, K, Cin]      bp [3*G*K*K] (NULL: no bias)
 *   off  [B, 2*G*K*K, Ho, Wo]      mask [B, G*K*K, Ho, Wo]
 * s->Cout is not used. */
int dcn_oracle_predict_offset_mask(const dcn_oracle_shape* s, const double* x, const double* wp, const double* bp,
                                   double* off, double* mask) {
    if (s->G <= 0 || s->K <= 0) return -1;
    const int Ho = dcn_oracle_out_h(s), Wo = dcn_oracle_out_w(s);
    const int K2 = s->K * s->K, NO = 2 * s->G * K2, NM = s->G * K2;
    long row;
    const long rows = (long)s->B * Ho;
#pragma omp parallel for schedule(dynamic, 4)
    for (row = 0; row < rows; ++row) {
        const int b = (int)(row / Ho), ho = (int)(row % Ho);
        for (int wo = 0; wo < Wo; ++wo) {
            for (int ch = 0; ch < NO + NM; ++ch) {
                double acc = bp ? bp[ch] : 0.0;
                for (int i = 0; i < s->K; ++i)
                    for (int j = 0; j < s->K; ++j)
                        for (int c = 0; c < s->Cin; ++c)
                            acc += wp[(((size_t)ch * s->K + i) * s->K + j) * s->Cin + c] *
                                   pixel_or_zero(x, s, b, ho * s->stride - s->pad + i * s->dil,
                                                 wo * s->stride - s->pad + j * s->dil, c);
                if (ch < NO)
                    off[(((size_t)b * NO + ch) * Ho + ho) * Wo + wo] = acc;
                else
                    mask[(((size_t)b * NM + (ch - NO)) * Ho + ho) * Wo + wo] = 1.0 / (1.0 + exp(-acc));
            }
        }
    }
    return 0;
}

/* --------------------------------------------------- deformable RoI pooling -- */

/* Deformable RoI pooling (notes, "可变形ROI pooling": RoI pooling cuts a RoI of
 * w x h into k x k bins and averages the pixels of each bin; the deformable form
 * first moves every bin as a whole by an offset given as a fraction of the RoI's
 * width and height, the moved positions being read by bilinear interpolation;
 * the explainer's "可变形RoI池化" paragraph: the offsets are normalised to the
 * RoI size; DCNv2 section 3.2: a modulation scalar per bin). The pages print no
 * formula for it; this follows the plainest reading of that text:
 *
 *   roi r = (b, x1, y1, x2, y2) in feature-map pixel coordinates,
 *   h = y2 - y1, w = x2 - x1 (a negative size counts as 0);
 *   bin (i, j), t = i*k + j, holds the integer offsets (u, v) with
 *     floor(i*h/k) <= u < ceil((i+1)*h/k),   floor(j*w/k) <= v < ceil((j+1)*w/k),
 *   n of them;
 *   its shift is (dy, dx) = gamma * (off[r][2t] * h, off[r][2t+1] * w);
 *   y[r][i][j][c] = m / n * sum over (u, v) of x_b(y1 + u + dy, x1 + v + dx, c),
 *   with m = mask[r][t] (1 without a mask), bilinear sampling whose neighbours
 *   outside the map contribute zero (as in the layer), and 0 for an empty bin.
 *
 * Layouts: x [B, H, W, C] (s->Cin = C; s->Cout, K, stride, pad, dil, G unused),
 * rois [R, 5], off [R, 2*k*k] or NULL (plain RoI pooling), mask [R, k*k] or
 * NULL, y and grad_y [R, k, k, C]. Returns -1 for a batch index out of range. */
static void roi_bin(const double* roi, int k, int i, int j, int* u0, int* u1, int* v0, int* v1, double* h,
                    double* w) {
    double hh = roi[4] - roi[2], ww = roi[3] - roi[1];
    if (hh < 0.0) hh = 0.0;
    if (ww < 0.0) ww = 0.0;
    *h = hh;
    *w = ww;
    *u0 = (int)floor(i * hh / k);
    *u1 = (int)ceil((i + 1) * hh / k);
    *v0 = (int)floor(j * ww / k);
    *v1 = (int)ceil((j + 1) * ww / k);
}

int dcn_oracle_droi_pool_forward(const dcn_oracle_shape* s, int R, int k, double gamma, const double* x,
                                 const double* rois, const double* off, const double* mask, double* y) {
    const int C = s->Cin, kk = k * k;
    for (int r = 0; r < R; ++r) {
        const double* roi = rois + (size_t)r * 5;
        const int b = (int)roi[0];
        if (b < 0 || b >= s->B) return -1;
        for (int i = 0; i < k; ++i)
            for (int j = 0; j < k; ++j) {
                int u0, u1, v0, v1;
                double h, w;
                roi_bin(roi, k, i, j, &u0, &u1, &v0, &v1, &h, &w);
                const int t = i * k + j;
                const double dy = off ? gamma * off[(size_t)r * 2 * kk + 2 * t] * h : 0.0;
                const double dx = off ? gamma * off[(size_t)r * 2 * kk + 2 * t + 1] * w : 0.0;
                const double m = mask ? mask[(size_t)r * kk + t] : 1.0;
                const int n = (u1 - u0) * (v1 - v0);
                double* yb = y + (((size_t)r * k + i) * k + j) * C;
                for (int c = 0; c < C; ++c) {
                    double acc = 0.0;
                    for (int u = u0; u < u1; ++u)
                        for (int v = v0; v < v1; ++v) acc += bilinear(x, s, b, c, roi[2] + u + dy, roi[1] + v + dx);
                    yb[c] = n > 0 ? m * acc / n : 0.0;
                }
            }
    }
    return 0;
}

/* Backward of the above: grad_x [B, H, W, C] (overwritten), grad_off [R, 2*k*k]
 * (the derivative with respect to the normalised offsets: gamma*h and gamma*w
 * times d/dy and d/dx of the bilinear samples, through floor() as in the layer),
 * grad_mask [R, k*k]; either of the last two may be NULL. */
int dcn_oracle_droi_pool_backward(const dcn_oracle_shape* s, int R, int k, double gamma, const double* x,
                                  const double* rois, const double* off, const double* mask, const double* gy,
                                  double* gx, double* goff, double* gmask) {
    const int C = s->Cin, kk = k * k;
    memset(gx, 0, sizeof(double) * (size_t)s->B * s->H * s->W * C);
    if (goff) memset(goff, 0, sizeof(double) * (size_t)R * 2 * kk);
    if (gmask) memset(gmask, 0, sizeof(double) * (size_t)R * kk);
    for (int r = 0; r < R; ++r) {
        const double* roi = rois + (size_t)r * 5;
        const int b = (int)roi[0];
        if (b < 0 || b >= s->B) return -1;
        for (int i = 0; i < k; ++i)
            for (int j = 0; j < k; ++j) {
                int u0, u1, v0, v1;
                double h, w;
                roi_bin(roi, k, i, j, &u0, &u1, &v0, &v1, &h, &w);
                const int t = i * k + j;
                const int n = (u1 - u0) * (v1 - v0);
                if (n == 0) continue;
                const double dy = off ? gamma * off[(size_t)r * 2 * kk + 2 * t] * h : 0.0;
                const double dx = off ? gamma * off[(size_t)r * 2 * kk + 2 * t + 1] * w : 0.0;
                const double m = mask ? mask[(size_t)r * kk + t] : 1.0;
                const double* gyb = gy + (((size_t)r * k + i) * k + j) * C;
                double g_dy = 0.0, g_dx = 0.0, g_m = 0.0;
                for (int c = 0; c < C; ++c) {
                    const double g = gyb[c] / n;
                    for (int u = u0; u < u1; ++u)
                        for (int v = v0; v < v1; ++v) {
                            const double py = roi[2] + u + dy, px = roi[1] + v + dx;
                            const double y0 = floor(py), x0 = floor(px);
                            for (int a = 0; a < 2; ++a)
                                for (int e = 0; e < 2; ++e) {
                                    const int rr = (int)y0 + a, qq = (int)x0 + e;
                                    if (rr < 0 || rr >= s->H || qq < 0 || qq >= s->W) continue;
                                    const double wt = (1.0 - fabs(py - rr)) * (1.0 - fabs(px - qq));
                                    gx[(((size_t)b * s->H + rr) * s->W + qq) * C + c] += g * m * wt;
                                }
                            double dpy, dpx;
                            bilinear_grad(x, s, b, c, py, px, &dpy, &dpx);
                            g_dy += g * m * dpy;
                            g_dx += g * m * dpx;
                            g_m += g * bilinear(x, s, b, c, py, px);
                        }
                }
                if (goff && off) {
                    goff[(size_t)r * 2 * kk + 2 * t] = g_dy * gamma * h;
                    goff[(size_t)r * 2 * kk + 2 * t + 1] = g_dx * gamma * w;
                }
                if (gmask && mask) gmask[(size_t)r * kk + t] = g_m;
            }
    }
    return 0;
}
