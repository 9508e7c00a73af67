/*
 * CPU oracle for deformable sampling-aggregation (DCNv3 / DCNv4 core) and
 * multi-scale deformable attention (MSDeformAttn core).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * definition that the CUDA path is checked against.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or constant with the CUDA library and includes nothing
 * from it.
 *
 * Everything is float64 loop nests over the definition, in the order the
 * sources state it; there is no blocking, fusion or reordering.
 *
 * Sources (page title, section):
 *   [P1] "InternImage: Deformable Convolutions at Scale", ch.1 (deformable taps
 *        p0 + p_k + dp_k), ch.2 (bilinear read: x0 = floor(px), a = px - x0,
 *        corner weights (1-a)(1-b), a(1-b), (1-a)b, ab, zero outside the map),
 *        ch.3 (DCNv3 operator, stable softmax over the K taps), ch.4 (G groups,
 *        each with its own K offsets and modulations shared by its C/G channels).
 *   [P2] "DCNv4" note, "Why Is Sampling Just 9 Points Still Slow?" (the group
 *        formula y_g(p0) = sum_k m_gk x_g(p0 + p_k + dp_gk)) and "1. Remove
 *        Softmax" (m used as given, any real value).
 *   [P4] "Deformable DETR: Learn Where to Read", "A learned location can fall
 *        between cells" and helper 2 (x = u W - 1/2, y = v H - 1/2, tent weights
 *        (1-|x-i|)+ (1-|y-j|)+ over the four floor/ceil neighbours, zero
 *        outside, no clamping, no renormalisation) and helper 3 (h_m = sum over
 *        levels and points of A_mlk times the sampled value); "A reference links
 *        resolutions without equating their pixels" (point and box references
 *        scaled by the level's valid ratio, offsets divided by the level size
 *        or scaled by the box size).
 *   [P5] "OverLoCK" note, "ContMix: Put the Whole Image into the Kernel"
 *        (steps 4-5: a softmax turns each location's K^2 numbers into its own
 *        K x K kernel per channel group, which is applied to the zero-padded
 *        K x K neighbourhood of that group's channels; the note's snippet
 *        unfolds with padding K // 2, so taps are row-major, ky * K + kx).
 *
 * Readings where the sources are silent (each also listed in the design notes):
 *   - tap index k = ix * kh + iy for a kh x kw window (the grid R of [P1] ch.1 is
 *     listed with its first, x, component varying slowest);
 *   - offsets are (dx, dy) pairs, x along W ([P1] ch.2 writes p = (px, py));
 *   - sampling location in convolution form:
 *       px = ox*stride - pad + ix*dil + dx,  py = oy*stride - pad + iy*dil + dy,
 *     output size Ho = (H + 2 pad - dil (kh - 1) - 1) / stride + 1 (same for Wo);
 *   - MSDA spatial shapes are (H_l, W_l) pairs and value row = start_l + y W_l + x.
 */
#include <math.h>
#include <stdlib.h>

/* Bilinear read, [P1] ch.2: channel c of a channels-last map whose pixel (yy, xx)
 * starts at map[(yy*W + xx) * pix_stride].  Corners outside the map read 0.  The
 * corner coordinates are compared as doubles, so huge or non-finite locations
 * never reach an integer conversion. */
static double bilinear_pixel(const double *map, long H, long W, long pix_stride,
                             long c, double px, double py)
{
    double x0 = floor(px);
    double y0 = floor(py);
    double a = px - x0;
    double b = py - y0;
    double total = 0.0;
    for (int j = 0; j < 2; ++j) {          /* row y0 + j */
        for (int i = 0; i < 2; ++i) {      /* column x0 + i */
            double xx = x0 + i;
            double yy = y0 + j;
            double wx = (i == 0) ? (1.0 - a) : a;
            double wy = (j == 0) ? (1.0 - b) : b;
            if (xx >= 0.0 && xx < (double)W && yy >= 0.0 && yy < (double)H) {
                long idx = ((long)yy * W + (long)xx) * pix_stride + c;
                total += wx * wy * map[idx];
            }
        }
    }
    return total;
}

/* Output size of the deformable window, convolution form. */
long oracle_out_size(long in, long k, long stride, long pad, long dil)
{
    return (in + 2 * pad - dil * (k - 1) - 1) / stride + 1;
}

/*
 * DCNv3 (softmax_flag = 1) / DCNv4 (softmax_flag = 0) forward, [P1] ch.3-4 and
 * [P2] recap formula.
 *   x      [N][H][W][C]            C = G * D, group g = channels [gD, (g+1)D)
 *   offset [N][Ho][Wo][G][K][2]    (dx, dy) per tap
 *   mask   [N][Ho][Wo][G][K]       m (softmax_flag = 0) or logits z (= 1)
 *   out    [N][Ho][Wo][C]
 * Returns 0, or -1 on a bad argument.
 */
int oracle_dcn_forward(const double *x, const double *offset, const double *mask,
                       double *out, long N, long H, long W, long C, long G,
                       long kh, long kw, long stride, long pad, long dil,
                       int softmax_flag)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || kh <= 0 ||
        kw <= 0 || stride <= 0 || pad < 0 || dil <= 0)
        return -1;
    long Ho = oracle_out_size(H, kh, stride, pad, dil);
    long Wo = oracle_out_size(W, kw, stride, pad, dil);
    if (Ho <= 0 || Wo <= 0)
        return -1;
    long D = C / G;
    long K = kh * kw;
    double *m = (double *)malloc(sizeof(double) * (size_t)K);
    if (!m)
        return -1;

    for (long n = 0; n < N; ++n)
    for (long oy = 0; oy < Ho; ++oy)
    for (long ox = 0; ox < Wo; ++ox)
    for (long g = 0; g < G; ++g) {
        long site = ((n * Ho + oy) * Wo + ox) * G + g;   /* (pixel, group) */
        const double *off = offset + site * K * 2;
        const double *msk = mask + site * K;

        /* modulation: the given m (DCNv4), or the stable softmax of the logits
         * over this group's K taps (DCNv3, [P1] ch.3 worked example) */
        if (softmax_flag) {
            double zmax = msk[0];
            for (long k = 1; k < K; ++k)
                if (msk[k] > zmax)
                    zmax = msk[k];
            double sum = 0.0;
            for (long k = 0; k < K; ++k) {
                m[k] = exp(msk[k] - zmax);
                sum += m[k];
            }
            for (long k = 0; k < K; ++k)
                m[k] = m[k] / sum;
        } else {
            for (long k = 0; k < K; ++k)
                m[k] = msk[k];
        }

        const double *xg = x + n * H * W * C + g * D;     /* this group's channels */
        for (long c = 0; c < D; ++c) {
            double acc = 0.0;
            for (long ix = 0; ix < kw; ++ix) {
                for (long iy = 0; iy < kh; ++iy) {
                    long k = ix * kh + iy;
                    double px = (double)(ox * stride - pad + ix * dil) + off[2 * k];
                    double py = (double)(oy * stride - pad + iy * dil) + off[2 * k + 1];
                    acc += m[k] * bilinear_pixel(xg, H, W, C, c, px, py);
                }
            }
            out[((n * Ho + oy) * Wo + ox) * C + g * D + c] = acc;
        }
    }
    free(m);
    return 0;
}

/* Sample of one level with align_corners = False and zero padding, [P4] helper 2:
 * the tent weights (1-|x-col|)(1-|y-row|) over the floor/ceil neighbours of
 * (x, y) = (u W - 1/2, v H - 1/2).  Pixel (row, col) of head h, channel c is
 * value[(row*W + col) * pix_stride + c]. */
static double sample_level(const double *value, long H, long W, long pix_stride,
                           long c, double u, double v)
{
    double x = u * (double)W - 0.5;
    double y = v * (double)H - 0.5;
    double left = floor(x);
    double top = floor(y);
    double total = 0.0;
    for (int r = 0; r < 2; ++r) {
        for (int q = 0; q < 2; ++q) {
            double row = top + r;
            double col = left + q;
            double weight = (1.0 - fabs(x - col)) * (1.0 - fabs(y - row));
            if (row >= 0.0 && row < (double)H && col >= 0.0 && col < (double)W)
                total += weight * value[((long)row * W + (long)col) * pix_stride + c];
        }
    }
    return total;
}

/*
 * MSDeformAttn core forward, [P4] "Mix samples with a per-head budget":
 *   out[n][q][h*D + c] = sum_{l<L, k<K} A[n][q][h][l][k] *
 *                        sample_level(level l of value[n][.][h][c], loc[n][q][h][l][k])
 *   value        [N][S][M][D]       S = sum_l H_l W_l, levels concatenated
 *   shapes       [L][2]             (H_l, W_l)
 *   level_start  [L]                first row of level l in value
 *   loc          [N][Lq][M][L][K][2]  normalised (u, v), not clamped
 *   attn         [N][Lq][M][L][K]   already normalised weights
 *   out          [N][Lq][M*D]
 * Returns 0, or -1 on a bad argument.
 */
int oracle_msda_forward(const double *value, const long long *shapes,
                        const long long *level_start, const double *loc,
                        const double *attn, double *out, long N, long S, long Lq,
                        long M, long D, long L, long K)
{
    if (N < 0 || S <= 0 || Lq < 0 || M <= 0 || D <= 0 || L <= 0 || K <= 0)
        return -1;
    for (long l = 0; l < L; ++l) {
        if (shapes[2 * l] <= 0 || shapes[2 * l + 1] <= 0 || level_start[l] < 0 ||
            level_start[l] + shapes[2 * l] * shapes[2 * l + 1] > S)
            return -1;
    }
    for (long n = 0; n < N; ++n)
    for (long q = 0; q < Lq; ++q)
    for (long h = 0; h < M; ++h)
    for (long c = 0; c < D; ++c) {
        double acc = 0.0;
        for (long l = 0; l < L; ++l) {
            long Hl = (long)shapes[2 * l];
            long Wl = (long)shapes[2 * l + 1];
            const double *lvl = value + ((n * S + (long)level_start[l]) * M + h) * D;
            for (long k = 0; k < K; ++k) {
                long t = (((n * Lq + q) * M + h) * L + l) * K + k;
                acc += attn[t] * sample_level(lvl, Hl, Wl, M * D, c,
                                              loc[2 * t], loc[2 * t + 1]);
            }
        }
        out[(n * Lq + q) * M * D + h * D + c] = acc;
    }
    return 0;
}

/*
 * Sampling locations of the reference-point variants, [P4] "A reference links
 * resolutions without equating their pixels" (the point formula and the
 * remark that a box reference has its centre and size scaled by the level's
 * valid ratio first) and its step "Translate a reference into each sampling
 * frame" (the box replaces the offset term by (dp / K) (w, h) r_l / 2).
 * Everything is componentwise, x with widths and y with heights:
 *   point p = (px, py):        s = p r_l + dp / (W_l, H_l)
 *   box (cx, cy, w, h):        s = (cx, cy) r_l + (dp / K) (w, h) r_l / 2
 * with r_l = (W_valid / W_l, H_valid / H_l) of the image and level (1 when
 * valid_ratios is NULL).  Nothing is clamped.
 *   reference     [N][Lq][ref_dim]      ref_dim 2 (point) or 4 (box)
 *   valid_ratios  [N][L][2]             (x ratio, y ratio), or NULL
 *   offsets       [N][Lq][M][L][K][2]   dp = (dx, dy)
 *   shapes        [L][2]                (H_l, W_l)
 *   loc           [N][Lq][M][L][K][2]   out: normalised (u, v)
 * Returns 0, or -1 on a bad argument.
 */
int oracle_msda_locations(const double *reference, long ref_dim, const double *valid_ratios,
                          const double *offsets, const long long *shapes, double *loc,
                          long N, long Lq, long M, long L, long K)
{
    if (N < 0 || Lq < 0 || M <= 0 || L <= 0 || K <= 0 || (ref_dim != 2 && ref_dim != 4))
        return -1;
    for (long l = 0; l < L; ++l)
        if (shapes[2 * l] <= 0 || shapes[2 * l + 1] <= 0)
            return -1;
    for (long n = 0; n < N; ++n)
    for (long q = 0; q < Lq; ++q)
    for (long h = 0; h < M; ++h)
    for (long l = 0; l < L; ++l) {
        const double *ref = reference + (n * Lq + q) * ref_dim;
        double level_h = (double)shapes[2 * l];
        double level_w = (double)shapes[2 * l + 1];
        double ratio_x = valid_ratios ? valid_ratios[(n * L + l) * 2] : 1.0;
        double ratio_y = valid_ratios ? valid_ratios[(n * L + l) * 2 + 1] : 1.0;
        for (long k = 0; k < K; ++k) {
            long t = (((n * Lq + q) * M + h) * L + l) * K + k;
            double dx = offsets[2 * t];
            double dy = offsets[2 * t + 1];
            double u, v;
            if (ref_dim == 2) {
                u = ref[0] * ratio_x + dx / level_w;
                v = ref[1] * ratio_y + dy / level_h;
            } else {
                u = ref[0] * ratio_x + (dx / (double)K) * ref[2] * ratio_x / 2.0;
                v = ref[1] * ratio_y + (dy / (double)K) * ref[3] * ratio_y / 2.0;
            }
            loc[2 * t] = u;
            loc[2 * t + 1] = v;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Backward (gradients of the forward above), the plain chain rule.
 *
 * With L the loss and g = dL/dout, each output channel is
 *   out = sum_k m_k * sum_corners w_corner(a_k, b_k) * v_corner,
 * so (the bilinear weights being (1-a)(1-b), a(1-b), (1-a)b, ab with
 * a = px - floor(px), da/dpx = 1, between integer points):
 *   dL/dv_corner += g * m_k * w_corner                   (corner inside the map)
 *   dL/dm_k      += g * sample_k
 *   dL/dpx_k     += g * m_k * ((1-b)(v01 - v00) + b (v11 - v10))
 *   dL/dpy_k     += g * m_k * ((1-a)(v10 - v00) + a (v11 - v01))
 * with v = 0 for a corner outside the map.  At an exactly integer coordinate
 * the floor convention (a = 0, corners x0 and x0+1) gives the right-hand
 * derivative.  DCNv3: m = softmax(z) over K, dL/dz_k = m_k (dL/dm_k -
 * sum_j m_j dL/dm_j).  MSDA: x = u W - 1/2, so dL/du = W dL/dx.
 * ---------------------------------------------------------------------- */

/* value of corner (xx, yy) of channel c, 0 outside the map */
static double corner_value(const double *map, long H, long W, long pix_stride, long c,
                           double xx, double yy)
{
    if (xx >= 0.0 && xx < (double)W && yy >= 0.0 && yy < (double)H)
        return map[((long)yy * W + (long)xx) * pix_stride + c];
    return 0.0;
}

static void corner_add(double *map, long H, long W, long pix_stride, long c, double xx,
                       double yy, double v)
{
    if (xx >= 0.0 && xx < (double)W && yy >= 0.0 && yy < (double)H)
        map[((long)yy * W + (long)xx) * pix_stride + c] += v;
}

/*
 * DCNv3 / DCNv4 backward.  Inputs as oracle_dcn_forward plus grad_out
 * [N][Ho][Wo][C]; outputs (overwritten) grad_x [N][H][W][C], grad_offset
 * [N][Ho][Wo][G][K][2], grad_mask [N][Ho][Wo][G][K] (the gradient with respect
 * to the mask argument: m itself, or the logits when softmax_flag = 1).
 */
int oracle_dcn_backward(const double *x, const double *offset, const double *mask,
                        const double *grad_out, double *grad_x, double *grad_offset,
                        double *grad_mask, long N, long H, long W, long C, long G, long kh,
                        long kw, long stride, long pad, long dil, int softmax_flag)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || kh <= 0 ||
        kw <= 0 || stride <= 0 || pad < 0 || dil <= 0)
        return -1;
    long Ho = oracle_out_size(H, kh, stride, pad, dil);
    long Wo = oracle_out_size(W, kw, stride, pad, dil);
    if (Ho <= 0 || Wo <= 0)
        return -1;
    long D = C / G;
    long K = kh * kw;
    double *m = (double *)malloc(sizeof(double) * (size_t)K * 2);
    if (!m)
        return -1;
    double *gm = m + K;

    for (long i = 0; i < N * H * W * C; ++i)
        grad_x[i] = 0.0;

    for (long n = 0; n < N; ++n)
    for (long oy = 0; oy < Ho; ++oy)
    for (long ox = 0; ox < Wo; ++ox)
    for (long g = 0; g < G; ++g) {
        long site = ((n * Ho + oy) * Wo + ox) * G + g;
        const double *off = offset + site * K * 2;
        const double *msk = mask + site * K;
        double *goff = grad_offset + site * K * 2;
        double *gmsk = grad_mask + site * K;
        if (softmax_flag) {
            double zmax = msk[0];
            for (long k = 1; k < K; ++k)
                if (msk[k] > zmax)
                    zmax = msk[k];
            double sum = 0.0;
            for (long k = 0; k < K; ++k) {
                m[k] = exp(msk[k] - zmax);
                sum += m[k];
            }
            for (long k = 0; k < K; ++k)
                m[k] = m[k] / sum;
        } else {
            for (long k = 0; k < K; ++k)
                m[k] = msk[k];
        }
        const double *xg = x + n * H * W * C + g * D;
        double *gxg = grad_x + n * H * W * C + g * D;
        const double *go = grad_out + ((n * Ho + oy) * Wo + ox) * C + g * D;

        for (long ix = 0; ix < kw; ++ix)
        for (long iy = 0; iy < kh; ++iy) {
            long k = ix * kh + iy;
            double px = (double)(ox * stride - pad + ix * dil) + off[2 * k];
            double py = (double)(oy * stride - pad + iy * dil) + off[2 * k + 1];
            double x0 = floor(px), y0 = floor(py);
            double a = px - x0, b = py - y0;
            double gdx = 0.0, gdy = 0.0, gmk = 0.0;
            for (long c = 0; c < D; ++c) {
                double v00 = corner_value(xg, H, W, C, c, x0, y0);
                double v01 = corner_value(xg, H, W, C, c, x0 + 1, y0);
                double v10 = corner_value(xg, H, W, C, c, x0, y0 + 1);
                double v11 = corner_value(xg, H, W, C, c, x0 + 1, y0 + 1);
                double sample = (1 - a) * (1 - b) * v00 + a * (1 - b) * v01 +
                                (1 - a) * b * v10 + a * b * v11;
                gmk += go[c] * sample;
                gdx += go[c] * m[k] * ((1 - b) * (v01 - v00) + b * (v11 - v10));
                gdy += go[c] * m[k] * ((1 - a) * (v10 - v00) + a * (v11 - v01));
                double gm_c = go[c] * m[k];
                corner_add(gxg, H, W, C, c, x0, y0, gm_c * (1 - a) * (1 - b));
                corner_add(gxg, H, W, C, c, x0 + 1, y0, gm_c * a * (1 - b));
                corner_add(gxg, H, W, C, c, x0, y0 + 1, gm_c * (1 - a) * b);
                corner_add(gxg, H, W, C, c, x0 + 1, y0 + 1, gm_c * a * b);
            }
            goff[2 * k] = gdx;
            goff[2 * k + 1] = gdy;
            gm[k] = gmk;
        }
        if (softmax_flag) {
            double dot = 0.0;
            for (long k = 0; k < K; ++k)
                dot += m[k] * gm[k];
            for (long k = 0; k < K; ++k)
                gmsk[k] = m[k] * (gm[k] - dot);
        } else {
            for (long k = 0; k < K; ++k)
                gmsk[k] = gm[k];
        }
    }
    free(m);
    return 0;
}

/*
 * MSDeformAttn core backward.  Inputs as oracle_msda_forward plus grad_out
 * [N][Lq][M*D]; outputs (overwritten) grad_value [N][S][M][D], grad_loc
 * [N][Lq][M][L][K][2], grad_attn [N][Lq][M][L][K].
 */
int oracle_msda_backward(const double *value, const long long *shapes,
                         const long long *level_start, const double *loc,
                         const double *attn, const double *grad_out, double *grad_value,
                         double *grad_loc, double *grad_attn, long N, long S, long Lq, long M,
                         long D, long L, long K)
{
    if (N < 0 || S <= 0 || Lq < 0 || M <= 0 || D <= 0 || L <= 0 || K <= 0)
        return -1;
    for (long l = 0; l < L; ++l) {
        if (shapes[2 * l] <= 0 || shapes[2 * l + 1] <= 0 || level_start[l] < 0 ||
            level_start[l] + shapes[2 * l] * shapes[2 * l + 1] > S)
            return -1;
    }
    for (long i = 0; i < N * S * M * D; ++i)
        grad_value[i] = 0.0;
    for (long i = 0; i < N * Lq * M * L * K; ++i) {
        grad_attn[i] = 0.0;
        grad_loc[2 * i] = 0.0;
        grad_loc[2 * i + 1] = 0.0;
    }
    for (long n = 0; n < N; ++n)
    for (long q = 0; q < Lq; ++q)
    for (long h = 0; h < M; ++h)
    for (long c = 0; c < D; ++c) {
        double go = grad_out[(n * Lq + q) * M * D + h * D + c];
        for (long l = 0; l < L; ++l) {
            long Hl = (long)shapes[2 * l];
            long Wl = (long)shapes[2 * l + 1];
            long off = ((n * S + (long)level_start[l]) * M + h) * D;
            const double *lvl = value + off;
            double *glvl = grad_value + off;
            for (long k = 0; k < K; ++k) {
                long t = (((n * Lq + q) * M + h) * L + l) * K + k;
                double A = attn[t];
                double x = loc[2 * t] * (double)Wl - 0.5;
                double y = loc[2 * t + 1] * (double)Hl - 0.5;
                double x0 = floor(x), y0 = floor(y);
                double a = x - x0, b = y - y0;
                double v00 = corner_value(lvl, Hl, Wl, M * D, c, x0, y0);
                double v01 = corner_value(lvl, Hl, Wl, M * D, c, x0 + 1, y0);
                double v10 = corner_value(lvl, Hl, Wl, M * D, c, x0, y0 + 1);
                double v11 = corner_value(lvl, Hl, Wl, M * D, c, x0 + 1, y0 + 1);
                double sample = (1 - a) * (1 - b) * v00 + a * (1 - b) * v01 +
                                (1 - a) * b * v10 + a * b * v11;
                grad_attn[t] += go * sample;
                grad_loc[2 * t] += go * A * ((1 - b) * (v01 - v00) + b * (v11 - v10)) * Wl;
                grad_loc[2 * t + 1] += go * A * ((1 - a) * (v10 - v00) + a * (v11 - v01)) * Hl;
                double ga = go * A;
                corner_add(glvl, Hl, Wl, M * D, c, x0, y0, ga * (1 - a) * (1 - b));
                corner_add(glvl, Hl, Wl, M * D, c, x0 + 1, y0, ga * a * (1 - b));
                corner_add(glvl, Hl, Wl, M * D, c, x0, y0 + 1, ga * (1 - a) * b);
                corner_add(glvl, Hl, Wl, M * D, c, x0 + 1, y0 + 1, ga * a * b);
            }
        }
    }
    return 0;
}

/*
 * Dynamic local aggregation (the ContMix core), [P5] "ContMix" steps 4-5.
 * x [N][H][W][C], w [N][H][W][G][K*K] (tap t = ky * K + kx), out [N][H][W][C]:
 *   out[n][y][x][g*D + c] = sum_{ky, kx} A[t] * x[n][y + ky - K/2][x + kx - K/2][g*D + c]
 * with 0 outside the map, A = softmax over the K*K weights of the location and
 * group (softmax_flag = 1) or the weights as given (0).  K must be odd (the
 * output keeps the input size).
 */
int oracle_dynconv_forward(const double *x, const double *w, double *out, long N, long H,
                           long W, long C, long G, long K, int softmax_flag)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || K <= 0 || K % 2 != 1)
        return -1;
    long D = C / G;
    long KK = K * K;
    long r = K / 2;
    double *A = (double *)malloc(sizeof(double) * (size_t)KK);
    if (!A)
        return -1;
    for (long n = 0; n < N; ++n)
    for (long y = 0; y < H; ++y)
    for (long xx = 0; xx < W; ++xx)
    for (long g = 0; g < G; ++g) {
        const double *wt = w + (((n * H + y) * W + xx) * G + g) * KK;
        if (softmax_flag) {
            double zmax = wt[0];
            for (long t = 1; t < KK; ++t)
                if (wt[t] > zmax)
                    zmax = wt[t];
            double sum = 0.0;
            for (long t = 0; t < KK; ++t) {
                A[t] = exp(wt[t] - zmax);
                sum += A[t];
            }
            for (long t = 0; t < KK; ++t)
                A[t] = A[t] / sum;
        } else {
            for (long t = 0; t < KK; ++t)
                A[t] = wt[t];
        }
        for (long c = 0; c < D; ++c) {
            double acc = 0.0;
            for (long ky = 0; ky < K; ++ky)
            for (long kx = 0; kx < K; ++kx) {
                long sy = y + ky - r, sx = xx + kx - r;
                if (sy < 0 || sy >= H || sx < 0 || sx >= W)
                    continue;
                acc += A[ky * K + kx] * x[((n * H + sy) * W + sx) * C + g * D + c];
            }
            out[((n * H + y) * W + xx) * C + g * D + c] = acc;
        }
    }
    free(A);
    return 0;
}
