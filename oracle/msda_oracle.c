/*
 * msda_oracle.c -- plain CPU oracle of the multi-scale deformable attention
 * (MSDeformAttn) core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes is the definition written out, loop by loop, with no
 * blocking, fusion or reordering:
 *
 *   out[n,q,m,:] = sum_l sum_k A[n,q,m,l,k] * bilinear(x^l_m, loc[n,q,m,l,k])
 *
 * ("Deformable DETR" wiki page, "Multi-scale deformable attention" equation:
 * the value projection W'_m is taken as already applied, so x^l_m is head m's
 * D-channel slice of the value map, and the output projection W_m is left to
 * the caller; heads are concatenated, "Deformable Attention" glossary page,
 * multi-head paragraph.)
 *
 * Precision: location -> pixel arithmetic is done either in fp32 (the way the
 * inputs are given, so that cell indices and fractions are reproducible bit for
 * bit) or entirely in fp64 (for finite-difference checks).  Corner weights,
 * products and sums are always accumulated in fp64.
 *
 * Readings of points the pages leave open (each one is stated beside the code
 * that takes it):
 *   R1 pixel convention: x = loc_x * W - 0.5, y = loc_y * H - 0.5 (pixel
 *      centres at half-integers in normalised units; this is
 *      grid_sample(align_corners=False)).
 *   R2 zero padding: a corner outside the map contributes 0; nothing is
 *      clamped or renormalised.  A sample with NaN/Inf coordinates, or one
 *      with no corner inside the map, contributes 0 and has zero gradient.
 *   R3 coordinate order (x, y), x along the width; spatial_shapes = (H, W).
 *   R4 fused offsets are level-l pixels: loc = ref + off / W_l (fp32 divide
 *      then fp32 add, both rounded to nearest).
 *   R5 softmax per (n, q, m) jointly over the L*K logits.
 *   R6 at a kink (integer x or y) the gradient is the one of the cell chosen
 *      by floor(), i.e. the right-hand derivative.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t N, Lq, S, M, D, L, K;
} ora_dims;

void ora_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int ora_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ *
 * Level metadata.  Level l occupies rows [start_l, start_l + H_l*W_l) of the
 * flattened value map; start_l is the exclusive prefix sum of H_j*W_j
 * ("Deformable DETR" wiki page, "Multi-scale deformable attention": L levels
 * x^l of sizes H^l x W^l).  Returns S = sum_l H_l*W_l.
 * ------------------------------------------------------------------------ */
int64_t ora_level_start_index(const int64_t *shapes, int64_t L, int64_t *starts)
{
    int64_t acc = 0;
    for (int64_t l = 0; l < L; ++l) {
        starts[l] = acc;
        acc += shapes[2 * l] * shapes[2 * l + 1];
    }
    return acc;
}

/* value is fp32, or bf16 stored as its 16-bit pattern (widening is exact). */
static double value_at(const void *value, int bf16, int64_t idx)
{
    if (bf16) {
        uint32_t u = ((const uint16_t *)value)[idx];
        u <<= 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)value)[idx];
}

/* A sampling point on level l: the cell (x0, y0) and the fractions. */
typedef struct {
    int valid;
    int64_t x0, y0;
    double fx, fy;
} ora_point;

/*
 * phi_l followed by the pixel convention R1 ("Deformable DETR" wiki page,
 * "Multi-scale deformable attention": phi_l rescales the normalised point by
 * the level's H^l, W^l).  In fp32 mode every operation is one IEEE fp32
 * operation, in the order written, with no fused multiply-add.
 */
static ora_point locate(double lx, double ly, int64_t H, int64_t W, int f32)
{
    ora_point p;
    p.valid = 0;
    p.x0 = p.y0 = 0;
    p.fx = p.fy = 0.0;
    if (f32) {
        float xf = (float)lx * (float)W;
        xf = xf - 0.5f;
        float yf = (float)ly * (float)H;
        yf = yf - 0.5f;
        /* R2: outside (-1, W) x (-1, H) no corner is inside the map; NaN fails too. */
        if (!(xf > -1.0f && xf < (float)W && yf > -1.0f && yf < (float)H))
            return p;
        /* From the fp32 pixel coordinate on, the arithmetic is exact: the
         * cell is floor(x) and the fraction x - floor(x) is taken in fp64
         * (in fp32 it would round for x in (-1, 0)). */
        float x0 = floorf(xf), y0 = floorf(yf);
        p.x0 = (int64_t)x0;
        p.y0 = (int64_t)y0;
        p.fx = (double)xf - (double)x0;
        p.fy = (double)yf - (double)y0;
    } else {
        double x = lx * (double)W - 0.5;
        double y = ly * (double)H - 0.5;
        if (!(x > -1.0 && x < (double)W && y > -1.0 && y < (double)H))
            return p;
        double x0 = floor(x), y0 = floor(y);
        p.x0 = (int64_t)x0;
        p.y0 = (int64_t)y0;
        p.fx = x - x0;
        p.fy = y - y0;
    }
    p.valid = 1;
    return p;
}

/* Row of pixel (yy, xx) of level l in the flattened map, or -1 if the pixel
 * lies outside the level (zero padding, R2). */
static int64_t pixel_row(const int64_t *shapes, const int64_t *starts,
                         int64_t l, int64_t yy, int64_t xx)
{
    int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
    if (xx < 0 || xx >= W || yy < 0 || yy >= H)
        return -1;
    return starts[l] + yy * W + xx;
}

/*
 * Forward ("Deformable DETR" wiki page, "Multi-scale deformable attention"
 * equation; each sample interpolated bilinearly between the four pixels
 * around it, same page, "Deformable attention module").
 *
 *   value [N,S,M,D]  fp32 or bf16 bits      loc  [N,Lq,M,L,K,2] (x,y)
 *   attn  [N,Lq,M,L,K] (fp64)              out  [N,Lq,M*D] (fp64)
 *
 * loc_f32 = 1: loc holds fp32 values and the pixel arithmetic is fp32.
 * loc_f32 = 0: the pixel arithmetic is fp64.
 * Queries [q_begin, q_end) of every batch entry are computed; other rows of
 * out are left untouched.
 */
void ora_forward(const void *value, int value_bf16, const int64_t *shapes,
                 const int64_t *starts, const double *loc, int loc_f32,
                 const double *attn, double *out, ora_dims d,
                 int64_t q_begin, int64_t q_end)
{
    const int64_t N = d.N, Lq = d.Lq, S = d.S, M = d.M, D = d.D, L = d.L, K = d.K;
    const int64_t nq_total = N * (q_end - q_begin);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nq_total; ++t) {
        const int64_t n = t / (q_end - q_begin);
        const int64_t q = q_begin + t % (q_end - q_begin);
        for (int64_t m = 0; m < M; ++m) {
            double *o = out + ((n * Lq + q) * M + m) * D;
            for (int64_t c = 0; c < D; ++c)
                o[c] = 0.0;
            for (int64_t l = 0; l < L; ++l) {
                const int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
                for (int64_t k = 0; k < K; ++k) {
                    const int64_t i = (((n * Lq + q) * M + m) * L + l) * K + k;
                    ora_point p = locate(loc[2 * i], loc[2 * i + 1], H, W, loc_f32);
                    if (!p.valid)
                        continue;
                    const double a = attn[i];
                    /* corners: (y0,x0) (y0,x0+1) (y0+1,x0) (y0+1,x0+1) */
                    const double w[4] = {(1.0 - p.fx) * (1.0 - p.fy), p.fx * (1.0 - p.fy),
                                         (1.0 - p.fx) * p.fy, p.fx * p.fy};
                    const int64_t r[4] = {pixel_row(shapes, starts, l, p.y0, p.x0),
                                          pixel_row(shapes, starts, l, p.y0, p.x0 + 1),
                                          pixel_row(shapes, starts, l, p.y0 + 1, p.x0),
                                          pixel_row(shapes, starts, l, p.y0 + 1, p.x0 + 1)};
                    for (int64_t c = 0; c < D; ++c) {
                        double s = 0.0;
                        for (int j = 0; j < 4; ++j)
                            if (r[j] >= 0)
                                s += w[j] * value_at(value, value_bf16,
                                                     ((n * S + r[j]) * M + m) * D + c);
                        o[c] += a * s;
                    }
                }
            }
        }
    }
}

/*
 * Joint softmax over the L*K logits of one (n, q, m) ("Deformable DETR" wiki
 * page, "Multi-scale deformable attention": sum_l sum_k A_mlqk = 1; "Deformable
 * attention module": the last MK projection channels go through a softmax).
 * Max-subtracted, fp64.  groups = N*Lq*M, LK = L*K.
 */
void ora_softmax(const double *logits, double *attn, int64_t groups, int64_t LK)
{
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < groups; ++g) {
        const double *z = logits + g * LK;
        double *a = attn + g * LK;
        double mx = z[0];
        for (int64_t j = 1; j < LK; ++j)
            if (z[j] > mx)
                mx = z[j];
        double s = 0.0;
        for (int64_t j = 0; j < LK; ++j) {
            a[j] = exp(z[j] - mx);
            s += a[j];
        }
        for (int64_t j = 0; j < LK; ++j)
            a[j] /= s;
    }
}

/*
 * Sampling location from the reference point and a pixel offset: phi_l(p) +
 * dp is a point in level-l pixels, so in normalised units it is p + dp / W_l
 * along x and p + dp / H_l along y (R4; "Deformable DETR" wiki page,
 * "Multi-scale deformable attention").  fp32: one IEEE divide, then one IEEE
 * add.
 *   ref [N,Lq,2]   off [N,Lq,M,L,K,2]   loc [N,Lq,M,L,K,2]
 */
void ora_locations_f32(const float *ref, const float *off, const int64_t *shapes,
                       ora_dims d, float *loc)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q)
            for (int64_t m = 0; m < M; ++m)
                for (int64_t l = 0; l < L; ++l)
                    for (int64_t k = 0; k < K; ++k) {
                        const int64_t i = (((n * Lq + q) * M + m) * L + l) * K + k;
                        const float Wf = (float)shapes[2 * l + 1];
                        const float Hf = (float)shapes[2 * l];
                        float dx = off[2 * i] / Wf;
                        float dy = off[2 * i + 1] / Hf;
                        loc[2 * i] = ref[2 * (n * Lq + q)] + dx;
                        loc[2 * i + 1] = ref[2 * (n * Lq + q) + 1] + dy;
                    }
}

/*
 * Box reference (iterative bounding-box refinement, "Deformable DETR" wiki
 * page, "Variants"): the previous layer's box (cx, cy, w, h) is the reference
 * and the offsets are scaled by the box size, so in normalised units
 * loc_x = cx + off_x * w, loc_y = cy + off_y * h (offsets in box units; the
 * page's 1/(2K) scaling of the initial offsets is a property of the offsets,
 * not of this map).  fp32: one IEEE multiply, then one IEEE add.
 *   box [N,Lq,4]   off [N,Lq,M,L,K,2]   loc [N,Lq,M,L,K,2]
 */
void ora_locations_box_f32(const float *box, const float *off, ora_dims d, float *loc)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q)
            for (int64_t j = 0; j < M * L * K; ++j) {
                const int64_t i = (n * Lq + q) * M * L * K + j;
                const float *b = box + 4 * (n * Lq + q);
                float dx = off[2 * i] * b[2];
                float dy = off[2 * i + 1] * b[3];
                loc[2 * i] = b[0] + dx;
                loc[2 * i + 1] = b[1] + dy;
            }
}

/* The same map in fp64 (finite-difference checks of the fused chain). */
void ora_locations_f64(const double *ref, const double *off, const int64_t *shapes,
                       ora_dims d, double *loc)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q)
            for (int64_t m = 0; m < M; ++m)
                for (int64_t l = 0; l < L; ++l)
                    for (int64_t k = 0; k < K; ++k) {
                        const int64_t i = (((n * Lq + q) * M + m) * L + l) * K + k;
                        loc[2 * i] = ref[2 * (n * Lq + q)] + off[2 * i] / (double)shapes[2 * l + 1];
                        loc[2 * i + 1] = ref[2 * (n * Lq + q) + 1] + off[2 * i + 1] / (double)shapes[2 * l];
                    }
}

/*
 * Backward of ora_forward: the gradients flow through the interpolation to
 * the value, the locations and the weights ("Deformable DETR" wiki page,
 * "Deformable attention module": the interpolation lets gradients reach
 * the offsets; "Deformable Attention" glossary page: the interpolation
 * passes gradients on to the offset prediction).
 *
 * With g = grad_out[n,q,m,:] and corner weights w_j(fx, fy):
 *   grad_attn[i]       = sum_j w_j <v_j, g>
 *   grad_value[row_j] += A_i w_j g              (corners inside the map)
 *   grad_loc_x[i]      = A_i * W * sum_j dw_j/dfx <v_j, g>
 *   grad_loc_y[i]      = A_i * H * sum_j dw_j/dfy <v_j, g>
 * (dx/dloc_x = W by R1; dfx/dx = 1 by R6; outside corners have v_j = 0.)
 * grad_value [N,S,M,D] is overwritten.  Serial per (n, m): rows of different
 * (n, m) are disjoint, so the result is deterministic.  grad_value may be
 * NULL: the per-sample gradients are then formed without the scatter (for
 * value maps too large to mirror in fp64).
 *
 * grad_loc_mass / grad_attn_mass (may be NULL) receive the absolute mass of
 * each sum, the same expression with every term replaced by its absolute
 * value (e.g. A*W*sum_j |dw_j/dfx| sum_c |v_jc g_c|).  They are not part of
 * the method: they scale the rounding-error bound of a finite-precision
 * evaluation of the same sum, |fl(sum) - sum| <= n*u*mass.
 */
void ora_backward(const void *value, int value_bf16, const int64_t *shapes,
                  const int64_t *starts, const double *loc, int loc_f32,
                  const double *attn, const double *grad_out, double *grad_value,
                  double *grad_loc, double *grad_attn, double *grad_loc_mass,
                  double *grad_attn_mass, ora_dims d)
{
    const int64_t N = d.N, Lq = d.Lq, S = d.S, M = d.M, D = d.D, L = d.L, K = d.K;
    if (grad_value)
        memset(grad_value, 0, sizeof(double) * (size_t)(N * S * M * D));
#pragma omp parallel for schedule(static)
    for (int64_t nm = 0; nm < N * M; ++nm) {
        const int64_t n = nm / M, m = nm % M;
        for (int64_t q = 0; q < Lq; ++q) {
            const double *g = grad_out + ((n * Lq + q) * M + m) * D;
            for (int64_t l = 0; l < L; ++l) {
                const int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
                for (int64_t k = 0; k < K; ++k) {
                    const int64_t i = (((n * Lq + q) * M + m) * L + l) * K + k;
                    ora_point p = locate(loc[2 * i], loc[2 * i + 1], H, W, loc_f32);
                    if (!p.valid) {
                        grad_attn[i] = 0.0;
                        grad_loc[2 * i] = 0.0;
                        grad_loc[2 * i + 1] = 0.0;
                        if (grad_loc_mass) {
                            grad_loc_mass[2 * i] = 0.0;
                            grad_loc_mass[2 * i + 1] = 0.0;
                        }
                        if (grad_attn_mass)
                            grad_attn_mass[i] = 0.0;
                        continue;
                    }
                    const double a = attn[i];
                    double dA = 0.0, dfx = 0.0, dfy = 0.0;
                    double mA = 0.0, mfx = 0.0, mfy = 0.0;
                    for (int cy = 0; cy < 2; ++cy)
                        for (int cx = 0; cx < 2; ++cx) {
                            const double wx = cx ? p.fx : 1.0 - p.fx;
                            const double wy = cy ? p.fy : 1.0 - p.fy;
                            const double w = wx * wy;
                            const double sx = cx ? 1.0 : -1.0; /* d wx / d fx */
                            const double sy = cy ? 1.0 : -1.0; /* d wy / d fy */
                            const int64_t r = pixel_row(shapes, starts, l, p.y0 + cy, p.x0 + cx);
                            if (r < 0)
                                continue; /* v = 0: no term, no scatter */
                            double vg = 0.0, vg_abs = 0.0;
                            for (int64_t c = 0; c < D; ++c) {
                                const int64_t e = ((n * S + r) * M + m) * D + c;
                                vg += value_at(value, value_bf16, e) * g[c];
                                vg_abs += fabs(value_at(value, value_bf16, e) * g[c]);
                                if (grad_value)
                                    grad_value[e] += a * w * g[c];
                            }
                            dA += w * vg;
                            dfx += sx * wy * vg;
                            dfy += sy * wx * vg;
                            mA += w * vg_abs;
                            mfx += wy * vg_abs;
                            mfy += wx * vg_abs;
                        }
                    grad_attn[i] = dA;
                    grad_loc[2 * i] = a * (double)W * dfx;
                    grad_loc[2 * i + 1] = a * (double)H * dfy;
                    if (grad_loc_mass) {
                        grad_loc_mass[2 * i] = fabs(a) * (double)W * mfx;
                        grad_loc_mass[2 * i + 1] = fabs(a) * (double)H * mfy;
                    }
                    if (grad_attn_mass)
                        grad_attn_mass[i] = mA;
                }
            }
        }
    }
}

/*
 * Chain rule from the sampled-point gradients back to the fused inputs
 * (loc = ref + off / W_l, A = softmax(z) over the L*K logits of a head):
 *   grad_off_x = grad_loc_x / W_l,  grad_off_y = grad_loc_y / H_l
 *   grad_ref   = sum over (m, l, k) of grad_loc
 *   grad_z     = A * (grad_A - sum_j A_j grad_A_j)       (softmax Jacobian)
 * All fp64.  grad_ref [N,Lq,2], grad_off like off, grad_logits like logits.
 */
void ora_fused_chain(const double *grad_loc, const double *grad_attn, const double *attn,
                     const int64_t *shapes, ora_dims d, double *grad_ref,
                     double *grad_off, double *grad_logits)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q) {
            double rx = 0.0, ry = 0.0;
            for (int64_t m = 0; m < M; ++m) {
                const int64_t base = ((n * Lq + q) * M + m) * L * K;
                double dot = 0.0;
                for (int64_t j = 0; j < L * K; ++j)
                    dot += attn[base + j] * grad_attn[base + j];
                for (int64_t j = 0; j < L * K; ++j)
                    grad_logits[base + j] = attn[base + j] * (grad_attn[base + j] - dot);
                for (int64_t l = 0; l < L; ++l)
                    for (int64_t k = 0; k < K; ++k) {
                        const int64_t i = base + l * K + k;
                        grad_off[2 * i] = grad_loc[2 * i] / (double)shapes[2 * l + 1];
                        grad_off[2 * i + 1] = grad_loc[2 * i + 1] / (double)shapes[2 * l];
                        rx += grad_loc[2 * i];
                        ry += grad_loc[2 * i + 1];
                    }
            }
            grad_ref[2 * (n * Lq + q)] = rx;
            grad_ref[2 * (n * Lq + q) + 1] = ry;
        }
}

/*
 * The same chain for box references (cx, cy, w, h) with loc = (cx, cy) +
 * off * (w, h) (iterative box refinement, "Deformable DETR" wiki page,
 * "Variants"):
 *   grad_off_x = grad_loc_x * w,  grad_off_y = grad_loc_y * h
 *   grad_box   = (sum grad_loc_x, sum grad_loc_y,
 *                 sum grad_loc_x * off_x, sum grad_loc_y * off_y)
 *   grad_z     = A * (grad_A - sum_j A_j grad_A_j)
 * box [N,Lq,4], off like grad_loc, grad_box [N,Lq,4].  fp64.
 */
void ora_fused_chain_box(const double *grad_loc, const double *grad_attn, const double *attn,
                         const double *box, const double *off, ora_dims d, double *grad_box,
                         double *grad_off, double *grad_logits)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q) {
            const double *b = box + 4 * (n * Lq + q);
            double gcx = 0.0, gcy = 0.0, gw = 0.0, gh = 0.0;
            for (int64_t m = 0; m < M; ++m) {
                const int64_t base = ((n * Lq + q) * M + m) * L * K;
                double dot = 0.0;
                for (int64_t j = 0; j < L * K; ++j)
                    dot += attn[base + j] * grad_attn[base + j];
                for (int64_t j = 0; j < L * K; ++j) {
                    const int64_t i = base + j;
                    grad_logits[i] = attn[i] * (grad_attn[i] - dot);
                    grad_off[2 * i] = grad_loc[2 * i] * b[2];
                    grad_off[2 * i + 1] = grad_loc[2 * i + 1] * b[3];
                    gcx += grad_loc[2 * i];
                    gcy += grad_loc[2 * i + 1];
                    gw += grad_loc[2 * i] * off[2 * i];
                    gh += grad_loc[2 * i + 1] * off[2 * i + 1];
                }
            }
            double *gb = grad_box + 4 * (n * Lq + q);
            gb[0] = gcx;
            gb[1] = gcy;
            gb[2] = gw;
            gb[3] = gh;
        }
}

/* fp64 box location map (finite-difference checks). */
void ora_locations_box_f64(const double *box, const double *off, ora_dims d, double *loc)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q)
            for (int64_t j = 0; j < M * L * K; ++j) {
                const int64_t i = (n * Lq + q) * M * L * K + j;
                const double *b = box + 4 * (n * Lq + q);
                loc[2 * i] = b[0] + off[2 * i] * b[2];
                loc[2 * i + 1] = b[1] + off[2 * i + 1] * b[3];
            }
}

/*
 * Per-sample index record, for bit-exact comparison of the cell arithmetic:
 * valid flag, the fp32 pixel coordinates (x, y) = (loc_x*W - 0.5,
 * loc_y*H - 0.5), the cell (x0, y0), and the flattened row of each of the
 * four corners in the order (y0,x0) (y0,x0+1) (y0+1,x0) (y0+1,x0+1), -1 for a
 * corner outside the map (R1, R2).  Invalid samples record x0 = y0 = 0.
 *   loc [N,Lq,M,L,K,2] fp32; every output has one entry (rows: four) per sample.
 */
void ora_sample_points_f32(const float *loc, const int64_t *shapes, const int64_t *starts,
                           ora_dims d, int32_t *valid, int32_t *x0, int32_t *y0,
                           float *px, float *py, int64_t *rows)
{
    const int64_t N = d.N, Lq = d.Lq, M = d.M, L = d.L, K = d.K;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < Lq; ++q)
            for (int64_t m = 0; m < M; ++m)
                for (int64_t l = 0; l < L; ++l)
                    for (int64_t k = 0; k < K; ++k) {
                        const int64_t i = (((n * Lq + q) * M + m) * L + l) * K + k;
                        ora_point p = locate((double)loc[2 * i], (double)loc[2 * i + 1],
                                             shapes[2 * l], shapes[2 * l + 1], 1);
                        float xf = loc[2 * i] * (float)shapes[2 * l + 1];
                        xf = xf - 0.5f;
                        float yf = loc[2 * i + 1] * (float)shapes[2 * l];
                        yf = yf - 0.5f;
                        valid[i] = p.valid;
                        x0[i] = (int32_t)p.x0;
                        y0[i] = (int32_t)p.y0;
                        px[i] = xf;
                        py[i] = yf;
                        for (int j = 0; j < 4; ++j)
                            rows[4 * i + j] = p.valid
                                ? pixel_row(shapes, starts, l, p.y0 + (j >> 1), p.x0 + (j & 1))
                                : -1;
                    }
}
