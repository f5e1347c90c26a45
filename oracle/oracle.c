/*
 * fp64 CPU oracle for the additive, differentiable 2D Gaussian-splatting
 * renderer ("predgsplat") of "Learning Video Dynamics with Predictive
 * Differentiable Rendering" (PDR).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg call this library.  The CUDA product path
 * never links, loads or calls it, and it shares no code with that path.
 *
 * What is computed (plain loops, fp64, no blocking, fusion or reordering):
 *   - each Gaussian has 5 + C parameters: position mu = (mu_x, mu_y),
 *     log-scales (s_1, s_2), rotation theta and C channel amplitudes a_c
 *     (paper abstract: "5 + C learnable parameters (position, scale,
 *     rotation, and C channel amplitudes)");
 *   - the field is an additive accumulation of the Gaussians (reading notes,
 *     "Method", first mechanism: additive accumulation; no opacity, no
 *     compositing, no depth order):
 *         I_c(p) = sum_i a_ic * exp(-1/2 (p - mu_i)^T Sigma_i^{-1} (p - mu_i)),
 *         Sigma_i = R(theta_i) diag(e^{2 s_i1}, e^{2 s_i2}) R(theta_i)^T,
 *     each Gaussian truncated to the k x k pixel window centred on
 *     round(mu_i) (the "kernel size" / "kernel support" knob of the reading
 *     notes, "Key Insight" and "Limitation");
 *   - the backward pass maps dL/dI to dL/d(mu, s, theta, a) for every
 *     Gaussian, pair by pair (Gaussian, window pixel), from the chain rule
 *     written out directly (abstract: a "differentiable" renderer).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - pixel (x, y) sits at the continuous coordinate p = (x, y), x = column,
 *     y = row; the window centre is round(mu) = floor(mu + 0.5), ties up,
 *     evaluated exactly for fp32 inputs (mu + 0.5 is exact in fp64);
 *   - R(theta) = [[cos, -sin], [sin, cos]]; u = R^T (p - mu) so
 *     q = e^{-2 s_1} u_1^2 + e^{-2 s_2} u_2^2;
 *   - window pixels outside the H x W grid are dropped (no wrap);
 *   - the window position is piecewise constant in mu: no gradient flows
 *     through round(mu);
 *   - a Gaussian with non-finite mu, or whose window misses the grid,
 *     contributes nothing and gets zero gradients;
 *   - the binning reference assigns Gaussian i to every 16 x 16 tile its
 *     clipped window touches, tiles in row-major order, ids ascending;
 *   - a frame may hold no Gaussians (N = 0): the empty sum, an all-zero
 *     image, no gradients and empty tile lists.
 *
 * Layouts: params [B][N][5+C] (mu_x, mu_y, s_1, s_2, theta, a_0..), fp32 for
 * the *_fwd / *_bwd / bin entry points and fp64 for the *_f64 ones (used by the
 * finite-difference checks); image and grad_image [B][C][H][W]; grad_params
 * like params.  All arithmetic is fp64.
 * Every function returns 0 on success and a negative value on bad arguments.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TILE 16

/* N = 0 is a frame with no Gaussians: the empty sum renders to zero. */
static int bad_sizes(int B, int N, int C, int H, int W, int k) {
    return B < 1 || N < 0 || C < 1 || H < 1 || W < 1 || k < 1 || (k % 2) == 0;
}

/* Clipped window of one Gaussian along one axis: pixels [lo, hi] of [0, n).
 * Returns 0 if the Gaussian has no pixel on this axis. */
static int window_axis(double mu, int r, int n, long long *lo, long long *hi) {
    if (!isfinite(mu)) return 0;
    double c = floor(mu + 0.5);              /* round half up, exact */
    if (c - r > (double)(n - 1) || c + r < 0.0) return 0;
    long long ci = (long long)c;             /* now |c| <= n + r: fits */
    long long a = ci - r, b = ci + r;
    if (a < 0) a = 0;
    if (b > n - 1) b = n - 1;
    *lo = a;
    *hi = b;
    return a <= b;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Forward render: image[b][c][y][x] = sum_i a_ic w_i(x, y), i ascending. */
int oracle_render_fwd_f64(const double *params, int B, int N, int C, int H,
                          int W, int k, double *image, int nthreads) {
    if (bad_sizes(B, N, C, H, W, k) || (N > 0 && !params) || !image) return -1;
    const int P = 5 + C;
    const int r = (k - 1) / 2;
    if (nthreads < 1) nthreads = 1;
    (void)nthreads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int b = 0; b < B; ++b) {
        double *img = image + (size_t)b * C * H * W;
        memset(img, 0, sizeof(double) * (size_t)C * H * W);
        for (int i = 0; i < N; ++i) {
            const double *g = params + ((size_t)b * N + i) * P;
            const double mx = g[0], my = g[1];
            const double e1 = exp(-2.0 * g[2]);
            const double e2 = exp(-2.0 * g[3]);
            const double ct = cos(g[4]), st = sin(g[4]);
            long long x0, x1, y0, y1;
            if (!window_axis(mx, r, W, &x0, &x1)) continue;
            if (!window_axis(my, r, H, &y0, &y1)) continue;
            for (long long y = y0; y <= y1; ++y) {
                for (long long x = x0; x <= x1; ++x) {
                    const double dx = (double)x - mx, dy = (double)y - my;
                    const double u1 = ct * dx + st * dy;
                    const double u2 = -st * dx + ct * dy;
                    const double q = e1 * u1 * u1 + e2 * u2 * u2;
                    const double w = exp(-0.5 * q);
                    for (int c = 0; c < C; ++c)
                        img[((size_t)c * H + y) * W + x] += g[5 + c] * w;
                }
            }
        }
    }
    return 0;
}

/* Backward: grad_params[b][i][.] = dL/d(mu_x, mu_y, s_1, s_2, theta, a_c),
 * accumulated pair by pair with
 *   G = sum_c g_c a_c,  t = dL/dq = -1/2 w G,
 *   da_c += g_c w,  ds_j += t (-2 u_j^2 e_j),  dtheta += t 2 u_1 u_2 (e_1 - e_2),
 *   dmu  += t (-2) R diag(e) u. */
int oracle_render_bwd_f64(const double *params, const double *grad_image,
                          int B, int N, int C, int H, int W, int k,
                          double *grad_params, int nthreads) {
    if (bad_sizes(B, N, C, H, W, k) || (N > 0 && (!params || !grad_params)) || !grad_image)
        return -1;
    const int P = 5 + C;
    const int r = (k - 1) / 2;
    if (nthreads < 1) nthreads = 1;
    (void)nthreads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int b = 0; b < B; ++b) {
        const double *gimg = grad_image + (size_t)b * C * H * W;
        for (int i = 0; i < N; ++i) {
            const double *g = params + ((size_t)b * N + i) * P;
            double *d = grad_params + ((size_t)b * N + i) * P;
            for (int j = 0; j < P; ++j) d[j] = 0.0;
            const double mx = g[0], my = g[1];
            const double e1 = exp(-2.0 * g[2]);
            const double e2 = exp(-2.0 * g[3]);
            const double ct = cos(g[4]), st = sin(g[4]);
            long long x0, x1, y0, y1;
            if (!window_axis(mx, r, W, &x0, &x1)) continue;
            if (!window_axis(my, r, H, &y0, &y1)) continue;
            for (long long y = y0; y <= y1; ++y) {
                for (long long x = x0; x <= x1; ++x) {
                    const double dx = (double)x - mx, dy = (double)y - my;
                    const double u1 = ct * dx + st * dy;
                    const double u2 = -st * dx + ct * dy;
                    const double q = e1 * u1 * u1 + e2 * u2 * u2;
                    const double w = exp(-0.5 * q);
                    double G = 0.0;
                    for (int c = 0; c < C; ++c) {
                        const double gc = gimg[((size_t)c * H + y) * W + x];
                        G += gc * g[5 + c];
                        d[5 + c] += gc * w;
                    }
                    const double t = -0.5 * w * G;
                    /* R diag(e) u */
                    const double rx = ct * e1 * u1 - st * e2 * u2;
                    const double ry = st * e1 * u1 + ct * e2 * u2;
                    d[0] += t * (-2.0) * rx;
                    d[1] += t * (-2.0) * ry;
                    d[2] += t * (-2.0 * u1 * u1 * e1);
                    d[3] += t * (-2.0 * u2 * u2 * e2);
                    d[4] += t * 2.0 * u1 * u2 * (e1 - e2);
                }
            }
        }
    }
    return 0;
}

/* fp32 entry points: the inputs are widened to fp64 once, then the fp64
 * loops above run unchanged. */
static double *widen(const float *src, size_t n) {
    double *dst = (double *)malloc(sizeof(double) * (n ? n : 1));
    if (dst)
        for (size_t j = 0; j < n; ++j) dst[j] = (double)src[j];
    return dst;
}

int oracle_render_fwd(const float *params, int B, int N, int C, int H, int W,
                      int k, double *image, int nthreads) {
    if (bad_sizes(B, N, C, H, W, k) || (N > 0 && !params) || !image) return -1;
    double *p = widen(params, (size_t)B * N * (5 + C));
    if (!p) return -2;
    int rc = oracle_render_fwd_f64(p, B, N, C, H, W, k, image, nthreads);
    free(p);
    return rc;
}

int oracle_render_bwd(const float *params, const float *grad_image, int B, int N,
                      int C, int H, int W, int k, double *grad_params,
                      int nthreads) {
    if (bad_sizes(B, N, C, H, W, k) || (N > 0 && (!params || !grad_params)) || !grad_image)
        return -1;
    double *p = widen(params, (size_t)B * N * (5 + C));
    double *g = widen(grad_image, (size_t)B * C * H * W);
    int rc = -2;
    if (p && g)
        rc = oracle_render_bwd_f64(p, g, B, N, C, H, W, k, grad_params, nthreads);
    free(p);
    free(g);
    return rc;
}

/* Brute-force binning: for every frame, every 16x16 tile (row-major) and every
 * Gaussian (ascending id), an integer rectangle-intersection test between the
 * Gaussian's clipped window and the tile.  tile_offsets has B*T + 1 entries
 * (global, frames concatenated); tile_ids holds the frame-local Gaussian index.
 * Returns the total number of entries E (>= 0); ids are written only while
 * they fit in cap (pass tile_ids = NULL, cap = 0 to count). */
long long oracle_bin(const float *params, int B, int N, int C, int H, int W, int k,
                     long long *tile_offsets, int *tile_ids, long long cap) {
    if (bad_sizes(B, N, C, H, W, k) || (N > 0 && !params)) return -1;
    const int P = 5 + C;
    const int r = (k - 1) / 2;
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE;
    long long e = 0;
    for (int b = 0; b < B; ++b) {
        for (int ty = 0; ty < TY; ++ty) {
            for (int tx = 0; tx < TX; ++tx) {
                if (tile_offsets) tile_offsets[((size_t)b * TY + ty) * TX + tx] = e;
                const long long px0 = (long long)tx * TILE, px1 = px0 + TILE - 1;
                const long long py0 = (long long)ty * TILE, py1 = py0 + TILE - 1;
                for (int i = 0; i < N; ++i) {
                    const float *g = params + ((size_t)b * N + i) * P;
                    long long x0, x1, y0, y1;
                    if (!window_axis(g[0], r, W, &x0, &x1)) continue;
                    if (!window_axis(g[1], r, H, &y0, &y1)) continue;
                    if (x1 < px0 || x0 > px1 || y1 < py0 || y0 > py1) continue;
                    if (tile_ids && e < cap) tile_ids[e] = i;
                    ++e;
                }
            }
        }
    }
    if (tile_offsets) tile_offsets[(size_t)B * TX * TY] = e;
    return e;
}
