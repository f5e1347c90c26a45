// L1 + SSIM training loss and its gradient dL/dI (the objective the reading
// notes, section "Method", name as essential for PDR; constants of the usual
// Gaussian-splatting form, see include/pdr.h):
//
//   L = (1 - lam) mean|I - T| + lam (1 - mean SSIM(I, T)),
//   SSIM per (frame, channel) image with an 11 x 11 Gaussian window (sigma
//   1.5), zero padding, C1 = (0.01 range)^2, C2 = (0.03 range)^2.
//
// Two tile kernels, one block per 32 x 32 tile of one (frame, channel)
// image, and a final reduction:
//   k_loss_coef  stages image and target with a 5-pixel apron, forms the five
//                window moments mu_x, mu_y, E xx, E yy, E xy on the tile by
//                separable sums (horizontal over the apron rows, then
//                vertical), the SSIM map S and the gradient coefficients
//                A = dS/dmu_x - 2 mu_x dS/ds_xx - mu_y dS/ds_xy,
//                B = dS/ds_xx,  Cxy = dS/ds_xy
//                (written to the workspace), and the tile's sums of |I - T|
//                and S;
//   k_loss_grad  stages A, B, Cxy with a 5-pixel apron (zero outside the
//                image) and forms dS_mean/dI = (G*A + 2 I (G*B) + T (G*Cxy)) / n
//                by separable sums, then dL/dI;
//   k_loss_final adds the per-block sums in block order (fp64) into L.
// Image and target are shifted by their values at the image centre: SSIM and
// its gradient are invariant under the shift (A is formed with the shifted
// means, the final combination with the shifted values: the shift cancels
// pixel pair by pixel pair), and it keeps the fp32 variances and the final
// combination free of large cancellations.  Taps come from the constant bank
// (a kernel argument); each separable pass is register-blocked (a thread
// produces RB neighbouring outputs from one streamed read of RB + 10
// inputs).  Fixed order throughout: bitwise reproducible.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "pdr.h"

namespace pdr {
namespace {

constexpr int kLT = 32;             // tile edge
constexpr int kLR = 5;              // window radius
constexpr int kLW = 2 * kLR + 1;    // window taps
constexpr int kLS = kLT + 2 * kLR;  // tile plus apron (42)
constexpr int kLossThreads = 256;
constexpr int kLU = (kLS * kLS + kLossThreads - 1) / kLossThreads;  // staged pixels per thread
constexpr int kRBH = 4;  // horizontal passes: 32 = 8 x 4 outputs per row
constexpr int kRBV = 2;  // vertical passes:   32 = 16 x 2 outputs per column

// The window taps travel as a kernel argument (constant bank).
struct Taps {
    float t[kLW];
};

struct CoefSmem {
    float x[kLS][kLS];      // shifted image over the tile and its apron, zero-padded
    float y[kLS][kLS];      // shifted target
    float h[5][kLS][kLT];   // horizontal window sums of x, y, xx, yy, xy
    float red[2][kLossThreads / 32];
};
struct GradSmem {
    float abc[3][kLS][kLS];  // A, B, Cxy over the tile and its apron
    float h[3][kLS][kLT];    // their horizontal window sums
};

struct LossTile {
    int im, X0, Y0;
    size_t base;
};
__device__ __forceinline__ LossTile loss_tile(int W, int H, int TX, int TY) {
    const int tiles = TX * TY;
    LossTile L;
    L.im = blockIdx.x / tiles;
    const int t = blockIdx.x - L.im * tiles;
    const int ty = t / TX;
    L.X0 = (t - ty * TX) * kLT;
    L.Y0 = ty * kLT;
    L.base = (size_t)L.im * H * W;
    return L;
}

__global__ void __launch_bounds__(kLossThreads) k_loss_coef(
    const float *__restrict__ img, const float *__restrict__ tgt, int H, int W, int TX, int TY,
    float C1, float C2, const Taps tp_, float *__restrict__ coef, size_t n,
    float *__restrict__ part) {
    extern __shared__ float4 lsm4[];
    CoefSmem &S = *reinterpret_cast<CoefSmem *>(lsm4);
    grid_dep_wait();
    const int tid = threadIdx.x;
    const LossTile T = loss_tile(W, H, TX, TY);
    const float *ip = img + T.base, *tp = tgt + T.base;
    const float *g = tp_.t;
    const size_t mid = (size_t)(H / 2) * W + W / 2;  // the image's shift
    const float sx = ip[mid], sy = tp[mid];

    // 1. stage [Y0 - 5, Y0 + 36] x [X0 - 5, X0 + 36]; |I - T| of the tile's pixels
    float lsum = 0.0f;
    {
        float xv[kLU], yv[kLU];
#pragma unroll
        for (int u = 0; u < kLU; ++u) {
            const int i = u * kLossThreads + tid;
            const int r = i / kLS, c = i - r * kLS;
            const int y = T.Y0 - kLR + r, x = T.X0 - kLR + c;
            const bool in = i < kLS * kLS && y >= 0 && y < H && x >= 0 && x < W;
            const size_t o = in ? (size_t)y * W + x : 0;
            xv[u] = in ? ip[o] : 0.0f;
            yv[u] = in ? tp[o] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kLU; ++u) {
            const int i = u * kLossThreads + tid;
            if (i >= kLS * kLS) continue;
            const int r = i / kLS, c = i - r * kLS;
            S.x[r][c] = xv[u] - sx;
            S.y[r][c] = yv[u] - sy;
            const int tr = r - kLR, tc = c - kLR;
            if (tr >= 0 && tr < kLT && tc >= 0 && tc < kLT && T.Y0 + tr < H && T.X0 + tc < W)
                lsum += fabsf(xv[u] - yv[u]);
        }
    }
    __syncthreads();

    // 2. horizontal sums of x, y, xx, yy, xy (all staged rows, the tile's columns)
    for (int it = tid; it < kLS * (kLT / kRBH); it += kLossThreads) {
        const int r = it / (kLT / kRBH), c0 = (it - r * (kLT / kRBH)) * kRBH;
        float m[5][kRBH];
#pragma unroll
        for (int j = 0; j < kRBH; ++j)
#pragma unroll
            for (int q = 0; q < 5; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRBH + kLW - 1; ++k) {
            const float a = S.x[r][c0 + k], b = S.y[r][c0 + k];
            const float aa = a * a, bb = b * b, ab = a * b;
#pragma unroll
            for (int j = 0; j < kRBH; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
                m[0][j] = fmaf(g[d], a, m[0][j]);
                m[1][j] = fmaf(g[d], b, m[1][j]);
                m[2][j] = fmaf(g[d], aa, m[2][j]);
                m[3][j] = fmaf(g[d], bb, m[3][j]);
                m[4][j] = fmaf(g[d], ab, m[4][j]);
            }
        }
#pragma unroll
        for (int q = 0; q < 5; ++q)
#pragma unroll
            for (int j = 0; j < kRBH; ++j) S.h[q][r][c0 + j] = m[q][j];
    }
    __syncthreads();

    // 3. vertical sums -> moments on the tile; SSIM and the coefficients
    float ssum = 0.0f;
    for (int it = tid; it < (kLT / kRBV) * kLT; it += kLossThreads) {
        const int rb = it / kLT, c = it - rb * kLT, r0 = rb * kRBV;
        float m[5][kRBV];
#pragma unroll
        for (int j = 0; j < kRBV; ++j)
#pragma unroll
            for (int q = 0; q < 5; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRBV + kLW - 1; ++k) {
            float v[5];
#pragma unroll
            for (int q = 0; q < 5; ++q) v[q] = S.h[q][r0 + k][c];
#pragma unroll
            for (int j = 0; j < kRBV; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
#pragma unroll
                for (int q = 0; q < 5; ++q) m[q][j] = fmaf(g[d], v[q], m[q][j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kRBV; ++j) {
            const int y = T.Y0 + r0 + j, x = T.X0 + c;
            if (y >= H || x >= W) continue;
            const float mx = m[0][j], my = m[1][j];  // shifted means
            const float vxx = fmaf(-mx, mx, m[2][j]), vyy = fmaf(-my, my, m[3][j]);
            const float vxy = fmaf(-mx, my, m[4][j]);
            const float ux = mx + sx, uy = my + sy;  // true means
            const float N1 = fmaf(2.0f * ux, uy, C1), N2 = fmaf(2.0f, vxy, C2);
            const float D1 = fmaf(ux, ux, fmaf(uy, uy, C1)), D2 = vxx + vyy + C2;
            const float rD1 = 1.0f / D1, rD2 = 1.0f / D2, rD = rD1 * rD2;
            const float sv = N1 * N2 * rD;
            const float dmu = 2.0f * uy * N2 * rD - 2.0f * ux * sv * rD1;
            const float Bc = -sv * rD2, Cc = 2.0f * N1 * rD;
            const size_t o = T.base + (size_t)y * W + x;
            coef[o] = dmu - 2.0f * mx * Bc - my * Cc;  // shifted means: the shift cancels
            coef[n + o] = Bc;
            coef[2 * n + o] = Cc;
            ssum += sv;
        }
    }

    // 4. block sums (fixed tree order)
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        lsum += __shfl_xor_sync(0xffffffffu, lsum, d);
        ssum += __shfl_xor_sync(0xffffffffu, ssum, d);
    }
    if (lane == 0) {
        S.red[0][warp] = lsum;
        S.red[1][warp] = ssum;
    }
    __syncthreads();
    if (tid == 0) {
        float l = 0.f, sm = 0.f;
        for (int w = 0; w < kLossThreads / 32; ++w) {
            l += S.red[0][w];
            sm += S.red[1][w];
        }
        part[2 * (size_t)blockIdx.x] = l;
        part[2 * (size_t)blockIdx.x + 1] = sm;
    }
}

__global__ void __launch_bounds__(kLossThreads) k_loss_grad(
    const float *__restrict__ img, const float *__restrict__ tgt, int H, int W, int TX, int TY,
    float lam, double inv_n, const Taps tp_, const float *__restrict__ coef, size_t n,
    float *__restrict__ grad) {
    extern __shared__ float4 lsm4[];
    GradSmem &S = *reinterpret_cast<GradSmem *>(lsm4);
    grid_dep_wait();
    const int tid = threadIdx.x;
    const LossTile T = loss_tile(W, H, TX, TY);
    const float *ip = img + T.base, *tp = tgt + T.base;
    const float *g = tp_.t;
    const size_t mid = (size_t)(H / 2) * W + W / 2;
    const float sx = ip[mid], sy = tp[mid];

    // 1. stage A, B, Cxy over [Y0 - 5, Y0 + 36] x [X0 - 5, X0 + 36], zero outside the image
    {
        float av[3][kLU];
#pragma unroll
        for (int u = 0; u < kLU; ++u) {
            const int i = u * kLossThreads + tid;
            const int r = i / kLS, c = i - r * kLS;
            const int y = T.Y0 - kLR + r, x = T.X0 - kLR + c;
            const bool in = i < kLS * kLS && y >= 0 && y < H && x >= 0 && x < W;
            const size_t o = in ? T.base + (size_t)y * W + x : 0;
#pragma unroll
            for (int q = 0; q < 3; ++q) av[q][u] = in ? coef[q * n + o] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kLU; ++u) {
            const int i = u * kLossThreads + tid;
            if (i >= kLS * kLS) continue;
            const int r = i / kLS, c = i - r * kLS;
#pragma unroll
            for (int q = 0; q < 3; ++q) S.abc[q][r][c] = av[q][u];
        }
    }
    __syncthreads();

    // 2. horizontal sums of A, B, Cxy
    for (int it = tid; it < kLS * (kLT / kRBH); it += kLossThreads) {
        const int r = it / (kLT / kRBH), c0 = (it - r * (kLT / kRBH)) * kRBH;
        float m[3][kRBH];
#pragma unroll
        for (int j = 0; j < kRBH; ++j)
#pragma unroll
            for (int q = 0; q < 3; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRBH + kLW - 1; ++k) {
            float v[3];
#pragma unroll
            for (int q = 0; q < 3; ++q) v[q] = S.abc[q][r][c0 + k];
#pragma unroll
            for (int j = 0; j < kRBH; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
#pragma unroll
                for (int q = 0; q < 3; ++q) m[q][j] = fmaf(g[d], v[q], m[q][j]);
            }
        }
#pragma unroll
        for (int q = 0; q < 3; ++q)
#pragma unroll
            for (int j = 0; j < kRBH; ++j) S.h[q][r][c0 + j] = m[q][j];
    }
    __syncthreads();

    // 3. vertical sums -> dL/dI on the tile
    const float wl1 = (float)((1.0 - (double)lam) * inv_n), wss = (float)((double)lam * inv_n);
    for (int it = tid; it < (kLT / kRBV) * kLT; it += kLossThreads) {
        const int rb = it / kLT, c = it - rb * kLT, r0 = rb * kRBV;
        float m[3][kRBV];
#pragma unroll
        for (int j = 0; j < kRBV; ++j)
#pragma unroll
            for (int q = 0; q < 3; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRBV + kLW - 1; ++k) {
            float v[3];
#pragma unroll
            for (int q = 0; q < 3; ++q) v[q] = S.h[q][r0 + k][c];
#pragma unroll
            for (int j = 0; j < kRBV; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
#pragma unroll
                for (int q = 0; q < 3; ++q) m[q][j] = fmaf(g[d], v[q], m[q][j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kRBV; ++j) {
            const int y = T.Y0 + r0 + j, x = T.X0 + c;
            if (y >= H || x >= W) continue;
            const size_t o = (size_t)y * W + x;
            const float xv = ip[o], yv = tp[o];
            const float dss = fmaf(2.0f * (xv - sx), m[1][j], fmaf(yv - sy, m[2][j], m[0][j]));
            const float diff = xv - yv;  // unshifted: ties stay exact zeros
            const float sg = diff > 0.0f ? 1.0f : (diff < 0.0f ? -1.0f : 0.0f);
            grad[T.base + o] = fmaf(wl1, sg, -wss * dss);
        }
    }
}

// loss = (1 - lam) sum|I - T| / n + lam (1 - sum S / n), partials added in
// block order in fp64 (each thread a contiguous range, then the threads in order).
__global__ void __launch_bounds__(256) k_loss_final(const float *__restrict__ part, int nblocks,
                                                    float lam, double inv_n,
                                                    float *__restrict__ loss) {
    __shared__ double sl[256], ss[256];
    grid_dep_wait();
    grid_dep_release();
    const int tid = threadIdx.x;
    const int per = (nblocks + 255) / 256;
    double l = 0.0, s = 0.0;
    for (int j = tid * per; j < min(nblocks, (tid + 1) * per); ++j) {
        l += part[2 * (size_t)j];
        s += part[2 * (size_t)j + 1];
    }
    sl[tid] = l;
    ss[tid] = s;
    __syncthreads();
    if (tid == 0) {
        double L = 0.0, Sm = 0.0;
        for (int j = 0; j < 256; ++j) {
            L += sl[j];
            Sm += ss[j];
        }
        *loss = (float)((1.0 - (double)lam) * L * inv_n + (double)lam * (1.0 - Sm * inv_n));
    }
}

bool loss_geometry(int B, int C, int H, int W, int *TX, int *TY, long long *nblocks) {
    if (B < 1 || C < 1 || H < 1 || W < 1) return false;
    *TX = (W + kLT - 1) / kLT;
    *TY = (H + kLT - 1) / kLT;
    *nblocks = (long long)B * C * (*TX) * (*TY);
    return *nblocks <= INT32_MAX && (long long)B * C * H * W <= (1ll << 40);
}

}  // namespace
}  // namespace pdr

using namespace pdr;

extern "C" {

size_t pdr_loss_workspace_bytes(int B, int C, int H, int W) {
    int TX, TY;
    long long nb;
    if (!loss_geometry(B, C, H, W, &TX, &TY, &nb)) return 0;
    const size_t part = ((2 * sizeof(float) * (size_t)nb) + 255) & ~(size_t)255;
    const size_t coef = 3 * sizeof(float) * (size_t)B * C * H * W;  // A, B, Cxy maps
    return part + ((coef + 255) & ~(size_t)255);
}

pdr_status pdr_loss_l1_ssim(const float *image, const float *target, int B, int C, int H,
                            int W, float lam, float data_range, float *loss, float *grad_image,
                            void *workspace, size_t workspace_bytes, void *stream) {
    int TX, TY;
    long long nb;
    if (!loss_geometry(B, C, H, W, &TX, &TY, &nb)) return PDR_ERR_INVALID_ARG;
    if (!(lam >= 0.0f && lam <= 1.0f) || !(data_range > 0.0f) || !isfinite(data_range))
        return PDR_ERR_INVALID_ARG;
    if (!image || !target || !loss || !grad_image || !workspace) return PDR_ERR_INVALID_ARG;
    if (((uintptr_t)image | (uintptr_t)target | (uintptr_t)loss | (uintptr_t)grad_image) & 3)
        return PDR_ERR_INVALID_ARG;
    if ((uintptr_t)workspace & 255) return PDR_ERR_INVALID_ARG;
    if (workspace_bytes < pdr_loss_workspace_bytes(B, C, H, W)) return PDR_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sc = sizeof(CoefSmem), sg = sizeof(GradSmem);
    if (cudaFuncSetAttribute(k_loss_coef, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k_loss_grad, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg) !=
            cudaSuccess)
        return PDR_ERR_CUDA;
    const size_t n = (size_t)B * C * H * W;
    const float C1 = (0.01f * data_range) * (0.01f * data_range);
    const float C2 = (0.03f * data_range) * (0.03f * data_range);
    float *part = static_cast<float *>(workspace);
    float *coef = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                            (((2 * sizeof(float) * (size_t)nb) + 255) & ~(size_t)255));
    // Window taps exp(-d^2 / (2 sigma^2)), sigma 1.5, normalised to sum 1.
    Taps taps;
    {
        double v[kLW], sum = 0.0;
        for (int d = 0; d < kLW; ++d) {
            const double o = d - kLR;
            v[d] = exp(-(o * o) / (2.0 * 1.5 * 1.5));
            sum += v[d];
        }
        for (int d = 0; d < kLW; ++d) taps.t[d] = (float)(v[d] / sum);
    }
    const double inv_n = 1.0 / (double)n;
    // Programmatic dependent launches: each kernel waits for its predecessor
    // at its top (k_loss_final needs k_loss_coef's partial sums, complete
    // once k_loss_grad, which waited for them, is).  k_loss_coef and
    // k_loss_grad do not release their successors early (measured on B200:
    // with early release the stress512-sized loss took 166 us against 152).
    if (launch_dependent(k_loss_coef, dim3((unsigned)nb), dim3(kLossThreads), sc, s,
                         (const float *)image, (const float *)target, H, W, TX, TY, C1, C2, taps,
                         coef, n, part) != cudaSuccess)
        return PDR_ERR_CUDA;
    if (launch_dependent(k_loss_grad, dim3((unsigned)nb), dim3(kLossThreads), sg, s,
                         (const float *)image, (const float *)target, H, W, TX, TY, lam, inv_n,
                         taps, (const float *)coef, n, grad_image) != cudaSuccess)
        return PDR_ERR_CUDA;
    if (launch_dependent(k_loss_final, dim3(1), dim3(256), 0, s, (const float *)part, (int)nb, lam,
                         inv_n, loss) != cudaSuccess)
        return PDR_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? PDR_OK : PDR_ERR_CUDA;
}

}  // extern "C"
