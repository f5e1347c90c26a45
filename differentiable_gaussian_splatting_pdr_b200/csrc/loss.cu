// L1 + SSIM training loss and its gradient dL/dI (the objective the reading
// notes, section "Method", name as essential for PDR; constants of the usual
// Gaussian-splatting form, see include/pdr.h):
//
//   L = (1 - lam) mean|I - T| + lam (1 - mean SSIM(I, T)),
//   SSIM per (frame, channel) image with an 11 x 11 Gaussian window (sigma
//   1.5), zero padding, C1 = (0.01 range)^2, C2 = (0.03 range)^2.
//
// k_loss_tile: one block per 32 x 32 output tile of one image.  The image and
// the target are staged with a 10-pixel apron, shifted by a per-block
// constant (the value at the tile centre): SSIM and its gradient are
// invariant under that shift, and it keeps the fp32 variances and the final
// gradient combination free of large cancellations.  Five separable window
// sums (horizontal then vertical) give the moments mu_x, mu_y, E xx, E yy,
// E xy on the tile plus a 5-pixel apron; there the SSIM map S and the
// gradient coefficients
//   A = dS/dmu_x - 2 mu_x dS/ds_xx - mu_y dS/ds_xy,  B = dS/ds_xx,  Cxy = dS/ds_xy
// are formed (zero outside the image), and three more separable window sums
// give dS_mean/dI = (G*A + 2 I (G*B) + T (G*Cxy)) / n on the tile.  Each block
// leaves its partial sums of |I - T| and S in the workspace; k_loss_final
// adds them in block order (fp64) into the loss.  Fixed order throughout:
// bitwise reproducible.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "pdr.h"

namespace pdr {
namespace {

constexpr int kLT = 32;             // output tile edge
constexpr int kLR = 5;              // window radius
constexpr int kLW = 2 * kLR + 1;    // window taps
constexpr int kLS = kLT + 2 * kLR;  // moment region edge (42)
constexpr int kLI = kLT + 4 * kLR;  // staged input edge (52)
constexpr int kLossThreads = 512;
constexpr int kLU = (kLI * kLI + kLossThreads - 1) / kLossThreads;  // staged pixels per thread

struct LossSmem {
    float x[kLI][kLI];            // shifted image, zero-padded
    float y[kLI][kLI];            // shifted target
    float h[5][kLI][kLS];         // horizontal window sums (reused for the gradient pass)
    float abc[3][kLS][kLS];       // A, B, Cxy on the tile and its apron
    signed char sgn[kLT][kLT];    // sign(I - T) on the tile
    float red[2][kLossThreads / 32];
};

// The window taps travel as a kernel argument (constant bank): every FMA
// reads its tap without a shared-memory load.
struct Taps {
    float t[kLW];
};

// Register-blocked passes: a thread produces RB neighbouring outputs of a
// window sum from one streamed read of the RB + 10 inputs they share.
constexpr int kRB2 = 6;  // horizontal moments: 42 = 7 x 6 outputs per row
constexpr int kRB3 = 3;  // vertical moments:   42 = 14 x 3 outputs per column
constexpr int kRB4 = 4;  // horizontal coefficients: 32 = 8 x 4
constexpr int kRB5 = 2;  // vertical coefficients:   32 = 16 x 2

__global__ void __launch_bounds__(kLossThreads) k_loss_tile(
    const float *__restrict__ img, const float *__restrict__ tgt, int BC, int H, int W, int TX,
    int TY, float lam, float C1, float C2, double inv_n, const Taps tp_,
    float *__restrict__ grad, float *__restrict__ part) {
    extern __shared__ float4 lsm4[];
    LossSmem &S = *reinterpret_cast<LossSmem *>(lsm4);
    const int tid = threadIdx.x;
    const int tiles = TX * TY;
    const int im = blockIdx.x / tiles, t = blockIdx.x - im * tiles;
    const int ty = t / TX, tx = t - ty * TX;
    const int X0 = tx * kLT, Y0 = ty * kLT;
    const size_t base = (size_t)im * H * W;
    const float *ip = img + base, *tp = tgt + base;
    const float *g = tp_.t;

    // Shift: the values at the tile centre (clamped into the image).
    const int cyy = min(Y0 + kLT / 2, H - 1), cxx = min(X0 + kLT / 2, W - 1);
    const float sx = ip[(size_t)cyy * W + cxx], sy = tp[(size_t)cyy * W + cxx];

    // 1. stage the shifted inputs over [Y0 - 10, Y0 + 41] x [X0 - 10, X0 + 41]
    //    (all of a thread's loads in flight together); the L1 term of the
    //    tile's own pixels is taken from the unshifted values here.
    float lsum = 0.0f;
    {
        float xv[kLU], yv[kLU];
#pragma unroll
        for (int u = 0; u < kLU; ++u) {
            const int i = u * kLossThreads + tid;
            const int r = i / kLI, c = i - r * kLI;
            const int y = Y0 - 2 * kLR + r, x = X0 - 2 * kLR + c;
            const bool in = i < kLI * kLI && y >= 0 && y < H && x >= 0 && x < W;
            const size_t o = in ? (size_t)y * W + x : 0;
            xv[u] = in ? ip[o] : 0.0f;
            yv[u] = in ? tp[o] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kLU; ++u) {
            const int i = u * kLossThreads + tid;
            if (i >= kLI * kLI) continue;
            const int r = i / kLI, c = i - r * kLI;
            S.x[r][c] = xv[u] - sx;
            S.y[r][c] = yv[u] - sy;
            const int tr = r - 2 * kLR, tc = c - 2 * kLR;
            if (tr >= 0 && tr < kLT && tc >= 0 && tc < kLT) {
                const float diff = xv[u] - yv[u];  // unshifted: ties stay exact zeros
                S.sgn[tr][tc] = diff > 0.0f ? 1 : (diff < 0.0f ? -1 : 0);
                if (Y0 + tr < H && X0 + tc < W) lsum += fabsf(diff);
            }
        }
    }
    __syncthreads();

    // 2. horizontal window sums of x, y, xx, yy, xy over all staged rows
    for (int it = tid; it < kLI * (kLS / kRB2); it += kLossThreads) {
        const int r = it / (kLS / kRB2), c0 = (it - r * (kLS / kRB2)) * kRB2;
        float m[5][kRB2];
#pragma unroll
        for (int j = 0; j < kRB2; ++j)
#pragma unroll
            for (int q = 0; q < 5; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRB2 + kLW - 1; ++k) {
            const float a = S.x[r][c0 + k], b = S.y[r][c0 + k];
            const float aa = a * a, bb = b * b, ab = a * b;
#pragma unroll
            for (int j = 0; j < kRB2; ++j) {
                const int d = k - j;  // tap of output c0 + j
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
            for (int j = 0; j < kRB2; ++j) S.h[q][r][c0 + j] = m[q][j];
    }
    __syncthreads();

    // 3. vertical sums -> moments; SSIM map and gradient coefficients
    float ssum = 0.0f;
    for (int it = tid; it < (kLS / kRB3) * kLS; it += kLossThreads) {
        const int rb = it / kLS, c = it - rb * kLS, r0 = rb * kRB3;
        float m[5][kRB3];
#pragma unroll
        for (int j = 0; j < kRB3; ++j)
#pragma unroll
            for (int q = 0; q < 5; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRB3 + kLW - 1; ++k) {
            float v[5];
#pragma unroll
            for (int q = 0; q < 5; ++q) v[q] = S.h[q][r0 + k][c];
#pragma unroll
            for (int j = 0; j < kRB3; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
#pragma unroll
                for (int q = 0; q < 5; ++q) m[q][j] = fmaf(g[d], v[q], m[q][j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kRB3; ++j) {
            const int r = r0 + j;
            const int y = Y0 - kLR + r, x = X0 - kLR + c;
            float A = 0.f, Bc = 0.f, Cc = 0.f;
            if (y >= 0 && y < H && x >= 0 && x < W) {
                const float mx = m[0][j], my = m[1][j];  // shifted means
                const float vxx = fmaf(-mx, mx, m[2][j]), vyy = fmaf(-my, my, m[3][j]);
                const float vxy = fmaf(-mx, my, m[4][j]);
                const float ux = mx + sx, uy = my + sy;  // true means
                const float N1 = fmaf(2.0f * ux, uy, C1), N2 = fmaf(2.0f, vxy, C2);
                const float D1 = fmaf(ux, ux, fmaf(uy, uy, C1)), D2 = vxx + vyy + C2;
                const float rD1 = 1.0f / D1, rD2 = 1.0f / D2, rD = rD1 * rD2;
                const float s = N1 * N2 * rD;
                const float dmu = 2.0f * uy * N2 * rD - 2.0f * ux * s * rD1;
                Bc = -s * rD2;
                Cc = 2.0f * N1 * rD;
                A = dmu - 2.0f * mx * Bc - my * Cc;  // shifted means: the shift cancels exactly
                if (r >= kLR && r < kLR + kLT && c >= kLR && c < kLR + kLT) ssum += s;
            }
            S.abc[0][r][c] = A;
            S.abc[1][r][c] = Bc;
            S.abc[2][r][c] = Cc;
        }
    }
    __syncthreads();

    // 4. horizontal window sums of A, B, Cxy over the moment rows
    for (int it = tid; it < kLS * (kLT / kRB4); it += kLossThreads) {
        const int r = it / (kLT / kRB4), c0 = (it - r * (kLT / kRB4)) * kRB4;
        float m[3][kRB4];
#pragma unroll
        for (int j = 0; j < kRB4; ++j)
#pragma unroll
            for (int q = 0; q < 3; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRB4 + kLW - 1; ++k) {
            float v[3];
#pragma unroll
            for (int q = 0; q < 3; ++q) v[q] = S.abc[q][r][c0 + k];
#pragma unroll
            for (int j = 0; j < kRB4; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
#pragma unroll
                for (int q = 0; q < 3; ++q) m[q][j] = fmaf(g[d], v[q], m[q][j]);
            }
        }
#pragma unroll
        for (int q = 0; q < 3; ++q)
#pragma unroll
            for (int j = 0; j < kRB4; ++j) S.h[q][r][c0 + j] = m[q][j];
    }
    __syncthreads();

    // 5. vertical sums -> dL/dI on the tile
    const float wl1 = (float)((1.0 - (double)lam) * inv_n), wss = (float)((double)lam * inv_n);
    for (int it = tid; it < (kLT / kRB5) * kLT; it += kLossThreads) {
        const int rb = it / kLT, c = it - rb * kLT, r0 = rb * kRB5;
        float m[3][kRB5];
#pragma unroll
        for (int j = 0; j < kRB5; ++j)
#pragma unroll
            for (int q = 0; q < 3; ++q) m[q][j] = 0.0f;
#pragma unroll
        for (int k = 0; k < kRB5 + kLW - 1; ++k) {
            float v[3];
#pragma unroll
            for (int q = 0; q < 3; ++q) v[q] = S.h[q][r0 + k][c];
#pragma unroll
            for (int j = 0; j < kRB5; ++j) {
                const int d = k - j;
                if (d < 0 || d >= kLW) continue;
#pragma unroll
                for (int q = 0; q < 3; ++q) m[q][j] = fmaf(g[d], v[q], m[q][j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kRB5; ++j) {
            const int r = r0 + j;
            const int y = Y0 + r, x = X0 + c;
            if (y >= H || x >= W) continue;
            const float xs = S.x[r + 2 * kLR][c + 2 * kLR], ys = S.y[r + 2 * kLR][c + 2 * kLR];
            const float dss = fmaf(2.0f * xs, m[1][j], fmaf(ys, m[2][j], m[0][j]));  // n * dS_mean/dI
            grad[base + (size_t)y * W + x] = fmaf(wl1, (float)S.sgn[r][c], -wss * dss);
        }
    }

    // 6. block partial sums (fixed tree order)
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
        float l = 0.f, s = 0.f;
        for (int w = 0; w < kLossThreads / 32; ++w) {
            l += S.red[0][w];
            s += S.red[1][w];
        }
        part[2 * (size_t)blockIdx.x] = l;
        part[2 * (size_t)blockIdx.x + 1] = s;
    }
}

// loss = (1 - lam) sum|I - T| / n + lam (1 - sum S / n), partials added in
// block order in fp64 (each thread a contiguous range, then the threads in order).
__global__ void __launch_bounds__(256) k_loss_final(const float *__restrict__ part, int nblocks,
                                                    float lam, double inv_n,
                                                    float *__restrict__ loss) {
    __shared__ double sl[256], ss[256];
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
    return (size_t)(((2 * sizeof(float) * (size_t)nb) + 255) & ~(size_t)255);
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
    const size_t smem = sizeof(LossSmem);
    if (cudaFuncSetAttribute(k_loss_tile, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return PDR_ERR_CUDA;
    const double n = (double)B * C * H * W;
    const float C1 = (0.01f * data_range) * (0.01f * data_range);
    const float C2 = (0.03f * data_range) * (0.03f * data_range);
    float *part = static_cast<float *>(workspace);
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
    k_loss_tile<<<(unsigned)nb, kLossThreads, smem, s>>>(image, target, B * C, H, W, TX, TY, lam,
                                                         C1, C2, 1.0 / n, taps, grad_image, part);
    if (cudaGetLastError() != cudaSuccess) return PDR_ERR_CUDA;
    k_loss_final<<<1, 256, 0, s>>>(part, (int)nb, lam, 1.0 / n, loss);
    return cudaGetLastError() == cudaSuccess ? PDR_OK : PDR_ERR_CUDA;
}

}  // extern "C"
