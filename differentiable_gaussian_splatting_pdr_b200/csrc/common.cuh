// Shared definitions of the sm_100a renderer kernels (tile binner, forward
// tile kernel, backward home-tile kernel).  Host API in api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pdr {

constexpr int kTile = 16;
// Window centre used for Gaussians whose mean is not finite: far outside any
// grid the library accepts, so their window never touches a pixel or a tile.
constexpr int kNoCenter = 0x40000000;
// Bits of the device error word (workspace), set by the kernels' own checks.
constexpr int kErrListBounds = 1;  // a tile list or list slot outside its frame's region
constexpr int kErrBadId = 2;       // a list entry that is not a Gaussian of the frame

// sqrt(kappa) with kappa = log2(e) / 2: scaling u by sqrt(kappa e^{-2 s})
// turns exp(-q / 2) into 2^{-(u1^2 + u2^2)}.
constexpr float kSqrtKappa = 0.849321800288019f;
// 1 / kappa = 2 ln 2: the factor between the moment sums and the gradients.
constexpr float kTwoLn2 = 1.38629436111989061883f;

struct Geom {
    int B, N, C, H, W, k, r;
    int TX, TY, T;      // tiles per row, per column, per frame
    int P;              // parameters per Gaussian (5 + C)
    int m;              // most tiles a window can touch along one axis
    int cap;            // tile-list capacity per frame (N * m * m)
    int chunk, nchunks; // Gaussians per binning chunk, chunks per frame
    int scatter_warps;  // warps per scatter block
    int out_vec2;       // 1 if the output image allows 8-byte pixel-pair stores
};

// Per-Gaussian record written by the binner and read by both render kernels
// (two float4 per Gaussian, 32 bytes):
//   [0] = (mu_x, mu_y, alpha_1, beta_1)
//   [1] = (alpha_2, beta_2, cx (int bits), cy (int bits))
// with  uhat_j = alpha_j (x - mu_x) + beta_j (y - mu_y) the rotated, scaled
// coordinates (uhat = sqrt(kappa) diag(e^{-s}) R^T (p - mu)), so that the
// weight is w = 2^{-(uhat_1^2 + uhat_2^2)} = exp(-q / 2).
struct Workspace {
    int *err;       // device error word
    float4 *gr;     // [B*N][2]
    int *hist;      // [B][nchunks][T]: chunk counts, then absolute list bases
    int *offs;      // [B][T + 1]: absolute list start of every tile, frame end
    int *ids;       // [B][cap]: frame-local Gaussian ids, tile-major
};

// Start and end of the list of tile t of frame b, checked against the frame's
// region; an inconsistent pair flags the error word and yields an empty list.
__device__ __forceinline__ void list_range(const int *offs, const Geom &g, int b, int t,
                                           int *err, int &L0, int &L1) {
    L0 = offs[(size_t)b * (g.T + 1) + t];
    L1 = offs[(size_t)b * (g.T + 1) + t + 1];
    const long long lo = (long long)b * g.cap, hi = lo + g.cap;
    if (L0 < lo || L1 > hi || L0 > L1) {
        atomicOr(err, kErrListBounds);
        L0 = L1 = 0;
    }
}

// round(mu) with ties up, exact: mu - floor(mu) is exact in fp32, whereas
// floor(mu + 0.5f) is not (0.49999997f + 0.5f rounds to 1).
__device__ __forceinline__ int round_half_up(float mu) {
    mu = fminf(fmaxf(mu, -16777216.0f), 16777216.0f);
    float c = floorf(mu);
    if (mu - c >= 0.5f) c += 1.0f;
    return (int)c;
}

// 2^x on the MUFU unit (flush-to-zero for results below the normal range).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Launchers (each returns the launch error, cudaSuccess otherwise).
cudaError_t launch_bin(const float *params, const Geom &g, const Workspace &ws,
                       cudaStream_t s);
cudaError_t launch_fwd(const float *params, const Geom &g, const Workspace &ws,
                       float *image, cudaStream_t s);
cudaError_t launch_bwd(const float *params, const float *grad_image, const Geom &g,
                       const Workspace &ws, float *grad_params, cudaStream_t s);

// Dynamic shared memory needed by the kernels for these sizes.
size_t bin_count_smem(const Geom &g);
size_t bin_scatter_smem(const Geom &g);
size_t bwd_smem(const Geom &g);

}  // namespace pdr
