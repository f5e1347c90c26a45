// Shared definitions of the sm_100a renderer kernels (tile binner, forward
// tile kernel, backward home-tile kernel).  Host API in api.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
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
constexpr int kErrSmemLayout = 4;  // a kernel got less dynamic shared memory than it lays out

// A tile-list entry is a frame-local Gaussian id; the binner sets kHomeFlag on
// the one entry of each Gaussian that sits in the list of its home tile (the
// tile of its clamped window centre), so that the backward pass finds its
// Gaussians from the ids alone.
constexpr unsigned kHomeFlag = 0x80000000u;
__device__ __forceinline__ int entry_id(int raw) { return raw & 0x7fffffff; }
__device__ __forceinline__ bool entry_home(int raw) { return raw < 0; }

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
    int slab;           // Gaussians per binning slab (32, 64, 128 or a multiple of 256)
    int nslab;          // binning slabs per frame
    int slab_warps;     // warps (slabs) per block of the slab scatter
    int frame_block;    // 1: small frames, one binning block per frame
    int frame_threads;  // threads of that block
    int cluster_fwd;    // 1: frames of <= kClusterTiles tiles, bins + forward in one launch
    int fwd_pl;         // forward pixels per lane (2 or 4)
    int out_vec2;       // 1 if the output image allows 2-pixel vector stores
    int out_vec4;       // 1 if the output image allows 4-pixel vector stores
    int img_dtype;      // storage of image / dL/dI: PDR_F32, PDR_F16 or PDR_BF16
    int stage_vec4;     // 1: dL/dI rows of a multiple of 4 elements, image aligned to 4 elements
    int bwd_threads;    // threads per backward block
    int bwd_rcap;       // home records a backward block stages at most (>= its threads)
};

constexpr int kFrameBlockMaxT = 256;   // small frames: at most this many tiles
constexpr int kFrameBlockMaxN = 16384; // and at most this many Gaussians
constexpr int kClusterTiles = 16;            // frames up to this many tiles: one cluster per frame
constexpr int kClusterMaxBlocks = 4 * 148;   // ... while the launch has at most this many blocks

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
    int *hist;      // [B][nslab][T]: slab counts, then exclusive prefix over slabs
    int *tot;       // [B][T]: entries per tile
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

// The per-Gaussian record (layout above) from its parameters.  One function
// for the binner and for the render kernels that find their Gaussians
// themselves, so both paths produce the same bits.
__device__ __forceinline__ void gaussian_record(const float *__restrict__ p, float4 &A,
                                                float4 &Q) {
    const float mx = p[0], my = p[1], s1 = p[2], s2 = p[3], th = p[4];
    int cx = kNoCenter, cy = kNoCenter;
    if (isfinite(mx) && isfinite(my)) {
        cx = round_half_up(mx);
        cy = round_half_up(my);
    }
    float sn, cs;
    sincosf(th, &sn, &cs);
    const float h1 = kSqrtKappa * expf(-s1), h2 = kSqrtKappa * expf(-s2);
    A = make_float4(mx, my, h1 * cs, h1 * sn);
    Q = make_float4(-h2 * sn, h2 * cs, __int_as_float(cx), __int_as_float(cy));
}

// Window centre of a Gaussian from its mean alone (as in gaussian_record).
__device__ __forceinline__ void window_centre(const float *__restrict__ p, int &cx, int &cy) {
    const float mx = p[0], my = p[1];
    cx = kNoCenter;
    cy = kNoCenter;
    if (isfinite(mx) && isfinite(my)) {
        cx = round_half_up(mx);
        cy = round_half_up(my);
    }
}

// The window clipped to the grid; false if it misses the grid.
__device__ __forceinline__ bool window_rect(int cx, int cy, const Geom &g, int &x0, int &x1,
                                            int &y0, int &y1) {
    x0 = max(cx - g.r, 0);
    x1 = min(cx + g.r, g.W - 1);
    y0 = max(cy - g.r, 0);
    y1 = min(cy + g.r, g.H - 1);
    return x0 <= x1 && y0 <= y1;
}

// Tile that owns a Gaussian in the backward pass: the tile of its window
// centre clamped to the grid (always one of the tiles its window touches).
__device__ __forceinline__ int home_tile(int cx, int cy, const Geom &g) {
    const int hx = min(max(cx, 0), g.W - 1) >> 4;
    const int hy = min(max(cy, 0), g.H - 1) >> 4;
    return hy * g.TX + hx;
}

// One element of an image stored as fp32, fp16 or bf16 (dtype uniform per
// launch), read or written as fp32.
__device__ __forceinline__ float img_load(const void *p, size_t i, int dtype) {
    if (dtype == 1) return __half2float(static_cast<const __half *>(p)[i]);
    if (dtype == 2) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    return static_cast<const float *>(p)[i];
}
// v rounded to nearest to fp16 (dtype 1) or bf16 (dtype 2), as raw bits.
__device__ __forceinline__ unsigned short half_bits(float v, int dtype) {
    return dtype == 1 ? __half_as_ushort(__float2half_rn(v))
                      : __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ void img_store(void *p, size_t i, int dtype, float v) {
    if (dtype == 1)
        static_cast<__half *>(p)[i] = __float2half_rn(v);
    else if (dtype == 2)
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
    else
        static_cast<float *>(p)[i] = v;
}

// 2^x on the MUFU unit (flush-to-zero for results below the normal range).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Programmatic dependent launch (sm_90 and later).  grid_dep_wait() returns
// once every grid this one depends on has completed and its writes are
// visible (at once for a grid launched without the attribute); every kernel
// calls it before its first access to global memory, so a kernel is correct
// whatever precedes it in the stream.  grid_dep_release() lets the next grid
// of the stream be scheduled as this one's blocks retire; the three slab
// binning kernels do not call it (measured on B200: with it, the next slab
// kernel's blocks resident early slowed a 1024-tile frame's binning from 39 to
// 58 us), so their successors start when they exit.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_release() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches kernel k on stream s as a programmatic dependent launch: its blocks
// may be scheduled while the previous kernel of the stream finishes, and wait
// in grid_dep_wait() for it.
template <typename... P, typename... A>
cudaError_t launch_dependent(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             A... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, args...);
}

__device__ __forceinline__ unsigned dynamic_smem_bytes() {
    unsigned n;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(n));
    return n;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive prefix over the block of one int per thread (any blockDim that is
// a multiple of 32, at most 1024); `total` gets the block sum.  warp_tot needs
// blockDim / 32 ints of shared memory.  Called by the whole block.
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    total = 0;
    for (int w = 0; w < nw; ++w) {
        const int c = warp_tot[w];
        before += w < warp ? c : 0;
        total += c;
    }
    __syncthreads();
    return before + incl - v;
}

// Launchers (each returns the launch error, cudaSuccess otherwise).
cudaError_t launch_bin(const float *params, const Geom &g, const Workspace &ws,
                       cudaStream_t s);
// bin_inside: bin and render in one launch (g.cluster_fwd frames only).
cudaError_t launch_fwd(const float *params, const Geom &g, const Workspace &ws,
                       void *image, cudaStream_t s, bool bin_inside);
cudaError_t launch_bwd(const float *params, const void *grad_image, const Geom &g,
                       const Workspace &ws, float *grad_params, cudaStream_t s);

// The fused bins + render launch (k_fwd_cluster) for these sizes can be
// scheduled on the current device (at least one cluster fits); cached.
bool fwd_cluster_schedulable(const Geom &g);
// dst[i] = frame-local id of tile-list entry src[i] (home flag cleared).
cudaError_t launch_copy_ids(int *dst, const int *src, size_t n, cudaStream_t s);

// Dynamic shared memory needed by the kernels for these sizes.
size_t bin_frame_smem(const Geom &g);
size_t bin_count_smem(const Geom &g);
size_t bin_scatter_smem(const Geom &g);
size_t bwd_smem(const Geom &g);
// The backward kernel for these sizes: the pixel-pair kernel (C <= 4, k 13 or
// 15) or the scalar one.
bool bwd_uses_pairs(int C, int k);

}  // namespace pdr
