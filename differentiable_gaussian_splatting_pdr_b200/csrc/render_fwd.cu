// Forward tile kernel: I_c(p) = sum_i a_ic * 2^{-(uhat_1^2 + uhat_2^2)} over
// the Gaussians whose k x k window contains p (paper abstract: 5 + C
// parameters, arbitrary C; reading notes, "Method": additive accumulation).
//
// One 128-thread block per (frame, 16x16 tile).  The tile is cut into sixteen
// 4x4 regions, one per group of 8 lanes; each lane owns a horizontal pixel
// pair and keeps all C channels of both pixels in registers.  Per batch of
// the tile's list (ascending Gaussian id):
//   1. stage: each entry's record is gathered from the per-Gaussian records
//      and rebased to the tile origin (uhat_j = alpha_j x + beta_j y + K_j in
//      tile-local pixels), with the window as a 16-bit column mask and a
//      16-bit row mask;
//   2. sub-lists: each warp compacts, in list order, the entries whose window
//      meets each of its four regions, together with the 16-bit mask of the
//      region's pixels inside the window (ballot + popcount);
//   3. evaluate: every group walks only its own sub-list, so lanes spend
//      their issue slots on pixels that can be inside a window.
// The per-pixel sum order is the list order: fixed, so results are bitwise
// reproducible.  Stores are float2 (pixel pairs), coalesced along rows.
#include "common.cuh"

namespace pdr {

namespace {

constexpr int kFwdThreads = 128;
constexpr int kFwdBatch = 128;  // list entries staged per batch

template <int C>
struct FwdRec {
    static constexpr int kFloats = 6 + C;
    static constexpr int kVec = (kFloats + 3) / 4;  // float4 per record
};

template <int C>
__global__ void __launch_bounds__(kFwdThreads) k_fwd(const float *__restrict__ params,
                                                     Geom g,
                                                     const float4 *__restrict__ gr,
                                                     const int *__restrict__ offs,
                                                     const int *__restrict__ ids,
                                                     float *__restrict__ image,
                                                     int *__restrict__ err) {
    constexpr int RV = FwdRec<C>::kVec;
    __shared__ float4 rec[kFwdBatch * RV];
    __shared__ unsigned win[kFwdBatch];
    __shared__ unsigned sub[16][kFwdBatch];
    __shared__ int subn[16];

    const int b = blockIdx.x / g.T, t = blockIdx.x - b * g.T;
    const int ty = t / g.TX, tx = t - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = tid >> 3, lig = tid & 7;
    const int gx = grp & 3;                     // region column; region row == warp
    const int li = lig & 1, lj = lig >> 1;
    const int lx = 4 * gx + 2 * li, ly = 4 * warp + lj;  // pixel pair (lx, ly), (lx + 1, ly)
    const float fx = (float)lx, fy = (float)ly;
    const unsigned bitA = 1u << (16 + 4 * lj + 2 * li), bitB = bitA << 1;
    const unsigned lt = lanemask_lt();

    float accA[C], accB[C];
#pragma unroll
    for (int c = 0; c < C; ++c) accA[c] = accB[c] = 0.0f;

    int L0, L1;
    list_range(offs, g, b, t, err, L0, L1);
    for (int e0 = L0; e0 < L1; e0 += kFwdBatch) {
        const int n = min(kFwdBatch, L1 - e0);
        __syncthreads();  // the previous batch is fully consumed
        for (int e = tid; e < n; e += kFwdThreads) {
            const int i = ids[e0 + e];
            if ((unsigned)i >= (unsigned)g.N) {  // never for consistent bins
                atomicOr(err, kErrBadId);
                win[e] = 0u;
                continue;
            }
            const size_t gid = (size_t)b * g.N + i;
            const float4 A = gr[2 * gid], Q = gr[2 * gid + 1];
            const float mx = A.x - (float)X0, my = A.y - (float)Y0;
            const float K1 = -fmaf(A.z, mx, A.w * my);
            const float K2 = -fmaf(Q.x, mx, Q.y * my);
            const int cx = __float_as_int(Q.z), cy = __float_as_int(Q.w);
            const int lx0 = max(cx - g.r - X0, 0), lx1 = min(cx + g.r - X0, kTile - 1);
            const int ly0 = max(cy - g.r - Y0, 0), ly1 = min(cy + g.r - Y0, kTile - 1);
            const unsigned cm = (2u << lx1) - (1u << lx0);
            const unsigned rm = (2u << ly1) - (1u << ly0);
            float r[RV * 4];
            r[0] = A.z; r[1] = A.w; r[2] = K1; r[3] = Q.x; r[4] = Q.y; r[5] = K2;
            const float *pa = params + gid * g.P + 5;
#pragma unroll
            for (int c = 0; c < C; ++c) r[6 + c] = pa[c];
#pragma unroll
            for (int c = 6 + C; c < RV * 4; ++c) r[c] = 0.0f;
#pragma unroll
            for (int v = 0; v < RV; ++v)
                rec[e * RV + v] = make_float4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            win[e] = (cm & 0xffffu) | ((rm & 0xffffu) << 16);
        }
        __syncthreads();
        {
            // Sub-lists of this warp's four regions (rows 4*warp .. 4*warp+3).
            int cnt[4] = {0, 0, 0, 0};
            const int nr = (n + 31) & ~31;
            for (int e = lane; e < nr; e += 32) {
                const unsigned wm = e < n ? win[e] : 0u;
                const unsigned rb = (wm >> (16 + 4 * warp)) & 0xfu;
                unsigned rs = (rb & 1u) | ((rb & 2u) << 3) | ((rb & 4u) << 6) | ((rb & 8u) << 9);
                rs *= 0xfu;  // one full nibble per window row of the region
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const unsigned cb = (wm >> (4 * q)) & 0xfu;
                    const unsigned pm = (cb * 0x1111u) & rs;
                    const unsigned bal = __ballot_sync(0xffffffffu, pm != 0u);
                    if (pm) sub[4 * warp + q][cnt[q] + __popc(bal & lt)] = (pm << 16) | (unsigned)e;
                    cnt[q] += __popc(bal);
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q) subn[4 * warp + q] = cnt[q];
            }
        }
        __syncthreads();
        const int ns = subn[grp];
        const unsigned *sl = sub[grp];
        for (int s = 0; s < ns; ++s) {
            const unsigned pk = sl[s];
            const float4 *r4 = rec + (pk & 0xffffu) * RV;
            float rr[RV * 4];
#pragma unroll
            for (int v = 0; v < RV; ++v) {
                const float4 q = r4[v];
                rr[4 * v] = q.x; rr[4 * v + 1] = q.y; rr[4 * v + 2] = q.z; rr[4 * v + 3] = q.w;
            }
            const float uA1 = fmaf(rr[0], fx, fmaf(rr[1], fy, rr[2]));
            const float uA2 = fmaf(rr[3], fx, fmaf(rr[4], fy, rr[5]));
            const float uB1 = uA1 + rr[0], uB2 = uA2 + rr[3];
            const float wA = ex2(fmaf(-uA1, uA1, -uA2 * uA2));
            const float wB = ex2(fmaf(-uB1, uB1, -uB2 * uB2));
            if (pk & bitA) {
#pragma unroll
                for (int c = 0; c < C; ++c) accA[c] = fmaf(rr[6 + c], wA, accA[c]);
            }
            if (pk & bitB) {
#pragma unroll
                for (int c = 0; c < C; ++c) accB[c] = fmaf(rr[6 + c], wB, accB[c]);
            }
        }
    }

    const int x = X0 + lx, y = Y0 + ly;
    if (y < g.H && x < g.W) {
        const bool pair = (x + 1 < g.W) && g.out_vec2;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float *dst = image + (((size_t)b * C + c) * g.H + y) * g.W + x;
            if (pair) {
                *reinterpret_cast<float2 *>(dst) = make_float2(accA[c], accB[c]);
            } else {
                dst[0] = accA[c];
                if (x + 1 < g.W) dst[1] = accB[c];
            }
        }
    }
}

template <int C>
cudaError_t launch_fwd_c(const float *params, const Geom &g, const Workspace &ws,
                         float *image, cudaStream_t s) {
    k_fwd<C><<<g.B * g.T, kFwdThreads, 0, s>>>(params, g, ws.gr, ws.offs, ws.ids, image, ws.err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const float *params, const Geom &g, const Workspace &ws,
                       float *image, cudaStream_t s) {
    switch (g.C) {
        case 1: return launch_fwd_c<1>(params, g, ws, image, s);
        case 2: return launch_fwd_c<2>(params, g, ws, image, s);
        case 3: return launch_fwd_c<3>(params, g, ws, image, s);
        case 4: return launch_fwd_c<4>(params, g, ws, image, s);
        case 5: return launch_fwd_c<5>(params, g, ws, image, s);
        case 6: return launch_fwd_c<6>(params, g, ws, image, s);
        case 7: return launch_fwd_c<7>(params, g, ws, image, s);
        case 8: return launch_fwd_c<8>(params, g, ws, image, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pdr
