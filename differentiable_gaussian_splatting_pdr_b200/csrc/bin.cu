// Tile binner: every Gaussian goes into the list of each 16x16 tile that its
// clipped k x k window touches, lists in ascending Gaussian id so that every
// fp32 sum downstream has a fixed order.  Three kernels, all on the caller's
// stream, no float atomics, no host synchronisation:
//
//   k_count   one block per (frame, chunk of Gaussians): per-Gaussian record
//             (window centre, rotated/scaled axes) and a chunk histogram over
//             the frame's tiles (integer shared-memory atomics count only);
//   k_scan    one block per frame: for every tile, exclusive prefix over the
//             chunks, then a block scan over tiles gives each (tile, chunk)
//             its absolute list base and each tile its list start;
//   k_scatter one block per (frame, chunk): stable in-chunk ranks from
//             per-warp lane bitmasks (rank = earlier warps' popcounts + the
//             lanes below in this warp), so positions never depend on the
//             order in which atomics land.
//
// The additive accumulation (reading notes, "Method") has no depth order, so
// any fixed order is correct; ascending id is the one the oracle also uses.
#include "common.cuh"

namespace pdr {

namespace {

__device__ __forceinline__ bool window_rect(int cx, int cy, const Geom &g, int &x0,
                                            int &x1, int &y0, int &y1) {
    x0 = max(cx - g.r, 0);
    x1 = min(cx + g.r, g.W - 1);
    y0 = max(cy - g.r, 0);
    y1 = min(cy + g.r, g.H - 1);
    return x0 <= x1 && y0 <= y1;
}

__global__ void __launch_bounds__(512) k_count(const float *__restrict__ params,
                                               Geom g, float4 *__restrict__ gr,
                                               int *__restrict__ hist, int *__restrict__ err) {
    extern __shared__ int hs[];  // [T]
    const int b = blockIdx.y, c = blockIdx.x;
    if (b == 0 && c == 0 && threadIdx.x == 0) *err = 0;
    for (int t = threadIdx.x; t < g.T; t += blockDim.x) hs[t] = 0;
    __syncthreads();
    const int i0 = c * g.chunk, i1 = min(i0 + g.chunk, g.N);
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
        const size_t gid = (size_t)b * g.N + i;
        const float *p = params + gid * g.P;
        const float mx = p[0], my = p[1], s1 = p[2], s2 = p[3], th = p[4];
        int cx = kNoCenter, cy = kNoCenter;
        if (isfinite(mx) && isfinite(my)) {
            cx = round_half_up(mx);
            cy = round_half_up(my);
        }
        float sn, cs;
        sincosf(th, &sn, &cs);
        const float h1 = kSqrtKappa * expf(-s1), h2 = kSqrtKappa * expf(-s2);
        gr[2 * gid] = make_float4(mx, my, h1 * cs, h1 * sn);
        gr[2 * gid + 1] = make_float4(-h2 * sn, h2 * cs, __int_as_float(cx),
                                      __int_as_float(cy));
        int x0, x1, y0, y1;
        if (window_rect(cx, cy, g, x0, x1, y0, y1)) {
            for (int ty = y0 >> 4; ty <= (y1 >> 4); ++ty)
                for (int tx = x0 >> 4; tx <= (x1 >> 4); ++tx)
                    atomicAdd(&hs[ty * g.TX + tx], 1);
        }
    }
    __syncthreads();
    int *h = hist + ((size_t)b * g.nchunks + c) * g.T;
    for (int t = threadIdx.x; t < g.T; t += blockDim.x) h[t] = hs[t];
}

// Block-wide inclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_incl_scan(int v, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w += u;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    total = warp_tot[31];
    int r = v + (warp ? warp_tot[warp - 1] : 0);
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(1024) k_scan(Geom g, int *__restrict__ hist,
                                               int *__restrict__ offs) {
    __shared__ int warp_tot[32];
    const int b = blockIdx.x;
    const int frame_base = b * g.cap;
    int carry = 0;
    for (int t0 = 0; t0 < g.T; t0 += blockDim.x) {
        const int t = t0 + threadIdx.x;
        int tot = 0;
        if (t < g.T) {
            for (int c = 0; c < g.nchunks; ++c) {
                int *h = hist + ((size_t)b * g.nchunks + c) * g.T + t;
                const int v = *h;
                *h = tot;
                tot += v;
            }
        }
        int total;
        const int incl = block_incl_scan(tot, warp_tot, total);
        const int base = frame_base + carry + incl - tot;
        if (t < g.T) {
            offs[(size_t)b * (g.T + 1) + t] = base;
            for (int c = 0; c < g.nchunks; ++c)
                hist[((size_t)b * g.nchunks + c) * g.T + t] += base;
        }
        carry += total;
    }
    if (threadIdx.x == 0) offs[(size_t)b * (g.T + 1) + g.T] = frame_base + carry;
}

__global__ void k_scatter(Geom g, const float4 *__restrict__ gr,
                          const int *__restrict__ base, int *__restrict__ ids,
                          int *__restrict__ err) {
    extern __shared__ unsigned sm[];
    const int nw = blockDim.x >> 5;
    unsigned *masks = sm;                                   // [nw][T]
    int *running = reinterpret_cast<int *>(sm + nw * g.T);  // [T]
    int *base_s = running + g.T;                            // [T]
    const int b = blockIdx.y, c = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = lanemask_lt();
    const int *bsrc = base + ((size_t)b * g.nchunks + c) * g.T;
    for (int t = threadIdx.x; t < g.T; t += blockDim.x) {
        base_s[t] = bsrc[t];
        running[t] = 0;
    }
    for (int t = threadIdx.x; t < nw * g.T; t += blockDim.x) masks[t] = 0u;
    __syncthreads();
    const int i0 = c * g.chunk, i1 = min(i0 + g.chunk, g.N);
    for (int s = i0; s < i1; s += blockDim.x) {
        const int i = s + threadIdx.x;
        int tx0 = 1, tx1 = 0, ty0 = 1, ty1 = 0;  // empty unless the window hits the grid
        if (i < i1) {
            const float4 q = gr[2 * ((size_t)b * g.N + i) + 1];
            int x0, x1, y0, y1;
            if (window_rect(__float_as_int(q.z), __float_as_int(q.w), g, x0, x1, y0, y1)) {
                tx0 = x0 >> 4; tx1 = x1 >> 4; ty0 = y0 >> 4; ty1 = y1 >> 4;
            }
        }
        unsigned *my = masks + warp * g.T;
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx)
                atomicOr(&my[ty * g.TX + tx], 1u << lane);
        __syncthreads();
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) {
                const int t = ty * g.TX + tx;
                int pre = running[t] + __popc(my[t] & lt);
                for (int w = 0; w < warp; ++w) pre += __popc(masks[w * g.T + t]);
                const long long slot = (long long)base_s[t] + pre;
                if (slot >= (long long)b * g.cap && slot < (long long)(b + 1) * g.cap)
                    ids[slot] = i;
                else
                    atomicOr(err, kErrListBounds);
            }
        __syncthreads();
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) {
                const int t = ty * g.TX + tx;
                const unsigned m = my[t];
                if (lane == __ffs(m) - 1) atomicAdd(&running[t], __popc(m));
            }
        __syncthreads();
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) my[ty * g.TX + tx] = 0u;
        __syncthreads();
    }
}

}  // namespace

size_t bin_count_smem(const Geom &g) { return sizeof(int) * (size_t)g.T; }

size_t bin_scatter_smem(const Geom &g) {
    return sizeof(int) * (size_t)g.T * (g.scatter_warps + 2);
}

cudaError_t launch_bin(const float *params, const Geom &g, const Workspace &ws,
                       cudaStream_t s) {
    const size_t sc = bin_count_smem(g), ss = bin_scatter_smem(g);
    cudaError_t e;
    if (sc > 48 * 1024) {
        e = cudaFuncSetAttribute(k_count, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc);
        if (e != cudaSuccess) return e;
    }
    if (ss > 48 * 1024) {
        e = cudaFuncSetAttribute(k_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ss);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(g.nchunks, g.B);
    k_count<<<grid, 512, sc, s>>>(params, g, ws.gr, ws.hist, ws.err);
    k_scan<<<g.B, 1024, 0, s>>>(g, ws.hist, ws.offs);
    k_scatter<<<grid, 32 * g.scatter_warps, ss, s>>>(g, ws.gr, ws.hist, ws.ids, ws.err);
    return cudaGetLastError();
}

}  // namespace pdr
