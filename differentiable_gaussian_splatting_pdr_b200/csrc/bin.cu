// Tile binner: every Gaussian goes into the list of each 16x16 tile that its
// clipped k x k window touches, lists in ascending Gaussian id so that every
// fp32 sum downstream has a fixed order.  The additive accumulation (reading
// notes, "Method") has no depth order, so any fixed order is correct;
// ascending id is the one the oracle also uses.  Four kernels on the
// caller's stream, no float atomics, no host synchronisation:
//
//   k_count   one block per (frame, chunk of kBinChunk Gaussians): the
//             per-Gaussian record (window centre, rotated and scaled axes)
//             and the chunk's per-tile counts (integer shared-memory atomics
//             count only; they never decide a position);
//   k_scan_tiles / k_scan_frames
//             exclusive prefix of each tile's counts over the chunks (32 tiles
//             x 32 chunks per step through shared memory), then one block per
//             frame scans the tile totals into the tiles' list starts;
//   k_scatter one block per (frame, chunk): stable ranks in rounds of
//             blockDim Gaussians -- rank in a tile = earlier chunks (the scans) +
//             earlier rounds + earlier warps' popcounts + lanes below in this
//             warp (per-warp lane bitmasks) -- so positions never depend on
//             the order in which atomics land.
// Small frames (g.frame_block) take one launch instead: k_bin_frame, one
// block per frame, does the records, the counts, the tile offsets and the
// stable scatter in shared memory (ranks from a per-tile prefix over the
// block's warps).  Same lists, same order.
#include "common.cuh"

namespace pdr {

namespace {

constexpr int kCountThreads = 256;

__global__ void __launch_bounds__(kCountThreads) k_count(const float *__restrict__ params,
                                                         Geom g, float4 *__restrict__ gr,
                                                         int *__restrict__ hist,
                                                         int *__restrict__ err) {
    extern __shared__ int hs[];  // [T]
    const int b = blockIdx.y, c = blockIdx.x;
    for (int t = threadIdx.x; t < g.T; t += blockDim.x) hs[t] = 0;
    __syncthreads();
    const int i0 = c * kBinChunk, i1 = min(i0 + kBinChunk, g.N);
    constexpr int U = kBinChunk / kCountThreads;  // Gaussians per thread, all in flight
    float4 A[U], Q[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kCountThreads + threadIdx.x;
        if (i < i1) gaussian_record(params + ((size_t)b * g.N + i) * g.P, A[u], Q[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kCountThreads + threadIdx.x;
        if (i >= i1) continue;
        const size_t gid = (size_t)b * g.N + i;
        gr[2 * gid] = A[u];
        gr[2 * gid + 1] = Q[u];
        int x0, x1, y0, y1;
        if (window_rect(__float_as_int(Q[u].z), __float_as_int(Q[u].w), g, x0, x1, y0, y1)) {
            for (int ty = y0 >> 4; ty <= (y1 >> 4); ++ty)
                for (int tx = x0 >> 4; tx <= (x1 >> 4); ++tx) atomicAdd(&hs[ty * g.TX + tx], 1);
        }
    }
    __syncthreads();
    int *h = hist + ((size_t)b * g.nchunks + c) * g.T;
    for (int t = threadIdx.x; t < g.T; t += blockDim.x) h[t] = hs[t];
}

// Block-wide inclusive scan of one int per thread (blockDim.x a multiple of 32).
__device__ __forceinline__ int block_incl_scan(int v, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w += u;
        }
        if (lane < nw) warp_tot[lane] = w;
    }
    __syncthreads();
    total = warp_tot[nw - 1];
    const int r = v + (warp ? warp_tot[warp - 1] : 0);
    __syncthreads();
    return r;
}

// hist[b][c][t] <- exclusive prefix over c of the counts (relative to the
// tile's list start); offs[b][t] <- the tile's total (turned into the
// absolute list start by k_scan_frames).  Block (x, b) takes tiles
// 32x .. 32x + 31 of frame b: the chunk counts pass through shared memory
// 32 chunks at a time (coalesced along the tiles on both sides), and warp w
// scans tile 32x + w over those chunks, carrying the running sum.
__global__ void __launch_bounds__(1024) k_scan_tiles(Geom g, int *__restrict__ hist,
                                                     int *__restrict__ offs) {
    __shared__ int v[32][33];  // [chunk][tile], padded against bank conflicts
    const int b = blockIdx.y, t0 = blockIdx.x * 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int *h = hist + (size_t)b * g.nchunks * g.T;
    int carry = 0;  // warp's tile: sum of the chunks already scanned
    for (int c0 = 0; c0 < g.nchunks; c0 += 32) {
        {
            const int c = c0 + warp, t = t0 + lane;  // load: warp = chunk, lane = tile
            v[warp][lane] = (c < g.nchunks && t < g.T) ? h[(size_t)c * g.T + t] : 0;
        }
        __syncthreads();
        {
            const int x = v[lane][warp];  // scan: warp = tile, lane = chunk
            int incl = x;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += u;
            }
            v[lane][warp] = carry + incl - x;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncthreads();
        {
            const int c = c0 + warp, t = t0 + lane;
            if (c < g.nchunks && t < g.T) h[(size_t)c * g.T + t] = v[warp][lane];
        }
        __syncthreads();
    }
    if (lane == 0 && t0 + warp < g.T) offs[(size_t)b * (g.T + 1) + t0 + warp] = carry;
}

// offs[b][t] <- frame start + exclusive prefix over the tiles of their totals.
__global__ void __launch_bounds__(1024) k_scan_frames(Geom g, int *__restrict__ offs) {
    __shared__ int warp_tot[32];
    const int b = blockIdx.x;
    int *o = offs + (size_t)b * (g.T + 1);
    int carry = b * g.cap;
    for (int t0 = 0; t0 < g.T; t0 += blockDim.x) {
        const int t = t0 + threadIdx.x;
        const int tot = t < g.T ? o[t] : 0;
        int total;
        const int incl = block_incl_scan(tot, warp_tot, total);
        if (t < g.T) o[t] = carry + incl - tot;
        carry += total;
    }
    if (threadIdx.x == 0) o[g.T] = carry;
}

__global__ void k_scatter(Geom g, const float4 *__restrict__ gr, const int *__restrict__ hist,
                          const int *__restrict__ offs, int *__restrict__ ids,
                          int *__restrict__ err) {
    extern __shared__ unsigned sm[];
    const int nw = blockDim.x >> 5;
    unsigned *masks = sm;                                   // [nw][T]
    int *running = reinterpret_cast<int *>(sm + nw * g.T);  // [T]
    int *base_s = running + g.T;                            // [T]
    const int b = blockIdx.y, c = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = lanemask_lt();
    const int *hsrc = hist + ((size_t)b * g.nchunks + c) * g.T;
    const int *osrc = offs + (size_t)b * (g.T + 1);
    for (int t = threadIdx.x; t < g.T; t += blockDim.x) {
        base_s[t] = osrc[t] + hsrc[t];
        running[t] = 0;
    }
    for (int t = threadIdx.x; t < nw * g.T; t += blockDim.x) masks[t] = 0u;
    __syncthreads();
    const long long lo = (long long)b * g.cap, hi = lo + g.cap;
    unsigned *my = masks + warp * g.T;
    const int i0 = c * kBinChunk, i1 = min(i0 + kBinChunk, g.N);
    for (int s = i0; s < i1; s += blockDim.x) {
        const int i = s + threadIdx.x;
        int tx0 = 1, tx1 = 0, ty0 = 1, ty1 = 0;  // empty unless the window hits the grid
        int ht = -1;                              // home tile
        if (i < i1) {
            const float4 Q = gr[2 * ((size_t)b * g.N + i) + 1];
            int x0, x1, y0, y1;
            if (window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
                tx0 = x0 >> 4; tx1 = x1 >> 4; ty0 = y0 >> 4; ty1 = y1 >> 4;
                ht = home_tile(__float_as_int(Q.z), __float_as_int(Q.w), g);
            }
        }
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) atomicOr(&my[ty * g.TX + tx], 1u << lane);
        __syncthreads();
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) {
                const int t = ty * g.TX + tx;
                int pre = running[t] + __popc(my[t] & lt);
                for (int w = 0; w < warp; ++w) pre += __popc(masks[w * g.T + t]);
                const long long slot = (long long)base_s[t] + pre;
                if (slot >= lo && slot < hi)
                    ids[slot] = (int)((unsigned)i | (t == ht ? kHomeFlag : 0u));
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

// One block per frame: the whole binner of a small frame in one launch.
__global__ void __launch_bounds__(1024) k_bin_frame(const float *__restrict__ params, Geom g,
                                                    float4 *__restrict__ gr,
                                                    int *__restrict__ offs,
                                                    int *__restrict__ ids,
                                                    int *__restrict__ err) {
    extern __shared__ int fsm[];
    const int T = g.T, nw = blockDim.x >> 5;
    int *run = fsm;                                            // [T] counts, then list cursor
    int *tot = run + T;                                        // [T] a round's per-tile total
    unsigned *masks = reinterpret_cast<unsigned *>(tot + T);  // [nw][T] lanes per (warp, tile)
    int *pre = reinterpret_cast<int *>(masks + nw * T);        // [nw][T] earlier warps' count
    __shared__ int warp_tot[32];
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    for (int t = tid; t < T; t += blockDim.x) run[t] = 0;
    for (int t = tid; t < nw * T; t += blockDim.x) masks[t] = 0u;
    __syncthreads();

    // 1. records and counts, four Gaussians per thread in flight
    constexpr int U = 4;
    for (int i0 = 0; i0 < g.N; i0 += U * blockDim.x) {
        float4 A[U], Q[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * blockDim.x + tid;
            if (i < g.N) gaussian_record(params + ((size_t)b * g.N + i) * g.P, A[u], Q[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * blockDim.x + tid;
            if (i >= g.N) continue;
            const size_t gid = (size_t)b * g.N + i;
            gr[2 * gid] = A[u];
            gr[2 * gid + 1] = Q[u];
            int x0, x1, y0, y1;
            if (window_rect(__float_as_int(Q[u].z), __float_as_int(Q[u].w), g, x0, x1, y0, y1)) {
                for (int ty = y0 >> 4; ty <= (y1 >> 4); ++ty)
                    for (int tx = x0 >> 4; tx <= (x1 >> 4); ++tx)
                        atomicAdd(&run[ty * g.TX + tx], 1);
            }
        }
    }
    __syncthreads();

    // 2. tile offsets; run[t] becomes the next free slot of tile t
    int carry = 0;
    for (int t0 = 0; t0 < T; t0 += blockDim.x) {
        const int t = t0 + tid;
        const int c = t < T ? run[t] : 0;
        int total;
        const int excl = block_excl_scan(c, warp_tot, total);
        const int start = b * g.cap + carry + excl;
        if (t < T) {
            offs[(size_t)b * (T + 1) + t] = start;
            run[t] = start;
        }
        carry += total;
    }
    if (tid == 0) offs[(size_t)b * (T + 1) + T] = b * g.cap + carry;
    __syncthreads();

    // 3. stable scatter, one round of blockDim Gaussians at a time
    const long long lo = (long long)b * g.cap, hi = lo + g.cap;
    unsigned *my = masks + warp * T;
    for (int s = 0; s < g.N; s += blockDim.x) {
        const int i = s + tid;
        int tx0 = 1, tx1 = 0, ty0 = 1, ty1 = 0;  // empty unless the window hits the grid
        int ht = -1;                              // home tile
        if (i < g.N) {
            const float4 Q = gr[2 * ((size_t)b * g.N + i) + 1];
            int x0, x1, y0, y1;
            if (window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
                tx0 = x0 >> 4; tx1 = x1 >> 4; ty0 = y0 >> 4; ty1 = y1 >> 4;
                ht = home_tile(__float_as_int(Q.z), __float_as_int(Q.w), g);
            }
        }
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) atomicOr(&my[ty * g.TX + tx], 1u << lane);
        __syncthreads();
        for (int t = tid; t < T; t += blockDim.x) {
            int acc = 0;
            for (int w = 0; w < nw; ++w) {
                pre[w * T + t] = acc;
                acc += __popc(masks[w * T + t]);
            }
            tot[t] = acc;
        }
        __syncthreads();
        for (int ty = ty0; ty <= ty1; ++ty)
            for (int tx = tx0; tx <= tx1; ++tx) {
                const int t = ty * g.TX + tx;
                const long long slot =
                    (long long)run[t] + pre[warp * T + t] + __popc(my[t] & lt);
                if (slot >= lo && slot < hi)
                    ids[slot] = (int)((unsigned)i | (t == ht ? kHomeFlag : 0u));
                else
                    atomicOr(err, kErrListBounds);
            }
        __syncthreads();
        for (int t = tid; t < T; t += blockDim.x) {
            run[t] += tot[t];
            for (int w = 0; w < nw; ++w) masks[w * T + t] = 0u;
        }
        __syncthreads();
    }
}

__global__ void k_copy_ids(int *__restrict__ dst, const int *__restrict__ src, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        dst[i] = entry_id(src[i]);
}

}  // namespace

cudaError_t launch_copy_ids(int *dst, const int *src, size_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const size_t blocks = (n + 255) / 256;
    k_copy_ids<<<(unsigned)(blocks < 4 * 148 ? blocks : 4 * 148), 256, 0, s>>>(dst, src, n);
    return cudaGetLastError();
}

size_t bin_frame_smem(const Geom &g) {
    return sizeof(int) * (size_t)g.T * (2 + 2 * (g.frame_threads / 32));
}

size_t bin_count_smem(const Geom &g) { return sizeof(int) * (size_t)g.T; }

size_t bin_scatter_smem(const Geom &g) {
    return sizeof(int) * (size_t)g.T * (g.scatter_warps + 2);
}

// Dynamic shared memory above which a launch needs the opt-in attribute: the
// 48 KB default less room for the kernel's static arrays.
constexpr size_t kStaticSmemRoom = 44 * 1024;

cudaError_t launch_bin(const float *params, const Geom &g, const Workspace &ws,
                       cudaStream_t s) {
    cudaError_t e;
    if (g.frame_block) {
        const size_t sf = bin_frame_smem(g);
        if (sf > kStaticSmemRoom) {
            e = cudaFuncSetAttribute(k_bin_frame, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sf);
            if (e != cudaSuccess) return e;
        }
        k_bin_frame<<<g.B, g.frame_threads, sf, s>>>(params, g, ws.gr, ws.offs, ws.ids, ws.err);
        return cudaGetLastError();
    }
    const size_t sc = bin_count_smem(g), ss = bin_scatter_smem(g);
    if (sc > 48 * 1024) {
        e = cudaFuncSetAttribute(k_count, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc);
        if (e != cudaSuccess) return e;
    }
    if (ss > 48 * 1024) {
        e = cudaFuncSetAttribute(k_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ss);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid(g.nchunks, g.B);
    const int scan_threads = g.T >= 1024 ? 1024 : ((g.T + 31) / 32) * 32;
    k_count<<<grid, kCountThreads, sc, s>>>(params, g, ws.gr, ws.hist, ws.err);
    k_scan_tiles<<<dim3((g.T + 31) / 32, g.B), 1024, 0, s>>>(g, ws.hist, ws.offs);
    k_scan_frames<<<g.B, scan_threads, 0, s>>>(g, ws.offs);
    k_scatter<<<grid, 32 * g.scatter_warps, ss, s>>>(g, ws.gr, ws.hist, ws.offs, ws.ids, ws.err);
    return cudaGetLastError();
}

}  // namespace pdr
