// Tile binner: every Gaussian goes into the list of each 16x16 tile that its
// clipped k x k window touches, lists in ascending Gaussian id so that every
// fp32 sum downstream has a fixed order.  The additive accumulation (reading
// notes, "Method") has no depth order, so any fixed order is correct;
// ascending id is the one the oracle also uses.  Three kernels on the
// caller's stream, no float atomics, no host synchronisation:
//
//   k_count   one block per (frame, chunk of 256 .. 1024 Gaussians): the
//             per-Gaussian record (window centre, rotated and scaled axes)
//             and the chunk's per-tile counts (integer shared-memory atomics
//             count only; they never decide a position);
//   k_scan_tiles
//             exclusive prefix of each tile's counts over the chunks (32 tiles
//             x 32 chunks per step through shared memory); the last block of
//             a frame to finish scans the frame's tile totals into the tiles'
//             list starts;
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
    const int i0 = c * g.chunk, i1 = min(i0 + g.chunk, g.N);
    constexpr int U = kBinChunk / kCountThreads;  // Gaussians per thread at most, all in flight
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
// tile's list start); offs[b][t] <- the tile's list start.  Block (x, b)
// takes tiles 32x .. 32x + 31 of frame b: the chunk counts pass through
// shared memory 32 chunks at a time (coalesced along the tiles on both
// sides), and warp w scans tile 32x + w over those chunks, carrying the
// running sum; the tile totals go to offs[b][t].  The last block of frame b
// to finish (a counter in the workspace, zeroed before the binner runs;
// nothing waits on it) then scans the frame's tile totals into list starts.
__global__ void __launch_bounds__(1024) k_scan_tiles(Geom g, int *__restrict__ hist,
                                                     int *__restrict__ offs,
                                                     int *__restrict__ done) {
    __shared__ int v[32][33];  // [chunk][tile], padded against bank conflicts
    __shared__ int warp_tot[32];
    __shared__ int last;
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
    int *o = offs + (size_t)b * (g.T + 1);
    if (lane == 0 && t0 + warp < g.T) {
        o[t0 + warp] = carry;
        __threadfence();  // this total is visible before the block is counted
    }
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&done[b], 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    int fcarry = b * g.cap;
    for (int s0 = 0; s0 < g.T; s0 += blockDim.x) {
        const int t = s0 + threadIdx.x;
        const int tot = t < g.T ? __ldcg(o + t) : 0;
        int total;
        const int incl = block_incl_scan(tot, warp_tot, total);
        if (t < g.T) o[t] = fcarry + incl - tot;
        fcarry += total;
    }
    if (threadIdx.x == 0) {
        o[g.T] = fcarry;
        done[b] = 0;
    }
}

// Stable scatter of one chunk: warp w of the block owns the contiguous slab
// [c * chunk + w * S, + S) of the chunk (S = chunk / warps), so list
// order = (warp, sub-round of 32, lane) = ascending id.  Each lane loads the
// window centres of all its Gaussians first (every load in flight at once)
// and keeps them in registers for both passes:
//   pass 1: per-(warp, tile) entry counts (shared-memory atomics that only
//           count, never decide a position);
//   prefix: each warp's first slot per tile, relative to the chunk's start
//           in that tile's list, from the counts of the earlier warps;
//   pass 2: each warp walks its slab again, 32 Gaussians at a time: the lane
//           bits of a warp-private mask per tile give the rank among this
//           sub-round's lanes, the warp's running slot per tile gives the
//           rest.  Only warp-level synchronisation inside the passes.
// The entry of each Gaussian in the list of its home tile carries kHomeFlag.
constexpr int kScatterSub = 8;  // sub-rounds of 32 per warp at most (S <= 256)

__device__ __forceinline__ void scatter_sub(const Geom &g, int b, int i, int cx, int cy,
                                            unsigned *mym, unsigned short *myslot,
                                            const int *tbase, int *__restrict__ ids,
                                            int *__restrict__ err) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = lanemask_lt();
    const long long lo = (long long)b * g.cap, hi = lo + g.cap;
    int tx0 = 1, tx1 = 0, ty0 = 1, ty1 = 0;  // empty unless the window hits the grid
    int ht = -1;                              // home tile
    int x0, x1, y0, y1;
    if (i >= 0 && window_rect(cx, cy, g, x0, x1, y0, y1)) {
        tx0 = x0 >> 4; tx1 = x1 >> 4; ty0 = y0 >> 4; ty1 = y1 >> 4;
        ht = home_tile(cx, cy, g);
    }
    for (int ty = ty0; ty <= ty1; ++ty)
        for (int tx = tx0; tx <= tx1; ++tx) atomicOr(&mym[ty * g.TX + tx], 1u << lane);
    __syncwarp();
    unsigned lead = 0u;  // bit k: this lane is the lowest lane on its k-th tile
    int k = 0;
    for (int ty = ty0; ty <= ty1; ++ty)
        for (int tx = tx0; tx <= tx1; ++tx, ++k) {
            const int t = ty * g.TX + tx;
            const unsigned m = mym[t];
            const long long slot = (long long)tbase[t] + myslot[t] + __popc(m & lt);
            if (slot >= lo && slot < hi)
                ids[slot] = (int)((unsigned)i | (t == ht ? kHomeFlag : 0u));
            else
                atomicOr(err, kErrListBounds);
            if (lane == __ffs(m) - 1) lead |= 1u << k;
        }
    __syncwarp();
    k = 0;
    for (int ty = ty0; ty <= ty1; ++ty)
        for (int tx = tx0; tx <= tx1; ++tx, ++k) {
            if (!((lead >> k) & 1u)) continue;
            const int t = ty * g.TX + tx;
            myslot[t] = (unsigned short)(myslot[t] + __popc(mym[t]));
            mym[t] = 0u;
        }
    __syncwarp();
}

// Window centres of this lane's Gaussians i0 + 32 j + lane (j < kScatterSub)
// below i1, kNoCenter elsewhere; all loads in flight at once.
__device__ __forceinline__ void load_centres(const Geom &g, const float4 *__restrict__ gr, int b,
                                             int i0, int i1, int (&cx)[kScatterSub],
                                             int (&cy)[kScatterSub]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < kScatterSub; ++j) {
        const int i = i0 + 32 * j + lane;
        cx[j] = cy[j] = kNoCenter;
        if (i < i1) {
            const float2 c2 = reinterpret_cast<const float2 *>(gr + 2 * ((size_t)b * g.N + i) + 1)[1];
            cx[j] = __float_as_int(c2.x);
            cy[j] = __float_as_int(c2.y);
        }
    }
}

// Passes 1 and 2 of one warp over its slab [i0, i1) (see above); counts,
// a block barrier and the prefix over warps happen between the passes, so
// this is called twice by every warp of the block (pass = 1, then 2).
// Slabs of at most 32 * kScatterSub Gaussians keep their centres in
// registers between the passes; longer ones reload them per group.
__device__ __forceinline__ void slab_pass(const Geom &g, const float4 *__restrict__ gr, int b,
                                          int i0, int i1, int pass, int (&cx)[kScatterSub],
                                          int (&cy)[kScatterSub], bool resident, int *mycnt,
                                          unsigned *mym, unsigned short *myslot,
                                          const int *tbase, int *__restrict__ ids,
                                          int *__restrict__ err) {
    const int lane = threadIdx.x & 31;
    for (int g0 = i0; g0 < i1; g0 += 32 * kScatterSub) {
        if (!resident) load_centres(g, gr, b, g0, i1, cx, cy);
#pragma unroll
        for (int j = 0; j < kScatterSub; ++j) {
            if (g0 + 32 * j >= i1) break;  // warp-uniform
            if (pass == 1) {
                int x0, x1, y0, y1;
                if (window_rect(cx[j], cy[j], g, x0, x1, y0, y1))
                    for (int ty = y0 >> 4; ty <= (y1 >> 4); ++ty)
                        for (int tx = x0 >> 4; tx <= (x1 >> 4); ++tx)
                            atomicAdd(&mycnt[ty * g.TX + tx], 1);
            } else {
                const int i = g0 + 32 * j + lane;
                scatter_sub(g, b, i < i1 ? i : -1, cx[j], cy[j], mym, myslot, tbase, ids, err);
            }
        }
    }
}

// Between the passes: each warp's first slot per tile (relative to tbase),
// and the count tables cleared to become pass 2's lane masks.
__device__ __forceinline__ void warp_prefix(int T, int nw, unsigned *masks, unsigned short *slots) {
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        int acc = 0;
        for (int w = 0; w < nw; ++w) {
            const int n = reinterpret_cast<int *>(masks)[w * T + t];
            slots[w * T + t] = (unsigned short)acc;
            masks[w * T + t] = 0u;
            acc += n;
        }
    }
}

__global__ void k_scatter(Geom g, const float4 *__restrict__ gr, const int *__restrict__ hist,
                          const int *__restrict__ offs, int *__restrict__ ids,
                          int *__restrict__ err) {
    extern __shared__ unsigned sm[];
    const int nw = blockDim.x >> 5, T = g.T;
    unsigned *masks = sm;                                                        // [nw][T]
    int *tbase = reinterpret_cast<int *>(sm + nw * T);                          // [T]
    unsigned short *slots = reinterpret_cast<unsigned short *>(tbase + T);      // [nw][T]
    const int b = blockIdx.y, c = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    for (int t = threadIdx.x; t < nw * T; t += blockDim.x) masks[t] = 0u;  // pass-1 counters
    const int *hsrc = hist + ((size_t)b * g.nchunks + c) * T;
    const int *osrc = offs + (size_t)b * (T + 1);
    for (int t = threadIdx.x; t < T; t += blockDim.x) tbase[t] = osrc[t] + hsrc[t];
    const int S = g.chunk / nw;
    const int c0 = c * g.chunk, c1 = min(c0 + g.chunk, g.N);
    const int i0 = min(c0 + warp * S, c1), i1 = min(i0 + S, c1);
    const bool resident = S <= 32 * kScatterSub;
    int cx[kScatterSub], cy[kScatterSub];
    if (resident) load_centres(g, gr, b, i0, i1, cx, cy);
    __syncthreads();
    int *mycnt = reinterpret_cast<int *>(masks + warp * T);
    unsigned *mym = masks + warp * T;
    unsigned short *myslot = slots + warp * T;
    slab_pass(g, gr, b, i0, i1, 1, cx, cy, resident, mycnt, mym, myslot, tbase, ids, err);
    __syncthreads();
    warp_prefix(T, nw, masks, slots);
    __syncthreads();
    slab_pass(g, gr, b, i0, i1, 2, cx, cy, resident, mycnt, mym, myslot, tbase, ids, err);
}

// One block per frame: the whole binner of a small frame in one launch.
// Warp w owns the contiguous slab [w * S, (w + 1) * S) of the frame's
// Gaussians: it computes their records and counts them per tile; one block
// scan turns the per-tile totals into the tiles' list starts; then every
// warp scatters its slab as in k_scatter.
__global__ void __launch_bounds__(1024) k_bin_frame(const float *__restrict__ params, Geom g,
                                                    float4 *__restrict__ gr,
                                                    int *__restrict__ offs,
                                                    int *__restrict__ ids,
                                                    int *__restrict__ err) {
    extern __shared__ unsigned fsm[];
    const int T = g.T, nw = blockDim.x >> 5;
    unsigned *masks = fsm;                                                   // [nw][T]
    int *tbase = reinterpret_cast<int *>(fsm + nw * T);                     // [T]
    unsigned short *slots = reinterpret_cast<unsigned short *>(tbase + T);  // [nw][T]
    __shared__ int warp_tot[32];
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int t = tid; t < nw * T; t += blockDim.x) masks[t] = 0u;
    __syncthreads();
    const int S = (((g.N + nw - 1) / nw) + 31) & ~31;
    const int i0 = min(warp * S, g.N), i1 = min(i0 + S, g.N);
    int *mycnt = reinterpret_cast<int *>(masks + warp * T);

    // 1. records and this warp's counts per tile, several Gaussians per lane in flight
    constexpr int U = 4;
    for (int s = i0; s < i1; s += 32 * U) {
        float4 A[U], Q[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = s + 32 * u + lane;
            if (i < i1) gaussian_record(params + ((size_t)b * g.N + i) * g.P, A[u], Q[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = s + 32 * u + lane;
            if (i >= i1) continue;
            const size_t gid = (size_t)b * g.N + i;
            gr[2 * gid] = A[u];
            gr[2 * gid + 1] = Q[u];
            int x0, x1, y0, y1;
            if (window_rect(__float_as_int(Q[u].z), __float_as_int(Q[u].w), g, x0, x1, y0, y1)) {
                for (int ty = y0 >> 4; ty <= (y1 >> 4); ++ty)
                    for (int tx = x0 >> 4; tx <= (x1 >> 4); ++tx)
                        atomicAdd(&mycnt[ty * g.TX + tx], 1);
            }
        }
    }
    __syncthreads();

    // 2. tile offsets (block scan of the per-tile totals), then each warp's
    //    first slot per tile relative to the tile's start
    int carry = 0;
    for (int t0 = 0; t0 < T; t0 += blockDim.x) {
        const int t = t0 + tid;
        int tot = 0;
        if (t < T)
            for (int w = 0; w < nw; ++w) tot += reinterpret_cast<int *>(masks)[w * T + t];
        int total;
        const int excl = block_excl_scan(tot, warp_tot, total);
        if (t < T) {
            const int start = b * g.cap + carry + excl;
            offs[(size_t)b * (T + 1) + t] = start;
            tbase[t] = start;
        }
        carry += total;
    }
    if (tid == 0) offs[(size_t)b * (T + 1) + T] = b * g.cap + carry;
    __syncthreads();
    warp_prefix(T, nw, masks, slots);
    __syncthreads();

    // 3. stable scatter of this warp's slab (its records are its own writes above)
    int cx[kScatterSub], cy[kScatterSub];
    slab_pass(g, gr, b, i0, i1, 2, cx, cy, false, mycnt, masks + warp * T, slots + warp * T,
              tbase, ids, err);
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

// Per-warp count / lane-mask table (4 bytes), per-warp slot table (2 bytes)
// and the tiles' bases (4 bytes).
static size_t bin_tables_bytes(int T, int nw) { return (size_t)T * (6 * (size_t)nw + 4) + 16; }

size_t bin_frame_smem(const Geom &g) { return bin_tables_bytes(g.T, g.frame_threads / 32); }

size_t bin_count_smem(const Geom &g) { return sizeof(int) * (size_t)g.T; }

size_t bin_scatter_smem(const Geom &g) { return bin_tables_bytes(g.T, g.scatter_warps); }

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
    k_count<<<grid, kCountThreads, sc, s>>>(params, g, ws.gr, ws.hist, ws.err);
    k_scan_tiles<<<dim3((g.T + 31) / 32, g.B), 1024, 0, s>>>(g, ws.hist, ws.offs, ws.done);
    k_scatter<<<grid, 32 * g.scatter_warps, ss, s>>>(g, ws.gr, ws.hist, ws.offs, ws.ids, ws.err);
    return cudaGetLastError();
}

}  // namespace pdr
