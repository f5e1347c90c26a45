// Tile binner: every Gaussian goes into the list of each 16x16 tile that its
// clipped k x k window touches, lists in ascending Gaussian id so that every
// fp32 sum downstream has a fixed order.  The additive accumulation (reading
// notes, "Method") has no depth order, so any fixed order is correct;
// ascending id is the one the oracle also uses.  No float atomics, no host
// synchronisation; integer shared-memory atomics only count or set lane bits,
// never decide a position.
//
// Large frames (three kernels on the caller's stream; a slab is g.slab
// consecutive Gaussians of a frame, one warp each):
//   k_slab_count    per slab: the per-Gaussian records (window centre,
//                   rotated and scaled axes) and the slab's count per tile;
//   k_slab_scan     per tile: exclusive prefix of the counts over the slabs,
//                   and the tile's total;
//   k_slab_scatter  per block: the tiles' list starts (block scan of the
//                   totals); per slab: stable ranks in rounds of 32 from
//                   lane masks, written at start + slab prefix + rank.
// Frames of at most 64 tiles take one launch instead: k_bin_cluster, one
// thread-block cluster per frame (chunk counts exchanged through distributed
// shared memory).  Other small frames (g.frame_block) take k_bin_frame, one
// block per frame doing the records, the counts, the tile offsets and the
// stable scatter in shared memory (ranks from a per-tile prefix over the
// block's warps).  Same lists, same order.
#include <cooperative_groups.h>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"

namespace pdr {

namespace cg = cooperative_groups;

namespace {

// Stable scatter of a frame by the block's warps (k_bin_frame): warp w owns
// the contiguous slab [w * S, (w + 1) * S) of the frame, so list order =
// (warp, sub-round of 32, lane) = ascending id.
//   pass 1: per-(warp, tile) entry counts;
//   prefix: each warp's first slot per tile, relative to the tile's start,
//           from the counts of the earlier warps;
//   pass 2: each warp walks its slab again, 32 Gaussians at a time: the lane
//           bits of a warp-private mask per tile give the rank among this
//           sub-round's lanes, the warp's running slot per tile gives the
//           rest.  Only warp-level synchronisation inside the passes.
// The entry of each Gaussian in the list of its home tile carries kHomeFlag.
constexpr int kScatterSub = 8;  // sub-rounds of 32 whose centres a lane holds

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

// ---- large frames: the slab binner ---------------------------------------
// A slab is g.slab consecutive Gaussians of one frame (a multiple of 32):
// counted by k_slab_count blocks of 256 threads, scattered by one warp of
// k_slab_scatter in rounds of 32.  k_slab_scan and k_slab_scatter are
// programmatic dependent launches (each waits for its predecessor at its
// top); none of the three releases its successor early.
constexpr int kSlabThreads = 256;
constexpr int kSlabWarps = 8;  // most warps (slabs) per k_slab_scatter block

// Window of a Gaussian as a tile rectangle: tiles (tx0 + dx, ty0 + dy) for
// dx < nx, dy < ny (nx = ny = 0 when the window misses the grid).
__device__ __forceinline__ void window_tiles(int cx, int cy, const Geom &g, int &tx0, int &ty0,
                                             int &nx, int &ny) {
    int x0, x1, y0, y1;
    if (window_rect(cx, cy, g, x0, x1, y0, y1)) {
        tx0 = x0 >> 4;
        ty0 = y0 >> 4;
        nx = (x1 >> 4) - tx0 + 1;
        ny = (y1 >> 4) - ty0 + 1;
    } else {
        tx0 = ty0 = nx = ny = 0;
    }
}

// Per slab: the records of its Gaussians (written to gr) and its entry
// count per tile, hist[b][s][t].  A block takes max(slab, 256) consecutive
// Gaussians, one per thread and round: one slab, or 256 / slab whole slabs
// (one shared-memory count table each).  Grid (ceil(N / max(slab, 256)), B).
__global__ void __launch_bounds__(kSlabThreads) k_slab_count(const float *__restrict__ params,
                                                             Geom g, float4 *__restrict__ gr,
                                                             int *__restrict__ hist) {
    extern __shared__ int cnt[];  // [slabs of the block][T]
    grid_dep_wait();
    const int T = g.T, b = blockIdx.y;
    const int span = max(g.slab, kSlabThreads), ntab = span / g.slab;
    const int s0 = blockIdx.x * ntab;  // first slab of the block
    for (int t = threadIdx.x; t < ntab * T; t += kSlabThreads) cnt[t] = 0;
    __syncthreads();
    int *mine = cnt + (ntab > 1 ? (int)threadIdx.x / g.slab : 0) * T;
    const int i1 = min((blockIdx.x + 1) * span, g.N);
    for (int i = blockIdx.x * span + threadIdx.x; i < i1; i += kSlabThreads) {
        const size_t gid = (size_t)b * g.N + i;
        float4 A, Q;
        gaussian_record(params + gid * g.P, A, Q);
        gr[2 * gid] = A;
        gr[2 * gid + 1] = Q;
        int tx0, ty0, nx, ny;
        window_tiles(__float_as_int(Q.z), __float_as_int(Q.w), g, tx0, ty0, nx, ny);
        for (int dy = 0; dy < ny; ++dy)
            for (int dx = 0; dx < nx; ++dx) atomicAdd(&mine[(ty0 + dy) * g.TX + tx0 + dx], 1);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < ntab * T; q += kSlabThreads) {
        const int tab = q / T, s = s0 + tab;
        if (s < g.nslab) hist[((size_t)b * g.nslab + s) * T + (q - tab * T)] = cnt[q];
    }
}

// hist[b][s][t] <- exclusive prefix over the slabs s (the slab's first slot
// in tile t, relative to the tile's list start); tot[b][t] <- the tile's
// entry count.  Block (x, b) takes tiles 32x .. 32x + 31 of frame b, lane =
// tile (coalesced rows); warp w takes a contiguous run of slabs, sums it,
// the 32 x 32 partial sums are scanned across the warps through shared
// memory, and each warp rescans its run from its offset.  Runs of at most
// kScanRegs slabs stay in registers between the two sweeps.
constexpr int kScanRegs = 8;

__global__ void __launch_bounds__(1024) k_slab_scan(Geom g, int *__restrict__ hist,
                                                    int *__restrict__ tot) {
    __shared__ int part[32][33];  // [warp][tile], padded against bank conflicts
    grid_dep_wait();
    const int b = blockIdx.y, t0 = blockIdx.x * 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = t0 + lane, T = g.T;
    const bool tin = t < T;
    const int spw = (g.nslab + 31) / 32;
    const int s0 = min(warp * spw, g.nslab), s1 = min(s0 + spw, g.nslab);
    int *h = hist + (size_t)b * g.nslab * T + t;
    const bool inreg = spw <= kScanRegs;  // block-uniform
    int x[kScanRegs];
    int sum = 0;
    if (inreg) {
#pragma unroll
        for (int q = 0; q < kScanRegs; ++q) {
            x[q] = (s0 + q < s1 && tin) ? h[(size_t)(s0 + q) * T] : 0;
            sum += x[q];
        }
    } else if (tin) {
        for (int s = s0; s < s1; ++s) sum += h[(size_t)s * T];
    }
    part[warp][lane] = sum;
    __syncthreads();
    {
        // warp = tile, lane = slab run
        const int v = part[lane][warp];
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += u;
        }
        part[lane][warp] = incl - v;
        if (lane == 31 && t0 + warp < T) tot[(size_t)b * T + t0 + warp] = incl;
    }
    __syncthreads();
    if (!tin) return;
    int run = part[warp][lane];
    if (inreg) {
#pragma unroll
        for (int q = 0; q < kScanRegs; ++q)
            if (s0 + q < s1) {
                h[(size_t)(s0 + q) * T] = run;
                run += x[q];
            }
    } else {
        for (int s = s0; s < s1; ++s) {
            const int v = h[(size_t)s * T];
            h[(size_t)s * T] = run;
            run += v;
        }
    }
}

// Stable scatter, one warp per slab, grid (ceil(nslab / slab_warps), B).  The
// block first turns the frame's tile totals into list starts (a block scan;
// block 0 of the frame also publishes them in offs).  Warp w then keeps two
// tables over the tiles: the next free slot of its slab in each tile (list
// start + the slab's exclusive prefix) and a lane mask.  Per round of 32
// Gaussians (lane = id order): every lane sets its bit in the masks of its
// tiles; its rank in a tile is the number of lower lanes in that mask; the
// lowest lane of each tile then advances the tile's slot by the mask's
// population and clears the mask.  List order = (slab, round, lane) =
// ascending id, whatever order the shared-memory atomics land in.  The
// entry in the list of the Gaussian's home tile carries kHomeFlag.
template <int M>  // most tiles a window touches along an axis (2: k <= 17, 3: k <= 33)
__global__ void __launch_bounds__(32 * kSlabWarps) k_slab_scatter(
    Geom g, const float4 *__restrict__ gr, const int *__restrict__ hist,
    const int *__restrict__ tot, int *__restrict__ offs, int *__restrict__ ids,
    int *__restrict__ err) {
    extern __shared__ int ssm[];
    grid_dep_wait();
    __shared__ int warp_tot[32];
    const int T = g.T, nwb = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y, s = blockIdx.x * nwb + warp;
    int *fofs = ssm;  // [T] list starts of the frame's tiles
    {
        // Thread j sums tiles [j * Q, j * Q + Q); one block scan.
        const int Q = (T + (int)blockDim.x - 1) / (int)blockDim.x;
        const int *tb = tot + (size_t)b * T;
        const int ta = min((int)threadIdx.x * Q, T), tz = min(ta + Q, T);
        int sum = 0;
        for (int t = ta; t < tz; ++t) sum += tb[t];
        int total;
        int run = b * g.cap + block_excl_scan(sum, warp_tot, total);
        for (int t = ta; t < tz; ++t) {
            fofs[t] = run;
            run += tb[t];
        }
        if (blockIdx.x == 0 && threadIdx.x == 0) offs[(size_t)b * (T + 1) + T] = b * g.cap + total;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        int *o = offs + (size_t)b * (T + 1);
        for (int t = threadIdx.x; t < T; t += blockDim.x) o[t] = fofs[t];
    }
    if (s >= g.nslab) return;  // warp-uniform, after the last block barrier
    int *nxt = ssm + T + warp * 2 * T;
    unsigned *msk = reinterpret_cast<unsigned *>(nxt + T);
    const int *h = hist + ((size_t)b * g.nslab + s) * T;
    for (int t = lane; t < T; t += 32) {
        nxt[t] = fofs[t] + h[t];
        msk[t] = 0u;
    }
    __syncwarp();
    const unsigned lt = lanemask_lt();
    const int lo = b * g.cap, hi = lo + g.cap;
    const int i0 = s * g.slab, i1 = min(i0 + g.slab, g.N);
    for (int g0 = i0; g0 < i1; g0 += 32 * kScatterSub) {
        int cx[kScatterSub], cy[kScatterSub];
        load_centres(g, gr, b, g0, i1, cx, cy);
#pragma unroll
        for (int j = 0; j < kScatterSub; ++j) {
            if (g0 + 32 * j >= i1) break;  // warp-uniform
            const int i = g0 + 32 * j + lane;  // past i1: no centre, no tiles
            int tx0, ty0, nx, ny;
            window_tiles(cx[j], cy[j], g, tx0, ty0, nx, ny);
            const int ht = nx ? home_tile(cx[j], cy[j], g) : -1;
            int tk[M * M];
#pragma unroll
            for (int dy = 0; dy < M; ++dy)
#pragma unroll
                for (int dx = 0; dx < M; ++dx) {
                    const int q = dy * M + dx;
                    tk[q] = (dx < nx && dy < ny) ? (ty0 + dy) * g.TX + tx0 + dx : -1;
                    if (tk[q] >= 0) atomicOr(&msk[tk[q]], 1u << lane);
                }
            __syncwarp();
            int nb[M * M];
#pragma unroll
            for (int q = 0; q < M * M; ++q) {
                nb[q] = -1;
                if (tk[q] < 0) continue;
                const unsigned m = msk[tk[q]];
                const int base = nxt[tk[q]];
                const int slot = base + __popc(m & lt);
                if (slot >= lo && slot < hi)
                    ids[slot] = (int)((unsigned)i | (tk[q] == ht ? kHomeFlag : 0u));
                else
                    atomicOr(err, kErrListBounds);
                if ((m & lt) == 0u) nb[q] = base + __popc(m);  // lowest lane of the tile
            }
            __syncwarp();
#pragma unroll
            for (int q = 0; q < M * M; ++q)
                if (nb[q] >= 0) {
                    nxt[tk[q]] = nb[q];
                    msk[tk[q]] = 0u;
                }
            __syncwarp();
        }
    }
}

// One block per frame: the whole binner of a small frame in one launch.
// Warp w owns the contiguous slab [w * S, (w + 1) * S) of the frame's
// Gaussians: it computes their records and counts them per tile; one block
// scan turns the per-tile totals into the tiles' list starts; then every
// warp scatters its slab with the lane-mask ranks described above.
__global__ void __launch_bounds__(1024) k_bin_frame(const float *__restrict__ params, Geom g,
                                                    float4 *__restrict__ gr,
                                                    int *__restrict__ offs,
                                                    int *__restrict__ ids,
                                                    int *__restrict__ err) {
    extern __shared__ unsigned fsm[];
    grid_dep_wait();
    grid_dep_release();
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

// Frames of at most kClusterBinMaxT tiles: one thread-block cluster of CS =
// min(T, 16) blocks per frame (grid (CS, B), cluster (CS, 1, 1)), block q
// owning the q-th chunk of the frame's Gaussians.  Each block computes its
// chunk's records and counts them per tile; the counts of all blocks are read
// through distributed shared memory, giving the tiles' list starts and this
// chunk's first slot in every tile (the counts of the chunks before it); the
// chunk is then scattered in rounds of kClusterBinThreads with the per-warp
// lane-mask ranks.  One launch, no counts in global memory.
constexpr int kClusterBinThreads = 256;
constexpr int kClusterBinMaxT = 64;    // most tiles per frame
constexpr int kClusterBinMaxCS = 16;   // most blocks per cluster (non-portable above 8)

__host__ __device__ constexpr int bin_cluster_size(int T) { return T < kClusterBinMaxCS ? T : kClusterBinMaxCS; }

__global__ void __launch_bounds__(kClusterBinThreads) k_bin_cluster(
    const float *__restrict__ params, Geom g, float4 *__restrict__ gr, int *__restrict__ offs,
    int *__restrict__ ids, int *__restrict__ err) {
    constexpr int NW = kClusterBinThreads / 32, MT = kClusterBinMaxT;
    __shared__ int cnt[MT];                          // this chunk's count per tile
    __shared__ int tab[kClusterBinMaxCS][MT];        // tab[r][t]: chunk r's count in tile t
    __shared__ int tstart[MT + 1];                   // frame-relative list start per tile
    __shared__ int base[MT];                         // next slot of this chunk per tile
    __shared__ unsigned masks[NW][MT];               // per-warp lane masks of a round
    grid_dep_wait();
    grid_dep_release();
    cg::cluster_group cluster = cg::this_cluster();
    const int T = g.T, CS = bin_cluster_size(T);
    const int q = (int)cluster.block_rank();
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    for (int t = tid; t < MT; t += kClusterBinThreads) cnt[t] = 0;
    for (int t = tid; t < NW * MT; t += kClusterBinThreads) masks[t / MT][t % MT] = 0u;
    __syncthreads();
    const int chunk = (g.N + CS - 1) / CS;
    const int i0 = min(q * chunk, g.N), i1 = min(i0 + chunk, g.N);
    for (int i = i0 + tid; i < i1; i += kClusterBinThreads) {
        const size_t gid = (size_t)b * g.N + i;
        float4 A, Q;
        gaussian_record(params + gid * g.P, A, Q);
        gr[2 * gid] = A;
        gr[2 * gid + 1] = Q;
        int tx0, ty0, nx, ny;
        window_tiles(__float_as_int(Q.z), __float_as_int(Q.w), g, tx0, ty0, nx, ny);
        for (int dy = 0; dy < ny; ++dy)
            for (int dx = 0; dx < nx; ++dx) atomicAdd(&cnt[(ty0 + dy) * g.TX + tx0 + dx], 1);
    }
    cluster.sync();  // every chunk's counts are final
    for (int j = tid; j < CS * T; j += kClusterBinThreads) {
        const int r = j / T, tt = j - r * T;
        tab[r][tt] = *cluster.map_shared_rank(cnt + tt, r);
    }
    cluster.sync();  // no block leaves while a peer may still read its counts
    if (warp == 0) {
        // Lane l takes tiles 2l and 2l + 1: their totals and the counts of the
        // chunks before this one; one warp scan over the pairs.
        int col[2] = {0, 0}, below[2] = {0, 0};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int tt = 2 * lane + h;
            if (tt < T)
                for (int r = 0; r < CS; ++r) {
                    const int v = tab[r][tt];
                    col[h] += v;
                    below[h] += r < q ? v : 0;
                }
        }
        const int pair = col[0] + col[1];
        int incl = pair;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += u;
        }
        const int ex0 = incl - pair, ex1 = ex0 + col[0];
        if (2 * lane < T) {
            tstart[2 * lane] = ex0;
            base[2 * lane] = ex0 + below[0];
        }
        if (2 * lane + 1 < T) {
            tstart[2 * lane + 1] = ex1;
            base[2 * lane + 1] = ex1 + below[1];
        }
        if (lane == 31) tstart[T] = incl;
    }
    __syncthreads();
    const int frame0 = b * g.cap;
    if (q == 0)
        for (int tt = tid; tt <= T; tt += kClusterBinThreads)
            offs[(size_t)b * (T + 1) + tt] = frame0 + tstart[tt];
    const int lo = frame0, hi = frame0 + g.cap;
    for (int s0 = i0; s0 < i1; s0 += kClusterBinThreads) {  // block-uniform rounds
        const int i = s0 + tid;
        int tx0 = 0, ty0 = 0, nx = 0, ny = 0, ht = -1;
        if (i < i1) {
            const float4 Q = gr[2 * ((size_t)b * g.N + i) + 1];
            const int cx = __float_as_int(Q.z), cy = __float_as_int(Q.w);
            window_tiles(cx, cy, g, tx0, ty0, nx, ny);
            if (nx) ht = home_tile(cx, cy, g);
        }
        for (int dy = 0; dy < ny; ++dy)
            for (int dx = 0; dx < nx; ++dx)
                atomicOr(&masks[warp][(ty0 + dy) * g.TX + tx0 + dx], 1u << lane);
        __syncthreads();
        for (int dy = 0; dy < ny; ++dy)
            for (int dx = 0; dx < nx; ++dx) {
                const int tt = (ty0 + dy) * g.TX + tx0 + dx;
                int pre = base[tt] + __popc(masks[warp][tt] & lt);
                for (int w = 0; w < warp; ++w) pre += __popc(masks[w][tt]);
                const int slot = frame0 + pre;
                if (slot >= lo && slot < hi)
                    ids[slot] = (int)((unsigned)i | (tt == ht ? kHomeFlag : 0u));
                else
                    atomicOr(err, kErrListBounds);
            }
        __syncthreads();
        for (int t = tid; t < T; t += kClusterBinThreads) {
            int add = 0;
            for (int w = 0; w < NW; ++w) add += __popc(masks[w][t]);
            base[t] += add;
        }
        __syncthreads();
        for (int t = tid; t < NW * MT; t += kClusterBinThreads) masks[t / MT][t % MT] = 0u;
        __syncthreads();
    }
}

__global__ void k_copy_ids(int *__restrict__ dst, const int *__restrict__ src, size_t n) {
    grid_dep_wait();
    grid_dep_release();
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

// k_slab_count: one count per tile; k_slab_scatter: the tiles' list starts,
// then a slot and a mask table per warp.
size_t bin_count_smem(const Geom &g) {
    const int ntab = g.slab < kSlabThreads ? kSlabThreads / g.slab : 1;
    return sizeof(int) * (size_t)g.T * ntab;
}

size_t bin_scatter_smem(const Geom &g) {
    return sizeof(int) * (size_t)g.T * (1 + 2 * (size_t)g.slab_warps);
}

// Dynamic shared memory above which a launch needs the opt-in attribute: the
// 48 KB default less room for the kernel's static arrays.
constexpr size_t kStaticSmemRoom = 44 * 1024;

template <typename K>
static cudaError_t allow_smem(K kernel, size_t bytes) {
    if (bytes <= kStaticSmemRoom) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// The clustered binner for these sizes can be scheduled on the current device
// (at least one cluster of min(T, 16) blocks fits); cached per device and T.
static bool bin_cluster_fits(const Geom &g) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    static std::mutex mu;
    static std::map<std::pair<int, int>, bool> known;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, g.T);
    const auto it = known.find(key);
    if (it != known.end()) return it->second;
    bool ok = true;
    const int CS = bin_cluster_size(g.T);
    if (CS > 8 && cudaFuncSetAttribute(k_bin_cluster, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                       1) != cudaSuccess) {
        cudaGetLastError();
        ok = false;
    }
    if (ok) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3(CS, 1, 1);
        cfg.blockDim = dim3(kClusterBinThreads, 1, 1);
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_bin_cluster, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        ok = n > 0;
    }
    known[key] = ok;
    return ok;
}

cudaError_t launch_bin(const float *params, const Geom &g, const Workspace &ws,
                       cudaStream_t s) {
    cudaError_t e;
    if (g.T <= kClusterBinMaxT && bin_cluster_fits(g)) {
        const int CS = bin_cluster_size(g.T);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3(CS, g.B, 1);
        cfg.blockDim = dim3(kClusterBinThreads, 1, 1);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_bin_cluster, params, g, ws.gr, ws.offs, ws.ids, ws.err);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    if (g.frame_block) {
        const size_t sf = bin_frame_smem(g);
        if ((e = allow_smem(k_bin_frame, sf)) != cudaSuccess) return e;
        k_bin_frame<<<g.B, g.frame_threads, sf, s>>>(params, g, ws.gr, ws.offs, ws.ids, ws.err);
        return cudaGetLastError();
    }
    const size_t sc = bin_count_smem(g), ss = bin_scatter_smem(g);
    if ((e = allow_smem(k_slab_count, sc)) != cudaSuccess) return e;
    const int span = g.slab > kSlabThreads ? g.slab : kSlabThreads;
    k_slab_count<<<dim3((g.N + span - 1) / span, g.B), kSlabThreads, sc, s>>>(params, g, ws.gr,
                                                                            ws.hist);
    if ((e = launch_dependent(k_slab_scan, dim3((g.T + 31) / 32, g.B), dim3(1024), 0, s, g,
                              ws.hist, ws.tot)) != cudaSuccess)
        return e;
    const dim3 grid((g.nslab + g.slab_warps - 1) / g.slab_warps, g.B);
    if (g.m <= 2) {
        if ((e = allow_smem(k_slab_scatter<2>, ss)) != cudaSuccess) return e;
        e = launch_dependent(k_slab_scatter<2>, grid, dim3(32 * g.slab_warps), ss, s, g,
                             (const float4 *)ws.gr, (const int *)ws.hist, (const int *)ws.tot,
                             ws.offs, ws.ids, ws.err);
        if (e != cudaSuccess) return e;
    } else {
        if ((e = allow_smem(k_slab_scatter<3>, ss)) != cudaSuccess) return e;
        e = launch_dependent(k_slab_scatter<3>, grid, dim3(32 * g.slab_warps), ss, s, g,
                             (const float4 *)ws.gr, (const int *)ws.hist, (const int *)ws.tot,
                             ws.offs, ws.ids, ws.err);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace pdr
