// Forward tile kernels: I_c(p) = sum_i a_ic * 2^{-(uhat_1^2 + uhat_2^2)} over
// the Gaussians whose k x k window contains p (paper abstract: 5 + C
// parameters, arbitrary C; reading notes, "Method": additive accumulation).
//
// A block renders one 16x16 tile.  The tile is cut into sixteen 4x4 regions,
// one per group of 16 / PL lanes; a lane owns PL pixels of one row of its
// region and keeps all C channels of them in registers (PL = 4: 64-thread
// blocks for large grids; PL = 2: 128-thread blocks, shorter per-lane work,
// for small grids).  Per batch of the tile's entries (ascending id):
//   1. stage: each entry's record is rebased to the tile origin
//      (uhat_j = alpha_j x + beta_j y + K_j in tile-local pixels), with the
//      window as a 16-bit column mask and a 16-bit row mask;
//   2. sub-lists: each warp compacts, in entry order, the entries whose
//      window meets each of its regions, with the 16-bit mask of the region's
//      pixels inside the window (ballot + popcount);
//   3. evaluate: every group walks only its own sub-list; a lane evaluates
//      its pixels from one rebased record (PL = 4: |uhat|^2 of its run as the
//      quadratic about the run's centre; PL = 2: stepping uhat along the row).
// The per-pixel sum order is the list order: fixed, so results are bitwise
// reproducible.
//
// k_fwd reads the tile lists the binner left in the workspace.  For frames of
// at most kClusterTiles tiles, k_fwd_cluster bins and renders in one launch:
// one thread-block cluster per frame, block q owning tile q and the q-th
// chunk of the frame's Gaussians.  Each block counts its chunk per tile; the
// counts are exchanged through distributed shared memory; each block writes
// its chunk's entries (stable ranks, as in the binner) into the global list
// for the backward pass and straight into the list of the owning block's
// shared memory; then every block renders its tile from its own list.
#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace pdr {

namespace {

constexpr int kFwdBatch = 64;          // entries staged per batch by k_fwd (byte offsets fit 16 bits)
constexpr int kClusterBatch = 128;     // ... and by k_fwd_cluster (fewer batch barriers)
constexpr int kClusterListCap = 1024;  // tile-list entries a clustered block keeps on chip
constexpr int kChunkSmem = 256;        // Gaussians per clustered block whose records stay on chip

template <int C>
struct FwdRec {
    static constexpr int kFloats = 6 + C;
    static constexpr int kVec = (kFloats + 3) / 4;  // float4 per record
};

template <int PL>
struct FwdLayout {
    static constexpr int kThreads = 256 / PL;          // one lane per PL pixels of the tile
    static constexpr int kLanes = 16 / PL;             // lanes per 4x4 region
};

// Shared-memory buffers of one rendering block.
template <int C, int NB>
struct FwdSmem {
    float4 rec[NB * FwdRec<C>::kVec];
    unsigned win[NB];  // window as column bits | row bits << 16 (tile pixels)
    unsigned sub[16][NB];
    int subn[16];
};

// Render the entries list[0 .. L) (frame-local ids, ascending) of the tile at
// (X0, Y0) of frame b into acc.  Called by the whole block.
// fetch(i, A, Q, amp) supplies the record and amplitudes of frame-local
// Gaussian i (from global memory, or from a cluster peer's shared memory).
template <int C, int PL, int NB, typename Fetch>
__device__ __forceinline__ void render_list(const Geom &g, Fetch fetch, const int *list,
                                            int L, int X0, int Y0, int *err,
                                            FwdSmem<C, NB> &S, float (&acc)[PL][C]) {
    using LY = FwdLayout<PL>;
    constexpr int RV = FwdRec<C>::kVec;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = tid / LY::kLanes, lig = tid % LY::kLanes;
    const int gx = grp & 3, gy = grp >> 2;
    const int lrow = lig / (4 / PL), lcol = (lig % (4 / PL)) * PL;  // lane's row / first column
    const float fx = (float)(4 * gx + lcol), fy = (float)(4 * gy + lrow);
    const int bitshift = 16 + 4 * lrow + lcol;  // this lane's bits of a packed sub-list entry

    const unsigned lt = lanemask_lt();
    static_assert(NB * FwdRec<C>::kVec * 16 <= 65536, "record offsets must fit 16 bits");
    // PL = 4: |uhat|^2 over the lane's run of 4 pixels as the quadratic about
    // the run's centre x_c = x + 1.5: with U = uhat(x_c), D = U . d uhat/dx and
    // Qc = |d uhat / dx|^2, the pixel at x_c + o has |uhat|^2 = |U|^2 + 2 o D + o^2 Qc,
    // o = +-0.5, +-1.5 (two operations per pixel instead of four; every term is
    // bounded by the expansion at the run's centre).  Qc rides in the record's
    // padding when it has a free float.
    constexpr bool kQcRec = 6 + C < RV * 4;
    const float fxc = fx + 0.5f * (float)(PL - 1);
    for (int e0 = 0; e0 < L; e0 += NB) {
        const int n = min(NB, L - e0);
        __syncthreads();  // the previous batch is fully consumed
        for (int e = tid; e < n; e += LY::kThreads) {
            const int i = entry_id(list[e0 + e]);
            if (i >= g.N) {  // never for consistent bins
                atomicOr(err, kErrBadId);
                S.win[e] = 0u;
                continue;
            }
            float4 A, Q;
            float amp[C];
            fetch(i, A, Q, amp);
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
#pragma unroll
            for (int c = 0; c < C; ++c) r[6 + c] = amp[c];
#pragma unroll
            for (int c = 6 + C; c < RV * 4; ++c) r[c] = 0.0f;
            if constexpr (kQcRec) r[6 + C] = fmaf(A.z, A.z, Q.x * Q.x);  // |d uhat / dx|^2
#pragma unroll
            for (int v = 0; v < RV; ++v)
                S.rec[e * RV + v] = make_float4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            // An entry whose window misses the tile (only possible with stale
            // bins) contributes nothing.
            S.win[e] = (lx0 <= lx1 && ly0 <= ly1) ? (cm & 0xffffu) | ((rm & 0xffffu) << 16) : 0u;
        }
        __syncthreads();
        {
            // Sub-lists of this warp's regions (region rows ROWS * warp ..).
            constexpr int RPW = 32 / LY::kLanes;  // regions per warp
            constexpr int ROWS = RPW / 4;         // region rows per warp
            int cnt[RPW];
#pragma unroll
            for (int q = 0; q < RPW; ++q) cnt[q] = 0;
            const int nr = (n + 31) & ~31;
            for (int e = lane; e < nr; e += 32) {
                const unsigned wm = e < n ? S.win[e] : 0u;
#pragma unroll
                for (int h = 0; h < ROWS; ++h) {
                    const int row = ROWS * warp + h;
                    const unsigned rb = (wm >> (16 + 4 * row)) & 0xfu;
                    unsigned rs = (rb & 1u) | ((rb & 2u) << 3) | ((rb & 4u) << 6) | ((rb & 8u) << 9);
                    rs *= 0xfu;  // one full nibble per window row of the region
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const unsigned cb = (wm >> (4 * q)) & 0xfu;
                        const unsigned pm = (cb * 0x1111u) & rs;
                        const unsigned bal = __ballot_sync(0xffffffffu, pm != 0u);
                        if (pm)  // pixel mask | byte offset of the entry's record
                            S.sub[4 * row + q][cnt[4 * h + q] + __popc(bal & lt)] =
                                (pm << 16) | (unsigned)(e * RV * 16);
                        cnt[4 * h + q] += __popc(bal);
                    }
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int q = 0; q < RPW; ++q) S.subn[RPW * warp + q] = cnt[q];
            }
        }
        __syncthreads();
        const int ns = S.subn[grp];
        const unsigned *sl = S.sub[grp];
        for (int s = 0; s < ns; ++s) {
            const unsigned pk = sl[s];
            const float4 *r4 = reinterpret_cast<const float4 *>(
                reinterpret_cast<const char *>(S.rec) + (pk & 0xffffu));
            float rr[RV * 4];
#pragma unroll
            for (int v = 0; v < RV; ++v) {
                const float4 q = r4[v];
                rr[4 * v] = q.x; rr[4 * v + 1] = q.y; rr[4 * v + 2] = q.z; rr[4 * v + 3] = q.w;
            }
            const unsigned bits = pk >> bitshift;
            if constexpr (PL == 4) {
                const float u1 = fmaf(rr[0], fxc, fmaf(rr[1], fy, rr[2]));
                const float u2 = fmaf(rr[3], fxc, fmaf(rr[4], fy, rr[5]));
                const float qc = fmaf(u1, u1, u2 * u2);
                const float D = fmaf(u1, rr[0], u2 * rr[3]);
                float Qc;
                if constexpr (kQcRec)
                    Qc = rr[6 + C];
                else
                    Qc = fmaf(rr[0], rr[0], rr[3] * rr[3]);
                const float s = fmaf(0.25f, Qc, qc), t = fmaf(2.25f, Qc, qc);
                const float q[4] = {fmaf(-3.0f, D, t), s - D, s + D, fmaf(3.0f, D, t)};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float w = ex2(-q[j]);
                    if (bits & (1u << j)) {
#pragma unroll
                        for (int c = 0; c < C; ++c) acc[j][c] = fmaf(rr[6 + c], w, acc[j][c]);
                    }
                }
            } else {
                float u1 = fmaf(rr[0], fx, fmaf(rr[1], fy, rr[2]));
                float u2 = fmaf(rr[3], fx, fmaf(rr[4], fy, rr[5]));
#pragma unroll
                for (int j = 0; j < PL; ++j) {
                    if (j) {
                        u1 += rr[0];
                        u2 += rr[3];
                    }
                    const float w = ex2(fmaf(-u1, u1, -u2 * u2));
                    if (bits & (1u << j)) {
#pragma unroll
                        for (int c = 0; c < C; ++c) acc[j][c] = fmaf(rr[6 + c], w, acc[j][c]);
                    }
                }
            }
        }
    }
}

template <int C, int PL>
__device__ __forceinline__ void store_tile(const Geom &g, int b, int X0, int Y0,
                                           void *__restrict__ image_, const float (&acc)[PL][C]) {
    using LY = FwdLayout<PL>;
    const int tid = threadIdx.x;
    const int grp = tid / LY::kLanes, lig = tid % LY::kLanes;
    const int lrow = lig / (4 / PL), lcol = (lig % (4 / PL)) * PL;
    const int x = X0 + 4 * (grp & 3) + lcol, y = Y0 + 4 * (grp >> 2) + lrow;
    if (y >= g.H) return;
    if (g.img_dtype != 0) {  // fp16 / bf16 storage: fp32 sums, rounded to nearest once
        const bool hvec = (x + PL - 1 < g.W) && (PL == 4 ? g.out_vec4 : g.out_vec2);
#pragma unroll
        for (int c = 0; c < C; ++c) {
            const size_t o = (((size_t)b * C + c) * g.H + y) * g.W + x;
            if (hvec) {
                unsigned short hb[PL];
#pragma unroll
                for (int j = 0; j < PL; ++j) hb[j] = half_bits(acc[j][c], g.img_dtype);
                unsigned short *dst = static_cast<unsigned short *>(image_) + o;
                if constexpr (PL == 4)
                    *reinterpret_cast<uint2 *>(dst) = make_uint2(hb[0] | ((unsigned)hb[1] << 16),
                                                                 hb[2] | ((unsigned)hb[3] << 16));
                else
                    *reinterpret_cast<unsigned *>(dst) = hb[0] | ((unsigned)hb[1] << 16);
            } else {
#pragma unroll
                for (int j = 0; j < PL; ++j)
                    if (x + j < g.W) img_store(image_, o + j, g.img_dtype, acc[j][c]);
            }
        }
        return;
    }
    float *image = static_cast<float *>(image_);
    const bool vec = (x + PL - 1 < g.W) && (PL == 4 ? g.out_vec4 : g.out_vec2);
#pragma unroll
    for (int c = 0; c < C; ++c) {
        float *dst = image + (((size_t)b * C + c) * g.H + y) * g.W + x;
        if (vec) {
            if constexpr (PL == 4)
                *reinterpret_cast<float4 *>(dst) = make_float4(acc[0][c], acc[1][c], acc[2][c], acc[3][c]);
            else
                *reinterpret_cast<float2 *>(dst) = make_float2(acc[0][c], acc[1][c]);
        } else {
#pragma unroll
            for (int j = 0; j < PL; ++j)
                if (x + j < g.W) dst[j] = acc[j][c];
        }
    }
}

template <int C, int PL>
__global__ void __launch_bounds__(FwdLayout<PL>::kThreads) k_fwd(const float *__restrict__ params,
                                                                 Geom g,
                                                                 const float4 *__restrict__ gr,
                                                                 const int *__restrict__ offs,
                                                                 const int *__restrict__ ids,
                                                                 void *__restrict__ image,
                                                                 int *__restrict__ err) {
    __shared__ FwdSmem<C, kFwdBatch> S;
    grid_dep_wait();
    grid_dep_release();
    const int b = blockIdx.x / g.T, t = blockIdx.x - b * g.T;
    const int ty = t / g.TX, tx = t - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    float acc[PL][C];
#pragma unroll
    for (int j = 0; j < PL; ++j)
#pragma unroll
        for (int c = 0; c < C; ++c) acc[j][c] = 0.0f;
    int L0, L1;
    list_range(offs, g, b, t, err, L0, L1);
    auto fetch = [&](int i, float4 &A, float4 &Q, float (&amp)[C]) {
        const size_t gid = (size_t)b * g.N + i;
        A = gr[2 * gid];
        Q = gr[2 * gid + 1];
        const float *pa = params + gid * g.P + 5;
#pragma unroll
        for (int c = 0; c < C; ++c) amp[c] = pa[c];
    };
    render_list<C, PL, kFwdBatch>(g, fetch, ids + L0, L1 - L0, X0, Y0, err, S, acc);
    store_tile<C, PL>(g, b, X0, Y0, image, acc);
}

// Bins and renders one small frame per thread-block cluster (grid (T, B),
// cluster (T, 1, 1)); block q = tile q owns the Gaussians [q * chunk, ...).
template <int C, int PL>
__global__ void __launch_bounds__(FwdLayout<PL>::kThreads) k_fwd_cluster(
    const float *__restrict__ params, Geom g, float4 *__restrict__ gr, int *__restrict__ offs,
    int *__restrict__ ids, void *__restrict__ image, int *__restrict__ err) {
    constexpr int NT = FwdLayout<PL>::kThreads;
    constexpr int NW = NT / 32;
    __shared__ FwdSmem<C, kClusterBatch> S;
    grid_dep_wait();
    grid_dep_release();
    __shared__ int cnt[kClusterTiles];                 // this chunk's count per tile
    __shared__ int tab[kClusterTiles][kClusterTiles];  // tab[r][t] = count of chunk r in tile t
    __shared__ int base[kClusterTiles];                // next list slot of this chunk, per tile
    __shared__ int tstart[kClusterTiles + 1];          // frame's tile offsets (relative)
    __shared__ unsigned masks[NW][kClusterTiles];
    __shared__ int list[kClusterListCap];              // this tile's entries, filled by the cluster
    __shared__ float4 crec[kChunkSmem][2];             // this chunk's records (read by the cluster)
    __shared__ float camp[kChunkSmem][C];              // and amplitudes

    cg::cluster_group cluster = cg::this_cluster();
    const int T = g.T;
    const int q = (int)cluster.block_rank();  // == tile index
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    if (tid < kClusterTiles) cnt[tid] = 0;
    if (tid < NW * kClusterTiles) masks[tid / kClusterTiles][tid % kClusterTiles] = 0u;
    __syncthreads();

    // 1. records and per-tile counts of this block's chunk
    const int chunk = (g.N + T - 1) / T;
    const bool onchip = chunk <= kChunkSmem;  // same for every block of the cluster
    const int i0 = min(q * chunk, g.N), i1 = min(i0 + chunk, g.N);
    for (int i = i0 + tid; i < i1; i += NT) {
        const size_t gid = (size_t)b * g.N + i;
        float4 A, Q;
        gaussian_record(params + gid * g.P, A, Q);
        gr[2 * gid] = A;
        gr[2 * gid + 1] = Q;
        if (onchip) {
            crec[i - i0][0] = A;
            crec[i - i0][1] = Q;
            const float *pa = params + gid * g.P + 5;
#pragma unroll
            for (int c = 0; c < C; ++c) camp[i - i0][c] = pa[c];
        }
        int x0, x1, y0, y1;
        if (window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
            for (int yy = y0 >> 4; yy <= (y1 >> 4); ++yy)
                for (int xx = x0 >> 4; xx <= (x1 >> 4); ++xx) atomicAdd(&cnt[yy * g.TX + xx], 1);
        }
    }
    cluster.sync();

    // 2. every block reads all chunks' counts (distributed shared memory)
    for (int j = tid; j < T * T; j += NT) {
        const int r = j / T, tt = j - r * T;
        tab[r][tt] = *cluster.map_shared_rank(cnt + tt, r);
    }
    __syncthreads();
    if (warp == 0) {  // tile offsets: lane tt sums column tt, then a warp scan over tiles
        int col = 0, below = 0;
        if (lane < T) {
            for (int r = 0; r < T; ++r) {
                const int v = tab[r][lane];
                col += v;
                below += r < q ? v : 0;
            }
        }
        int incl = col;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += u;
        }
        if (lane < T) {
            tstart[lane] = incl - col;
            base[lane] = incl - col + below;
        }
        if (lane == T - 1) tstart[T] = incl;
    }
    __syncthreads();
    const int frame0 = b * g.cap;
    if (q == 0)
        for (int tt = tid; tt <= T; tt += NT) offs[(size_t)b * (T + 1) + tt] = frame0 + tstart[tt];

    // 3. stable scatter of this chunk: global list + the owning block's list
    const long long lo = frame0, hi = lo + g.cap;
    for (int s = i0; s < i1; s += NT) {
        const int i = s + tid;
        int tx0 = 1, tx1 = 0, ty0 = 1, ty1 = 0;
        int ht = -1;  // home tile
        if (i < i1) {
            const float4 Q = gr[2 * ((size_t)b * g.N + i) + 1];
            int x0, x1, y0, y1;
            if (window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
                tx0 = x0 >> 4; tx1 = x1 >> 4; ty0 = y0 >> 4; ty1 = y1 >> 4;
                ht = home_tile(__float_as_int(Q.z), __float_as_int(Q.w), g);
            }
        }
        for (int yy = ty0; yy <= ty1; ++yy)
            for (int xx = tx0; xx <= tx1; ++xx) atomicOr(&masks[warp][yy * g.TX + xx], 1u << lane);
        __syncthreads();
        for (int yy = ty0; yy <= ty1; ++yy)
            for (int xx = tx0; xx <= tx1; ++xx) {
                const int tt = yy * g.TX + xx;
                int pre = base[tt] + __popc(masks[warp][tt] & lt);
                for (int w = 0; w < warp; ++w) pre += __popc(masks[w][tt]);
                const long long slot = (long long)frame0 + pre;
                if (slot >= lo && slot < hi) {
                    ids[slot] = (int)((unsigned)i | (tt == ht ? kHomeFlag : 0u));
                    const int local = pre - tstart[tt];
                    if (local < kClusterListCap) *cluster.map_shared_rank(list + local, tt) = i;
                } else {
                    atomicOr(err, kErrListBounds);
                }
            }
        __syncthreads();
        if (tid < T) {
            int add = 0;
            for (int w = 0; w < NW; ++w) add += __popc(masks[w][tid]);
            base[tid] += add;
        }
        __syncthreads();
        if (tid < NW * kClusterTiles) masks[tid / kClusterTiles][tid % kClusterTiles] = 0u;
        __syncthreads();
    }
    cluster.sync();  // every list is complete; only the records are read across blocks after this

    // 4. render this tile from its own list
    const int ty = q / g.TX, tx = q - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    float acc[PL][C];
#pragma unroll
    for (int j = 0; j < PL; ++j)
#pragma unroll
        for (int c = 0; c < C; ++c) acc[j][c] = 0.0f;
    const int L = tstart[q + 1] - tstart[q];
    const int *src = L <= kClusterListCap ? list : ids + frame0 + tstart[q];
    if (onchip) {
        // Records from the chunk owners' shared memory (distributed shared memory).
        auto fetch = [&](int i, float4 &A, float4 &Q, float (&amp)[C]) {
            const int r = i / chunk, li = i - r * chunk;
            const float4 *pr = cluster.map_shared_rank(&crec[li][0], r);
            const float *pa = cluster.map_shared_rank(&camp[li][0], r);
            A = pr[0];
            Q = pr[1];
#pragma unroll
            for (int c = 0; c < C; ++c) amp[c] = pa[c];
        };
        render_list<C, PL, kClusterBatch>(g, fetch, src, L, X0, Y0, err, S, acc);
    } else {
        auto fetch = [&](int i, float4 &A, float4 &Q, float (&amp)[C]) {
            const size_t gid = (size_t)b * g.N + i;
            A = gr[2 * gid];
            Q = gr[2 * gid + 1];
            const float *pa = params + gid * g.P + 5;
#pragma unroll
            for (int c = 0; c < C; ++c) amp[c] = pa[c];
        };
        render_list<C, PL, kClusterBatch>(g, fetch, src, L, X0, Y0, err, S, acc);
    }
    store_tile<C, PL>(g, b, X0, Y0, image, acc);
    if (onchip) cluster.sync();  // peers may still read this block's records
}

template <int C, int PL>
cudaError_t launch_fwd_cluster(const float *params, const Geom &g, const Workspace &ws,
                               void *image, cudaStream_t s) {
        cudaError_t e;
        if (g.T > 8) {
            e = cudaFuncSetAttribute(k_fwd_cluster<C, PL>,
                                     cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3(g.T, g.B, 1);
        cfg.blockDim = dim3(FwdLayout<PL>::kThreads, 1, 1);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = g.T;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_fwd_cluster<C, PL>, params, g, ws.gr, ws.offs, ws.ids,
                               image, ws.err);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
}

// At least one cluster of g.T blocks of k_fwd_cluster<C, PL> fits on the
// current device (a cluster of more than 8 blocks needs the non-portable size).
template <int C, int PL>
bool cluster_fits(const Geom &g) {
    if (g.T > 8 && cudaFuncSetAttribute(k_fwd_cluster<C, PL>,
                                        cudaFuncAttributeNonPortableClusterSizeAllowed,
                                        1) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(g.T, 1, 1);
    cfg.blockDim = dim3(FwdLayout<PL>::kThreads, 1, 1);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g.T;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_fwd_cluster<C, PL>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return n > 0;
}

template <int C>
bool cluster_fits_c(const Geom &g) {
    return g.fwd_pl == 2 ? cluster_fits<C, 2>(g) : cluster_fits<C, 4>(g);
}

template <int C>
cudaError_t launch_fwd_c(const float *params, const Geom &g, const Workspace &ws, void *image,
                         cudaStream_t s, bool bin_inside) {
    if (bin_inside)
        return g.fwd_pl == 2 ? launch_fwd_cluster<C, 2>(params, g, ws, image, s)
                             : launch_fwd_cluster<C, 4>(params, g, ws, image, s);
    const cudaError_t e =
        g.fwd_pl == 2
            ? launch_dependent(k_fwd<C, 2>, dim3(g.B * g.T), dim3(FwdLayout<2>::kThreads), 0, s,
                               params, g, (const float4 *)ws.gr, (const int *)ws.offs,
                               (const int *)ws.ids, image, ws.err)
            : launch_dependent(k_fwd<C, 4>, dim3(g.B * g.T), dim3(FwdLayout<4>::kThreads), 0, s,
                               params, g, (const float4 *)ws.gr, (const int *)ws.offs,
                               (const int *)ws.ids, image, ws.err);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

bool fwd_cluster_schedulable(const Geom &g) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int>, bool> known;  // (device, C, PL, T)
    const auto key = std::make_tuple(dev, g.C, g.fwd_pl, g.T);
    std::lock_guard<std::mutex> lock(mu);
    const auto it = known.find(key);
    if (it != known.end()) return it->second;
    bool ok = false;
    switch (g.C) {
        case 1: ok = cluster_fits_c<1>(g); break;
        case 2: ok = cluster_fits_c<2>(g); break;
        case 3: ok = cluster_fits_c<3>(g); break;
        case 4: ok = cluster_fits_c<4>(g); break;
        case 5: ok = cluster_fits_c<5>(g); break;
        case 6: ok = cluster_fits_c<6>(g); break;
        case 7: ok = cluster_fits_c<7>(g); break;
        case 8: ok = cluster_fits_c<8>(g); break;
        default: ok = false;
    }
    known[key] = ok;
    return ok;
}

cudaError_t launch_fwd(const float *params, const Geom &g, const Workspace &ws, void *image,
                       cudaStream_t s, bool bin_inside) {
    switch (g.C) {
        case 1: return launch_fwd_c<1>(params, g, ws, image, s, bin_inside);
        case 2: return launch_fwd_c<2>(params, g, ws, image, s, bin_inside);
        case 3: return launch_fwd_c<3>(params, g, ws, image, s, bin_inside);
        case 4: return launch_fwd_c<4>(params, g, ws, image, s, bin_inside);
        case 5: return launch_fwd_c<5>(params, g, ws, image, s, bin_inside);
        case 6: return launch_fwd_c<6>(params, g, ws, image, s, bin_inside);
        case 7: return launch_fwd_c<7>(params, g, ws, image, s, bin_inside);
        case 8: return launch_fwd_c<8>(params, g, ws, image, s, bin_inside);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pdr
