// Backward kernels: dL/d(mu, s, theta, a) from dL/dI (paper abstract: a
// "differentiable" renderer; the forward is the additive accumulation of the
// reading notes, "Method").
//
// With uhat = sqrt(kappa) diag(e^{-s}) R^T (p - mu)  (kappa = log2(e) / 2),
// w = 2^{-|uhat|^2} = exp(-q / 2), G = sum_c g_c a_c and v = w G, the whole
// gradient of one Gaussian follows from seven sums over its window:
//     S1 = sum v uhat_1,  S2 = sum v uhat_2,
//     S11 = sum v uhat_1^2,  S12 = sum v uhat_1 uhat_2,  S22 = sum v uhat_2^2,
//     DA_c = sum g_c w,
// as  dL/dmu_x = 2 ln2 (alpha_1 S1 + alpha_2 S2),  dL/dmu_y = 2 ln2 (beta_1 S1 + beta_2 S2),
//     dL/ds_j = 2 ln2 S_jj,  dL/dtheta = 2 ln2 * 2 sinh(s_1 - s_2) * S12,  dL/da_c = DA_c
// (uhat_j = alpha_j dx + beta_j dy; dL/duhat_j = -2 ln2 v uhat_j).
//
// Work decomposition ("home tile"): a Gaussian is processed exactly once, by
// the block of the tile that contains its clamped window centre, over its
// full k x k window; dL/dI is staged once per tile in shared memory with a
// zero-padded halo, so pixels outside the grid contribute exactly zero and
// the inner loop needs no bounds tests.  A block finds its Gaussians from the
// ids of its tile list alone: the binner flags the one entry of each Gaussian
// that lies in its home tile's list, so the block reads its list contiguously,
// compacts the flagged entries in list order (ballots and a prefix over the
// warps), and only then gathers the records of those Gaussians into shared
// memory, each prepared once (window origin, offset into the staged halo,
// 2 ln2 * 2 sinh(s1 - s2), amplitudes).  Eight lanes share one Gaussian; for
// k = 7 .. 15 (C <= 4) a lane walks window columns and forms their share of
// the five uhat sums from three row moments per column (see the pixel-pair
// section).  The chain rule, linear in the sums, is applied by each lane to
// its own partial sums, which are then combined with a fixed xor-shuffle tree
// (a segmented reduction with segments of 8 lanes), so no per-pixel atomics
// and no partial-gradient buffer are needed.  Every sum has a fixed order.  Block sizes (NT) are template parameters: 128-thread
// blocks keep the last round of a tile's Gaussians short when a tile holds
// few of them.
#include "common.cuh"

namespace pdr {

namespace {

constexpr int kGroup = 8;   // lanes per Gaussian

// Home record staged in shared memory (float4 units):
//   [0] = (alpha_1, beta_1, K_1, alpha_2)   K_j = uhat_j at the window corner
//   [1] = (beta_2, K_2, 2 ln2 * 2 sinh(s_1 - s_2), id bits; -1: bad id)
//   [2] = (kernel-specific offsets into the staged halo, as int bits)
//   [3..] = amplitudes a_0 .. a_{C-1} (zero padded)
template <int C>
struct HRec {
    static constexpr int RV = 3 + (C + 3) / 4;
};

// Channels of dL/dI stored per shared-memory pixel (padded to a vector width).
template <int C> struct GPix { static constexpr int n = C <= 1 ? 1 : C <= 2 ? 2 : C <= 4 ? 4 : 8; };

// Row pitch (pixels) of the staged region: at least RS, congruent to k mod 8.
__host__ __device__ __forceinline__ int staged_pitch(int RS, int k) {
    return RS + (((k - RS) % 8) + 8) % 8;
}

// List entries each thread holds per pass (a pass is KP * NT entries).
constexpr int kPer = 2;

// One pass of a tile list: entry e0 + j * NT + tid (j < KP) is held by thread
// tid as raw[j] (the binner's entry with its home flag) when valid[j].
// Returns each entry's rank among the pass's home entries in list order (-1
// if it is not a home entry) and their total.  Called by the whole block;
// wcnt holds KP * NT / 32 ints (consecutive passes alternate between two such
// areas, so that no thread can overwrite counts another thread of the
// previous pass is still reading).
template <int NT, int KP>
__device__ __forceinline__ void home_ranks(const int (&raw)[KP], const bool (&valid)[KP],
                                           int *wcnt, int (&pos)[KP], int &total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = lanemask_lt();
#pragma unroll
    for (int j = 0; j < KP; ++j) {
        const bool h = valid[j] && entry_home(raw[j]);
        const unsigned bal = __ballot_sync(0xffffffffu, h);
        pos[j] = h ? (int)__popc(bal & lt) : -1;
        if (lane == 0) wcnt[j * NW + warp] = __popc(bal);
    }
    __syncthreads();
    // List order is (j, warp, lane): add the counts of every earlier (j, warp).
    int before[KP];
#pragma unroll
    for (int j = 0; j < KP; ++j) before[j] = 0;
    total = 0;
#pragma unroll
    for (int q = 0; q < KP * NW; ++q) {
        const int c = wcnt[q];
#pragma unroll
        for (int j = 0; j < KP; ++j) before[j] += q < j * NW + warp ? c : 0;
        total += c;
    }
#pragma unroll
    for (int j = 0; j < KP; ++j)
        if (pos[j] >= 0) pos[j] += before[j];
}

// The ids of pass 0 of a tile list, requested by the caller before its
// halo staging so that both are in flight together.
template <int NT, int KP>
__device__ __forceinline__ void load_pass(const int *__restrict__ ids, int e0, int L1,
                                          int (&raw)[KP], bool (&valid)[KP]) {
#pragma unroll
    for (int j = 0; j < KP; ++j) {
        const int e = e0 + j * NT + (int)threadIdx.x;
        valid[j] = e < L1;
        raw[j] = valid[j] ? ids[e] : 0;
    }
}

// Walks the tile list [L0, L1) in passes of KP * NT entries (pass 0 already
// in raw / valid), ranks each pass's home entries in list order and gathers
// all their records in one round of loads (make(raw entry, slot) writes the
// record of slot `slot`), calling process(n) on the staged records whenever
// the record area (rcap) is full and once at the end.  Called by the whole
// block; the staging done before it is visible to process.
template <int NT, int KP, typename Make, typename Process>
__device__ __forceinline__ void gather_homes(const int *__restrict__ ids, int L0, int L1,
                                             int rcap, int *wcnt2, int (&raw)[KP],
                                             bool (&valid)[KP], Make make, Process process) {
    constexpr int W = KP * NT / 32;
    int nh = 0, pass = 0;
    for (int e0 = L0; e0 < L1; e0 += KP * NT, ++pass) {
        if (e0 != L0) load_pass<NT, KP>(ids, e0, L1, raw, valid);
        int pos[KP], tot;
        home_ranks<NT, KP>(raw, valid, wcnt2 + (pass & 1) * W, pos, tot);
        for (int done = 0; done < tot;) {  // block-uniform
            if (nh == rcap) {
                __syncthreads();  // the staged records visible
                process(nh);
                __syncthreads();  // records consumed before they are overwritten
                nh = 0;
            }
            const int take = min(tot - done, rcap - nh);
#pragma unroll
            for (int j = 0; j < KP; ++j)
                if (pos[j] >= done && pos[j] < done + take) make(raw[j], nh + pos[j] - done);
            nh += take;
            done += take;
        }
    }
    __syncthreads();  // the last records (and the staging) visible
    process(nh);
}

// The part of a home record that both kernels share: rows 0, 1 and the
// amplitudes.  id < 0 marks an entry that is not a Gaussian of the frame.
template <int C>
__device__ __forceinline__ void home_record_common(const float *__restrict__ params,
                                                   const float4 *__restrict__ gr, const Geom &g,
                                                   int b, int id, int &cx, int &cy,
                                                   float4 *R) {
    constexpr int RV = HRec<C>::RV;
    const size_t gid = (size_t)b * g.N + id;
    const float4 A = gr[2 * gid], Q = gr[2 * gid + 1];
    const float *pp = params + gid * g.P;
    float amp[4 * (RV - 3)];
#pragma unroll
    for (int c = 0; c < 4 * (RV - 3); ++c) amp[c] = c < C ? pp[5 + c] : 0.0f;
    const float s1 = pp[2], s2 = pp[3];
    cx = __float_as_int(Q.z);
    cy = __float_as_int(Q.w);
    const float a1 = A.z, b1 = A.w, a2 = Q.x, b2 = Q.y;
    const float dx0 = (float)(cx - g.r) - A.x, dy0 = (float)(cy - g.r) - A.y;
    const float K1 = fmaf(a1, dx0, b1 * dy0), K2 = fmaf(a2, dx0, b2 * dy0);
    // 2 sinh(s1 - s2) = e^{d} - e^{-d}, via the base-2 exponential.
    const float dl = (s1 - s2) * 1.44269504088896340736f;
    R[0] = make_float4(a1, b1, K1, a2);
    R[1] = make_float4(b2, K2, kTwoLn2 * (ex2(dl) - ex2(-dl)), __int_as_float(id));
#pragma unroll
    for (int v = 0; v < RV - 3; ++v)
        R[3 + v] = make_float4(amp[4 * v], amp[4 * v + 1], amp[4 * v + 2], amp[4 * v + 3]);
}

// Gaussians whose window misses the grid (or whose mean is not finite)
// appear in no list: the block of tile t zeroes a slice of its frame's.
__device__ __forceinline__ void zero_missing(const float4 *__restrict__ gr, const Geom &g, int b,
                                             int t, float *__restrict__ dparams) {
    const int per = (g.N + g.T - 1) / g.T;
    const int i0 = t * per, i1 = min(i0 + per, g.N);
    for (int i = i0 + (int)threadIdx.x; i < i1; i += blockDim.x) {
        const size_t gid = (size_t)b * g.N + i;
        const float4 Q = gr[2 * gid + 1];
        int x0, x1, y0, y1;
        if (!window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
            float *d = dparams + gid * g.P;
            for (int j = 0; j < g.P; ++j) d[j] = 0.0f;
        }
    }
}

// The group's partial sums -> lane j of the group holds gradient component j
// (j < 8, summed over the group in a fixed order), written with one store per
// lane; components 8.. (C > 3) go through a plain tree to the group leader.
template <int C>
struct Extra { static constexpr int n = C > 3 ? C - 3 : 1; };  // components 8 .. 4 + C

template <int C>
__device__ __forceinline__ void group_write(float (&v)[8], const float (&extra)[Extra<C>::n],
                                            unsigned gmask, int lig, float *__restrict__ d) {
    constexpr int NV = 5 + C;
    const bool h2 = lig & 4, h1 = lig & 2, h0 = lig & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = h2 ? v[i] : v[i + 4], keep = h2 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(gmask, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = h1 ? v[i] : v[i + 2], keep = h1 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(gmask, send, 2);
    }
    {
        const float send = h0 ? v[0] : v[1], keep = h0 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(gmask, send, 1);
    }
    if (lig < NV) d[lig] = v[0];
#pragma unroll
    for (int j = 8; j < NV; ++j) {
        float e = extra[j - 8];
#pragma unroll
        for (int dd = 1; dd < kGroup; dd <<= 1) e += __shfl_xor_sync(gmask, e, dd);
        if (lig == 0) d[j] = e;
    }
}

template <int C>
__device__ __forceinline__ void load_gpix(const float *gh, int pix, float (&gv)[C]) {
    constexpr int GP = GPix<C>::n;
    if constexpr (GP == 1) {
        gv[0] = gh[pix];
    } else if constexpr (GP == 2) {
        const float2 v = reinterpret_cast<const float2 *>(gh)[pix];
        gv[0] = v.x;
        if constexpr (C > 1) gv[1] = v.y;
    } else if constexpr (GP == 4) {
        const float4 v = reinterpret_cast<const float4 *>(gh)[pix];
        const float t[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < C; ++c) gv[c] = t[c];
    } else {
        const float4 v0 = reinterpret_cast<const float4 *>(gh)[2 * pix];
        const float4 v1 = reinterpret_cast<const float4 *>(gh)[2 * pix + 1];
        const float t[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int c = 0; c < C; ++c) gv[c] = t[c];
    }
}

// ---------------------------------------------------------------------------
// Scalar backward (any C, any k; common k compiled in).  Eight lanes share a
// Gaussian's k*k window.  For k = 7, 9, 11 (compiled in, C <= 4) lane l walks
// window column l (l < min(k, 8)) and forms the column's share of the five
// sums from its row moments, as the pixel-pair kernel does (see there); the
// pixels of columns 8 .. k - 1 are dealt to the lanes in row-major order from
// a per-block offset table.  For every other k the lanes stride over all the
// window's pixels that way (lane l takes pixels l, l + 8, ...).  dL/dI is staged over
// [X0 - 2r, X0 + 15 + 2r]^2, zero outside the core [X0 - r, X0 + 15 + r]^2
// and outside the grid: the core holds the whole window of every home
// Gaussian centred on the grid, and the outer ring is only read by home
// Gaussians centred off the grid (a border tile's), at pixels that are
// themselves off the grid, so every home Gaussian reads shared memory only.
// The staged rows have a pitch congruent to k modulo 8, so the 8 pixels the
// lanes of a group read together fall in 8 distinct 16-byte bank groups even
// across a row wrap.
// ---------------------------------------------------------------------------
template <int C, int KT, int NT>
__global__ void __launch_bounds__(NT, C > 4 ? 1 : 1024 / NT) k_bwd(const float *__restrict__ params,
                                            const void *__restrict__ gimg, Geom g,
                                            const float4 *__restrict__ gr,
                                            const int *__restrict__ offs,
                                            const int *__restrict__ ids,
                                            float *__restrict__ dparams,
                                            int *__restrict__ err) {
    grid_dep_wait();
    grid_dep_release();
    constexpr int GP = GPix<C>::n;
    constexpr int NV = 5 + C;
    constexpr int RV = HRec<C>::RV;
    constexpr int NG = NT / kGroup;
    extern __shared__ float4 smem4[];
    __shared__ int wcnt[2 * kPer * NT / 32];
    const int k = KT ? KT : g.k, r = (k - 1) / 2;
    const int RS = kTile + 4 * r;                 // staged region edge (pixels)
    const int RP = staged_pitch(RS, k);           // its row pitch
    const int kk = k * k;
    const int full = kk / kGroup, tail = kk - full * kGroup;  // compile-time when KT > 0
    const int rcap = g.bwd_rcap;                  // home records staged at most
    float4 *table = smem4;                        // [(full + 1) * 8]: (ox, oy, offset, 0)
    float4 *recs = table + (full + 1) * kGroup;   // [rcap][RV]
    float *gh = reinterpret_cast<float *>(recs + (size_t)rcap * RV);  // [RS*RP][GP]
    {
        // The launch must have provided this layout; otherwise report, touch nothing.
        const unsigned need = (unsigned)(sizeof(float4) * ((full + 1) * kGroup + rcap * RV) +
                                         sizeof(float) * RS * RP * GP);
        if (dynamic_smem_bytes() < need || rcap < NT) {
            if (threadIdx.x == 0) atomicOr(err, kErrSmemLayout);
            return;
        }
    }

    const int b = blockIdx.x / g.T, t = blockIdx.x - b * g.T;
    const int ty = t / g.TX, tx = t - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    const int RX0 = X0 - 2 * r, RY0 = Y0 - 2 * r;  // staged region origin (grid coordinates)
    const int tid = threadIdx.x;
    const int grp = tid / kGroup, lig = tid % kGroup;
    // Groups of one warp may run different numbers of Gaussians, so the
    // group's reduction names only its own lanes.
    const unsigned gmask = ((1u << kGroup) - 1u) << (kGroup * (grp % (32 / kGroup)));

    int L0, L1;
    list_range(offs, g, b, t, err, L0, L1);
    // The first pass's entries, requested before the staging loads so that
    // both are in flight together.
    int raw[kPer];
    bool valid[kPer];
    load_pass<NT, kPer>(ids, L0, L1, raw, valid);

    zero_missing(gr, g, b, t, dparams);

    // Window enumeration table: lane l of a group takes window pixels
    // l, l + 8, l + 16, ... in row-major order -- with column moments, only
    // the pixels of columns 8 .. k - 1 (XW wide), the others being walked by
    // column.
    constexpr bool kCols = KT >= 7 && KT <= 11;
    constexpr int XW = kCols ? (KT > kGroup ? KT - kGroup : 0) : 0;
    const int tabn = kCols ? XW * k : kk;  // pixels enumerated by the table
    const int tfull = tabn / kGroup, ttail = tabn - tfull * kGroup;
    for (int j = tid; j < (tfull + 1) * kGroup; j += NT) {
        const int p = j < tabn ? j : 0;
        const int ox = kCols ? kGroup + p % (XW > 0 ? XW : 1) : p % k;
        const int oy = kCols ? p / (XW > 0 ? XW : 1) : p / k;
        table[j] = make_float4((float)ox, (float)oy, __int_as_float(oy * RP + ox), 0.0f);
    }
    // dL/dI of the core (zero outside it and outside the grid).
    constexpr int kStageU = 4;  // pixels per thread with their loads in flight together
    for (int p0 = 0; p0 < RS * RS; p0 += kStageU * NT) {
        float v[kStageU][GP];
#pragma unroll
        for (int u = 0; u < kStageU; ++u) {
            const int pix = p0 + u * NT + tid;
            const int ry = pix / RS, rx = pix - ry * RS;
            const int x = RX0 + rx, y = RY0 + ry;
            const bool core = rx >= r && rx < RS - r && ry >= r && ry < RS - r;
            const bool in = pix < RS * RS && core && x >= 0 && x < g.W && y >= 0 && y < g.H;
#pragma unroll
            for (int c = 0; c < GP; ++c)
                v[u][c] = (in && c < C) ? img_load(gimg, (((size_t)b * C + c) * g.H + y) * g.W + x, g.img_dtype) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kStageU; ++u) {
            const int pix = p0 + u * NT + tid;
            if (pix >= RS * RS) continue;
            const int ry = pix / RS, rx = pix - ry * RS;
            const int spix = ry * RP + rx;
            if constexpr (GP == 1) {
                gh[spix] = v[u][0];
            } else if constexpr (GP == 2) {
                reinterpret_cast<float2 *>(gh)[spix] = make_float2(v[u][0], v[u][1]);
            } else if constexpr (GP == 4) {
                reinterpret_cast<float4 *>(gh)[spix] = make_float4(v[u][0], v[u][1], v[u][2], v[u][3]);
            } else {
                reinterpret_cast<float4 *>(gh)[2 * spix] = make_float4(v[u][0], v[u][1], v[u][2], v[u][3]);
                reinterpret_cast<float4 *>(gh)[2 * spix + 1] = make_float4(v[u][4], v[u][5], v[u][6], v[u][7]);
            }
        }
    }

    // The staged home Gaussians recs[0 .. n), one per group at a time.
    auto process = [&](int n) {
        for (int h = grp; h < n; h += NG) {
            const float4 *R = recs + h * RV;
            const float4 r0 = R[0], r1 = R[1], r2 = R[2];
            const int id = __float_as_int(r1.w);
            if (id < 0) continue;
            const float a1 = r0.x, b1 = r0.y, K1 = r0.z, a2 = r0.w, b2 = r1.x, K2 = r1.y;
            float amp[4 * (RV - 3)];
#pragma unroll
            for (int v = 0; v < RV - 3; ++v) {
                const float4 q = R[3 + v];
                amp[4 * v] = q.x; amp[4 * v + 1] = q.y; amp[4 * v + 2] = q.z; amp[4 * v + 3] = q.w;
            }
            float acc[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) acc[j] = 0.0f;

            auto pixel = [&](float ox, float oy, const float (&gv)[C]) {
                const float u1 = fmaf(a1, ox, fmaf(b1, oy, K1));
                const float u2 = fmaf(a2, ox, fmaf(b2, oy, K2));
                const float w = ex2(fmaf(-u1, u1, -u2 * u2));
                float G = gv[0] * amp[0];
#pragma unroll
                for (int c = 1; c < C; ++c) G = fmaf(gv[c], amp[c], G);
                const float v = w * G;
#pragma unroll
                for (int c = 0; c < C; ++c) acc[5 + c] = fmaf(gv[c], w, acc[5 + c]);
                const float vu1 = v * u1, vu2 = v * u2;
                acc[0] += vu1;
                acc[1] += vu2;
                acc[2] = fmaf(vu1, u1, acc[2]);
                acc[3] = fmaf(vu1, u2, acc[3]);
                acc[4] = fmaf(vu2, u2, acc[4]);
            };
            const float *gb = gh + __float_as_int(r2.x);
            auto eval = [&](int j) {
                const float4 tb = table[j * kGroup + lig];
                float gv[C];
                load_gpix<C>(gb, __float_as_int(tb.z), gv);
                pixel(tb.x, tb.y, gv);
            };
            if constexpr (kCols) {
                // Columns 8 .. k - 1 pixel by pixel, then lane l walks window
                // column l (l < min(k, 8)) by row moments: with jc = row - r and
                // U = uhat at the column's pixel of the centre row,
                // uhat = U + jc (beta_1, beta_2), |uhat|^2 = Qa + jc (Qb + jc Qc),
                // and the five sums follow from M0 = sum v, MY = sum jc v,
                // MYY = sum jc^2 v (S_j = U_j M0 + beta_j MY,
                // S_jl = U_l (U_j M0 + beta_j MY) + beta_l (U_j MY + beta_j MYY)).
                if constexpr (XW > 0) {
#pragma unroll
                    for (int j = 0; j < tfull; ++j) eval(j);
                    if (lig < ttail) eval(tfull);
                }
                constexpr int KC = KT < kGroup ? KT : kGroup;
                constexpr int RR = (KT - 1) / 2;
                if (KC == kGroup || lig < KC) {
                    const float ox = (float)lig;
                    const float U1 = fmaf(a1, ox, fmaf(b1, (float)RR, K1));
                    const float U2 = fmaf(a2, ox, fmaf(b2, (float)RR, K2));
                    const float Qa = fmaf(U1, U1, U2 * U2);
                    const float Qb = 2.0f * fmaf(U1, b1, U2 * b2);
                    const float Qc = fmaf(b1, b1, b2 * b2);
                    float M0 = 0.0f, MY = 0.0f, MYY = 0.0f;
                    const float *gcol = gb + lig * GP;
#pragma unroll
                    for (int j = 0; j < KT; ++j) {
                        const int jc = j - RR;
                        float gv[C];
                        load_gpix<C>(gcol, j * RP, gv);
                        const float q = jc == 0 ? Qa : fmaf(fmaf(Qc, (float)jc, Qb), (float)jc, Qa);
                        const float w = ex2(-q);
                        float G = gv[0] * amp[0];
#pragma unroll
                        for (int c = 1; c < C; ++c) G = fmaf(gv[c], amp[c], G);
#pragma unroll
                        for (int c = 0; c < C; ++c) acc[5 + c] = fmaf(gv[c], w, acc[5 + c]);
                        const float v = w * G;
                        M0 += v;
                        if (jc != 0) {
                            MY = fmaf(v, (float)jc, MY);
                            MYY = fmaf(v, (float)(jc * jc), MYY);
                        }
                    }
                    const float t1 = fmaf(b1, MY, U1 * M0), t2 = fmaf(b2, MY, U2 * M0);
                    const float q1 = fmaf(b1, MYY, U1 * MY), q2 = fmaf(b2, MYY, U2 * MY);
                    acc[0] += t1;
                    acc[1] += t2;
                    acc[2] += fmaf(b1, q1, U1 * t1);
                    acc[3] += fmaf(b2, q1, U2 * t1);
                    acc[4] += fmaf(b2, q2, U2 * t2);
                }
            } else if constexpr (KT > 0) {
#pragma unroll 8
                for (int j = 0; j < full; ++j) eval(j);
                if (lig < tail) eval(full);
            } else {
                for (int j = 0; j < full; ++j) eval(j);
                if (lig < tail) eval(full);
            }

            // The chain rule is linear in the sums, so each lane applies it to
            // its own partial sums before the group reduction.
            float v[8];
            v[0] = kTwoLn2 * fmaf(a1, acc[0], a2 * acc[1]);  // dL/dmu_x
            v[1] = kTwoLn2 * fmaf(b1, acc[0], b2 * acc[1]);  // dL/dmu_y
            v[2] = kTwoLn2 * acc[2];                         // dL/ds_1
            v[3] = kTwoLn2 * acc[4];                         // dL/ds_2
            v[4] = r1.z * acc[3];                            // dL/dtheta
#pragma unroll
            for (int j = 5; j < 8; ++j) v[j] = j < NV ? acc[j < NV ? j : 0] : 0.0f;
            float extra[Extra<C>::n];
#pragma unroll
            for (int j = 0; j < Extra<C>::n; ++j) extra[j] = 8 + j < NV ? acc[8 + j < NV ? 8 + j : 0] : 0.0f;
            group_write<C>(v, extra, gmask, lig, dparams + ((size_t)b * g.N + id) * g.P);
        }
    };

    auto make = [&](int rawe, int slot) {
        const int id = entry_id(rawe);
        if (id >= g.N) {  // never for consistent bins
            atomicOr(err, kErrBadId);
            recs[slot * RV + 1] = make_float4(0.0f, 0.0f, 0.0f, __int_as_float(-1));
            return;
        }
        float4 R[RV];
        int cx, cy;
        home_record_common<C>(params, gr, g, b, id, cx, cy, R);
        const int wx0 = cx - r, wy0 = cy - r;  // inside the staged region
        R[2] = make_float4(__int_as_float(((wy0 - RY0) * RP + (wx0 - RX0)) * GP), 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int v = 0; v < RV; ++v) recs[slot * RV + v] = R[v];
    };
    gather_homes<NT, kPer>(ids, L0, L1, rcap, wcnt, raw, valid, make, process);
}

// ---------------------------------------------------------------------------
// Pixel-pair backward (C <= 4, k in {13, 15} compiled in).  Same home-tile
// decomposition and the same seven sums per Gaussian as k_bwd, but every
// lane works on two horizontally adjacent pixels at once with the packed
// f32x2 arithmetic of sm_100 (one instruction issues two FP32 FMAs), which
// halves the issue slots of the inner loop.
//
// A window row of k pixels (k odd) is covered by (k + 1) / 2 pairs, one of
// whose pixels lies just outside the window and is masked (its weight is
// 2^-inf = 0).  dL/dI is staged once, in pairs that start at even x: a window
// that starts at even x takes its pairs from its first pixel and masks the
// pixel after its last; one that starts at odd x takes them from the pixel
// before its first, which it masks.  Two channels of a pair share one float4
// (c lo, c hi, c+1 lo, c+1 hi) and an odd last channel has a float2 plane of
// its own, so one vector load per two channels yields the packed operands
// directly.  Lane l of a group takes pair column l of every window row
// (k = 13 leaves lane 7 idle).
//
// Per lane, the sums are formed from three row moments of its column: with
// jc = row - r and U = uhat at the column's pixel of the window's centre row,
// uhat = U + jc (beta_1, beta_2) along the column, so |uhat|^2 is the
// quadratic Qa + jc (Qb + jc Qc) in jc, and S1, S2, S11, S12, S22 follow
// exactly (up to rounding) from M0 = sum v, MY = sum jc v, MYY = sum jc^2 v:
//   S_j  = U_j M0 + beta_j MY,
//   S_jl = U_l (U_j M0 + beta_j MY) + beta_l (U_j MY + beta_j MYY).
// That takes three accumulations per pixel instead of seven.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2dup(float a) { return make_float2(a, a); }

template <int C, int K, int NT>
struct PairShape {
    static constexpr int R = (K - 1) / 2;
    static constexpr int NPW = (K + 1) / 2;                  // pairs per window row
    static constexpr int SLOTS = NPW * K;                    // pair slots per window
    static constexpr int NP4 = C / 2;                        // float4 planes (two channels each)
    static constexpr int NP2 = C & 1;                        // float2 plane (the odd channel)
    // Staged rows Y0 - r - 1 .. Y0 + 16 + r and columns X0 - 8 .. X0 + 23:
    // every pair read by the window of a home Gaussian whose centre lies in
    // [X0 - 1, X0 + 16] x [Y0 - 1, Y0 + 16] (on the grid, or one pixel off
    // it).  Its pairs start at x0 = cx - r or, x0 being odd, at x0 - 1 (X0 is
    // even): at X0 - 8 or later for r <= 7, and its last pair ends at
    // X0 + 17 + r - (r & 1) <= X0 + 23.
    static constexpr int ROWS = kTile + 2 * R + 2;
    static constexpr int XOFF = 8;
    static constexpr int PAIRS = kTile / 2 + XOFF;           // staged pairs per row
    static constexpr int PITCH = PAIRS;
    static constexpr int PLANE = ROWS * PITCH;               // elements per plane
    static constexpr int NIT = ROWS * PAIRS;                 // staging items
    static constexpr int RV = HRec<C>::RV;
    static constexpr size_t HALO4 = sizeof(float4) * NP4 * PLANE;
    static constexpr size_t HALO2 = sizeof(float2) * NP2 * PLANE;
    static_assert(R < XOFF, "window apron within the staged columns");
    // Dynamic shared memory for a record capacity of rcap home Gaussians.
    __host__ __device__ static constexpr size_t smem(int rcap) { return HALO4 + HALO2 + sizeof(float4) * RV * rcap; }
};

// Stages dL/dI of the pair kernels' region, rows [Y0 - r - 1, Y0 + 16 + r]
// and the pairs of columns X0 - 8 .. X0 + 23, zero outside [X0 - r, X0 + 15 + r]
// and outside the grid, for rows of a multiple of 4 elements and an image
// aligned to 4 elements: item (row, j) loads the aligned 4 elements from
// X0 - 8 + 4j of every channel (one vector load each: a float4, or 8 bytes of
// fp16 / bf16 widened to fp32; guarded scalar loads where it crosses the
// grid's edge) and writes staged pairs 2j and 2j + 1.
template <int C, int K, int NT, bool HALF>
__device__ __forceinline__ void stage_pairs_vec4(const void *__restrict__ gimg, const Geom &g,
                                                 int b, int X0, int Y0, float4 *halo4,
                                                 float2 *halo2) {
    using S = PairShape<C, K, NT>;
    constexpr int R = S::R, NP4 = S::NP4, NP2 = S::NP2;
    constexpr int NJ = S::PAIRS / 2;  // float4 columns per row
    constexpr int NCH = 2 * NP4 + NP2;
    for (int it = (int)threadIdx.x; it < S::ROWS * NJ; it += NT) {
        const int row = it / NJ, j = it - row * NJ;
        const int y = Y0 - R - 1 + row;
        const int x4 = X0 - S::XOFF + 4 * j;
        float v[NCH][4];
        const bool rowin = y >= 0 && y < g.H;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            v[c][0] = v[c][1] = v[c][2] = v[c][3] = 0.0f;
            if (rowin) {
                const size_t row0 = (((size_t)b * C + c) * g.H + y) * g.W;
                if (x4 >= 0 && x4 + 3 < g.W) {
                    if constexpr (!HALF) {
                        const float4 q = *reinterpret_cast<const float4 *>(static_cast<const float *>(gimg) + row0 + x4);
                        v[c][0] = q.x; v[c][1] = q.y; v[c][2] = q.z; v[c][3] = q.w;
                    } else {
                        const uint2 q = *reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(gimg) + row0 + x4);
                        const unsigned hw[4] = {q.x & 0xffffu, q.x >> 16, q.y & 0xffffu, q.y >> 16};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            v[c][e] = g.img_dtype == 1  // fp16, else bf16
                                          ? __half2float(__ushort_as_half((unsigned short)hw[e]))
                                          : __bfloat162float(__ushort_as_bfloat16((unsigned short)hw[e]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (x4 + e >= 0 && x4 + e < g.W) v[c][e] = img_load(gimg, row0 + x4 + e, g.img_dtype);
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (x4 + e < X0 - R || x4 + e > X0 + kTile - 1 + R) v[c][e] = 0.0f;
        }
        const int el = row * S::PITCH + 2 * j;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int pl = 0; pl < NP4; ++pl)
                halo4[pl * S::PLANE + el + h] = make_float4(v[2 * pl][2 * h], v[2 * pl][2 * h + 1],
                                                            v[2 * pl + 1][2 * h], v[2 * pl + 1][2 * h + 1]);
            if constexpr (NP2) halo2[el + h] = make_float2(v[C - 1][2 * h], v[C - 1][2 * h + 1]);
        }
    }
}

template <int C, int K, int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) k_bwd_pairs(const float *__restrict__ params,
                                                  const void *__restrict__ gimg, Geom g,
                                                  const float4 *__restrict__ gr,
                                                  const int *__restrict__ offs,
                                                  const int *__restrict__ ids,
                                                  float *__restrict__ dparams,
                                                  int *__restrict__ err) {
    grid_dep_wait();
    grid_dep_release();
    using S = PairShape<C, K, NT>;
    constexpr int R = S::R, NPW = S::NPW, NP4 = S::NP4, NP2 = S::NP2;
    constexpr int RV = S::RV, NG = NT / kGroup;
    constexpr int NCH = 2 * NP4 + NP2;  // channels staged per pixel (C, rounded to the planes)
    extern __shared__ float4 smem4[];
    __shared__ int wcnt[2 * kPer * NT / 32];
    const int rcap = g.bwd_rcap;  // home records staged at most
    float4 *halo4 = smem4;                                                // [NP4][ROWS][PITCH]
    float2 *halo2 = reinterpret_cast<float2 *>(smem4 + NP4 * S::PLANE);  // [ROWS][PITCH]
    float4 *recs = smem4 + (S::HALO4 + S::HALO2) / sizeof(float4);       // [rcap][RV]
    static_assert(S::HALO2 % sizeof(float4) == 0, "record area must stay 16-byte aligned");
    if (dynamic_smem_bytes() < (unsigned)S::smem(rcap) || g.k != K || rcap < NT) {
        if (threadIdx.x == 0) atomicOr(err, kErrSmemLayout);  // launch/layout mismatch
        return;
    }

    const int b = blockIdx.x / g.T, t = blockIdx.x - b * g.T;
    const int ty = t / g.TX, tx = t - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    const int SX0 = X0 - S::XOFF, RY0 = Y0 - R - 1;  // staged region origin (grid coordinates)
    const int tid = threadIdx.x;
    const int grp = tid / kGroup, lig = tid % kGroup;
    const unsigned gmask = ((1u << kGroup) - 1u) << (kGroup * (grp % (32 / kGroup)));

    int L0, L1;
    list_range(offs, g, b, t, err, L0, L1);
    // The first pass's entries, requested before the staging loads so that
    // both are in flight together.
    int raw[kPer];
    bool valid[kPer];
    load_pass<NT, kPer>(ids, L0, L1, raw, valid);

    if (g.stage_vec4) {
        if (g.img_dtype == 0)
            stage_pairs_vec4<C, K, NT, false>(gimg, g, b, X0, Y0, halo4, halo2);
        else
            stage_pairs_vec4<C, K, NT, true>(gimg, g, b, X0, Y0, halo4, halo2);
    } else {
        // The same region element by element: item (row, m) holds pixels
        // SX0 + 2m and SX0 + 2m + 1 (zero outside [X0 - r, X0 + 15 + r] and
        // outside the grid).  Two items per thread have their loads in
        // flight together.
        constexpr int SU = 2;
        for (int i0 = 0; i0 < S::NIT; i0 += SU * NT) {
            float v[SU][2][NCH];
#pragma unroll
            for (int u = 0; u < SU; ++u) {
                const int it = i0 + u * NT + tid;
                const int row = it / S::PAIRS, m = it - row * S::PAIRS;
                const int y = RY0 + row;
                const bool rowin = it < S::NIT && y >= 0 && y < g.H;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int x = SX0 + 2 * m + q;
                    const bool in = rowin && x >= 0 && x < g.W && x >= X0 - R && x <= X0 + kTile - 1 + R;
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
                        v[u][q][c] = (in && c < C) ? img_load(gimg, (((size_t)b * C + c) * g.H + y) * g.W + x, g.img_dtype) : 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < SU; ++u) {
                const int it = i0 + u * NT + tid;
                if (it >= S::NIT) continue;
                const int row = it / S::PAIRS, m = it - row * S::PAIRS;
                const int el = row * S::PITCH + m;
#pragma unroll
                for (int pl = 0; pl < NP4; ++pl)
                    halo4[pl * S::PLANE + el] = make_float4(v[u][0][2 * pl], v[u][1][2 * pl],
                                                            v[u][0][2 * pl + 1], v[u][1][2 * pl + 1]);
                if constexpr (NP2) halo2[el] = make_float2(v[u][0][C - 1], v[u][1][C - 1]);
            }
        }
    }

    zero_missing(gr, g, b, t, dparams);

    // This lane's pair column (independent of the Gaussian).  A lane walks
    // every row of its column; with all 8 lanes active (k = 15) no lane idles
    // and the test is a compile-time constant.
    constexpr bool kAllOn = NPW == kGroup;
    static_assert(NPW <= kGroup, "one pair column per lane");
    const bool lane_on = kAllOn || lig < NPW;
    const int pc = lig % NPW;
    const float kInf = __int_as_float(0x7f800000);  // 2^-inf = 0: a masked pixel

    // The staged home Gaussians recs[0 .. n), one per group at a time.
    auto process = [&](int n) {
        for (int h = grp; h < n; h += NG) {
            const float4 *Rh = recs + h * RV;
            const float4 q0 = Rh[0], q1 = Rh[1], q2 = Rh[2];
            const int id = __float_as_int(q1.w);
            if (id < 0) continue;
            const float2 A1 = f2dup(q0.x), B1 = f2dup(q0.y), K1 = f2dup(q0.z);
            const float2 A2 = f2dup(q0.w), B2 = f2dup(q1.x), K2 = f2dup(q1.y);
            float2 AMP[C];
            {
                const float4 P = Rh[3];
                AMP[0] = f2dup(P.x);
                if constexpr (C > 1) AMP[1] = f2dup(P.y);
                if constexpr (C > 2) AMP[2] = f2dup(P.z);
                if constexpr (C > 3) AMP[3] = f2dup(P.w);
            }
            const float2 z2 = make_float2(0.0f, 0.0f);
            float2 S1 = z2, S2 = z2, S11 = z2, S12 = z2, S22 = z2, DA[C];
#pragma unroll
            for (int c = 0; c < C; ++c) DA[c] = z2;

            // One pair slot: u = uhat of the two pixels, q = |uhat|^2 (+inf
            // on a masked pixel), w = 2^-q, gc = dL/dI of the pair.
            auto slot = [&](float2 u1, float2 u2, float mhi, const float2 (&gc)[C]) {
                float2 q = f2fma(u1, u1, f2mul(u2, u2));
                q.y += mhi;
                const float2 w = make_float2(ex2(-q.x), ex2(-q.y));
                float2 G = f2mul(gc[0], AMP[0]);
#pragma unroll
                for (int c = 1; c < C; ++c) G = f2fma(gc[c], AMP[c], G);
#pragma unroll
                for (int c = 0; c < C; ++c) DA[c] = f2fma(gc[c], w, DA[c]);
                const float2 v = f2mul(w, G);
                const float2 vu1 = f2mul(v, u1), vu2 = f2mul(v, u2);
                S1 = f2add(S1, vu1);
                S2 = f2add(S2, vu2);
                S11 = f2fma(vu1, u1, S11);
                S12 = f2fma(vu1, u2, S12);
                S22 = f2fma(vu2, u2, S22);
            };

            const bool staged = __float_as_int(q2.w) != 0;
            if (staged && lane_on) {
                // Row moments of the lane's column (see the section comment).
                // par = 1: the window starts at odd x and its pairs one pixel
                // before it, so the pixel offsets of the lane's pair are
                // 2 pc - 1 and 2 pc, and lane 0's first pixel is masked;
                // par = 0: offsets 2 pc and 2 pc + 1, the last lane's second
                // pixel masked.
                const int el = __float_as_int(q2.x), par = __float_as_int(q2.y);
                const float4 *hp4 = halo4 + el + pc;
                const float2 *hp2 = halo2 + el + pc;
                const float2 sfx = make_float2((float)(2 * pc - par), (float)(2 * pc + 1 - par));
                const float2 U1 = f2fma(A1, sfx, f2fma(B1, f2dup((float)R), K1));
                const float2 U2 = f2fma(A2, sfx, f2fma(B2, f2dup((float)R), K2));
                float2 Qa = f2fma(U1, U1, f2mul(U2, U2));
                if (par) {
                    if (pc == 0) Qa.x = kInf;
                } else if (pc == NPW - 1) {
                    Qa.y = kInf;
                }
                const float2 Qb = f2mul(f2dup(2.0f), f2fma(U1, B1, f2mul(U2, B2)));
                const float2 Qc = f2dup(fmaf(q0.y, q0.y, q1.x * q1.x));
                float2 M0 = z2, MY = z2, MYY = z2;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int jc = j - R;
                    const float2 JC = f2dup((float)jc);
                    float2 gc[C];
#pragma unroll
                    for (int pl = 0; pl < NP4; ++pl) {
                        const float4 P = hp4[j * S::PITCH + pl * S::PLANE];
                        gc[2 * pl] = make_float2(P.x, P.y);
                        gc[2 * pl + 1] = make_float2(P.z, P.w);
                    }
                    if constexpr (NP2) gc[C - 1] = hp2[j * S::PITCH];
                    const float2 q = jc == 0 ? Qa : f2fma(f2fma(Qc, JC, Qb), JC, Qa);
                    const float2 w = make_float2(ex2(-q.x), ex2(-q.y));
                    float2 G = f2mul(gc[0], AMP[0]);
#pragma unroll
                    for (int c = 1; c < C; ++c) G = f2fma(gc[c], AMP[c], G);
#pragma unroll
                    for (int c = 0; c < C; ++c) DA[c] = f2fma(gc[c], w, DA[c]);
                    const float2 v = f2mul(w, G);
                    M0 = f2add(M0, v);
                    if (jc != 0) {
                        MY = f2fma(v, JC, MY);
                        MYY = f2fma(v, f2dup((float)(jc * jc)), MYY);
                    }
                }
                const float2 t1 = f2fma(B1, MY, f2mul(U1, M0));   // sum v uhat_1
                const float2 t2 = f2fma(B2, MY, f2mul(U2, M0));   // sum v uhat_2
                const float2 r1 = f2fma(B1, MYY, f2mul(U1, MY));  // sum v jc uhat_1
                const float2 r2 = f2fma(B2, MYY, f2mul(U2, MY));  // sum v jc uhat_2
                S1 = t1;
                S2 = t2;
                S11 = f2fma(B1, r1, f2mul(U1, t1));
                S12 = f2fma(B2, r1, f2mul(U2, t1));
                S22 = f2fma(B2, r2, f2mul(U2, t2));
            } else if (!staged) {
                // Centred more than one pixel off the grid: read dL/dI from
                // global memory, zero outside the grid (rare).
                const int wx0 = __float_as_int(q2.x), wy0 = __float_as_int(q2.y);
                for (int sl = lig; sl < S::SLOTS; sl += kGroup) {
                    const int row = sl / NPW, pcs = sl - row * NPW;
                    const int x = wx0 + 2 * pcs, y = wy0 + row;
                    const float2 fx = make_float2((float)(2 * pcs), (float)(2 * pcs + 1));
                    const float2 fy = f2dup((float)row);
                    const float2 u1 = f2fma(A1, fx, f2fma(B1, fy, K1));
                    const float2 u2 = f2fma(A2, fx, f2fma(B2, fy, K2));
                    float2 gc[C];
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        float lo = 0.0f, hi = 0.0f;
                        if (y >= 0 && y < g.H) {
                            const size_t rowo = (((size_t)b * C + c) * g.H + y) * g.W;
                            if (x >= 0 && x < g.W) lo = img_load(gimg, rowo + x, g.img_dtype);
                            if (x + 1 >= 0 && x + 1 < g.W && pcs < NPW - 1)
                                hi = img_load(gimg, rowo + x + 1, g.img_dtype);
                        }
                        gc[c] = make_float2(lo, hi);
                    }
                    slot(u1, u2, pcs == NPW - 1 ? __int_as_float(0x7f800000) : 0.0f, gc);
                }
            }

            // The chain rule is linear in the sums, so each lane applies it to
            // its own partial sums before the group reduction.
            float v[8];
            {
                const float s1 = S1.x + S1.y, s2 = S2.x + S2.y;
                v[0] = kTwoLn2 * fmaf(q0.x, s1, q0.w * s2);  // dL/dmu_x
                v[1] = kTwoLn2 * fmaf(q0.y, s1, q1.x * s2);  // dL/dmu_y
                v[2] = kTwoLn2 * (S11.x + S11.y);             // dL/ds_1
                v[3] = kTwoLn2 * (S22.x + S22.y);             // dL/ds_2
                v[4] = q1.z * (S12.x + S12.y);                // dL/dtheta
#pragma unroll
                for (int j = 5; j < 8; ++j) v[j] = j - 5 < C ? DA[j - 5 < C ? j - 5 : 0].x + DA[j - 5 < C ? j - 5 : 0].y : 0.0f;
            }
            float extra[Extra<C>::n] = {C > 3 ? DA[C > 3 ? 3 : 0].x + DA[C > 3 ? 3 : 0].y : 0.0f};
            group_write<C>(v, extra, gmask, lig, dparams + ((size_t)b * g.N + id) * g.P);
        }
    };

    auto make = [&](int rawe, int slot) {
        const int id = entry_id(rawe);
        if (id >= g.N) {  // never for consistent bins
            atomicOr(err, kErrBadId);
            recs[slot * RV + 1] = make_float4(0.0f, 0.0f, 0.0f, __int_as_float(-1));
            return;
        }
        float4 Rr[RV];
        int cx, cy;
        home_record_common<C>(params, gr, g, b, id, cx, cy, Rr);
        const int wx0 = cx - R, wy0 = cy - R;
        // Centred on the grid or at most one pixel off it: the window lies in
        // the staged region (its off-grid pixels are staged as zero).
        const bool staged = cx >= -1 && cx <= g.W && cy >= -1 && cy <= g.H;
        const int par = wx0 & 1;
        const int el = (wy0 - RY0) * S::PITCH + ((wx0 - par - SX0) >> 1);  // first staged pair
        Rr[2] = staged ? make_float4(__int_as_float(el), __int_as_float(par), 0.0f, __int_as_float(1))
                       : make_float4(__int_as_float(wx0), __int_as_float(wy0), 0.0f,
                                     __int_as_float(0));
#pragma unroll
        for (int v = 0; v < RV; ++v) recs[slot * RV + v] = Rr[v];
    };
    gather_homes<NT, kPer>(ids, L0, L1, rcap, wcnt, raw, valid, make, process);
}

template <int C, int K, int NT>
cudaError_t launch_bwd_pairs(const float *params, const void *grad_image, const Geom &g,
                             const Workspace &ws, float *grad_params, cudaStream_t s) {
    const size_t smem = PairShape<C, K, NT>::smem(g.bwd_rcap);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_bwd_pairs<C, K, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const cudaError_t e = launch_dependent(k_bwd_pairs<C, K, NT>, dim3(g.B * g.T), dim3(NT), smem,
                                           s, params, grad_image, g, (const float4 *)ws.gr,
                                           (const int *)ws.offs, (const int *)ws.ids,
                                           grad_params, ws.err);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int C, int KT, int NT>
cudaError_t launch_bwd_ck(const float *params, const void *grad_image, const Geom &g,
                          const Workspace &ws, float *grad_params, cudaStream_t s) {
    const size_t smem = bwd_smem(g);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_bwd<C, KT, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const cudaError_t e = launch_dependent(k_bwd<C, KT, NT>, dim3(g.B * g.T), dim3(NT), smem, s,
                                           params, grad_image, g, (const float4 *)ws.gr,
                                           (const int *)ws.offs, (const int *)ws.ids,
                                           grad_params, ws.err);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int C, int KT>
cudaError_t launch_bwd_scalar(const float *params, const void *grad_image, const Geom &g,
                              const Workspace &ws, float *grad_params, cudaStream_t s) {
    return launch_bwd_ck<C, KT, 256>(params, grad_image, g, ws, grad_params, s);
}

template <int C>
cudaError_t launch_bwd_c(const float *params, const void *grad_image, const Geom &g,
                         const Workspace &ws, float *grad_params, cudaStream_t s) {
    // Measured on B200: the pixel-pair kernel pays off for wide windows
    // (k >= 13); for smaller windows the per-Gaussian work is short and the
    // scalar kernel, with more blocks resident, is faster.
    if constexpr (C <= 4) {
        switch (g.k) {
            case 7: return launch_bwd_scalar<C, 7>(params, grad_image, g, ws, grad_params, s);
            case 9: return launch_bwd_scalar<C, 9>(params, grad_image, g, ws, grad_params, s);
            case 11: return launch_bwd_scalar<C, 11>(params, grad_image, g, ws, grad_params, s);
            case 13: return launch_bwd_pairs<C, 13, 128>(params, grad_image, g, ws, grad_params, s);
            case 15: return launch_bwd_pairs<C, 15, 128>(params, grad_image, g, ws, grad_params, s);
            default: break;
        }
    }
    return launch_bwd_scalar<C, 0>(params, grad_image, g, ws, grad_params, s);
}

}  // namespace

bool bwd_uses_pairs(int C, int k) { return C <= 4 && (k == 13 || k == 15); }

size_t bwd_smem(const Geom &g) {
    const int kk = g.k * g.k;
    const int full = kk / kGroup;
    const int RS = kTile + 4 * g.r;
    const int RP = staged_pitch(RS, g.k);
    const int GP = g.C <= 1 ? 1 : g.C <= 2 ? 2 : g.C <= 4 ? 4 : 8;
    const int RV = 3 + (g.C + 3) / 4;
    return sizeof(float4) * ((size_t)(full + 1) * kGroup + (size_t)g.bwd_rcap * RV) +
           sizeof(float) * (size_t)RS * RP * GP;
}

cudaError_t launch_bwd(const float *params, const void *grad_image, const Geom &g,
                       const Workspace &ws, float *grad_params, cudaStream_t s) {
    switch (g.C) {
        case 1: return launch_bwd_c<1>(params, grad_image, g, ws, grad_params, s);
        case 2: return launch_bwd_c<2>(params, grad_image, g, ws, grad_params, s);
        case 3: return launch_bwd_c<3>(params, grad_image, g, ws, grad_params, s);
        case 4: return launch_bwd_c<4>(params, grad_image, g, ws, grad_params, s);
        case 5: return launch_bwd_c<5>(params, grad_image, g, ws, grad_params, s);
        case 6: return launch_bwd_c<6>(params, grad_image, g, ws, grad_params, s);
        case 7: return launch_bwd_c<7>(params, grad_image, g, ws, grad_params, s);
        case 8: return launch_bwd_c<8>(params, grad_image, g, ws, grad_params, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pdr
