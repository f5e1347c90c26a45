// Backward kernel: dL/d(mu, s, theta, a) from dL/dI (paper abstract: a
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
// the inner loop needs no bounds tests.  Eight lanes share one Gaussian and
// stride over its k*k window pixels (a lane takes pixels l, l + 8, ... in
// row-major order, from a per-block offset table).  The staged rows have a
// pitch congruent to k modulo 8, so the 8 pixels the lanes of a group read
// together fall in 8 distinct 16-byte bank groups even across a row wrap: the
// loads of dL/dI are free of bank conflicts.  The lanes' partial sums are
// combined with a fixed xor-shuffle tree (a segmented reduction with segments
// of 8 lanes), and the chain rule is applied once, so no per-pixel atomics
// and no partial-gradient buffer are needed.  Every sum has a fixed order.
// The common window sizes are compiled in (KT = k), which lets the window
// loop unroll with constant table offsets; other sizes use KT = 0.
#include "common.cuh"

namespace pdr {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kGroup = 8;                          // lanes per Gaussian
constexpr int kGroups = kBwdThreads / kGroup;      // Gaussians in flight per block
constexpr int kPer = 2;                            // entries tested per thread per pass
constexpr int kPass = kPer * kBwdThreads;          // entries scanned per pass
constexpr int kHomeCap = 2 * kPass;                // home Gaussians gathered before processing

// Channels of dL/dI stored per shared-memory pixel (padded to a vector width).
template <int C> struct GPix { static constexpr int n = C <= 1 ? 1 : C <= 2 ? 2 : C <= 4 ? 4 : 8; };

// Row pitch (pixels) of the staged region: at least RS, congruent to k mod 8.
__host__ __device__ __forceinline__ int staged_pitch(int RS, int k) {
    return RS + (((k - RS) % 8) + 8) % 8;
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

template <int C, int KT>
__global__ void __launch_bounds__(kBwdThreads) k_bwd(const float *__restrict__ params,
                                                     const void *__restrict__ gimg, Geom g,
                                                     const float4 *__restrict__ gr,
                                                     const int *__restrict__ offs,
                                                     const int *__restrict__ ids,
                                                     float *__restrict__ dparams,
                                                     int *__restrict__ err) {
    constexpr int GP = GPix<C>::n;
    constexpr int NV = 5 + C;
    extern __shared__ float4 smem4[];
    const int k = KT ? KT : g.k, r = (k - 1) / 2;
    const int RS = kTile + 4 * r;                 // staged region edge (pixels)
    const int RP = staged_pitch(RS, k);           // its row pitch
    const int kk = k * k;
    const int full = kk / kGroup, tail = kk - full * kGroup;  // compile-time when KT > 0
    float4 *table = smem4;                        // [(full + 1) * 8]: (ox, oy, offset, 0)
    int *home = reinterpret_cast<int *>(table + (full + 1) * kGroup);  // [kHomeCap]
    float *gh = reinterpret_cast<float *>(home + kHomeCap);            // [RS*RS][GP]
    {
        // The launch must have provided this layout; otherwise report, touch nothing.
        const unsigned need = (unsigned)(sizeof(float4) * (full + 1) * kGroup +
                                         sizeof(int) * kHomeCap + sizeof(float) * RS * RP * GP);
        if (dynamic_smem_bytes() < need) {
            if (threadIdx.x == 0) atomicOr(err, kErrSmemLayout);
            return;
        }
    }

    const int b = blockIdx.x / g.T, t = blockIdx.x - b * g.T;
    const int ty = t / g.TX, tx = t - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    const int RX0 = X0 - 2 * r, RY0 = Y0 - 2 * r;  // region origin (grid coordinates)
    const int tid = threadIdx.x;
    const int grp = tid / kGroup, lig = tid % kGroup;
    // Groups of one warp may run different numbers of Gaussians, so the
    // group's reduction names only its own lanes.
    const unsigned gmask = ((1u << kGroup) - 1u) << (kGroup * (grp % (32 / kGroup)));

    // Gaussians whose window misses the grid (or whose mean is not finite)
    // appear in no list: this block zeroes a slice of them.
    {
        const int per = (g.N + g.T - 1) / g.T;
        const int i0 = t * per, i1 = min(i0 + per, g.N);
        for (int i = i0 + tid; i < i1; i += kBwdThreads) {
            const size_t gid = (size_t)b * g.N + i;
            const float4 Q = gr[2 * gid + 1];
            int x0, x1, y0, y1;
            if (!window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
                float *d = dparams + gid * g.P;
                for (int j = 0; j < g.P; ++j) d[j] = 0.0f;
            }
        }
    }

    // Window enumeration table: lane l of a group takes window pixels
    // l, l + 8, l + 16, ... in row-major order.
    for (int j = tid; j < (full + 1) * kGroup; j += kBwdThreads) {
        const int p = j < kk ? j : 0;
        const int ox = p % k, oy = p / k;
        table[j] = make_float4((float)ox, (float)oy, __int_as_float(oy * RP + ox), 0.0f);
    }
    // dL/dI of the core [X0 - r, X0 + 15 + r]^2 (zero outside the grid); the
    // outer ring is only ever read by Gaussians centred off the grid, at
    // pixels that are themselves off the grid, so it is all zeros.
    constexpr int kStageU = 4;  // pixels per thread with their loads in flight together
    for (int p0 = 0; p0 < RS * RS; p0 += kStageU * kBwdThreads) {
        float v[kStageU][GP];
#pragma unroll
        for (int u = 0; u < kStageU; ++u) {
            const int pix = p0 + u * kBwdThreads + tid;
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
            const int pix = p0 + u * kBwdThreads + tid;
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

    // Home Gaussians are gathered from the tile's list (in list order) until
    // enough are there to keep all groups busy, then processed.
    int L0, L1;
    list_range(offs, g, b, t, err, L0, L1);
    __shared__ int wtot[kBwdThreads / 32];
    int nh = 0;
    for (int e0 = L0; e0 < L1; e0 += kPass) {
        // Each thread tests a contiguous stripe of entries (all loads in
        // flight at once); a block scan keeps the home Gaussians in order.
        const int e1 = min(e0 + kPass, L1);
        const int per = (e1 - e0 + kBwdThreads - 1) / kBwdThreads;
        const int my0 = e0 + tid * per;
        int found[kPer];
        unsigned hits = 0u;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            found[j] = -1;
            const int e = my0 + j;
            if (j < per && e < e1) {
                const int i = ids[e];
                if ((unsigned)i >= (unsigned)g.N) {  // never for consistent bins
                    atomicOr(err, kErrBadId);
                    continue;
                }
                const float4 Q = gr[2 * ((size_t)b * g.N + i) + 1];
                if (home_tile(__float_as_int(Q.z), __float_as_int(Q.w), g) == t) {
                    found[j] = i;
                    hits |= 1u << j;
                }
            }
        }
        __syncthreads();  // staging done / previous homes consumed
        int total;
        int at = nh + block_excl_scan(__popc(hits), wtot, total);
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (hits & (1u << j)) home[at++] = found[j];
        nh += total;
        if (nh <= kHomeCap - kPass && e1 < L1) continue;  // gather more
        __syncthreads();

        for (int h = grp; h < nh; h += kGroups) {
            const size_t gid = (size_t)b * g.N + home[h];
            const float4 A = gr[2 * gid], Q = gr[2 * gid + 1];
            const float a1 = A.z, b1 = A.w, a2 = Q.x, b2 = Q.y;
            const int cx = __float_as_int(Q.z), cy = __float_as_int(Q.w);
            const int wx0 = cx - r, wy0 = cy - r;
            const float dx0 = (float)wx0 - A.x, dy0 = (float)wy0 - A.y;
            const float K1 = fmaf(a1, dx0, b1 * dy0), K2 = fmaf(a2, dx0, b2 * dy0);
            const float *gb = gh + (size_t)((wy0 - RY0) * RP + (wx0 - RX0)) * GP;
            const float *pp = params + gid * g.P;
            float amp[C];
#pragma unroll
            for (int c = 0; c < C; ++c) amp[c] = pp[5 + c];
            float acc[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) acc[j] = 0.0f;

            auto eval = [&](int j) {
                const float4 tb = table[j * kGroup + lig];
                float gv[C];
                load_gpix<C>(gb, __float_as_int(tb.z), gv);
                const float u1 = fmaf(a1, tb.x, fmaf(b1, tb.y, K1));
                const float u2 = fmaf(a2, tb.x, fmaf(b2, tb.y, K2));
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
            if constexpr (KT > 0) {
#pragma unroll 8
                for (int j = 0; j < full; ++j) eval(j);
            } else {
                for (int j = 0; j < full; ++j) eval(j);
            }
            if (lig < tail) eval(full);

            // The chain rule is linear in the sums, so each lane applies it to
            // its own partial sums; a transposing xor tree then leaves lane j
            // of the group with gradient component j (j < 8), summed over the
            // group in a fixed order; components 8.. (C > 3) use a plain tree.
            // 2 sinh(s1 - s2) = e^{d} - e^{-d}, via the base-2 exponential.
            const float dl = (pp[2] - pp[3]) * 1.44269504088896340736f;
            const float sh2 = kTwoLn2 * (ex2(dl) - ex2(-dl));
            float v[8];
            v[0] = kTwoLn2 * fmaf(a1, acc[0], a2 * acc[1]);  // dL/dmu_x
            v[1] = kTwoLn2 * fmaf(b1, acc[0], b2 * acc[1]);  // dL/dmu_y
            v[2] = kTwoLn2 * acc[2];                         // dL/ds_1
            v[3] = kTwoLn2 * acc[4];                         // dL/ds_2
            v[4] = sh2 * acc[3];                             // dL/dtheta
#pragma unroll
            for (int j = 5; j < 8; ++j) v[j] = j < NV ? acc[j < NV ? j : 0] : 0.0f;
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
            float *d = dparams + gid * g.P;
            if (lig < NV) d[lig] = v[0];
#pragma unroll
            for (int j = 8; j < NV; ++j) {
                float e = acc[j];
#pragma unroll
                for (int dd = 1; dd < kGroup; dd <<= 1) e += __shfl_xor_sync(gmask, e, dd);
                if (lig == 0) d[j] = e;
            }
        }
        nh = 0;
    }
}

// ---------------------------------------------------------------------------
// Pixel-pair backward (C <= 4, k <= 15 compiled in).  Same home-tile
// decomposition and the same seven sums per Gaussian as k_bwd, but every
// lane works on two horizontally adjacent pixels at once with the packed
// f32x2 arithmetic of sm_100 (one instruction issues two FP32 FMAs), which
// halves the issue slots of the inner loop; the loop is then bound by the
// FMA pipe itself.
//
// A window row of k pixels (k odd) is covered by (k + 1) / 2 pairs whose
// last pixel lies just outside the window and is masked (its weight is
// 2^-inf = 0).  So that every window starts on a pair boundary whatever its
// parity, dL/dI is staged twice: pairs starting at even x and pairs starting
// at odd x.  Each staged element is a float4 holding two channels of the
// pair: (c0 lo, c0 hi, c1 lo, c1 hi), so a single vector load yields the
// packed operands directly.  The pair slots of a window (rows x pairs,
// row-major) are dealt to the 8 lanes of a group in turn: lane l takes slots
// l, l + 8, l + 16, ...  When the pairs of a row divide 8 (k = 3, 7, 15)
// the lanes tile whole rows and the slot coordinates follow from the lane
// and a compile-time step; otherwise they are kept per lane in registers.
// Staged rows have a pitch congruent to the pairs per row modulo 8, so the
// 8 lanes of a group always read 8 consecutive 16-byte bank groups.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2dup(float a) { return make_float2(a, a); }

// A home Gaussian as the groups need it, prepared once per block by the
// thread that found it: the packed (duplicated) operands of the pair loop.
struct HomeRec {
    float4 ab1;   // alpha_1, alpha_1, beta_1, beta_1
    float4 ab2;   // alpha_2, alpha_2, beta_2, beta_2
    float4 kk;    // K_1, K_1, K_2, K_2: uhat at the window corner (wx0, wy0)
    float4 a01;   // a_0, a_0, a_1, a_1
    float4 a23;   // a_2, a_2, a_3, a_3
    float4 aux;   // 2 ln2 * 2 sinh(s_1 - s_2), id, staged offset (or wx0 off the grid), wy0
};
constexpr int kPairPass = kBwdThreads;       // list entries tested per pass (one per thread)
constexpr int kRecCap = kPairPass;           // home records gathered before processing

template <int C, int K>
struct PairShape {
    static constexpr int R = (K - 1) / 2;
    static constexpr int NPW = (K + 1) / 2;                  // pairs per window row
    static constexpr int SLOTS = NPW * K;                    // pair slots per window
    // Lane l takes pair column l % NPW of rows l / NPW, l / NPW + RPS, ...;
    // when NPW does not divide 8, lanes NPW .. 7 idle.
    static constexpr int RPS = (kGroup % NPW) == 0 ? kGroup / NPW : 1;  // rows per lane step
    static constexpr int LANES = RPS * NPW;                  // active lanes of a group
    static constexpr int NS = (K + RPS - 1) / RPS;           // rows (slots) per active lane
    static constexpr int NPL = (C + 1) / 2;                  // float4 planes (two channels each)
    static constexpr int ROWS = kTile + 2 * R;               // staged rows: the tile and its apron
    static constexpr int PAIRS = kTile / 2 + R;              // staged pairs per row and parity
    static constexpr int PITCH = PAIRS + (((NPW - PAIRS) % 8) + 8) % 8;
    static constexpr int PLANE = ROWS * PITCH;               // float4 per (parity, plane)
    static constexpr int NIT = ROWS * PAIRS;                 // staging items
    static constexpr int SU = (NIT + kBwdThreads - 1) / kBwdThreads;  // items per thread
    static constexpr size_t SMEM = sizeof(float4) * 2 * NPL * PLANE + sizeof(HomeRec) * kRecCap;
};

template <int C, int K>
__global__ void __launch_bounds__(kBwdThreads, 3) k_bwd_pairs(const float *__restrict__ params,
                                                           const void *__restrict__ gimg, Geom g,
                                                           const float4 *__restrict__ gr,
                                                           const int *__restrict__ offs,
                                                           const int *__restrict__ ids,
                                                           float *__restrict__ dparams,
                                                           int *__restrict__ err) {
    using S = PairShape<C, K>;
    constexpr int R = S::R, NPW = S::NPW, NS = S::NS, NPL = S::NPL;
    constexpr int NV = 5 + C;
    extern __shared__ float4 smem4[];
    float4 *halo = smem4;  // [parity][plane][ROWS][PITCH]
    // Home records: Gaussians centred on the grid from the front, the rare
    // ones centred off the grid (their window leaves the staged apron) from
    // the back.
    HomeRec *recs = reinterpret_cast<HomeRec *>(halo + 2 * NPL * S::PLANE);  // [kRecCap]
    if (dynamic_smem_bytes() < (unsigned)S::SMEM || g.k != K) {  // launch/layout mismatch
        if (threadIdx.x == 0) atomicOr(err, kErrSmemLayout);
        return;
    }

    const int b = blockIdx.x / g.T, t = blockIdx.x - b * g.T;
    const int ty = t / g.TX, tx = t - ty * g.TX;
    const int X0 = tx * kTile, Y0 = ty * kTile;
    const int RX0 = X0 - R, RY0 = Y0 - R;  // staged region origin (grid coordinates)
    const int tid = threadIdx.x;
    const int grp = tid / kGroup, lig = tid % kGroup;
    const unsigned gmask = ((1u << kGroup) - 1u) << (kGroup * (grp % (32 / kGroup)));

    int L0, L1;
    list_range(offs, g, b, t, err, L0, L1);
    // The first pass's list entry, requested before the staging loads so that
    // both are in flight together.
    int id = L0 + tid < L1 ? ids[L0 + tid] : -1;

    // Stage dL/dI over [X0 - r, X0 + 15 + r]^2 (zero outside the grid; the
    // column after it, read only as the masked pixel of a last pair, is zero
    // too): item (row, m) holds pixels RX0 + 2m + {0, 1, 2}; the even plane
    // gets pair (0, 1), the odd plane pair (1, 2).
    {
        float v[S::SU][3][2 * NPL];
#pragma unroll
        for (int u = 0; u < S::SU; ++u) {
            const int it = u * kBwdThreads + tid;
            const int row = it / S::PAIRS, m = it - row * S::PAIRS;
            const int y = RY0 + row;
            const bool rowin = it < S::NIT && y >= 0 && y < g.H;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int x = RX0 + 2 * m + q;
                const bool in = rowin && x >= 0 && x < g.W && x <= X0 + kTile - 1 + R;
#pragma unroll
                for (int c = 0; c < 2 * NPL; ++c)
                    v[u][q][c] = (in && c < C) ? img_load(gimg, (((size_t)b * C + c) * g.H + y) * g.W + x, g.img_dtype) : 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < S::SU; ++u) {
            const int it = u * kBwdThreads + tid;
            if (it >= S::NIT) continue;
            const int row = it / S::PAIRS, m = it - row * S::PAIRS;
            float4 *dst = halo + row * S::PITCH + m;
#pragma unroll
            for (int pl = 0; pl < NPL; ++pl) {
                dst[pl * S::PLANE] = make_float4(v[u][0][2 * pl], v[u][1][2 * pl],
                                                 v[u][0][2 * pl + 1], v[u][1][2 * pl + 1]);
                dst[(NPL + pl) * S::PLANE] = make_float4(v[u][1][2 * pl], v[u][2][2 * pl],
                                                         v[u][1][2 * pl + 1], v[u][2][2 * pl + 1]);
            }
        }
    }

    // Gaussians whose window misses the grid appear in no list: zero a slice.
    {
        const int per = (g.N + g.T - 1) / g.T;
        const int i0 = t * per, i1 = min(i0 + per, g.N);
        for (int i = i0 + tid; i < i1; i += kBwdThreads) {
            const size_t gid = (size_t)b * g.N + i;
            const float4 Q = gr[2 * gid + 1];
            int x0, x1, y0, y1;
            if (!window_rect(__float_as_int(Q.z), __float_as_int(Q.w), g, x0, x1, y0, y1)) {
                float *d = dparams + gid * g.P;
                for (int j = 0; j < g.P; ++j) d[j] = 0.0f;
            }
        }
    }

    // This lane's pair column and first row (independent of the Gaussian),
    // with the mask of the pair's second pixel (last pair of a row).
    const bool lane_on = lig < S::LANES;
    const int pc = lig % NPW, r0 = lig / NPW;
    const float2 sfx = make_float2((float)(2 * pc), (float)(2 * pc + 1));
    const float2 sfy = f2dup((float)r0);
    const float smask = pc == NPW - 1 ? __int_as_float(0x7f800000) : 0.0f;  // +inf: 2^-inf = 0
    const int soff = r0 * S::PITCH + pc;
    const bool last_ok = r0 + (NS - 1) * S::RPS < K;  // the lane's last row lies in the window

    __shared__ int wtot[kBwdThreads / 32];
    int nh = 0, no = 0;  // home records on / off the grid gathered so far
    for (int e0 = L0; e0 < L1; e0 += kPairPass) {
        // Test this thread's entry; a home Gaussian's record is loaded along
        // with the test (one round trip for all of them).
        int kind = 0;  // 1: home, centred on the grid; 1 << 16: home, centred off it
        HomeRec rec;
        if (e0 + tid < L1) {
            if ((unsigned)id >= (unsigned)g.N) {  // never for consistent bins
                atomicOr(err, kErrBadId);
            } else {
                const size_t gid = (size_t)b * g.N + id;
                const float4 A = gr[2 * gid], Q = gr[2 * gid + 1];
                const float *pp = params + gid * g.P;
                const float s1 = pp[2], s2 = pp[3];
                float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int c = 0; c < C; ++c) a[c] = pp[5 + c];
                const int cx = __float_as_int(Q.z), cy = __float_as_int(Q.w);
                if (home_tile(cx, cy, g) == t) {
                    const bool ongrid = cx >= 0 && cx < g.W && cy >= 0 && cy < g.H;
                    kind = ongrid ? 1 : (1 << 16);
                    const float a1 = A.z, b1 = A.w, a2 = Q.x, b2 = Q.y;
                    const int wx0 = cx - R, wy0 = cy - R;
                    const float dx0 = (float)wx0 - A.x, dy0 = (float)wy0 - A.y;
                    const float K1 = fmaf(a1, dx0, b1 * dy0), K2 = fmaf(a2, dx0, b2 * dy0);
                    const int lx = wx0 - RX0;  // in [0, 15] on the grid
                    const int base = (lx & 1) * NPL * S::PLANE + (wy0 - RY0) * S::PITCH + (lx >> 1);
                    // 2 sinh(s1 - s2) = e^{d} - e^{-d}, via the base-2 exponential.
                    const float dl = (s1 - s2) * 1.44269504088896340736f;
                    rec.ab1 = make_float4(a1, a1, b1, b1);
                    rec.ab2 = make_float4(a2, a2, b2, b2);
                    rec.kk = make_float4(K1, K1, K2, K2);
                    rec.a01 = make_float4(a[0], a[0], a[1], a[1]);
                    rec.a23 = make_float4(a[2], a[2], a[3], a[3]);
                    rec.aux = make_float4(kTwoLn2 * (ex2(dl) - ex2(-dl)), __int_as_float(id),
                                          __int_as_float(ongrid ? base : wx0), __int_as_float(wy0));
                }
            }
        }
        {
            const int en = e0 + kPairPass + tid;  // the next pass's entry, in flight meanwhile
            id = en < L1 ? ids[en] : -1;
        }
        int total;
        const int at = block_excl_scan(kind, wtot, total);  // also orders the staging
        if (kind == 1) recs[nh + (at & 0xffff)] = rec;
        if (kind > 1) recs[kRecCap - 1 - (no + (at >> 16))] = rec;
        nh += total & 0xffff;
        no += total >> 16;
        __syncthreads();

        for (int h = grp; h < nh + no; h += kGroups) {
            const bool off = h >= nh;
            const HomeRec &hr = off ? recs[kRecCap - 1 - (h - nh)] : recs[h];
            const float4 AB1 = hr.ab1, AB2 = hr.ab2, KK = hr.kk, AX = hr.aux;
            const float2 A1 = make_float2(AB1.x, AB1.y), B1 = make_float2(AB1.z, AB1.w);
            const float2 A2 = make_float2(AB2.x, AB2.y), B2 = make_float2(AB2.z, AB2.w);
            const float2 K1 = make_float2(KK.x, KK.y), K2 = make_float2(KK.z, KK.w);
            float2 AMP[C];
            {
                const float4 P = hr.a01;
                AMP[0] = make_float2(P.x, P.y);
                if constexpr (C > 1) AMP[1] = make_float2(P.z, P.w);
            }
            if constexpr (C > 2) {
                const float4 P = hr.a23;
                AMP[2] = make_float2(P.x, P.y);
                if constexpr (C > 3) AMP[3] = make_float2(P.z, P.w);
            }
            const float2 z2 = make_float2(0.0f, 0.0f);
            float2 S1 = z2, S2 = z2, S11 = z2, S12 = z2, S22 = z2, DA[C];
#pragma unroll
            for (int c = 0; c < C; ++c) DA[c] = z2;

            // One pair slot: u = uhat of the two pixels, q = |uhat|^2 (+inf
            // on a masked pixel), w = 2^-q, gc = dL/dI of the pair.
            auto slot = [&](float2 u1, float2 u2, float mhi, const float2 (&gc)[2 * NPL]) {
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

            if (!off && lane_on) {
                const float4 *hp = halo + __float_as_int(AX.z) + soff;
                float2 u1 = f2fma(A1, sfx, f2fma(B1, sfy, K1));
                float2 u2 = f2fma(A2, sfx, f2fma(B2, sfy, K2));
                const float2 RB1 = S::RPS == 1 ? B1 : f2mul(B1, f2dup((float)S::RPS));
                const float2 RB2 = S::RPS == 1 ? B2 : f2mul(B2, f2dup((float)S::RPS));
#pragma unroll
                for (int j = 0; j < NS; ++j) {
                    if (j > 0) {
                        u1 = f2add(u1, RB1);
                        u2 = f2add(u2, RB2);
                    }
                    if (j < NS - 1 || last_ok) {
                        float2 gc[2 * NPL];
#pragma unroll
                        for (int pl = 0; pl < NPL; ++pl) {
                            const float4 P = hp[j * S::RPS * S::PITCH + pl * S::PLANE];
                            gc[2 * pl] = make_float2(P.x, P.y);
                            gc[2 * pl + 1] = make_float2(P.z, P.w);
                        }
                        slot(u1, u2, smask, gc);
                    }
                }
            } else if (off) {
                // Centred off the grid: read dL/dI from global memory, zero
                // outside the grid (rare: a centre within r of the border).
                const int wx0 = __float_as_int(AX.z), wy0 = __float_as_int(AX.w);
                for (int sl = lig; sl < S::SLOTS; sl += kGroup) {
                    const int row = sl / NPW, pc = sl - row * NPW;
                    const int x = wx0 + 2 * pc, y = wy0 + row;
                    const float2 fx = make_float2((float)(2 * pc), (float)(2 * pc + 1));
                    const float2 fy = f2dup((float)row);
                    const float2 u1 = f2fma(A1, fx, f2fma(B1, fy, K1));
                    const float2 u2 = f2fma(A2, fx, f2fma(B2, fy, K2));
                    float2 gc[2 * NPL];
#pragma unroll
                    for (int c = 0; c < 2 * NPL; ++c) {
                        float lo = 0.0f, hi = 0.0f;
                        if (c < C && y >= 0 && y < g.H) {
                            const size_t row = (((size_t)b * C + c) * g.H + y) * g.W;
                            if (x >= 0 && x < g.W) lo = img_load(gimg, row + x, g.img_dtype);
                            if (x + 1 >= 0 && x + 1 < g.W && pc < NPW - 1)
                                hi = img_load(gimg, row + x + 1, g.img_dtype);
                        }
                        gc[c] = make_float2(lo, hi);
                    }
                    slot(u1, u2, pc == NPW - 1 ? __int_as_float(0x7f800000) : 0.0f, gc);
                }
            }

            // The chain rule is linear in the sums, so each lane applies it to
            // its own partial sums; a transposing xor tree then leaves lane j
            // of the group with gradient component j, summed over the group.
            float v[8];
            {
                const float s1 = S1.x + S1.y, s2 = S2.x + S2.y;
                v[0] = kTwoLn2 * fmaf(AB1.x, s1, AB2.x * s2);  // dL/dmu_x
                v[1] = kTwoLn2 * fmaf(AB1.z, s1, AB2.z * s2);  // dL/dmu_y
                v[2] = kTwoLn2 * (S11.x + S11.y);               // dL/ds_1
                v[3] = kTwoLn2 * (S22.x + S22.y);               // dL/ds_2
                v[4] = AX.x * (S12.x + S12.y);                  // dL/dtheta
#pragma unroll
                for (int j = 5; j < 8; ++j) v[j] = j - 5 < C ? DA[j - 5 < C ? j - 5 : 0].x + DA[j - 5 < C ? j - 5 : 0].y : 0.0f;
            }
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
            float *d = dparams + ((size_t)b * g.N + __float_as_int(AX.y)) * g.P;
            if (lig < NV) d[lig] = v[0];
            if constexpr (C > 3) {  // the ninth component: dL/da_3
                float e = DA[3].x + DA[3].y;
#pragma unroll
                for (int dd = 1; dd < kGroup; dd <<= 1) e += __shfl_xor_sync(gmask, e, dd);
                if (lig == 0) d[8] = e;
            }
        }
        nh = 0;
        no = 0;
    }
}

template <int C, int K>
cudaError_t launch_bwd_pairs(const float *params, const void *grad_image, const Geom &g,
                             const Workspace &ws, float *grad_params, cudaStream_t s) {
    constexpr size_t smem = PairShape<C, K>::SMEM;
    static_assert(smem <= 200 * 1024, "staged dL/dI does not fit");
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_bwd_pairs<C, K>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_bwd_pairs<C, K><<<g.B * g.T, kBwdThreads, smem, s>>>(params, grad_image, g, ws.gr, ws.offs,
                                                           ws.ids, grad_params, ws.err);
    return cudaGetLastError();
}

template <int C, int KT>
cudaError_t launch_bwd_ck(const float *params, const void *grad_image, const Geom &g,
                          const Workspace &ws, float *grad_params, cudaStream_t s) {
    const size_t smem = bwd_smem(g);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_bwd<C, KT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_bwd<C, KT><<<g.B * g.T, kBwdThreads, smem, s>>>(params, grad_image, g, ws.gr, ws.offs,
                                                      ws.ids, grad_params, ws.err);
    return cudaGetLastError();
}

template <int C>
cudaError_t launch_bwd_c(const float *params, const void *grad_image, const Geom &g,
                         const Workspace &ws, float *grad_params, cudaStream_t s) {
    // Measured on B200: the pixel-pair kernel pays off for wide windows
    // (k >= 13); for smaller windows the per-Gaussian work is short and the
    // scalar kernel, with more blocks resident, is faster.
    if constexpr (C <= 4) {
        switch (g.k) {
            case 7: return launch_bwd_ck<C, 7>(params, grad_image, g, ws, grad_params, s);
            case 9: return launch_bwd_ck<C, 9>(params, grad_image, g, ws, grad_params, s);
            case 11: return launch_bwd_ck<C, 11>(params, grad_image, g, ws, grad_params, s);
            case 13: return launch_bwd_pairs<C, 13>(params, grad_image, g, ws, grad_params, s);
            case 15: return launch_bwd_pairs<C, 15>(params, grad_image, g, ws, grad_params, s);
            default: break;
        }
    }
    return launch_bwd_ck<C, 0>(params, grad_image, g, ws, grad_params, s);
}

}  // namespace

size_t bwd_smem(const Geom &g) {
    const int kk = g.k * g.k;
    const int full = kk / kGroup;
    const int RS = kTile + 4 * g.r;
    const int RP = staged_pitch(RS, g.k);
    const int GP = g.C <= 1 ? 1 : g.C <= 2 ? 2 : g.C <= 4 ? 4 : 8;
    return sizeof(float4) * (size_t)(full + 1) * kGroup + sizeof(int) * kHomeCap +
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
