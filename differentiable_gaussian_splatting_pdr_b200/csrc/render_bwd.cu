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
                                                     const float *__restrict__ gimg, Geom g,
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
                v[u][c] = (in && c < C) ? gimg[(((size_t)b * C + c) * g.H + y) * g.W + x] : 0.0f;
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

            // Fixed xor tree over the lanes of the group.
#pragma unroll
            for (int d = 1; d < kGroup; d <<= 1) {
#pragma unroll
                for (int j = 0; j < NV; ++j) acc[j] += __shfl_xor_sync(gmask, acc[j], d);
            }
            if (lig == 0) {
                const float s1 = pp[2], s2 = pp[3];
                float *d = dparams + gid * g.P;
                d[0] = kTwoLn2 * fmaf(a1, acc[0], a2 * acc[1]);
                d[1] = kTwoLn2 * fmaf(b1, acc[0], b2 * acc[1]);
                d[2] = kTwoLn2 * acc[2];
                d[3] = kTwoLn2 * acc[4];
                d[4] = kTwoLn2 * 2.0f * sinhf(s1 - s2) * acc[3];
#pragma unroll
                for (int c = 0; c < C; ++c) d[5 + c] = acc[5 + c];
            }
        }
        nh = 0;
    }
}

template <int C, int KT>
cudaError_t launch_bwd_ck(const float *params, const float *grad_image, const Geom &g,
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
cudaError_t launch_bwd_c(const float *params, const float *grad_image, const Geom &g,
                         const Workspace &ws, float *grad_params, cudaStream_t s) {
    if constexpr (C <= 4) {
        switch (g.k) {
            case 7: return launch_bwd_ck<C, 7>(params, grad_image, g, ws, grad_params, s);
            case 9: return launch_bwd_ck<C, 9>(params, grad_image, g, ws, grad_params, s);
            case 11: return launch_bwd_ck<C, 11>(params, grad_image, g, ws, grad_params, s);
            case 13: return launch_bwd_ck<C, 13>(params, grad_image, g, ws, grad_params, s);
            case 15: return launch_bwd_ck<C, 15>(params, grad_image, g, ws, grad_params, s);
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

cudaError_t launch_bwd(const float *params, const float *grad_image, const Geom &g,
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
