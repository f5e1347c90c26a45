// C ABI of libpdr.so (declared in include/pdr.h): host-side validation,
// geometry, workspace layout and kernel launches on the caller's stream.
// The library allocates no device memory: everything lives in the caller's
// workspace and buffers.
#include <limits.h>
#include <stdint.h>

#include "common.cuh"
#include "pdr.h"

namespace pdr {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

int tiles_per_axis(int k) { return (k - 1 + kTile - 1) / kTile + 1; }

struct Layout {
    size_t err, gr, hist, tot, offs, ids, total;
};

// Forward pixels per lane: 2 for small grids (at most 2368 tiles in all:
// more, shorter lanes per tile), else 4 (measured on B200).
int fwd_pixels_per_lane(long long B, long long T) { return B * T <= 2368 ? 2 : 4; }

pdr_status make_geom(int B, int N, int C, int H, int W, int k, Geom *g) {
    // N = 0: frames with no Gaussians (the entry points launch no kernel then).
    if (B < 1 || N < 0 || C < 1 || H < 1 || W < 1 || k < 1 || (k & 1) == 0)
        return PDR_ERR_INVALID_ARG;
    if (C > PDR_MAX_C || k > PDR_MAX_K) return PDR_ERR_TOO_LARGE;
    const long long TX = (W + kTile - 1) / kTile, TY = (H + kTile - 1) / kTile;
    const long long T = TX * TY;
    if (T > PDR_MAX_TILES_PER_FRAME) return PDR_ERR_TOO_LARGE;
    const long long m = tiles_per_axis(k);
    const long long cap = (long long)N * m * m;
    if ((long long)B * cap > INT_MAX || (long long)B * T > INT_MAX || B > 65535 ||
        (long long)B * N * (5 + C) > (long long)INT_MAX * 64)
        return PDR_ERR_TOO_LARGE;
    g->B = B; g->N = N; g->C = C; g->H = H; g->W = W; g->k = k; g->r = (k - 1) / 2;
    g->TX = (int)TX; g->TY = (int)TY; g->T = (int)T;
    g->P = 5 + C;
    g->m = (int)m;
    g->cap = (int)cap;
    // Binning slabs of 32 * R Gaussians (one scatter warp each): R = 8, halved
    // while the frames would give fewer than eight scatter warps per SM, but
    // at least T / 64 so that the per-slab counts (B x slabs x T ints) stay
    // within about two ints per Gaussian (measured on B200: 512-Gaussian slabs
    // bin a 1024-tile frame faster than 256).  Slabs under 256 Gaussians
    // divide 256 (R = 1, 2, 4).
    {
        int R = 8;
        while (R > 1 && (long long)B * ((N + 32 * R - 1) / (32 * R)) < 8 * 148) R >>= 1;
        int rmin = (int)((T + 63) / 64);
        if (rmin <= 8) rmin = rmin <= 1 ? 1 : rmin <= 2 ? 2 : rmin <= 4 ? 4 : 8;  // divides 256
        if (R < rmin) R = rmin;
        g->slab = 32 * R;
        g->nslab = (N + g->slab - 1) / g->slab;
    }
    if (m > 3) return PDR_ERR_TOO_LARGE;  // the slab scatter handles windows over at most 3 tiles per axis
    // Slab-scatter block: up to 8 warps while its tables (a list start per
    // tile, and a slot and a mask table per warp) stay within 100 KB.
    {
        int nw = 8;
        while (nw > 1 && (size_t)T * 4 * (1 + 2 * nw) > 100 * 1024) nw >>= 1;
        g->slab_warps = nw;  // one warp: 12 bytes per tile, <= 192 KB for the most tiles
    }
    // Small frames: one binning block per frame (its shared-memory tables
    // hold [2 + 2 * warps] x T ints).
    // (only when the frames alone give at least one block per SM; otherwise
    // the slab kernels spread the work over more blocks)
    g->frame_block = T <= kFrameBlockMaxT && N <= kFrameBlockMaxN && B >= 148;
    int ft = ((N + 31) / 32) * 32;
    if (ft > 1024) ft = 1024;
    if (ft < 32) ft = 32;
    // More frames than SMs: smaller blocks, so that all frames are resident in
    // one wave (about 1024 binning threads per SM).
    const long long per_sm = ((long long)B + 147) / 148;
    while (ft > 128 && per_sm * ft > 1024) ft = ((ft / 2 + 31) / 32) * 32;
    g->frame_threads = ft;
    // Bins + render in one clustered launch only while the launch is small
    // (latency-bound); larger batches of small frames run faster as separate
    // binning and render launches (measured on B200).
    g->cluster_fwd = T <= kClusterTiles && (long long)B * T <= kClusterMaxBlocks;
    g->fwd_pl = fwd_pixels_per_lane(B, T);
    g->out_vec2 = 0;
    g->out_vec4 = 0;
    g->img_dtype = PDR_F32;
    g->stage_vec4 = 0;
    // Backward record capacity: room for the home Gaussians of a tile at 1.5x
    // the mean count (a tile with more is processed in several rounds), at
    // least one block's worth of list entries, at most 512.
    // The pixel-pair kernel runs 128-thread blocks (short last rounds of its
    // 16 groups per tile); the scalar kernel 256-thread blocks (measured on B200).
    {
        const long long mean = ((long long)N + T - 1) / T;
        long long cap = ((mean * 3 / 2 + 32 + 31) / 32) * 32;
        const int nt = bwd_uses_pairs(C, k) ? 128 : 256;
        if (cap < nt) cap = nt;
        if (cap > 512) cap = 512;
        g->bwd_threads = nt;
        g->bwd_rcap = (int)cap;
    }
    return PDR_OK;
}

Layout make_layout(const Geom &g) {
    Layout L;
    size_t o = 0;
    L.err = o; o += align_up(sizeof(int));  // the device error word
    L.gr = o; o += align_up(sizeof(float4) * 2 * (size_t)g.B * g.N);
    L.hist = o; o += align_up(sizeof(int) * (size_t)g.B * g.nslab * g.T);
    L.tot = o; o += align_up(sizeof(int) * (size_t)g.B * g.T);
    L.offs = o; o += align_up(sizeof(int) * (size_t)g.B * (g.T + 1));
    L.ids = o; o += align_up(sizeof(int) * (size_t)g.B * g.cap);
    L.total = o;
    return L;
}

Workspace carve(void *base, const Layout &L) {
    char *p = static_cast<char *>(base);
    Workspace w;
    w.err = reinterpret_cast<int *>(p + L.err);
    w.gr = reinterpret_cast<float4 *>(p + L.gr);
    w.hist = reinterpret_cast<int *>(p + L.hist);
    w.tot = reinterpret_cast<int *>(p + L.tot);
    w.offs = reinterpret_cast<int *>(p + L.offs);
    w.ids = reinterpret_cast<int *>(p + L.ids);
    return w;
}

pdr_status check_ws(const Geom &g, void *ws, size_t bytes, Layout *L) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return PDR_ERR_INVALID_ARG;
    *L = make_layout(g);
    if (bytes < L->total) return PDR_ERR_WORKSPACE_TOO_SMALL;
    return PDR_OK;
}

pdr_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PDR_OK : PDR_ERR_CUDA; }

// Side streams and events of pdr_step_host, one set per host thread and
// device, created on first use and kept for the thread's lifetime: `up` for
// the dL/dI upload, `down` for the image download, so that the download can
// run while the upload is still in flight (PCIe carries both directions at
// once).
constexpr int kStepChunks = 4;                       // frame chunks of a host step
constexpr size_t kStepChunkMinBytes = 8u << 20;      // ... when it moves this much each way
constexpr int kStepEvents = 2 + 4 * kStepChunks;
struct StepSide {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t ev[kStepEvents] = {};
};
constexpr int kMaxDevices = 64;

cudaError_t step_side(StepSide **out) {
    static thread_local StepSide sides[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    StepSide &d = sides[dev];
    if (!d.up) {
        StepSide n;
        e = cudaStreamCreateWithFlags(&n.up, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&n.down, cudaStreamNonBlocking);
        for (int j = 0; j < kStepEvents && e == cudaSuccess; ++j)
            e = cudaEventCreateWithFlags(&n.ev[j], cudaEventDisableTiming);
        if (e != cudaSuccess) {
            for (cudaEvent_t v : n.ev)
                if (v) cudaEventDestroy(v);
            if (n.up) cudaStreamDestroy(n.up);
            if (n.down) cudaStreamDestroy(n.down);
            return e;
        }
        d = n;
    }
    *out = &d;
    return cudaSuccess;
}

// Binning starts a new use of the workspace: the device error word is
// cleared first, stream-ordered, so that no kernel of this call (or of a
// render that reuses these bins) can have set a bit that the clear then wipes.
cudaError_t clear_error_word(const Workspace &ws, cudaStream_t s) {
    return cudaMemsetAsync(ws.err, 0, sizeof(int), s);
}

cudaError_t bin(const float *params, const Geom &g, const Workspace &ws, cudaStream_t s) {
    cudaError_t e = clear_error_word(ws, s);
    if (e != cudaSuccess) return e;
    if (g.N == 0)  // no Gaussians: every tile list empty at 0
        return cudaMemsetAsync(ws.offs, 0, sizeof(int) * (size_t)g.B * (g.T + 1), s);
    return launch_bin(params, g, ws, s);
}

// params (and grad_params) may be null only when there are no Gaussians.
bool params_ok(const Geom &g, const void *p) { return g.N == 0 || p != nullptr; }

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace
}  // namespace pdr

using namespace pdr;

extern "C" {

int pdr_abi_version(void) { return 1; }

const char *pdr_status_string(pdr_status s) {
    switch (s) {
        case PDR_OK: return "PDR_OK";
        case PDR_ERR_INVALID_ARG: return "PDR_ERR_INVALID_ARG: bad size, even k, null or misaligned pointer";
        case PDR_ERR_WORKSPACE_TOO_SMALL: return "PDR_ERR_WORKSPACE_TOO_SMALL";
        case PDR_ERR_CUDA: return "PDR_ERR_CUDA: a CUDA call or kernel launch failed";
        case PDR_ERR_DEVICE_TIMEOUT: return "PDR_ERR_DEVICE_TIMEOUT";
        case PDR_ERR_INTERNAL: return "PDR_ERR_INTERNAL: a device-side check failed";
        case PDR_ERR_TOO_LARGE: return "PDR_ERR_TOO_LARGE: sizes beyond the library limits";
    }
    return "unknown pdr_status";
}

size_t pdr_workspace_bytes(int B, int N, int C, int H, int W, int k) {
    Geom g;
    if (make_geom(B, N, C, H, W, k, &g) != PDR_OK) return 0;
    return make_layout(g).total;
}

long long pdr_list_capacity_per_frame(int N, int k) {
    if (N < 1 || k < 1 || (k & 1) == 0) return 0;
    const long long m = tiles_per_axis(k);
    return (long long)N * m * m;
}

pdr_status pdr_build_bins(const float *params, int B, int N, int C, int H, int W, int k,
                          void *workspace, size_t workspace_bytes, void *stream) {
    Geom g;
    pdr_status st = make_geom(B, N, C, H, W, k, &g);
    if (st != PDR_OK) return st;
    if (!params_ok(g, params) || !aligned4(params)) return PDR_ERR_INVALID_ARG;
    Layout L;
    st = check_ws(g, workspace, workspace_bytes, &L);
    if (st != PDR_OK) return st;
    return from_cuda(bin(params, g, carve(workspace, L), static_cast<cudaStream_t>(stream)));
}

static bool dtype_ok(int dtype, const void *p) {
    if (dtype == PDR_F32) return (reinterpret_cast<uintptr_t>(p) & 3) == 0;
    if (dtype == PDR_F16 || dtype == PDR_BF16) return (reinterpret_cast<uintptr_t>(p) & 1) == 0;
    return false;
}

namespace {
// The forward of frames that belong to a batch of B_batch frames: the pixels
// per lane (the one choice that changes how a pixel's weights are evaluated,
// hence the last bits of the image) follow the whole batch, so that rendering
// the batch in chunks gives bitwise the image of one call.
pdr_status render_fwd_in_batch(const float *params, int B, int N, int C, int H, int W, int k,
                               void *image, int image_dtype, void *workspace,
                               size_t workspace_bytes, int workspace_holds_bins, void *stream,
                               int B_batch) {
    Geom g;
    pdr_status st = make_geom(B, N, C, H, W, k, &g);
    if (st != PDR_OK) return st;
    g.fwd_pl = fwd_pixels_per_lane(B_batch, g.T);
    if (!params_ok(g, params) || !image || !aligned4(params) || !dtype_ok(image_dtype, image))
        return PDR_ERR_INVALID_ARG;
    Layout L;
    st = check_ws(g, workspace, workspace_bytes, &L);
    if (st != PDR_OK) return st;
    const Workspace ws = carve(workspace, L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (g.N == 0) {  // the empty sum (all-zero bits are 0.0 in every storage type)
        st = from_cuda(bin(params, g, ws, s));
        if (st != PDR_OK) return st;
        const size_t esize = image_dtype == PDR_F32 ? sizeof(float) : 2;
        return from_cuda(
            cudaMemsetAsync(image, 0, esize * (size_t)g.B * g.C * g.H * g.W, s));
    }
    g.img_dtype = image_dtype;
    // 2- and 4-pixel vector stores: rows of a multiple of 2 / 4 pixels and an
    // image aligned to 2 / 4 elements.
    const uintptr_t esz = image_dtype == PDR_F32 ? 4 : 2;
    g.out_vec2 = ((g.W & 1) == 0) && ((reinterpret_cast<uintptr_t>(image) & (2 * esz - 1)) == 0);
    g.out_vec4 = ((g.W & 3) == 0) && ((reinterpret_cast<uintptr_t>(image) & (4 * esz - 1)) == 0);
    if (!workspace_holds_bins && g.cluster_fwd && fwd_cluster_schedulable(g)) {
        // Small frames: bins + render in one clustered launch.
        st = from_cuda(clear_error_word(ws, s));
        if (st != PDR_OK) return st;
        return from_cuda(launch_fwd(params, g, ws, image, s, true));
    }
    if (!workspace_holds_bins) {
        st = from_cuda(bin(params, g, ws, s));
        if (st != PDR_OK) return st;
    }
    return from_cuda(launch_fwd(params, g, ws, image, s, false));
}
}  // namespace

pdr_status pdr_render_fwd_ex(const float *params, int B, int N, int C, int H, int W, int k,
                             void *image, int image_dtype, void *workspace,
                             size_t workspace_bytes, int workspace_holds_bins, void *stream) {
    return render_fwd_in_batch(params, B, N, C, H, W, k, image, image_dtype, workspace,
                               workspace_bytes, workspace_holds_bins, stream, B);
}

pdr_status pdr_render_fwd(const float *params, int B, int N, int C, int H, int W, int k,
                          float *image, void *workspace, size_t workspace_bytes,
                          int workspace_holds_bins, void *stream) {
    return pdr_render_fwd_ex(params, B, N, C, H, W, k, image, PDR_F32, workspace, workspace_bytes,
                             workspace_holds_bins, stream);
}

pdr_status pdr_render_bwd_ex(const float *params, const void *grad_image, int grad_dtype, int B,
                             int N, int C, int H, int W, int k, float *grad_params,
                             void *workspace, size_t workspace_bytes,
                             int workspace_holds_fwd_bins, void *stream) {
    Geom g;
    pdr_status st = make_geom(B, N, C, H, W, k, &g);
    if (st != PDR_OK) return st;
    if (!params_ok(g, params) || !grad_image || !params_ok(g, grad_params) ||
        !aligned4(params) || !dtype_ok(grad_dtype, grad_image) || !aligned4(grad_params))
        return PDR_ERR_INVALID_ARG;
    Layout L;
    st = check_ws(g, workspace, workspace_bytes, &L);
    if (st != PDR_OK) return st;
    if (g.N == 0) return PDR_OK;  // no Gaussians: no gradients to write
    const Workspace ws = carve(workspace, L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    g.img_dtype = grad_dtype;
    // Four consecutive dL/dI elements per vector load: rows of a multiple of 4
    // elements and an image aligned to 4 elements (16 bytes fp32, 8 bytes half).
    g.stage_vec4 = (g.W & 3) == 0 &&
                   (reinterpret_cast<uintptr_t>(grad_image) & (grad_dtype == PDR_F32 ? 15 : 7)) == 0;
    if (!workspace_holds_fwd_bins) {
        st = from_cuda(bin(params, g, ws, s));
        if (st != PDR_OK) return st;
    }
    return from_cuda(launch_bwd(params, grad_image, g, ws, grad_params, s));
}

pdr_status pdr_render_bwd(const float *params, const float *grad_image, int B, int N, int C,
                          int H, int W, int k, float *grad_params, void *workspace,
                          size_t workspace_bytes, int workspace_holds_fwd_bins,
                          void *stream) {
    return pdr_render_bwd_ex(params, grad_image, PDR_F32, B, N, C, H, W, k, grad_params,
                             workspace, workspace_bytes, workspace_holds_fwd_bins, stream);
}

pdr_status pdr_bin(const float *params, int B, int N, int C, int H, int W, int k,
                   int *tile_offsets, int *tile_ids, void *workspace, size_t workspace_bytes,
                   void *stream) {
    Geom g;
    pdr_status st = make_geom(B, N, C, H, W, k, &g);
    if (st != PDR_OK) return st;
    if (!params_ok(g, params) || !tile_offsets || (g.N > 0 && !tile_ids) || !aligned4(params))
        return PDR_ERR_INVALID_ARG;
    Layout L;
    st = check_ws(g, workspace, workspace_bytes, &L);
    if (st != PDR_OK) return st;
    const Workspace ws = carve(workspace, L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = from_cuda(bin(params, g, ws, s));
    if (st != PDR_OK) return st;
    st = from_cuda(cudaMemcpyAsync(tile_offsets, ws.offs, sizeof(int) * (size_t)g.B * (g.T + 1),
                                   cudaMemcpyDeviceToDevice, s));
    if (st != PDR_OK || g.cap == 0) return st;
    // The lists as frame-local ids (the workspace copy also marks each
    // Gaussian's home-tile entry for the backward pass).
    return from_cuda(launch_copy_ids(tile_ids, ws.ids, (size_t)g.B * g.cap, s));
}

pdr_status pdr_workspace_part(int B, int N, int C, int H, int W, int k, int part,
                              size_t *offset, size_t *bytes) {
    Geom g;
    pdr_status st = make_geom(B, N, C, H, W, k, &g);
    if (st != PDR_OK) return st;
    if (!offset || !bytes) return PDR_ERR_INVALID_ARG;
    const Layout L = make_layout(g);
    switch (part) {
        case PDR_WS_ERROR_WORD: *offset = L.err; *bytes = sizeof(int); return PDR_OK;
        case PDR_WS_RECORDS: *offset = L.gr; *bytes = L.hist - L.gr; return PDR_OK;
        case PDR_WS_TILE_OFFSETS:
            *offset = L.offs;
            *bytes = sizeof(int) * (size_t)g.B * (g.T + 1);
            return PDR_OK;
        case PDR_WS_TILE_IDS:
            *offset = L.ids;
            *bytes = sizeof(int) * (size_t)g.B * g.cap;
            return PDR_OK;
        default: return PDR_ERR_INVALID_ARG;
    }
}

pdr_status pdr_step_host(const float *h_params, const float *h_grad_image, float *h_image,
                         float *h_grad_params, int B, int N, int C, int H, int W, int k,
                         float *d_params, float *d_grad_image, float *d_image,
                         float *d_grad_params, void *workspace, size_t workspace_bytes,
                         void *stream) {
    Geom g;
    pdr_status st = make_geom(B, N, C, H, W, k, &g);
    if (st != PDR_OK) return st;
    if (!params_ok(g, h_params) || !h_grad_image || !h_image || !params_ok(g, h_grad_params) ||
        !params_ok(g, d_params) || !d_grad_image || !d_image || !params_ok(g, d_grad_params))
        return PDR_ERR_INVALID_ARG;
    Layout L;
    st = check_ws(g, workspace, workspace_bytes, &L);
    if (st != PDR_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    StepSide *side = nullptr;
    st = from_cuda(step_side(&side));
    if (st != PDR_OK) return st;
    cudaStream_t up = side->up, down = side->down;
    cudaEvent_t *ev = side->ev;
    // Frames are independent, so the step runs in up to kStepChunks chunks of
    // consecutive frames, pipelined over three streams:
    //   up:     params_c H2D, dL/dI_c H2D, for c = 0, 1, ...
    //   stream: forward_c (bins inside) after params_c, backward_c after
    //           dL/dI_c (reusing forward_c's bins), chunk after chunk
    //   down:   image_c D2H after forward_c, grads_c D2H after backward_c
    // so that the downloads of early chunks run while later chunks upload
    // (PCIe carries both directions at once).  Every chunk's results are those
    // of the whole batch (each frame is rendered from its own lists), and the
    // workspace, used by one chunk at a time on `stream`, is reused.  `up`
    // starts after everything already on `stream`, so a previous step is done
    // with the device buffers before they are overwritten; `stream` joins both
    // side streams before the call's last operation.
    const size_t pframe = (size_t)N * g.P, iframe = (size_t)C * H * W;  // floats per frame
    // Steps that move under 8 MB each way are bound by fixed per-copy and
    // per-launch latencies, which chunking would multiply: one chunk.
    const bool small = sizeof(float) * (size_t)B * (pframe + iframe) < kStepChunkMinBytes;
    const int nch = small ? 1 : (B < kStepChunks ? B : kStepChunks);
    cudaEvent_t ev_start = ev[0], ev_end = ev[1];
    pdr_status st_out = PDR_OK;
    cudaError_t e = cudaEventRecord(ev_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(up, ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(down, ev_start, 0);
    for (int c = 0; c < nch && e == cudaSuccess && st_out == PDR_OK; ++c) {
        const int b0 = (int)((long long)B * c / nch), b1 = (int)((long long)B * (c + 1) / nch);
        const int Bc = b1 - b0;
        cudaEvent_t ev_p = ev[2 + 4 * c], ev_g = ev[3 + 4 * c];
        cudaEvent_t ev_f = ev[4 + 4 * c], ev_b = ev[5 + 4 * c];
        const size_t po = (size_t)b0 * pframe, io = (size_t)b0 * iframe;
        const size_t pbytes = sizeof(float) * (size_t)Bc * pframe;
        const size_t ibytes = sizeof(float) * (size_t)Bc * iframe;
        if (pbytes) e = cudaMemcpyAsync(d_params + po, h_params + po, pbytes, cudaMemcpyHostToDevice, up);
        if (e == cudaSuccess) e = cudaEventRecord(ev_p, up);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(d_grad_image + io, h_grad_image + io, ibytes, cudaMemcpyHostToDevice, up);
        if (e == cudaSuccess) e = cudaEventRecord(ev_g, up);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_p, 0);
        if (e != cudaSuccess) break;
        st_out = render_fwd_in_batch(d_params + po, Bc, N, C, H, W, k, d_image + io, PDR_F32,
                                     workspace, workspace_bytes, 0, stream, B);
        if (st_out != PDR_OK) break;
        e = cudaEventRecord(ev_f, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(down, ev_f, 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(h_image + io, d_image + io, ibytes, cudaMemcpyDeviceToHost, down);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_g, 0);
        if (e != cudaSuccess) break;
        st_out = pdr_render_bwd(d_params + po, d_grad_image + io, Bc, N, C, H, W, k,
                                d_grad_params + po, workspace, workspace_bytes, 1, stream);
        if (st_out != PDR_OK) break;
        e = cudaEventRecord(ev_b, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(down, ev_b, 0);
        if (e == cudaSuccess && pbytes)
            e = cudaMemcpyAsync(h_grad_params + po, d_grad_params + po, pbytes,
                                cudaMemcpyDeviceToHost, down);
    }
    // Join both side streams whatever happened, so that `stream` covers their copies.
    cudaError_t ej = cudaEventRecord(ev_end, up);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, ev_end, 0);
    if (ej == cudaSuccess) ej = cudaEventRecord(ev_end, down);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, ev_end, 0);
    if (st_out != PDR_OK) return st_out;
    if (e != cudaSuccess || ej != cudaSuccess) return PDR_ERR_CUDA;
    return PDR_OK;
}

pdr_status pdr_check_device_error(void *workspace, void *stream) {
    if (!workspace) return PDR_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return PDR_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return PDR_ERR_CUDA;
    if (word != 0) {
        if (cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return PDR_ERR_CUDA;
        return PDR_ERR_INTERNAL;
    }
    return PDR_OK;
}

}  // extern "C"
