/*
 * pdr.h -- C ABI of libpdr.so: the additive, differentiable 2D Gaussian
 * splatting renderer of "Learning Video Dynamics with Predictive
 * Differentiable Rendering" (PDR), forward and backward, for NVIDIA B200
 * (sm_100a).
 *
 * What is rendered (paper abstract: each Gaussian has "5 + C learnable
 * parameters (position, scale, rotation, and C channel amplitudes)"; reading
 * notes, "Method": the render is an additive accumulation; "Key Insight" and
 * "Limitation": the kernel size / support is a tuned knob):
 *
 *     I_c(p) = sum_i a_ic * exp(-1/2 (p - mu_i)^T Sigma_i^{-1} (p - mu_i)),
 *     Sigma_i = R(theta_i) diag(e^{2 s_i1}, e^{2 s_i2}) R(theta_i)^T,
 *
 * each Gaussian truncated to the k x k pixel window centred on round(mu_i)
 * (ties round up), window pixels outside the grid dropped.  Pixel (x, y) sits
 * at p = (x, y); x is the column, y the row; R(t) = [[cos t, -sin t],
 * [sin t, cos t]].  No opacity, no compositing, no depth order.
 *
 * Layouts (all fp32, row-major, device memory unless stated):
 *   params       [B][N][5+C]  per Gaussian (mu_x, mu_y, s_1, s_2, theta, a_0..a_{C-1})
 *   image        [B][C][H][W]
 *   grad_image   [B][C][H][W]  dL/dI
 *   grad_params  [B][N][5+C]   dL/dparams, same order as params
 *
 * Ownership: the caller allocates every buffer, including the workspace
 * (size from pdr_workspace_bytes); the library allocates no device memory.
 * Outputs are overwritten, never accumulated into.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  All work is enqueued on it and the calls return without waiting.
 * A PDR_ERR_CUDA return reports a launch error; errors during execution show
 * up at the caller's next synchronisation.
 *
 * Validation (host side, before anything is launched; on failure nothing is
 * launched and outputs are untouched): B, C, H, W >= 1 and N >= 0; k odd and
 * >= 1; sizes within the limits below (else PDR_ERR_TOO_LARGE); non-null
 * pointers, except that the arrays sized by N (params, grad_params, tile_ids)
 * may be NULL when N = 0; workspace_bytes >= pdr_workspace_bytes(...) and a
 * 256-byte aligned workspace.
 *
 * Frames with no Gaussians (N = 0) are the empty sum: the forward zeroes the
 * image and leaves empty bins, the backward writes nothing, pdr_bin writes
 * all-zero offsets; no kernel is launched (stream-ordered memsets only).
 *
 * Numerics: fp32 arithmetic with a hardware base-2 exponential; fixed
 * summation order (every list is in ascending Gaussian id), so results are
 * bitwise reproducible run to run.  A Gaussian with a non-finite mean, or
 * whose window misses the grid, contributes nothing and receives zero
 * gradients; other non-finite parameters propagate NaN/Inf into that
 * Gaussian's window pixels and its own gradients.  mu is clamped to
 * [-2^24, 2^24] before the window centre is taken.  No gradient flows through
 * round(mu) (the window position is piecewise constant in mu).
 */
#ifndef PDR_H
#define PDR_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PDR_OK = 0,
    PDR_ERR_INVALID_ARG = 1,          /* bad size, even k, null pointer, misaligned workspace */
    PDR_ERR_WORKSPACE_TOO_SMALL = 2,  /* workspace_bytes < pdr_workspace_bytes(...) */
    PDR_ERR_CUDA = 3,                 /* a CUDA runtime call or launch failed */
    PDR_ERR_DEVICE_TIMEOUT = 4,       /* reserved: a bounded device-side wait gave up */
    PDR_ERR_INTERNAL = 5,             /* a device-side consistency check failed */
    PDR_ERR_TOO_LARGE = 6             /* sizes beyond the limits below */
} pdr_status;

/* Library limits (checked on the host). */
#define PDR_TILE 16                    /* tile edge in pixels */
#define PDR_MAX_C 8                    /* channels */
#define PDR_MAX_K 31                   /* window size */
#define PDR_MAX_TILES_PER_FRAME 16384  /* ceil(H/16) * ceil(W/16) */

/* ABI version of this header (bumped on any incompatible change). */
int pdr_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *pdr_status_string(pdr_status s);

/* Bytes of device workspace that pdr_render_fwd / pdr_render_bwd / pdr_bin
 * need for these sizes; 0 if the sizes are invalid or beyond the limits.
 * Computed on the host from a worst-case bound (every Gaussian touching the
 * most tiles a k x k window can touch), so no device-to-host synchronisation
 * is ever needed to size the tile lists. */
size_t pdr_workspace_bytes(int B, int N, int C, int H, int W, int k);

/* Tile binning into the workspace (no rendering): every Gaussian enters the
 * list of each 16x16 tile its clipped window touches, lists in ascending
 * Gaussian id, together with a per-Gaussian record (window centre, rotated and
 * scaled axes).  The window is the k x k "kernel support" of the reading
 * notes ("Key Insight", "Limitation"); the ascending order gives every sum a
 * fixed order (the additive accumulation itself has none).  The bins stay
 * valid for pdr_render_fwd / pdr_render_bwd on the same params and sizes. */
pdr_status pdr_build_bins(const float *params, int B, int N, int C, int H, int W,
                          int k, void *workspace, size_t workspace_bytes,
                          void *stream);

/* Forward render (abstract: "differentiable 2D Gaussian renderer supporting
 * arbitrary channels"; reading notes, "Method": additive accumulation).
 * Writes image[B][C][H][W].  workspace_holds_bins = 1 uses the bins that
 * pdr_build_bins (or a previous call) left in this workspace for the same
 * params and sizes; 0 bins first.  The bins stay valid in the workspace for a
 * following pdr_render_bwd on the same params and sizes. */
pdr_status pdr_render_fwd(const float *params, int B, int N, int C, int H, int W,
                          int k, float *image, void *workspace,
                          size_t workspace_bytes, int workspace_holds_bins,
                          void *stream);

/* Backward pass: dL/dparams from dL/dI (abstract: "differentiable").
 * grad_params[B][N][5+C] = (dL/dmu_x, dL/dmu_y, dL/ds_1, dL/ds_2,
 * dL/dtheta, dL/da_0 .. dL/da_{C-1}) for every Gaussian.
 * workspace_holds_fwd_bins = 1 reuses the bins a preceding pdr_render_fwd,
 * pdr_build_bins or pdr_bin left in this workspace for the same params and
 * sizes; 0 re-bins first. */
pdr_status pdr_render_bwd(const float *params, const float *grad_image, int B,
                          int N, int C, int H, int W, int k, float *grad_params,
                          void *workspace, size_t workspace_bytes,
                          int workspace_holds_fwd_bins, void *stream);

/* Tile binning only (exported for tests and tools).  Each frame b owns the
 * list region [b * cap, (b + 1) * cap) of tile_ids, with
 * cap = pdr_list_capacity_per_frame(N, k).  tile_offsets[b * (T + 1) + t] is
 * the absolute start of tile t of frame b (T = tiles per frame, row-major);
 * tile_offsets[b * (T + 1) + T] is the end of frame b's entries.  Entries are
 * frame-local Gaussian indices, ascending within each tile.
 * tile_offsets: [B * (T + 1)] int32, tile_ids: [B * cap] int32, device. */
pdr_status pdr_bin(const float *params, int B, int N, int C, int H, int W, int k,
                   int *tile_offsets, int *tile_ids, void *workspace,
                   size_t workspace_bytes, void *stream);

/* List capacity per frame used by pdr_bin: N times the most 16x16 tiles a
 * k x k window can touch. */
long long pdr_list_capacity_per_frame(int N, int k);

/* One whole step from HOST memory, for callers whose data lives on the host:
 * copies h_params and h_grad_image to the caller's device buffers d_params and
 * d_grad_image, renders forward into d_image, runs the backward into
 * d_grad_params, and copies the image and the gradients back to h_image and
 * h_grad_params (cudaMemcpyAsync; pinned host memory makes the copies
 * asynchronous).  A step that moves 8 MB or more each way is processed in up
 * to 4 chunks of consecutive frames, pipelined: the uploads (params, then dL/dI, chunk after chunk) run on
 * one side stream of the library, the forward and backward of each chunk on
 * `stream` (results bitwise those of one call over all frames; the workspace
 * is reused chunk after chunk), and the downloads (image after the chunk's
 * forward, gradients after its backward) on a second side stream, so that
 * early chunks download while later ones upload.  The side streams (one pair
 * per host thread and device, created on first use) start after the work
 * already on `stream`, which joins both before the call's last operation.  The call returns after enqueueing; synchronise
 * `stream` before reading h_image / h_grad_params. */
pdr_status pdr_step_host(const float *h_params, const float *h_grad_image,
                         float *h_image, float *h_grad_params, int B, int N,
                         int C, int H, int W, int k, float *d_params,
                         float *d_grad_image, float *d_image,
                         float *d_grad_params, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Bytes of the library's built-in device scratch (see pdr_render_fwd_noalloc). */
#define PDR_STATIC_SCRATCH_BYTES (16u << 20)

/* Forward render without any caller-provided workspace, for callers that
 * cannot allocate device memory -- e.g. a plugin whose host application owns
 * all device memory through its own pool, or a real-time loop that must not
 * allocate after start-up.  The paper has no counterpart (this is an interface
 * convenience, not a step of the method).
 *
 * Same inputs, output and numerics as pdr_render_fwd (params and image are the
 * caller's device buffers); the bins live in a scratch array compiled into the
 * library, PDR_STATIC_SCRATCH_BYTES (16 MiB) on every GPU that loads the
 * library, held until the process exits.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine.
 *   - Sizes whose pdr_workspace_bytes(...) exceeds PDR_STATIC_SCRATCH_BYTES
 *     (e.g. 16 frames of 64x64 with 1024 Gaussians each fit; 320 frames of
 *     32x64 with 2048 each do not) return PDR_ERR_TOO_LARGE; bad sizes or null
 *     pointers return PDR_ERR_INVALID_ARG; nothing is launched then.
 *   - The first call made with a given device current looks up the scratch's
 *     device address (cudaGetSymbolAddress) and caches it; make that first
 *     call before any stream capture.
 *   - All calls on a device share the one scratch, which keeps the last
 *     call's contents.  Each call rebuilds everything it reads (its device
 *     error word included, cleared before its first kernel), so nothing
 *     needs clearing, but calls that overlap on the GPU (other streams, other
 *     host threads) race on it: serialise them.
 *   - The kernels' own bounds checks report into that scratch's error word;
 *     pdr_check_device_error_noalloc reads it. */
pdr_status pdr_render_fwd_noalloc(const float *params, int B, int N, int C, int H,
                                  int W, int k, float *image, void *stream);

/* pdr_check_device_error for the built-in scratch of pdr_render_fwd_noalloc
 * on the current device: synchronises `stream`, returns PDR_ERR_INTERNAL if a
 * kernel's bounds check fired since the last call of pdr_render_fwd_noalloc
 * began, and clears the word.  Allocates nothing. */
pdr_status pdr_check_device_error_noalloc(void *stream);

/* ---- Reduced-precision image storage ------------------------------------------
 * Image and dL/dI stored as fp16 or bf16 (half the bytes of the two largest
 * tensors), every sum still in fp32: the forward rounds each pixel's fp32
 * total to the storage type once (round to nearest even), the backward
 * widens each dL/dI element to fp32 on load.  Motivated by the mixed-precision
 * study of the hardware-rasterizer page ("contour-based differentiable
 * rendering"); params and grad_params stay fp32 (small, and mu feeds the
 * exact window centre).  The fp16/bf16 image of pdr_render_fwd_ex equals the
 * fp32 image of pdr_render_fwd rounded to that type. */
typedef enum { PDR_F32 = 0, PDR_F16 = 1, PDR_BF16 = 2 } pdr_dtype;

/* pdr_render_fwd with the image stored as image_dtype (a pdr_dtype; the
 * image pointer aligned to its element size).  pdr_render_fwd(...) is
 * pdr_render_fwd_ex(..., image, PDR_F32, ...).  An unknown dtype returns
 * PDR_ERR_INVALID_ARG. */
pdr_status pdr_render_fwd_ex(const float *params, int B, int N, int C, int H, int W, int k,
                             void *image, int image_dtype, void *workspace,
                             size_t workspace_bytes, int workspace_holds_bins, void *stream);

/* pdr_render_bwd with dL/dI stored as grad_dtype (a pdr_dtype). */
pdr_status pdr_render_bwd_ex(const float *params, const void *grad_image, int grad_dtype, int B,
                             int N, int C, int H, int W, int k, float *grad_params,
                             void *workspace, size_t workspace_bytes,
                             int workspace_holds_fwd_bins, void *stream);

/* Synchronises `stream` and reports the device-side error word in the
 * workspace (PDR_ERR_INTERNAL if a kernel's own bounds check fired), then
 * clears it.  The word is also cleared, stream-ordered, by every call that
 * bins (pdr_build_bins, pdr_bin, and the render calls with their
 * workspace_holds_*bins flag at 0) before its first kernel; kernels only ever
 * set bits in it, so a bit set by any kernel since the last binning stays set
 * until it is read here. */
pdr_status pdr_check_device_error(void *workspace, void *stream);

/* Where a part of the workspace lies, for tools and tests that inspect or
 * plant values in it: byte offset from the workspace start and size in bytes
 * of part `part` (a pdr_ws_part) for these sizes.  The tile offsets are
 * int32 [B][T + 1] absolute list positions (as pdr_bin returns them); the
 * tile ids are int32 [B * cap] entries whose bit 31 marks the one entry of
 * each Gaussian in the list of its home tile (the tile of its window centre
 * clamped to the grid), bits 0..30 the frame-local id.  Returns
 * PDR_ERR_INVALID_ARG for an unknown part or null outputs, and the sizes'
 * own validation errors. */
typedef enum {
    PDR_WS_ERROR_WORD = 0,
    PDR_WS_RECORDS = 1,
    PDR_WS_TILE_OFFSETS = 2,
    PDR_WS_TILE_IDS = 3
} pdr_ws_part;
pdr_status pdr_workspace_part(int B, int N, int C, int H, int W, int k, int part,
                              size_t *offset, size_t *bytes);

/* ---- Training loss: L1 + SSIM, producing dL/dI ------------------------------
 * The objective the reading notes (section "Method", third point; "Key
 * Insight / Why It Works") name as essential for PDR: an L1 term plus a
 * structural-similarity term.  The pages give no weights or SSIM constants;
 * the library takes the usual Gaussian-splatting ones:
 *
 *   L = (1 - lam) mean|I - T| + lam (1 - mean SSIM(I, T)),
 *
 * SSIM computed per (frame, channel) image with an 11 x 11 Gaussian window
 * (sigma 1.5, taps normalised to sum 1), zero padding at the borders (maps of
 * the image's size), C1 = (0.01 data_range)^2, C2 = (0.03 data_range)^2; the
 * means run over all B*C*H*W elements.  dL/dI is the exact derivative of that
 * definition (sign(0) = 0 for the L1 term); T gets no gradient. */

/* Workspace bytes for pdr_loss_l1_ssim (per-block partial sums); 0 if the
 * sizes are invalid. */
size_t pdr_loss_workspace_bytes(int B, int C, int H, int W);

/* image, target: [B][C][H][W] fp32 device; lam in [0, 1] (0.2 is the usual
 * choice); data_range > 0 (1 for images in [0, 1]).  Writes the scalar loss to
 * `loss` (one fp32 on the device) and dL/dimage to grad_image
 * ([B][C][H][W], overwritten; it may not alias image or target).  The
 * workspace (device, 256-byte aligned, pdr_loss_workspace_bytes) holds
 * per-block partial sums, added in a fixed order: bitwise reproducible.
 * Errors: PDR_ERR_INVALID_ARG for sizes < 1, lam outside [0, 1], a
 * non-positive or non-finite data_range, null or misaligned pointers;
 * PDR_ERR_WORKSPACE_TOO_SMALL; nothing is launched then.  Asynchronous on
 * `stream` like the render calls. */
pdr_status pdr_loss_l1_ssim(const float *image, const float *target, int B, int C, int H,
                            int W, float lam, float data_range, float *loss, float *grad_image,
                            void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PDR_H */
