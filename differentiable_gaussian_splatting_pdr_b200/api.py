"""PyTorch-facing API of the renderer: device memory and streams only.

    image = render(params, H, W, k)           # differentiable (autograd)
    image, ws = render_fwd(params, H, W, k)   # forward, bins kept in ws
    grad = render_bwd(params, grad_image, H, W, k, ws)

params is a contiguous fp32 CUDA tensor [B, N, 5 + C] holding, per Gaussian,
(mu_x, mu_y, s_1, s_2, theta, a_0 .. a_{C-1}) -- the "5 + C learnable
parameters (position, scale, rotation, and C channel amplitudes)" of the
paper's abstract.  Images are [B, C, H, W].  Every call enqueues the
library's kernels on the current torch stream; nothing is computed here.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_params(params: torch.Tensor):
    if not isinstance(params, torch.Tensor) or not params.is_cuda:
        raise ValueError("params must be a CUDA tensor")
    if params.dtype != torch.float32 or params.dim() != 3 or params.shape[2] < 6:
        raise ValueError("params must be fp32 [B, N, 5 + C] with C >= 1")
    if not params.is_contiguous():
        raise ValueError("params must be contiguous")
    B, N, P = params.shape
    return B, N, P - 5


def workspace_bytes(B: int, N: int, C: int, H: int, W: int, k: int) -> int:
    n = _lib.load().pdr_workspace_bytes(B, N, C, H, W, k)
    if n == 0:
        raise ValueError("invalid or unsupported sizes B=%d N=%d C=%d H=%d W=%d k=%d"
                         % (B, N, C, H, W, k))
    return int(n)


def list_capacity_per_frame(N: int, k: int) -> int:
    return int(_lib.load().pdr_list_capacity_per_frame(N, k))


@dataclass
class Workspace:
    """Caller-owned device workspace (tile bins and per-Gaussian records)."""
    buf: torch.Tensor
    shape: tuple  # (B, N, C, H, W, k) the bins in it were built for, or ()

    @staticmethod
    def for_sizes(B, N, C, H, W, k, device) -> "Workspace":
        n = workspace_bytes(B, N, C, H, W, k)
        return Workspace(torch.empty(n, dtype=torch.uint8, device=device), ())

    def fits(self, B, N, C, H, W, k) -> bool:
        return self.buf.numel() >= workspace_bytes(B, N, C, H, W, k)


def _workspace(ws, B, N, C, H, W, k, device) -> Workspace:
    if ws is None or not ws.fits(B, N, C, H, W, k) or ws.buf.device != device:
        ws = Workspace.for_sizes(B, N, C, H, W, k, device)
    return ws


def build_bins(params: torch.Tensor, H: int, W: int, k: int,
               workspace: Workspace | None = None) -> Workspace:
    """Bin the Gaussians into 16x16 tiles inside a (new or given) workspace."""
    B, N, C = _check_params(params)
    dev = params.device
    ws = _workspace(workspace, B, N, C, H, W, k, dev)
    lib = _lib.load()
    _lib.check("pdr_build_bins", lib.pdr_build_bins(
        _ptr(params), B, N, C, H, W, k, _ptr(ws.buf), ws.buf.numel(), _stream(dev)))
    ws.shape = (B, N, C, H, W, k)
    return ws


# Image storage types of the _ex entry points (pdr_dtype in include/pdr.h).
_DTYPES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


def render_fwd(params: torch.Tensor, H: int, W: int, k: int, workspace: Workspace | None = None,
               out: torch.Tensor | None = None, reuse_bins: bool = False,
               dtype: torch.dtype = torch.float32):
    """Forward render; returns (image [B, C, H, W], workspace holding the bins).

    reuse_bins=True renders from the bins already in `workspace` (built by
    build_bins or an earlier call on the same params and sizes).  dtype
    float16 / bfloat16 stores the image in that type (fp32 sums, rounded once)."""
    B, N, C = _check_params(params)
    dev = params.device
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32, float16 or bfloat16")
    holds = bool(reuse_bins and workspace is not None and workspace.shape == (B, N, C, H, W, k))
    ws = _workspace(workspace, B, N, C, H, W, k, dev)
    if ws is not workspace:
        holds = False
    if out is None:
        out = torch.empty((B, C, H, W), dtype=dtype, device=dev)
    elif out.shape != (B, C, H, W) or out.dtype != dtype or not out.is_contiguous():
        raise ValueError("out must be contiguous %s [B, C, H, W]" % dtype)
    lib = _lib.load()
    _lib.check("pdr_render_fwd_ex", lib.pdr_render_fwd_ex(
        _ptr(params), B, N, C, H, W, k, _ptr(out), _DTYPES[dtype], _ptr(ws.buf), ws.buf.numel(),
        1 if holds else 0, _stream(dev)))
    ws.shape = (B, N, C, H, W, k)
    return out, ws


def render_bwd(params: torch.Tensor, grad_image: torch.Tensor, H: int, W: int, k: int,
               workspace: Workspace | None = None, out: torch.Tensor | None = None,
               reuse_bins: bool = True) -> torch.Tensor:
    """dL/dparams [B, N, 5 + C] from dL/dI [B, C, H, W].

    reuse_bins=True uses the bins a render_fwd on the same params left in
    `workspace`; otherwise (or without a matching workspace) they are rebuilt."""
    B, N, C = _check_params(params)
    dev = params.device
    if grad_image.shape != (B, C, H, W) or grad_image.dtype not in _DTYPES or not grad_image.is_cuda:
        raise ValueError("grad_image must be a float32 / float16 / bfloat16 CUDA [B, C, H, W]")
    grad_image = grad_image.contiguous()
    holds = bool(reuse_bins and workspace is not None and workspace.shape == (B, N, C, H, W, k))
    ws = _workspace(workspace, B, N, C, H, W, k, dev)
    if ws is not workspace:
        holds = False
    if out is None:
        out = torch.empty_like(params)
    lib = _lib.load()
    _lib.check("pdr_render_bwd_ex", lib.pdr_render_bwd_ex(
        _ptr(params), _ptr(grad_image), _DTYPES[grad_image.dtype], B, N, C, H, W, k, _ptr(out),
        _ptr(ws.buf), ws.buf.numel(), 1 if holds else 0, _stream(dev)))
    ws.shape = (B, N, C, H, W, k)
    return out


def check_device_error(ws: Workspace, device=None) -> None:
    """Synchronise the stream and raise if a kernel's own check fired."""
    device = ws.buf.device if device is None else device
    _lib.check("pdr_check_device_error",
               _lib.load().pdr_check_device_error(_ptr(ws.buf), _stream(device)))


# Parts of the workspace (pdr_ws_part in include/pdr.h).
WS_PARTS = {"error_word": 0, "records": 1, "tile_offsets": 2, "tile_ids": 3}


def workspace_part(B: int, N: int, C: int, H: int, W: int, k: int, part: str):
    """(byte offset, bytes) of a part of the workspace for these sizes."""
    import ctypes
    off, n = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _lib.check("pdr_workspace_part", _lib.load().pdr_workspace_part(
        B, N, C, H, W, k, WS_PARTS[part], ctypes.byref(off), ctypes.byref(n)))
    return int(off.value), int(n.value)


def bin_tiles(params: torch.Tensor, H: int, W: int, k: int):
    """Tile lists as the library builds them.

    Returns (tile_offsets [B, T + 1] int32, tile_ids [B * cap] int32, cap):
    frame b's entries live in tile_ids[b * cap : (b + 1) * cap]; tile t of
    frame b is tile_ids[tile_offsets[b, t] : tile_offsets[b, t + 1]]."""
    B, N, C = _check_params(params)
    dev = params.device
    T = ((H + 15) // 16) * ((W + 15) // 16)
    cap = list_capacity_per_frame(N, k)
    ws = Workspace.for_sizes(B, N, C, H, W, k, dev)
    offs = torch.empty((B, T + 1), dtype=torch.int32, device=dev)
    ids = torch.empty(B * cap, dtype=torch.int32, device=dev)
    lib = _lib.load()
    _lib.check("pdr_bin", lib.pdr_bin(_ptr(params), B, N, C, H, W, k, _ptr(offs), _ptr(ids),
                                      _ptr(ws.buf), ws.buf.numel(), _stream(dev)))
    check_device_error(ws)
    return offs, ids, cap


def step_host(h_params: torch.Tensor, h_grad_image: torch.Tensor, H: int, W: int, k: int,
              dev_bufs: dict | None = None, device=None):
    """One forward + backward pass from host (ideally pinned) tensors.

    Copies inputs to the device, renders, back-propagates dL/dI, and copies the
    image and dL/dparams back, all enqueued by one C-ABI call (pdr_step_host):
    the dL/dI upload and the image download overlap the render on a side
    stream of the library that the current stream joins.  Returns (h_image,
    h_grad_params, dev_bufs); the host outputs are valid after the current
    stream is synchronised.  N = 0 (no Gaussians) gives a zero image."""
    if h_params.is_cuda or h_grad_image.is_cuda:
        raise ValueError("step_host takes host tensors")
    B, N, P = h_params.shape
    C = P - 5
    device = torch.device(device or "cuda")
    if dev_bufs is None:
        dev_bufs = {
            "params": torch.empty((B, N, P), dtype=torch.float32, device=device),
            "grad_image": torch.empty((B, C, H, W), dtype=torch.float32, device=device),
            "image": torch.empty((B, C, H, W), dtype=torch.float32, device=device),
            "grad_params": torch.empty((B, N, P), dtype=torch.float32, device=device),
            "ws": Workspace.for_sizes(B, N, C, H, W, k, device),
            "h_image": torch.empty((B, C, H, W), dtype=torch.float32, pin_memory=True),
            "h_grad_params": torch.empty((B, N, P), dtype=torch.float32, pin_memory=True),
        }
    d = dev_bufs
    lib = _lib.load()
    _lib.check("pdr_step_host", lib.pdr_step_host(
        _ptr(h_params), _ptr(h_grad_image), _ptr(d["h_image"]), _ptr(d["h_grad_params"]),
        B, N, C, H, W, k, _ptr(d["params"]), _ptr(d["grad_image"]), _ptr(d["image"]),
        _ptr(d["grad_params"]), _ptr(d["ws"].buf), d["ws"].buf.numel(), _stream(device)))
    return d["h_image"], d["h_grad_params"], d


class _Render(torch.autograd.Function):
    @staticmethod
    def forward(ctx, params, H, W, k):
        image, ws = render_fwd(params, H, W, k)
        ctx.save_for_backward(params)
        ctx.ws = ws
        ctx.hwk = (H, W, k)
        return image

    @staticmethod
    def backward(ctx, grad_image):
        (params,) = ctx.saved_tensors
        H, W, k = ctx.hwk
        # fp16 / bf16 upstream gradients go to the library as they are (it
        # widens each element to fp32 on load); other types become fp32.
        if grad_image.dtype not in _DTYPES:
            grad_image = grad_image.float()
        grad = render_bwd(params, grad_image.contiguous(), H, W, k, ctx.ws, reuse_bins=True)
        ctx.ws = None
        return grad, None, None, None


def render(params: torch.Tensor, H: int, W: int, k: int) -> torch.Tensor:
    """Differentiable render: image [B, C, H, W] from params [B, N, 5 + C]."""
    return _Render.apply(params.contiguous(), H, W, k)


def loss_workspace_bytes(B: int, C: int, H: int, W: int) -> int:
    return int(_lib.load().pdr_loss_workspace_bytes(B, C, H, W))


def l1_ssim_loss(image: torch.Tensor, target: torch.Tensor, lam: float = 0.2,
                 data_range: float = 1.0, workspace: torch.Tensor | None = None,
                 grad_out: torch.Tensor | None = None, loss_out: torch.Tensor | None = None):
    """L1 + SSIM training loss and dL/dimage (see pdr_loss_l1_ssim).

    image, target: contiguous fp32 CUDA tensors [B, C, H, W].  Returns
    (loss, grad): a 1-element device tensor and a tensor like image.  The
    target receives no gradient."""
    lib = _lib.load()
    for t in (image, target):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 \
                or t.dim() != 4 or not t.is_contiguous():
            raise ValueError("image and target must be contiguous fp32 CUDA tensors [B, C, H, W]")
    if image.shape != target.shape:
        raise ValueError("image and target shapes differ")
    B, C, H, W = image.shape
    dev = image.device
    nb = loss_workspace_bytes(B, C, H, W)
    if workspace is None or workspace.numel() < nb:
        workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    grad = torch.empty_like(image) if grad_out is None else grad_out
    loss = torch.empty(1, dtype=torch.float32, device=dev) if loss_out is None else loss_out
    _lib.check("pdr_loss_l1_ssim", lib.pdr_loss_l1_ssim(
        _ptr(image), _ptr(target), B, C, H, W, float(lam), float(data_range), _ptr(loss),
        _ptr(grad), _ptr(workspace), workspace.numel(), _stream(dev)))
    return loss, grad


class _L1Ssim(torch.autograd.Function):
    @staticmethod
    def forward(ctx, image, target, lam, data_range):
        loss, grad = l1_ssim_loss(image, target, lam, data_range)
        ctx.save_for_backward(grad)
        return loss[0]

    @staticmethod
    def backward(ctx, g):
        (grad,) = ctx.saved_tensors
        return grad * g, None, None, None


def l1_ssim(image: torch.Tensor, target: torch.Tensor, lam: float = 0.2,
            data_range: float = 1.0) -> torch.Tensor:
    """Differentiable L1 + SSIM loss (scalar); dL/dimage flows to image."""
    return _L1Ssim.apply(image.contiguous(), target.contiguous(), lam, data_range)
