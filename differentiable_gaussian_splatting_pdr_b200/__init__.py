"""B200-native (sm_100a) additive, differentiable 2D Gaussian-splatting renderer.

The hot path of "Learning Video Dynamics with Predictive Differentiable
Rendering" (PDR): N anisotropic Gaussians per frame, each with 5 + C
parameters, accumulated additively into a C-channel H x W field, forward and
backward.  The kernels and their C ABI live in libpdr.so (include/pdr.h);
this package is the thin PyTorch binding around it.
"""
from .api import (  # noqa: F401
    Workspace,
    bin_tiles,
    build_bins,
    check_device_error,
    l1_ssim,
    l1_ssim_loss,
    list_capacity_per_frame,
    loss_workspace_bytes,
    render,
    render_bwd,
    render_fwd,
    step_host,
    workspace_bytes,
)
