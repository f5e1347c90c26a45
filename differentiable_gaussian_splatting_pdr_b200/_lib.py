"""ctypes binding of libpdr.so (C ABI in include/pdr.h).

Argument marshalling only: every step of the renderer runs in the library's
CUDA kernels.  If the library cannot be loaded, every entry point raises;
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpdr.so")

PDR_OK = 0
STATUS_NAMES = {
    0: "PDR_OK",
    1: "PDR_ERR_INVALID_ARG",
    2: "PDR_ERR_WORKSPACE_TOO_SMALL",
    3: "PDR_ERR_CUDA",
    4: "PDR_ERR_DEVICE_TIMEOUT",
    5: "PDR_ERR_INTERNAL",
    6: "PDR_ERR_TOO_LARGE",
}

STATUS_CODES = {name: code for code, name in STATUS_NAMES.items()}

# Every symbol include/pdr.h declares, with (restype, argtypes).
_vp, _i, _sz, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
SIGNATURES = {
    "pdr_abi_version": (_i, []),
    "pdr_status_string": (ctypes.c_char_p, [_i]),
    "pdr_workspace_bytes": (_sz, [_i] * 6),
    "pdr_list_capacity_per_frame": (_ll, [_i, _i]),
    "pdr_build_bins": (_i, [_vp] + [_i] * 6 + [_vp, _sz, _vp]),
    "pdr_render_fwd": (_i, [_vp] + [_i] * 6 + [_vp, _vp, _sz, _i, _vp]),
    "pdr_render_bwd": (_i, [_vp, _vp] + [_i] * 6 + [_vp, _vp, _sz, _i, _vp]),
    "pdr_bin": (_i, [_vp] + [_i] * 6 + [_vp, _vp, _vp, _sz, _vp]),
    "pdr_step_host": (_i, [_vp, _vp, _vp, _vp] + [_i] * 6 + [_vp] * 5 + [_sz, _vp]),
    "pdr_check_device_error": (_i, [_vp, _vp]),
    "pdr_render_fwd_noalloc": (_i, [_vp] + [_i] * 6 + [_vp, _vp]),
    "pdr_check_device_error_noalloc": (_i, [_vp]),
    "pdr_workspace_part": (_i, [_i] * 7 + [ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "pdr_loss_workspace_bytes": (_sz, [_i] * 4),
    "pdr_render_fwd_ex": (_i, [_vp] + [_i] * 6 + [_vp, _i, _vp, _sz, _i, _vp]),
    "pdr_render_bwd_ex": (_i, [_vp, _vp, _i] + [_i] * 6 + [_vp, _vp, _sz, _i, _vp]),
    "pdr_loss_l1_ssim": (_i, [_vp, _vp] + [_i] * 4 + [ctypes.c_float, ctypes.c_float] + [_vp] * 3 + [_sz, _vp]),
}

_lib = None


class PdrError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = STATUS_NAMES.get(status, "status %d" % status)
        if _lib is not None:
            try:
                msg = _lib.pdr_status_string(status).decode()
            except Exception:  # pragma: no cover - diagnostic only
                pass
        super().__init__("%s failed: %s" % (fn, msg))


def load(path: str = LIB_PATH):
    """Load libpdr.so once; raise (never fall back) if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            "libpdr.so not found at %s: build it with "
            "`python -m differentiable_gaussian_splatting_pdr_b200.build`" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != PDR_OK:
        raise PdrError(fn, status)
