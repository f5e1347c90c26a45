"""Host-side tests of the C-ABI boundary: the library loads and exports every
symbol include/pdr.h declares, validation rejects bad arguments before any
launch, and the workspace / capacity arithmetic matches brute force.  No
kernel runs here."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from differentiable_gaussian_splatting_pdr_b200 import _lib, build as pdr_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pdr.h")


@pytest.fixture(scope="module")
def lib():
    pdr_build.build()
    return _lib.load()


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pdr_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ["pdr_render_fwd", "pdr_render_bwd", "pdr_workspace_bytes", "pdr_bin",
              "pdr_status_string", "pdr_step_host"]:
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert set(syms) == set(_lib.SIGNATURES), "binding and header disagree"
    for s in syms:
        assert hasattr(lib, s), s
    assert lib.pdr_abi_version() == 1


def test_status_strings(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.pdr_status_string(code).decode().startswith(name)
    assert b"unknown" in lib.pdr_status_string(99)


@pytest.mark.parametrize("args", [
    (0, 10, 1, 32, 32, 7), (1, -1, 1, 32, 32, 7), (1, 10, 0, 32, 32, 7),
    (1, 10, 1, 0, 32, 7), (1, 10, 1, 32, 0, 7), (1, 10, 1, 32, 32, 0),
    (1, 10, 1, 32, 32, 8), (1, 10, 1, 32, 32, -3),
    (1, 10, 9, 32, 32, 7),            # C beyond PDR_MAX_C
    (1, 10, 1, 32, 32, 33),           # k beyond PDR_MAX_K
    (1, 10, 1, 4096, 4096, 7),        # more tiles per frame than allowed
])
def test_workspace_bytes_rejects_bad_sizes(lib, args):
    assert lib.pdr_workspace_bytes(*args) == 0


def test_frames_without_gaussians_are_valid_sizes(lib):
    """N = 0 (the empty sum) is accepted: a workspace for the bins' offsets, no
    list capacity."""
    n0 = lib.pdr_workspace_bytes(3, 0, 2, 40, 24, 9)
    assert 0 < n0 < lib.pdr_workspace_bytes(3, 1, 2, 40, 24, 9)
    assert lib.pdr_list_capacity_per_frame(0, 9) == 0


def _max_tiles_touched(k):
    """Brute force: most 16-pixel tiles a run of k pixels can touch."""
    return max(len({x // 16 for x in range(s, s + k)}) for s in range(0, 64))


@pytest.mark.parametrize("k", [1, 3, 7, 9, 11, 15, 17, 19, 31])
def test_list_capacity_matches_brute_force(lib, k):
    m = _max_tiles_touched(k)
    assert lib.pdr_list_capacity_per_frame(100, k) == 100 * m * m


def test_workspace_bytes_grows_with_sizes(lib):
    a = lib.pdr_workspace_bytes(1, 64, 1, 32, 32, 7)
    b = lib.pdr_workspace_bytes(2, 64, 1, 32, 32, 7)
    c = lib.pdr_workspace_bytes(1, 128, 1, 32, 32, 7)
    d = lib.pdr_workspace_bytes(1, 64, 1, 32, 32, 31)   # 3x3 tiles per window
    assert 0 < a < b and a < c and a < d
    # worst case: every Gaussian in m*m lists
    assert a >= 4 * 64 * 4


# Fake, never-dereferenced pointers: every case below must fail host-side
# validation before anything is enqueued.  They are skipped where a GPU is
# visible, so that a validation bug can never launch a kernel on them.
no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers only without a GPU")
FAKE = 0x10000


@no_gpu
def test_fwd_validation_order(lib):
    ws = lib.pdr_workspace_bytes(1, 64, 1, 32, 32, 7)
    f = lib.pdr_render_fwd
    assert f(FAKE, 0, 64, 1, 32, 32, 7, FAKE, FAKE, ws, 0, None) == 1
    assert f(FAKE, 1, 64, 1, 32, 32, 6, FAKE, FAKE, ws, 0, None) == 1
    assert f(FAKE, 1, 64, 9, 32, 32, 7, FAKE, FAKE, ws, 0, None) == 6
    assert f(None, 1, 64, 1, 32, 32, 7, FAKE, FAKE, ws, 0, None) == 1
    assert f(FAKE, 1, 64, 1, 32, 32, 7, None, FAKE, ws, 0, None) == 1
    assert f(FAKE + 2, 1, 64, 1, 32, 32, 7, FAKE, FAKE, ws, 0, None) == 1   # misaligned params
    assert f(FAKE, 1, 64, 1, 32, 32, 7, FAKE, None, ws, 0, None) == 1
    assert f(FAKE, 1, 64, 1, 32, 32, 7, FAKE, FAKE + 16, ws, 0, None) == 1  # workspace not 256-aligned
    assert f(FAKE, 1, 64, 1, 32, 32, 7, FAKE, FAKE, ws - 1, 0, None) == 2
    assert lib.pdr_build_bins(FAKE, 1, 64, 1, 32, 32, 7, FAKE, ws - 1, None) == 2
    assert lib.pdr_build_bins(None, 1, 64, 1, 32, 32, 7, FAKE, ws, None) == 1


@no_gpu
def test_bwd_bin_and_host_step_validation(lib):
    ws = lib.pdr_workspace_bytes(2, 64, 3, 40, 24, 9)
    assert lib.pdr_render_bwd(FAKE, FAKE, 2, 64, 3, 40, 24, 9, FAKE, FAKE, ws - 256, 1, None) == 2
    assert lib.pdr_render_bwd(FAKE, None, 2, 64, 3, 40, 24, 9, FAKE, FAKE, ws, 1, None) == 1
    assert lib.pdr_render_bwd(FAKE, FAKE, 2, 64, 3, 40, 24, 9, None, FAKE, ws, 1, None) == 1
    assert lib.pdr_bin(FAKE, 2, 64, 3, 40, 24, 9, None, FAKE, FAKE, ws, None) == 1
    assert lib.pdr_bin(FAKE, 2, 64, 3, 40, 24, 9, FAKE, FAKE, FAKE, 16, None) == 2
    assert lib.pdr_step_host(FAKE, FAKE, FAKE, None, 2, 64, 3, 40, 24, 9,
                             FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == 1
    assert lib.pdr_check_device_error(None, None) == 1


@no_gpu
def test_null_arrays_only_for_frames_without_gaussians(lib):
    """params / grad_params / tile_ids may be NULL only when N = 0; the N = 0
    calls here stop at the workspace check (size 16), before any launch."""
    ws = lib.pdr_workspace_bytes(2, 64, 3, 40, 24, 9)
    assert lib.pdr_render_fwd(None, 2, 64, 3, 40, 24, 9, FAKE, FAKE, ws, 0, None) == 1
    assert lib.pdr_render_fwd(None, 2, 0, 3, 40, 24, 9, FAKE, FAKE, 16, 0, None) == 2
    assert lib.pdr_render_bwd(None, FAKE, 2, 0, 3, 40, 24, 9, None, FAKE, 16, 1, None) == 2
    assert lib.pdr_render_bwd(None, None, 2, 0, 3, 40, 24, 9, None, FAKE, 16, 1, None) == 1
    assert lib.pdr_bin(None, 2, 0, 3, 40, 24, 9, FAKE, None, FAKE, 16, None) == 2
    assert lib.pdr_bin(None, 2, 64, 3, 40, 24, 9, FAKE, None, FAKE, ws, None) == 1
    assert lib.pdr_render_fwd(None, 2, -1, 3, 40, 24, 9, FAKE, FAKE, ws, 0, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="libpdr.so not found"):
        saved = _lib._lib
        try:
            _lib._lib = None
            _lib.load(str(tmp_path / "missing.so"))
        finally:
            _lib._lib = saved


def test_python_api_surface():
    import differentiable_gaussian_splatting_pdr_b200 as pkg
    from differentiable_gaussian_splatting_pdr_b200 import api
    for name in ["render", "render_fwd", "render_bwd", "bin_tiles", "step_host", "build_bins",
                 "workspace_bytes", "check_device_error", "Workspace"]:
        assert callable(getattr(api, name)), name
    assert pkg.render is api.render


def test_loss_workspace_sizes_and_validation_without_gpu():
    """Loss entry points: sizes and argument checks that run before any launch."""
    lib = _lib.load()
    assert lib.pdr_loss_workspace_bytes(0, 1, 8, 8) == 0
    assert lib.pdr_loss_workspace_bytes(1, 1, 8, -1) == 0
    n1 = lib.pdr_loss_workspace_bytes(2, 3, 64, 96)      # 2 x 3 x 2 x 3 tiles, 2 floats each
    assert n1 >= 2 * 4 * 36 and n1 % 256 == 0
    assert lib.pdr_loss_workspace_bytes(2, 3, 65, 96) > n1 or lib.pdr_loss_workspace_bytes(2, 3, 65, 96) == n1
    fake = 1 << 20  # never dereferenced: validation fails before any CUDA call
    bad = [
        (fake, fake, 0, 1, 8, 8, 0.2, 1.0, fake, fake, fake, 1 << 20, None),
        (fake, fake, 1, 1, 8, 8, -0.1, 1.0, fake, fake, fake, 1 << 20, None),
        (fake, fake, 1, 1, 8, 8, 0.2, float("nan"), fake, fake, fake, 1 << 20, None),
        (0, fake, 1, 1, 8, 8, 0.2, 1.0, fake, fake, fake, 1 << 20, None),
        (fake + 2, fake, 1, 1, 8, 8, 0.2, 1.0, fake, fake, fake, 1 << 20, None),
        (fake, fake, 1, 1, 8, 8, 0.2, 1.0, fake, fake, fake + 16, 1 << 20, None),
    ]
    for args in bad:
        assert lib.pdr_loss_l1_ssim(*args) == _lib.STATUS_CODES["PDR_ERR_INVALID_ARG"], args
    assert lib.pdr_loss_l1_ssim(fake, fake, 1, 1, 8, 8, 0.2, 1.0, fake, fake, fake, 0, None) == \
        _lib.STATUS_CODES["PDR_ERR_WORKSPACE_TOO_SMALL"]


def test_plain_c_caller(lib, tmp_path):
    """include/pdr.h is plain C99 and libpdr.so is callable from C without
    Python: a C program built against them runs the host-only entry points."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(r'''
#include <stdio.h>
#include "pdr.h"
int main(void) {
    if (pdr_abi_version() != 1) return 1;
    if (pdr_workspace_bytes(2, 64, 3, 40, 24, 9) == 0) return 2;
    if (pdr_workspace_bytes(2, 64, 3, 40, 24, 8) != 0) return 3;      /* even k */
    if (pdr_list_capacity_per_frame(100, 9) != 400) return 4;
    if (pdr_render_fwd(NULL, 2, 64, 3, 40, 24, 9, NULL, NULL, 0, 0, NULL)
        != PDR_ERR_INVALID_ARG) return 5;
    printf("%s\n", pdr_status_string(PDR_ERR_TOO_LARGE));
    return 0;
}
''')
    exe = tmp_path / "caller"
    libdir = os.path.dirname(_lib.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                         str(src), "-o", str(exe), "-L", libdir, "-lpdr", "-Wl,-rpath," + libdir],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert run.stdout.startswith("PDR_ERR_TOO_LARGE")
