"""The C ABI library loads, exports every symbol include/flare.h declares, and
rejects invalid arguments with status codes before touching the device.

These run without a GPU.  The argument-validation tests pass fake
(never dereferenced) device addresses, so they are skipped when a CUDA
device is present: with a GPU the same checks run in the gpu tests with
real buffers.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import rank_latent_attention_flare_b200 as fl
from rank_latent_attention_flare_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flare.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = 0, 1, 2, 3, 4

no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="fake-pointer validation tests run on CPU-only hosts")


@pytest.fixture(scope="module")
def lib():
    from rank_latent_attention_flare_b200 import build
    build.build()
    return fl.load()


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FLARE_API\s+[\w\s\*]+?\b(flare_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    for name in ("flare_fwd", "flare_pp_fwd", "flare_bwd", "flare_workspace_size",
                 "flare_status_string", "flare_encode", "flare_combine", "flare_decode"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    syms = header_symbols()
    assert set(syms) == set(_lib.SIGNATURES), "binding signatures out of sync with flare.h"
    out = subprocess.run(["nm", "-D", "--defined-only", fl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(flare_\w+)", out))
    missing = set(syms) - exported
    assert not missing, missing
    for s in syms:
        assert getattr(lib, s) is not None


def test_library_targets_sm100a_only(lib):
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", fl.LIB_PATH],
                         capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    archs = set(re.findall(r"sm_(\d+a?)", out.stdout))
    assert archs == {"100a"}, archs


def test_version_and_status_strings(lib):
    assert lib.flare_version() >= 100
    for code in range(6):
        s = lib.flare_status_string(code).decode()
        assert s.startswith("FLARE"), s
    assert b"unknown" in lib.flare_status_string(99)


def test_workspace_size(lib):
    ws = lib.flare_workspace_size
    assert ws(0, 1, 16, 1 << 20, 256, 32, 1) > 0
    assert ws(1, 2, 8, 1 << 18, 256, 32, 1) > ws(0, 2, 8, 1 << 18, 256, 32, 1)
    # the tensor-core backward keeps two floats of statistics per token
    assert ws(2, 8, 8, 16384, 128, 32, 1) > 8 * 8 * 16384 * 8
    # the CUDA-core backward (fp32) holds the fp32 decode-stage dK
    assert ws(2, 8, 8, 16384, 128, 32, 0) > 8 * 8 * 16384 * 32 * 4
    assert ws(0, 1, 1, 1, 16, 16, 0) > 0
    # invalid or unsupported sizes -> 0
    assert ws(0, 0, 1, 100, 16, 16, 0) == 0
    assert ws(0, 1, 1, 0, 16, 16, 0) == 0
    assert ws(0, 1, 1, 100, 24, 16, 0) == 0
    assert ws(0, 1, 1, 100, 16, 64, 0) == 0
    assert ws(0, 1, 1, 100, 512, 16, 0) == 0
    assert ws(7, 1, 1, 100, 16, 16, 0) == 0
    assert ws(0, 1, 1, 100, 16, 16, 5) == 0


def test_fwd_path_selection(lib):
    assert lib.flare_fwd_path(1, 4, 1024, 32, 16, 0) == 0        # fp32 -> CUDA cores
    assert lib.flare_fwd_path(1, 16, 1 << 20, 256, 32, 1) == 1     # bf16 headline -> tcgen05
    assert lib.flare_fwd_path(4, 8, 1 << 16, 128, 16, 1) == 1
    assert lib.flare_fwd_path(1, 4, 1000, 64, 32, 1) == 1         # bf16, M=64 -> tcgen05 (padded)
    assert lib.flare_fwd_path(1, 4, 1000, 16, 16, 1) == 1
    assert lib.flare_fwd_path(1, 4, 1000, 192, 32, 1) == 1
    assert lib.flare_fwd_path(1, 4, 1000, 64, 32, 0) == 0         # fp32, M=64 -> CUDA cores
    assert lib.flare_fwd_path(1, 4, 1024, 40, 16, 1) == -1
    assert lib.flare_bwd_path(8, 8, 16384, 128, 32, 1) == 1      # bf16, M=128 -> tcgen05
    assert lib.flare_bwd_path(1, 2, 300, 128, 16, 1) == 1
    assert lib.flare_bwd_path(1, 2, 300, 256, 32, 1) == 1        # bf16, M=256 -> tcgen05
    assert lib.flare_bwd_path(1, 2, 300, 64, 32, 1) == 0         # bf16, M=64 -> CUDA cores
    assert lib.flare_bwd_path(1, 2, 300, 128, 32, 0) == 0        # fp32 -> CUDA cores
    assert lib.flare_bwd_path(1, 2, 300, 40, 32, 1) == -1


# ------------------------------------------------ validation before launch ---

FAKE = 0x7F0000000000       # 16- and 256-byte aligned, never dereferenced


def _p(x):
    return ctypes.c_void_p(x)


def _fwd(lib, Q=FAKE, qbs=0, K=FAKE + 0x100000, V=FAKE + 0x200000, Y=FAKE + 0x300000,
         B=1, H=2, N=100, M=32, D=16, dt=0, scale=0.25, Z=None, lse=None,
         ws=FAKE + 0x400000, wsb=None):
    if wsb is None:
        wsb = lib.flare_workspace_size(0, B, H, N, M, D, dt) or (1 << 30)
    return lib.flare_fwd(_p(Q), qbs, _p(K), _p(V), _p(Y), B, H, N, M, D, dt, scale,
                         _p(Z) if Z else None, _p(lse) if lse else None, _p(ws), wsb, None)


@no_gpu_only
def test_fwd_rejects_bad_pointers(lib):
    assert _fwd(lib, Q=0) == INVALID
    assert _fwd(lib, K=0) == INVALID
    assert _fwd(lib, V=0) == INVALID
    assert _fwd(lib, Y=0) == INVALID
    assert _fwd(lib, Q=FAKE + 8) == INVALID          # misaligned
    assert _fwd(lib, Y=FAKE + 0x300002) == INVALID
    assert _fwd(lib, Z=FAKE + 0x500004) == INVALID   # optional but misaligned


@no_gpu_only
def test_fwd_rejects_bad_sizes_and_scale(lib):
    assert _fwd(lib, N=0) == INVALID
    assert _fwd(lib, B=0) == INVALID
    assert _fwd(lib, H=-1) == INVALID
    assert _fwd(lib, dt=3) == INVALID
    for s in (0.0, -1.0, float("nan"), float("inf")):
        assert _fwd(lib, scale=s) == INVALID
    assert _fwd(lib, D=24) == UNSUPPORTED
    assert _fwd(lib, D=64) == UNSUPPORTED
    assert _fwd(lib, M=8) == UNSUPPORTED
    assert _fwd(lib, M=100) == UNSUPPORTED
    assert _fwd(lib, M=272) == UNSUPPORTED
    assert _fwd(lib, qbs=7) == UNSUPPORTED
    assert _fwd(lib, B=1 << 21) == INVALID


@no_gpu_only
def test_fwd_rejects_bad_workspace(lib):
    need = lib.flare_workspace_size(0, 1, 2, 100, 32, 16, 0)
    assert _fwd(lib, wsb=need - 1) == WORKSPACE
    assert _fwd(lib, ws=0) == WORKSPACE
    assert _fwd(lib, ws=FAKE + 0x400010) == WORKSPACE   # not 256-byte aligned


@no_gpu_only
def test_other_entry_points_validate(lib):
    F = FAKE
    ws_pp = lib.flare_workspace_size(1, 1, 2, 100, 32, 16, 0)
    assert lib.flare_pp_fwd(None, _p(F), _p(F), _p(F), None, 1, 2, 100, 32, 16, 0, 0.25, None,
                            None, _p(F), ws_pp, None) == INVALID
    assert lib.flare_pp_fwd(_p(F), _p(F), _p(F), _p(F), None, 1, 2, 100, 32, 16, 0, 0.25, None,
                            None, _p(F), ws_pp - 1, None) == WORKSPACE
    ws_b = lib.flare_workspace_size(2, 1, 2, 100, 32, 16, 0)
    # Z_save and lse_save are required by the backward
    assert lib.flare_bwd(_p(F), 0, _p(F), _p(F), _p(F), None, _p(F), _p(F), _p(F), _p(F),
                         1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_b, None) == INVALID
    assert lib.flare_bwd(_p(F), 0, _p(F), _p(F), _p(F), _p(F), None, _p(F), _p(F), _p(F),
                         1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_b, None) == INVALID
    assert lib.flare_bwd(_p(F), 0, _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F),
                         1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_b - 1, None) == WORKSPACE
    ws_ppb = lib.flare_workspace_size(3, 1, 2, 100, 32, 16, 0)
    assert ws_ppb > ws_b
    # FLARE++ backward: Q_dyn, Z_save and lse_save are required
    assert lib.flare_pp_bwd(_p(F), _p(F), _p(F), _p(F), None, _p(F), _p(F), _p(F), _p(F), _p(F),
                            1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_ppb, None) == INVALID
    assert lib.flare_pp_bwd(_p(F), _p(F), _p(F), _p(F), _p(F), _p(F), None, _p(F), _p(F), _p(F),
                            1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_ppb, None) == INVALID
    assert lib.flare_pp_bwd(_p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F),
                            1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_ppb - 1, None) == WORKSPACE
    ws_f = lib.flare_workspace_size(0, 1, 2, 100, 32, 16, 0)
    assert lib.flare_encode(None, 0, _p(F), _p(F), 1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_f,
                            None) == INVALID
    assert lib.flare_combine(1, 2, 100, 32, 16, 0, None, None, _p(F), ws_f - 1,
                             None) == WORKSPACE
    assert lib.flare_decode(_p(F), 0, _p(F), None, 1, 2, 100, 32, 16, 0, 0.25, _p(F), ws_f,
                            None) == INVALID
    assert lib.flare_device_status(None, 256, None, None) == WORKSPACE


@no_gpu_only
def test_fwd_host_validates(lib):
    F = FAKE
    host = ctypes.create_string_buffer(64)   # never read: validation fails first
    hp = ctypes.cast(host, ctypes.c_void_p)
    need = lib.flare_fwd_host_workspace_size(1, 2, 100, 32, 16, 0)
    assert need > 0
    assert lib.flare_fwd_host_workspace_size(1, 2, 100, 40, 16, 0) == 0   # M not a multiple of 16
    args = dict(B=1, H=2, N=100, M=32, D=16)

    def call(q=hp, y=hp, qd=_p(F), wsb=need, scale=0.25):
        return lib.flare_fwd_host(q, 0, hp, hp, y, qd, _p(F), _p(F), _p(F), args["B"], args["H"],
                                  args["N"], args["M"], args["D"], 0, scale, _p(F), wsb, None,
                                  None)
    assert call(q=None) == INVALID          # host pointers are required
    assert call(y=None) == INVALID
    assert call(qd=None) == INVALID         # and device buffers
    assert call(scale=-1.0) == INVALID
    assert call(wsb=need - 1) == WORKSPACE


@no_gpu_only
def test_valid_call_without_device_reports_cuda_error(lib):
    # Arguments pass validation; the first enqueue fails because there is no
    # device, which must surface as FLARE_ERR_CUDA (not a crash).
    assert _fwd(lib) == CUDA


def test_binding_fails_loudly_without_cuda_tensors():
    x = torch.zeros(1, 2, 8, 16)
    with pytest.raises(ValueError):
        fl.flare_fwd(torch.zeros(2, 16, 16), x, x)


def _st(*triples):
    arr = (_lib.FlareStrides * len(triples))()
    for i, t in enumerate(triples):
        arr[i] = _lib.FlareStrides(*t)
    return arr


@no_gpu_only
def test_strided_entry_points_validate_strides(lib):
    # B2 H2 N100 M32 D16 float32: rows must start on 16 bytes (4 elements)
    B, H, N, M, D = 2, 2, 100, 32, 16
    F = FAKE
    ws = lib.flare_workspace_size(0, B, H, N, M, D, 0)
    contig = (H * N * D, N * D, D)
    bnhd = (N * H * D, D, H * D)

    def fwd(*triples):
        st = _st(*triples) if triples else None
        return lib.flare_fwd_ex(_p(F), 0, _p(F), _p(F), _p(F), st, None, B, H, N, M, D, 0, 0.25,
                                     None, None, _p(F), ws, None)

    # valid layouts pass validation and fail only at the first enqueue
    assert fwd() == CUDA
    assert fwd(contig, contig, contig) == CUDA
    assert fwd(bnhd, bnhd, bnhd) == CUDA
    assert fwd(contig, bnhd, (N * H * D, D, H * D)) == CUDA
    # an input may overlap itself (rows 8 elements apart); an output may not
    assert fwd((H * N * 8, N * 8, 8), contig, contig) == CUDA
    assert fwd(contig, contig, (H * N * 8, N * 8, 8)) == INVALID
    assert fwd(contig, contig, (N * D, N * D, D)) == INVALID   # b and h rows coincide
    # strides must be positive multiples of 16 bytes
    assert fwd((0, N * D, D), contig, contig) == INVALID
    assert fwd(contig, (H * N * D, N * D, -D), contig) == INVALID
    assert fwd(contig, contig, (H * N * 18, N * 18, 18)) == UNSUPPORTED
    assert fwd((1 << 40, N * D, D), contig, contig) == INVALID
    # the backward's outputs dK, dV are the 4th and 5th entries
    wsb = lib.flare_workspace_size(2, B, H, N, M, D, 0)

    def bwd(*triples):
        return lib.flare_bwd_ex(_p(F), 0, _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F),
                                _p(F), _st(*triples), None, B, H, N, M, D, 0, 0.25, _p(F), wsb,
                                None)

    assert bwd(bnhd, bnhd, bnhd, bnhd, bnhd) == CUDA
    assert bwd(bnhd, bnhd, bnhd, bnhd, (N * H * D, D, 8)) == INVALID
    assert bwd(bnhd, bnhd, (N * H * D, D, 8), bnhd, bnhd) == CUDA
    wsp = lib.flare_workspace_size(1, B, H, N, M, D, 0)
    assert lib.flare_pp_fwd_ex(_p(F), _p(F), _p(F), _p(F), None, _st(bnhd, bnhd, bnhd), None, B,
                               H, N, M, D, 0, 0.25, None, None, _p(F), wsp, None) == CUDA
    assert lib.flare_pp_fwd_ex(_p(F), _p(F), _p(F), _p(F), None,
                               _st(bnhd, bnhd, (N * D, N * D, D)), None, B, H, N, M, D, 0, 0.25,
                               None, None, _p(F), wsp, None) == INVALID
    wspb = lib.flare_workspace_size(3, B, H, N, M, D, 0)
    assert lib.flare_pp_bwd_ex(_p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F), _p(F),
                               _p(F), _p(F), _st(bnhd, bnhd, bnhd, (0, D, H * D), bnhd), None, B,
                               H, N, M, D, 0, 0.25, _p(F), wspb, None) == INVALID
    # seq_lens: a device array of int32, 4-byte aligned
    assert lib.flare_fwd_ex(_p(F), 0, _p(F), _p(F), _p(F), None, _p(F + 0x600002), B, H, N, M,
                            D, 0, 0.25, None, None, _p(F), ws, None) == INVALID
    assert lib.flare_fwd_ex(_p(F), 0, _p(F), _p(F), _p(F), None, _p(F + 0x600004), B, H, N, M,
                            D, 0, 0.25, None, None, _p(F), ws, None) == CUDA
