"""Thin PyTorch binding over the C ABI (argument marshalling only).

Every function here allocates outputs and the workspace with torch (the
library never allocates), passes raw device pointers and the current CUDA
stream to ``libflare.so``, and raises :class:`FlareError` on a non-OK status.
All computation happens in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _lib
from ._lib import FlareError  # noqa: F401  (re-export)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _lib.FLARE_F32
    if t.dtype == torch.bfloat16:
        return _lib.FLARE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("FLARE tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("FLARE tensors must be contiguous")


def _need_tokens(*ts):
    """Token tensors [B,H,N,D]: on the device, D contiguous, any other strides."""
    shape = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("FLARE tensors must live on a CUDA device")
        if t.dim() != 4 or t.stride(-1) != 1:
            raise ValueError("token tensors must be [B,H,N,D] views with D contiguous")
        if shape is not None and t.shape != shape:
            raise ValueError(f"token tensors differ in shape: {tuple(t.shape)} vs {tuple(shape)}")
        shape = t.shape


def _strides(*ts):
    """None when every token tensor is contiguous, else the flare_strides_t
    array (one entry per tensor, in the C entry point's order)."""
    if all(t.is_contiguous() for t in ts):
        return None
    arr = (_lib.FlareStrides * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _lib.FlareStrides(t.stride(0), t.stride(1), t.stride(2))
    return arr


def _seq_lens(seq_lens, B: int, device):
    """Device int32 [B] lengths (or None), checked for shape, dtype and device."""
    if seq_lens is None:
        return None
    if (not isinstance(seq_lens, torch.Tensor) or seq_lens.dtype != torch.int32
            or seq_lens.shape != (B,) or seq_lens.device != device
            or not seq_lens.is_contiguous()):
        raise ValueError("seq_lens must be a contiguous int32 tensor of shape [B] on the "
                         "tensors' device")
    return seq_lens


def _like(t: torch.Tensor) -> torch.Tensor:
    """An output with t's layout (empty_like keeps the strides of a dense
    tensor); a contiguous one where t's layout has gaps or overlaps."""
    return torch.empty_like(t)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dims(Q: torch.Tensor, K: torch.Tensor):
    if K.dim() != 4:
        raise ValueError("K must be [B,H,N,D]")
    B, H, N, D = K.shape
    M = Q.shape[-2]
    if Q.dim() == 3:
        qbs = 0
    elif Q.dim() == 4:
        qbs = H * M * D
    else:
        raise ValueError("Q must be [H,M,D] or [B,H,M,D]")
    return B, H, N, M, D, qbs


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def workspace_size(op: int, B: int, H: int, N: int, M: int, D: int, dtype: torch.dtype) -> int:
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    return int(_lib.load().flare_workspace_size(op, B, H, N, M, D, code))


def fwd_path(B: int, H: int, N: int, M: int, D: int, dtype: torch.dtype) -> int:
    """1 = tcgen05 tensor-core kernels, 0 = CUDA-core kernels, -1 = unsupported."""
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    return int(_lib.load().flare_fwd_path(B, H, N, M, D, code))


def bwd_path(B: int, H: int, N: int, M: int, D: int, dtype: torch.dtype) -> int:
    """1 = tcgen05 tensor-core backward, 0 = CUDA-core kernels, -1 = unsupported."""
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    return int(_lib.load().flare_bwd_path(B, H, N, M, D, code))


def alloc_workspace(op: int, B, H, N, M, D, dtype, device) -> torch.Tensor:
    n = workspace_size(op, B, H, N, M, D, dtype)
    if n == 0:
        raise FlareError(2, "flare_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream; returns the device error site (0 = none)."""
    detail = ctypes.c_uint32(0)
    st = _lib.load().flare_device_status(_ptr(workspace), workspace.numel(),
                                         ctypes.byref(detail), _stream(stream))
    if st not in (0, 5):
        _lib.check(st, "flare_device_status")
    return int(detail.value)


def flare_fwd(Q, K, V, scale: Optional[float] = None, *, save: bool = False,
              workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
              seq_lens: Optional[torch.Tensor] = None, stream=None):
    """FLARE forward.  Returns Y, or (Y, Z, lse) when ``save``.

    K, V (and ``out``) may be any [B,H,N,D] views with D contiguous, e.g.
    ``x.transpose(1, 2)`` of a [B,N,H,D] projection output; Y then takes K's
    layout.  ``seq_lens`` (int32 [B] on the device): valid tokens per batch
    element; padding is never read, and Y is 0 there."""
    _need_cuda(Q, workspace)
    _need_tokens(K, V, out)
    B, H, N, M, D, qbs = _dims(Q, K)
    dt = _dtype_code(K)
    s = default_scale(D) if scale is None else float(scale)
    Y = _like(K) if out is None else out
    Z = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device) if save else None
    lse = torch.empty((B, H, M), dtype=torch.float32, device=K.device) if save else None
    ws = workspace if workspace is not None else alloc_workspace(
        _lib.FLARE_OP_FWD, B, H, N, M, D, K.dtype, K.device)
    strides = _strides(K, V, Y)
    lens = _seq_lens(seq_lens, B, K.device)
    if strides is None and lens is None:
        st = _lib.load().flare_fwd(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(Y), B, H, N, M, D, dt, s,
                                   _ptr(Z), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    else:
        st = _lib.load().flare_fwd_ex(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(Y), strides,
                                      _ptr(lens), B, H, N, M, D, dt, s, _ptr(Z), _ptr(lse),
                                      _ptr(ws), ws.numel(), _stream(stream))
    _lib.check(st, "flare_fwd")
    return (Y, Z, lse) if save else Y


def flare_fwd_host(Q, K, V, scale: Optional[float] = None, *, out: Optional[torch.Tensor] = None,
                   device_buffers=None, workspace: Optional[torch.Tensor] = None, device=None,
                   stream=None, copy_stream=None):
    """FLARE forward from and to host memory (flare_fwd_host): Q, K, V are
    contiguous CPU tensors (pinned for the copies to overlap the compute),
    and Y comes back in ``out`` (a pinned CPU tensor shaped like K, created
    if not given).  ``device_buffers``: an optional dict of device tensors
    "Q", "K", "V", "Y" shaped like the host ones, reused across calls.
    Returns Y once ``stream`` is synchronised (this call does not wait)."""
    for t in (Q, K, V, out):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("flare_fwd_host takes contiguous host tensors")
    if K.dim() != 4:
        raise ValueError("K must be [B,H,N,D]")
    B, H, N, D = K.shape
    M = Q.shape[-2]
    qbs = 0 if Q.dim() == 3 else H * M * D
    dt = _dtype_code(K)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    s = default_scale(D) if scale is None else float(scale)
    Y = torch.empty(K.shape, dtype=K.dtype, pin_memory=True) if out is None else out
    buf = device_buffers if device_buffers is not None else {
        "Q": torch.empty(Q.shape, dtype=Q.dtype, device=dev),
        **{k: torch.empty(K.shape, dtype=K.dtype, device=dev) for k in ("K", "V", "Y")}}
    lib = _lib.load()
    if workspace is None:
        n = int(lib.flare_fwd_host_workspace_size(B, H, N, M, D, dt))
        if n == 0:
            raise FlareError(2, "flare_fwd_host_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    st = _stream(stream)
    cs = _stream(copy_stream) if copy_stream is not None else st
    _lib.check(lib.flare_fwd_host(ctypes.c_void_p(Q.data_ptr()), qbs, ctypes.c_void_p(K.data_ptr()),
                                  ctypes.c_void_p(V.data_ptr()), ctypes.c_void_p(Y.data_ptr()),
                                  _ptr(buf["Q"]), _ptr(buf["K"]), _ptr(buf["V"]), _ptr(buf["Y"]),
                                  B, H, N, M, D, dt, s, _ptr(workspace), workspace.numel(), st, cs),
               "flare_fwd_host")
    return Y


def flare_pp_fwd(Q, K, V, scale: Optional[float] = None, *, save: bool = False,
                 workspace: Optional[torch.Tensor] = None,
                 seq_lens: Optional[torch.Tensor] = None, stream=None):
    """FLARE++ forward with learned Q [H,M,D].  Returns (Y, Q_dyn) or
    (Y, Q_dyn, Z, lse) when ``save``."""
    _need_cuda(Q, workspace)
    _need_tokens(K, V)
    B, H, N, M, D, qbs = _dims(Q, K)
    if qbs != 0:
        raise ValueError("FLARE++ takes learned latents Q of shape [H,M,D]")
    dt = _dtype_code(K)
    s = default_scale(D) if scale is None else float(scale)
    Y = _like(K)
    Qd = torch.empty((B, H, M, D), dtype=K.dtype, device=K.device)
    Z = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device) if save else None
    lse = torch.empty((B, H, M), dtype=torch.float32, device=K.device) if save else None
    ws = workspace if workspace is not None else alloc_workspace(
        _lib.FLARE_OP_PP_FWD, B, H, N, M, D, K.dtype, K.device)
    strides = _strides(K, V, Y)
    lens = _seq_lens(seq_lens, B, K.device)
    if strides is None and lens is None:
        st = _lib.load().flare_pp_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(Y), _ptr(Qd), B, H, N, M,
                                      D, dt, s, _ptr(Z), _ptr(lse), _ptr(ws), ws.numel(),
                                      _stream(stream))
    else:
        st = _lib.load().flare_pp_fwd_ex(_ptr(Q), _ptr(K), _ptr(V), _ptr(Y), _ptr(Qd), strides,
                                         _ptr(lens), B, H, N, M, D, dt, s, _ptr(Z), _ptr(lse),
                                         _ptr(ws), ws.numel(), _stream(stream))
    _lib.check(st, "flare_pp_fwd")
    return (Y, Qd, Z, lse) if save else (Y, Qd)


def flare_bwd(Q, K, V, dY, Z, lse, scale: Optional[float] = None, *,
              workspace: Optional[torch.Tensor] = None,
              seq_lens: Optional[torch.Tensor] = None, stream=None):
    """FLARE backward.  Returns (dQ, dK, dV); dK and dV take K's and V's
    layouts (token tensors may be strided as in flare_fwd)."""
    _need_cuda(Q, Z, lse, workspace)
    _need_tokens(K, V, dY)
    B, H, N, M, D, qbs = _dims(Q, K)
    dt = _dtype_code(K)
    s = default_scale(D) if scale is None else float(scale)
    dQ = torch.empty_like(Q)
    dK = _like(K)
    dV = _like(V)
    ws = workspace if workspace is not None else alloc_workspace(
        _lib.FLARE_OP_BWD, B, H, N, M, D, K.dtype, K.device)
    strides = _strides(K, V, dY, dK, dV)
    lens = _seq_lens(seq_lens, B, K.device)
    if strides is None and lens is None:
        st = _lib.load().flare_bwd(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(dY), _ptr(Z), _ptr(lse),
                                   _ptr(dQ), _ptr(dK), _ptr(dV), B, H, N, M, D, dt, s, _ptr(ws),
                                   ws.numel(), _stream(stream))
    else:
        st = _lib.load().flare_bwd_ex(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(dY), _ptr(Z),
                                      _ptr(lse), _ptr(dQ), _ptr(dK), _ptr(dV), strides,
                                      _ptr(lens), B, H, N, M, D, dt, s, _ptr(ws), ws.numel(),
                                      _stream(stream))
    _lib.check(st, "flare_bwd")
    return dQ, dK, dV


def flare_pp_bwd(Q, K, V, dY, Q_dyn, Z, lse, scale: Optional[float] = None, *,
                 workspace: Optional[torch.Tensor] = None,
                 seq_lens: Optional[torch.Tensor] = None, stream=None):
    """FLARE++ backward with learned Q [H,M,D] (Q_dyn, Z, lse from
    flare_pp_fwd(..., save=True)).  Returns (dQ [H,M,D], dK, dV)."""
    _need_cuda(Q, Q_dyn, Z, lse, workspace)
    _need_tokens(K, V, dY)
    B, H, N, M, D, qbs = _dims(Q, K)
    if qbs != 0:
        raise ValueError("FLARE++ takes learned latents Q of shape [H,M,D]")
    dt = _dtype_code(K)
    s = default_scale(D) if scale is None else float(scale)
    dQ = torch.empty_like(Q)
    dK = _like(K)
    dV = _like(V)
    ws = workspace if workspace is not None else alloc_workspace(
        _lib.FLARE_OP_PP_BWD, B, H, N, M, D, K.dtype, K.device)
    strides = _strides(K, V, dY, dK, dV)
    lens = _seq_lens(seq_lens, B, K.device)
    if strides is None and lens is None:
        st = _lib.load().flare_pp_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(dY), _ptr(Q_dyn), _ptr(Z),
                                      _ptr(lse), _ptr(dQ), _ptr(dK), _ptr(dV), B, H, N, M, D, dt,
                                      s, _ptr(ws), ws.numel(), _stream(stream))
    else:
        st = _lib.load().flare_pp_bwd_ex(_ptr(Q), _ptr(K), _ptr(V), _ptr(dY), _ptr(Q_dyn),
                                         _ptr(Z), _ptr(lse), _ptr(dQ), _ptr(dK), _ptr(dV),
                                         strides, _ptr(lens), B, H, N, M, D, dt, s, _ptr(ws),
                                         ws.numel(), _stream(stream))
    _lib.check(st, "flare_pp_bwd")
    return dQ, dK, dV


def flare_encode(Q, K, V, scale: Optional[float] = None, *, workspace: torch.Tensor,
                 stream=None) -> None:
    """Stage 1: encode partials into ``workspace`` (FLARE_OP_FWD size)."""
    _need_cuda(Q, K, V, workspace)
    B, H, N, M, D, qbs = _dims(Q, K)
    s = default_scale(D) if scale is None else float(scale)
    st = _lib.load().flare_encode(_ptr(Q), qbs, _ptr(K), _ptr(V), B, H, N, M, D, _dtype_code(K),
                                  s, _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(st, "flare_encode")


def flare_combine(B, H, N, M, D, dtype: torch.dtype, *, workspace: torch.Tensor,
                  Z_save: Optional[torch.Tensor] = None, lse_save: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    """Stage 2: merge the encode partials in ``workspace``."""
    _need_cuda(workspace, Z_save, lse_save)
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    st = _lib.load().flare_combine(B, H, N, M, D, code, _ptr(Z_save), _ptr(lse_save),
                                   _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(st, "flare_combine")


def flare_decode(Q, K, scale: Optional[float] = None, *, workspace: torch.Tensor,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Stage 3: decode with the Z left in ``workspace`` by flare_combine."""
    _need_cuda(Q, K, workspace, out)
    B, H, N, M, D, qbs = _dims(Q, K)
    s = default_scale(D) if scale is None else float(scale)
    Y = torch.empty_like(K) if out is None else out
    st = _lib.load().flare_decode(_ptr(Q), qbs, _ptr(K), _ptr(Y), B, H, N, M, D, _dtype_code(K),
                                  s, _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(st, "flare_decode")
    return Y


def flare_fwd_noalloc(Q, K, V, scale: Optional[float] = None, *, save: bool = False,
                      out: Optional[torch.Tensor] = None, stream=None):
    """FLARE forward without a workspace, for callers that cannot allocate.

    The library keeps the scratch in a fixed device array of
    ``NOALLOC_SCRATCH_BYTES`` bytes shared by every call on the device, so
    calls that overlap on the GPU race; sizes that need more scratch raise
    FlareError(FLARE_ERR_WORKSPACE).  This wrapper still allocates the
    outputs with torch for convenience; the C entry point allocates nothing.
    """
    _need_cuda(Q, K, V, out)
    B, H, N, M, D, qbs = _dims(Q, K)
    dt = _dtype_code(K)
    s = default_scale(D) if scale is None else float(scale)
    Y = torch.empty_like(K) if out is None else out
    Z = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device) if save else None
    lse = torch.empty((B, H, M), dtype=torch.float32, device=K.device) if save else None
    lib = _lib.load()
    st = lib.flare_fwd_noalloc(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(Y), B, H, N, M, D, dt, s,
                               _ptr(Z), _ptr(lse), _stream(stream))
    if st == 3:
        detail = (lib.flare_last_error_detail() or b"").decode(errors="replace")
        raise FlareError(st, "flare_fwd_noalloc" + (f" [{detail}]" if detail else ""))
    _lib.check(st, "flare_fwd_noalloc")
    return (Y, Z, lse) if save else Y


# ------------------------------------------------- context parallelism (stages)

def noalloc_device_status(stream=None) -> int:
    """Reads and clears the device error word of flare_fwd_noalloc's scratch
    array on the current device (synchronises the stream); returns its
    detail code (0: no bounded wait ran out)."""
    detail = ctypes.c_uint32(0)
    st = _lib.load().flare_noalloc_device_status(ctypes.byref(detail), _stream(stream))
    if st not in (0, 5):
        _lib.check(st, "flare_noalloc_device_status")
    return int(detail.value)


def probe_unit_rates(device=None, stream=None) -> dict:
    """Measured throughputs of the units the kernels are bound by
    (flare_probe_unit_rates): MUFU exponentials, scalar and packed fp32 FMAs
    and their mix, per SM per SM clock, with the SM clock seen by the probe
    kernels.  Synchronises the device."""
    lib = _lib.load()
    n = int(lib.flare_probe_scratch_bytes())
    if n == 0:
        raise RuntimeError("flare_probe_scratch_bytes: no CUDA device")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    scratch = torch.empty(n, dtype=torch.uint8, device=dev)
    out = _lib.UnitRates()
    _lib.check(lib.flare_probe_unit_rates(_ptr(scratch), n, ctypes.byref(out), _stream(stream)),
               "flare_probe_unit_rates")
    return {name: getattr(out, name) for name, _ in _lib.UnitRates._fields_}


def probe_mma_rates(cases=None, device=None, stream=None) -> dict:
    """SM clocks per tcgen05.mma of the kernels' shapes (flare_probe_mma_rate)
    for each (n, a_in_tmem, issuers) case: with one issuer the issue latency
    of a thread, with several the SM's own cost of a product.  Synchronises
    the device."""
    lib = _lib.load()
    nbytes = int(lib.flare_probe_scratch_bytes())
    if nbytes == 0:
        raise RuntimeError("flare_probe_scratch_bytes: no CUDA device")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    scratch = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if cases is None:
        cases = [(n, t, i) for t in (0, 1) for n in (32, 48) for i in (1, 4)] + \
                [(128, 0, 1), (256, 0, 1)]
    out = {}
    for n, tm, iss in cases:
        v = ctypes.c_double(0.0)
        _lib.check(lib.flare_probe_mma_rate(int(n), int(tm), int(iss), _ptr(scratch), nbytes,
                                            ctypes.byref(v), _stream(stream)),
                   "flare_probe_mma_rate")
        out[f"{'ts' if tm else 'ss'}_n{n}_x{iss}"] = float(v.value)
    return out


def exp_split(kernel: int, M: int, D: int, dtype: torch.dtype) -> float:
    """Share of the forward encode's (kernel 0) or decode's (kernel 1)
    exponentials computed by the FMA-pipe polynomial (flare_exp_split)."""
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    out = ctypes.c_double(0.0)
    _lib.check(_lib.load().flare_exp_split(int(kernel), M, D, code, ctypes.byref(out)),
               "flare_exp_split")
    return float(out.value)


def eval_exp2(x: torch.Tensor, form: int, stream=None) -> torch.Tensor:
    """2^x with one of the kernels' exponentials (flare_eval_exp2): form 0 =
    MUFU ex2.approx, 1 = FMA-pipe polynomial, 2 = the packed polynomial,
    3 = the packed polynomial with its exponent clamped to [-125, 126]."""
    _need_cuda(x)
    if x.dtype != torch.float32:
        raise TypeError("eval_exp2 takes float32")
    y = torch.empty_like(x)
    _lib.check(_lib.load().flare_eval_exp2(_ptr(x), _ptr(y), x.numel(), form, _stream(stream)),
               "flare_eval_exp2")
    return y


def selftest_wait_timeout(workspace: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Launches the bounded-wait self-test (flare_selftest_wait_timeout) on
    a workspace of at least 512 bytes; read the result with device_status."""
    _lib.check(_lib.load().flare_selftest_wait_timeout(_ptr(workspace), workspace.numel(),
                                                       int(limit_ns), _stream(stream)),
               "flare_selftest_wait_timeout")


def records_layout(B: int, H: int, N: int, M: int, D: int, dtype: torch.dtype):
    """(records_per_bh, ml_offset, acc_offset): where flare_encode leaves its
    chunk records in a FLARE_OP_FWD workspace."""
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    r, mo, ao = ctypes.c_int64(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = _lib.load().flare_records_layout(B, H, N, M, D, code, ctypes.byref(r),
                                          ctypes.byref(mo), ctypes.byref(ao))
    _lib.check(st, "flare_records_layout")
    return int(r.value), int(mo.value), int(ao.value)


def encode_records(workspace: torch.Tensor, B: int, H: int, N: int, M: int, D: int,
                   dtype: torch.dtype):
    """Views of the records flare_encode left in ``workspace``: ml
    [B*H, R, M, 2] (running max in log2 units, sum) and acc [B*H, R, M, D],
    float32."""
    R, mo, ao = records_layout(B, H, N, M, D, dtype)
    n_ml, n_acc = B * H * R * M * 2 * 4, B * H * R * M * D * 4
    ml = workspace[mo:mo + n_ml].view(torch.float32).view(B * H, R, M, 2)
    acc = workspace[ao:ao + n_acc].view(torch.float32).view(B * H, R, M, D)
    return ml, acc


def flare_combine_shards(ml: torch.Tensor, acc: torch.Tensor, B: int, H: int, N: int, M: int,
                         D: int, dtype: torch.dtype, *, workspace: torch.Tensor,
                         Z_save: Optional[torch.Tensor] = None,
                         lse_save: Optional[torch.Tensor] = None,
                         Q_learned: Optional[torch.Tensor] = None,
                         Q_dyn_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """Merges the gathered records of every shard (ml [shards, B*H, R, M, 2],
    acc [shards, B*H, R, M, D]) into the whole sequence's Z, left in
    ``workspace`` for flare_decode (and written to Z_save / lse_save).  With
    Q_dyn_out (FLARE++'s first encode) also Q_dyn = Q_learned + Z."""
    _need_cuda(ml, acc, workspace, Z_save, lse_save, Q_learned, Q_dyn_out)
    if ml.dim() != 5 or acc.dim() != 5 or ml.shape[:4] != acc.shape[:4]:
        raise ValueError("ml must be [shards, B*H, R, M, 2] and acc [shards, B*H, R, M, D]")
    code = _lib.FLARE_F32 if dtype == torch.float32 else _lib.FLARE_BF16
    st = _lib.load().flare_combine_shards(ml.shape[0], _ptr(ml), _ptr(acc), ml.shape[2], B, H, N,
                                          M, D, code, _ptr(Z_save), _ptr(lse_save),
                                          _ptr(Q_learned), _ptr(Q_dyn_out), _ptr(workspace),
                                          workspace.numel(), _stream(stream))
    _lib.check(st, "flare_combine_shards")


def flare_bwd_shard_dz(Q, K, V, dY, Z, lse, scale: Optional[float] = None, *,
                       workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """First half of a sharded backward: the decode stage over this shard's
    tokens.  Returns the shard's part of dZ (float32 [B,H,M,D]); keep
    ``workspace`` (FLARE_OP_BWD size) for flare_bwd_shard_finish."""
    _need_cuda(Q, K, V, dY, Z, lse, workspace)
    B, H, N, M, D, qbs = _dims(Q, K)
    s = default_scale(D) if scale is None else float(scale)
    dZ = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device)
    st = _lib.load().flare_bwd_shard_dz(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(dY), _ptr(Z),
                                        _ptr(lse), _ptr(dZ), B, H, N, M, D, _dtype_code(K), s,
                                        _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(st, "flare_bwd_shard_dz")
    return dZ


def flare_bwd_shard_finish(Q, K, V, dY, Z, lse, dZ, scale: Optional[float] = None, *,
                           workspace: torch.Tensor, stream=None):
    """Second half, given dZ summed over the shards: returns (the shard's
    float32 part of dQ, its rows of dK, dV)."""
    _need_cuda(Q, K, V, dY, Z, lse, dZ, workspace)
    B, H, N, M, D, qbs = _dims(Q, K)
    s = default_scale(D) if scale is None else float(scale)
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=K.device)
    dK = torch.empty_like(K)
    dV = torch.empty_like(V)
    st = _lib.load().flare_bwd_shard_finish(_ptr(Q), qbs, _ptr(K), _ptr(V), _ptr(dY), _ptr(Z),
                                            _ptr(lse), _ptr(dZ), _ptr(dQ), _ptr(dK), _ptr(dV), B,
                                            H, N, M, D, _dtype_code(K), s, _ptr(workspace),
                                            workspace.numel(), _stream(stream))
    _lib.check(st, "flare_bwd_shard_finish")
    return dQ, dK, dV


def flare_pp_bwd_shard_tail(Q, K, V, Z1, lse1, dQ_dyn, dK, dV, scale: Optional[float] = None, *,
                            workspace: torch.Tensor, add_dq_dyn: bool = False,
                            stream=None) -> torch.Tensor:
    """FLARE++'s first-encode gradient over this shard, given dQ_dyn summed
    over the shards (input dtype) and the first encode's Z1, lse1 of the
    whole sequence: adds into dK, dV (in place) and returns the shard's
    float32 part of dQ [H,M,D]; with ``add_dq_dyn`` (on exactly one shard)
    that part also holds the sum over the batch of dQ_dyn, so that dQ is the
    sum of the parts.  ``workspace``: FLARE_OP_PP_BWD size."""
    _need_cuda(Q, K, V, Z1, lse1, dQ_dyn, dK, dV, workspace)
    B, H, N, M, D, qbs = _dims(Q, K)
    if qbs != 0:
        raise ValueError("FLARE++ takes learned latents Q of shape [H,M,D]")
    s = default_scale(D) if scale is None else float(scale)
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=K.device)
    st = _lib.load().flare_pp_bwd_shard_tail(_ptr(Q), _ptr(K), _ptr(V), _ptr(Z1), _ptr(lse1),
                                             _ptr(dQ_dyn), int(bool(add_dq_dyn)), _ptr(dQ),
                                             _ptr(dK), _ptr(dV), B, H, N,
                                             M, D, _dtype_code(K), s, _ptr(workspace),
                                             workspace.numel(), _stream(stream))
    _lib.check(st, "flare_pp_bwd_shard_tail")
    return dQ
