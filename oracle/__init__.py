"""Double-precision CPU oracle for FLARE / FLARE++ (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never touches it, and it never touches the product path:
the two share only the seeded input generators in ``flare_inputs``.

The arithmetic lives in ``flare_oracle.c`` (plain loops, double precision,
OpenMP over independent rows).  This module compiles it with gcc, loads it
with ctypes and converts numpy arrays to float64 before every call.

Sources: "Flare Fast Low Rank Attention" skill page, sections 2 and 4
(encode); FLARE arXiv 2508.12594 abstract (two SDPA calls, rank-M mixing
matrix, hence the decode); FLARE++ arXiv 2608.11519 abstract (input-
conditioned queries).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flare_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_c_dp = ctypes.POINTER(ctypes.c_double)
_c_i64p = ctypes.POINTER(ctypes.c_int64)
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_encode.argtypes = [_c_dp, _i64, _c_dp, _c_dp, _c_i32p, _i64, _i64, _i64,
                                      _i64, _i64, ctypes.c_double, _c_dp, _c_dp]
        lib.oracle_decode.argtypes = [_c_dp, _i64, _c_dp, _c_dp, _c_i32p, _i64, _i64, _i64,
                                      _i64, _i64, ctypes.c_double, _c_dp]
        lib.oracle_decode_rows.argtypes = [_c_dp, _i64, _c_dp, _c_dp, _i64, _i64, _i64, _i64,
                                           _i64, ctypes.c_double, _c_i64p, _i64, _c_dp]
        lib.oracle_flare_fwd.argtypes = [_c_dp, _i64, _c_dp, _c_dp, _c_i32p, _i64, _i64, _i64,
                                         _i64, _i64, ctypes.c_double, _c_dp, _c_dp, _c_dp]
        lib.oracle_flare_pp_fwd.argtypes = [_c_dp, _c_dp, _c_dp, _c_i32p, _i64, _i64, _i64, _i64,
                                            _i64, ctypes.c_double, _c_dp, _c_dp, _c_dp, _c_dp]
        lib.oracle_flare_bwd.argtypes = [_c_dp, _i64, _c_dp, _c_dp, _c_dp, _c_i32p, _i64, _i64,
                                         _i64, _i64, _i64, ctypes.c_double, _c_dp, _c_dp, _c_dp]
        lib.oracle_flare_pp_bwd.argtypes = [_c_dp, _c_dp, _c_dp, _c_dp, _c_i32p, _i64, _i64,
                                            _i64, _i64, _i64, ctypes.c_double, _c_dp, _c_dp,
                                            _c_dp]
        lib.oracle_encode_bwd.argtypes = lib.oracle_flare_pp_bwd.argtypes
        for f in ("oracle_encode", "oracle_decode", "oracle_decode_rows", "oracle_flare_fwd",
                  "oracle_flare_pp_fwd", "oracle_flare_bwd", "oracle_flare_pp_bwd",
                  "oracle_encode_bwd"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (CPU): exact widening to float64
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(_c_dp)


def _lens(seq_lens, B):
    """The per-batch valid token counts as a ctypes int32 array (None: all
    N); keeps the array alive through the returned tuple."""
    if seq_lens is None:
        return None, None
    if hasattr(seq_lens, "detach"):
        seq_lens = seq_lens.detach().to("cpu").numpy()
    a = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    assert a.shape == (B,), a.shape
    return a, a.ctypes.data_as(_c_i32p)


def _shapes(Q, K, shared_q):
    B, H, N, D = K.shape
    M = Q.shape[-2]
    if shared_q:
        assert Q.shape == (H, M, D), Q.shape
        qbs = 0
    else:
        assert Q.shape == (B, H, M, D), Q.shape
        qbs = H * M * D
    return B, H, N, M, D, qbs


def encode(Q, K, V, scale: float, seq_lens=None):
    """Z [B,H,M,D] and natural-log lse [B,H,M] of softmax_N(s Q K^T) V.

    Q is [H,M,D] (shared over the batch) or [B,H,M,D].  ``seq_lens`` ([B]
    ints, optional): the softmax runs over the first seq_lens[b] tokens only;
    a sequence with none gives Z = 0, lse = -inf.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, N, M, D, qbs = _shapes(Q, K, Q.ndim == 3)
    keep, lp = _lens(seq_lens, B)
    Z = np.empty((B, H, M, D))
    lse = np.empty((B, H, M))
    _load().oracle_encode(_p(Q), qbs, _p(K), _p(V), lp, B, H, N, M, D, float(scale), _p(Z),
                          _p(lse))
    return Z, lse


def decode(Q, K, Z, scale: float, seq_lens=None):
    """Y [B,H,N,D] = softmax_M(s K Q^T) Z (Y = 0 at padded tokens)."""
    Q, K, Z = _f64(Q), _f64(K), _f64(Z)
    B, H, N, M, D, qbs = _shapes(Q, K, Q.ndim == 3)
    keep, lp = _lens(seq_lens, B)
    Y = np.empty((B, H, N, D))
    _load().oracle_decode(_p(Q), qbs, _p(K), _p(Z), lp, B, H, N, M, D, float(scale), _p(Y))
    return Y


def decode_rows(Q, K, Z, scale: float, rows):
    """Y at the flat token indices ``rows`` ((b*H+h)*N+n); returns [len(rows), D]."""
    Q, K, Z = _f64(Q), _f64(K), _f64(Z)
    B, H, N, M, D, qbs = _shapes(Q, K, Q.ndim == 3)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    Yr = np.empty((rows.shape[0], D))
    _load().oracle_decode_rows(_p(Q), qbs, _p(K), _p(Z), B, H, N, M, D, float(scale),
                               rows.ctypes.data_as(_c_i64p), rows.shape[0], _p(Yr))
    return Yr


def flare_fwd(Q, K, V, scale: float, seq_lens=None):
    """FLARE forward: returns (Y, Z, lse).  ``seq_lens``: see encode/decode."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, N, M, D, qbs = _shapes(Q, K, Q.ndim == 3)
    keep, lp = _lens(seq_lens, B)
    Y = np.empty((B, H, N, D))
    Z = np.empty((B, H, M, D))
    lse = np.empty((B, H, M))
    _load().oracle_flare_fwd(_p(Q), qbs, _p(K), _p(V), lp, B, H, N, M, D, float(scale),
                             _p(Y), _p(Z), _p(lse))
    return Y, Z, lse


def flare_pp_fwd(Q, K, V, scale: float, seq_lens=None):
    """FLARE++ forward with learned Q [H,M,D]: returns (Y, Q_dyn, Z, lse)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, N, M, D, _ = _shapes(Q, K, True)
    keep, lp = _lens(seq_lens, B)
    Y = np.empty((B, H, N, D))
    Qd = np.empty((B, H, M, D))
    Z = np.empty((B, H, M, D))
    lse = np.empty((B, H, M))
    _load().oracle_flare_pp_fwd(_p(Q), _p(K), _p(V), lp, B, H, N, M, D, float(scale),
                                _p(Y), _p(Qd), _p(Z), _p(lse))
    return Y, Qd, Z, lse


def flare_bwd(Q, K, V, dY, scale: float, seq_lens=None):
    """Gradients (dQ, dK, dV) of sum(Y * dY) for FLARE.

    dQ is [H,M,D] summed over the batch when Q is shared ([H,M,D] input),
    else [B,H,M,D].
    """
    Q, K, V, dY = _f64(Q), _f64(K), _f64(V), _f64(dY)
    shared = Q.ndim == 3
    B, H, N, M, D, qbs = _shapes(Q, K, shared)
    keep, lp = _lens(seq_lens, B)
    dQ = np.empty(Q.shape)
    dK = np.empty((B, H, N, D))
    dV = np.empty((B, H, N, D))
    _load().oracle_flare_bwd(_p(Q), qbs, _p(K), _p(V), _p(dY), lp, B, H, N, M, D, float(scale),
                             _p(dQ), _p(dK), _p(dV))
    return dQ, dK, dV


def encode_bwd(Q, K, V, dZ, scale: float, seq_lens=None):
    """Gradients (dQ [H,M,D] summed over the batch, dK, dV) of sum(Z * dZ) for
    the encode Z = softmax_N(s Q K^T) V with Q [H,M,D] shared over the batch
    (the FLARE paper's encode step; FLARE++ uses it for the first encode)."""
    Q, K, V, dZ = _f64(Q), _f64(K), _f64(V), _f64(dZ)
    B, H, N, M, D, _ = _shapes(Q, K, True)
    assert dZ.shape == (B, H, M, D), dZ.shape
    keep, lp = _lens(seq_lens, B)
    dQ = np.empty(Q.shape)
    dK = np.empty((B, H, N, D))
    dV = np.empty((B, H, N, D))
    _load().oracle_encode_bwd(_p(Q), _p(K), _p(V), _p(dZ), lp, B, H, N, M, D, float(scale),
                              _p(dQ), _p(dK), _p(dV))
    return dQ, dK, dV


def flare_pp_bwd(Q, K, V, dY, scale: float, seq_lens=None):
    """Gradients (dQ [H,M,D], dK, dV) of sum(Y * dY) for FLARE++ with learned
    Q [H,M,D] (FLARE++ abstract: the encoder's outputs correct the learned
    queries; the chain rule runs through both uses of Q_dyn and through the
    first encode)."""
    Q, K, V, dY = _f64(Q), _f64(K), _f64(V), _f64(dY)
    B, H, N, M, D, _ = _shapes(Q, K, True)
    keep, lp = _lens(seq_lens, B)
    dQ = np.empty(Q.shape)
    dK = np.empty((B, H, N, D))
    dV = np.empty((B, H, N, D))
    _load().oracle_flare_pp_bwd(_p(Q), _p(K), _p(V), _p(dY), lp, B, H, N, M, D, float(scale),
                                _p(dQ), _p(dK), _p(dV))
    return dQ, dK, dV
