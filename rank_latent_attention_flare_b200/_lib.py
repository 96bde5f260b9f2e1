"""ctypes declarations of the C ABI in include/flare.h.

Loads the in-tree ``libflare.so``.  There is no fallback: if the library is
missing or does not load, importing the binding raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libflare.so")

FLARE_F32 = 0
FLARE_BF16 = 1

FLARE_OP_FWD = 0
FLARE_OP_PP_FWD = 1
FLARE_OP_BWD = 2
FLARE_OP_PP_BWD = 3

# Size of the fixed device scratch array behind flare_fwd_noalloc.
NOALLOC_SCRATCH_BYTES = 32 << 20

STATUS_NAMES = {
    0: "FLARE_OK",
    1: "FLARE_ERR_INVALID_ARG",
    2: "FLARE_ERR_UNSUPPORTED",
    3: "FLARE_ERR_WORKSPACE",
    4: "FLARE_ERR_CUDA",
    5: "FLARE_ERR_DEVICE_TIMEOUT",
}

# Every symbol include/flare.h declares, with (restype, argtypes).
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_f32 = ctypes.c_float
_sz = ctypes.c_size_t
_u32p = ctypes.POINTER(ctypes.c_uint32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_szp = ctypes.POINTER(ctypes.c_size_t)


class FlareStrides(ctypes.Structure):
    """flare_strides_t: element strides of a [B,H,N,D] token tensor."""
    _fields_ = [("b_stride", ctypes.c_int64), ("h_stride", ctypes.c_int64),
                ("n_stride", ctypes.c_int64)]


_stp = ctypes.POINTER(FlareStrides)


class UnitRates(ctypes.Structure):
    """flare_unit_rates_t: probe throughputs per SM per SM clock."""
    _fields_ = [("sms", ctypes.c_int), ("sm_mhz", ctypes.c_double),
                ("ex2_per_clk_sm", ctypes.c_double), ("fma_per_clk_sm", ctypes.c_double),
                ("fma2_per_clk_sm", ctypes.c_double), ("mix_ex2_per_clk_sm", ctypes.c_double),
                ("mix_fma_per_clk_sm", ctypes.c_double), ("ex2_ms", ctypes.c_double),
                ("fma_ms", ctypes.c_double), ("fma2_ms", ctypes.c_double),
                ("mix_ms", ctypes.c_double)]

SIGNATURES = {
    "flare_version": (_i32, []),
    "flare_last_error_detail": (ctypes.c_char_p, []),
    "flare_status_string": (ctypes.c_char_p, [_i32]),
    "flare_workspace_size": (_sz, [_i32, _i64, _i64, _i64, _i64, _i64, _i32]),
    "flare_fwd": (_i32, [_vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i32, _f32,
                         _vp, _vp, _vp, _sz, _vp]),
    "flare_pp_fwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i32, _f32,
                            _vp, _vp, _vp, _sz, _vp]),
    "flare_fwd_host": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                              _i64, _i32, _f32, _vp, _sz, _vp, _vp]),
    "flare_fwd_host_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i64, _i32]),
    "flare_bwd": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                         _i64, _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_pp_bwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                            _i64, _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_fwd_ex": (_i32, [_vp, _i64, _vp, _vp, _vp, _stp, _vp, _i64, _i64, _i64, _i64, _i64,
                                 _i32, _f32, _vp, _vp, _vp, _sz, _vp]),
    "flare_pp_fwd_ex": (_i32, [_vp, _vp, _vp, _vp, _vp, _stp, _vp, _i64, _i64, _i64, _i64, _i64,
                                    _i32, _f32, _vp, _vp, _vp, _sz, _vp]),
    "flare_bwd_ex": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _stp, _vp, _i64,
                                 _i64, _i64, _i64, _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_pp_bwd_ex": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _stp, _vp, _i64,
                                    _i64, _i64, _i64, _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_records_layout": (_i32, [_i64, _i64, _i64, _i64, _i64, _i32, _i64p, _szp, _szp]),
    "flare_combine_shards": (_i32, [_i64, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _i32, _vp,
                                    _vp, _vp, _vp, _vp, _sz, _vp]),
    "flare_pp_bwd_shard_tail": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i64, _i64,
                                       _i64, _i64, _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_bwd_shard_dz": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                  _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_bwd_shard_finish": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                      _i64, _i64, _i64, _i64, _i32, _f32, _vp, _sz, _vp]),
    "flare_encode": (_i32, [_vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i32, _f32, _vp,
                            _sz, _vp]),
    "flare_combine": (_i32, [_i64, _i64, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _sz, _vp]),
    "flare_decode": (_i32, [_vp, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i32, _f32, _vp,
                            _sz, _vp]),
    "flare_device_status": (_i32, [_vp, _sz, _u32p, _vp]),
    "flare_fwd_path": (_i32, [_i64, _i64, _i64, _i64, _i64, _i32]),
    "flare_bwd_path": (_i32, [_i64, _i64, _i64, _i64, _i64, _i32]),
    "flare_fwd_noalloc": (_i32, [_vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i32,
                                 _f32, _vp, _vp, _vp]),
    "flare_noalloc_device_status": (_i32, [_u32p, _vp]),
    "flare_probe_scratch_bytes": (_sz, []),
    "flare_probe_unit_rates": (_i32, [_vp, _sz, ctypes.POINTER(UnitRates), _vp]),
    "flare_eval_exp2": (_i32, [_vp, _vp, _i64, _i32, _vp]),
    "flare_exp_split": (_i32, [_i32, _i64, _i64, _i32, ctypes.POINTER(ctypes.c_double)]),
    "flare_probe_mma_rate": (_i32, [_i32, _i32, _i32, _vp, _sz, ctypes.POINTER(ctypes.c_double),
                                    _vp]),
    "flare_selftest_wait_timeout": (_i32, [_vp, _sz, ctypes.c_uint64, _vp]),
}

_lib = None


class FlareError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        text = STATUS_NAMES.get(status, f"status {status}")
        super().__init__(f"{where}: {text}")


def load() -> ctypes.CDLL:
    """Load libflare.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m rank_latent_attention_flare_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(status: int, where: str) -> None:
    if status != 0:
        detail = ""
        if status == 4 and _lib is not None:
            detail = (_lib.flare_last_error_detail() or b"").decode(errors="replace")
        raise FlareError(status, where + (f" [{detail}]" if detail else ""))
