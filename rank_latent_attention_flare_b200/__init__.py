"""FLARE / FLARE++ low-rank attention routing on B200 (sm_100a).

The compute lives in ``libflare.so`` (hand-written CUDA: tcgen05/TMEM/TMA
tensor-core kernels and CUDA-core kernels) behind the C ABI declared in
``include/flare.h``.  This package is a thin ctypes binding over it.
"""
from ._lib import (FLARE_BF16, FLARE_F32, FLARE_OP_BWD, FLARE_OP_FWD, FLARE_OP_PP_BWD,
                   FLARE_OP_PP_FWD,
                   NOALLOC_SCRATCH_BYTES, FlareError, LIB_PATH, SIGNATURES, load)
from .autograd import FlareFunction, FlarePPFunction, flare, flare_pp
from .flare import (alloc_workspace, bwd_path, default_scale, device_status, encode_records,
                    flare_bwd, flare_bwd_shard_dz, flare_bwd_shard_finish, flare_combine,
                    flare_combine_shards, flare_decode, flare_encode, flare_fwd, flare_fwd_host,
                    flare_fwd_noalloc,
                    flare_pp_bwd, flare_pp_bwd_shard_tail, flare_pp_fwd, fwd_path, records_layout,
                    workspace_size, noalloc_device_status, probe_unit_rates, probe_mma_rates, eval_exp2,
                    selftest_wait_timeout, exp_split)
from . import parallel

__all__ = [
    "FLARE_BF16", "FLARE_F32", "FLARE_OP_BWD", "FLARE_OP_FWD", "FLARE_OP_PP_BWD",
    "FLARE_OP_PP_FWD", "FlareError",
    "LIB_PATH", "SIGNATURES", "load", "alloc_workspace", "default_scale", "device_status",
    "flare_bwd", "flare_combine", "flare_decode", "flare_encode", "flare_fwd", "flare_fwd_host",
    "flare_fwd_noalloc",
    "flare_pp_bwd", "flare_pp_fwd", "NOALLOC_SCRATCH_BYTES",
    "bwd_path", "fwd_path", "workspace_size",
    "FlareFunction", "FlarePPFunction", "flare", "flare_pp",
    "encode_records", "flare_bwd_shard_dz", "flare_bwd_shard_finish", "flare_combine_shards",
    "records_layout", "parallel", "flare_pp_bwd_shard_tail", "noalloc_device_status",
    "probe_unit_rates", "probe_mma_rates", "eval_exp2", "selftest_wait_timeout", "exp_split",
]
