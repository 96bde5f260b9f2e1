"""The measurement and self-test calls on the device: the unit-rate probe
behind the roofline, the kernels' exponentials against their error bounds,
and a bounded wait that runs out (no fault, no hang: the wait's own limit
ends it and the device stays usable)."""
import math

import numpy as np
import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import assert_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

# The polynomial's stated relative error on [-1/2, 1/2] (Remez fit).
POLY_REL = 7.5e-5


def test_probe_unit_rates_are_plausible():
    r = fl.probe_unit_rates()
    assert r["sms"] == torch.cuda.get_device_properties(0).multi_processor_count
    assert 500.0 < r["sm_mhz"] < 2500.0, r
    # B200: 16 ex2 / clk / SM, 128 fp32 FMA / clk / SM (within a broad margin)
    assert 8.0 < r["ex2_per_clk_sm"] < 40.0, r
    assert 64.0 < r["fma_per_clk_sm"] < 300.0, r
    assert 64.0 < r["fma2_per_clk_sm"] < 600.0, r
    assert 4.0 < r["mix_ex2_per_clk_sm"] < 40.0, r


def test_probe_mma_rates_are_plausible():
    # The tensor core's math alone takes 2 M N K / 8192 clocks per product
    # at B200's dense bf16 rate (~8K flops / clk / SM), so no product is
    # cheaper than that; a product of N = 256 is math-bound, and an A operand
    # read from shared memory (4 KB) costs at least 4096 / 128 = 32 clocks
    # of the shared-memory port once several threads keep the SM busy.
    r = fl.probe_mma_rates()
    for k, v in r.items():
        assert 1.0 < v < 1000.0, (k, v)
    assert r["ss_n256_x1"] >= 0.9 * 2 * 128 * 256 * 16 / 8192, r
    assert r["ss_n32_x4"] >= 0.9 * 4096 / 128, r
    # with A in TMEM, four issuers get more products per clock than with A
    # in shared memory
    assert r["ts_n32_x4"] < r["ss_n32_x4"], r
    with pytest.raises(fl.FlareError):   # 4 issuers x 128 columns do not fit
        fl.probe_mma_rates(cases=[(128, 0, 4)])


def _grid():
    xs = [np.linspace(-130.0, 126.0, 1 << 20)]
    k = np.arange(-130, 127, dtype=np.float64)
    # integers, half-integers (the rounding boundary of the range reduction)
    # and their float32 neighbours
    for base in (k, k + 0.5):
        b = base.astype(np.float32)
        xs += [b, np.nextafter(b, np.float32(np.inf)), np.nextafter(b, np.float32(-np.inf))]
    x = np.concatenate([np.asarray(v, dtype=np.float32) for v in xs])
    return x[(x >= -130.0) & (x <= 126.0)]


@pytest.mark.parametrize("form", [1, 2], ids=["scalar", "packed"])
def test_exp2_polynomial_within_its_bound(form):
    x = _grid()
    y = fl.eval_exp2(torch.from_numpy(x).to(DEV), form).cpu().numpy().astype(np.float64)
    x64 = x.astype(np.float64)
    valid = x64 >= -125.0
    rel = np.abs(y[valid] / np.exp2(x64[valid]) - 1.0)
    assert float(rel.max()) <= POLY_REL, (float(rel.max()), float(x64[valid][rel.argmax()]))
    # below -125 the input is clamped: the result is 2^-125 within the bound
    low = np.abs(y[~valid] / 2.0 ** -125 - 1.0)
    assert low.size > 0 and float(low.max()) <= POLY_REL


def test_exp2_clamped_polynomial_within_its_bound():
    # the softmax loops' form: exponent clamped to [-125, 126] by a
    # saturating FMA that computes y = x (1/251) + 125/251.  Error in the
    # exponent: the float32 constants' rounding ((|x| + 125) 2^-24) and y's
    # own (251 * 2^-25), on top of the polynomial's 7.5e-5 relative.
    x = np.concatenate([_grid(), np.linspace(126.0, 400.0, 4096, dtype=np.float32),
                        np.float32([np.inf, -np.inf, 1e30, -1e30])])
    y = fl.eval_exp2(torch.from_numpy(x).to(DEV), 3).cpu().numpy().astype(np.float64)
    xc = np.clip(x.astype(np.float64), -125.0, 126.0)
    bound = POLY_REL + math.log(2.0) * ((np.abs(xc) + 125.0) * 2.0 ** -24 + 251.0 * 2.0 ** -25)
    rel = np.abs(y / np.exp2(xc) - 1.0)
    assert np.isfinite(y).all()
    assert (rel <= bound).all(), (float(rel.max()), float(x[rel.argmax()]))


def test_exp2_forms_agree_bitwise():
    # the packed form is the scalar one in packed instructions: same result
    x = torch.from_numpy(_grid()).to(DEV)
    assert torch.equal(fl.eval_exp2(x, 1), fl.eval_exp2(x, 2))


def test_exp2_mufu_reference():
    x = _grid()
    x = x[x >= -126.0]   # ftz: results below 2^-126 flush to zero
    y = fl.eval_exp2(torch.from_numpy(x).to(DEV), 0).cpu().numpy().astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert float(rel.max()) <= 2.0 ** -21


@pytest.mark.parametrize("limit_ns", [0, 2_000_000], ids=["immediate", "2ms"])
def test_bounded_wait_runs_out_and_reports(limit_ns):
    ws = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    fl.selftest_wait_timeout(ws, limit_ns)
    detail = ctypes_status(ws)
    assert detail == (5, 0x701)
    # read and cleared: a second read is clean
    assert ctypes_status(ws) == (0, 0)
    # the device is still usable: a forward call afterwards is correct
    B, H, N, M, D = 1, 2, 700, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=4)
    g = {k: v.to(DEV) for k, v in x.items()}
    wsf = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, torch.bfloat16, DEV)
    Y = fl.flare_fwd(g["Q"], g["K"], g["V"], s, workspace=wsf)
    assert fl.device_status(wsf) == 0
    Yo, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Y, Yo, torch.bfloat16, "Y after a timed-out wait")


def ctypes_status(ws):
    import ctypes
    detail = ctypes.c_uint32(0)
    st = fl.load().flare_device_status(ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                       ctypes.byref(detail),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return int(st), int(detail.value)


def test_selftest_rejects_bad_arguments():
    ws = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(fl.FlareError) as e:
        fl.selftest_wait_timeout(ws[:256], 1000)
    assert e.value.status == 3
    with pytest.raises(fl.FlareError) as e:
        fl.selftest_wait_timeout(ws, 5_000_000_000)
    assert e.value.status == 1
