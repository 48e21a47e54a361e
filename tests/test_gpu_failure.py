"""Failure detection on the device without a GPU fault.

A kernel whose partner never signals must not hang: every pipeline wait in
the library is bounded, records TP_DEVERR_TIMEOUT in the caller's status
word and returns.  The self-test kernel waits on a barrier nothing arrives
on; afterwards the context must still run the real kernels correctly.
"""
import time

import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, assert_close, to_dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    st = tpl.new_status()
    t0 = time.perf_counter()
    tpl.tp_selftest_wait_timeout(st, limit_us=2000)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) & tpl.DEVERR_TIMEOUT
    assert dt < 5.0
    # the context is intact: a real call still runs and matches the oracle
    inp = tp_inputs.mlp_inputs(130, 64, 256, w_std=0.1, seed=11)
    d = to_dev(inp)
    st2 = tpl.new_status()
    Z, U, Y = tpl.tp_mlp_fwd(d["X"], d["A"], d["bias"], d["B"], 2, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert_close("Z after timeout", Z, O.mlp_fwd(inp["X"], inp["A"], inp["bias"], inp["B"])[2],
                 TOL_BF16)


def test_selftest_argument_checks():
    with pytest.raises(tpl.TPError):
        tpl.tp_selftest_wait_timeout(tpl.new_status(), limit_us=0)


def _clean_mlp_matches_oracle(seed):
    inp = tp_inputs.mlp_inputs(300, 256, 1024, w_std=0.05, bias_std=0.02, seed=seed)
    d = to_dev(inp)
    st = tpl.new_status()
    Z, U, Y = tpl.tp_mlp_fwd(d["X"], d["A"], d["bias"], d["B"], 4, dev_status=st)
    g = tpl.tp_mlp_bwd(d["X"], d["A"], d["B"], U, Y, d["dZ"], 4, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    oU, oY, oZ = O.mlp_fwd(inp["X"], inp["A"], inp["bias"], inp["B"])
    ob = O.mlp_bwd(inp["X"], inp["A"], inp["bias"], inp["B"], inp["dZ"])
    assert_close("Z", Z, oZ, TOL_BF16)
    for k in ("dX", "dA", "dB", "dbias"):
        assert_close(k, g[k], ob[k], TOL_BF16)


@pytest.mark.parametrize("tile", ["2x256", "2x256t", "2x128", "1x256", "1x128"])
@pytest.mark.parametrize("unit,kblock", [(0, 1), (0, 0), (1, 2)])
def test_gemm_producer_stall_times_out_drains_and_recovers(tile, unit, kblock, monkeypatch):
    """The real GEMM pipeline's failure path: the producers of one CTA (pair)
    stop before a k-block (the injection), the MMA issuer's bounded wait runs
    out, the launch reports TP_DEVERR_TIMEOUT within the limit, drains its
    copies and MMAs, frees its tensor memory and returns; the next calls on
    the same context are correct."""
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    inp = tp_inputs.mlp_inputs(300, 256, 1024, w_std=0.05, seed=13)   # 4 k-blocks per unit
    d = to_dev(inp)
    torch.cuda.synchronize()
    st = tpl.new_status()
    tpl.tp_debug_stall_next_gemm(unit, kblock, wait_limit_us=50000)
    t0 = time.perf_counter()
    tpl.tp_mlp_fwd(d["X"], d["A"], d["bias"], d["B"], 4, dev_status=st)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) & tpl.DEVERR_TIMEOUT
    assert dt < 2.0, dt          # a few 50 ms waits, not a hang
    _clean_mlp_matches_oracle(seed=14)


def test_split_sum_stall_times_out_and_recovers():
    """The same on the row-parallel GEMM's split shard sum (partials and
    arrival counters of the stalled tile are left behind; the next call
    clears the counters and is correct)."""
    inp = tp_inputs.mlp_inputs(512, 4096, 256, w_std=0.02, seed=15)
    Xin, W = inp["X"].cuda(), inp["A"].cuda()            # [512, 4096] x [4096, 256], 8 shards
    st = tpl.new_status()
    tpl.tp_debug_stall_next_gemm(0, 3, wait_limit_us=50000)
    tpl.tp_row_linear_fwd(Xin, W, 8, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tpl.DEVERR_TIMEOUT
    st2 = tpl.new_status()
    Z = tpl.tp_row_linear_fwd(Xin, W, 8, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert_close("Z after a stalled split sum", Z, O.row_linear_fwd(inp["X"], inp["A"])[0], TOL_BF16)


def test_injection_argument_checks():
    with pytest.raises(tpl.TPError):
        tpl.tp_debug_stall_next_gemm(-1, 0)
    with pytest.raises(tpl.TPError):
        tpl.tp_debug_stall_next_gemm(0, 0, wait_limit_us=0)
