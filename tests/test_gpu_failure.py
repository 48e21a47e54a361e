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
