"""tp_row_linear_fwd_noalloc: the row-parallel forward for callers that
cannot allocate device memory.

Such callers (code inside a host framework that owns every device
allocation, or a plugin whose interface only hands over input and output
pointers) get the shards' partial products kept in the library's static
scratch instead of a workspace.  Each call is checked against the fp64
oracle's row-parallel product (the g sum of [TP-ILL] §1.1) and against the
regular entry point, tp_row_linear_fwd, within the bf16 tolerance the other
GPU tests use.  Two calls run back to back on DIFFERENT inputs and shard
counts: the scratch keeps the previous call's partials and counters, so a
call that read a stale partial or a counter left from the call before would
produce the first call's numbers and fail the second comparison.  This file
is collected last so that a run stopping at the first failure has already
run every other test.
"""
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, assert_close, f64, guarded

pytestmark = pytest.mark.gpu


def _inputs(M, Kin, Nout, seed):
    p = tp_inputs.mlp_inputs(M, Kin, Nout, w_std=0.03, seed=seed)
    return p["X"], p["A"]      # Xin [M, Kin], W [Kin, Nout]


# (M, Kin, Nout, N, offsets) of the first and the second call: same output
# shape, other inputs and another shard count each time
PAIRS = [
    ((512, 1024, 1024, 4, None), (512, 1024, 1024, 2, None)),
    ((300, 1600, 1600, 4, [0, 448, 832, 1216, 1600]),      # per-shard heads 7/6/6/6 of 64
     (300, 1600, 1600, 5, None)),
    ((129, 256, 264, 2, None), (129, 256, 264, 4, None)),   # ragged row and column tiles
    ((64, 512, 128, 1, None), (64, 512, 128, 8, None)),     # one shard: nothing to sum
]


@pytest.mark.parametrize("first,second", PAIRS)
def test_noalloc_matches_oracle_on_two_different_calls(first, second):
    M, _, Nout, _, _ = first
    Z, guard = guarded((M, Nout), torch.bfloat16)
    for call, (Mc, Kin, Nc, N, offsets) in enumerate((first, second)):
        Xin, W = _inputs(Mc, Kin, Nc, seed=1000 * call + Mc + N)
        if call == 1:
            Xin = -Xin        # nothing of the first call's partials can be right here
        Xd, Wd = Xin.cuda(), W.cuda()
        Z.fill_(float("nan"))
        st = tpl.new_status()
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        tpl.tp_row_linear_fwd_noalloc(Xd, Wd, N, shard_offsets=offsets, Z=Z, dev_status=st)
        torch.cuda.synchronize()
        # the library allocated nothing on the device (the first call of the
        # process may load the module's static scratch; later calls reserve nothing)
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
        assert int(st.item()) == 0
        guard.check(f"noalloc Z, call {call}")
        want = O.row_linear_fwd(Xin, W, offsets=offsets, N=N)[0]
        assert_close(f"noalloc call {call} vs oracle", Z, want, TOL_BF16)
        ref = tpl.tp_row_linear_fwd(Xd, Wd, N, shard_offsets=offsets)
        torch.cuda.synchronize()
        assert_close(f"noalloc call {call} vs tp_row_linear_fwd", Z, f64(ref), TOL_BF16)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    # 32 x 16 output tiles x 8 shards of 128 KB partials = 512 MB > 32 MB
    Xin = torch.empty(4096, 4096, dtype=torch.bfloat16, device="cuda")
    W = torch.empty(4096, 4096, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tpl.TPError) as e:
        tpl.tp_row_linear_fwd_noalloc(Xin, W, 8)
    assert e.value.status == 7   # TP_ERR_WORKSPACE: the static scratch is too small
    with pytest.raises(tpl.TPError) as e:
        tpl.tp_row_linear_fwd_noalloc(Xin[:64].float(), W.float(), 8)
    assert e.value.status == 4   # TP_ERR_DTYPE: bf16 only
