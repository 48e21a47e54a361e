"""tp_row_linear_fwd_noalloc: the row-parallel forward for callers that
cannot allocate device memory.

Such callers (code inside a host framework that owns every device
allocation, or a plugin whose interface only hands over input and output
pointers) get the shards' partial products kept in the library's static
scratch instead of a workspace.  Its result must match the regular entry
point, tp_row_linear_fwd, on the same inputs, within the bf16 tolerance the
other GPU tests use, on two calls in a row (the scratch keeps the previous
call's contents, so the second call checks that nothing stale leaks in).
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from tests.gpu_helpers import TOL_BF16, assert_close, f64

pytestmark = pytest.mark.gpu


def _inputs(M, Kin, Nout, seed):
    p = tp_inputs.mlp_inputs(M, Kin, Nout, w_std=0.03, seed=seed)
    return p["X"].cuda(), p["A"].cuda()      # Xin [M, Kin], W [Kin, Nout]


@pytest.mark.parametrize("M,Kin,Nout,N,offsets", [
    (512, 1024, 1024, 4, None),
    (300, 1600, 1600, 4, [0, 448, 832, 1216, 1600]),   # per-shard heads 7/6/6/6 of 64
    (129, 256, 264, 2, None),                           # ragged row and column tiles
    (64, 512, 128, 1, None),                            # one shard: nothing to sum
])
def test_noalloc_matches_regular_entry_point_twice(M, Kin, Nout, N, offsets):
    Xin, W = _inputs(M, Kin, Nout, seed=M + N)
    ref = tpl.tp_row_linear_fwd(Xin, W, N, shard_offsets=offsets)
    torch.cuda.synchronize()
    Z = torch.empty(M, Nout, dtype=torch.bfloat16, device="cuda")
    for call in range(2):
        Z.fill_(float("nan"))
        st = tpl.new_status()
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        tpl.tp_row_linear_fwd_noalloc(Xin, W, N, shard_offsets=offsets, Z=Z, dev_status=st)
        torch.cuda.synchronize()
        if call == 1:
            # the library allocated nothing on the device
            assert torch.cuda.mem_get_info()[0] == free_before
        assert int(st.item()) == 0
        assert_close(f"noalloc call {call}", Z, f64(ref), TOL_BF16)


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
