"""Attention projections with per-shard heads (GPT-2 1.5B layer slice:
h=1600, 25 heads of 64 over N=4 shards -> 7, 6, 6, 6 heads): column-parallel
QKV and row-parallel output projection with its shard sum, forward and
backward, on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, assert_close, f64, guarded, to_dev

pytestmark = pytest.mark.gpu


def _head_offsets(n_heads, head_dim, N, per_head_cols):
    heads = tp_inputs.head_split(n_heads, N)
    offs = [0]
    for nh in heads:
        offs.append(offs[-1] + nh * head_dim * per_head_cols)
    return heads, offs


def _case(M, seed, zpart):
    w = tp_inputs.WORKLOADS["gpt2_1p5b_slice"]
    h, nh, hd, N = w["h"], w["n_heads"], w["head_dim"], w["N"]
    inp = tp_inputs.attn_proj_inputs(M, h, nh, hd, N, seed=seed)
    d = to_dev(inp)
    heads, qkv_offs = _head_offsets(nh, hd, N, 3)
    _, ctx_offs = _head_offsets(nh, hd, N, 1)
    assert heads == [7, 6, 6, 6]
    assert ctx_offs == [0, 448, 832, 1216, 1600]
    bf = torch.bfloat16
    # every output inside a guard band (NaN-filled, sentinel margins): the
    # 1600-wide outputs end in a 64-column tile and M=640 in a half row tile
    shapes = {"QKV": ((M, 3 * h), bf), "dX": ((M, h), bf), "dWq": ((h, 3 * h), bf),
              "dbq": ((3 * h,), torch.float32), "Z": ((M, h), bf), "dctx": ((M, h), bf),
              "dWo": ((h, h), bf)}
    if zpart:
        shapes["Zp"] = ((N, M, h), torch.float32)
    o, guards = {}, {}
    for k, (shape, t) in shapes.items():
        o[k], guards[k] = guarded(shape, t)
    st = tpl.new_status()
    # QKV: column-parallel, shard-major columns (own Q, K, V heads per shard)
    QKV, _ = tpl.tp_col_linear_fwd(d["X"], d["Wqkv"], d["bqkv"], N, shard_offsets=qkv_offs,
                                   Y=o["QKV"], dev_status=st)
    gq = tpl.tp_col_linear_bwd(d["X"], d["Wqkv"], None, d["dQKV"], N, shard_offsets=qkv_offs,
                               dX=o["dX"], dW=o["dWq"], dbias=o["dbq"], dev_status=st)
    # output projection: row-parallel over the per-shard context, summed
    Zp = o.get("Zp")
    Z = tpl.tp_row_linear_fwd(d["ctx"], d["Wo"], N, shard_offsets=ctx_offs, Zpart=Zp, Z=o["Z"],
                              dev_status=st)
    go = tpl.tp_row_linear_bwd(d["ctx"], d["Wo"], d["dZ"], N, shard_offsets=ctx_offs,
                               dXin=o["dctx"], dW=o["dWo"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for k, gd in guards.items():
        gd.check(k)
    return inp, qkv_offs, ctx_offs, QKV, gq, Z, Zp, go


@pytest.mark.parametrize("zpart", [False, True])
def test_attention_projections(zpart):
    inp, qkv_offs, ctx_offs, QKV, gq, Z, Zp, go = _case(640, 3, zpart)
    _, oQKV = O.col_linear_fwd(inp["X"], inp["Wqkv"], inp["bqkv"])
    assert_close("QKV", QKV, oQKV, TOL_BF16)
    ob = O.col_linear_bwd(inp["X"], inp["Wqkv"], oQKV, inp["dQKV"])
    assert_close("dX (f sum over QKV shards)", gq["dX"], ob["dX"], TOL_BF16)
    assert_close("dWqkv", gq["dW"], ob["dW"], TOL_BF16)
    assert_close("dbqkv", gq["dbias"], ob["dbias"], TOL_BF16)
    oZ, parts = O.row_linear_fwd(inp["ctx"], inp["Wo"], offsets=ctx_offs)
    assert_close("Z (g sum over uneven shards)", Z, oZ, TOL_BF16)
    if zpart:
        for i in range(4):
            assert_close(f"Zpart[{i}]", Zp[i], parts[i], TOL_BF16)
    obo = O.row_linear_bwd(inp["ctx"], inp["Wo"], inp["dZ"])
    assert_close("dctx", go["dXin"], obo["dXin"], TOL_BF16)
    assert_close("dWo", go["dW"], obo["dW"], TOL_BF16)


def test_shard_major_heads_are_the_standard_heads():
    """The per-shard Q/K/V blocks are a column permutation of the standard
    [Q | K | V] projection: permuting the weight and the output agrees."""
    M = 256
    w = tp_inputs.WORKLOADS["gpt2_1p5b_slice"]
    h, nh, hd, N = w["h"], w["n_heads"], w["head_dim"], w["N"]
    inp = tp_inputs.attn_proj_inputs(M, h, nh, hd, N, seed=7)
    perm, offs = O.qkv_shard_columns(nh, hd, tp_inputs.head_split(nh, N))
    W_std = torch.empty_like(inp["Wqkv"])
    W_std[:, torch.as_tensor(perm)] = inp["Wqkv"]   # shard-major column j is standard perm[j]
    Y_sm, _ = tpl.tp_col_linear_fwd(inp["X"].cuda(), inp["Wqkv"].cuda(), None, N, shard_offsets=offs)
    Y_std, _ = tpl.tp_col_linear_fwd(inp["X"].cuda(), W_std.cuda(), None, 1)
    torch.cuda.synchronize()
    assert_close("permuted heads", Y_std[:, torch.as_tensor(perm).cuda()], f64(Y_sm), 1e-3)


@pytest.mark.slow
def test_attention_projections_full_m():
    M = tp_inputs.WORKLOADS["gpt2_1p5b_slice"]["M"]
    inp, qkv_offs, ctx_offs, QKV, gq, Z, Zp, go = _case(M, 0, False)
    rows = torch.as_tensor(np.r_[0:128, 1000:1064, M - 64:M])
    _, oQKV = O.col_linear_fwd(inp["X"][rows], inp["Wqkv"], inp["bqkv"])
    assert_close("QKV[rows]", QKV[rows.cuda()], oQKV, TOL_BF16)
    oZ, _ = O.row_linear_fwd(inp["ctx"][rows], inp["Wo"], offsets=ctx_offs)
    assert_close("Z[rows]", Z[rows.cuda()], oZ, TOL_BF16)
    ob = O.row_linear_bwd(inp["ctx"][rows], inp["Wo"], inp["dZ"][rows])
    assert_close("dctx[rows]", go["dXin"][rows.cuda()], ob["dXin"], TOL_BF16)
    cols = torch.as_tensor(np.r_[0:64, 700:764])
    obw = O.row_linear_bwd(inp["ctx"], inp["Wo"][:, cols], inp["dZ"][:, cols])
    assert_close("dWo[:,cols]", go["dW"][:, cols.cuda()], obw["dW"], TOL_BF16)
    obq = O.col_linear_bwd(inp["X"], inp["Wqkv"][:, cols], None, inp["dQKV"][:, cols])
    assert_close("dWqkv[:,cols]", gq["dW"][:, cols.cuda()], obq["dW"], TOL_BF16)
    assert_close("dbqkv[cols]", gq["dbias"][cols.cuda()], obq["dbias"], TOL_BF16)


@pytest.mark.parametrize("act", [tpl.ACT_GELU_TANH, tpl.ACT_GELU_ERF, tpl.ACT_NONE])
@pytest.mark.parametrize("M,K,Nout,N", [(200, 192, 1600, 4), (1000, 320, 648, 3)])
def test_col_linear_bwd_with_activation(M, K, Nout, N, act):
    """The column-parallel backward with an activation: dU = dY ⊙ act'(U)
    and dbias = Σ_rows dU come from the element-wise column-sum kernel
    (32-row partial sums, ragged last block), then dW and dX."""
    g = torch.Generator().manual_seed(M + Nout + act)
    X = (torch.randn(M, K, generator=g) * 0.5).bfloat16()
    W = (torch.randn(K, Nout, generator=g) * 0.05).bfloat16()
    U = torch.randn(M, Nout, generator=g).bfloat16()
    dY = torch.randn(M, Nout, generator=g).bfloat16()
    bf = torch.bfloat16
    dX, gx = guarded((M, K), bf)
    dW, gw = guarded((K, Nout), bf)
    dbias, gb = guarded((Nout,), torch.float32)
    dU, gu = guarded((M, Nout), bf) if act != tpl.ACT_NONE else (None, None)
    st = tpl.new_status()
    out = tpl.tp_col_linear_bwd(X.cuda(), W.cuda(), U.cuda() if act != tpl.ACT_NONE else None,
                                dY.cuda(), N, act=act, dU=dU, dX=dX, dW=dW, dbias=dbias,
                                dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for gd, name in ((gx, "dX"), (gw, "dW"), (gb, "dbias"), (gu, "dU")):
        if gd is not None:
            gd.check(name)
    ref = O.col_linear_bwd(X, W, U, dY, act)   # act' = 1 everywhere without an activation
    if act != tpl.ACT_NONE:
        assert_close("dU", f64(out["dU"]), ref["dU"], TOL_BF16)
    assert_close("dbias", f64(out["dbias"]), ref["dbias"], TOL_BF16)
    assert_close("dW", f64(out["dW"]), ref["dW"], TOL_BF16)
    assert_close("dX", f64(out["dX"]), ref["dX"], TOL_BF16)
