"""Vocabulary-parallel backward on the GPU against the fp64 oracle: the bf16
gradient of the cross-entropy, the output-embedding backward (dH, dE), the
input-embedding scatter-add, and the gradient of a table shared by both
(the sum the pages prescribe for tied input/output embeddings)."""
import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, TOL_XENT, assert_close, f64

pytestmark = pytest.mark.gpu
TOL_F32_SUM = 1e-6   # fp32 sums of bf16 rows in token order vs fp64


@pytest.mark.parametrize("v,N", [(1024, 4), (50304, 8), (1002, 3)])
def test_xent_bf16_gradient(v, N):
    inp = tp_inputs.xent_logits(129, v, seed=31)
    st = tpl.new_status()
    r = tpl.vp_xent_bf16_grad(inp["logits"].cuda(), inp["targets"].cuda(), N, grad_scale=0.5,
                              dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = O.xent(inp["logits"], inp["targets"], 0.5)
    rel = np.abs(f64(r["loss"]) - ref["loss"]) / np.abs(ref["loss"])
    assert rel.max() <= TOL_XENT
    assert r["dlogits"].dtype == torch.bfloat16
    assert_close("bf16 dlogits", r["dlogits"], ref["dlogits"], TOL_BF16)
    assert np.array_equal(r["argmax"].cpu().numpy().astype(np.int64), ref["argmax"])


def test_logits_bwd_ragged():
    T, v, h, N = 300, 1000, 264, 4
    b = tp_inputs.vocab_bwd_inputs(T, v, h, seed=32)
    f = tp_inputs.vocab_inputs(T, v, h, seed=33)
    st = tpl.new_status()
    dH, dE = tpl.tp_logits_bwd(b["dlogits"].cuda(), f["H"].cuda(), f["E"].cuda(), N, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = O.logits_bwd(b["dlogits"], f["H"], f["E"])
    assert_close("dH", dH, ref["dH"], TOL_BF16)
    assert_close("dE", dE, ref["dE"], 1e-4)
    s = O.logits_bwd_sharded(b["dlogits"], f["H"], f["E"], N)
    for i in range(N):   # each shard's block of dE is its own
        assert_close(f"dE shard {i}", dE[i * 250:(i + 1) * 250], s["dE"][i * 250:(i + 1) * 250], 1e-4)


@pytest.mark.slow
def test_logits_bwd_full_size_sampled():
    w = tp_inputs.WORKLOADS["vocab_v50304"]
    T, v, h, N = w["T"], w["v"], w["h"], w["N"]
    b = tp_inputs.vocab_bwd_inputs(T, v, h, seed=0)
    f = tp_inputs.vocab_inputs(T, v, h, seed=0)
    dH, dE = tpl.tp_logits_bwd(b["dlogits"].cuda(), f["H"].cuda(), f["E"].cuda(), N)
    torch.cuda.synchronize()
    rows = torch.as_tensor(np.r_[0:32, 9000:9032, T - 32:T])
    ref = O.logits_bwd(b["dlogits"][rows], f["H"][rows], f["E"])
    assert_close("dH[rows]", dH[rows.cuda()], ref["dH"], TOL_BF16)
    vrows = torch.as_tensor(np.r_[0:32, 25000:25032, v - 32:v])
    refE = O.f64(b["dlogits"][:, vrows]).T @ O.f64(f["H"])
    assert_close("dE[vocab rows]", dE[vrows.cuda()], refE, 1e-4)


def _embed_bwd_case(T, v, h, N, seed, ids=None):
    b = tp_inputs.vocab_bwd_inputs(T, v, h, seed=seed)
    if ids is not None:
        b["ids"] = ids
    dE = b["dE0"].cuda().clone()
    st = tpl.new_status()
    tpl.vp_embed_bwd(b["ids"].cuda(), b["dout"].cuda(), dE, N, dev_status=st)
    torch.cuda.synchronize()
    ref = O.f64(b["dE0"]) + O.embed_bwd(b["ids"], b["dout"], v)
    return dE, ref, st, b


def test_embed_bwd_repeats_and_out_of_range():
    ids = torch.tensor([3, 17, 3, 39, 0, 17, 3, 25, -1, 40, 39], dtype=torch.int64)
    dE, ref, st, b = _embed_bwd_case(ids.shape[0], 40, 64, 4, 34, ids=ids)
    assert int(st.item()) & tpl.DEVERR_RANGE
    assert_close("dE", dE, ref, TOL_F32_SUM)
    sharded = O.f64(b["dE0"]) + O.embed_bwd_sharded(ids, b["dout"], 40, 4)
    assert_close("dE sharded", dE, sharded, TOL_F32_SUM)


@pytest.mark.parametrize("T,v,h,N", [(3000, 4096, 264, 8), (20000, 2048, 64, 2)])
def test_embed_bwd_random_and_deterministic(T, v, h, N):
    # T=20000 exceeds the 16384 keys sorted in shared memory: global sort path
    dE, ref, st, b = _embed_bwd_case(T, v, h, N, 35)
    assert int(st.item()) == 0
    assert_close("dE", dE, ref, TOL_F32_SUM)
    dE2 = b["dE0"].cuda().clone()
    tpl.vp_embed_bwd(b["ids"].cuda(), b["dout"].cuda(), dE2, N)
    torch.cuda.synchronize()
    assert torch.equal(dE, dE2)


@pytest.mark.slow
def test_embed_bwd_full_size():
    w = tp_inputs.WORKLOADS["vocab_v50304"]
    dE, ref, st, _ = _embed_bwd_case(w["T"], w["v"], w["h"], w["N"], 0)
    assert int(st.item()) == 0
    assert_close("dE", dE, ref, TOL_F32_SUM)


def test_tied_table_gradient_chain():
    """Logits → bf16 cross-entropy gradient → dH, dE → plus the input-side
    scatter-add: the shared table's gradient, against the oracle chain."""
    T, v, h, N = 256, 2048, 128, 8
    f = tp_inputs.vocab_inputs(T, v, h, seed=36)
    b = tp_inputs.vocab_bwd_inputs(T, v, h, seed=37)
    H, E = f["H"].cuda(), f["E"].cuda()
    L = tpl.tp_logits_fwd(H, E, N)
    x = tpl.vp_xent_bf16_grad(L, f["targets"].cuda(), N, grad_scale=1.0 / T)
    dH, dE = tpl.tp_logits_bwd(x["dlogits"], H, E, N)
    tpl.vp_embed_bwd(f["ids"].cuda(), b["dout"].cuda(), dE, N)
    torch.cuda.synchronize()
    oL = O.logits(f["H"], f["E"])
    oG = O.xent(oL, f["targets"], 1.0 / T)["dlogits"]
    og = O.logits_bwd(oG, f["H"], f["E"])
    total = O.tied_embedding_grad(og["dE"], O.embed_bwd(f["ids"], b["dout"], v))
    assert_close("dH", dH, og["dH"], TOL_BF16)
    assert_close("tied dE", dE, total, TOL_BF16)
