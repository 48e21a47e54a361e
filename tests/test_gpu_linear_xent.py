"""Output layer and cross-entropy without the logits matrix, on the GPU
against the fp64 oracle (through the C ABI).

The loss statistics come from the GEMM's fp32 accumulators of bf16 H and E;
the oracle computes the same logits in fp64 from the same bf16 values.  The
loss and log-sum-exp are compared per token (relative, TOL_XENT); the bf16
gradient with TOL_BF16.  The arg-max is decided in fp32 on the GPU and in
fp64 in the oracle, so it is compared where it is unique at fp32 accuracy
(top-two gap above ARGMAX_EPS) and checked to be a maximum within ARGMAX_EPS
elsewhere.
"""
import math

import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, TOL_XENT, assert_close, f64

pytestmark = pytest.mark.gpu

# fp32 accumulation of h products of size ~|H||E| = O(0.02): error well below this
ARGMAX_EPS = 1e-4


def _check_argmax(got, L64):
    got = np.asarray(got, dtype=np.int64)
    rows = np.arange(L64.shape[0])
    top = L64.max(axis=1)
    assert np.all(L64[rows, got] >= top - ARGMAX_EPS)
    part = np.partition(L64, -2, axis=1)
    unique = part[:, -1] - part[:, -2] > 2 * ARGMAX_EPS
    assert np.array_equal(got[unique], np.argmax(L64, axis=1)[unique])
    return int(unique.sum())


def _check_fwd(r, ref, rows=None):
    sel = slice(None) if rows is None else rows
    loss = f64(r["loss"])[sel]
    ok = np.isfinite(ref["loss"])
    rel = np.abs(loss[ok] - ref["loss"][ok]) / np.maximum(np.abs(ref["loss"][ok]), 1e-30)
    assert rel.max() <= TOL_XENT, rel.max()
    assert np.all(np.isnan(loss[~ok]))
    lse = f64(r["lse"])[sel]
    assert (np.abs(lse - ref["lse"]) / np.abs(ref["lse"])).max() <= TOL_XENT


@pytest.mark.parametrize("T,v,h,N", [(300, 1000, 256, 4),    # ragged rows, partial last slice
                                     (16, 2048, 64, 8),      # one 128-row tile
                                     (200, 136, 512, 2),     # two slices, one mostly empty
                                     (513, 4096, 328, 1)])   # K not a multiple of 64, one row past 512
def test_linear_xent_small(T, v, h, N):
    inp = tp_inputs.vocab_inputs(T, v, h, e_std=1.0 / math.sqrt(h) * 1.28, seed=11)
    H, E, y = inp["H"], inp["E"], inp["targets"]
    st = tpl.new_status()
    r = tpl.tp_linear_xent_fwd(H.cuda(), E.cuda(), y.cuda(), N, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = O.linear_xent(H, E, y, grad_scale=1.0 / T)
    _check_fwd(r, ref)
    assert abs(float(r["loss_sum"].item()) - ref["loss_sum"]) <= TOL_XENT * abs(ref["loss_sum"])
    _check_argmax(r["argmax"].cpu().numpy(), O.logits(H, E))
    d = tpl.tp_linear_xent_dlogits(H.cuda(), E.cuda(), y.cuda(), r["lse"], N, grad_scale=1.0 / T,
                                   dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close("dlogits", d, ref["dlogits"], TOL_BF16)
    # partitioned form of the pages' combine gives the same loss
    part = O.linear_xent_partitioned(H, E, y, list(range(0, v, 128)) + [v])
    _check_fwd(r, part)


def test_linear_xent_matches_unfused_path():
    """Same fp32 accumulators as the logits GEMM: the arg-max is identical and
    the loss agrees with vp_xent on the stored logits to fp32 rounding."""
    T, v, h, N = 1024, 8192, 1024, 8
    inp = tp_inputs.vocab_inputs(T, v, h, e_std=0.04, seed=12)
    H, E, y = inp["H"].cuda(), inp["E"].cuda(), inp["targets"].cuda()
    r = tpl.tp_linear_xent_fwd(H, E, y, N)
    L = tpl.tp_logits_fwd(H, E, N)
    u = tpl.vp_xent(L, y, N, with_grad=False)
    torch.cuda.synchronize()
    assert torch.equal(r["argmax"], u["argmax"])
    assert torch.allclose(r["loss"], u["loss"], rtol=1e-5, atol=1e-5)


def test_linear_xent_bad_targets_and_ties():
    v, h, N = 256, 64, 2
    E = torch.zeros(v, h)
    E[3, 0] = E[200, 0] = 1.0           # equal rows 3 and 200: tie across the slice cut
    E[17, 1] = E[18, 1] = 1.0           # tie inside a slice
    H = torch.zeros(5, h)
    H[0, 0] = 4.0
    H[1, 1] = 2.0
    H[2, 2] = 0.5                       # all logits 0: uniform row, arg-max 0
    H[3, 0] = 1.0
    H[4, 1] = 1.0
    y = torch.tensor([3, 0, 10, -1, v], dtype=torch.int64)
    Hb, Eb = H.bfloat16(), E.bfloat16()
    st = tpl.new_status()
    r = tpl.tp_linear_xent_fwd(Hb.cuda(), Eb.cuda(), y.cuda(), N, dev_status=st)
    d = tpl.tp_linear_xent_dlogits(Hb.cuda(), Eb.cuda(), y.cuda(), r["lse"], N, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tpl.DEVERR_RANGE
    ref = O.linear_xent(Hb, Eb, y)
    _check_fwd(r, ref)
    assert r["argmax"].cpu().tolist() == [3, 17, 0, 3, 17]
    assert abs(float(r["loss"][2]) - math.log(v)) < 1e-5
    dd = f64(d)
    assert np.all(np.isnan(dd[3:])) and np.all(np.isfinite(dd[:3]))
    assert_close("dlogits", dd[:3], ref["dlogits"][:3], TOL_BF16)


def test_linear_xent_backward_chain():
    """dlogits recomputed by the GEMM, then the output-layer backward:
    dH and dE against the oracle's chain on the same inputs."""
    T, v, h, N = 384, 2048, 256, 4
    inp = tp_inputs.vocab_inputs(T, v, h, e_std=0.08, seed=13)
    H, E, y = inp["H"], inp["E"], inp["targets"]
    Hd, Ed, yd = H.cuda(), E.cuda(), y.cuda()
    r = tpl.tp_linear_xent_fwd(Hd, Ed, yd, N)
    d = tpl.tp_linear_xent_dlogits(Hd, Ed, yd, r["lse"], N, grad_scale=1.0 / T)
    dH, dE = tpl.tp_logits_bwd(d, Hd, Ed, N)
    torch.cuda.synchronize()
    ref = O.linear_xent(H, E, y, grad_scale=1.0 / T)
    g = O.logits_bwd(ref["dlogits"], H, E)
    # dH and dE contract the bf16-rounded dlogits (the oracle's stay fp64):
    # per tensor the stated 2e-2, per element twice that for the rounding
    # the chain adds before the contraction
    assert_close("dH", dH, g["dH"], TOL_BF16, elem_tol=2 * TOL_BF16)
    assert_close("dE", dE, g["dE"], TOL_BF16, elem_tol=2 * TOL_BF16)


@pytest.mark.slow
def test_linear_xent_full_size_sampled_rows():
    """T=16384 tokens, v=50304 over 8 shards, h=4096 in the launch shape the
    benchmark times; the oracle recomputes 48 sampled rows in fp64."""
    w = tp_inputs.WORKLOADS["vocab_v50304"]
    inp = tp_inputs.vocab_inputs(w["T"], w["v"], w["h"], e_std=w["e_std"], seed=0)
    H, E, y = inp["H"], inp["E"], inp["targets"]
    Hd, Ed, yd = H.cuda(), E.cuda(), y.cuda()
    st = tpl.new_status()
    r = tpl.tp_linear_xent_fwd(Hd, Ed, yd, w["N"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.arange(5, w["T"], w["T"] // 48)[:48]
    rows[-1] = w["T"] - 1
    ref = O.linear_xent(H[rows], E, y[rows], grad_scale=1.0 / w["T"])
    _check_fwd(r, ref, rows)
    _check_argmax(r["argmax"].cpu().numpy()[rows], O.logits(H[rows], E))
    # the fixed-order sum equals the sum of the per-token losses it reduces
    tot = float(r["loss"].double().sum().item())
    assert abs(float(r["loss_sum"].item()) - tot) <= 1e-5 * abs(tot)
    d = tpl.tp_linear_xent_dlogits(Hd, Ed, yd, r["lse"], w["N"], grad_scale=1.0 / w["T"])
    torch.cuda.synchronize()
    rsel = torch.as_tensor(rows).cuda()
    assert_close("dlogits[rows]", d[rsel], ref["dlogits"], TOL_BF16)
    del d
