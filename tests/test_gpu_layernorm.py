"""Sequence-parallel dropout-add-LayerNorm on the GPU against the fp64 oracle
(through the C ABI).

The dropout mask is an integer decision taken on both sides from the same
Philox4x32-10 words: compared bit for bit.  p is a power of two so that the
threshold floor(p·2^32) is the same in the float the kernel receives and the
double the oracle uses.  hs and y are stored in bf16 (TOL_BF16).  The
kernel takes the statistics from hs as stored, so every quantity built from
xhat carries the bf16 rounding of hs (relative 2^-9 per element, 1.1e-3
rms): rstd within 1e-3; the row mean, a quantity near zero, within 1e-2 of
its own size; the fp32 parameter gradients within 5e-3; the backward's bf16
outputs within TOL_BF16.
"""
import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, assert_close, f64

pytestmark = pytest.mark.gpu

TOL_STAT = 1e-3
TOL_MEAN = 1e-2
TOL_PGRAD = 5e-3


def _inputs(M, h, seed, with_bias=True):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *s, std=1.0: (std * torch.randn(*s, generator=g)).bfloat16()
    return dict(x=bf(M, h), res=bf(M, h), bias=bf(h, std=0.1) if with_bias else None,
                gamma=(1 + 0.2 * torch.randn(h, generator=g)).bfloat16(), beta=bf(h, std=0.1),
                dy=bf(M, h), dhs=bf(M, h, std=0.5))


def _run(d, M, h, N, p, seed, offset, use_dhs):
    dev = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    st = tpl.new_status()
    f = tpl.tp_sp_dropout_add_ln_fwd(dev["x"], dev["bias"], dev["res"], dev["gamma"], dev["beta"],
                                     N, p=p, seed=seed, offset=offset, with_keep=True,
                                     dev_status=st)
    b = tpl.tp_sp_dropout_add_ln_bwd(dev["dy"], dev["dhs"] if use_dhs else None, f["hs"],
                                     dev["gamma"], f["mean"], f["rstd"], N, p=p, seed=seed,
                                     offset=offset, with_dbias=d["bias"] is not None,
                                     dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return f, b


@pytest.mark.parametrize("M,h,N,p,use_dhs,with_bias", [
    (300, 1600, 4, 0.125, True, True),     # the GPT-2 slice width, ragged chunk count per thread
    (64, 4096, 8, 0.25, False, True),
    (8, 8, 1, 0.5, True, False),           # one chunk per row
    (130, 1000, 2, 0.0, True, True),       # no dropout
    (40, 8192, 4, 0.125, True, True),      # the widest supported row
])
def test_layernorm_against_oracle(M, h, N, p, use_dhs, with_bias):
    d = _inputs(M, h, seed=M + h, with_bias=with_bias)
    seed, offset = 0x1234ABCD5678, 77
    f, b = _run(d, M, h, N, p, seed, offset, use_dhs)
    ref = O.dropout_add_layernorm(d["x"], d["bias"], d["res"], d["gamma"], d["beta"], p, seed, offset)
    assert np.array_equal(f["keep"].cpu().numpy().astype(bool), ref["keep"])
    assert_close("hs", f["hs"], ref["hs"], TOL_BF16)
    assert_close("y", f["y"], ref["y"], TOL_BF16)
    assert_close("mean", f["mean"], ref["mean"], TOL_MEAN)
    # per element twice TOL_STAT: a row of 8 values (the smallest case) has
    # the statistics of 8 bf16-rounded hs values
    assert_close("rstd", f["rstd"], ref["rstd"], TOL_STAT, elem_tol=2 * TOL_STAT)
    rb = O.dropout_add_layernorm_bwd_sharded(d["dy"], d["dhs"] if use_dhs else None, ref["hs"],
                                             d["gamma"], ref["mean"], ref["rstd"], ref["keep"], p, N)
    assert_close("dx", b["dx"], rb["dx"], TOL_BF16)
    assert_close("dresidual", b["dresidual"], rb["dresidual"], TOL_BF16)
    assert_close("dgamma", b["dgamma"], rb["dgamma"], TOL_PGRAD, elem_tol=TOL_BF16)
    assert_close("dbeta", b["dbeta"], rb["dbeta"], TOL_PGRAD, elem_tol=TOL_BF16)
    if with_bias:
        assert_close("dbias", b["dbias"], rb["dbias"], TOL_PGRAD, elem_tol=TOL_BF16)


def test_dropout_mask_depends_only_on_seed_and_offset():
    M, h = 64, 1024
    d = _inputs(M, h, seed=3)
    f1, _ = _run(d, M, h, 2, 0.25, seed=5, offset=9, use_dhs=False)
    f2, _ = _run(d, M, h, 2, 0.25, seed=5, offset=9, use_dhs=False)
    f3, _ = _run(d, M, h, 2, 0.25, seed=5, offset=10, use_dhs=False)
    assert torch.equal(f1["keep"], f2["keep"]) and torch.equal(f1["hs"], f2["hs"])
    assert not torch.equal(f1["keep"], f3["keep"])
    frac = f1["keep"].float().mean().item()
    assert abs(frac - 0.75) < 5 * (0.25 * 0.75 / (M * h)) ** 0.5


@pytest.mark.slow
def test_layernorm_gpt2_slice_full():
    """M = 4096 tokens of width 1600 over 4 sequence shards, p = 0.125: every
    element against the oracle."""
    M, h, N, p = 4096, 1600, 4, 0.125
    d = _inputs(M, h, seed=11)
    f, b = _run(d, M, h, N, p, 2024, 0, True)
    ref = O.dropout_add_layernorm(d["x"], d["bias"], d["res"], d["gamma"], d["beta"], p, 2024, 0)
    assert np.array_equal(f["keep"].cpu().numpy().astype(bool), ref["keep"])
    assert_close("y", f["y"], ref["y"], TOL_BF16)
    rb = O.dropout_add_layernorm_bwd(d["dy"], d["dhs"], ref["hs"], d["gamma"], ref["mean"],
                                     ref["rstd"], ref["keep"], p)
    assert_close("dx", b["dx"], rb["dx"], TOL_BF16)
    assert_close("dgamma", b["dgamma"], rb["dgamma"], TOL_PGRAD, elem_tol=TOL_BF16)


def test_layernorm_deterministic():
    M, h = 200, 1600
    d = _inputs(M, h, seed=4)
    _, b1 = _run(d, M, h, 4, 0.125, 1, 2, True)
    _, b2 = _run(d, M, h, 4, 0.125, 1, 2, True)
    for k in ("dx", "dresidual", "dgamma", "dbeta", "dbias"):
        assert torch.equal(b1[k], b2[k]), k


@pytest.mark.parametrize("M,h", [
    (16384, 1600),   # more rows per CTA than row slots: every slot refilled
    (1000, 2048),    # the widest row the staged forward takes
    (5, 24),         # fewer rows than CTAs, three chunks per row
])
def test_layernorm_forward_staged_shapes(M, h):
    """The staged forward (rows bulk-copied into shared-memory slots) at the
    shapes that take its other paths."""
    d = _inputs(M, h, seed=M + 7 * h)
    seed, offset, p = 99, 5, 0.125
    f, b = _run(d, M, h, 1, p, seed, offset, True)
    ref = O.dropout_add_layernorm(d["x"], d["bias"], d["res"], d["gamma"], d["beta"], p, seed, offset)
    assert np.array_equal(f["keep"].cpu().numpy().astype(bool), ref["keep"])
    assert_close("hs", f["hs"], ref["hs"], TOL_BF16)
    assert_close("y", f["y"], ref["y"], TOL_BF16)
    assert_close("rstd", f["rstd"], ref["rstd"], TOL_STAT, elem_tol=2 * TOL_STAT)


def test_layernorm_forward_warp_path(monkeypatch):
    """The register-only warp-per-row forward (TP_LN_FWD_WARP=1), the path
    the staged one replaced, kept for sweeps: same results."""
    monkeypatch.setenv("TP_LN_FWD_WARP", "1")
    M, h, p, seed, offset = 300, 1600, 0.125, 7, 3
    d = _inputs(M, h, seed=21)
    f, _ = _run(d, M, h, 4, p, seed, offset, False)
    ref = O.dropout_add_layernorm(d["x"], d["bias"], d["res"], d["gamma"], d["beta"], p, seed, offset)
    assert np.array_equal(f["keep"].cpu().numpy().astype(bool), ref["keep"])
    assert_close("hs", f["hs"], ref["hs"], TOL_BF16)
    assert_close("y", f["y"], ref["y"], TOL_BF16)
