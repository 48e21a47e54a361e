"""Attention core between the projections (per-shard heads) on the GPU
against the fp64 oracle (through the C ABI).

The scores are fp32 accumulations of bf16 Q·Kᵀ; P is rounded to bf16 for the
P·V product and the context is stored in bf16, so the context is compared
with TOL_BF16 (relative Frobenius per head and sequence) and the
log-sum-exp per query with TOL_XENT.
"""
import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, TOL_XENT, assert_close, f64, guarded

pytestmark = pytest.mark.gpu

HD = 64


def _qkv(b, s, nh, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (std * torch.randn(b * s, 3 * nh * HD, generator=g)).bfloat16()


def _offsets(nh, N):
    heads = tp_inputs.head_split(nh, N)
    return [0] + list(np.cumsum(heads))


def _check(QKV, b, s, nh, N, causal, offs=None, scale=None):
    st = tpl.new_status()
    ctx, gctx = guarded((b * s, nh * HD), torch.bfloat16)
    lse, glse = guarded((b, nh, s), torch.float32)
    tpl.tp_attention_fwd(QKV.cuda(), b, s, nh, N, head_offsets=offs, causal=causal, scale=scale,
                         ctx=ctx, lse=lse, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gctx.check("ctx")
    glse.check("lse")
    shards = np.diff(offs if offs is not None else _offsets(nh, N)).tolist()
    rctx, rlse = O.attention_sharded(QKV, b, s, nh, HD, shards, causal=causal, scale=scale)
    g = f64(ctx)
    for bb in range(b):
        for hh in range(nh):
            rows, cols = slice(bb * s, (bb + 1) * s), slice(hh * HD, (hh + 1) * HD)
            assert_close(f"ctx[b={bb},h={hh}]", g[rows, cols], rctx[rows, cols], TOL_BF16)
    gl = f64(lse)
    assert (np.abs(gl - rlse) / np.maximum(np.abs(rlse), 1.0)).max() <= TOL_XENT
    return ctx


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("b,s,nh,N", [(2, 200, 5, 3),     # ragged second query tile
                                      (1, 128, 2, 2),     # one full tile
                                      (3, 37, 4, 1),      # shorter than one tile
                                      (1, 1, 1, 1),       # a single token
                                      (2, 384, 3, 3)])    # three tiles, causal diagonal blocks
def test_attention_small(b, s, nh, N, causal):
    _check(_qkv(b, s, nh, seed=s + nh), b, s, nh, N, causal)


def test_attention_explicit_offsets_and_scale():
    b, s, nh = 2, 260, 6
    _check(_qkv(b, s, nh, seed=7), b, s, nh, 3, True, offs=[0, 1, 4, 6], scale=0.05)


def test_attention_large_scores():
    """Scores of size ~±60 after scaling: the running maximum and the
    rescaling of O keep the softmax exact in fp32."""
    b, s, nh = 1, 512, 2
    _check(_qkv(b, s, nh, seed=8, std=3.0), b, s, nh, 2, True)


@pytest.mark.slow
def test_attention_gpt2_slice():
    """b=4, s=1024, 25 heads of 64 over 4 shards (7, 6, 6, 6): every head of
    two sequences against the oracle; the other two by their log-sum-exp."""
    w = tp_inputs.WORKLOADS["gpt2_1p5b_slice"]
    b, s, nh, N = 4, 1024, w["n_heads"], w["N"]
    QKV = _qkv(b, s, nh, seed=9)
    st = tpl.new_status()
    ctx, lse = tpl.tp_attention_fwd(QKV.cuda(), b, s, nh, N, with_lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    shards = tp_inputs.head_split(nh, N)
    for bb in (0, 3):
        rows = slice(bb * s, (bb + 1) * s)
        rctx, rlse = O.attention_sharded(QKV[rows], 1, s, nh, HD, shards, causal=True)
        assert_close(f"ctx[b={bb}]", ctx[rows], rctx, TOL_BF16)
        assert (np.abs(f64(lse[bb]) - rlse[0]) / np.maximum(np.abs(rlse[0]), 1.0)).max() <= TOL_XENT


def test_attention_layer_chain():
    """X -> column-parallel QKV (per-shard heads) -> attention core ->
    row-parallel output projection with its shard sum, against the oracle's
    chain of the same three steps."""
    b, s, nh, N, h = 2, 192, 5, 2, 5 * HD
    inp = tp_inputs.attn_proj_inputs(b * s, h, nh, HD, N, seed=10, w_std=0.05)
    shards = tp_inputs.head_split(nh, N)
    qkv_offs = [0] + list(np.cumsum([3 * k * HD for k in shards]))
    ctx_offs = [0] + list(np.cumsum([k * HD for k in shards]))
    X, Wqkv, Wo = (inp[k].cuda() for k in ("X", "Wqkv", "Wo"))
    QKV, _ = tpl.tp_col_linear_fwd(X, Wqkv, None, N, shard_offsets=qkv_offs)
    ctx, _ = tpl.tp_attention_fwd(QKV, b, s, nh, N)
    Z = tpl.tp_row_linear_fwd(ctx, Wo, N, shard_offsets=ctx_offs)
    torch.cuda.synchronize()
    _, rQKV = O.col_linear_fwd(inp["X"], inp["Wqkv"])
    rctx, _ = O.attention_sharded(rQKV, b, s, nh, HD, shards, causal=True)
    rZ, _ = O.row_linear_fwd(rctx, inp["Wo"], offsets=ctx_offs)
    assert_close("QKV", QKV, rQKV, TOL_BF16)
    # ctx and Z are taken from the bf16-rounded QKV (the oracle's stays
    # fp64) and the softmax amplifies that rounding: twice the bound per element
    assert_close("ctx", ctx, rctx, TOL_BF16, elem_tol=2 * TOL_BF16)
    assert_close("Z", Z, rZ, TOL_BF16, elem_tol=2 * TOL_BF16)


def test_attention_deterministic():
    b, s, nh = 2, 300, 4
    QKV = _qkv(b, s, nh, seed=11).cuda()
    a, _ = tpl.tp_attention_fwd(QKV, b, s, nh, 2)
    c, _ = tpl.tp_attention_fwd(QKV, b, s, nh, 2)
    torch.cuda.synchronize()
    assert torch.equal(a, c)


# ---------------------------------------------------------------- backward
def _bwd_elem_tol(causal):
    """Per-element bound of the backward's gradients.  P and dS enter their
    products rounded to bf16; under the causal mask the first rows of a
    sequence sum over a handful of keys, so that rounding does not average
    out there.  Emulating exactly those rounding points in float64 (one
    head, s=1024, three seeds) gives relative Frobenius errors of 2.5e-3 and
    worst elements of up to 6.8e-2 causal, 1.7e-2 not causal: the causal
    bound is 0.1, still far below the ~1 of an element that is wrong."""
    return 5 * TOL_BF16 if causal else TOL_BF16


def _bwd_check(b, s, nh, N, causal, seed, offs=None, scale=None):
    QKV = _qkv(b, s, nh, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    dctx = torch.randn(b * s, nh * HD, generator=g).bfloat16()
    st = tpl.new_status()
    ctx, lse = tpl.tp_attention_fwd(QKV.cuda(), b, s, nh, N, head_offsets=offs, causal=causal,
                                    scale=scale, with_lse=True, dev_status=st)
    dQKV, gd = guarded((b * s, 3 * nh * HD), torch.bfloat16)
    tpl.tp_attention_bwd(QKV.cuda(), ctx, dctx.cuda(), lse, b, s, nh, N, head_offsets=offs,
                         causal=causal, scale=scale, dQKV=dQKV, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gd.check("dQKV")
    shards = np.diff(offs if offs is not None else _offsets(nh, N)).tolist()
    ref = O.attention_sharded_bwd(QKV, dctx, b, s, nh, HD, shards, causal=causal, scale=scale)
    got = f64(dQKV)
    for bb in range(b):
        rows = slice(bb * s, (bb + 1) * s)
        for c0 in range(0, 3 * nh * HD, HD):     # every head's Q, K and V block
            cols = slice(c0, c0 + HD)
            assert_close(f"dQKV[b={bb},cols={c0}]", got[rows, cols], ref[rows, cols], TOL_BF16,
                         elem_tol=_bwd_elem_tol(causal))
    return dQKV


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("b,s,nh,N", [(2, 200, 5, 3), (1, 128, 2, 2), (3, 37, 4, 1), (1, 1, 1, 1),
                                      (2, 384, 3, 3)])
def test_attention_backward_small(b, s, nh, N, causal):
    _bwd_check(b, s, nh, N, causal, seed=100 + s + nh)


def test_attention_backward_offsets_and_scale():
    _bwd_check(2, 260, 6, 3, True, seed=12, offs=[0, 1, 4, 6], scale=0.05)


def test_attention_backward_reproducible():
    """dK and dV come from one CTA per key row: bit for bit the same on a
    second run.  dQ sums the key tiles' fp32 contributions in arrival order,
    so a second run may differ by the rounding of that sum: at most one bf16
    step of the element (or of the tensor's scale near zero)."""
    nh = 4
    a = _bwd_check(2, 300, nh, 2, True, seed=13)
    c = _bwd_check(2, 300, nh, 2, True, seed=13)
    q_cols = torch.zeros(3 * nh * HD, dtype=torch.bool)
    for first, cnt in ((0, 2), (2, 2)):          # shard-major: [Q heads | K heads | V heads]
        q_cols[3 * HD * first:3 * HD * first + cnt * HD] = True
    assert torch.equal(a[:, ~q_cols], c[:, ~q_cols])
    qa, qc = a[:, q_cols].float(), c[:, q_cols].float()
    step = torch.maximum(qa.abs(), qc.abs()) * 2.0 ** -7 + qa.abs().max() * 2.0 ** -16
    assert bool(((qa - qc).abs() <= step).all())


@pytest.mark.slow
def test_attention_backward_gpt2_slice():
    """b=4, s=1024, 25 heads over 4 shards: every head of the first sequence
    against the oracle."""
    b, s, nh, N = 4, 1024, 25, 4
    QKV = _qkv(b, s, nh, seed=14)
    g = torch.Generator().manual_seed(15)
    dctx = torch.randn(b * s, nh * HD, generator=g).bfloat16()
    st = tpl.new_status()
    ctx, lse = tpl.tp_attention_fwd(QKV.cuda(), b, s, nh, N, with_lse=True, dev_status=st)
    dQKV = tpl.tp_attention_bwd(QKV.cuda(), ctx, dctx.cuda(), lse, b, s, nh, N, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    shards = tp_inputs.head_split(nh, N)
    ref = O.attention_sharded_bwd(QKV[:s], dctx[:s], 1, s, nh, HD, shards, causal=True)
    assert_close("dQKV[b=0]", dQKV[:s], ref, TOL_BF16, elem_tol=_bwd_elem_tol(True))
