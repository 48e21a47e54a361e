"""TP-MLP forward/backward on the GPU against the fp64 oracle (through the C ABI).

Sizes the oracle finishes in seconds span several 128x256 tiles with ragged
edges; the full-size shapes (h=1024, the GPT-2 1.5B slice, h=4096) are
checked on sampled rows (row-local outputs) and sampled ffn columns
(column-local outputs), which the oracle computes exactly from the same
inputs.
"""
import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, TOL_F32, assert_close, f64, guarded, to_dev

pytestmark = pytest.mark.gpu


def _run(inp, N, act, offsets=None, zpart=False):
    """Forward + backward with every output inside a guard band (NaN-filled,
    sentinel margins before and after) so that a missed store fails the
    parity check and a store past either end fails the guard check."""
    d = to_dev(inp)
    M, h = d["X"].shape
    F = d["A"].shape[1]
    dt = d["X"].dtype
    shapes = {"U": ((M, F), dt), "Y": ((M, F), dt), "Z": ((M, h), dt), "dU": ((M, F), dt),
              "dX": ((M, h), dt), "dA": ((h, F), dt), "dB": ((F, h), dt),
              "dbias": ((F,), torch.float32)}
    if zpart:
        shapes["Zpart"] = ((N, M, h), torch.float32)
    out, guards = {}, {}
    for k, (shape, t) in shapes.items():
        out[k], guards[k] = guarded(shape, t)
    st = tpl.new_status()
    Z, U, Y = tpl.tp_mlp_fwd(d["X"], d["A"], d["bias"], d["B"], N, shard_offsets=offsets,
                             act=act, U=out["U"], Y=out["Y"], Z=out["Z"], Zpart=out.get("Zpart"),
                             dev_status=st)
    g = tpl.tp_mlp_bwd(d["X"], d["A"], d["B"], U, Y, d["dZ"], N, shard_offsets=offsets, act=act,
                       dU=out["dU"], dX=out["dX"], dA=out["dA"], dbias=out["dbias"], dB=out["dB"],
                       dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for k, gd in guards.items():
        gd.check(k)
    return Z, U, Y, g, out.get("Zpart")


def _check_full(inp, N, act, tol, offsets=None, zpart=False):
    Z, U, Y, g, Zpart = _run(inp, N, act, offsets, zpart)
    oU, oY, oZ = O.mlp_fwd(inp["X"], inp["A"], inp["bias"], inp["B"], act)
    ob = O.mlp_bwd(inp["X"], inp["A"], inp["bias"], inp["B"], inp["dZ"], act)
    assert_close("U", U, oU, tol)
    assert_close("Y", Y, oY, tol)
    assert_close("Z", Z, oZ, tol)
    for k in ("dX", "dA", "dB", "dbias", "dU"):
        assert_close(k, g[k], ob[k], tol)
    if zpart:
        s = O.mlp_fwd_sharded(inp["X"], inp["A"], inp["bias"], inp["B"], N, offsets, act)
        for i in range(N):
            assert_close(f"Zpart[{i}]", Zpart[i], s["Zparts"][i], tol)
    return Z, U, Y, g


@pytest.mark.parametrize("act", [tpl.ACT_GELU_TANH, tpl.ACT_GELU_ERF, tpl.ACT_NONE])
def test_mlp_ragged_tiles(act):
    # M=200 (one full and one ragged 128-row tile), h=264 (ragged k-block and
    # a ragged 256-column tile of Z), F=1024 over N=4 shards, non-zero bias
    inp = tp_inputs.mlp_inputs(200, 264, 1024, w_std=0.05, bias_std=0.02, seed=1)
    _check_full(inp, 4, act, TOL_BF16)


def test_mlp_shard_partials_and_uneven_shards():
    inp = tp_inputs.mlp_inputs(130, 128, 768, w_std=0.05, bias_std=0.02, seed=2)
    _check_full(inp, 3, tpl.ACT_GELU_TANH, TOL_BF16, offsets=[0, 128, 448, 768], zpart=True)
    _check_full(inp, 4, tpl.ACT_GELU_TANH, TOL_BF16, zpart=True)
    # one shard: Zpart[0] is the whole product in fp32 (the per-rank partial
    # a multi-GPU layer all-reduces)
    _check_full(inp, 1, tpl.ACT_GELU_TANH, TOL_BF16, zpart=True)


def test_mlp_degenerate_sizes():
    # one token row, one shard, K = 8 (a single zero-padded k-block)
    inp = tp_inputs.mlp_inputs(1, 8, 16, w_std=0.3, bias_std=0.1, seed=3)
    _check_full(inp, 1, tpl.ACT_GELU_TANH, TOL_BF16)
    inp = tp_inputs.mlp_inputs(3, 16, 64, w_std=0.3, bias_std=0.1, seed=4)
    _check_full(inp, 8, tpl.ACT_GELU_TANH, TOL_BF16)


def test_mlp_tiny_fp32_path():
    w = tp_inputs.WORKLOADS["mlp_tiny_fp32"]
    inp = tp_inputs.mlp_inputs(w["M"], w["h"], w["F"], dtype=torch.float32, w_std=w["w_std"],
                               x_std=w["x_std"], bias_std=0.0, seed=0)
    _check_full(inp, w["N"], tpl.ACT_GELU_TANH, TOL_F32, zpart=True)
    inp = tp_inputs.mlp_inputs(w["M"], w["h"], w["F"], dtype=torch.float32, w_std=0.5,
                               bias_std=0.1, seed=5)
    _check_full(inp, w["N"], tpl.ACT_GELU_ERF, TOL_F32)


def test_mlp_h1024_full():
    w = tp_inputs.WORKLOADS["mlp_h1024"]
    inp = tp_inputs.mlp_inputs(w["M"], w["h"], w["F"], w_std=w["w_std"], seed=0)
    _check_full(inp, w["N"], tpl.ACT_GELU_TANH, TOL_BF16)


def _check_sampled(inp, N, act, rows, cols, offsets=None):
    """Row-local outputs on sampled rows, column-local outputs on sampled ffn columns."""
    Z, U, Y, g, _ = _run(inp, N, act, offsets)
    X, A, b, B, dZ = (inp[k] for k in ("X", "A", "bias", "B", "dZ"))
    r = torch.as_tensor(rows)
    c = torch.as_tensor(cols)
    oU, oY, oZ = O.mlp_fwd(X[r], A, b, B, act)
    assert_close("Z[rows]", Z[r.cuda()], oZ, TOL_BF16)
    assert_close("U[rows]", U[r.cuda()], oU, TOL_BF16)
    assert_close("Y[rows]", Y[r.cuda()], oY, TOL_BF16)
    ob_rows = O.mlp_bwd(X[r], A, b, B, dZ[r], act)
    assert_close("dX[rows]", g["dX"][r.cuda()], ob_rows["dX"], TOL_BF16)
    assert_close("dU[rows]", g["dU"][r.cuda()], ob_rows["dU"], TOL_BF16)
    # every output that is local to an ffn column: restrict A's columns and B's rows
    ob_cols = O.mlp_bwd(X, A[:, c], b[c], B[c], dZ, act)
    cc = c.cuda()
    assert_close("dA[:,cols]", g["dA"][:, cc], ob_cols["dA"], TOL_BF16)
    assert_close("dB[cols]", g["dB"][cc], ob_cols["dB"], TOL_BF16)
    assert_close("dbias[cols]", g["dbias"][cc], ob_cols["dbias"], TOL_BF16)
    assert_close("dU[:,cols]", g["dU"][:, cc], ob_cols["dU"], TOL_BF16)


def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    head = np.arange(min(128, n))
    rest = rng.choice(np.arange(128, n), size=min(k, n - 128), replace=False) if n > 128 else []
    return np.sort(np.concatenate([head, rest]).astype(np.int64))


@pytest.mark.slow
def test_mlp_gpt2_slice_sampled():
    w = tp_inputs.WORKLOADS["gpt2_1p5b_slice"]
    inp = tp_inputs.mlp_inputs(w["M"], w["h"], w["F"], w_std=w["w_std"], seed=0)
    _check_sampled(inp, w["N"], tpl.ACT_GELU_TANH, _sample(w["M"], 128, 1), _sample(w["F"], 128, 2))


@pytest.mark.slow
def test_mlp_h4096_sampled():
    w = tp_inputs.WORKLOADS["mlp_h4096"]
    inp = tp_inputs.mlp_inputs(w["M"], w["h"], w["F"], w_std=w["w_std"], seed=0)
    _check_sampled(inp, w["N"], tpl.ACT_GELU_TANH, _sample(w["M"], 128, 1), _sample(w["F"], 128, 2))


def test_mlp_deterministic():
    inp = tp_inputs.mlp_inputs(300, 512, 2048, w_std=0.02, bias_std=0.02, seed=6)
    a = _run(inp, 8, tpl.ACT_GELU_TANH, zpart=True)
    b = _run(inp, 8, tpl.ACT_GELU_TANH, zpart=True)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    for k in ("dX", "dA", "dB", "dbias", "dU"):
        assert torch.equal(a[3][k], b[3][k]), k
    assert torch.equal(a[4], b[4])


@pytest.mark.parametrize("tile", ["2x256", "2x256t", "2x128", "1x256", "1x128"])
def test_mlp_every_tile_shape(tile, monkeypatch):
    """Each tile shape of the GEMM engine (CTA pairs or single CTAs, 256- or
    128-column tiles), forced for every GEMM of the layer: ragged rows and
    columns, uneven shards with their partials, and the split shard sum."""
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    inp = tp_inputs.mlp_inputs(300, 264, 1024, w_std=0.05, bias_std=0.02, seed=21)
    _check_full(inp, 4, tpl.ACT_GELU_TANH, TOL_BF16, zpart=True)
    _check_full(inp, 3, tpl.ACT_GELU_TANH, TOL_BF16, offsets=[0, 128, 448, 1024])
    # long K over 8 shards: the split shard sum (two or more K ranges per tile)
    inp = tp_inputs.mlp_inputs(512, 256, 4096, w_std=0.02, bias_std=0.02, seed=22)
    _check_full(inp, 8, tpl.ACT_GELU_TANH, TOL_BF16)


@pytest.mark.parametrize("switch", ["TP_GEMM_NO_TMA_STORE", "TP_GEMM_SPLIT_ALL"])
def test_mlp_alternate_gemm_paths(switch, monkeypatch):
    """The two GEMM paths the defaults leave unused: outputs stored from
    registers instead of through staged tensor-map stores, and the shard sum
    split on every tile instead of on the tail that does not fill the
    persistent slots."""
    monkeypatch.setenv(switch, "1")
    inp = tp_inputs.mlp_inputs(300, 264, 1024, w_std=0.05, bias_std=0.02, seed=23)
    _check_full(inp, 4, tpl.ACT_GELU_TANH, TOL_BF16, zpart=True)
    _check_full(inp, 3, tpl.ACT_GELU_ERF, TOL_BF16, offsets=[0, 128, 448, 1024])
    inp = tp_inputs.mlp_inputs(512, 256, 4096, w_std=0.02, bias_std=0.02, seed=24)
    _check_full(inp, 8, tpl.ACT_GELU_TANH, TOL_BF16)
