"""Vocabulary-parallel embedding, logits and cross-entropy on the GPU against
the fp64 oracle (through the C ABI)."""
import math

import numpy as np
import pytest
import torch

import linear_layers_b200 as tpl
import tp_inputs
from oracle import tp_oracle as O
from tests.gpu_helpers import TOL_BF16, TOL_XENT, assert_close, f64, guarded

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- embedding
def test_embed_page_example_bit_exact():
    """300-word table over 2 GPUs, ids [0, 212, 7, 9]: every row exact."""
    E = tp_inputs.vocab_inputs(4, 300, 64, seed=1)["E"]
    ids = torch.tensor([0, 212, 7, 9], dtype=torch.int64)
    st = tpl.new_status()
    out = tpl.vp_embed(ids.cuda(), E.cuda(), 2, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(f64(out), O.vp_embed_sharded(ids, E, 2))
    assert np.array_equal(f64(out), O.embed_lookup(ids, E))


@pytest.mark.parametrize("h,N", [(8, 1), (64, 4), (1000, 8), (4096, 8)])
def test_embed_random_bit_exact(h, N):
    v = 4096 if h < 4096 else 50304
    inp = tp_inputs.vocab_inputs(3000, v, h, seed=2)
    out = tpl.vp_embed(inp["ids"].cuda(), inp["E"].cuda(), N)
    torch.cuda.synchronize()
    assert np.array_equal(f64(out), O.embed_lookup(inp["ids"], inp["E"]))


def test_embed_out_of_range_rows_are_zero_and_flagged():
    E = tp_inputs.vocab_inputs(4, 256, 32, seed=3)["E"]
    ids = torch.tensor([5, -1, 256, 255, 1 << 40], dtype=torch.int64)
    st = tpl.new_status()
    out = tpl.vp_embed(ids.cuda(), E.cuda(), 4, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tpl.DEVERR_RANGE
    assert np.array_equal(f64(out), O.vp_embed_sharded(ids, E, 4))


@pytest.mark.slow
def test_embed_full_size_bit_exact():
    w = tp_inputs.WORKLOADS["vocab_v50304"]
    inp = tp_inputs.vocab_inputs(w["T"], w["v"], w["h"], e_std=w["e_std"], seed=0)
    out = tpl.vp_embed(inp["ids"].cuda(), inp["E"].cuda(), w["N"])
    torch.cuda.synchronize()
    # bf16 copies compared bit for bit (as int16 words)
    ref = inp["E"][inp["ids"]]
    assert torch.equal(out.cpu().view(torch.int16), ref.view(torch.int16))
    rows = torch.arange(0, w["T"], 97)
    assert np.array_equal(f64(out[rows.cuda()]), O.embed_lookup(inp["ids"][rows], inp["E"]))


# ---------------------------------------------------------------- logits
def test_logits_ragged():
    inp = tp_inputs.vocab_inputs(300, 1000, 264, seed=4)
    L, gl = guarded((300, 1000), torch.float32)       # ragged row and column tiles
    tpl.tp_logits_fwd(inp["H"].cuda(), inp["E"].cuda(), 4, logits=L)
    gl.check("logits")
    assert_close("logits", L, O.logits(inp["H"], inp["E"]), TOL_BF16)
    blocks = O.logits_sharded(inp["H"], inp["E"], 4)
    for i, b in enumerate(blocks):
        assert_close(f"logits shard {i}", L[:, i * 250:(i + 1) * 250], b, TOL_BF16)


def test_logits_ragged_register_store(monkeypatch):
    """The fp32 logits stored from registers instead of through tensor-map
    stores (the path taken when the output is not 16-byte aligned)."""
    monkeypatch.setenv("TP_GEMM_NO_TMA_STORE", "1")
    inp = tp_inputs.vocab_inputs(300, 1000, 264, seed=5)
    L, gl = guarded((300, 1000), torch.float32)
    tpl.tp_logits_fwd(inp["H"].cuda(), inp["E"].cuda(), 4, logits=L)
    gl.check("logits")
    assert_close("logits", L, O.logits(inp["H"], inp["E"]), TOL_BF16)


def test_logits_column_bands_bit_identical(monkeypatch):
    """With 32 or more tile rows and B the larger operand the GEMM visits its
    tiles in bands of columns; the order of the tiles changes nothing in any
    tile's arithmetic, so the logits equal those of the row-band order bit
    for bit (and the oracle on sampled rows)."""
    inp = tp_inputs.vocab_inputs(8192, 20000, 128, seed=9)
    H, E = inp["H"].cuda(), inp["E"].cuda()
    L1 = tpl.tp_logits_fwd(H, E, 8)
    monkeypatch.setenv("TP_GEMM_NO_COLUMN_BANDS", "1")
    L2 = tpl.tp_logits_fwd(H, E, 8)
    torch.cuda.synchronize()
    assert torch.equal(L1, L2)
    rows = torch.as_tensor(np.r_[0:16, 4000:4016, 8176:8192])
    assert_close("logits[rows]", L1[rows.cuda()], O.logits(inp["H"][rows], inp["E"]), TOL_BF16)


@pytest.mark.slow
def test_logits_full_size_sampled_rows():
    w = tp_inputs.WORKLOADS["vocab_v50304"]
    inp = tp_inputs.vocab_inputs(w["T"], w["v"], w["h"], e_std=w["e_std"], seed=0)
    L = tpl.tp_logits_fwd(inp["H"].cuda(), inp["E"].cuda(), w["N"])
    torch.cuda.synchronize()
    rows = torch.as_tensor(np.r_[0:32, 8000:8032, w["T"] - 32:w["T"]])
    assert_close("logits[rows]", L[rows.cuda()], O.logits(inp["H"][rows], inp["E"]), TOL_BF16)


# ---------------------------------------------------------------- cross-entropy
def _xent_check(logits, targets, N, grad_scale, rows=None):
    st = tpl.new_status()
    dl, gdl = guarded(tuple(logits.shape), torch.float32)
    r = tpl.vp_xent(logits.cuda(), targets.cuda(), N, grad_scale=grad_scale, dlogits=dl,
                    dev_status=st)
    gdl.check("dlogits")
    sel = torch.arange(logits.shape[0]) if rows is None else torch.as_tensor(rows)
    ref = O.xent(logits[sel], targets[sel], grad_scale)
    dsel = sel.cuda()
    loss = f64(r["loss"][dsel])
    ok = np.isfinite(ref["loss"])
    rel = np.abs(loss[ok] - ref["loss"][ok]) / np.maximum(np.abs(ref["loss"][ok]), 1e-30)
    assert rel.max() <= TOL_XENT, rel.max()
    assert np.all(np.isnan(loss[~ok]))
    g = f64(r["dlogits"][dsel])
    assert_close("dlogits", g[ok], ref["dlogits"][ok], TOL_XENT)
    assert np.array_equal(r["argmax"][dsel].cpu().numpy().astype(np.int64), ref["argmax"])
    return r, st


@pytest.mark.parametrize("v,N", [(1024, 4), (48, 8), (50304, 8), (1002, 3), (4096, 1), (4000, 16),
                                 (32768, 2), (8192, 8)])
def test_xent_small(v, N):
    inp = tp_inputs.xent_logits(257, v, seed=5)
    r, st = _xent_check(inp["logits"], inp["targets"], N, 1.0 / 257)
    assert int(st.item()) == 0
    ref = O.xent(inp["logits"], inp["targets"])
    assert abs(float(r["loss_sum"].item()) - ref["loss_sum"]) <= TOL_XENT * abs(ref["loss_sum"])


def test_xent_alternating_slice_sizes():
    """Calls with a smaller shard slice between two with a larger one (the
    same kernel instance): every launch keeps enough shared memory."""
    for v, N in [(8192, 8), (1024, 4), (8192, 8), (1024, 4)]:
        inp = tp_inputs.xent_logits(64, v, seed=v + N)
        _xent_check(inp["logits"], inp["targets"], N, 1.0)


def test_xent_ties_uniform_and_bad_targets():
    v, N = 64, 4
    L = torch.zeros(5, v)
    L[0, [3, 40]] = 5.0        # tie across shards -> 3
    L[1, [17, 18]] = 2.0       # tie inside a shard -> 17
    L[2, :] = 0.25             # uniform -> loss log v, argmax 0
    L[3, 63] = 9.0
    targets = torch.tensor([3, 0, 10, -1, v], dtype=torch.int64)
    r, st = _xent_check(L, targets, N, 1.0)
    assert int(st.item()) & tpl.DEVERR_RANGE
    assert r["argmax"].cpu().tolist()[:4] == [3, 17, 0, 63]
    assert abs(float(r["loss"][2]) - math.log(v)) < 1e-5


def test_xent_in_place_gradient():
    inp = tp_inputs.xent_logits(64, 2048, seed=6)
    ref = O.xent(inp["logits"], inp["targets"], 0.5)
    L = inp["logits"].cuda()
    r = tpl.vp_xent(L, inp["targets"].cuda(), 8, grad_scale=0.5, dlogits=L)
    torch.cuda.synchronize()
    assert_close("in-place dlogits", L, ref["dlogits"], TOL_XENT)


@pytest.mark.slow
def test_xent_full_size_sampled_rows():
    w = tp_inputs.WORKLOADS["vocab_v50304"]
    inp = tp_inputs.xent_logits(w["T"], w["v"], seed=0)
    rows = np.r_[0:64, 9000:9064, w["T"] - 64:w["T"]]
    r, st = _xent_check(inp["logits"], inp["targets"], w["N"], 1.0 / w["T"], rows=rows)
    assert int(st.item()) == 0
    # loss_sum is the fixed-order sum of the per-token losses
    s = float(r["loss"].double().sum())
    assert abs(float(r["loss_sum"].item()) - s) <= 1e-5 * abs(s)


def test_xent_deterministic():
    inp = tp_inputs.xent_logits(300, 50304, seed=8)
    a = tpl.vp_xent(inp["logits"].cuda(), inp["targets"].cuda(), 8)
    b = tpl.vp_xent(inp["logits"].cuda(), inp["targets"].cuda(), 8)
    torch.cuda.synchronize()
    for k in ("loss", "loss_sum", "dlogits", "argmax"):
        assert torch.equal(a[k], b[k]), k
