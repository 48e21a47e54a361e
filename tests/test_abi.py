"""The C ABI on the host: the library builds, loads and exports every symbol
include/tplayers.h declares; argument validation answers before anything is
enqueued; and with no sm_100 device current a valid call fails loudly
(TP_ERR_DEVICE) instead of falling back to a CPU path."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import linear_layers_b200 as tpl
from linear_layers_b200 import build as tpbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tplayers.h")

TP_OK, TP_ERR_NULL, TP_ERR_SHAPE, TP_ERR_ALIGN, TP_ERR_DTYPE = 0, 1, 2, 3, 4
TP_ERR_DEVICE = 8


@pytest.fixture(scope="module")
def L():
    tpbuild.build()
    return tpl.lib()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^TP_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("tp_mlp_fwd", "tp_mlp_bwd", "vp_embed", "vp_xent", "tp_logits_fwd",
                 "tp_col_linear_fwd", "tp_col_linear_bwd", "tp_row_linear_fwd",
                 "tp_row_linear_bwd", "tp_workspace_bytes", "tp_status_string", "tp_version"):
        assert must in names, must


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", tpl.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    declared = set(_declared())
    assert declared <= exported, declared - exported
    # nothing but the API leaks out (the static CUDA runtime stays private)
    assert exported == declared, exported - declared
    for name in declared:
        assert getattr(L, name) is not None


def test_status_strings_and_version(L):
    assert tpl.tp_version() == 100
    assert tpl.tp_status_string(0) == "ok"
    for s in range(1, 9):
        assert tpl.tp_status_string(s) not in ("ok", "unknown status")
    assert tpl.tp_status_string(99) == "unknown status"


def test_workspace_sizes_are_host_only(L):
    # h=4096, F=16384, N=8: room for split partials plus dbias partials
    fwd = tpl.tp_workspace_bytes(tpl.OP_MLP_FWD, 4096, 4096, 16384, 8)
    bwd = tpl.tp_workspace_bytes(tpl.OP_MLP_BWD, 4096, 4096, 16384, 8)
    assert fwd > 0 and bwd > fwd
    assert bwd - fwd >= (4096 // 32) * 16384 * 4
    assert tpl.tp_workspace_bytes(tpl.OP_ROW_LINEAR_BWD, 16, 64, 256, 2) == 0
    assert tpl.tp_workspace_bytes(tpl.OP_MLP_FWD, 0, 64, 256, 2) == 0


FAKE = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: validation answers first


def _mlp_fwd(L, **kw):
    a = dict(X=FAKE, A=FAKE, bias=None, B=FAKE, M=16, h=64, F=256, N=2, offs=None, dt=0, act=1,
             U=FAKE, Y=FAKE, Z=FAKE, Zpart=None, ws=None, wsb=0, st=None, stream=None)
    a.update(kw)
    return L.tp_mlp_fwd(a["X"], a["A"], a["bias"], a["B"], a["M"], a["h"], a["F"], a["N"],
                        a["offs"], a["dt"], a["act"], a["U"], a["Y"], a["Z"], a["Zpart"], a["ws"],
                        a["wsb"], a["st"], a["stream"])


def test_validation_errors_before_any_launch(L):
    assert _mlp_fwd(L, X=None) == TP_ERR_NULL
    assert _mlp_fwd(L, Z=None) == TP_ERR_NULL
    assert _mlp_fwd(L, dt=7) == TP_ERR_DTYPE
    assert _mlp_fwd(L, act=9) == TP_ERR_DTYPE
    assert _mlp_fwd(L, M=0) == TP_ERR_SHAPE
    assert _mlp_fwd(L, M=(1 << 30) + 1) == TP_ERR_SHAPE        # sizes are bounded by 2^30
    assert _mlp_fwd(L, h=-8) == TP_ERR_SHAPE
    assert _mlp_fwd(L, F=250, N=4) == TP_ERR_SHAPE            # F % N without offsets
    assert _mlp_fwd(L, h=60) == TP_ERR_ALIGN                   # bf16 rows need 8 | h
    assert _mlp_fwd(L, X=ctypes.c_void_p((1 << 20) + 8)) == TP_ERR_ALIGN
    bad = (ctypes.c_int64 * 3)(0, 300, 256)                    # not increasing
    assert _mlp_fwd(L, offs=bad) == TP_ERR_SHAPE
    short = (ctypes.c_int64 * 3)(0, 100, 250)                  # does not end at F
    assert _mlp_fwd(L, offs=short) == TP_ERR_SHAPE
    # vocabulary entry points
    assert L.vp_embed(FAKE, 4, FAKE, 300, 64, 7, 0, FAKE, None, None) == TP_ERR_SHAPE   # 7 ∤ 300
    assert L.vp_embed(None, 4, FAKE, 300, 64, 2, 0, FAKE, None, None) == TP_ERR_NULL
    assert L.vp_xent(FAKE, FAKE, 4, 300, 7, 1.0, FAKE, None, None, None, None, None) == TP_ERR_SHAPE
    assert L.tp_logits_fwd(FAKE, FAKE, 4, 64, 302, 2, FAKE, None, None) == TP_ERR_ALIGN
    # fused output layer + loss: workspace is checked before the device
    wsb = tpl.tp_workspace_bytes(tpl.OP_LINEAR_XENT, 4, 64, 300, 2)
    assert wsb >= 3 * 3 * 4 * 4 + 4 * 4                       # 3 slices x 4 tokens, 3 planes
    lx = L.tp_linear_xent_fwd
    assert lx(FAKE, FAKE, FAKE, 4, 64, 300, 7, FAKE, None, None, None, FAKE, wsb, None,
              None) == TP_ERR_SHAPE
    assert lx(FAKE, FAKE, None, 4, 64, 300, 2, FAKE, None, None, None, FAKE, wsb, None,
              None) == TP_ERR_NULL
    assert lx(FAKE, FAKE, FAKE, 4, 60, 300, 2, FAKE, None, None, None, FAKE, wsb, None,
              None) == TP_ERR_ALIGN
    assert lx(FAKE, FAKE, FAKE, 4, 64, 300, 2, FAKE, None, None, None, FAKE, wsb - 1, None,
              None) == 7                                       # TP_ERR_WORKSPACE
    assert L.tp_linear_xent_dlogits(FAKE, FAKE, FAKE, FAKE, 4, 64, 300, 2, 1.0, FAKE, None,
                                    None) == TP_ERR_ALIGN     # bf16 rows need 8 | v
    # attention core: head_dim 64 only, shards cover the heads
    at = L.tp_attention_fwd
    assert at(FAKE, 2, 16, 4, 128, 2, None, 1, 0.0, FAKE, None, None, None) == 5   # UNSUPPORTED
    assert at(FAKE, 2, 16, 4, 64, 5, None, 1, 0.0, FAKE, None, None, None) == TP_ERR_SHAPE
    bad = (ctypes.c_int64 * 3)(0, 3, 3)                        # empty shard
    assert at(FAKE, 2, 16, 3, 64, 2, bad, 1, 0.0, FAKE, None, None, None) == TP_ERR_SHAPE
    assert at(None, 2, 16, 4, 64, 2, None, 1, 0.0, FAKE, None, None, None) == TP_ERR_NULL
    # attention backward: the lse and a workspace are required
    ab = L.tp_attention_bwd
    wsa = tpl.tp_workspace_bytes(tpl.OP_ATTENTION_BWD, 32, 4, 64, 2)
    assert wsa >= 32 * 4 * 4 + 32 * 4 * 64 * 4                  # D, then the fp32 dQ accumulator
    assert ab(FAKE, FAKE, FAKE, None, 2, 16, 4, 64, 2, None, 1, 0.0, FAKE, FAKE, wsa, None,
              None) == TP_ERR_NULL
    assert ab(FAKE, FAKE, FAKE, FAKE, 2, 16, 4, 64, 2, None, 1, 0.0, FAKE, FAKE, wsa - 1, None,
              None) == 7                                       # TP_ERR_WORKSPACE
    assert ab(FAKE, FAKE, FAKE, FAKE, 2, 16, 4, 32, 2, None, 1, 0.0, FAKE, FAKE, wsa, None,
              None) == 5                                       # head_dim 64 only
    # dropout-add-LayerNorm: 0 <= p < 1, rows split evenly, h a multiple of 8
    ln = L.tp_sp_dropout_add_ln_fwd
    args = lambda **k: dict(dict(x=FAKE, b=None, r=FAKE, g=FAKE, be=FAKE, M=64, h=1600, N=4,
                                 p=0.1, seed=1, off=0, eps=1e-5, hs=FAKE, y=FAKE, m=FAKE, rs=FAKE,
                                 keep=None), **k)
    call = lambda a: ln(a["x"], a["b"], a["r"], a["g"], a["be"], a["M"], a["h"], a["N"], a["p"],
                        a["seed"], a["off"], a["eps"], a["hs"], a["y"], a["m"], a["rs"], a["keep"],
                        None, None)
    assert call(args(p=1.0)) == TP_ERR_SHAPE
    assert call(args(p=-0.1)) == TP_ERR_SHAPE
    assert call(args(M=66)) == TP_ERR_SHAPE                  # 4 ∤ 66
    assert call(args(h=1604)) == TP_ERR_ALIGN
    assert call(args(h=16384)) == 5                           # wider than 8192
    assert call(args(x=None)) == TP_ERR_NULL
    lb = L.tp_sp_dropout_add_ln_bwd
    wsl = tpl.tp_workspace_bytes(tpl.OP_SP_LN_BWD, 64, 1600, 1600, 4)
    assert wsl >= 3 * (64 // 8) * 1600 * 4
    assert lb(FAKE, None, FAKE, FAKE, FAKE, FAKE, 64, 1600, 4, 0.1, 1, 0, FAKE, FAKE, FAKE, FAKE,
              None, FAKE, wsl - 1, None, None) == 7           # TP_ERR_WORKSPACE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_fails_loudly(L):
    assert _mlp_fwd(L) == TP_ERR_DEVICE
    assert L.vp_embed(FAKE, 4, FAKE, 300, 64, 2, 0, FAKE, None, None) == TP_ERR_DEVICE
    assert L.vp_xent(FAKE, FAKE, 4, 300, 2, 1.0, FAKE, None, None, None, None, None) == TP_ERR_DEVICE
    wsb = tpl.tp_workspace_bytes(tpl.OP_LINEAR_XENT, 4, 64, 304, 2)
    assert L.tp_linear_xent_fwd(FAKE, FAKE, FAKE, 4, 64, 304, 2, FAKE, None, None, None, FAKE,
                                wsb, None, None) == TP_ERR_DEVICE
    assert L.tp_linear_xent_dlogits(FAKE, FAKE, FAKE, FAKE, 4, 64, 304, 2, 1.0, FAKE, None,
                                    None) == TP_ERR_DEVICE
    assert L.tp_attention_fwd(FAKE, 2, 16, 25, 64, 4, None, 1, 0.0, FAKE, None, None,
                              None) == TP_ERR_DEVICE
    wsa = tpl.tp_workspace_bytes(tpl.OP_ATTENTION_BWD, 32, 25, 64, 4)
    assert L.tp_attention_bwd(FAKE, FAKE, FAKE, FAKE, 2, 16, 25, 64, 4, None, 1, 0.0, FAKE, FAKE,
                              wsa, None, None) == TP_ERR_DEVICE
    assert L.tp_sp_dropout_add_ln_fwd(FAKE, None, FAKE, FAKE, FAKE, 64, 1600, 4, 0.1, 1, 0, 1e-5,
                                      FAKE, FAKE, FAKE, FAKE, None, None, None) == TP_ERR_DEVICE
    with pytest.raises(RuntimeError, match="no CPU path"):
        X = torch.zeros(16, 64, dtype=torch.bfloat16)
        tpl.tp_mlp_fwd(X, torch.zeros(64, 256, dtype=torch.bfloat16), None,
                       torch.zeros(256, 64, dtype=torch.bfloat16), 2)


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "linear_layers_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in text.lower().replace("oracle is the oracle", ""), f
