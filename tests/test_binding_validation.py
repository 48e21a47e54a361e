"""The binding's argument checks, on the CPU (no kernel runs).

The C entry points receive bare pointers and the sizes read from the leading
operands, so a caller's tensor of the wrong shape, dtype or device would be
read or written past its end on the GPU.  The binding rejects such a call
before anything reaches the library.  On the CPU a call that passes every
check stops at the binding's "CUDA tensors only" error, which is how these
tests tell a passed check from a rejected one.
"""
import pytest
import torch

import linear_layers_b200 as tpl

BF, F32, I64, I32, U8 = torch.bfloat16, torch.float32, torch.int64, torch.int32, torch.uint8


def t(*shape, dtype=BF):
    return torch.zeros(*shape, dtype=dtype)


def passes(fn, *a, **k):
    with pytest.raises(RuntimeError, match="no CPU path"):
        fn(*a, **k)


def rejected(fn, *a, **k):
    with pytest.raises((ValueError, TypeError)):
        fn(*a, **k)


M, h, F, N = 16, 64, 256, 2


def test_mlp_fwd_checks():
    X, A, b, B = t(M, h), t(h, F), t(F), t(F, h)
    passes(tpl.tp_mlp_fwd, X, A, b, B, N)
    passes(tpl.tp_mlp_fwd, X, A, None, B, N, Zpart=t(N, M, h, dtype=F32))
    rejected(tpl.tp_mlp_fwd, X, A, b, t(h, F), N)              # B in the [out, in] layout
    rejected(tpl.tp_mlp_fwd, X, A, t(h), B, N)                 # bias of the wrong length
    rejected(tpl.tp_mlp_fwd, X, A.float(), b, B, N)            # mixed dtypes
    rejected(tpl.tp_mlp_fwd, X, A, b, B, N, Z=t(M, h + 8))     # output too wide
    rejected(tpl.tp_mlp_fwd, X, A, b, B, N, Zpart=t(N, M, h))  # partials must be fp32
    rejected(tpl.tp_mlp_fwd, X, A, b, B, N, dev_status=t(1, dtype=I64))


def test_mlp_bwd_checks():
    X, A, B, U, Y, dZ = t(M, h), t(h, F), t(F, h), t(M, F), t(M, F), t(M, h)
    passes(tpl.tp_mlp_bwd, X, A, B, U, Y, dZ, N)
    passes(tpl.tp_mlp_bwd_recompute, X, A, B, U, dZ, N, Y=U)
    rejected(tpl.tp_mlp_bwd, X, A, B, U, Y, t(M, F), N)        # dZ of the wrong width
    rejected(tpl.tp_mlp_bwd, X, A, B, U, Y, dZ, N, dbias=t(F))  # dbias must be fp32
    rejected(tpl.tp_mlp_bwd, X, A, B, U[:8], Y, dZ, N)
    rejected(tpl.tp_mlp_bwd_recompute, X, A, B, U, dZ, N, Y=t(M, h))


def test_linear_block_checks():
    X, W, b = t(M, h), t(h, F), t(F)
    passes(tpl.tp_col_linear_fwd, X, W, b, N)
    passes(tpl.tp_col_linear_fwd, X, W, b, N, act=tpl.ACT_GELU_TANH)
    rejected(tpl.tp_col_linear_fwd, X, W, b, N, Y=t(M, F + 8))
    passes(tpl.tp_col_linear_bwd, X, W, None, t(M, F), N)
    rejected(tpl.tp_col_linear_bwd, X, W, None, t(M, h), N)
    rejected(tpl.tp_col_linear_bwd, X, W, None, t(M, F), N, dW=t(F, h))
    Xin, Wr = t(M, F), t(F, h)
    passes(tpl.tp_row_linear_fwd, Xin, Wr, N)
    passes(tpl.tp_row_linear_fwd_noalloc, Xin, Wr, N)
    passes(tpl.tp_row_linear_bwd, Xin, Wr, t(M, h), N)
    rejected(tpl.tp_row_linear_fwd, Xin, t(h, F), N)
    rejected(tpl.tp_row_linear_fwd, Xin, Wr, N, Zpart=t(N + 1, M, h, dtype=F32))
    rejected(tpl.tp_row_linear_fwd_noalloc, Xin, Wr, N, Z=t(M, h, dtype=F32))
    rejected(tpl.tp_row_linear_bwd, Xin, Wr, t(M, F), N)


def test_vocabulary_checks():
    T, v, hv = 32, 128, 64
    ids, E, H = t(T, dtype=I64), t(v, hv), t(T, hv)
    passes(tpl.vp_embed, ids, E, 4)
    rejected(tpl.vp_embed, ids, E, 4, out=t(T, hv + 8))
    rejected(tpl.vp_embed, t(T, dtype=I32), E, 4)
    passes(tpl.tp_logits_fwd, H, E, 4)
    rejected(tpl.tp_logits_fwd, H, t(v, hv + 8), 4)             # E with another hidden size
    rejected(tpl.tp_logits_fwd, H, E, 4, logits=t(T, v))        # logits must be fp32
    L, y = t(T, v, dtype=F32), t(T, dtype=I64)
    passes(tpl.vp_xent, L, y, 4)
    passes(tpl.vp_xent, L, y, 4, dlogits=L)                     # in place over the logits
    rejected(tpl.vp_xent, L, t(T + 1, dtype=I64), 4)
    rejected(tpl.vp_xent, L, y, 4, dlogits=t(T, v))
    rejected(tpl.vp_xent, L, y, 4, argmax=t(T, dtype=I64))
    passes(tpl.vp_xent_bf16_grad, L, y, 4)
    rejected(tpl.vp_xent_bf16_grad, L, y, 4, dlogits=t(T, v, dtype=F32))
    passes(tpl.tp_logits_bwd, t(T, v), H, E, 4)
    rejected(tpl.tp_logits_bwd, t(T, v), H, E, 4, dE=t(v, hv))
    passes(tpl.vp_embed_bwd, ids, t(T, hv), t(v, hv, dtype=F32), 4)
    rejected(tpl.vp_embed_bwd, ids, t(T, hv), t(v, hv), 4)
    rejected(tpl.vp_embed_bwd, ids[:8], t(T, hv), t(v, hv, dtype=F32), 4)
    passes(tpl.tp_linear_xent_fwd, H, E, y, 4)
    rejected(tpl.tp_linear_xent_fwd, H, E, y, 4, lse=t(T, dtype=F32)[:8])
    passes(tpl.tp_linear_xent_dlogits, H, E, y, t(T, dtype=F32), 4)
    rejected(tpl.tp_linear_xent_dlogits, H, E, y, t(T), 4)


def test_attention_and_layernorm_checks():
    b, s, nh = 2, 64, 3
    QKV = t(b * s, 3 * nh * 64)
    passes(tpl.tp_attention_fwd, QKV, b, s, nh, 3, with_lse=True)
    rejected(tpl.tp_attention_fwd, QKV, b, s + 1, nh, 3)       # rows do not match b·s
    rejected(tpl.tp_attention_fwd, QKV, b, s, nh, 3, lse=t(b, s, nh, dtype=F32))
    ctx, lse = t(b * s, nh * 64), t(b, nh, s, dtype=F32)
    passes(tpl.tp_attention_bwd, QKV, ctx, ctx, lse, b, s, nh, 3)
    rejected(tpl.tp_attention_bwd, QKV, ctx, t(b * s, nh * 64 + 8), lse, b, s, nh, 3)
    Ml, hl = 8, 64
    x, g = t(Ml, hl), t(hl)
    passes(tpl.tp_sp_dropout_add_ln_fwd, x, None, x, g, g, 2, with_keep=True)
    rejected(tpl.tp_sp_dropout_add_ln_fwd, x, None, t(Ml, hl + 8), g, g, 2)
    rejected(tpl.tp_sp_dropout_add_ln_fwd, x, None, x, g.float(), g, 2)
    mean = t(Ml, dtype=F32)
    passes(tpl.tp_sp_dropout_add_ln_bwd, x, None, x, g, mean, mean, 2)
    rejected(tpl.tp_sp_dropout_add_ln_bwd, x, t(Ml + 1, hl), x, g, mean, mean, 2)
    rejected(tpl.tp_sp_dropout_add_ln_bwd, x, None, x, g, mean[:4], mean, 2)


def test_device_mismatch_is_rejected():
    X, A, b, B = t(M, h), t(h, F), t(F), t(F, h)
    meta = torch.empty(F, h, dtype=BF, device="meta")
    rejected(tpl.tp_mlp_fwd, X, A, b, meta, N)
