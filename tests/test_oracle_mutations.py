"""Plant plausible mistakes in the oracle (on the CPU) and require the pins
to catch each one: a pin set that a dropped term, a wrong sign or index, or
a transposed operand slips through would not be worth trusting."""
import math

import numpy as np
import pytest

from oracle import tp_oracle as O
from tests import oracle_checks as C


def _m_gelu_grad_drop_term(mp):
    def bad(u, act):
        if act == O.ACT_GELU_TANH:
            t = np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3))
            return 0.5 * (1.0 + t)           # dropped the x·(1 − t²)·dinner term
        return O.__dict__["_orig_act_grad"](u, act)
    mp.setitem(O.__dict__, "_orig_act_grad", O.act_grad)
    mp.setattr(O, "act_grad", bad)


def _m_gelu_wrong_constant(mp):
    mp.setattr(O, "_SQRT_2_OVER_PI", math.sqrt(math.pi / 2))


def _m_gelu_sign(mp):
    orig = O.act_fwd

    def bad(u, act):
        if act == O.ACT_GELU_TANH:
            return 0.5 * u * (1.0 - np.tanh(O._SQRT_2_OVER_PI * (u + O._GELU_CUBIC * u ** 3)))
        return orig(u, act)
    mp.setattr(O, "act_fwd", bad)


def _m_fwd_drop_bias(mp):
    orig = O.mlp_fwd
    mp.setattr(O, "mlp_fwd", lambda X, A, bias, B, act=O.ACT_GELU_TANH: orig(X, A, None, B, act))


def _m_bwd_no_act_grad(mp):
    orig = O.mlp_bwd

    def bad(X, A, bias, B, dZ, act=O.ACT_GELU_TANH):
        g = orig(X, A, bias, B, dZ, act)
        g["dA"] = O.f64(X).T @ g["dY"]
        return g
    mp.setattr(O, "mlp_bwd", bad)


def _m_bwd_transposed_dB(mp):
    orig = O.mlp_bwd

    def bad(X, A, bias, B, dZ, act=O.ACT_GELU_TANH):
        g = orig(X, A, bias, B, dZ, act)
        g["dB"] = g["dB"].reshape(g["dB"].shape[1], g["dB"].shape[0]).T.copy()  # wrong index order
        return g
    mp.setattr(O, "mlp_bwd", bad)


def _m_bwd_dX_no_sum_of_shards(mp):
    orig = O.mlp_bwd_sharded

    def bad(*a, **k):
        r = orig(*a, **k)
        r["dX"] = r["dXparts"][0]        # f backward without its all-reduce
        return r
    mp.setattr(O, "mlp_bwd_sharded", bad)


def _m_allreduce_drops_last(mp):
    mp.setattr(O, "all_reduce_sum", lambda parts: np.sum(np.stack(parts[:-1] or parts), axis=0)
               if len(parts) > 1 else np.array(parts[0], dtype=np.float64))


def _m_offsets_off_by_one(mp):
    def bad(total, N):
        step = total // N
        return [0] + [i * step - 1 for i in range(1, N)] + [total]
    mp.setattr(O, "even_offsets", bad)


def _m_embed_index_shift(mp):
    def bad(ids, E):
        ids, E = O.i64(ids), O.f64(E)
        out = np.zeros((ids.shape[0], E.shape[1]))
        ok = (ids >= 0) & (ids < E.shape[0])
        out[ok] = E[np.maximum(ids[ok] - 1, 0)]
        return out
    mp.setattr(O, "embed_lookup", bad)


def _m_xent_loss_sign(mp):
    orig = O.xent

    def bad(L, y, grad_scale=1.0):
        r = orig(L, y, grad_scale)
        Lf, yy = O.f64(L), O.i64(y)
        tgt = Lf[np.arange(Lf.shape[0]), np.clip(yy, 0, Lf.shape[1] - 1)]
        r["loss"] = r["loss"] + 2 * tgt
        return r
    mp.setattr(O, "xent", bad)


def _m_xent_no_onehot(mp):
    orig = O.xent

    def bad(L, y, grad_scale=1.0):
        r = orig(L, y, grad_scale)
        Lf = O.f64(L)
        p = np.exp(Lf - Lf.max(1, keepdims=True))
        r["dlogits"] = grad_scale * p / p.sum(1, keepdims=True)
        return r
    mp.setattr(O, "xent", bad)


def _m_xent_combine_no_rescale(mp):
    orig = O.xent_sharded

    def bad(L, y, N, grad_scale=1.0):
        r = orig(L, y, N, grad_scale)
        Lf = O.f64(L)
        offs = O.even_offsets(Lf.shape[1], N)
        S = sum(np.exp(Lf[:, offs[i]:offs[i + 1]] - Lf[:, offs[i]:offs[i + 1]].max(1, keepdims=True)).sum(1)
                for i in range(N))
        r["S"] = S
        r["loss"] = r["m"] + np.log(S) - Lf[np.arange(Lf.shape[0]), O.i64(y)]
        return r
    mp.setattr(O, "xent_sharded", bad)


def _m_argmax_last(mp):
    orig = O.xent

    def bad(L, y, grad_scale=1.0):
        r = orig(L, y, grad_scale)
        Lf = O.f64(L)
        r["argmax"] = Lf.shape[1] - 1 - np.argmax(Lf[:, ::-1], axis=1)
        return r
    mp.setattr(O, "xent", bad)


def _m_embed_bwd_overwrites_repeats(mp):
    def bad(ids, dout, v):
        ids, G = O.i64(ids), O.f64(dout)
        dE = np.zeros((v, G.shape[1]))
        ok = (ids >= 0) & (ids < v)
        dE[ids[ok]] = G[ok]            # assignment instead of accumulation
        return dE
    mp.setattr(O, "embed_bwd", bad)


def _m_logits_bwd_shards_reversed(mp):
    orig = O.logits_bwd_sharded

    def bad(dlogits, H, E, N):
        r = orig(dlogits, H, E, N)
        offs = O.even_offsets(O.f64(E).shape[0], N)
        blocks = [r["dE"][offs[i]:offs[i + 1]] for i in range(N)]
        r["dE"] = np.concatenate(blocks[::-1], axis=0)
        return r
    mp.setattr(O, "logits_bwd_sharded", bad)


def _m_logits_bwd_drops_scale(mp):
    orig = O.logits_bwd

    def bad(dlogits, H, E):
        r = orig(dlogits, H, E)
        r["dE"] = 0.5 * r["dE"]
        return r
    mp.setattr(O, "logits_bwd", bad)


def _m_lxent_transposed_table(mp):
    def bad(H, E, targets, grad_scale=1.0):
        return O.xent(O.f64(H) @ O.f64(E), targets, grad_scale)   # E used as [h,v]
    mp.setattr(O, "linear_xent", bad)


def _m_lxent_lse_without_max(mp):
    orig = O.linear_xent

    def bad(H, E, targets, grad_scale=1.0):
        r = orig(H, E, targets, grad_scale)
        L = O.logits(H, E)
        r["lse"] = np.log(np.exp(L - L.max(axis=1)[:, None]).sum(axis=1))   # dropped + m
        return r
    mp.setattr(O, "linear_xent", bad)


def _m_partitioned_tie_to_later_part(mp):
    orig = O.xent_sharded

    def bad(logits_, targets, N, grad_scale=1.0, offsets=None):
        r = orig(logits_, targets, N, grad_scale, offsets)
        L = O.f64(logits_)
        r["argmax"] = (L.shape[1] - 1 - np.argmax(L[:, ::-1], axis=1)).astype(np.int64)
        return r
    mp.setattr(O, "xent_sharded", bad)


def _m_recompute_uses_derivative(mp):
    orig = O.mlp_bwd_recompute

    def bad(X, A, B, U, dZ, act=O.ACT_GELU_TANH):
        r = orig(X, A, B, U, dZ, act)
        Y = O.act_grad(O.f64(U), act)                     # derivative in place of the value
        r["Y"] = Y
        r["dB"] = Y.T @ O.f64(dZ)
        return r
    mp.setattr(O, "mlp_bwd_recompute", bad)


def _m_attention_mask_off_by_one(mp):
    orig = O.attention_head

    def bad(Q, K, V, causal=True, scale=None):
        if not causal:
            return orig(Q, K, V, causal, scale)
        Q, K, V = O.f64(Q), O.f64(K), O.f64(V)
        s, d = Q.shape
        sc = (1.0 / math.sqrt(d)) if scale is None else float(scale)
        S = (Q @ K.T) * sc
        S = np.where(np.tril(np.ones((s, s), dtype=bool), k=-1), S, -np.inf)   # drops the diagonal
        S[0, 0] = 0.0
        m = S.max(axis=1)
        P = np.exp(S - m[:, None])
        l = P.sum(axis=1)
        return (P / l[:, None]) @ V, m + np.log(l)
    mp.setattr(O, "attention_head", bad)


def _m_attention_kv_swapped(mp):
    orig = O.attention_sharded

    def bad(QKV, b, s, n_heads, head_dim, heads_per_shard, causal=True, scale=None):
        X = O.f64(QKV).copy()
        col = 0
        for nh in heads_per_shard:                    # reads V where K should be and back
            k0, v0 = col + nh * head_dim, col + 2 * nh * head_dim
            X[:, k0:k0 + nh * head_dim], X[:, v0:v0 + nh * head_dim] = (
                X[:, v0:v0 + nh * head_dim].copy(), X[:, k0:k0 + nh * head_dim].copy())
            col += 3 * nh * head_dim
        return orig(X, b, s, n_heads, head_dim, heads_per_shard, causal, scale)
    mp.setattr(O, "attention_sharded", bad)


def _m_philox_wrong_weyl(mp):
    mp.setattr(O, "_PHILOX_W1", 0xBB67AE86)


def _m_layernorm_unbiased_variance(mp):
    orig = O.dropout_add_layernorm

    def bad(x, bias, residual, gamma, beta, p, seed, offset, eps=1e-5):
        f = orig(x, bias, residual, gamma, beta, p, seed, offset, eps)
        hs = f["hs"]
        var = hs.var(axis=1, ddof=1)                     # n − 1 in place of n
        f["rstd"] = 1.0 / np.sqrt(var + eps)
        xhat = (hs - f["mean"][:, None]) * f["rstd"][:, None]
        f["y"] = xhat * O.f64(gamma)[None, :] + O.f64(beta)[None, :]
        return f
    mp.setattr(O, "dropout_add_layernorm", bad)


def _m_dropout_no_rescale(mp):
    orig = O.dropout_add_layernorm_bwd

    def bad(dy, dhs_in, hs, gamma, mean, rstd, keep, p):
        r = orig(dy, dhs_in, hs, gamma, mean, rstd, keep, p)
        r["dx"] = r["dx"] * (1.0 - p)                   # dropped the 1/(1 − p)
        r["dbias"] = r["dx"].sum(axis=0)
        return r
    mp.setattr(O, "dropout_add_layernorm_bwd", bad)


def _m_layernorm_dgamma_without_xhat(mp):
    orig = O.dropout_add_layernorm_bwd

    def bad(dy, dhs_in, hs, gamma, mean, rstd, keep, p):
        r = orig(dy, dhs_in, hs, gamma, mean, rstd, keep, p)
        r["dgamma"] = O.f64(dy).sum(axis=0)
        return r
    mp.setattr(O, "dropout_add_layernorm_bwd", bad)


def _m_attention_bwd_drops_rowsum(mp):
    orig = O.attention_head_bwd

    def bad(Q, K, V, dO, causal=True, scale=None):
        Qf, Kf, Vf, dOf = O.f64(Q), O.f64(K), O.f64(V), O.f64(dO)
        s, d = Qf.shape
        sc = (1.0 / math.sqrt(d)) if scale is None else float(scale)
        S = (Qf @ Kf.T) * sc
        if causal:
            S = np.where(np.tril(np.ones((s, s), dtype=bool)), S, -np.inf)
        P = np.exp(S - S.max(axis=1)[:, None])
        P = P / P.sum(axis=1)[:, None]
        dS = P * (dOf @ Vf.T)                         # dropped − rowsum(dO ⊙ O)
        return sc * dS @ Kf, sc * dS.T @ Qf, P.T @ dOf
    mp.setattr(O, "attention_head_bwd", bad)


def _m_col_dbias_without_act_grad(mp):
    orig = O.col_linear_bwd

    def bad(X, W, U, dY, act=O.ACT_NONE):
        g = orig(X, W, U, dY, act)
        g["dbias"] = O.f64(dY).sum(axis=0)            # dbias from dY, act'(U) forgotten
        return g
    mp.setattr(O, "col_linear_bwd", bad)


def _m_col_dbias_mean_not_sum(mp):
    orig = O.col_linear_bwd

    def bad(X, W, U, dY, act=O.ACT_NONE):
        g = orig(X, W, U, dY, act)
        g["dbias"] = g["dU"].mean(axis=0)             # averaged over rows instead of summed
        return g
    mp.setattr(O, "col_linear_bwd", bad)


def _m_row_bwd_dW_rows_misaligned(mp):
    orig = O.row_linear_bwd

    def bad(Xin, W, dZ):
        g = orig(Xin, W, dZ)
        g["dW"] = O.f64(Xin)[::-1].T @ O.f64(dZ)      # token rows of Xin and dZ out of step
        return g
    mp.setattr(O, "row_linear_bwd", bad)


def _m_row_bwd_dX_sign(mp):
    orig = O.row_linear_bwd

    def bad(Xin, W, dZ):
        g = orig(Xin, W, dZ)
        g["dXin"] = -g["dXin"]
        return g
    mp.setattr(O, "row_linear_bwd", bad)


def _m_col_fwd_drops_bias(mp):
    orig = O.col_linear_fwd
    mp.setattr(O, "col_linear_fwd", lambda X, W, bias=None, act=O.ACT_NONE: orig(X, W, None, act))


def _m_row_fwd_drops_last_shard(mp):
    orig = O.row_linear_fwd

    def bad(Xin, W, offsets=None, N=None):
        Z, parts = orig(Xin, W, offsets, N)
        if parts is None:
            return Z, parts
        return O.all_reduce_sum(parts[:-1] or parts), parts   # the g sum without the last shard
    mp.setattr(O, "row_linear_fwd", bad)


def _m_qkv_columns_k_v_swapped(mp):
    orig = O.qkv_shard_columns

    def bad(n_heads, head_dim, heads_per_shard):
        perm, offs = orig(n_heads, head_dim, heads_per_shard)
        perm = list(perm)
        h = n_heads * head_dim
        perm = [c + h if h <= c < 2 * h else (c - h if c >= 2 * h else c) for c in perm]
        return perm, offs
    mp.setattr(O, "qkv_shard_columns", bad)


def _m_embed_owner_inclusive_range(mp):
    def bad(ids, v, N):
        ids = O.i64(ids)
        offs = O.even_offsets(v, N)
        own = np.full(ids.shape, -1, dtype=np.int64)
        for i in range(N):
            own[(ids >= offs[i]) & (ids <= offs[i + 1])] = i   # hi taken as inclusive
        return own
    mp.setattr(O, "embed_owner", bad)


def _m_vp_embed_shard_base_off(mp):
    def bad(ids, E, N):
        ids, E = O.i64(ids), O.f64(E)
        v, h = E.shape
        offs = O.even_offsets(v, N)
        parts = []
        for i in range(N):
            lo, hi = offs[i], offs[i + 1]
            mine = (ids >= lo) & (ids < hi)
            part = np.zeros((ids.shape[0], h))
            part[mine] = E[np.minimum(ids[mine] - lo + (1 if i else 0), v - 1)]   # wrong base
            parts.append(part)
        return O.all_reduce_sum(parts)
    mp.setattr(O, "vp_embed_sharded", bad)


def _m_logits_sharded_wrong_rows(mp):
    def bad(H, E, N):
        H, E = O.f64(H), O.f64(E)
        offs = O.even_offsets(E.shape[0], N)
        return [H @ E[offs[N - 1 - i]:offs[N - i]].T for i in range(N)]   # shards in reverse
    mp.setattr(O, "logits_sharded", bad)


def _m_dropout_keep_next_word(mp):
    orig = O.dropout_keep

    def bad(M, h, p, seed, offset):
        k = orig(M, h, p, seed, offset).reshape(-1)
        n = k.size
        w = np.arange(n)
        return k[np.minimum((w // 4) * 4 + (w + 1) % 4, n - 1)].reshape(M, h)   # word e+1 mod 4
    mp.setattr(O, "dropout_keep", bad)


def _m_tied_grad_output_only(mp):
    mp.setattr(O, "tied_embedding_grad", lambda dE_output, dE_input: O.f64(dE_output))


def _m_embed_bwd_sharded_wrong_shard(mp):
    orig = O.embed_bwd_sharded

    def bad(ids, dout, v, N):
        blocks = orig(ids, dout, v, N)
        if isinstance(blocks, list) and len(blocks) > 1:
            blocks = blocks[1:] + blocks[:1]     # blocks rotated by one shard
        elif isinstance(blocks, np.ndarray):
            blocks = np.roll(blocks, v // max(N, 1), axis=0)
        return blocks
    mp.setattr(O, "embed_bwd_sharded", bad)


def _m_mlp_fwd_sharded_no_bias(mp):
    orig = O.mlp_fwd_sharded
    mp.setattr(O, "mlp_fwd_sharded",
               lambda X, A, bias, B, N, offsets=None, act=O.ACT_GELU_TANH: orig(X, A, None, B, N, offsets, act))


def _m_ln_bwd_sharded_first_shard_params(mp):
    orig = O.dropout_add_layernorm_bwd_sharded

    def bad(dy, dhs_in, hs, gamma, mean, rstd, keep, p, N):
        r = orig(dy, dhs_in, hs, gamma, mean, rstd, keep, p, N)
        M = O.f64(dy).shape[0]
        first = O.dropout_add_layernorm_bwd(O.f64(dy)[: M // N], None if dhs_in is None else O.f64(dhs_in)[: M // N],
                                            O.f64(hs)[: M // N], gamma, O.f64(mean)[: M // N],
                                            O.f64(rstd)[: M // N], keep[: M // N], p)
        r["dgamma"] = first["dgamma"]     # the parameter gradients without their all-reduce
        return r
    mp.setattr(O, "dropout_add_layernorm_bwd_sharded", bad)


def _m_attention_sharded_bwd_no_dv(mp):
    orig = O.attention_sharded_bwd

    def bad(QKV, dctx, b, s, n_heads, head_dim, heads_per_shard, causal=True, scale=None):
        d = orig(QKV, dctx, b, s, n_heads, head_dim, heads_per_shard, causal, scale)
        col = 0
        for nh in heads_per_shard:            # zero every shard's V block
            d[:, col + 2 * nh * head_dim: col + 3 * nh * head_dim] = 0.0
            col += 3 * nh * head_dim
        return d
    mp.setattr(O, "attention_sharded_bwd", bad)


MUTATIONS = [v for k, v in sorted(globals().items()) if k.startswith("_m_")]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__[3:])
def test_pins_catch_mutation(mutate, monkeypatch):
    mutate(monkeypatch)
    failed = []
    for check in C.ALL_CHECKS:
        try:
            check(O)
        except Exception:  # AssertionError, or a shape error from a bad transpose
            failed.append(check.__name__)
    assert failed, "no pin caught this planted mistake"
