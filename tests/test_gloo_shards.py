"""The pages' sharded algorithm run on real ranks (gloo, world_size 2, CPU).

Each rank holds one column block of A and one row block of B, computes its
partial Z_i and dX_i, and a real torch.distributed all-reduce forms the sums
(the g and f operators).  The result must equal the oracle's unsharded layer.
The vocabulary-parallel loss is checked the same way: each rank owns half of
the vocabulary, max and sum-exp are all-reduced.  So are the other exchange
steps: the sequence-parallel LayerNorm's parameter gradients, the attention
block's output projection over per-rank heads, and the vocabulary
backward's dH.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from oracle import tp_oracle as O
        import tp_inputs

        inp = tp_inputs.mlp_inputs(12, 16, 32, dtype=torch.float32, w_std=0.3, bias_std=0.1, seed=3)
        X, A, b, B, dZ = (O.f64(inp[k]) for k in ("X", "A", "bias", "B", "dZ"))
        offs = O.even_offsets(32, world)
        lo, hi = offs[rank], offs[rank + 1]
        Ui = X @ A[:, lo:hi] + b[lo:hi]
        Yi = O.act_fwd(Ui, O.ACT_GELU_TANH)
        Zi = torch.from_numpy(Yi @ B[lo:hi])
        dist.all_reduce(Zi)                                   # g forward
        dUi = (dZ @ B[lo:hi].T) * O.act_grad(Ui, O.ACT_GELU_TANH)
        dXi = torch.from_numpy(dUi @ A[:, lo:hi].T)
        dist.all_reduce(dXi)                                  # f backward
        _, _, Z = O.mlp_fwd(X, A, b, B)
        g = O.mlp_bwd(X, A, b, B, dZ)
        ok_mlp = (np.abs(Zi.numpy() - Z).max() < 1e-12 and np.abs(dXi.numpy() - g["dX"]).max() < 1e-12
                  and np.abs(X.T @ dUi - g["dA"][:, lo:hi]).max() < 1e-12)

        lg = tp_inputs.xent_logits(5, 40, seed=4)
        L, y = O.f64(lg["logits"]), O.i64(lg["targets"])
        vo = O.even_offsets(40, world)
        Li = L[:, vo[rank]:vo[rank + 1]]
        mi = torch.from_numpy(Li.max(1))
        m = mi.clone()
        dist.all_reduce(m, op=dist.ReduceOp.MAX)
        s = torch.from_numpy(np.exp(Li - m.numpy()[:, None]).sum(1))
        dist.all_reduce(s)
        mine = (y >= vo[rank]) & (y < vo[rank + 1])
        t = torch.from_numpy(np.where(mine, L[np.arange(5), y], 0.0))
        dist.all_reduce(t)
        loss = m.numpy() + np.log(s.numpy()) - t.numpy()
        ok_xent = np.abs(loss - O.xent(L, y)["loss"]).max() < 1e-12

        # sequence-parallel dropout-add-LayerNorm: this rank's token rows,
        # the parameter gradients all-reduced
        r = np.random.default_rng(5)
        M, h, p = 8, 6, 0.25
        x, res, dy = r.normal(size=(M, h)), r.normal(size=(M, h)), r.normal(size=(M, h))
        gam, bet = 1 + 0.2 * r.normal(size=h), 0.1 * r.normal(size=h)
        full = O.dropout_add_layernorm(x, None, res, gam, bet, p, seed=3, offset=1)
        ref = O.dropout_add_layernorm_bwd(dy, None, full["hs"], gam, full["mean"], full["rstd"],
                                          full["keep"], p)
        ro = O.even_offsets(M, world)
        rs = slice(ro[rank], ro[rank + 1])
        mine_f = {k: v[rs] for k, v in full.items() if k in ("hs", "mean", "rstd", "keep")}
        part = O.dropout_add_layernorm_bwd(dy[rs], None, mine_f["hs"], gam, mine_f["mean"],
                                           mine_f["rstd"], mine_f["keep"], p)
        dg, db = torch.from_numpy(part["dgamma"]), torch.from_numpy(part["dbeta"])
        dist.all_reduce(dg)
        dist.all_reduce(db)
        ok_ln = (np.abs(dg.numpy() - ref["dgamma"]).max() < 1e-12
                 and np.abs(db.numpy() - ref["dbeta"]).max() < 1e-12
                 and np.abs(part["dx"] - ref["dx"][rs]).max() < 1e-12)

        # attention block: this rank's heads need no communication; the
        # row-parallel output projection's partials are all-reduced
        bq, sq, nh, hd = 2, 5, 4, 3
        shards = [2, 2]
        std = r.normal(size=(bq * sq, 3 * nh * hd))
        perm, qoffs = O.qkv_shard_columns(nh, hd, shards)
        qkv = std[:, perm]
        Wo = r.normal(size=(nh * hd, 7))
        ctx_all, _ = O.attention_sharded(qkv, bq, sq, nh, hd, shards)
        my = slice(qoffs[rank], qoffs[rank + 1])          # this rank's QKV columns
        ctx_i, _ = O.attention_sharded(qkv[:, my], bq, sq, shards[rank], hd, [shards[rank]])
        co = slice(rank * 2 * hd, (rank + 1) * 2 * hd)    # its context columns / rows of Wo
        Zo = torch.from_numpy(ctx_i @ Wo[co])
        dist.all_reduce(Zo)
        ok_attn = (np.abs(ctx_i - ctx_all[:, co]).max() < 1e-12
                   and np.abs(Zo.numpy() - ctx_all @ Wo).max() < 1e-12)

        # vocabulary backward: dH is the all-reduce of the shards' dlogits_i·E_i
        T, v, hh = 4, 10, 3
        G, Hm, E = r.normal(size=(T, v)), r.normal(size=(T, hh)), r.normal(size=(v, hh))
        vo2 = O.even_offsets(v, world)
        vs = slice(vo2[rank], vo2[rank + 1])
        dH = torch.from_numpy(G[:, vs] @ E[vs])
        dist.all_reduce(dH)
        ok_vbwd = np.abs(dH.numpy() - O.logits_bwd(G, Hm, E)["dH"]).max() < 1e-12
        q.put((rank, bool(ok_mlp), bool(ok_xent), bool(ok_ln), bool(ok_attn), bool(ok_vbwd)))
    finally:
        dist.destroy_process_group()


def test_two_rank_allreduce_matches_unsharded():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(res) == [(0,) + (True,) * 5, (1,) + (True,) * 5], res
