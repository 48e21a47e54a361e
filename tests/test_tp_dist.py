"""The multi-GPU driver (linear_layers_b200.tp_dist): shard i on rank i and
the g / f all-reduces through torch.distributed.

CPU: two and three gloo ranks, each computing its shard with a float64
stand-in for the library (the per-shard compute is a parameter of the
driver), must reproduce the oracle's unsharded layer; this checks the
partitioning, which rank holds what, and which sums are all-reduced.
GPU: one NCCL rank on the GPU running the library's own single-shard calls,
against the oracle.
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


class _Float64Shard:
    """The per-shard math of one rank written with torch float64 CPU ops (a
    test stand-in for the library's single-shard calls)."""

    def __init__(self, O):
        self.O = O

    def mlp_fwd(self, X, A_i, bias_i, B_i, act):
        U = X @ A_i + (0 if bias_i is None else bias_i)
        Y = torch.from_numpy(self.O.act_fwd(U.numpy(), act))
        return Y @ B_i, U, Y

    def mlp_bwd(self, X, A_i, B_i, U_i, Y_i, dZ, act):
        dU = (dZ @ B_i.T) * torch.from_numpy(self.O.act_grad(U_i.numpy(), act))
        return {"dX": dU @ A_i.T, "dA": X.T @ dU, "dbias": dU.sum(0), "dB": Y_i.T @ dZ}

    def col_fwd(self, X, W_i, bias_i):
        return X @ W_i + (0 if bias_i is None else bias_i)

    def col_bwd(self, X, W_i, dY_i):
        return {"dX": dY_i @ W_i.T, "dW": X.T @ dY_i, "dbias": dY_i.sum(0)}

    def row_fwd(self, Xin_i, W_i):
        return Xin_i @ W_i

    def row_bwd(self, Xin_i, W_i, dZ):
        return {"dXin": dZ @ W_i.T, "dW": Xin_i.T @ dZ}


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from linear_layers_b200 import tp_dist as D
        from oracle import tp_oracle as O
        import tp_inputs

        ok = []
        comp = _Float64Shard(O)
        # count the collectives: [MLP-TP] §2.3 / [TP-ILL] §2.2 put exactly one
        # all-reduce of b·s·h elements in the MLP's forward (g) and one in its
        # backward (f); the column-parallel block all-reduces only dX, the
        # row-parallel block only Z
        sent = []
        plain_all_reduce = dist.all_reduce

        def counting_all_reduce(t, *a, **k):
            sent.append(t.numel())
            return plain_all_reduce(t, *a, **k)

        D.dist.all_reduce = counting_all_reduce

        def moved(fn, *a):
            sent.clear()
            r = fn(*a)
            return r, list(sent)
        F = 48
        inp = tp_inputs.mlp_inputs(10, 16, F, dtype=torch.float32, w_std=0.3, bias_std=0.1, seed=7)
        X, A, b, B, dZ = (inp[k].double() for k in ("X", "A", "bias", "B", "dZ"))
        uneven = {2: [0, 16, 48], 3: [0, 8, 24, 48]}[world]
        for offsets in (None, uneven):
            A_i, b_i, B_i = D.shard_mlp_weights(A, b, B, rank, world, offsets)
            layer = D.TPMLP(A_i, b_i, B_i, compute=comp)
            (Z, state), n_fwd = moved(layer.forward, X)
            g, n_bwd = moved(layer.backward, X, state, dZ)
            ok.append(n_fwd == [X.shape[0] * X.shape[1]] and n_bwd == [X.shape[0] * X.shape[1]])
            _, _, oZ = O.mlp_fwd(X, A, b, B)
            og = O.mlp_bwd(X, A, b, B, dZ)
            offs = D.shard_bounds(F, world, offsets)
            lo, hi = offs[rank], offs[rank + 1]
            ok.append(np.abs(Z.numpy() - oZ).max() < 1e-12)
            ok.append(np.abs(g["dX"].numpy() - og["dX"]).max() < 1e-12)
            ok.append(np.abs(g["dA"].numpy() - og["dA"][:, lo:hi]).max() < 1e-12)
            ok.append(np.abs(g["dB"].numpy() - og["dB"][lo:hi]).max() < 1e-12)
            ok.append(np.abs(g["dbias"].numpy() - og["dbias"][lo:hi]).max() < 1e-12)

        # the linear blocks: column-parallel QKV-like projection, row-parallel output
        r = np.random.default_rng(11)
        Xl = torch.from_numpy(r.normal(size=(6, 9)))
        Wc = torch.from_numpy(r.normal(size=(9, 12)))
        bc = torch.from_numpy(r.normal(size=12))
        offs = D.shard_bounds(12, world, None)
        lo, hi = offs[rank], offs[rank + 1]
        col = D.ColumnParallelLinear(Wc[:, lo:hi].contiguous(), bc[lo:hi].contiguous(), compute=comp)
        Yi, n_cf = moved(col.forward, Xl)
        dY = torch.from_numpy(r.normal(size=(6, 12)))
        gc, n_cb = moved(col.backward, Xl, dY[:, lo:hi].contiguous())
        ok.append(n_cf == [] and n_cb == [6 * 9])
        _, oY = O.col_linear_fwd(Xl, Wc, bc)
        ocb = O.col_linear_bwd(Xl, Wc, oY, dY)
        ok.append(np.abs(Yi.numpy() - oY[:, lo:hi]).max() < 1e-12)
        ok.append(np.abs(gc["dX"].numpy() - ocb["dX"]).max() < 1e-12)
        ok.append(np.abs(gc["dW"].numpy() - ocb["dW"][:, lo:hi]).max() < 1e-12)
        ok.append(np.abs(gc["dbias"].numpy() - ocb["dbias"][lo:hi]).max() < 1e-12)
        Wr = torch.from_numpy(r.normal(size=(12, 5)))
        row = D.RowParallelLinear(Wr[lo:hi].contiguous(), compute=comp)
        Zr, n_rf = moved(row.forward, Yi)
        dZr = torch.from_numpy(r.normal(size=(6, 5)))
        gr, n_rb = moved(row.backward, Yi, dZr)
        ok.append(n_rf == [6 * 5] and n_rb == [])
        oZr, _ = O.row_linear_fwd(oY, Wr)
        orb = O.row_linear_bwd(oY, Wr, dZr)
        ok.append(np.abs(Zr.numpy() - oZr).max() < 1e-12)
        ok.append(np.abs(gr["dXin"].numpy() - orb["dXin"][:, lo:hi]).max() < 1e-12)
        ok.append(np.abs(gr["dW"].numpy() - orb["dW"][lo:hi]).max() < 1e-12)
        q.put((rank, [bool(x) for x in ok]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_tp_dist_gloo_ranks_match_unsharded(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, oks in res:
        assert all(oks), (rank, oks)


def _failing_worker(rank, world, port, q):
    """Rank 1 fails between steps (raises before the forward, its process
    ends); rank 0 must learn of it from its next collective, which ends with
    an error within the process group's short timeout instead of waiting."""
    import time
    from datetime import timedelta

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=5))
    from linear_layers_b200 import tp_dist as D
    from oracle import tp_oracle as O

    comp = _Float64Shard(O)
    r = np.random.default_rng(3)
    X = torch.from_numpy(r.normal(size=(4, 8)))
    A_i = torch.from_numpy(r.normal(size=(8, 6)))
    B_i = torch.from_numpy(r.normal(size=(6, 8)))
    layer = D.TPMLP(A_i, None, B_i, compute=comp)
    layer.forward(X)                      # one good step on both ranks
    dist.barrier()
    if rank == 1:
        q.put((rank, "left", 0.0))
        q.close()
        q.join_thread()                   # the message is out before the process ends
        os._exit(3)                       # the failure: this rank is gone
    t0 = time.monotonic()
    try:
        layer.forward(X)
        q.put((rank, "no error", time.monotonic() - t0))
    except Exception as e:                # gloo: peer closed, or the timeout
        q.put((rank, type(e).__name__, time.monotonic() - t0))
    q.close()
    q.join_thread()
    os._exit(0)                           # the broken group is not torn down


def test_tp_dist_rank_failure_ends_the_next_collective_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        rank, what, secs = q.get(timeout=120)
        res[rank] = (what, secs)
    for p in procs:
        p.join(timeout=60)
    assert res[1][0] == "left"
    what, secs = res[0]
    assert what != "no error", "the surviving rank's all-reduce completed without its peer"
    assert secs < 30, secs                 # ended by the error, not by waiting for good
    assert procs[1].exitcode == 3


def test_shard_bounds_validation():
    from linear_layers_b200 import tp_dist as D

    assert D.shard_bounds(48, 3) == [0, 16, 32, 48]
    with pytest.raises(ValueError):
        D.shard_bounds(50, 3)
    with pytest.raises(ValueError):
        D.shard_bounds(48, 2, [0, 30, 20, 48])
    with pytest.raises(ValueError):
        D.shard_bounds(48, 2, [0, 48, 48])


@pytest.mark.gpu
def test_tp_dist_one_nccl_rank_on_the_gpu():
    """One NCCL rank on the GPU: the library's single-shard calls plus a real
    (one-member) all-reduce, against the oracle."""
    from datetime import timedelta

    import linear_layers_b200  # noqa: F401  (loads the library)
    from linear_layers_b200 import tp_dist as D
    from oracle import tp_oracle as O
    import tp_inputs
    from tests.gpu_helpers import TOL_BF16, assert_close

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60))
    try:
        inp = tp_inputs.mlp_inputs(300, 256, 1024, w_std=0.05, bias_std=0.02, seed=12)
        d = {k: v.cuda() for k, v in inp.items()}
        A_i, b_i, B_i = D.shard_mlp_weights(d["A"], d["bias"], d["B"], 0, 1)
        layer = D.TPMLP(A_i, b_i, B_i)
        Z, state = layer.forward(d["X"])
        g = layer.backward(d["X"], state, d["dZ"])
        torch.cuda.synchronize()
        _, _, oZ = O.mlp_fwd(inp["X"], inp["A"], inp["bias"], inp["B"])
        og = O.mlp_bwd(inp["X"], inp["A"], inp["bias"], inp["B"], inp["dZ"])
        assert_close("Z", Z, oZ, TOL_BF16)
        for k in ("dX", "dA", "dB", "dbias"):
            assert_close(k, g[k], og[k], TOL_BF16)
    finally:
        dist.destroy_process_group()
