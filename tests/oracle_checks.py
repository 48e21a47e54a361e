"""Checks that pin the fp64 oracle to facts outside itself.

Each ``check_*`` takes the oracle module and raises AssertionError when the
oracle disagrees with what the pages or the mathematics fix.  The pin tests
run every check on the real oracle; the mutation tests plant plausible
mistakes in the oracle and require at least one check to fail for each.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.linalg.norm(b), 1e-300)
    return float(np.linalg.norm(a - b) / den)


def _rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------
# GeLU
# ----------------------------------------------------------------------------
def check_gelu_erf_table(o):
    """x·Φ(x) at the textbook values of the normal CDF."""
    g = _golden("normal_cdf.json")
    x = np.array(g["x"])
    want = x * np.array(g["phi"])
    got = o.act_fwd(x, o.ACT_GELU_ERF)
    assert np.max(np.abs(got - want)) < 1e-15, (got, want)


def check_gelu_tanh_vs_erf(o):
    """The tanh closed form approximates x·Φ(x) to within 1e-3 on [-10, 10]
    (the measured gap of this approximation is 4.73e-4, at |x| ≈ 2.70)."""
    x = np.linspace(-10.0, 10.0, 200001)
    gap = np.max(np.abs(o.act_fwd(x, o.ACT_GELU_TANH) - o.act_fwd(x, o.ACT_GELU_ERF)))
    assert 1e-5 < gap < 1e-3, gap


def check_gelu_special_values(o):
    for act in (o.ACT_GELU_TANH, o.ACT_GELU_ERF):
        assert o.act_fwd(np.array([0.0]), act)[0] == 0.0
        assert abs(o.act_grad(np.array([0.0]), act)[0] - 0.5) < 1e-15
        big = o.act_fwd(np.array([10.0, -10.0]), act)
        assert abs(big[0] - 10.0) < 1e-12 and abs(big[1]) < 1e-12, big
        # gelu(x) - gelu(-x) = x for both forms (Φ(x) + Φ(-x) = 1, tanh odd)
        x = np.linspace(-6, 6, 1001)
        assert np.max(np.abs(o.act_fwd(x, act) - o.act_fwd(-x, act) - x)) < 1e-12
    # identity "activation"
    x = np.linspace(-3, 3, 7)
    assert np.array_equal(o.act_fwd(x, o.ACT_NONE), x)
    assert np.array_equal(o.act_grad(x, o.ACT_NONE), np.ones_like(x))


def check_gelu_derivative_fd(o):
    x = np.linspace(-8.0, 8.0, 3201)
    eps = 1e-6
    for act in (o.ACT_GELU_TANH, o.ACT_GELU_ERF):
        fd = (o.act_fwd(x + eps, act) - o.act_fwd(x - eps, act)) / (2 * eps)
        assert np.max(np.abs(fd - o.act_grad(x, act))) < 1e-8, act


# ----------------------------------------------------------------------------
# TP-MLP
# ----------------------------------------------------------------------------
def _tiny_mlp(seed=0, M=3, h=4, F=8):
    r = _rng(seed)
    return (r.normal(size=(M, h)), r.normal(size=(h, F)) * 0.5,
            r.normal(size=F) * 0.3, r.normal(size=(F, h)) * 0.5,
            r.normal(size=(M, h)))


def check_mlp_bruteforce_loops(o):
    """Z of the oracle against triple loops over scalars (act = NONE and the
    erf form, whose Φ comes from math.erf)."""
    X, A, b, B, _ = _tiny_mlp(1, M=3, h=4, F=6)
    M, h = X.shape
    F = A.shape[1]
    for act, fn in ((o.ACT_NONE, lambda u: u),
                    (o.ACT_GELU_ERF, lambda u: u * 0.5 * (1 + math.erf(u / math.sqrt(2))))):
        U = [[sum(X[m][k] * A[k][f] for k in range(h)) + b[f] for f in range(F)]
             for m in range(M)]
        Y = [[fn(U[m][f]) for f in range(F)] for m in range(M)]
        Z = [[sum(Y[m][f] * B[f][j] for f in range(F)) for j in range(h)]
             for m in range(M)]
        oU, oY, oZ = o.mlp_fwd(X, A, b, B, act)
        assert _rel(oU, U) < 1e-14 and _rel(oY, Y) < 1e-14 and _rel(oZ, Z) < 1e-14, act


def check_mlp_identity_closed_form(o):
    """With the identity activation Z = X·(A·B) + bias·B (re-associated)."""
    X, A, b, B, _ = _tiny_mlp(2, M=5, h=6, F=12)
    _, _, Z = o.mlp_fwd(X, A, b, B, o.ACT_NONE)
    AB = A @ B
    want = X @ AB + (b @ B)[None, :]
    assert _rel(Z, want) < 1e-13


def check_mlp_fd_gradients(o):
    """Central differences of L = Σ Z⊙dZ against dX, dA, dbias, dB
    (M=2, h=4, F=8, eps=1e-6)."""
    X, A, b, B, dZ = _tiny_mlp(3, M=2, h=4, F=8)
    eps = 1e-6
    for act in (o.ACT_GELU_TANH, o.ACT_GELU_ERF):
        g = o.mlp_bwd(X, A, b, B, dZ, act)

        def loss(X_, A_, b_, B_):
            return float((o.mlp_fwd(X_, A_, b_, B_, act)[2] * dZ).sum())

        for name, arr in (("dX", X), ("dA", A), ("dbias", b), ("dB", B)):
            fd = np.zeros_like(arr)
            it = np.nditer(arr, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                args = {"X": X, "A": A, "b": b, "B": B}
                key = {"dX": "X", "dA": "A", "dbias": "b", "dB": "B"}[name]
                plus = arr.copy()
                plus[idx] += eps
                minus = arr.copy()
                minus[idx] -= eps
                args[key] = plus
                lp = loss(args["X"], args["A"], args["b"], args["B"])
                args[key] = minus
                lm = loss(args["X"], args["A"], args["b"], args["B"])
                fd[idx] = (lp - lm) / (2 * eps)
            assert _rel(g[name], fd) < 1e-7, (act, name, _rel(g[name], fd))


def check_mlp_recompute(o):
    """Backward from the saved pre-activation alone: with U = X·A + bias it is
    the full backward; with a perturbed U it is the gradient at that U (torch
    autograd through Y = gelu(U) in float64 on the recomputed path)."""
    import torch

    X, A, b, B, dZ = _tiny_mlp(5, M=3, h=4, F=8)
    for act in (o.ACT_GELU_TANH, o.ACT_GELU_ERF, o.ACT_NONE):
        full = o.mlp_bwd(X, A, b, B, dZ, act)
        U = X @ A + b[None, :]
        rc = o.mlp_bwd_recompute(X, A, B, U, dZ, act)
        for k in ("dX", "dA", "dbias", "dB", "dU"):
            assert _rel(rc[k], full[k]) < 1e-15, (act, k)
    U2 = X @ A + b[None, :] + 0.3                       # any saved tensor
    Ut = torch.from_numpy(U2).requires_grad_(True)
    Bt = torch.from_numpy(B).requires_grad_(True)
    Yt = torch.nn.functional.gelu(Ut, approximate="tanh")
    ((Yt @ Bt) * torch.from_numpy(dZ)).sum().backward()
    rc = o.mlp_bwd_recompute(X, A, B, U2, dZ, o.ACT_GELU_TANH)
    assert _rel(rc["Y"], Yt.detach().numpy()) < 1e-15
    assert _rel(rc["dB"], Bt.grad.numpy()) < 1e-14
    assert _rel(rc["dU"], Ut.grad.numpy()) < 1e-14


def check_mlp_sharded_equals_unsharded(o):
    """Column split of A and row split of B with one all-reduce reproduce the
    unsharded layer exactly up to rounding (N = 1, 2, 4, 8 and uneven shards)."""
    X, A, b, B, dZ = _tiny_mlp(4, M=6, h=8, F=32)
    for act in (o.ACT_GELU_TANH, o.ACT_GELU_ERF, o.ACT_NONE):
        U, Y, Z = o.mlp_fwd(X, A, b, B, act)
        g = o.mlp_bwd(X, A, b, B, dZ, act)
        cases = [dict(N=n) for n in (1, 2, 4, 8)] + [dict(N=3, offsets=[0, 5, 19, 32])]
        for c in cases:
            s = o.mlp_fwd_sharded(X, A, b, B, c["N"], c.get("offsets"), act)
            assert _rel(s["Z"], Z) < 1e-12 and _rel(s["U"], U) < 1e-14 and _rel(s["Y"], Y) < 1e-14
            sb = o.mlp_bwd_sharded(X, A, b, B, dZ, c["N"], c.get("offsets"), act)
            for k in ("dX", "dA", "dB", "dbias", "dU"):
                assert _rel(sb[k], g[k]) < 1e-12, (act, c, k)
            # each partial is its shard's own product (not a share of the sum)
            offs = c.get("offsets") or o.even_offsets(32, c["N"])
            for i, Zi in enumerate(s["Zparts"]):
                lo, hi = offs[i], offs[i + 1]
                assert _rel(Zi, Y[:, lo:hi] @ B[lo:hi]) < 1e-13


def check_row_split_of_A_breaks_gelu(o):
    """Why A is split by columns: splitting A by rows (X by columns) and
    applying GeLU per shard before the sum does not give GeLU(X·A)."""
    X, A, b, B, _ = _tiny_mlp(5, M=4, h=8, F=8)
    full = o.act_fwd(X @ A, o.ACT_GELU_TANH)
    wrong = sum(o.act_fwd(X[:, i * 4:(i + 1) * 4] @ A[i * 4:(i + 1) * 4], o.ACT_GELU_TANH)
                for i in range(2))
    assert _rel(wrong, full) > 1e-2
    # column split: GeLU of each column block equals the block of GeLU
    blocks = np.concatenate([o.act_fwd(X @ A[:, i * 4:(i + 1) * 4], o.ACT_GELU_TANH)
                             for i in range(2)], axis=1)
    assert np.array_equal(blocks, full)


def check_apx_shape_example(o):
    g = _golden("apx_linear_shapes.json")
    r = _rng(6)
    x = r.normal(size=(g["batch"], g["in_features"]))
    W = r.normal(size=(g["in_features"], g["out_features"])) * 0.02
    _, full = o.col_linear_fwd(x, W)
    assert list(full.shape) == g["full_shape"]
    offs = o.even_offsets(g["out_features"], g["tp"])
    parts = [o.col_linear_fwd(x, W[:, offs[i]:offs[i + 1]])[1] for i in range(g["tp"])]
    for p in parts:
        assert list(p.shape) == g["shard_shape"]
    assert np.array_equal(np.concatenate(parts, axis=1), full)


def check_linear_blocks(o):
    """Column/row linear blocks: sharded == unsharded, gradients by FD."""
    r = _rng(7)
    X = r.normal(size=(5, 6))
    W = r.normal(size=(6, 10))
    b = r.normal(size=10)
    U, Y = o.col_linear_fwd(X, W, b, o.ACT_GELU_TANH)
    assert _rel(U, X @ W + b) < 1e-14
    dY = r.normal(size=U.shape)
    g = o.col_linear_bwd(X, W, U, dY, o.ACT_GELU_TANH)
    eps = 1e-6
    fdW = np.zeros_like(W)
    for i in range(W.shape[0]):
        for j in range(W.shape[1]):
            Wp, Wm = W.copy(), W.copy()
            Wp[i, j] += eps
            Wm[i, j] -= eps
            fdW[i, j] = ((o.col_linear_fwd(X, Wp, b, o.ACT_GELU_TANH)[1]
                          - o.col_linear_fwd(X, Wm, b, o.ACT_GELU_TANH)[1]) * dY).sum() / (2 * eps)
    assert _rel(g["dW"], fdW) < 1e-7
    fdX = np.zeros_like(X)
    for i in range(X.shape[0]):
        for j in range(X.shape[1]):
            Xp, Xm = X.copy(), X.copy()
            Xp[i, j] += eps
            Xm[i, j] -= eps
            fdX[i, j] = ((o.col_linear_fwd(Xp, W, b, o.ACT_GELU_TANH)[1]
                          - o.col_linear_fwd(Xm, W, b, o.ACT_GELU_TANH)[1]) * dY).sum() / (2 * eps)
    assert _rel(g["dX"], fdX) < 1e-7
    # row-parallel: sum of per-shard partials == unsharded product
    Xin = r.normal(size=(4, 12))
    Wr = r.normal(size=(12, 5))
    Z, _ = o.row_linear_fwd(Xin, Wr)
    Zs, parts = o.row_linear_fwd(Xin, Wr, offsets=[0, 7, 12])
    assert _rel(Zs, Z) < 1e-14 and len(parts) == 2
    dZ = r.normal(size=Z.shape)
    gb = o.row_linear_bwd(Xin, Wr, dZ)
    assert _rel(gb["dW"], np.einsum("mi,mj->ij", Xin, dZ)) < 1e-14
    assert _rel(gb["dXin"], np.einsum("mj,ij->mi", dZ, Wr)) < 1e-14


def _fd_grad(f, P, eps=1e-6):
    """Central differences of the scalar f() with respect to every entry of
    the array P (modified in place and restored)."""
    g = np.zeros_like(P)
    it = np.nditer(P, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        keep = P[i]
        P[i] = keep + eps
        fp = f()
        P[i] = keep - eps
        fm = f()
        P[i] = keep
        g[i] = (fp - fm) / (2 * eps)
    return g


def check_linear_bwd_fd(o):
    """Every gradient of the two linear blocks against central differences of
    L = Σ out ⊙ dOut ([TP-ILL] §1.1/§1.2: each shard's gradient is the local
    one, the f/g operators only sum or pass through):
    - col_linear_bwd: dbias (with a GeLU, so dbias = Σ_rows dY ⊙ act'(U)
      and not Σ_rows dY) and dU;
    - row_linear_bwd: dXin and dW of Z = Σ_i Xin_i·W_i over uneven shards."""
    r = _rng(71)
    X = r.normal(size=(5, 6))
    W = r.normal(size=(6, 10)) * 0.5
    b = r.normal(size=10)
    for act in (o.ACT_GELU_TANH, o.ACT_GELU_ERF, o.ACT_NONE):
        U, _ = o.col_linear_fwd(X, W, b, act)
        dY = r.normal(size=U.shape)
        g = o.col_linear_bwd(X, W, U, dY, act)
        L = lambda: float((o.col_linear_fwd(X, W, b, act)[1] * dY).sum())
        assert _rel(g["dbias"], _fd_grad(L, b)) < 1e-7, act
        # dU is the gradient with respect to the pre-activation itself
        Uw = U.copy()
        LU = lambda: float((o.act_fwd(Uw, act) * dY).sum())
        assert _rel(g["dU"], _fd_grad(LU, Uw)) < 1e-7, act
    Xin = r.normal(size=(4, 12))
    Wr = r.normal(size=(12, 5))
    dZ = r.normal(size=(4, 5))
    offs = [0, 7, 12]
    Lr = lambda: float((o.row_linear_fwd(Xin, Wr, offsets=offs)[0] * dZ).sum())
    gb = o.row_linear_bwd(Xin, Wr, dZ)
    assert _rel(gb["dXin"], _fd_grad(Lr, Xin)) < 1e-8
    assert _rel(gb["dW"], _fd_grad(Lr, Wr)) < 1e-8


def check_qkv_head_split(o):
    """25 heads over 4 shards -> 7, 6, 6, 6; shard-major columns are a
    permutation of [Q | K | V] and shard i's block holds exactly its heads."""
    perm, offs = o.qkv_shard_columns(25, 64, [7, 6, 6, 6])
    assert offs == [0, 7 * 192, 13 * 192, 19 * 192, 25 * 192]
    assert sorted(perm.tolist()) == list(range(3 * 1600))
    # shard 1 starts with Q of head 7, then its K block starts at Q-offset 1600 + 7*64
    s1 = perm[offs[1]:offs[2]]
    assert s1[0] == 7 * 64 and s1[6 * 64] == 1600 + 7 * 64 and s1[12 * 64] == 3200 + 7 * 64


# ----------------------------------------------------------------------------
# embedding
# ----------------------------------------------------------------------------
def check_embed_page_example(o):
    g = _golden("embed_vocab300_n2.json")
    v, N, ids = g["v"], g["N"], np.array(g["ids"])
    assert [[o.even_offsets(v, N)[i], o.even_offsets(v, N)[i + 1]] for i in range(N)] == g["shard_ranges"]
    assert o.embed_owner(ids, v, N).tolist() == g["owner"]
    # the ranges are half-open: each shard's first id is its own, its end id is the
    # next shard's (or nobody's past the table)
    edge = np.array([-1, 0, 149, 150, 299, 300])
    assert o.embed_owner(edge, v, N).tolist() == [-1, 0, 0, 1, 1, -1]
    E = _rng(8).normal(size=(v, 16))
    out = o.vp_embed_sharded(ids, E, N)
    for t, i in enumerate(ids):
        assert np.array_equal(out[t], E[i])


def check_embed_sharded_equals_lookup(o):
    import torch

    r = _rng(9)
    v, h = 96, 24
    E = r.normal(size=(v, h))
    ids = r.integers(0, v, size=50)
    ref = torch.nn.functional.embedding(torch.from_numpy(ids), torch.from_numpy(E)).numpy()
    assert np.array_equal(o.embed_lookup(ids, E), ref)
    for N in (1, 2, 3, 4, 8):
        assert np.array_equal(o.vp_embed_sharded(ids, E, N), ref), N
    bad = np.array([-1, v, 5])
    out = o.vp_embed_sharded(bad, E, 4)
    assert not out[0].any() and not out[1].any() and np.array_equal(out[2], E[5])
    assert np.array_equal(o.embed_lookup(bad, E), out)


# ----------------------------------------------------------------------------
# logits
# ----------------------------------------------------------------------------
def check_logits(o):
    import torch

    r = _rng(10)
    H = r.normal(size=(7, 16))
    E = r.normal(size=(40, 16))
    L = o.logits(H, E)
    ref = torch.nn.functional.linear(torch.from_numpy(H), torch.from_numpy(E)).numpy()
    assert _rel(L, ref) < 1e-14
    blocks = o.logits_sharded(H, E, 4)
    assert _rel(np.concatenate(blocks, axis=1), L) < 1e-15
    # brute force single entry
    assert abs(L[3, 17] - sum(H[3, k] * E[17, k] for k in range(16))) < 1e-12


# ----------------------------------------------------------------------------
# cross-entropy
# ----------------------------------------------------------------------------
def check_xent_uniform(o):
    """Equal logits: loss = log v, dlogits = 1/v − onehot."""
    v = 48
    L = np.full((3, v), 0.7)
    y = np.array([0, 17, 47])
    r = o.xent(L, y)
    assert np.max(np.abs(r["loss"] - math.log(v))) < 1e-13
    want = np.full((3, v), 1.0 / v)
    want[[0, 1, 2], y] -= 1.0
    assert np.max(np.abs(r["dlogits"] - want)) < 1e-15
    assert r["argmax"].tolist() == [0, 0, 0]


def check_xent_dominant(o):
    v = 32
    L = np.zeros((2, v))
    L[0, 5] = 1000.0
    L[1, 9] = 1000.0
    r = o.xent(L, np.array([5, 3]))
    assert abs(r["loss"][0]) < 1e-12 and abs(r["loss"][1] - 1000.0) < 1e-9
    assert r["argmax"].tolist() == [5, 9]


def check_xent_vs_torch(o):
    import torch

    r = _rng(11)
    L = r.normal(size=(9, 37)) * 2.0
    y = r.integers(0, 37, size=9)
    Lt = torch.from_numpy(L).requires_grad_(True)
    loss = torch.nn.functional.cross_entropy(Lt, torch.from_numpy(y), reduction="none")
    loss.sum().backward()
    got = o.xent(L, y, grad_scale=1.0)
    assert _rel(got["loss"], loss.detach().numpy()) < 1e-13
    assert abs(got["loss_sum"] - float(loss.detach().sum())) < 1e-12
    assert _rel(got["dlogits"], Lt.grad.numpy()) < 1e-13
    assert np.array_equal(got["argmax"], np.argmax(L, axis=1))
    got2 = o.xent(L, y, grad_scale=0.25)
    assert _rel(got2["dlogits"], 0.25 * Lt.grad.numpy()) < 1e-14


def check_xent_invariants(o):
    r = _rng(12)
    L = r.normal(size=(6, 50)) * 3
    y = r.integers(0, 50, size=6)
    a = o.xent(L, y)
    assert np.max(np.abs(a["dlogits"].sum(axis=1))) < 1e-14      # rows sum to 0
    b = o.xent(L + 123.0, y)                                       # shift invariance
    assert np.max(np.abs(a["loss"] - b["loss"])) < 1e-10
    eps = 1e-6                                                     # FD of loss_t
    for t in range(2):
        for j in (0, y[t], 49):
            Lp, Lm = L.copy(), L.copy()
            Lp[t, j] += eps
            Lm[t, j] -= eps
            fd = (o.xent(Lp, y)["loss"][t] - o.xent(Lm, y)["loss"][t]) / (2 * eps)
            assert abs(fd - a["dlogits"][t, j]) < 1e-8
    bad = o.xent(L[:2], np.array([-1, 50]))
    assert np.all(np.isnan(bad["loss"]))


def check_xent_sharded(o):
    r = _rng(13)
    v = 48
    L = r.normal(size=(11, v)) * 2
    y = r.integers(0, v, size=11)
    ref = o.xent(L, y, grad_scale=0.5)
    for N in (1, 2, 3, 4, 8):
        s = o.xent_sharded(L, y, N, grad_scale=0.5)
        assert _rel(s["loss"], ref["loss"]) < 1e-12, N
        assert abs(s["loss_sum"] - ref["loss_sum"]) < 1e-11
        assert _rel(s["dlogits"], ref["dlogits"]) < 1e-12
        assert np.array_equal(s["argmax"], ref["argmax"])
        assert _rel(np.log(s["S"]) + s["m"], ref["loss"] + L[np.arange(11), y]) < 1e-12


def check_xent_argmax_ties(o):
    """Equal maxima go to the lowest index, also across shard boundaries."""
    v = 16
    L = np.zeros((3, v))
    L[0, [3, 12]] = 5.0   # tie across shards (N=4: ranges of 4)
    L[1, [9, 10]] = 2.0   # tie inside one shard
    L[2, :] = -1.0        # all equal
    y = np.array([0, 0, 0])
    for fn in (lambda: o.xent(L, y), lambda: o.xent_sharded(L, y, 4)):
        assert fn()["argmax"].tolist() == [3, 9, 0]


# ----------------------------------------------------------------------------
# vocabulary-parallel backward
# ----------------------------------------------------------------------------
def check_logits_bwd_fd_through_xent(o):
    """dH, dE of L = Σ_t xent(H·Eᵀ)_t against central differences, and the
    sharded form (per-shard dH partials summed) equal to the unsharded one."""
    r = _rng(21)
    T, h, v = 3, 4, 12
    H = r.normal(size=(T, h))
    E = r.normal(size=(v, h)) * 0.5
    y = np.array([1, 7, 11])

    def loss(H_, E_):
        return float(o.xent(o.logits(H_, E_), y)["loss_sum"])

    G = o.xent(o.logits(H, E), y, grad_scale=1.0)["dlogits"]
    g = o.logits_bwd(G, H, E)
    eps = 1e-6
    for name, arr in (("dH", H), ("dE", E)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += eps
            m[idx] -= eps
            fd[idx] = ((loss(p, E) - loss(m, E)) if name == "dH" else (loss(H, p) - loss(H, m))) / (2 * eps)
        assert _rel(g[name], fd) < 1e-7, (name, _rel(g[name], fd))
    for N in (1, 2, 3, 4):
        s = o.logits_bwd_sharded(G, H, E, N)
        assert _rel(s["dH"], g["dH"]) < 1e-13 and _rel(s["dE"], g["dE"]) < 1e-14
        assert len(s["dHparts"]) == N


def check_embed_bwd_vs_torch(o):
    """Scatter-add of the embedding gradient against torch autograd (float64),
    with repeated ids, and the sharded accumulation equal to it."""
    import torch

    r = _rng(22)
    v, h = 40, 6
    ids = np.array([3, 17, 3, 39, 0, 17, 3, 25])
    G = r.normal(size=(ids.shape[0], h))
    E = torch.from_numpy(r.normal(size=(v, h))).requires_grad_(True)
    out = torch.nn.functional.embedding(torch.from_numpy(ids), E)
    (out * torch.from_numpy(G)).sum().backward()
    got = o.embed_bwd(ids, G, v)
    assert _rel(got, E.grad.numpy()) < 1e-15
    assert abs(got[3] - (G[0] + G[2] + G[6])).max() < 1e-15      # three repeats of id 3
    for N in (1, 2, 4, 5, 8):
        assert np.array_equal(o.embed_bwd_sharded(ids, G, v, N), got), N
    bad = o.embed_bwd(np.array([-1, 40, 2]), r.normal(size=(3, h)), v)
    assert not bad[:2].any() and bad[2].any() and not np.delete(bad, 2, axis=0).any()


def check_tied_embedding_grad(o):
    """One table used twice (input lookup and output logits): its gradient is
    the sum of both paths' gradients (torch autograd in float64)."""
    import torch

    r = _rng(23)
    v, h, T = 10, 4, 5
    ids = np.array([1, 4, 4, 9, 0])
    y = np.array([2, 4, 8, 0, 1])
    W = r.normal(size=(h, h)) * 0.7
    E = torch.from_numpy(r.normal(size=(v, h))).requires_grad_(True)
    x = torch.nn.functional.embedding(torch.from_numpy(ids), E)
    Hh = torch.tanh(x @ torch.from_numpy(W))            # any layer between the two uses
    L = torch.nn.functional.cross_entropy(Hh @ E.T, torch.from_numpy(y), reduction="sum")
    L.backward()
    Hn = Hh.detach().numpy()
    G = o.xent(o.logits(Hn, E.detach().numpy()), y)["dlogits"]
    g_out = o.logits_bwd(G, Hn, E.detach().numpy())
    # back through tanh(x W) to the looked-up rows
    dx = (g_out["dH"] * (1 - Hn ** 2)) @ W.T
    total = o.tied_embedding_grad(g_out["dE"], o.embed_bwd(ids, dx, v))
    assert _rel(total, E.grad.numpy()) < 1e-12


# ----------------------------------------------------------------------------
# output layer and loss together
# ----------------------------------------------------------------------------
def check_linear_xent_zero_hidden(o):
    """H = 0 makes every logit 0: loss = lse = log v, dlogits = 1/v − onehot,
    arg-max 0 (the lowest index of a v-way tie)."""
    v, h = 37, 6
    E = _rng(30).normal(size=(v, h))
    y = np.array([0, 36, 5])
    r = o.linear_xent(np.zeros((3, h)), E, y, grad_scale=2.0)
    assert np.allclose(r["loss"], math.log(v), rtol=0, atol=1e-14)
    assert np.allclose(r["lse"], math.log(v), rtol=0, atol=1e-14)
    want = np.full((3, v), 1.0 / v)
    want[np.arange(3), y] -= 1.0
    assert np.allclose(r["dlogits"], 2.0 * want, rtol=0, atol=1e-15)
    assert list(r["argmax"]) == [0, 0, 0]


def check_linear_xent_permutation_table(o):
    """E = c·P (a permutation that is not its own inverse, v = h) gives logits
    c·H[:, π]; torch's cross_entropy and logsumexp in float64 on those."""
    import torch

    h = 9
    perm = np.array([3, 0, 7, 1, 8, 2, 4, 6, 5])      # row j of E picks hidden unit perm[j]
    assert not np.array_equal(perm[perm], np.arange(h))
    c = 1.7
    E = np.zeros((h, h))
    E[np.arange(h), perm] = c
    H = _rng(31).normal(size=(6, h))
    y = np.array([0, 8, 3, 3, 5, 1])
    r = o.linear_xent(H, E, y, grad_scale=1.0)
    Lt = torch.from_numpy(c * H[:, perm])
    yt = torch.from_numpy(y)
    ref = torch.nn.functional.cross_entropy(Lt, yt, reduction="none").numpy()
    assert _rel(r["loss"], ref) < 1e-14
    assert _rel(r["lse"], torch.logsumexp(Lt, dim=1).numpy()) < 1e-14
    assert np.array_equal(r["argmax"], torch.argmax(Lt, dim=1).numpy())
    Lg = Lt.clone().requires_grad_(True)
    torch.nn.functional.cross_entropy(Lg, yt, reduction="sum").backward()
    assert _rel(r["dlogits"], Lg.grad.numpy()) < 1e-14


def check_linear_xent_bruteforce(o):
    """Scalar loops: loss_t = log Σ_j exp(Σ_k H_tk·E_jk) − Σ_k H_tk·E_{y_t,k}."""
    r = _rng(32)
    T, v, h = 3, 7, 5
    H = r.normal(size=(T, h))
    E = r.normal(size=(v, h))
    y = [4, 0, 6]
    got = o.linear_xent(H, E, np.array(y), grad_scale=0.5)
    for t in range(T):
        lt = [sum(H[t][k] * E[j][k] for k in range(h)) for j in range(v)]
        z = sum(math.exp(x) for x in lt)
        assert abs(got["lse"][t] - math.log(z)) < 1e-12
        assert abs(got["loss"][t] - (math.log(z) - lt[y[t]])) < 1e-12
        best = 0
        for j in range(1, v):
            if lt[j] > lt[best]:
                best = j
        assert got["argmax"][t] == best
        for j in range(v):
            want = 0.5 * (math.exp(lt[j]) / z - (1.0 if j == y[t] else 0.0))
            assert abs(got["dlogits"][t, j] - want) < 1e-13


def check_linear_xent_partitioned(o):
    """Any cut of the vocabulary (128-wide slices with a short tail, a single
    column, the whole range) combines to the unpartitioned loss; a maximum
    tied across a cut goes to the lower index."""
    r = _rng(33)
    T, v, h = 5, 300, 8
    H = r.normal(size=(T, h))
    E = r.normal(size=(v, h))
    y = np.array([0, 127, 128, 299, 150])
    ref = o.linear_xent(H, E, y, grad_scale=0.25)
    for offs in ([0, 128, 256, 300], [0, 1, 300], [0, 300], [0, 7, 8, 200, 299, 300]):
        got = o.linear_xent_partitioned(H, E, y, offs, grad_scale=0.25)
        assert _rel(got["loss"], ref["loss"]) < 1e-13, offs
        assert _rel(got["lse"], ref["lse"]) < 1e-13, offs
        assert _rel(got["dlogits"], ref["dlogits"]) < 1e-13, offs
        assert np.array_equal(got["argmax"], ref["argmax"]), offs
    # rows 40 and 200 of the table are equal: the tie straddles the cut at 128
    E2 = E.copy()
    E2[200] = E2[40] = 10.0 * H[2] / np.linalg.norm(H[2])
    tie = o.linear_xent_partitioned(H, E2, y, [0, 128, 256, 300])
    assert tie["argmax"][2] == 40
    assert o.linear_xent(H, E2, y)["argmax"][2] == 40


# ----------------------------------------------------------------------------
# attention core
# ----------------------------------------------------------------------------
def check_attention_vs_torch(o):
    """One head against torch's scaled_dot_product_attention in float64,
    causal and not, default and explicit scale."""
    import torch

    r = _rng(40)
    s, d = 9, 8
    Q, K, V = (r.normal(size=(s, d)) for _ in range(3))
    for causal in (True, False):
        for scale in (None, 0.3):
            O, lse = o.attention_head(Q, K, V, causal, scale)
            t = lambda x: torch.from_numpy(x)[None, None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                t(Q), t(K), t(V), is_causal=causal, scale=scale)[0, 0].numpy()
            assert _rel(O, ref) < 1e-14, (causal, scale)
            sc = 1 / math.sqrt(d) if scale is None else scale
            S = torch.from_numpy(Q @ K.T * sc)
            if causal:
                S = S.masked_fill(~torch.ones(s, s, dtype=torch.bool).tril(), float("-inf"))
            assert _rel(lse, torch.logsumexp(S, dim=1).numpy()) < 1e-14


def check_attention_bruteforce_and_closed_forms(o):
    """Scalar loops on a tiny head; constant V gives V back; zero scores give
    the running mean of V under the causal mask (row i averages rows 0..i)."""
    r = _rng(41)
    s, d = 5, 3
    Q, K, V = (r.normal(size=(s, d)) for _ in range(3))
    O, _ = o.attention_head(Q, K, V, causal=True, scale=0.7)
    for i in range(s):
        w = [math.exp(0.7 * sum(Q[i][k] * K[j][k] for k in range(d))) for j in range(i + 1)]
        for c in range(d):
            want = sum(w[j] * V[j][c] for j in range(i + 1)) / sum(w)
            assert abs(O[i, c] - want) < 1e-13
    Vc = np.tile(r.normal(size=(1, d)), (s, 1))
    assert np.allclose(o.attention_head(Q, K, Vc)[0], Vc, rtol=0, atol=1e-14)
    O0, lse0 = o.attention_head(np.zeros((s, d)), K, V, causal=True)
    want = np.cumsum(V, axis=0) / np.arange(1, s + 1)[:, None]
    assert _rel(O0, want) < 1e-14
    assert np.allclose(lse0, np.log(np.arange(1, s + 1)), rtol=0, atol=1e-14)


def check_attention_sharded_layout(o):
    """Shard-major QKV of uneven head shards: the per-shard core equals
    standard multi-head attention on the [Q | K | V] layout (torch, float64),
    batch rows kept apart."""
    import torch

    r = _rng(42)
    b, s, nh, hd = 2, 6, 5, 4
    shards = [2, 1, 1, 1]
    std = r.normal(size=(b * s, 3 * nh * hd))            # standard [Q | K | V], heads in order
    perm, offs = o.qkv_shard_columns(nh, hd, shards)
    ctx, lse = o.attention_sharded(std[:, perm], b, s, nh, hd, shards, causal=True)
    t = torch.from_numpy(std).view(b, s, 3, nh, hd).permute(2, 0, 3, 1, 4)   # [3, b, nh, s, hd]
    ref = torch.nn.functional.scaled_dot_product_attention(t[0], t[1], t[2], is_causal=True)
    ref = ref.permute(0, 2, 1, 3).reshape(b * s, nh * hd).numpy()
    assert _rel(ctx, ref) < 1e-14
    assert lse.shape == (b, nh, s)


# ----------------------------------------------------------------------------
# sequence-parallel dropout-add-LayerNorm
# ----------------------------------------------------------------------------
def check_philox_known_answers(o):
    """Philox4x32-10 against the generator's published known-answer vectors."""
    g = _golden("philox4x32_10_kat.json")
    for v in g["vectors"]:
        got = o.philox4x32_10(np.array([int(w, 16) for w in v["ctr"]], dtype=np.uint64),
                              np.array([int(w, 16) for w in v["key"]], dtype=np.uint64))
        assert ["%08x" % w for w in got] == v["out"], (v, got)


def check_dropout_mask_properties(o):
    """Keep fraction within 5 sigma of 1 − p; p = 0 keeps everything; the mask is a
    function of (seed, offset) alone; element e uses word e mod 4 of counter e div 4."""
    M, h, p = 511, 1001, 0.1
    k = o.dropout_keep(M, h, p, seed=1234, offset=7)
    n = M * h
    assert abs(k.mean() - (1 - p)) < 5 * math.sqrt(p * (1 - p) / n)
    assert o.dropout_keep(M, h, 0.0, 1234, 7).all()
    assert np.array_equal(k, o.dropout_keep(M, h, p, 1234, 7))
    assert not np.array_equal(k, o.dropout_keep(M, h, p, 1234, 8))
    assert not np.array_equal(k, o.dropout_keep(M, h, p, 1235, 7))
    thr = int(math.floor(p * 2 ** 32))
    flat = k.reshape(-1)
    # every word of the first 64 counters and of the last (partial) one, each counter
    # drawn on its own; h = 1001 makes rows start in the middle of a counter
    for q in list(range(64)) + [(n - 1) // 4]:
        w = o.philox4x32_10(np.array([q, 0, 7, 0], dtype=np.uint64), np.array([1234, 0], dtype=np.uint64))
        for j in range(4):
            if 4 * q + j < n:
                assert flat[4 * q + j] == (int(w[j]) >= thr), (q, j)


def check_layernorm_vs_torch(o):
    """Forward and backward of hs = residual + dropout(x + bias), y = LN(hs)
    against torch (float64 autograd) with the oracle's keep mask as input."""
    import torch

    r = _rng(50)
    M, h, p, eps = 6, 10, 0.25, 1e-5
    x, res, bias = r.normal(size=(M, h)), r.normal(size=(M, h)), r.normal(size=h)
    gamma, beta = 1 + 0.3 * r.normal(size=h), 0.2 * r.normal(size=h)
    f = o.dropout_add_layernorm(x, bias, res, gamma, beta, p, seed=3, offset=11, eps=eps)
    keep = torch.from_numpy(f["keep"].astype(np.float64))
    T = {k: torch.from_numpy(v).requires_grad_(True)
         for k, v in dict(x=x, res=res, bias=bias, gamma=gamma, beta=beta).items()}
    hs = T["res"] + keep * (T["x"] + T["bias"]) / (1 - p)
    y = torch.nn.functional.layer_norm(hs, (h,), T["gamma"], T["beta"], eps)
    assert _rel(f["hs"], hs.detach().numpy()) < 1e-15
    assert _rel(f["y"], y.detach().numpy()) < 1e-14
    dy, dhs = r.normal(size=(M, h)), r.normal(size=(M, h))
    (y * torch.from_numpy(dy)).sum().add((hs * torch.from_numpy(dhs)).sum()).backward()
    b = o.dropout_add_layernorm_bwd(dy, dhs, f["hs"], gamma, f["mean"], f["rstd"], f["keep"], p)
    for name, t in (("dx", "x"), ("dresidual", "res"), ("dbias", "bias"), ("dgamma", "gamma"),
                    ("dbeta", "beta")):
        assert _rel(b[name], T[t].grad.numpy()) < 1e-13, name
    assert f["keep"].any() and not f["keep"].all()


def check_layernorm_sequence_shards(o):
    """Each shard of token rows gives its own rows' gradients; the parameter
    gradients are the sum of the shards' partials (uneven last shard)."""
    r = _rng(51)
    M, h, p = 12, 8, 0.1
    x, res = r.normal(size=(M, h)), r.normal(size=(M, h))
    gamma, beta = 1 + 0.3 * r.normal(size=h), 0.2 * r.normal(size=h)
    f = o.dropout_add_layernorm(x, None, res, gamma, beta, p, seed=9, offset=0)
    dy = r.normal(size=(M, h))
    ref = o.dropout_add_layernorm_bwd(dy, None, f["hs"], gamma, f["mean"], f["rstd"], f["keep"], p)
    for N in (1, 3, 4):
        s = o.dropout_add_layernorm_bwd_sharded(dy, None, f["hs"], gamma, f["mean"], f["rstd"],
                                                f["keep"], p, N)
        for k in ref:
            assert _rel(s[k], ref[k]) < 1e-14, (N, k)


def check_attention_backward_vs_torch(o):
    """dQ, dK, dV of one head against torch autograd through
    scaled_dot_product_attention in float64, causal and not; and the sharded
    backward against autograd through the whole shard-major layout."""
    import torch

    r = _rng(43)
    s, d = 7, 4
    Q, K, V, dO = (r.normal(size=(s, d)) for _ in range(4))
    for causal in (True, False):
        for scale in (None, 0.4):
            T = [torch.from_numpy(x).requires_grad_(True) for x in (Q, K, V)]
            out = torch.nn.functional.scaled_dot_product_attention(
                *(t[None, None] for t in T), is_causal=causal, scale=scale)[0, 0]
            (out * torch.from_numpy(dO)).sum().backward()
            got = o.attention_head_bwd(Q, K, V, dO, causal, scale)
            for g, t in zip(got, T):
                assert _rel(g, t.grad.numpy()) < 1e-13, (causal, scale)
    b, s2, nh, hd = 2, 5, 3, 4
    shards = [2, 1]
    std = r.normal(size=(b * s2, 3 * nh * hd))
    perm, _ = o.qkv_shard_columns(nh, hd, shards)
    X = torch.from_numpy(std).requires_grad_(True)
    t = X.view(b, s2, 3, nh, hd).permute(2, 0, 3, 1, 4)
    ctx = torch.nn.functional.scaled_dot_product_attention(t[0], t[1], t[2], is_causal=True)
    ctx = ctx.permute(0, 2, 1, 3).reshape(b * s2, nh * hd)
    G = r.normal(size=(b * s2, nh * hd))
    (ctx * torch.from_numpy(G)).sum().backward()
    got = o.attention_sharded_bwd(std[:, perm], G, b, s2, nh, hd, shards, causal=True)
    assert _rel(got, X.grad.numpy()[:, perm]) < 1e-13


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
