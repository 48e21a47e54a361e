"""fp64 CPU oracle for Megatron-style tensor-parallel layers.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The CUDA path
in ``linear_layers_b200`` never imports it and shares no code with it.

Everything here is plain numpy in float64 (matrix products through ``@``,
element-wise maps through numpy ufuncs).  There is no blocking, fusion or
reordering beyond what the definitions below state.  Inputs arrive in their
storage dtype (bf16 / fp32 torch tensors or numpy arrays) and are widened
exactly to float64 before any arithmetic.

Sources (web pages on Megatron-LM tensor parallelism), cited by page title
and section:

* [MLP-TP] "Megatron-LM：张量并行与大规模训练" (astro-blog-cod.pages.dev),
  §2.1 "MLP 层的张量并行": Y = GeLU(XA)B with A [h,4h] split by columns,
  B [4h,h] split by rows, one all-reduce of the Z_i after the row GEMM;
  §2.2 "Self-Attention 的张量并行": per-shard heads, QKV column-split,
  output projection row-split followed by one all-reduce.
* [TP-ILL] 张量模型并行图解 page (m.youleyou.com/wenzhang/3143730),
  §1.1 "按行切分权重" and §1.2 "按列切分权重" (the f and g operators and
  their backward), §2.1 "MLP层的张量模型并行计算方法", §3.1
  "Multihead-Attention的计算方法", §4.1 "输入层Embedding", §4.2
  "输出层Embedding", §5 "Cross-Entropy层".
* [APX] "Megatron-LM 介绍" (apxml.com), §"核心贡献": column-parallel
  Y_i = X A_i and the Linear(1024→4096), TP=2 shape example.
* [FW] "Megatron-LM框架概览" page (5688vip.com, chapter 03), §3.2
  "核心特性": activation recompute drops activations and rebuilds them in
  the backward.
* [EVO] Megatron history page (discosf.com/news/5875844), §2.3
  "序列并行与激活重计算": recompute keeps only each layer's inputs, or
  selectively the costliest part of the MLP or attention.

Readings where the pages are silent or garbled (each also listed with the
design notes):

* GeLU has no formula on any page.  Default: the tanh closed form
  0.5·x·(1 + tanh(√(2/π)·(x + 0.044715·x³))); the erf form x·Φ(x) is the
  selectable alternative.
* No page has a bias.  A column bias [F] is added before the activation and
  is split with A's columns.
* The vocabulary split of §4.1's example is printed as [0,150) and
  [150,299) for v=300; read as contiguous half-open ranges
  [i·v/N, (i+1)·v/N).
* §5 sums raw exponentials; the per-shard maximum is subtracted first
  (mathematically equal, numerically safe).  The loss is returned per token
  and as the sum over tokens ("按行加总得到 scalar Loss").
* Ties in the arg-max go to the lowest vocabulary index.
* [EVO] §2.3 names sequence-parallel LayerNorm and Dropout without
  formulas; the plain reading is the transformer's residual step
  hs = residual + dropout(x + bias), y = LayerNorm(hs) (biased variance,
  eps = 1e-5) on each shard's token rows, with the parameter gradients
  summed over shards.  Dropout draws from Philox4x32-10 (its published
  definition), one 32-bit word per element, kept when the word is at least
  floor(p·2^32).
* The attention core's formula is an image lost from the pages; the plain
  reading is scaled dot-product attention softmax(Q·Kᵀ/√d)·V per head, with
  the causal mask of a decoder (the GPT-2 layer) selectable, and no dropout.

Pins (tests that hold this oracle to something other than itself) live in
``tests/test_oracle_pins.py`` and ``tests/test_oracle_mutations.py``.
No function here is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

ACT_NONE = 0
ACT_GELU_TANH = 1
ACT_GELU_ERF = 2

_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)
_GELU_CUBIC = 0.044715


# ----------------------------------------------------------------------------
# conversions
# ----------------------------------------------------------------------------
def f64(x) -> np.ndarray:
    """Widen a torch tensor (any float dtype, incl. bf16) or array to float64."""
    if hasattr(x, "detach"):  # torch tensor; bf16 has no numpy dtype
        import torch

        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


# ----------------------------------------------------------------------------
# activation (no page gives the formula; see module docstring)
# ----------------------------------------------------------------------------
def _erf(x: np.ndarray) -> np.ndarray:
    from scipy.special import erf

    return erf(x)


def act_fwd(u: np.ndarray, act: int) -> np.ndarray:
    if act == ACT_NONE:
        return u.copy()
    if act == ACT_GELU_TANH:
        inner = _SQRT_2_OVER_PI * (u + _GELU_CUBIC * u ** 3)
        return 0.5 * u * (1.0 + np.tanh(inner))
    if act == ACT_GELU_ERF:
        return 0.5 * u * (1.0 + _erf(u / math.sqrt(2.0)))
    raise ValueError(f"unknown activation {act}")


def act_grad(u: np.ndarray, act: int) -> np.ndarray:
    """d act(u) / du, element-wise."""
    if act == ACT_NONE:
        return np.ones_like(u)
    if act == ACT_GELU_TANH:
        t = np.tanh(_SQRT_2_OVER_PI * (u + _GELU_CUBIC * u ** 3))
        dinner = _SQRT_2_OVER_PI * (1.0 + 3.0 * _GELU_CUBIC * u ** 2)
        return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * dinner
    if act == ACT_GELU_ERF:
        cdf = 0.5 * (1.0 + _erf(u / math.sqrt(2.0)))
        pdf = np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
        return cdf + u * pdf
    raise ValueError(f"unknown activation {act}")


# ----------------------------------------------------------------------------
# shards
# ----------------------------------------------------------------------------
def even_offsets(total: int, N: int) -> list[int]:
    """Contiguous half-open ranges [i·total/N, (i+1)·total/N); needs N | total.

    [TP-ILL] §4.1 splits the vocabulary into contiguous ranges, one per GPU;
    [MLP-TP] §2.1 gives each GPU 1/N of A's columns ([h, 4h/N]).
    """
    if total % N:
        raise ValueError(f"{total} is not divisible by {N}")
    step = total // N
    return [i * step for i in range(N + 1)]


def all_reduce_sum(parts):
    """The all-reduce of the pages, written out: sum the N partials in shard order."""
    acc = np.array(parts[0], dtype=np.float64, copy=True)
    for p in parts[1:]:
        acc = acc + p
    return acc


# ----------------------------------------------------------------------------
# TP-MLP, unsharded definition  ([MLP-TP] §2.1; [TP-ILL] §2.1)
# ----------------------------------------------------------------------------
def mlp_fwd(X, A, bias, B, act=ACT_GELU_TANH):
    """U = X·A + bias, Y = act(U), Z = Y·B.   Returns (U, Y, Z) in fp64."""
    X, A, B = f64(X), f64(A), f64(B)
    U = X @ A
    if bias is not None:
        U = U + f64(bias)[None, :]
    Y = act_fwd(U, act)
    Z = Y @ B
    return U, Y, Z


def mlp_bwd(X, A, bias, B, dZ, act=ACT_GELU_TANH):
    """Gradient of L = Σ Z⊙dZ for Z = act(X·A + bias)·B.

    Returns dict(dX, dA, dbias, dB, dU, dY).  The forward is recomputed here
    in fp64 from the inputs.
    """
    X, A, B, dZ = f64(X), f64(A), f64(B), f64(dZ)
    U, Y, _ = mlp_fwd(X, A, bias, B, act)
    dY = dZ @ B.T
    dU = dY * act_grad(U, act)
    return {
        "dY": dY,
        "dU": dU,
        "dB": Y.T @ dZ,
        "dA": X.T @ dU,
        "dbias": dU.sum(axis=0),
        "dX": dU @ A.T,
    }


def mlp_bwd_recompute(X, A, B, U, dZ, act=ACT_GELU_TANH):
    """The same gradient when the forward kept only the pre-activation U.

    Activation recompute ([FW] §3.2, the recompute row of its feature table;
    [EVO] §2.3): the activation Y is dropped after the forward and rebuilt
    from the saved U when the backward needs it, Y = act(U); everything else
    is mlp_bwd.  ``U`` is taken as given (the saved tensor), so the result is
    the gradient at that U.
    """
    X, A, B, U, dZ = f64(X), f64(A), f64(B), f64(U), f64(dZ)
    Y = act_fwd(U, act)                      # recomputed, not stored
    dY = dZ @ B.T
    dU = dY * act_grad(U, act)
    return {
        "Y": Y,
        "dY": dY,
        "dU": dU,
        "dB": Y.T @ dZ,
        "dA": X.T @ dU,
        "dbias": dU.sum(axis=0),
        "dX": dU @ A.T,
    }


# ----------------------------------------------------------------------------
# TP-MLP, sharded algorithm with an explicit host all-reduce
# ([MLP-TP] §2.1 pseudocode; [TP-ILL] §1.1, §1.2 and §2.1 f/g operators)
# ----------------------------------------------------------------------------
def mlp_fwd_sharded(X, A, bias, B, N, offsets=None, act=ACT_GELU_TANH):
    """Per shard i: Y_i = act(X·A_i + bias_i), Z_i = Y_i·B_i; Z = all-reduce(Z_i).

    f forward is the identity (every shard sees the same X).  Returns
    dict(Z, Zparts, U, Y) with U, Y assembled from the shards' column blocks.
    """
    X, A, B = f64(X), f64(A), f64(B)
    F = A.shape[1]
    offs = even_offsets(F, N) if offsets is None else list(offsets)
    b = np.zeros(F) if bias is None else f64(bias)
    Zparts, Us, Ys = [], [], []
    for i in range(N):
        lo, hi = offs[i], offs[i + 1]
        Ui = X @ A[:, lo:hi] + b[None, lo:hi]
        Yi = act_fwd(Ui, act)
        Zparts.append(Yi @ B[lo:hi, :])
        Us.append(Ui)
        Ys.append(Yi)
    return {
        "Z": all_reduce_sum(Zparts),
        "Zparts": Zparts,
        "U": np.concatenate(Us, axis=1),
        "Y": np.concatenate(Ys, axis=1),
    }


def mlp_bwd_sharded(X, A, bias, B, dZ, N, offsets=None, act=ACT_GELU_TANH):
    """g backward = identity (dZ to every shard); local dA_i, dB_i, dbias_i;
    f backward = all-reduce of the N partials dX_i = dU_i·A_iᵀ."""
    X, A, B, dZ = f64(X), f64(A), f64(B), f64(dZ)
    F = A.shape[1]
    offs = even_offsets(F, N) if offsets is None else list(offsets)
    b = np.zeros(F) if bias is None else f64(bias)
    dXparts, dAs, dBs, dbs, dUs = [], [], [], [], []
    for i in range(N):
        lo, hi = offs[i], offs[i + 1]
        Ai, Bi = A[:, lo:hi], B[lo:hi, :]
        Ui = X @ Ai + b[None, lo:hi]
        Yi = act_fwd(Ui, act)
        dYi = dZ @ Bi.T
        dUi = dYi * act_grad(Ui, act)
        dBs.append(Yi.T @ dZ)
        dAs.append(X.T @ dUi)
        dbs.append(dUi.sum(axis=0))
        dUs.append(dUi)
        dXparts.append(dUi @ Ai.T)
    return {
        "dX": all_reduce_sum(dXparts),
        "dXparts": dXparts,
        "dA": np.concatenate(dAs, axis=1),
        "dB": np.concatenate(dBs, axis=0),
        "dbias": np.concatenate(dbs),
        "dU": np.concatenate(dUs, axis=1),
    }


# ----------------------------------------------------------------------------
# Linear building blocks ([TP-ILL] §1.1, §1.2; [APX] §核心贡献)
# ----------------------------------------------------------------------------
def col_linear_fwd(X, W, bias=None, act=ACT_NONE):
    """Column-parallel linear over all shards: U = X·W + bias, Y = act(U)."""
    X, W = f64(X), f64(W)
    U = X @ W
    if bias is not None:
        U = U + f64(bias)[None, :]
    return U, act_fwd(U, act)


def col_linear_bwd(X, W, U, dY, act=ACT_NONE):
    """dU = dY ⊙ act'(U); dW = Xᵀ·dU; dbias = Σ_rows dU; dX = dU·Wᵀ (the f sum)."""
    X, W, U, dY = f64(X), f64(W), f64(U), f64(dY)
    dU = dY * act_grad(U, act)
    return {"dU": dU, "dW": X.T @ dU, "dbias": dU.sum(axis=0), "dX": dU @ W.T}


def row_linear_fwd(Xin, W, offsets=None, N=None):
    """Row-parallel linear: Z = Σ_i Xin[:, lo_i:hi_i]·W[lo_i:hi_i, :] (the g sum).

    With no offsets this is the unsharded product Xin·W.
    Returns (Z, parts) where parts is None for the unsharded call.
    """
    Xin, W = f64(Xin), f64(W)
    if offsets is None and N is None:
        return Xin @ W, None
    offs = even_offsets(W.shape[0], N) if offsets is None else list(offsets)
    parts = [Xin[:, offs[i]:offs[i + 1]] @ W[offs[i]:offs[i + 1], :]
             for i in range(len(offs) - 1)]
    return all_reduce_sum(parts), parts


def row_linear_bwd(Xin, W, dZ):
    """g backward is the identity: dXin = dZ·Wᵀ (per shard columns), dW = Xinᵀ·dZ."""
    Xin, W, dZ = f64(Xin), f64(W), f64(dZ)
    return {"dXin": dZ @ W.T, "dW": Xin.T @ dZ}


def qkv_shard_columns(n_heads: int, head_dim: int, heads_per_shard):
    """Column permutation from the standard [Q | K | V] layout (heads in order
    inside each block) to the shard-major layout in which shard i holds its
    own Q heads, then its K heads, then its V heads ([MLP-TP] §2.2;
    [TP-ILL] §3.1: Q, K and V are column-split, one or more heads per GPU).

    Returns (perm, offsets): shard-major column j holds standard column
    perm[j]; shard i owns shard-major columns [offsets[i], offsets[i+1]).
    """
    hd = head_dim
    h = n_heads * hd
    perm, offsets, head0 = [], [0], 0
    for nh in heads_per_shard:
        for block in range(3):  # Q, K, V
            for hh in range(head0, head0 + nh):
                base = block * h + hh * hd
                perm.extend(range(base, base + hd))
        head0 += nh
        offsets.append(len(perm))
    if head0 != n_heads:
        raise ValueError("heads_per_shard does not cover all heads")
    return np.asarray(perm, dtype=np.int64), offsets


# ----------------------------------------------------------------------------
# Attention core between the projections ([MLP-TP] §2.2; [TP-ILL] §3.1)
# ----------------------------------------------------------------------------
def attention_head(Q, K, V, causal=True, scale=None):
    """One head of scaled dot-product attention over one sequence.

    O = softmax(Q·Kᵀ·scale + mask)·V with Q, K, V [s, d], scale = 1/√d by
    default and, when causal, position j masked out of row i for j > i (the
    decoder form of the GPT-2 layer).  Each row's softmax subtracts its
    maximum first.  Returns (O [s, d], lse [s]) with lse the natural-log
    sum of exp of the scaled, masked scores.
    """
    Q, K, V = f64(Q), f64(K), f64(V)
    s, d = Q.shape
    sc = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    S = (Q @ K.T) * sc
    if causal:
        S = np.where(np.tril(np.ones((s, K.shape[0]), dtype=bool)), S, -np.inf)
    m = S.max(axis=1)
    P = np.exp(S - m[:, None])
    l = P.sum(axis=1)
    return (P / l[:, None]) @ V, m + np.log(l)


def attention_sharded(QKV, b, s, n_heads, head_dim, heads_per_shard, causal=True, scale=None):
    """The attention core of the tensor-parallel layer, shard by shard.

    QKV [b·s, 3h] is the column-parallel projection's output in the
    shard-major layout (shard i: its Q heads, then its K heads, then its V
    heads; see qkv_shard_columns).  Each shard runs attention on its own heads
    with no communication; the context [b·s, h] keeps the heads in order,
    so shard i's block of columns is the input of its rows of the
    row-parallel output projection.  Returns (ctx, lse [b, n_heads, s]).
    """
    X = f64(QKV)
    hd = head_dim
    ctx = np.zeros((b * s, n_heads * hd))
    lse = np.zeros((b, n_heads, s))
    col, head = 0, 0
    for nh in heads_per_shard:
        q0, k0, v0 = col, col + nh * hd, col + 2 * nh * hd
        for j in range(nh):
            for bb in range(b):
                rows = slice(bb * s, (bb + 1) * s)
                O, L = attention_head(X[rows, q0 + j * hd:q0 + (j + 1) * hd],
                                      X[rows, k0 + j * hd:k0 + (j + 1) * hd],
                                      X[rows, v0 + j * hd:v0 + (j + 1) * hd], causal, scale)
                ctx[rows, (head + j) * hd:(head + j + 1) * hd] = O
                lse[bb, head + j] = L
        col += 3 * nh * hd
        head += nh
    if head != n_heads:
        raise ValueError("heads_per_shard does not cover all heads")
    return ctx, lse


def attention_head_bwd(Q, K, V, dO, causal=True, scale=None):
    """Gradient of one head of attention_head for the upstream gradient dO.

    With P = softmax(Q·Kᵀ·scale + mask) and O = P·V:
    dV = Pᵀ·dO,  dP = dO·Vᵀ,  dS = P ⊙ (dP − rowsum(dO ⊙ O)),
    dQ = scale·dS·K,  dK = scale·dSᵀ·Q.  Returns (dQ, dK, dV)."""
    Q, K, V, dO = f64(Q), f64(K), f64(V), f64(dO)
    s, d = Q.shape
    sc = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    S = (Q @ K.T) * sc
    if causal:
        S = np.where(np.tril(np.ones((s, K.shape[0]), dtype=bool)), S, -np.inf)
    P = np.exp(S - S.max(axis=1)[:, None])
    P = P / P.sum(axis=1)[:, None]
    O = P @ V
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - (dO * O).sum(axis=1)[:, None])
    return sc * dS @ K, sc * dS.T @ Q, dV


def attention_sharded_bwd(QKV, dctx, b, s, n_heads, head_dim, heads_per_shard, causal=True,
                          scale=None):
    """Backward of attention_sharded: each shard differentiates its own heads
    with no communication.  Returns dQKV [b·s, 3h] in the same shard-major
    layout as QKV (the upstream gradient of the column-parallel projection)."""
    X, G = f64(QKV), f64(dctx)
    hd = head_dim
    dX = np.zeros_like(X)
    col, head = 0, 0
    for nh in heads_per_shard:
        q0, k0, v0 = col, col + nh * hd, col + 2 * nh * hd
        for j in range(nh):
            cq = slice(q0 + j * hd, q0 + (j + 1) * hd)
            ck = slice(k0 + j * hd, k0 + (j + 1) * hd)
            cv = slice(v0 + j * hd, v0 + (j + 1) * hd)
            co = slice((head + j) * hd, (head + j + 1) * hd)
            for bb in range(b):
                rows = slice(bb * s, (bb + 1) * s)
                dq, dk, dv = attention_head_bwd(X[rows, cq], X[rows, ck], X[rows, cv],
                                                G[rows, co], causal, scale)
                dX[rows, cq], dX[rows, ck], dX[rows, cv] = dq, dk, dv
        col += 3 * nh * hd
        head += nh
    return dX


# ----------------------------------------------------------------------------
# Sequence-parallel dropout-add-LayerNorm ([EVO] §2.3: LayerNorm and Dropout
# split along the sequence, each shard handling its own token rows)
# ----------------------------------------------------------------------------
_PHILOX_M0, _PHILOX_M1 = 0xD2511F53, 0xCD9E8D57
_PHILOX_W0, _PHILOX_W1 = 0x9E3779B9, 0xBB67AE85
_U32 = 0xFFFFFFFF


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random
    numbers: as easy as 1, 2, 3", SC 2011).  ctr: uint32 array [..., 4], key:
    uint32 array [..., 2].  Each round multiplies words 0 and 2 by the two
    constants, crosses the high halves with words 1 and 3 and the key, and
    bumps the key by the two Weyl constants.  Returns uint32 [..., 4]."""
    c = np.asarray(ctr, dtype=np.uint64) & _U32
    k = np.asarray(key, dtype=np.uint64) & _U32
    c0, c1, c2, c3 = (c[..., i].copy() for i in range(4))
    k0, k1 = k[..., 0].copy(), k[..., 1].copy()
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _PHILOX_W0) & _U32
            k1 = (k1 + _PHILOX_W1) & _U32
        p0 = c0 * _PHILOX_M0                      # exact in uint64
        p1 = c2 * _PHILOX_M1
        hi0, lo0 = p0 >> 32, p0 & _U32
        hi1, lo1 = p1 >> 32, p1 & _U32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def dropout_keep(M, h, p, seed, offset):
    """Keep mask [M, h] of dropout with drop probability p.

    Element e = row·h + col draws word e mod 4 of Philox4x32-10 at counter
    (e div 4 as two 32-bit words, offset as two 32-bit words) under key
    seed (two 32-bit words); it is kept when that word u satisfies
    u >= floor(p·2^32), so the keep probability is 1 − p to 2^-32.
    """
    n = M * h
    q = np.arange((n + 3) // 4, dtype=np.uint64)
    ctr = np.stack([q & _U32, q >> 32, np.full_like(q, offset & _U32),
                    np.full_like(q, (offset >> 32) & _U32)], axis=-1)
    key = np.broadcast_to(np.array([seed & _U32, (seed >> 32) & _U32], dtype=np.uint64),
                          (q.size, 2))
    words = philox4x32_10(ctr, key).reshape(-1)[:n]
    thr = np.uint64(int(math.floor(p * 2.0 ** 32)))
    return (words.astype(np.uint64) >= thr).reshape(M, h)


def dropout_add_layernorm(x, bias, residual, gamma, beta, p, seed, offset, eps=1e-5):
    """Forward: hs = residual + keep·(x + bias)/(1 − p);  y = LayerNorm(hs)·gamma + beta,
    the LayerNorm over the hidden dimension with the biased variance.
    Returns dict(hs, y, mean, rstd, keep)."""
    x, residual, gamma, beta = f64(x), f64(residual), f64(gamma), f64(beta)
    M, h = x.shape
    keep = dropout_keep(M, h, p, seed, offset)
    xb = x + (f64(bias)[None, :] if bias is not None else 0.0)
    hs = residual + np.where(keep, xb / (1.0 - p), 0.0)
    mean = hs.mean(axis=1)
    var = ((hs - mean[:, None]) ** 2).mean(axis=1)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (hs - mean[:, None]) * rstd[:, None]
    return {"hs": hs, "y": xhat * gamma[None, :] + beta[None, :], "mean": mean, "rstd": rstd,
            "keep": keep}


def dropout_add_layernorm_bwd(dy, dhs_in, hs, gamma, mean, rstd, keep, p):
    """Backward of dropout_add_layernorm.  dy: gradient at y; dhs_in
    (nullable): gradient reaching the residual stream hs from later layers.
    Returns dict(dx, dresidual, dbias, dgamma, dbeta)."""
    dy, hs, gamma = f64(dy), f64(hs), f64(gamma)
    xhat = (hs - f64(mean)[:, None]) * f64(rstd)[:, None]
    g = dy * gamma[None, :]
    dh = f64(rstd)[:, None] * (g - g.mean(axis=1, keepdims=True)
                               - xhat * (g * xhat).mean(axis=1, keepdims=True))
    if dhs_in is not None:
        dh = dh + f64(dhs_in)
    dx = np.where(keep, dh / (1.0 - p), 0.0)
    return {"dx": dx, "dresidual": dh, "dbias": dx.sum(axis=0),
            "dgamma": (dy * xhat).sum(axis=0), "dbeta": dy.sum(axis=0)}


def dropout_add_layernorm_bwd_sharded(dy, dhs_in, hs, gamma, mean, rstd, keep, p, N):
    """The sequence-parallel backward: shard i owns token rows [i·M/N, (i+1)·M/N)
    and computes its rows' gradients and its partial dgamma, dbeta, dbias;
    the parameter gradients are the all-reduce of the shards' partials."""
    M = f64(dy).shape[0]
    offs = even_offsets(M, N)
    parts = []
    for i in range(N):
        r = slice(offs[i], offs[i + 1])
        parts.append(dropout_add_layernorm_bwd(
            f64(dy)[r], None if dhs_in is None else f64(dhs_in)[r], f64(hs)[r], gamma,
            f64(mean)[r], f64(rstd)[r], keep[r], p))
    out = {k: np.concatenate([q[k] for q in parts], axis=0) for k in ("dx", "dresidual")}
    for k in ("dbias", "dgamma", "dbeta"):
        out[k] = all_reduce_sum([q[k] for q in parts])
    return out


# ----------------------------------------------------------------------------
# Vocabulary-parallel embedding ([TP-ILL] §4.1)
# ----------------------------------------------------------------------------
def embed_lookup(ids, E):
    """Plain row lookup out[t] = E[id_t]; ids outside [0, v) give a zero row."""
    ids, E = i64(ids), f64(E)
    v, h = E.shape
    out = np.zeros((ids.shape[0], h))
    ok = (ids >= 0) & (ids < v)
    out[ok] = E[ids[ok]]
    return out


def vp_embed_sharded(ids, E, N):
    """Each shard looks up the ids inside its vocabulary range and writes a
    zero row for the rest; the N partial outputs are then all-reduced."""
    ids, E = i64(ids), f64(E)
    v, h = E.shape
    offs = even_offsets(v, N)
    parts = []
    for i in range(N):
        lo, hi = offs[i], offs[i + 1]
        Ei = E[lo:hi]
        mine = (ids >= lo) & (ids < hi)
        part = np.zeros((ids.shape[0], h))
        part[mine] = Ei[ids[mine] - lo]
        parts.append(part)
    return all_reduce_sum(parts)


def embed_owner(ids, v, N):
    """Index of the shard whose vocabulary range holds each id (-1 if none)."""
    ids = i64(ids)
    offs = even_offsets(v, N)
    own = np.full(ids.shape, -1, dtype=np.int64)
    for i in range(N):
        own[(ids >= offs[i]) & (ids < offs[i + 1])] = i
    return own


# ----------------------------------------------------------------------------
# Output embedding / logits ([TP-ILL] §4.2)
# ----------------------------------------------------------------------------
def logits(H, E):
    """logits = H·Eᵀ (shared word-embedding table E [v,h])."""
    return f64(H) @ f64(E).T


def logits_sharded(H, E, N):
    """Shard i computes H·E_iᵀ for its vocabulary rows; the blocks sit side by side."""
    H, E = f64(H), f64(E)
    offs = even_offsets(E.shape[0], N)
    return [H @ E[offs[i]:offs[i + 1]].T for i in range(N)]


# ----------------------------------------------------------------------------
# Vocabulary-parallel softmax cross-entropy ([TP-ILL] §5)
# ----------------------------------------------------------------------------
def xent(logits_, targets, grad_scale=1.0):
    """Unsharded softmax cross-entropy per row.

    loss_t = log Σ_j exp(l_tj) − l_t,y_t;  loss_sum = Σ_t loss_t;
    dlogits = grad_scale · (softmax(l_t) − onehot(y_t));
    argmax_t = smallest j with l_tj = max_j l_tj.
    Targets outside [0, v) give loss NaN and a dlogits row of NaN.
    """
    L = f64(logits_)
    y = i64(targets)
    T, v = L.shape
    m = L.max(axis=1)
    lse = m + np.log(np.exp(L - m[:, None]).sum(axis=1))
    ok = (y >= 0) & (y < v)
    tgt = np.full(T, np.nan)
    tgt[ok] = L[np.nonzero(ok)[0], y[ok]]
    loss = lse - tgt
    p = np.exp(L - lse[:, None])
    d = p.copy()
    d[np.nonzero(ok)[0], y[ok]] -= 1.0
    d[~ok] = np.nan
    return {
        "loss": loss,
        "loss_sum": loss.sum(),
        "dlogits": grad_scale * d,
        "argmax": np.argmax(L, axis=1).astype(np.int64),  # first maximum
        "lse": lse,
    }


def xent_sharded(logits_, targets, N, grad_scale=1.0, offsets=None):
    """The vocabulary-parallel algorithm of [TP-ILL] §5, written out per shard.

    Shard i holds columns [lo_i, hi_i): the even split [i·v/N, (i+1)·v/N) of
    §4.1, or the boundaries ``offsets`` (N+1 increasing column indices from 0
    to v) when given.  It computes its maximum m_i, its sum
    s_i = Σ exp(l − m_i), its masked target logit and its local arg-max; the
    all-reduce combines m = max m_i, S = Σ s_i·exp(m_i − m) and the target
    logit; every shard then forms its own block of softmax − onehot and its
    share of the loss, and a last all-reduce sums the per-shard loss scalars.
    """
    L = f64(logits_)
    y = i64(targets)
    T, v = L.shape
    offs = even_offsets(v, N) if offsets is None else [int(o) for o in offsets]
    assert len(offs) == N + 1 and offs[0] == 0 and offs[-1] == v
    ms, ss, tg, amax_i, amax_v = [], [], [], [], []
    for i in range(N):
        Li = L[:, offs[i]:offs[i + 1]]
        mi = Li.max(axis=1)
        ms.append(mi)
        ss.append(np.exp(Li - mi[:, None]).sum(axis=1))
        mine = (y >= offs[i]) & (y < offs[i + 1])
        t = np.zeros(T)
        t[mine] = Li[np.nonzero(mine)[0], y[mine] - offs[i]]
        tg.append(t)
        amax_i.append(np.argmax(Li, axis=1) + offs[i])
        amax_v.append(mi)
    # all-reduce (max) of the maxima, then (sum) of the rescaled sums
    m = ms[0].copy()
    for mi in ms[1:]:
        m = np.maximum(m, mi)
    S = all_reduce_sum([ss[i] * np.exp(ms[i] - m) for i in range(N)])
    tgt = all_reduce_sum(tg)
    ok = (y >= 0) & (y < v)
    tgt[~ok] = np.nan
    lse = m + np.log(S)
    loss = lse - tgt
    dblocks, loss_parts = [], []
    for i in range(N):
        Li = L[:, offs[i]:offs[i + 1]]
        d = np.exp(Li - lse[:, None])
        mine = (y >= offs[i]) & (y < offs[i + 1])
        d[np.nonzero(mine)[0], y[mine] - offs[i]] -= 1.0
        d[~ok] = np.nan
        dblocks.append(grad_scale * d)
        loss_parts.append(np.where(mine, loss, 0.0).sum())
    # arg-max across shards: larger value wins, equal values go to the lower shard
    best_v = amax_v[0].copy()
    best_i = amax_i[0].copy()
    for i in range(1, N):
        better = amax_v[i] > best_v
        best_v = np.where(better, amax_v[i], best_v)
        best_i = np.where(better, amax_i[i], best_i)
    return {
        "loss": loss,
        "loss_sum": all_reduce_sum([np.array(x) for x in loss_parts]),
        "dlogits": np.concatenate(dblocks, axis=1),
        "argmax": best_i.astype(np.int64),
        "m": m,
        "S": S,
        "lse": lse,
    }


# ----------------------------------------------------------------------------
# Output layer and loss together ([TP-ILL] §4.2 followed by §5)
# ----------------------------------------------------------------------------
def linear_xent(H, E, targets, grad_scale=1.0):
    """Softmax cross-entropy of the output-layer logits l = H·Eᵀ.

    The result is defined by the two steps in sequence: the logits of §4.2
    (vocabulary rows of the shared table E against the hidden states H), then
    §5's loss on them.  Returns xent's outputs, among them the per-token
    log-sum-exp lse_t = log Σ_j exp(l_tj) that the gradient
    grad_scale·(exp(l − lse) − onehot(y)) is formed from.
    """
    return xent(logits(H, E), targets, grad_scale)


def linear_xent_partitioned(H, E, targets, offsets, grad_scale=1.0):
    """The same loss with the vocabulary cut at ``offsets`` (any increasing
    column boundaries, not only an even split): per-part maxima, rescaled
    sums and target logits combined by §5's rule."""
    return xent_sharded(logits(H, E), targets, len(offsets) - 1, grad_scale, offsets=offsets)


# ----------------------------------------------------------------------------
# Vocabulary-parallel backward ([TP-ILL] §4.2: the output layer shares the
# word embedding with the input layer; the table's gradient is the sum of the
# two layers' gradients)
# ----------------------------------------------------------------------------
def logits_bwd(dlogits, H, E):
    """Backward of logits = H·Eᵀ:  dH = dlogits·E,  dE = dlogitsᵀ·H."""
    G, H, E = f64(dlogits), f64(H), f64(E)
    return {"dH": G @ E, "dE": G.T @ H}


def logits_bwd_sharded(dlogits, H, E, N):
    """Shard i owns vocabulary rows [lo_i, hi_i): dE_i = dlogits_iᵀ·H is local,
    dH = Σ_i dlogits_i·E_i is the all-reduce of the shards' partials."""
    G, H, E = f64(dlogits), f64(H), f64(E)
    offs = even_offsets(E.shape[0], N)
    parts = [G[:, offs[i]:offs[i + 1]] @ E[offs[i]:offs[i + 1]] for i in range(N)]
    dE = np.concatenate([G[:, offs[i]:offs[i + 1]].T @ H for i in range(N)], axis=0)
    return {"dH": all_reduce_sum(parts), "dHparts": parts, "dE": dE}


def embed_bwd(ids, dout, v):
    """Gradient of out[t] = E[id_t] with respect to E: row x of the result is
    the sum of dout[t] over the tokens with id_t = x (ids outside [0, v)
    contribute nothing)."""
    ids, G = i64(ids), f64(dout)
    dE = np.zeros((v, G.shape[1]))
    ok = (ids >= 0) & (ids < v)
    np.add.at(dE, ids[ok], G[ok])
    return dE


def embed_bwd_sharded(ids, dout, v, N):
    """Each shard accumulates the gradient rows of the ids in its own range."""
    ids, G = i64(ids), f64(dout)
    offs = even_offsets(v, N)
    blocks = []
    for i in range(N):
        lo, hi = offs[i], offs[i + 1]
        blk = np.zeros((hi - lo, G.shape[1]))
        mine = (ids >= lo) & (ids < hi)
        np.add.at(blk, ids[mine] - lo, G[mine])
        blocks.append(blk)
    return np.concatenate(blocks, axis=0)


def tied_embedding_grad(dE_output, dE_input):
    """The shared table's gradient: output-layer part plus input-layer part."""
    return f64(dE_output) + f64(dE_input)
