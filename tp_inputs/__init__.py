"""Seeded synthetic inputs shared by the GPU tests, the oracle tests and bench.py.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the layers' arithmetic, so both the CUDA path and the fp64
oracle can consume its output without sharing any method code.

Recipe (one generator per call, ``torch.Generator('cpu').manual_seed(seed)``):

* TP-MLP: draws in the fixed order X, A, bias, B, dZ.  Each is drawn in fp32
  with ``torch.randn`` and scaled by its standard deviation, then rounded to
  the storage dtype (round-to-nearest-even).  The same storage bits go to the
  GPU and, widened exactly to fp64, to the oracle.
* Vocabulary path: draws in the order ids, E, H, targets.  ids and targets are
  uniform integers in [0, v) (two independent draws); E ~ N(0, e_std) and
  H ~ N(0, 1) in bf16.
* Cross-entropy logits drawn directly (for parity of the loss kernel on its
  own): fp32 N(0, logit_std); the default 1.28 is the spread of H·Eᵀ with
  H ~ N(0,1), E ~ N(0,0.02), h = 4096 (sqrt(4096)·0.02).
"""
from __future__ import annotations

import torch

__all__ = [
    "mlp_inputs",
    "vocab_inputs",
    "xent_logits",
    "attn_proj_inputs",
    "vocab_bwd_inputs",
    "head_split",
    "WORKLOADS",
]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, std, dtype):
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def mlp_inputs(M, h, F, *, dtype=torch.bfloat16, w_std=0.02, x_std=1.0,
               bias_std=0.0, dz_std=1.0, seed=0):
    """X [M,h], A [h,F], bias [F], B [F,h], dZ [M,h] in ``dtype``.

    bias_std == 0 gives an all-zero bias (the timing configuration); the
    draw for it is still made so the later draws do not depend on it.
    """
    g = _gen(seed)
    X = _randn(g, (M, h), x_std, dtype)
    A = _randn(g, (h, F), w_std, dtype)
    bias = _randn(g, (F,), bias_std if bias_std > 0 else 1.0, dtype)
    if bias_std == 0:
        bias.zero_()
    B = _randn(g, (F, h), w_std, dtype)
    dZ = _randn(g, (M, h), dz_std, dtype)
    return {"X": X, "A": A, "bias": bias, "B": B, "dZ": dZ}


def vocab_inputs(T, v, h, *, e_std=0.02, seed=0, id_dtype=torch.int64):
    """ids [T] int64, E [v,h] bf16, H [T,h] bf16, targets [T] int64."""
    g = _gen(seed)
    ids = torch.randint(0, v, (T,), generator=g, dtype=id_dtype)
    E = _randn(g, (v, h), e_std, torch.bfloat16)
    H = _randn(g, (T, h), 1.0, torch.bfloat16)
    targets = torch.randint(0, v, (T,), generator=g, dtype=id_dtype)
    return {"ids": ids, "E": E, "H": H, "targets": targets}


def xent_logits(T, v, *, logit_std=1.28, seed=0):
    """fp32 logits [T,v] ~ N(0, logit_std) and targets [T] uniform in [0,v)."""
    g = _gen(seed)
    logits = _randn(g, (T, v), logit_std, torch.float32)
    targets = torch.randint(0, v, (T,), generator=g, dtype=torch.int64)
    return {"logits": logits, "targets": targets}


def vocab_bwd_inputs(T, v, h, *, seed=0, dlogit_std=1e-4):
    """Inputs of the vocabulary backward: dlogits [T,v] bf16 ~ N(0, dlogit_std),
    dout [T,h] bf16 ~ N(0,1) (gradient at the embedding output), dE0 [v,h]
    fp32 ~ N(0, 1e-3) (a gradient the scatter-add accumulates onto), ids [T]
    uniform in [0, v)."""
    g = _gen(seed)
    dlogits = _randn(g, (T, v), dlogit_std, torch.bfloat16)
    dout = _randn(g, (T, h), 1.0, torch.bfloat16)
    dE0 = _randn(g, (v, h), 1e-3, torch.float32)
    ids = torch.randint(0, v, (T,), generator=g, dtype=torch.int64)
    return {"dlogits": dlogits, "dout": dout, "dE0": dE0, "ids": ids}


def head_split(n_heads: int, N: int):
    """Contiguous uneven split of ``n_heads`` heads over N shards.

    Shard i gets floor(n_heads/N) heads plus one more while i < n_heads mod N
    (25 heads over 4 shards -> 7, 6, 6, 6).  This is a pure partition of
    integers, used to size the inputs; it carries no layer arithmetic.
    """
    base, extra = divmod(n_heads, N)
    return [base + (1 if i < extra else 0) for i in range(N)]


def attn_proj_inputs(M, h, n_heads, head_dim, N, *, dtype=torch.bfloat16,
                     w_std=0.02, seed=0):
    """Inputs of the attention projections with per-shard heads.

    X [M,h]; Wqkv [h, 3h] stored shard-major (shard i's columns are its
    Q heads, then its K heads, then its V heads); bqkv [3h] zeros;
    ctx [M, h] (the per-shard attention context, synthetic because the
    attention core itself is not on this path); Wo [h, h] (rows split like
    ctx's columns); dQKV [M, 3h] and dZ [M, h] upstream gradients.
    """
    g = _gen(seed)
    X = _randn(g, (M, h), 1.0, dtype)
    Wqkv = _randn(g, (h, 3 * n_heads * head_dim), w_std, dtype)
    bqkv = torch.zeros(3 * n_heads * head_dim, dtype=dtype)
    ctx = _randn(g, (M, n_heads * head_dim), 1.0, dtype)
    Wo = _randn(g, (n_heads * head_dim, h), w_std, dtype)
    dQKV = _randn(g, (M, 3 * n_heads * head_dim), 1.0, dtype)
    dZ = _randn(g, (M, h), 1.0, dtype)
    return {"X": X, "Wqkv": Wqkv, "bqkv": bqkv, "ctx": ctx, "Wo": Wo,
            "dQKV": dQKV, "dZ": dZ}


# The workloads the tests and the benchmark draw from (sizes only).
WORKLOADS = {
    # tiny fp32 MLP: b=2, s=8, h=64, ffn=256, N=2
    "mlp_tiny_fp32": dict(M=16, h=64, F=256, N=2, dtype=torch.float32,
                          w_std=0.02, x_std=0.02, bias_std=0.0),
    # b=8, s=512, h=1024, ffn=4096, N=8
    "mlp_h1024": dict(M=4096, h=1024, F=4096, N=8, dtype=torch.bfloat16,
                      w_std=0.02, bias_std=0.0),
    # GPT-2 1.5B layer slice: b=4, s=1024, h=1600, 25 heads, ffn=6400, N=4
    "gpt2_1p5b_slice": dict(M=4096, h=1600, F=6400, N=4, n_heads=25,
                            head_dim=64, dtype=torch.bfloat16, w_std=0.02,
                            bias_std=0.0),
    # b=2, s=2048, h=4096, ffn=16384, N=8 (headline roofline shape)
    "mlp_h4096": dict(M=4096, h=4096, F=16384, N=8, dtype=torch.bfloat16,
                      w_std=0.006, bias_std=0.0),
    # vocab path: b=8, s=2048, v=50304 over N=8, h=4096
    "vocab_v50304": dict(T=16384, v=50304, h=4096, N=8, e_std=0.02),
}
