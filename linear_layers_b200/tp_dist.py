"""Tensor parallelism over several GPUs: shard i of a layer on rank i.

The single-GPU entry points keep all N shards of a layer on one device and
fuse the shard sums into the kernels.  This module places ONE shard per
rank instead, as the pages lay the method out ([MLP-TP] §2.1, the forward
pseudocode that all-reduces Y_i·B_i; [TP-ILL] §2.2, one all-reduce of Z in
the forward and one of dX in the backward, 2·b·s·h elements each):

  rank i holds   A_i = A[:, off_i:off_{i+1}], bias_i, B_i = B[off_i:off_{i+1}, :]
  forward        U_i, Y_i, Z_i = library call on shard i (N = 1)
                 Z = all_reduce(Z_i)                       (the g operator)
  backward       dU_i, dA_i, dbias_i, dB_i, dX_i = library call on shard i
                 dX = all_reduce(dX_i)                     (the f operator)

The per-shard arithmetic is the library's single-shard call (every step in
its sm_100a kernels); torch.distributed supplies the all-reduce (NCCL on
GPUs).  The partials travel in the activation dtype (bf16), as the
reference design does; no TMA load of this path reads another GPU's memory.

The per-shard compute is a parameter (`compute`): LibraryShard (the
default) runs the library on the rank's GPU; tests pass a CPU stand-in so
that the partitioning and the collectives run on gloo ranks without a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

ACT_NONE, ACT_GELU_TANH, ACT_GELU_ERF = 0, 1, 2


def shard_bounds(total: int, world: int, offsets=None):
    """Offsets [off_0 = 0, ..., off_world = total] of the contiguous shards
    (the even split unless given; the even split needs total % world == 0)."""
    if offsets is None:
        if total % world:
            raise ValueError(f"{total} does not split evenly over {world} ranks")
        return [total // world * i for i in range(world + 1)]
    offs = [int(x) for x in offsets]
    if len(offs) != world + 1 or offs[0] != 0 or offs[-1] != total or \
            any(b <= a for a, b in zip(offs, offs[1:])):
        raise ValueError(f"bad shard offsets {offs} for {total} over {world} ranks")
    return offs


def shard_mlp_weights(A, bias, B, rank: int, world: int, offsets=None):
    """Rank `rank`'s contiguous copies of A's column block, bias's block and
    B's row block (what a rank holds in memory)."""
    offs = shard_bounds(A.shape[1], world, offsets)
    lo, hi = offs[rank], offs[rank + 1]
    A_i = A[:, lo:hi].contiguous()
    b_i = None if bias is None else bias[lo:hi].contiguous()
    B_i = B[lo:hi, :].contiguous()
    return A_i, b_i, B_i


class LibraryShard:
    """Per-shard compute through the library (the rank's GPU, N = 1)."""

    def __init__(self):
        import linear_layers_b200 as tpl

        self.tpl = tpl

    def mlp_fwd(self, X, A_i, bias_i, B_i, act):
        Z_i, U_i, Y_i = self.tpl.tp_mlp_fwd(X, A_i, bias_i, B_i, 1, act=act)
        return Z_i, U_i, Y_i

    def mlp_bwd(self, X, A_i, B_i, U_i, Y_i, dZ, act):
        g = self.tpl.tp_mlp_bwd(X, A_i, B_i, U_i, Y_i, dZ, 1, act=act)
        return {"dX": g["dX"], "dA": g["dA"], "dbias": g["dbias"], "dB": g["dB"]}

    def col_fwd(self, X, W_i, bias_i):
        Y, _ = self.tpl.tp_col_linear_fwd(X, W_i, bias_i, 1)
        return Y

    def col_bwd(self, X, W_i, dY_i):
        g = self.tpl.tp_col_linear_bwd(X, W_i, None, dY_i, 1)
        return {"dX": g["dX"], "dW": g["dW"], "dbias": g["dbias"]}

    def row_fwd(self, Xin_i, W_i):
        return self.tpl.tp_row_linear_fwd(Xin_i, W_i, 1)

    def row_bwd(self, Xin_i, W_i, dZ):
        g = self.tpl.tp_row_linear_bwd(Xin_i, W_i, dZ, 1)
        return {"dXin": g["dXin"], "dW": g["dW"]}


@dataclass
class MLPState:
    U: torch.Tensor
    Y: torch.Tensor


class TPMLP:
    """The TP-MLP with this rank's shard: forward all-reduces Z, backward
    all-reduces dX; the weight gradients stay local to the shard."""

    def __init__(self, A_i, bias_i, B_i, group=None, compute=None, act=ACT_GELU_TANH):
        self.A_i, self.bias_i, self.B_i = A_i, bias_i, B_i
        self.group = group
        self.compute = compute if compute is not None else LibraryShard()
        self.act = act

    def forward(self, X):
        """Z = Σ_ranks GeLU(X·A_i + bias_i)·B_i.  Returns (Z, state for backward)."""
        Z, U_i, Y_i = self.compute.mlp_fwd(X, self.A_i, self.bias_i, self.B_i, self.act)
        dist.all_reduce(Z, group=self.group)                 # g forward
        return Z, MLPState(U_i, Y_i)

    def backward(self, X, state: MLPState, dZ):
        """dX (all-reduced over the ranks) and this shard's dA_i, dbias_i, dB_i."""
        g = self.compute.mlp_bwd(X, self.A_i, self.B_i, state.U, state.Y, dZ, self.act)
        dist.all_reduce(g["dX"], group=self.group)           # f backward
        return g


class ColumnParallelLinear:
    """Y_i = X·W_i + bias_i on this rank ([TP-ILL] §1.2): no communication
    forward; the backward all-reduces dX (the f operator)."""

    def __init__(self, W_i, bias_i=None, group=None, compute=None):
        self.W_i, self.bias_i, self.group = W_i, bias_i, group
        self.compute = compute if compute is not None else LibraryShard()

    def forward(self, X):
        return self.compute.col_fwd(X, self.W_i, self.bias_i)

    def backward(self, X, dY_i):
        g = self.compute.col_bwd(X, self.W_i, dY_i)
        dist.all_reduce(g["dX"], group=self.group)
        return g


class RowParallelLinear:
    """Z = Σ_ranks Xin_i·W_i ([TP-ILL] §1.1): the forward all-reduces Z (the
    g operator); the backward is local (dXin_i = dZ·W_iᵀ, dW_i = Xin_iᵀ·dZ)."""

    def __init__(self, W_i, group=None, compute=None):
        self.W_i, self.group = W_i, group
        self.compute = compute if compute is not None else LibraryShard()

    def forward(self, Xin_i):
        Z = self.compute.row_fwd(Xin_i, self.W_i)
        dist.all_reduce(Z, group=self.group)
        return Z

    def backward(self, Xin_i, dZ):
        return self.compute.row_bwd(Xin_i, self.W_i, dZ)
