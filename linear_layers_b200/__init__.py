"""Megatron-style tensor-parallel layers on one B200 (sm_100a).

Thin ctypes binding over ``libtplayers.so`` (declared in ``include/tplayers.h``).
Every function here has the name of the C entry point it calls and does
argument marshalling only: it reads sizes from the tensors' shapes,
allocates missing outputs with torch (device memory is torch's job), checks
that every other tensor has the shape, dtype and device those sizes imply,
passes raw device pointers and the current CUDA stream, and raises
``TPError`` on a non-zero status.  All arithmetic happens in the library's CUDA kernels; there
is no CPU or PyTorch fallback, and importing a function whose library is
missing fails loudly.

The N tensor-parallel shards are partitions of the same device tensors:
shard i of A owns columns [off_i, off_{i+1}), shard i of B the same rows,
shard i of the vocabulary the rows [i·v/N, (i+1)·v/N) of E.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "TPError", "lib", "library_path", "ACT_NONE", "ACT_GELU_TANH", "ACT_GELU_ERF",
    "tp_status_string", "tp_version", "tp_launch_count", "tp_selftest_wait_timeout",
    "tp_debug_stall_next_gemm",
    "tp_workspace_bytes", "tp_mlp_fwd", "tp_mlp_bwd",
    "tp_col_linear_fwd", "tp_col_linear_bwd", "tp_row_linear_fwd", "tp_row_linear_bwd",
    "tp_row_linear_fwd_noalloc", "NOALLOC_SCRATCH_BYTES",
    "vp_embed", "tp_logits_fwd", "vp_xent", "vp_xent_bf16_grad", "tp_logits_bwd", "vp_embed_bwd",
    "OP_EMBED_BWD", "new_status", "DEVERR_RANGE", "DEVERR_TIMEOUT",
    "tp_linear_xent_fwd", "tp_linear_xent_dlogits", "OP_LINEAR_XENT", "tp_mlp_bwd_recompute",
    "tp_attention_fwd", "tp_sp_dropout_add_ln_fwd", "tp_sp_dropout_add_ln_bwd", "OP_SP_LN_BWD",
    "tp_attention_bwd", "OP_ATTENTION_BWD",
    "OP_MLP_FWD", "OP_MLP_BWD", "OP_ROW_LINEAR_FWD", "OP_COL_LINEAR_BWD", "OP_ROW_LINEAR_BWD",
]

ACT_NONE, ACT_GELU_TANH, ACT_GELU_ERF = 0, 1, 2
DTYPE_BF16, DTYPE_F32 = 0, 1
(OP_MLP_FWD, OP_MLP_BWD, OP_ROW_LINEAR_FWD, OP_COL_LINEAR_BWD, OP_ROW_LINEAR_BWD, OP_EMBED_BWD,
 OP_LINEAR_XENT, OP_SP_LN_BWD, OP_ATTENTION_BWD) = range(9)
DEVERR_RANGE, DEVERR_TIMEOUT = 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libtplayers.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t
_F = ctypes.c_float

_SIGS = {
    "tp_status_string": ([_I32], ctypes.c_char_p),
    "tp_version": ([], _I32),
    "tp_launch_count": ([], ctypes.c_uint64),
    "tp_selftest_wait_timeout": ([_P, ctypes.c_uint32, _P], _I32),
    "tp_debug_stall_next_gemm": ([_I32, _I32, ctypes.c_uint32], _I32),
    "tp_workspace_bytes": ([_I32, _I64, _I64, _I64, _I32], _SZ),
    "tp_mlp_fwd": ([_P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I32, _I32,
                    _P, _P, _P, _P, _P, _SZ, _P, _P], _I32),
    "tp_mlp_bwd": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I32, _I32,
                    _P, _P, _P, _P, _P, _P, _SZ, _P, _P], _I32),
    "tp_col_linear_fwd": ([_P, _P, _P, _I64, _I64, _I64, _I32, _P, _I32, _I32,
                           _P, _P, _P, _P], _I32),
    "tp_col_linear_bwd": ([_P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I32, _I32,
                           _P, _P, _P, _P, _P, _SZ, _P, _P], _I32),
    "tp_row_linear_fwd": ([_P, _P, _I64, _I64, _I64, _I32, _P, _I32, _P, _P, _P, _SZ,
                           _P, _P], _I32),
    "tp_row_linear_bwd": ([_P, _P, _P, _I64, _I64, _I64, _I32, _P, _I32, _P, _P, _P, _P], _I32),
    "tp_row_linear_fwd_noalloc": ([_P, _P, _I64, _I64, _I64, _I32, _P, _I32, _P, _P, _P], _I32),
    "vp_embed": ([_P, _I64, _P, _I64, _I64, _I32, _I32, _P, _P, _P], _I32),
    "tp_logits_fwd": ([_P, _P, _I64, _I64, _I64, _I32, _P, _P, _P], _I32),
    "vp_xent": ([_P, _P, _I64, _I64, _I32, _F, _P, _P, _P, _P, _P, _P], _I32),
    "vp_xent_bf16_grad": ([_P, _P, _I64, _I64, _I32, _F, _P, _P, _P, _P, _P, _P], _I32),
    "tp_logits_bwd": ([_P, _P, _P, _I64, _I64, _I64, _I32, _P, _P, _P, _P], _I32),
    "vp_embed_bwd": ([_P, _P, _I64, _I64, _I64, _I32, _P, _P, _SZ, _P, _P], _I32),
    "tp_linear_xent_fwd": ([_P, _P, _P, _I64, _I64, _I64, _I32, _P, _P, _P, _P, _P, _SZ,
                            _P, _P], _I32),
    "tp_linear_xent_dlogits": ([_P, _P, _P, _P, _I64, _I64, _I64, _I32, _F, _P, _P, _P], _I32),
    "tp_sp_dropout_add_ln_fwd": ([_P, _P, _P, _P, _P, _I64, _I64, _I32, _F, ctypes.c_uint64,
                                  ctypes.c_uint64, _F, _P, _P, _P, _P, _P, _P, _P], _I32),
    "tp_sp_dropout_add_ln_bwd": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, _F, ctypes.c_uint64,
                                  ctypes.c_uint64, _P, _P, _P, _P, _P, _P, _SZ, _P, _P], _I32),
    "tp_attention_bwd": ([_P, _P, _P, _P, _I64, _I64, _I32, _I32, _I32, _P, _I32, _F, _P, _P, _SZ,
                          _P, _P], _I32),
    "tp_attention_fwd": ([_P, _I64, _I64, _I32, _I32, _I32, _P, _I32, _F, _P, _P, _P, _P], _I32),
    "tp_mlp_bwd_recompute": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I32, _I32,
                              _P, _P, _P, _P, _P, _P, _SZ, _P, _P], _I32),
}


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({_status_text(status)})")


def lib():
    """Load libtplayers.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"{library_path} is missing: build it with `python -m linear_layers_b200.build`")
        handle = ctypes.CDLL(library_path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def _status_text(s: int) -> str:
    try:
        return lib().tp_status_string(int(s)).decode()
    except Exception:  # pragma: no cover - library missing while formatting an error
        return "?"


def _check(status: int, where: str):
    if status != 0:
        raise TPError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    if torch.device(device).type != "cuda":
        raise RuntimeError("linear_layers_b200 runs on CUDA tensors only; there is no CPU path")
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _offsets(offsets, N):
    if offsets is None:
        return None, None
    arr = (ctypes.c_int64 * (N + 1))(*[int(x) for x in offsets])
    return arr, arr


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major, no padding)")


_BF, _F32, _I64T, _I32T, _U8 = torch.bfloat16, torch.float32, torch.int64, torch.int32, torch.uint8


def _want(dev, *specs):
    """Check (name, tensor, shape, dtype) entries before anything is enqueued.

    The library receives bare pointers and the sizes read from the leading
    operands, so a tensor of another shape, dtype or device would be read or
    written past its end on the GPU.  A None tensor (an optional argument)
    passes; a None shape or dtype is not checked.  The status word must be
    an int32 tensor on the same device."""
    for name, t, shape, dtype in specs:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor, not {type(t).__name__}")
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the operands on {dev}")
        if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} is {t.dtype}, expected {dtype}")


def _status_spec(dev_status):
    if dev_status is not None and isinstance(dev_status, torch.Tensor) and dev_status.numel() < 1:
        raise ValueError("dev_status must hold at least one int32 word")
    return ("dev_status", dev_status, None, _I32T)


def _ws_spec(ws):
    return ("ws", ws, None, None)


def new_status(device="cuda") -> torch.Tensor:
    """A zeroed int32 device word for the kernels' TP_DEVERR_* bits."""
    return torch.zeros(1, dtype=torch.int32, device=device)


def tp_status_string(s: int) -> str:
    return _status_text(s)


def tp_version() -> int:
    return int(lib().tp_version())


def tp_launch_count() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(lib().tp_launch_count())


def tp_selftest_wait_timeout(dev_status, limit_us=1000):
    """Run the device self-test of the bounded wait; returns the status word."""
    _check(lib().tp_selftest_wait_timeout(_ptr(dev_status), int(limit_us),
                                          _stream(dev_status.device)), "tp_selftest_wait_timeout")
    return dev_status


def tp_debug_stall_next_gemm(unit: int, kblock: int, wait_limit_us: int = 50000):
    """Arm the one-shot producer stall of the next tensor-core GEMM launch
    (diagnostics of the bounded-wait failure path; see tplayers.h)."""
    _check(lib().tp_debug_stall_next_gemm(int(unit), int(kblock), int(wait_limit_us)),
           "tp_debug_stall_next_gemm")


def tp_workspace_bytes(op: int, M: int, h: int, F: int, N: int) -> int:
    return int(lib().tp_workspace_bytes(int(op), int(M), int(h), int(F), int(N)))


def _workspace(ws, op, M, h, F, N, device):
    need = tp_workspace_bytes(op, M, h, F, N)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws, (0 if ws is None else ws.numel() * ws.element_size())


def tp_mlp_fwd(X, A, bias, B, N, *, shard_offsets=None, act=ACT_GELU_TANH, U=None, Y=None,
               Z=None, Zpart=None, ws=None, dev_status=None):
    """Z = Σ_i act(X·A_i + bias_i)·B_i.  Returns (Z, U, Y)."""
    M, h = X.shape
    F = A.shape[1]
    dev = X.device
    U = torch.empty(M, F, dtype=X.dtype, device=dev) if U is None else U
    Y = torch.empty(M, F, dtype=X.dtype, device=dev) if Y is None else Y
    Z = torch.empty(M, h, dtype=X.dtype, device=dev) if Z is None else Z
    _contig(X, A, bias, B, U, Y, Z, Zpart)
    dt = X.dtype
    _want(dev, ("A", A, (h, F), dt), ("bias", bias, (F,), dt), ("B", B, (F, h), dt),
          ("U", U, (M, F), dt), ("Y", Y, (M, F), dt), ("Z", Z, (M, h), dt),
          ("Zpart", Zpart, (N, M, h), _F32), _ws_spec(ws), _status_spec(dev_status))
    ws, wsb = _workspace(ws, OP_MLP_FWD, M, h, F, N, dev)
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_mlp_fwd(_ptr(X), _ptr(A), _ptr(bias), _ptr(B), M, h, F, N, offs, _dt(X),
                            act, _ptr(U), _ptr(Y), _ptr(Z), _ptr(Zpart), _ptr(ws), wsb,
                            _ptr(dev_status), _stream(dev)), "tp_mlp_fwd")
    return Z, U, Y


def _mlp_bwd_specs(M, h, F, dt, A, B, U, Y, dZ, dU, dX, dA, dbias, dB, ws, dev_status):
    return (("A", A, (h, F), dt), ("B", B, (F, h), dt), ("U", U, (M, F), dt),
            ("Y", Y, (M, F), dt), ("dZ", dZ, (M, h), dt), ("dU", dU, (M, F), dt),
            ("dX", dX, (M, h), dt), ("dA", dA, (h, F), dt), ("dbias", dbias, (F,), _F32),
            ("dB", dB, (F, h), dt), _ws_spec(ws), _status_spec(dev_status))


def tp_mlp_bwd(X, A, B, U, Y, dZ, N, *, shard_offsets=None, act=ACT_GELU_TANH, with_dbias=True,
               dU=None, dX=None, dA=None, dbias=None, dB=None, ws=None, dev_status=None):
    """Returns dict(dX, dA, dbias, dB, dU)."""
    M, h = X.shape
    F = A.shape[1]
    dev = X.device
    dt = X.dtype
    dU = torch.empty(M, F, dtype=dt, device=dev) if dU is None else dU
    dX = torch.empty(M, h, dtype=dt, device=dev) if dX is None else dX
    dA = torch.empty(h, F, dtype=dt, device=dev) if dA is None else dA
    dB = torch.empty(F, h, dtype=dt, device=dev) if dB is None else dB
    if dbias is None and with_dbias:
        dbias = torch.empty(F, dtype=torch.float32, device=dev)
    _contig(X, A, B, U, Y, dZ, dU, dX, dA, dB, dbias)
    _want(dev, *_mlp_bwd_specs(M, h, F, dt, A, B, U, Y, dZ, dU, dX, dA, dbias, dB, ws,
                               dev_status))
    ws, wsb = _workspace(ws, OP_MLP_BWD, M, h, F, N, dev)
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_mlp_bwd(_ptr(X), _ptr(A), _ptr(B), _ptr(U), _ptr(Y), _ptr(dZ), M, h, F, N,
                            offs, _dt(X), act, _ptr(dU), _ptr(dX), _ptr(dA), _ptr(dbias), _ptr(dB),
                            _ptr(ws), wsb, _ptr(dev_status), _stream(dev)), "tp_mlp_bwd")
    return {"dX": dX, "dA": dA, "dbias": dbias, "dB": dB, "dU": dU}


def tp_mlp_bwd_recompute(X, A, B, U, dZ, N, *, Y=None, shard_offsets=None, act=ACT_GELU_TANH,
                         with_dbias=True, dU=None, dX=None, dA=None, dbias=None, dB=None, ws=None,
                         dev_status=None):
    """Backward from the saved pre-activation U alone: Y = act(U) is rebuilt
    into ``Y`` (scratch, or U itself for in place).  Returns dict(dX, dA,
    dbias, dB, dU, Y)."""
    M, h = X.shape
    F = A.shape[1]
    dev = X.device
    dt = X.dtype
    Y = torch.empty(M, F, dtype=dt, device=dev) if Y is None else Y
    dU = torch.empty(M, F, dtype=dt, device=dev) if dU is None else dU
    dX = torch.empty(M, h, dtype=dt, device=dev) if dX is None else dX
    dA = torch.empty(h, F, dtype=dt, device=dev) if dA is None else dA
    dB = torch.empty(F, h, dtype=dt, device=dev) if dB is None else dB
    if dbias is None and with_dbias:
        dbias = torch.empty(F, dtype=torch.float32, device=dev)
    _contig(X, A, B, U, Y, dZ, dU, dX, dA, dB, dbias)
    _want(dev, *_mlp_bwd_specs(M, h, F, dt, A, B, U, Y, dZ, dU, dX, dA, dbias, dB, ws,
                               dev_status))
    ws, wsb = _workspace(ws, OP_MLP_BWD, M, h, F, N, dev)
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_mlp_bwd_recompute(_ptr(X), _ptr(A), _ptr(B), _ptr(U), _ptr(Y), _ptr(dZ), M, h,
                                      F, N, offs, _dt(X), act, _ptr(dU), _ptr(dX), _ptr(dA),
                                      _ptr(dbias), _ptr(dB), _ptr(ws), wsb, _ptr(dev_status),
                                      _stream(dev)), "tp_mlp_bwd_recompute")
    return {"dX": dX, "dA": dA, "dbias": dbias, "dB": dB, "dU": dU, "Y": Y}


def tp_col_linear_fwd(X, W, bias, N, *, shard_offsets=None, act=ACT_NONE, U=None, Y=None,
                      dev_status=None):
    """Y = act(X·W + bias) over all column shards.  Returns (Y, U) (U is None for act NONE
    unless given)."""
    M, K = X.shape
    Nout = W.shape[1]
    dev = X.device
    if U is None and act != ACT_NONE:
        U = torch.empty(M, Nout, dtype=X.dtype, device=dev)
    Y = torch.empty(M, Nout, dtype=X.dtype, device=dev) if Y is None else Y
    _contig(X, W, bias, U, Y)
    dt = X.dtype
    _want(dev, ("W", W, (K, Nout), dt), ("bias", bias, (Nout,), dt), ("U", U, (M, Nout), dt),
          ("Y", Y, (M, Nout), dt), _status_spec(dev_status))
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_col_linear_fwd(_ptr(X), _ptr(W), _ptr(bias), M, K, Nout, N, offs, _dt(X),
                                   act, _ptr(U), _ptr(Y), _ptr(dev_status), _stream(dev)),
           "tp_col_linear_fwd")
    return Y, U


def tp_col_linear_bwd(X, W, U, dY, N, *, shard_offsets=None, act=ACT_NONE, with_dbias=True,
                      dU=None, dX=None, dW=None, dbias=None, ws=None, dev_status=None):
    """Returns dict(dX, dW, dbias, dU)."""
    M, K = X.shape
    Nout = W.shape[1]
    dev = X.device
    dt = X.dtype
    if dU is None and act != ACT_NONE:
        dU = torch.empty(M, Nout, dtype=dt, device=dev)
    dX = torch.empty(M, K, dtype=dt, device=dev) if dX is None else dX
    dW = torch.empty(K, Nout, dtype=dt, device=dev) if dW is None else dW
    if dbias is None and with_dbias:
        dbias = torch.empty(Nout, dtype=torch.float32, device=dev)
    _contig(X, W, U, dY, dU, dX, dW, dbias)
    _want(dev, ("W", W, (K, Nout), dt), ("U", U, (M, Nout), dt), ("dY", dY, (M, Nout), dt),
          ("dU", dU, (M, Nout), dt), ("dX", dX, (M, K), dt), ("dW", dW, (K, Nout), dt),
          ("dbias", dbias, (Nout,), _F32), _ws_spec(ws), _status_spec(dev_status))
    ws, wsb = _workspace(ws, OP_COL_LINEAR_BWD, M, K, Nout, N, dev)
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_col_linear_bwd(_ptr(X), _ptr(W), _ptr(U), _ptr(dY), M, K, Nout, N, offs,
                                   _dt(X), act, _ptr(dU), _ptr(dX), _ptr(dW), _ptr(dbias),
                                   _ptr(ws), wsb, _ptr(dev_status), _stream(dev)),
           "tp_col_linear_bwd")
    return {"dX": dX, "dW": dW, "dbias": dbias, "dU": dU if dU is not None else dY}


def tp_row_linear_fwd(Xin, W, N, *, shard_offsets=None, Z=None, Zpart=None, ws=None,
                      dev_status=None):
    """Z = Σ_i Xin_i·W_i.  Returns Z."""
    M, Kin = Xin.shape
    Nout = W.shape[1]
    dev = Xin.device
    Z = torch.empty(M, Nout, dtype=Xin.dtype, device=dev) if Z is None else Z
    _contig(Xin, W, Z, Zpart)
    dt = Xin.dtype
    _want(dev, ("W", W, (Kin, Nout), dt), ("Z", Z, (M, Nout), dt),
          ("Zpart", Zpart, (N, M, Nout), _F32), _ws_spec(ws), _status_spec(dev_status))
    ws, wsb = _workspace(ws, OP_ROW_LINEAR_FWD, M, Nout, Kin, N, dev)
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_row_linear_fwd(_ptr(Xin), _ptr(W), M, Kin, Nout, N, offs, _dt(Xin), _ptr(Z),
                                   _ptr(Zpart), _ptr(ws), wsb, _ptr(dev_status), _stream(dev)),
           "tp_row_linear_fwd")
    return Z


NOALLOC_SCRATCH_BYTES = 32 << 20   # TP_NOALLOC_SCRATCH_BYTES in tplayers.h


def tp_row_linear_fwd_noalloc(Xin, W, N, *, shard_offsets=None, Z=None, dev_status=None):
    """Z = Σ_i Xin_i·W_i without any device allocation by the library.

    For callers that cannot allocate device memory (a host framework that
    owns every allocation, or a plugin interface that only passes input and
    output pointers): the shards' partials live in the library's static
    scratch of NOALLOC_SCRATCH_BYTES per GPU.  Only Z is allocated here, and
    only if the caller does not pass it.  Calls that overlap on the GPU share
    that scratch and race: serialise them.
    """
    M, Kin = Xin.shape
    Nout = W.shape[1]
    dev = Xin.device
    Z = torch.empty(M, Nout, dtype=Xin.dtype, device=dev) if Z is None else Z
    _contig(Xin, W, Z)
    dt = Xin.dtype
    _want(dev, ("W", W, (Kin, Nout), dt), ("Z", Z, (M, Nout), dt), _status_spec(dev_status))
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_row_linear_fwd_noalloc(_ptr(Xin), _ptr(W), M, Kin, Nout, N, offs, _dt(Xin),
                                           _ptr(Z), _ptr(dev_status), _stream(dev)),
           "tp_row_linear_fwd_noalloc")
    return Z


def tp_row_linear_bwd(Xin, W, dZ, N, *, shard_offsets=None, dXin=None, dW=None, dev_status=None):
    """Returns dict(dXin, dW)."""
    M, Kin = Xin.shape
    Nout = W.shape[1]
    dev = Xin.device
    dXin = torch.empty(M, Kin, dtype=Xin.dtype, device=dev) if dXin is None else dXin
    dW = torch.empty(Kin, Nout, dtype=Xin.dtype, device=dev) if dW is None else dW
    _contig(Xin, W, dZ, dXin, dW)
    dt = Xin.dtype
    _want(dev, ("W", W, (Kin, Nout), dt), ("dZ", dZ, (M, Nout), dt), ("dXin", dXin, (M, Kin), dt),
          ("dW", dW, (Kin, Nout), dt), _status_spec(dev_status))
    offs, keep = _offsets(shard_offsets, N)
    _check(lib().tp_row_linear_bwd(_ptr(Xin), _ptr(W), _ptr(dZ), M, Kin, Nout, N, offs, _dt(Xin),
                                   _ptr(dXin), _ptr(dW), _ptr(dev_status), _stream(dev)),
           "tp_row_linear_bwd")
    return {"dXin": dXin, "dW": dW}


def vp_embed(ids, E, N, *, out=None, dev_status=None):
    """out[t] = E[ids[t]] through the vocabulary shards (zero row for ids outside [0, v))."""
    T = ids.shape[0]
    v, h = E.shape
    dev = E.device
    out = torch.empty(T, h, dtype=E.dtype, device=dev) if out is None else out
    _contig(ids, E, out)
    if ids.dtype != torch.int64:
        raise TypeError("ids must be int64")
    _want(dev, ("ids", ids, (T,), _I64T), ("out", out, (T, h), E.dtype), _status_spec(dev_status))
    _check(lib().vp_embed(_ptr(ids), T, _ptr(E), v, h, N, _dt(E), _ptr(out), _ptr(dev_status),
                          _stream(dev)), "vp_embed")
    return out


def tp_logits_fwd(H, E, N, *, logits=None, dev_status=None):
    """logits [T, v] fp32 = H·Eᵀ, written shard block by shard block."""
    T, h = H.shape
    v = E.shape[0]
    dev = H.device
    logits = torch.empty(T, v, dtype=torch.float32, device=dev) if logits is None else logits
    _contig(H, E, logits)
    _want(dev, ("H", H, (T, h), _BF), ("E", E, (v, h), _BF), ("logits", logits, (T, v), _F32),
          _status_spec(dev_status))
    _check(lib().tp_logits_fwd(_ptr(H), _ptr(E), T, h, v, N, _ptr(logits), _ptr(dev_status),
                               _stream(dev)), "tp_logits_fwd")
    return logits


def _xent_specs(T, v, logits, targets, loss, loss_sum, argmax, dev_status):
    return (("logits", logits, (T, v), _F32), ("targets", targets, (T,), _I64T),
            ("loss", loss, (T,), _F32), ("loss_sum", loss_sum, (1,), _F32),
            ("argmax", argmax, (T,), _I32T), _status_spec(dev_status))


def vp_xent(logits, targets, N, *, grad_scale=1.0, with_grad=True, with_argmax=True,
            loss=None, loss_sum=None, dlogits=None, argmax=None, dev_status=None):
    """Returns dict(loss [T], loss_sum [1], dlogits [T,v] or None, argmax [T] or None)."""
    T, v = logits.shape
    dev = logits.device
    loss = torch.empty(T, dtype=torch.float32, device=dev) if loss is None else loss
    loss_sum = torch.empty(1, dtype=torch.float32, device=dev) if loss_sum is None else loss_sum
    if with_grad and dlogits is None:
        dlogits = torch.empty_like(logits)
    if with_argmax and argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=dev)
    _contig(logits, targets, loss, dlogits, argmax)
    if targets.dtype != torch.int64:
        raise TypeError("targets must be int64")
    _want(dev, *_xent_specs(T, v, logits, targets, loss, loss_sum, argmax, dev_status),
          ("dlogits", dlogits, (T, v), _F32))
    _check(lib().vp_xent(_ptr(logits), _ptr(targets), T, v, N, float(grad_scale), _ptr(loss),
                         _ptr(loss_sum), _ptr(dlogits), _ptr(argmax), _ptr(dev_status),
                         _stream(dev)), "vp_xent")
    return {"loss": loss, "loss_sum": loss_sum, "dlogits": dlogits, "argmax": argmax}


def vp_xent_bf16_grad(logits, targets, N, *, grad_scale=1.0, with_argmax=True, loss=None,
                      loss_sum=None, dlogits=None, argmax=None, dev_status=None):
    """vp_xent with the gradient written in bf16.  Returns the same dict."""
    T, v = logits.shape
    dev = logits.device
    loss = torch.empty(T, dtype=torch.float32, device=dev) if loss is None else loss
    loss_sum = torch.empty(1, dtype=torch.float32, device=dev) if loss_sum is None else loss_sum
    dlogits = torch.empty(T, v, dtype=torch.bfloat16, device=dev) if dlogits is None else dlogits
    if with_argmax and argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=dev)
    _contig(logits, targets, loss, dlogits, argmax)
    if targets.dtype != torch.int64:
        raise TypeError("targets must be int64")
    _want(dev, *_xent_specs(T, v, logits, targets, loss, loss_sum, argmax, dev_status),
          ("dlogits", dlogits, (T, v), _BF))
    _check(lib().vp_xent_bf16_grad(_ptr(logits), _ptr(targets), T, v, N, float(grad_scale),
                                   _ptr(loss), _ptr(loss_sum), _ptr(dlogits), _ptr(argmax),
                                   _ptr(dev_status), _stream(dev)), "vp_xent_bf16_grad")
    return {"loss": loss, "loss_sum": loss_sum, "dlogits": dlogits, "argmax": argmax}


def tp_logits_bwd(dlogits, H, E, N, *, dH=None, dE=None, dev_status=None):
    """dH = Σ_i dlogits_i·E_i (bf16), dE = dlogitsᵀ·H (fp32).  Returns (dH, dE)."""
    T, v = dlogits.shape
    h = H.shape[1]
    dev = H.device
    dH = torch.empty(T, h, dtype=H.dtype, device=dev) if dH is None else dH
    dE = torch.empty(v, h, dtype=torch.float32, device=dev) if dE is None else dE
    _contig(dlogits, H, E, dH, dE)
    _want(dev, ("dlogits", dlogits, (T, v), _BF), ("H", H, (T, h), _BF), ("E", E, (v, h), _BF),
          ("dH", dH, (T, h), _BF), ("dE", dE, (v, h), _F32), _status_spec(dev_status))
    _check(lib().tp_logits_bwd(_ptr(dlogits), _ptr(H), _ptr(E), T, h, v, N, _ptr(dH), _ptr(dE),
                               _ptr(dev_status), _stream(dev)), "tp_logits_bwd")
    return dH, dE


def vp_embed_bwd(ids, dout, dE, N, *, ws=None, dev_status=None):
    """dE[x] += Σ_{t: ids[t] = x} dout[t] (in place, token order).  Returns dE."""
    T, h = dout.shape
    v = dE.shape[0]
    dev = dout.device
    _contig(ids, dout, dE)
    if ids.dtype != torch.int64:
        raise TypeError("ids must be int64")
    _want(dev, ("ids", ids, (T,), _I64T), ("dout", dout, (T, h), _BF), ("dE", dE, (v, h), _F32),
          _ws_spec(ws), _status_spec(dev_status))
    ws, wsb = _workspace(ws, OP_EMBED_BWD, T, h, v, N, dev)
    _check(lib().vp_embed_bwd(_ptr(ids), _ptr(dout), T, v, h, N, _ptr(dE), _ptr(ws), wsb,
                              _ptr(dev_status), _stream(dev)), "vp_embed_bwd")
    return dE


def tp_linear_xent_fwd(H, E, targets, N, *, with_argmax=True, loss=None, loss_sum=None, lse=None,
                       argmax=None, ws=None, dev_status=None):
    """Cross-entropy of logits = H·Eᵀ without storing the logits.

    Returns {"loss" [T] fp32, "loss_sum" [1] fp32, "lse" [T] fp32, "argmax" [T] int32 or None}.
    """
    T, h = H.shape
    v = E.shape[0]
    dev = H.device
    loss = torch.empty(T, dtype=torch.float32, device=dev) if loss is None else loss
    loss_sum = torch.empty(1, dtype=torch.float32, device=dev) if loss_sum is None else loss_sum
    lse = torch.empty(T, dtype=torch.float32, device=dev) if lse is None else lse
    if with_argmax and argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=dev)
    _contig(H, E, targets, loss, lse, argmax)
    if targets.dtype != torch.int64:
        raise TypeError("targets must be int64")
    _want(dev, ("H", H, (T, h), _BF), ("E", E, (v, h), _BF), ("targets", targets, (T,), _I64T),
          ("loss", loss, (T,), _F32), ("loss_sum", loss_sum, (1,), _F32), ("lse", lse, (T,), _F32),
          ("argmax", argmax, (T,), _I32T), _ws_spec(ws), _status_spec(dev_status))
    ws, wsb = _workspace(ws, OP_LINEAR_XENT, T, h, v, N, dev)
    _check(lib().tp_linear_xent_fwd(_ptr(H), _ptr(E), _ptr(targets), T, h, v, N, _ptr(loss),
                                    _ptr(loss_sum), _ptr(lse), _ptr(argmax), _ptr(ws), wsb,
                                    _ptr(dev_status), _stream(dev)), "tp_linear_xent_fwd")
    return {"loss": loss, "loss_sum": loss_sum, "lse": lse, "argmax": argmax}


def tp_linear_xent_dlogits(H, E, targets, lse, N, *, grad_scale=1.0, dlogits=None,
                           dev_status=None):
    """bf16 dlogits = grad_scale·(exp(H·Eᵀ − lse) − onehot), logits recomputed on chip."""
    T, h = H.shape
    v = E.shape[0]
    dev = H.device
    dlogits = torch.empty(T, v, dtype=torch.bfloat16, device=dev) if dlogits is None else dlogits
    _contig(H, E, targets, lse, dlogits)
    if targets.dtype != torch.int64:
        raise TypeError("targets must be int64")
    _want(dev, ("H", H, (T, h), _BF), ("E", E, (v, h), _BF), ("targets", targets, (T,), _I64T),
          ("lse", lse, (T,), _F32), ("dlogits", dlogits, (T, v), _BF), _status_spec(dev_status))
    _check(lib().tp_linear_xent_dlogits(_ptr(H), _ptr(E), _ptr(targets), _ptr(lse), T, h, v, N,
                                        float(grad_scale), _ptr(dlogits), _ptr(dev_status),
                                        _stream(dev)), "tp_linear_xent_dlogits")
    return dlogits


def tp_attention_fwd(QKV, b, s, n_heads, N, *, head_offsets=None, causal=True, scale=None,
                     ctx=None, lse=None, with_lse=False, dev_status=None):
    """Per-shard attention core on the shard-major QKV [b·s, 3·n_heads·64].

    Returns (ctx [b·s, n_heads·64] bf16, lse [b, n_heads, s] fp32 or None)."""
    dev = QKV.device
    hd = 64
    ctx = torch.empty(b * s, n_heads * hd, dtype=QKV.dtype, device=dev) if ctx is None else ctx
    if with_lse and lse is None:
        lse = torch.empty(b, n_heads, s, dtype=torch.float32, device=dev)
    _contig(QKV, ctx, lse)
    _want(dev, ("QKV", QKV, (b * s, 3 * n_heads * hd), _BF), ("ctx", ctx, (b * s, n_heads * hd), _BF),
          ("lse", lse, (b, n_heads, s), _F32), _status_spec(dev_status))
    offs, keep = _offsets(head_offsets, N)
    _check(lib().tp_attention_fwd(_ptr(QKV), b, s, n_heads, hd, N, offs, 1 if causal else 0,
                                  float(scale) if scale else 0.0, _ptr(ctx), _ptr(lse),
                                  _ptr(dev_status), _stream(dev)), "tp_attention_fwd")
    return ctx, lse


def tp_sp_dropout_add_ln_fwd(x, bias, residual, gamma, beta, N, *, p=0.0, seed=0, offset=0,
                             eps=1e-5, with_keep=False, hs=None, y=None, mean=None, rstd=None,
                             keep=None, dev_status=None):
    """hs = residual + dropout(x + bias), y = LayerNorm(hs) on N sequence shards.

    Returns dict(hs, y, mean, rstd, keep or None)."""
    M, h = x.shape
    dev = x.device
    hs = torch.empty_like(x) if hs is None else hs
    y = torch.empty_like(x) if y is None else y
    mean = torch.empty(M, dtype=torch.float32, device=dev) if mean is None else mean
    rstd = torch.empty(M, dtype=torch.float32, device=dev) if rstd is None else rstd
    if with_keep and keep is None:
        keep = torch.empty(M, h, dtype=torch.uint8, device=dev)
    _contig(x, bias, residual, gamma, beta, hs, y, mean, rstd, keep)
    _want(dev, ("x", x, (M, h), _BF), ("bias", bias, (h,), _BF), ("residual", residual, (M, h), _BF),
          ("gamma", gamma, (h,), _BF), ("beta", beta, (h,), _BF), ("hs", hs, (M, h), _BF),
          ("y", y, (M, h), _BF), ("mean", mean, (M,), _F32), ("rstd", rstd, (M,), _F32),
          ("keep", keep, (M, h), _U8), _status_spec(dev_status))
    _check(lib().tp_sp_dropout_add_ln_fwd(_ptr(x), _ptr(bias), _ptr(residual), _ptr(gamma),
                                          _ptr(beta), M, h, N, float(p), int(seed), int(offset),
                                          float(eps), _ptr(hs), _ptr(y), _ptr(mean), _ptr(rstd),
                                          _ptr(keep), _ptr(dev_status), _stream(dev)),
           "tp_sp_dropout_add_ln_fwd")
    return {"hs": hs, "y": y, "mean": mean, "rstd": rstd, "keep": keep}


def tp_sp_dropout_add_ln_bwd(dy, dhs_in, hs, gamma, mean, rstd, N, *, p=0.0, seed=0, offset=0,
                             with_dbias=True, dx=None, dresidual=None, dgamma=None, dbeta=None,
                             dbias=None, ws=None, dev_status=None):
    """Backward of tp_sp_dropout_add_ln_fwd.  Returns dict(dx, dresidual, dgamma, dbeta, dbias)."""
    M, h = dy.shape
    dev = dy.device
    dx = torch.empty_like(dy) if dx is None else dx
    dresidual = torch.empty_like(dy) if dresidual is None else dresidual
    dgamma = torch.empty(h, dtype=torch.float32, device=dev) if dgamma is None else dgamma
    dbeta = torch.empty(h, dtype=torch.float32, device=dev) if dbeta is None else dbeta
    if with_dbias and dbias is None:
        dbias = torch.empty(h, dtype=torch.float32, device=dev)
    _contig(dy, dhs_in, hs, gamma, mean, rstd, dx, dresidual, dgamma, dbeta, dbias)
    _want(dev, ("dy", dy, (M, h), _BF), ("dhs_in", dhs_in, (M, h), _BF), ("hs", hs, (M, h), _BF),
          ("gamma", gamma, (h,), _BF), ("mean", mean, (M,), _F32), ("rstd", rstd, (M,), _F32),
          ("dx", dx, (M, h), _BF), ("dresidual", dresidual, (M, h), _BF),
          ("dgamma", dgamma, (h,), _F32), ("dbeta", dbeta, (h,), _F32), ("dbias", dbias, (h,), _F32),
          _ws_spec(ws), _status_spec(dev_status))
    ws, wsb = _workspace(ws, OP_SP_LN_BWD, M, h, h, N, dev)
    _check(lib().tp_sp_dropout_add_ln_bwd(_ptr(dy), _ptr(dhs_in), _ptr(hs), _ptr(gamma),
                                          _ptr(mean), _ptr(rstd), M, h, N, float(p), int(seed),
                                          int(offset), _ptr(dx), _ptr(dresidual), _ptr(dgamma),
                                          _ptr(dbeta), _ptr(dbias), _ptr(ws), wsb,
                                          _ptr(dev_status), _stream(dev)),
           "tp_sp_dropout_add_ln_bwd")
    return {"dx": dx, "dresidual": dresidual, "dgamma": dgamma, "dbeta": dbeta, "dbias": dbias}


def tp_attention_bwd(QKV, ctx, dctx, lse, b, s, n_heads, N, *, head_offsets=None, causal=True,
                     scale=None, dQKV=None, ws=None, dev_status=None):
    """Gradient of the attention core with respect to QKV (shard-major layout).
    lse from tp_attention_fwd(..., with_lse=True).  Returns dQKV."""
    dev = QKV.device
    dQKV = torch.empty_like(QKV) if dQKV is None else dQKV
    _contig(QKV, ctx, dctx, lse, dQKV)
    _want(dev, ("QKV", QKV, (b * s, 3 * n_heads * 64), _BF), ("ctx", ctx, (b * s, n_heads * 64), _BF),
          ("dctx", dctx, (b * s, n_heads * 64), _BF), ("lse", lse, (b, n_heads, s), _F32),
          ("dQKV", dQKV, (b * s, 3 * n_heads * 64), _BF), _ws_spec(ws), _status_spec(dev_status))
    offs, keep = _offsets(head_offsets, N)
    ws, wsb = _workspace(ws, OP_ATTENTION_BWD, b * s, n_heads, 64, N, dev)
    _check(lib().tp_attention_bwd(_ptr(QKV), _ptr(ctx), _ptr(dctx), _ptr(lse), b, s, n_heads, 64,
                                  N, offs, 1 if causal else 0, float(scale) if scale else 0.0,
                                  _ptr(dQKV), _ptr(ws), wsb, _ptr(dev_status), _stream(dev)),
           "tp_attention_bwd")
    return dQKV
