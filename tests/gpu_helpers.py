"""Shared helpers for the GPU parity tests (comparison metrics, tolerances,
guard bands around outputs)."""
import os

import numpy as np
import torch

# bf16 storage, fp32 accumulation: the stated relative error of every GEMM
# output and gradient against the fp64 oracle, applied both per tensor
# (relative Frobenius) and per element (see elem_ratio).
TOL_BF16 = 2e-2
# fp32 CUDA-core path (tiny fp32 configuration); the inputs are exact fp32
# values, so only fp32 accumulation order and the library's tanh/erf differ.
TOL_F32 = 1e-5
# fp32 cross-entropy: loss per token (relative) and dlogits (relative Frobenius)
TOL_XENT = 1e-4


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _as64(x):
    return f64(x) if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)


def rel_fro(gpu, ref):
    g = _as64(gpu)
    r = _as64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / (den if den > 0 else 1.0))


def elem_ratio(gpu, ref):
    """max over elements of |gpu − ref| / max(|ref|, rms(ref)).

    The element-wise reading of "relative error ≤ tol": an element's error is
    measured against its own magnitude, and against the tensor's root mean
    square where the true value is smaller than that (near zero a relative
    error is undefined, and a value there still carries the absolute rounding
    of the sums that produced it).  One element that is entirely wrong (a
    missed or misplaced store, a stale value) gives a ratio near 1, far above
    any tolerance here.  NaN anywhere gives NaN, which fails every bound.
    """
    g = _as64(gpu)
    r = _as64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    floor = rms if rms > 0 else 1.0
    d = np.abs(g - r)
    if np.isnan(d).any():
        return float("nan")
    return float(np.max(d / np.maximum(np.abs(r), floor)))


def assert_close(name, gpu, ref, tol, elem_tol=None):
    """Relative Frobenius error ≤ tol for the tensor AND every element within
    elem_tol (default tol) by elem_ratio.  Returns (frobenius, element) errors."""
    e = rel_fro(gpu, ref)
    m = elem_ratio(gpu, ref)
    et = tol if elem_tol is None else elem_tol
    if os.environ.get("TP_PARITY_LOG"):
        with open(os.environ["TP_PARITY_LOG"], "a") as fh:
            fh.write(f"{name}\t{e:.3e}\t{m:.3e}\t{tol:.1e}\t{et:.1e}\n")
    assert e <= tol, f"{name}: relative Frobenius error {e:.3e} > {tol:.1e}"
    assert m <= et, f"{name}: element-wise relative error {m:.3e} > {et:.1e}"
    return e, m


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


# ----------------------------------------------------------------------------
# canaries: outputs inside a larger buffer whose margins hold a sentinel
# ----------------------------------------------------------------------------
GUARD_BYTES = 4096        # a multiple of 256, so the output keeps its alignment
SENTINEL = 0x5A


class Guarded:
    """An output tensor with GUARD_BYTES of sentinel bytes right before and
    right after it in the same allocation.  A kernel that stores past either
    end of the output (a ragged edge tile that does not mask its rows or
    columns) overwrites a sentinel; check() then fails."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((n + 2 * GUARD_BYTES,), SENTINEL, dtype=torch.uint8, device=device)
        self.t = self.buf[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, name="output"):
        torch.cuda.synchronize()
        head = self.buf[:GUARD_BYTES]
        tail = self.buf[GUARD_BYTES + self.n:]
        bad_head = int((head != SENTINEL).sum())
        bad_tail = int((tail != SENTINEL).sum())
        assert bad_head == 0 and bad_tail == 0, \
            f"{name}: {bad_head} guard bytes before and {bad_tail} after the tensor were overwritten"


def guarded(shape, dtype, device="cuda", fill=float("nan")):
    """(tensor, Guarded) with the tensor pre-filled (NaN by default, so an
    element that no kernel writes fails the parity check)."""
    g = Guarded(shape, dtype, device, fill)
    return g.t, g
