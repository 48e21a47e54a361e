"""Shared helpers for the GPU parity tests (comparison metrics, tolerances)."""
import numpy as np
import torch

# bf16 storage, fp32 accumulation: relative Frobenius error of every GEMM
# output and gradient against the fp64 oracle.
TOL_BF16 = 2e-2
# fp32 CUDA-core path (tiny fp32 configuration); the inputs are exact fp32
# values, so only fp32 accumulation order and the library's tanh/erf differ.
TOL_F32 = 1e-5
# fp32 cross-entropy: loss per token (relative) and dlogits (relative Frobenius)
TOL_XENT = 1e-4


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(gpu, ref):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / (den if den > 0 else 1.0))


def assert_close(name, gpu, ref, tol):
    e = rel_fro(gpu, ref)
    assert e <= tol, f"{name}: relative Frobenius error {e:.3e} > {tol:.1e}"
    return e


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
