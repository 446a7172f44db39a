"""Helpers shared by the GPU parity tests: device transfer and comparison metrics."""
import numpy as np
import torch

# Tolerances: max-abs-error / max|ref|
TOL_FP32 = 1e-4
TOL_BF16 = 2e-2
# relative tolerance of P_i and the auxiliary loss
TOL_STATS = 1e-5
# routing of GPU-computed logits is compared on tokens whose fp64 top-k margin exceeds this
MARGIN = 1e-5


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda().contiguous()


def host(t):
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def norm_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def torch_dtype(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def tol(name):
    return TOL_BF16 if name == "bf16" else TOL_FP32
