"""Helpers shared by the GPU parity tests (tolerances, conversions)."""
import numpy as np
import torch

# Tolerances of the parity bar (per quantity).
TOL_GAUSS = 2e-6        # absolute, eps
TOL_LOSS = 2e-5         # absolute, clean loss and rewards (perturbed loss = loss - reward)
TOL_G = 1e-4            # relative Frobenius, g
TOL_GW_BF16 = 2e-3      # relative Frobenius, G_W with bf16 GEMM operands
TOL_GW_F32 = 1e-5       # relative Frobenius, G_W on the fp32 path


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


def to_dev(x, dtype, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        return t.to(torch.bfloat16).to(device)
    if dtype == "i32":
        return t.to(torch.int32).to(device)
    return t.to(torch.float32).to(device)


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()
