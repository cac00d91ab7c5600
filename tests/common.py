"""Helpers shared by the test files (no arithmetic of the method lives here)."""
import numpy as np
import torch


def rel_l2(x, ref) -> float:
    """||x - ref||_2 / ||ref||_2 in float64."""
    x = np.asarray(x.detach().double().cpu().numpy() if hasattr(x, "detach") else x,
                   dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


# Tolerances on relative L2 error against the fp64 oracle: fp32 inputs and
# bf16 q/k/v (with fp32 gates and state).
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to_cuda(d):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in d.items()}


def cpu(d):
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in d.items()}
