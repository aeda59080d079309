"""Shared helpers for the parity tests (no method arithmetic here)."""
import numpy as np
import torch

# Tolerances on relative L2 error, as the target statement fixes them:
# fp32 path 1e-4; bf16 inputs with fp32 accumulation 2e-2.
REL_F32 = 1e-4
REL_BF16 = 2e-2
# Two retained sets may differ only where the boundary scores differ by less
# than this, relative to the larger score.
TIE_REL = 1e-4


def rel_l2(got, want) -> float:
    g = np.asarray(got.detach().cpu().double() if hasattr(got, "detach") else got, np.float64)
    w = np.asarray(want, np.float64)
    return float(np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-300))


def cuda(*ts):
    out = tuple(t.cuda() for t in ts)
    return out if len(out) > 1 else out[0]


def tol(dtype: str) -> float:
    return REL_F32 if dtype == "f32" else REL_BF16


def allowed_swap(scores: np.ndarray, keep_a, keep_b, m: int) -> bool:
    """Two kept sets of size m from one candidate list may differ only inside
    the band of candidates whose score is within TIE_REL (relative) of the
    m-th largest score."""
    a, b = set(int(x) for x in keep_a), set(int(x) for x in keep_b)
    if a == b:
        return True
    if m == 0 or m >= len(scores):
        return False
    boundary = np.sort(scores)[::-1][m - 1]
    for j in a ^ b:
        if abs(scores[j] - boundary) > TIE_REL * max(abs(scores[j]), abs(boundary)):
            return False
    return True


def set_seed(seed: int = 0) -> None:
    torch.manual_seed(seed)
