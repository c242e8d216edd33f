"""Shared test helpers: the error metric and the parity tolerances."""
from __future__ import annotations

import numpy as np
import torch



def rel_frob(x, ref) -> float:
    """||x - ref||_F / ||ref||_F over the whole tensor (float64)."""
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = ref.detach().double().cpu().numpy() if hasattr(ref, "detach") else np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
