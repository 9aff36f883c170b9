"""Shared helpers of the GPU parity tests (no arithmetic of the method lives here)."""
import numpy as np
import pytest
import torch

import seeded

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

BF16_ATOL = 2e-2      # bf16 logits / attention outputs
F32_ATOL = 1e-4       # fp32 configuration
LOSS_RTOL = 1e-3      # loss, relative


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def model_inputs(name: str, stress: bool = False, B=None, T=None, ignore_frac=0.0, **over):
    """(cfg dict, stored weights, fp64 weights, idx, targets) for a named workload."""
    w = seeded.WORKLOADS[name]
    cfg = dict(w.model_dict(), **over)
    W = seeded.make_weights(cfg, stress=stress)
    B = B or w.batch
    T = T or w.seq_len
    idx, tgt = seeded.make_tokens(B, T, w.token_high, ignore_frac=ignore_frac)
    return cfg, W, seeded.to_f64(W), idx, tgt
