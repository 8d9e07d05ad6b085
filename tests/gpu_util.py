"""Helpers for the GPU parity tests: error metric, oracle-side fp64 views, device copies."""
import numpy as np
import pytest
import torch


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def err(gpu, ref):
    """max|gpu - ref| / rms(ref), in fp64."""
    g = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt((r ** 2).mean()))
    return float(np.abs(g - r).max() / max(rms, 1e-300))


def dev(t):
    return t.contiguous().cuda()


def bf16_round(x):
    """Round an fp64 array to bf16 (RNE) and back, as the GPU's bf16 output does."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


# Tolerances: BASELINE-stated max|err|/rms(ref) bars for the raw and post-epilogue outputs.
TOL_F32 = 1e-4
TOL_BF16 = 1e-2
