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


def err_bf16_out(gpu, ref):
    """Error of a bf16 OUTPUT against the fp64 reference, net of the output's own rounding.

    Rounding a correct value to bf16 moves it by up to 2^-8 |ref| (8-bit significand, round to
    nearest), so each element's excess over that is what the max|err|/rms bar applies to.
    """
    g = gpu.detach().double().cpu().numpy()
    r = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt((r ** 2).mean()))
    excess = np.maximum(np.abs(g - r) - 2.0 ** -8 * np.abs(r), 0.0)
    return float(excess.max() / max(rms, 1e-300))


def bf16_round(x):
    """Round an fp64 array to bf16 (RNE) and back, as the GPU's bf16 output does."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


# Tolerances on max|err|/rms(ref), for the raw and the post-epilogue outputs: 1e-4 with fp32
# inputs, 1e-2 with bf16 inputs and fp32 accumulation.
TOL_F32 = 1e-4
TOL_BF16 = 1e-2
