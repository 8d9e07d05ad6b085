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


def err_msr(gpu, ref, y_ref, g, heads, eps=1e-5, bf16_out=False):
    """Error of an MSR output against the oracle's ``ref`` = swish(g) (.) GroupNorm(y_ref), in
    units of the bar that the retention output y itself meets.

    If y carries errors |dy| <= tol * rms(y) (the chunkwise bar), then within one (token, head)
    row of mean m and deviation sd, the normalised value y^ = (y - m) / sd moves by at most
    tol * rms(y) * (2 + |y^|) / sd (one term for dy, one for dm, |y^| for d sd; m and sd are
    1-Lipschitz in the row's max norm), and the output by |swish(g)| times that.  Returned: the
    smallest tol that explains the observed differences, max over elements of
    |out - ref| * sd_row / (rms(y) * (2 + |y^|) * |swish(g)|), net of a bf16 output's own
    rounding when bf16_out.  (m, sd, y^ and swish(g) here only size the bound.)
    """
    y = np.asarray(y_ref, dtype=np.float64)
    dv = y.shape[-1]
    rows = y.reshape(-1, heads, dv)
    gg = np.asarray(g.double().numpy() if hasattr(g, "double") else g, dtype=np.float64).reshape(rows.shape)
    r = np.asarray(ref, dtype=np.float64).reshape(rows.shape)
    m = rows.mean(axis=-1, keepdims=True)
    sd = np.sqrt(((rows - m) ** 2).mean(axis=-1, keepdims=True) + eps)
    yh = (rows - m) / sd
    sw = np.abs(gg / (1.0 + np.exp(-gg)))
    out = gpu.detach().double().cpu().numpy().reshape(rows.shape)
    diff = np.abs(out - r)
    if bf16_out:
        diff = np.maximum(diff - 2.0 ** -8 * np.abs(r), 0.0)
    rms_y = float(np.sqrt((y ** 2).mean()))
    scale = rms_y * (2.0 + np.abs(yh)) * sw / sd
    ok = scale > 0
    if not ok.all() and diff[~ok].max() > 0:
        return float("inf")
    return float((diff[ok] / scale[ok]).max())
