"""The error measures the GPU parity tests apply, checked against their own definitions on the
CPU: a perturbation that meets the retention bar stays within the post-GroupNorm measure, and a
correct value rounded to bf16 has no excess over the bf16-output allowance."""
import numpy as np
import torch

import oracle
import synth_inputs as si
from gpu_util import bf16_round, err_bf16_out, err_msr


def test_err_msr_bounds_a_perturbation_at_the_retention_bar():
    rng = np.random.default_rng(5)
    b, L, h, dv = 2, 40, 3, 64
    y = rng.standard_normal((b, L, h, dv)) * rng.uniform(0.1, 3.0, (b, L, h, 1))  # rows of mixed size
    g = si.randn((b, L, h, dv), 6, "bf16")
    ref = oracle.msr_epilogue(y, g, h, eps=1e-5)
    rms = np.sqrt((y ** 2).mean())
    for tol in (1e-3, 1e-2):
        for trial in range(3):
            dy = rng.choice([-1.0, 1.0], size=y.shape) * tol * rms * rng.uniform(0.5, 1.0, y.shape)
            out = oracle.msr_epilogue(y + dy, g, h, eps=1e-5)
            assert err_msr(torch.from_numpy(out), ref, y, g, h) <= tol * (1 + 1e-9)
    # and a real error shows: a wrong mean (a constant shift of the output rows) is far above
    bad = ref + 0.05
    assert err_msr(torch.from_numpy(bad), ref, y, g, h) > 1e-2


def test_bf16_output_allowance():
    rng = np.random.default_rng(7)
    ref = rng.standard_normal((50, 64)) * 3
    rounded = torch.from_numpy(bf16_round(ref)).float()
    assert err_bf16_out(rounded, ref) == 0.0
    assert err_bf16_out(rounded + 0.1, ref) > 1e-2
