"""Host-side checks of the C interface (no GPU needed, no compute calls).

The library must load here, export every function include/retnet.h declares, and reject
bad arguments with the documented status before it touches a device.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import linear_attention_sequence_chunkwise_b200 as rn
from linear_attention_sequence_chunkwise_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "retnet.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return rn.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RETNET_API\s+[\w\s\*]+?\b(retnet_\w+)\s*\(", text)))


def test_header_declares_the_interface():
    names = declared_functions()
    assert set(names) == set(rn.EXPORTS), names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (retnet_\w+)", out.stdout))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_header_compiles_as_c():
    src = '#include "retnet.h"\nint main(void){ retnet_dims_t d = {1,2,3,4,5}; return (int)d.batch - 1; }\n'
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-x", "c", "-",
                        "-fsyntax-only"], input=src, text=True, capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings(lib):
    for code in range(7):
        s = rn.retnet_status_string(code)
        assert isinstance(s, str) and len(s) > 0
    assert rn.retnet_status_string(99) == "unknown status"
    assert lib.retnet_version() >= 100


# Fake, never-dereferenced device addresses: every call below must fail validation first.
FAKE = 0x10000


def _gamma(h, val=0.9):
    return np.full(h, val, dtype=np.float32)


def _par(lib, dims, gamma, theta=None, flags=0, q=FAKE, in_dt=0, out_dt=0, pos0=0):
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    th = None if theta is None else np.ascontiguousarray(theta, dtype=np.float32)
    return lib.retnet_retention_parallel(q, FAKE, FAKE, FAKE, rn.Dims(*dims), in_dt, out_dt,
                                         g.ctypes.data_as(rn._fp), None if th is None else th.ctypes.data_as(rn._fp),
                                         pos0, flags, None)


def test_parallel_validation(lib):
    ok = (1, 8, 2, 4, 4)
    assert _par(lib, ok, _gamma(2), q=0) == 1                            # NULL q
    assert _par(lib, (0, 8, 2, 4, 4), _gamma(2)) == 2                    # batch 0
    assert _par(lib, (1, 8, 2, 0, 4), _gamma(2)) == 2                    # d_k 0
    assert _par(lib, (1, 8, 2, 4, 2000), _gamma(2)) == 2                 # d_v over the limit
    assert _par(lib, (1, 8, 300, 4, 4), _gamma(300)) == 2                # heads over the limit
    assert _par(lib, ok, _gamma(2), in_dt=7) == 3                        # bad dtype
    assert _par(lib, ok, _gamma(2, 1.0)) == 4                            # gamma = 1
    assert _par(lib, ok, _gamma(2, 0.0)) == 4                            # gamma = 0
    assert _par(lib, ok, np.array([0.9, np.nan], np.float32)) == 4       # gamma NaN
    assert _par(lib, ok, _gamma(2), flags=32) == 4                       # unknown flag bit
    assert _par(lib, (1, 8, 2, 5, 4), _gamma(2), np.ones(2), flags=rn.F_XPOS) == 4  # odd d_k with xPos
    assert _par(lib, ok, _gamma(2), None, flags=rn.F_XPOS) == 1          # xPos without theta
    assert _par(lib, ok, _gamma(2), np.array([1.0, np.inf]), flags=rn.F_XPOS) == 4  # theta inf
    assert _par(lib, ok, _gamma(2), pos0=-1) == 4                        # negative position
    assert _par(lib, (1, 0, 2, 4, 4), _gamma(2)) == 0                    # empty sequence: no work


def test_chunkwise_and_step_validation(lib):
    g = _gamma(2)
    gp = g.ctypes.data_as(rn._fp)
    d = rn.Dims(1, 8, 2, 4, 4)
    # chunk <= 0
    assert lib.retnet_retention_chunkwise(FAKE, FAKE, FAKE, FAKE, d, 0, 0, gp, None, 0, 0, 0, None, None, None,
                                          None, None) == 4
    # NULL o
    assert lib.retnet_retention_chunkwise(FAKE, FAKE, FAKE, None, d, 0, 0, gp, None, 0, 0, 16, None, None, None,
                                          None, None) == 1
    # step: NORM_R without z
    assert lib.retnet_retention_step(FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 4, 0, 0, FAKE, None, gp, None, 0,
                                     rn.F_NORM_R, None) == 5
    # step: misaligned state
    assert lib.retnet_retention_step(FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 4, 0, 0, FAKE + 4, None, gp, None, 0, 0,
                                     None) == 4
    # step: NULL state
    assert lib.retnet_retention_step(FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 4, 0, 0, None, None, gp, None, 0, 0,
                                     None) == 1
    # step: negative position
    assert lib.retnet_retention_step(FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 4, 0, 0, FAKE, None, gp, None, -3, 0,
                                     None) == 4


def test_chunkwise_workspace_entry_points(lib):
    """Workspace size is the documented bound; the workspace variant validates like the plain call
    and rejects a misaligned workspace before touching a device."""
    a256 = lambda x: (x + 255) // 256 * 256
    for dims in ((2, 100, 3, 128, 64), (1, 4096, 2, 64, 128), (2, 1000, 3, 256, 128), (2, 8192, 16, 256, 512)):
        b, L, h, dk, dv = dims
        states = 6 * b * h * dk * dv * 4
        copies = 4 * a256(b * L * h * dk * 2) + a256(b * L * h * dv * 2)  # q~, k~ hi and lo; v
        # d_k 256: the P pass's tiles (at most 36 tiles of 64 x 64 fp16 per 512 tokens) after single copies
        ptiles = a256(b * h * ((L + 511) // 512) * 36 * 64 * 64 * 2) if dk == 256 else 0
        single = 2 * a256(b * L * h * dk * 2) + a256(b * L * h * dv * 2)
        rden = a256(b * L * h * 4) + a256(b * h * dk * 64 * 4)  # R~ row factors and key-sum segments, in front
        assert rn.retnet_chunkwise_workspace_size(dims) == rden + max(states, copies, single + ptiles)
    assert rn.retnet_chunkwise_workspace_size((0, 0, 0, 0, 0)) == 0
    out = ctypes.c_size_t(0)
    assert lib.retnet_chunkwise_workspace_size(rn.Dims(1, 8, -2, 4, 4), ctypes.byref(out)) == 2
    assert lib.retnet_chunkwise_workspace_size(rn.Dims(1, 8, 2, 4, 4), None) == 1
    g = _gamma(2)
    gp = g.ctypes.data_as(rn._fp)
    d = rn.Dims(1, 8, 2, 4, 4)
    # chunk <= 0, NULL o: as the plain call
    assert lib.retnet_retention_chunkwise_ws(FAKE, FAKE, FAKE, FAKE, d, 0, 0, gp, None, 0, 0, 0, None, None, None,
                                             None, FAKE, 4096, None) == 4
    assert lib.retnet_retention_chunkwise_ws(FAKE, FAKE, FAKE, None, d, 0, 0, gp, None, 0, 0, 16, None, None, None,
                                             None, FAKE, 4096, None) == 1
    # misaligned workspace
    assert lib.retnet_retention_chunkwise_ws(FAKE, FAKE, FAKE, FAKE, d, 0, 0, gp, None, 0, 0, 16, None, None, None,
                                             None, FAKE + 8, 4096, None) == 4


def test_static_scratch_entry_point_limits(lib):
    """The allocation-free chunkwise call rejects, before touching a device, a call whose one
    segment state exceeds the static scratch; the header and the binding agree on its size."""
    m = re.search(r"#define RETNET_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(HEADER).read())
    assert m and int(m.group(1)) << int(m.group(2)) == rn.STATIC_SCRATCH_BYTES
    g = _gamma(16)
    gp = g.ctypes.data_as(rn._fp)
    big = rn.Dims(64, 8, 16, 256, 512)  # one state = 512 MiB
    assert lib.retnet_retention_chunkwise_static(FAKE, FAKE, FAKE, FAKE, big, 1, 1, gp, None, 0, 0, 64, None, None,
                                                 None, None, None) == 5


def test_epilogue_validation(lib):
    f = lib.retnet_msr_epilogue
    assert f(FAKE, FAKE, FAKE, 4, 2, 12, 1e-5, 0, 0, None) == 2          # d_v not a multiple of 8
    assert f(FAKE, FAKE, FAKE, 4, 2, 16, -1.0, 0, 0, None) == 4          # eps < 0
    assert f(FAKE, FAKE, FAKE, 4, 2, 16, float("nan"), 0, 0, None) == 4  # eps NaN
    assert f(None, FAKE, FAKE, 4, 2, 16, 1e-5, 0, 0, None) == 1          # NULL y
    assert f(FAKE + 2, FAKE, FAKE, 4, 2, 16, 1e-5, 0, 0, None) == 4      # misaligned
    assert f(FAKE, FAKE, FAKE, 4, 2, 16, 1e-5, 5, 0, None) == 3          # bad dtype
    assert f(FAKE, FAKE, FAKE, 0, 2, 16, 1e-5, 0, 0, None) == 0          # no tokens: no work


def test_fused_msr_validation(lib):
    """The fused MSR entry point checks eps, the gate pointer and, for R~, that there is a
    workspace for the row factors, on the host."""
    g = _gamma(2)
    gp = g.ctypes.data_as(rn._fp)
    d = rn.Dims(1, 64, 2, 128, 128)
    f = lib.retnet_msr_chunkwise
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, d, 1, 0, gp, None, 0, 0, 64, -1.0, None, None, None, 0, None) == 4
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, d, 1, 0, gp, None, 0, 0, 64, float("inf"), None, None, None, 0,
             None) == 4
    assert f(FAKE, FAKE, FAKE, None, FAKE, d, 1, 0, gp, None, 0, 0, 64, 1e-5, None, None, None, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, d, 1, 0, gp, None, 0, rn.F_NORM_R, 64, 1e-5, None, None, None, 0,
             None) == 5
    assert lib.retnet_msr_chunkwise_launches(d, 1, rn.F_NORM_R, 64, gp, 0) == -5
    assert lib.retnet_msr_chunkwise_launches(rn.Dims(1, 64, 2, 128, 128), 1, 0, 0, gp, 0) == -4  # chunk 0


def test_backward_validation(lib):
    """The gradient entry point: workspace size formula, R~ unsupported, NULL and workspace
    checks before any device access."""
    assert rn.retnet_backward_workspace_size((2, 10, 3, 64, 32)) >= 2 * 4 * 2 * 10 * 3 * 64  # CUDA-core path
    g = _gamma(2)
    gp = g.ctypes.data_as(rn._fp)
    d = rn.Dims(1, 8, 2, 64, 64)
    f = lib.retnet_retention_backward
    args = lambda q=FAKE, ws=FAKE, wsb=1 << 20, flags=0: (q, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, 0, gp, None, 0,
                                                          flags, None, None, ws, wsb, None)
    assert f(*args(flags=rn.F_NORM_R)) == 5
    assert f(*args(q=None)) == 1
    assert f(*args(ws=None)) == 1
    assert f(*args(wsb=16)) == 4
    assert f(*args(ws=FAKE + 8)) == 4
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, rn.Dims(1, 8, 2, 512, 64), 0, gp, None, 0, 0, None, None,
             FAKE, 1 << 30, None) == 5  # d_k beyond the gradient kernels' 256


def test_binding_raises_without_library(tmp_path):
    import importlib
    mod = importlib.import_module("linear_attention_sequence_chunkwise_b200")
    saved = mod._lib
    try:
        mod._lib = None
        with pytest.raises(RuntimeError, match="not found"):
            mod.load(str(tmp_path / "missing.so"))
    finally:
        mod._lib = saved


def test_chunkwise_kernel_choice(lib):
    g8 = np.array([1.0 - 2.0 ** (-5 - i) for i in range(8)], np.float32)
    f = rn.F_XPOS | rn.F_SCALE_SQRT_D | rn.F_NORM_D
    assert rn.retnet_chunkwise_kernel((8, 2048, 8, 128), 128, rn.BF16, f, 64, g8) == 1
    assert rn.retnet_chunkwise_kernel((2, 8192, 8, 256), 512, rn.BF16, f, 128, g8) == 1
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 64), 64, rn.BF16, f, 128, g8) == 1
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 128), 128, rn.F32, f, 64, g8) == 0      # fp32 inputs
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 128), 128, rn.BF16, f | rn.F_NORM_R, 64, g8) == 0
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 96), 128, rn.BF16, f, 64, g8) == 0      # d_k 96
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 128), 96, rn.BF16, f, 64, g8) == 0      # d_v 96
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 128), 128, rn.BF16, f, 32, g8) == 0     # chunk 32
    assert rn.retnet_chunkwise_kernel((4, 4096, 8, 256), 256, rn.BF16, f, 256, g8) == 1  # chunk 256
    assert rn.retnet_chunkwise_kernel((2, 8192, 8, 256), 512, rn.BF16, f, 512, g8) == 1  # chunk 512
    assert rn.retnet_chunkwise_kernel((1, 64, 8, 128), 128, rn.BF16, f, 384, g8) == 0    # chunk 384
    # gamma^B < 2^-12 for some head: the scaled tensor-core form does not apply
    assert rn.retnet_chunkwise_kernel((1, 64, 2, 128), 128, rn.BF16, f, 128, np.array([0.9, 0.99], np.float32)) == 0
    assert rn.retnet_chunkwise_kernel((1, 64, 2, 128), 128, rn.BF16, f, 0, g8) == -4
    assert rn.retnet_chunkwise_kernel((1, 64, 2, 128), 128, 9, f, 64, g8) == -3
