"""RetNet multi-scale retention on B200 (sm_100a): Python binding of libretnet.so.

The compute lives in the CUDA kernels behind the C interface ``include/retnet.h``; this
module only marshals arguments (device pointers, sizes, dtype codes, the caller's stream)
and turns a non-zero status into an exception.  PyTorch is used for device memory and
streams.  There is no CPU path: if the library is missing, ``load()`` raises.

The functions carry the C names:
  retnet_retention_parallel   -- §2.3 Parallel Mode of "阅读笔记：RetNet" (mzeromiko blog)
  retnet_retention_chunkwise  -- §2.4 Chunkwise Recurrent Mode
  retnet_retention_step       -- §2.2 Recurrent Mode, one decode token for a batch
  retnet_msr_epilogue         -- §三.2 GroupNorm per head, then the swish gate
  retnet_msr_chunkwise        -- §2.4 and §三.2 in one kernel (the retention output stays on chip)
  retnet_retention_backward   -- gradient of the forward (dq, dk, dv, d state) for training
with the §三.3 normalisations chosen by flags.  Tensors are dense BLHD (see the header).
"""
import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libretnet.so")

F_XPOS = 1
F_SCALE_SQRT_D = 2
F_NORM_D = 4
F_NORM_R = 8
F_PRECISE = 16  # split fp16 operands (hi + lo) on the tensor-core kernel
F_ALL = F_XPOS | F_SCALE_SQRT_D | F_NORM_D | F_NORM_R
F32 = 0
BF16 = 1

STATUS = {0: "RETNET_OK", 1: "RETNET_ERR_NULL_PTR", 2: "RETNET_ERR_BAD_SHAPE", 3: "RETNET_ERR_BAD_DTYPE",
          4: "RETNET_ERR_BAD_PARAM", 5: "RETNET_ERR_UNSUPPORTED", 6: "RETNET_ERR_CUDA"}
STATIC_SCRATCH_BYTES = 16 << 20  # RETNET_STATIC_SCRATCH_BYTES
EXPORTS = ("retnet_retention_parallel", "retnet_retention_chunkwise", "retnet_retention_chunkwise_ws",
           "retnet_retention_chunkwise_static", "retnet_chunkwise_segment_state", "retnet_state_advance",
           "retnet_chunkwise_workspace_size", "retnet_retention_step", "retnet_msr_epilogue",
           "retnet_msr_chunkwise", "retnet_msr_chunkwise_launches", "retnet_retention_backward",
           "retnet_backward_workspace_size", "retnet_backward_kernel", "retnet_backward_launches",
           "retnet_chunkwise_kernel", "retnet_chunkwise_launches", "retnet_debug_wait_timeouts",
           "retnet_fp16_range_errors", "retnet_debug_set_wait_budget",
           "retnet_status_string", "retnet_version")


class RetnetError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("heads", ctypes.c_int64),
                ("d_k", ctypes.c_int64), ("d_v", ctypes.c_int64)]


_lib = None
_vp = ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_u32 = ctypes.c_uint32


def load(path: str = None):
    """Load libretnet.so (built in-tree by ``_build.build()``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libretnet.so not found at {path}: build it with "
                           "linear_attention_sequence_chunkwise_b200._build.build()")
    lib = ctypes.CDLL(path)
    lib.retnet_retention_parallel.argtypes = [_vp, _vp, _vp, _vp, Dims, _i32, _i32, _fp, _fp, _i64, _u32, _vp]
    lib.retnet_retention_chunkwise.argtypes = [_vp, _vp, _vp, _vp, Dims, _i32, _i32, _fp, _fp, _i64, _u32, _i64,
                                               _vp, _vp, _vp, _vp, _vp]
    lib.retnet_retention_chunkwise_ws.argtypes = [_vp, _vp, _vp, _vp, Dims, _i32, _i32, _fp, _fp, _i64, _u32,
                                                  _i64, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.retnet_retention_chunkwise_static.argtypes = [_vp, _vp, _vp, _vp, Dims, _i32, _i32, _fp, _fp, _i64, _u32,
                                                      _i64, _vp, _vp, _vp, _vp, _vp]
    lib.retnet_chunkwise_segment_state.argtypes = [_vp, _vp, Dims, _i32, _fp, _fp, _i64, _u32, _i64, _vp, _vp]
    lib.retnet_chunkwise_segment_state.restype = _i32
    lib.retnet_state_advance.argtypes = [_vp, _vp, _i64, _i64, _i64, _i64, _fp, _i64, _vp]
    lib.retnet_state_advance.restype = _i32
    lib.retnet_chunkwise_workspace_size.argtypes = [Dims, ctypes.POINTER(ctypes.c_size_t)]
    lib.retnet_chunkwise_workspace_size.restype = _i32
    lib.retnet_retention_step.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _fp,
                                          _fp, _i64, _u32, _vp]
    lib.retnet_msr_epilogue.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float, _i32, _i32, _vp]
    lib.retnet_msr_chunkwise.argtypes = [_vp, _vp, _vp, _vp, _vp, Dims, _i32, _i32, _fp, _fp, _i64, _u32, _i64,
                                         ctypes.c_float, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.retnet_msr_chunkwise_launches.argtypes = [Dims, _i32, _u32, _i64, _fp, ctypes.c_size_t]
    lib.retnet_retention_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, Dims, _i32, _fp, _fp, _i64, _u32,
                                              _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.retnet_retention_backward.restype = _i32
    lib.retnet_backward_workspace_size.argtypes = [Dims, ctypes.POINTER(ctypes.c_size_t)]
    lib.retnet_backward_workspace_size.restype = _i32
    lib.retnet_backward_kernel.argtypes = [Dims, _i32, _u32, _fp, ctypes.c_size_t]
    lib.retnet_backward_kernel.restype = _i32
    lib.retnet_backward_launches.argtypes = [Dims, _i32, _u32, _fp, ctypes.c_size_t, _i32, _i32]
    lib.retnet_backward_launches.restype = _i32
    lib.retnet_msr_chunkwise_launches.restype = _i32
    for name in ("retnet_retention_parallel", "retnet_retention_chunkwise", "retnet_retention_chunkwise_ws",
                 "retnet_retention_chunkwise_static", "retnet_retention_step", "retnet_msr_epilogue",
                 "retnet_msr_chunkwise"):
        getattr(lib, name).restype = _i32
    lib.retnet_chunkwise_kernel.argtypes = [Dims, _i32, _u32, _i64, _fp]
    lib.retnet_chunkwise_kernel.restype = _i32
    lib.retnet_chunkwise_launches.argtypes = [Dims, _i32, _u32, _i64, _fp, ctypes.c_size_t]
    lib.retnet_chunkwise_launches.restype = _i32
    lib.retnet_debug_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint), _i32]
    lib.retnet_debug_wait_timeouts.restype = _i32
    lib.retnet_fp16_range_errors.argtypes = [ctypes.POINTER(ctypes.c_uint), _i32]
    lib.retnet_fp16_range_errors.restype = _i32
    lib.retnet_debug_set_wait_budget.argtypes = [ctypes.c_longlong]
    lib.retnet_debug_set_wait_budget.restype = _i32
    lib.retnet_status_string.argtypes = [_i32]
    lib.retnet_status_string.restype = ctypes.c_char_p
    lib.retnet_version.argtypes = []
    lib.retnet_version.restype = _i32
    _lib = lib
    return lib


def retnet_status_string(status: int) -> str:
    return load().retnet_status_string(int(status)).decode()


def _check(status):
    if status != 0:
        raise RetnetError(status, retnet_status_string(status))


# ---- marshalling helpers ------------------------------------------------------------------

def _ptr(t):
    """Device pointer of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}: the library takes float32 or bfloat16")


def _require_cuda(*ts):
    for t in ts:
        if t is None or isinstance(t, int):
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (the library takes device pointers)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (dense BLHD layout)")


def _host_f32(a, n):
    """Host float32 array of at least n entries (kept alive by the caller's frame)."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    if arr.size < n:
        raise ValueError(f"parameter array has {arr.size} entries, needs {n}")
    return arr


def _fptr(arr):
    return None if arr is None else arr.ctypes.data_as(_fp)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---- the C entry points -------------------------------------------------------------------

def retnet_retention_parallel(q, k, v, o, gamma, theta=None, pos0=0, flags=F_ALL, stream=None):
    """Parallel form into ``o``: q,k (b,L,h,d_k), v,o (b,L,h,d_v); gamma (h,), theta (d_k/2,) on the host."""
    _require_cuda(q, k, v, o)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (b, L, h, dk) or tuple(v.shape) != (b, L, h, dv) or tuple(o.shape) != (b, L, h, dv):
        raise ValueError("shape mismatch between q, k, v, o")
    g = _host_f32(gamma, h)
    th = _host_f32(theta, dk // 2)
    _check(load().retnet_retention_parallel(_ptr(q), _ptr(k), _ptr(v), _ptr(o), Dims(b, L, h, dk, dv),
                                            _dtype_code(q), _dtype_code(o), _fptr(g), _fptr(th), int(pos0),
                                            int(flags), _stream(stream)))


def _chunkwise_args(q, k, v, o, gamma, theta, state_in, state_out, z_in, z_out):
    _require_cuda(q, k, v, o, state_in, state_out, z_in, z_out)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (b, L, h, dk) or tuple(v.shape) != (b, L, h, dv) or tuple(o.shape) != (b, L, h, dv):
        raise ValueError("shape mismatch between q, k, v, o")
    for s in (state_in, state_out):
        if s is not None and not isinstance(s, int) and tuple(s.shape) != (b, h, dk, dv):
            raise ValueError("state must be (batch, heads, d_k, d_v) float32")
    for z in (z_in, z_out):
        if z is not None and not isinstance(z, int) and tuple(z.shape) != (b, h, dk):
            raise ValueError("z must be (batch, heads, d_k) float32")
    return Dims(b, L, h, dk, dv), _host_f32(gamma, h), _host_f32(theta, dk // 2)


def retnet_chunkwise_workspace_size(dims) -> int:
    """Bytes of workspace for retnet_retention_chunkwise_ws; dims = (batch, seqlen, heads, d_k, d_v)."""
    out = ctypes.c_size_t(0)
    _check(load().retnet_chunkwise_workspace_size(Dims(*[int(x) for x in dims]), ctypes.byref(out)))
    return out.value


def retnet_retention_chunkwise_ws(q, k, v, o, gamma, theta=None, pos0=0, flags=F_ALL, chunk=64, state_in=None,
                                  state_out=None, z_in=None, z_out=None, workspace=None, stream=None):
    """Chunkwise form with a caller-owned device workspace (a uint8 CUDA tensor, or None)."""
    d, g, th = _chunkwise_args(q, k, v, o, gamma, theta, state_in, state_out, z_in, z_out)
    _require_cuda(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().retnet_retention_chunkwise_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(o), d, _dtype_code(q),
                                                _dtype_code(o), _fptr(g), _fptr(th), int(pos0), int(flags),
                                                int(chunk), _ptr(state_in), _ptr(state_out), _ptr(z_in),
                                                _ptr(z_out), _ptr(workspace), ws_bytes, _stream(stream)))


def retnet_retention_chunkwise_static(q, k, v, o, gamma, theta=None, pos0=0, flags=F_ALL, chunk=64, state_in=None,
                                      state_out=None, z_in=None, z_out=None, stream=None):
    """Chunkwise form with the library's static device scratch (no workspace argument, no
    allocation); calls that overlap on the GPU race on the scratch -- see the C header."""
    d, g, th = _chunkwise_args(q, k, v, o, gamma, theta, state_in, state_out, z_in, z_out)
    _check(load().retnet_retention_chunkwise_static(_ptr(q), _ptr(k), _ptr(v), _ptr(o), d, _dtype_code(q),
                                                    _dtype_code(o), _fptr(g), _fptr(th), int(pos0), int(flags),
                                                    int(chunk), _ptr(state_in), _ptr(state_out), _ptr(z_in),
                                                    _ptr(z_out), _stream(stream)))


def retnet_chunkwise_segment_state(k, v, state_out, gamma, theta=None, pos0=0, flags=F_ALL, chunk=64, stream=None):
    """State a sequence's chunks leave behind from a zero start (no outputs): k (b,L,h,d_k),
    v (b,L,h,d_v) bf16; state_out (b,h,d_k,d_v) float32."""
    _require_cuda(k, v, state_out)
    b, L, h, dk = k.shape
    dv = v.shape[-1]
    if tuple(v.shape) != (b, L, h, dv) or tuple(state_out.shape) != (b, h, dk, dv):
        raise ValueError("shape mismatch between k, v, state_out")
    g = _host_f32(gamma, h)
    th = _host_f32(theta, dk // 2)
    _check(load().retnet_chunkwise_segment_state(_ptr(k), _ptr(v), Dims(b, L, h, dk, dv), _dtype_code(k), _fptr(g),
                                                 _fptr(th), int(pos0), int(flags), int(chunk), _ptr(state_out),
                                                 _stream(stream)))


def retnet_state_advance(state, w, gamma, length, stream=None):
    """state <- gamma^length * state + w in place (both (b,h,d_k,d_v) float32 CUDA tensors)."""
    _require_cuda(state, w)
    b, h, dk, dv = state.shape
    if tuple(w.shape) != (b, h, dk, dv):
        raise ValueError("state and w must have the same shape")
    g = _host_f32(gamma, h)
    _check(load().retnet_state_advance(_ptr(state), _ptr(w), b, h, dk, dv, _fptr(g), int(length), _stream(stream)))


def retnet_retention_chunkwise(q, k, v, o, gamma, theta=None, pos0=0, flags=F_ALL, chunk=64, state_in=None,
                               state_out=None, z_in=None, z_out=None, stream=None):
    """Chunkwise form into ``o`` (and ``state_out``/``z_out`` when given); see the C header."""
    _require_cuda(q, k, v, o, state_in, state_out, z_in, z_out)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (b, L, h, dk) or tuple(v.shape) != (b, L, h, dv) or tuple(o.shape) != (b, L, h, dv):
        raise ValueError("shape mismatch between q, k, v, o")
    for s in (state_in, state_out):
        if s is not None and not isinstance(s, int) and tuple(s.shape) != (b, h, dk, dv):
            raise ValueError("state must be (batch, heads, d_k, d_v) float32")
    for z in (z_in, z_out):
        if z is not None and not isinstance(z, int) and tuple(z.shape) != (b, h, dk):
            raise ValueError("z must be (batch, heads, d_k) float32")
    g = _host_f32(gamma, h)
    th = _host_f32(theta, dk // 2)
    _check(load().retnet_retention_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(o), Dims(b, L, h, dk, dv),
                                             _dtype_code(q), _dtype_code(o), _fptr(g), _fptr(th), int(pos0),
                                             int(flags), int(chunk), _ptr(state_in), _ptr(state_out),
                                             _ptr(z_in), _ptr(z_out), _stream(stream)))


def retnet_retention_step(q, k, v, o, state, gamma, theta=None, pos=0, flags=F_ALL, z=None, stream=None):
    """One decode step in place on ``state``: q,k (b,h,d_k), v,o (b,h,d_v), state (b,h,d_k,d_v) fp32."""
    _require_cuda(q, k, v, o, state, z)
    b, h, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (b, h, dk) or tuple(v.shape) != (b, h, dv) or tuple(o.shape) != (b, h, dv):
        raise ValueError("shape mismatch between q, k, v, o")
    if tuple(state.shape) != (b, h, dk, dv):
        raise ValueError("state must be (batch, heads, d_k, d_v) float32")
    g = _host_f32(gamma, h)
    th = _host_f32(theta, dk // 2)
    _check(load().retnet_retention_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o), b, h, dk, dv, _dtype_code(q),
                                        _dtype_code(o), _ptr(state), _ptr(z), _fptr(g), _fptr(th), int(pos),
                                        int(flags), _stream(stream)))


def retnet_msr_epilogue(y, g, out, heads, eps=1e-5, stream=None):
    """GroupNorm per (token, head) row of d_v values, times swish(g), into ``out`` (shape of y)."""
    _require_cuda(y, g, out)
    if tuple(g.shape) != tuple(y.shape) or tuple(out.shape) != tuple(y.shape):
        raise ValueError("y, g and out must have one shape")
    if g.dtype != y.dtype:
        raise ValueError("y and g must have one dtype (the C call reads both as in_dtype)")
    total = y.numel()
    last = y.shape[-1]
    dv = last if (y.dim() >= 2 and y.shape[-2] == heads) else last // heads
    tokens = total // (heads * dv)
    _check(load().retnet_msr_epilogue(_ptr(y), _ptr(g), _ptr(out), tokens, heads, dv, float(eps), _dtype_code(y),
                                      _dtype_code(out), _stream(stream)))


def retnet_msr_chunkwise(q, k, v, g, out, gamma, theta=None, pos0=0, flags=F_XPOS | F_SCALE_SQRT_D | F_NORM_D,
                         chunk=64, eps=1e-5, state_in=None, state_out=None, workspace=None, stream=None):
    """swish(g) (.) GroupNorm_h(chunkwise retention) into ``out`` in one fused kernel: q,k (b,L,h,d_k),
    v,g,out (b,L,h,d_v); raises with RETNET_ERR_UNSUPPORTED for shapes the fused kernel does not take."""
    d, gm, th = _chunkwise_args(q, k, v, out, gamma, theta, state_in, state_out, None, None)
    _require_cuda(g, workspace)
    if tuple(g.shape) != tuple(v.shape) or g.dtype != q.dtype:
        raise ValueError("g must have the shape of v and the dtype of q")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().retnet_msr_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out), d, _dtype_code(q),
                                       _dtype_code(out), _fptr(gm), _fptr(th), int(pos0), int(flags), int(chunk),
                                       float(eps), _ptr(state_in), _ptr(state_out), _ptr(workspace), ws_bytes,
                                       _stream(stream)))


def retnet_msr_chunkwise_launches(shape_qk, d_v, in_dtype, flags, chunk, gamma, workspace_bytes=0):
    """Kernel launches retnet_msr_chunkwise makes (negative: the negated status it would return)."""
    b, L, h, dk = shape_qk
    gm = _host_f32(gamma, h)
    return load().retnet_msr_chunkwise_launches(Dims(b, L, h, dk, d_v), int(in_dtype), int(flags), int(chunk),
                                                _fptr(gm), int(workspace_bytes))


def retnet_backward_workspace_size(dims) -> int:
    """Bytes of workspace for retnet_retention_backward; dims = (batch, seqlen, heads, d_k, d_v)."""
    out = ctypes.c_size_t(0)
    _check(load().retnet_backward_workspace_size(Dims(*[int(x) for x in dims]), ctypes.byref(out)))
    return out.value


def retnet_backward_kernel(shape_qk, d_v, in_dtype, flags, gamma, workspace_bytes):
    """1 if a gradient call of this shape runs on the tensor cores, 0 for the CUDA-core path."""
    b, L, h, dk = shape_qk
    return load().retnet_backward_kernel(Dims(b, L, h, dk, d_v), int(in_dtype), int(flags),
                                         _fptr(_host_f32(gamma, h)), int(workspace_bytes))


def retnet_backward_launches(shape_qk, d_v, in_dtype, flags, gamma, workspace_bytes, with_state=False,
                             with_dstate=False):
    """Kernel launches of a gradient call (negative: the negated status it would return)."""
    b, L, h, dk = shape_qk
    return load().retnet_backward_launches(Dims(b, L, h, dk, d_v), int(in_dtype), int(flags),
                                           _fptr(_host_f32(gamma, h)), int(workspace_bytes), int(bool(with_state)),
                                           int(bool(with_dstate)))


def retnet_retention_backward(q, k, v, dout, dq, dk, dv, gamma, theta=None, pos0=0,
                              flags=F_XPOS | F_SCALE_SQRT_D | F_NORM_D, state_in=None, dstate=None, workspace=None,
                              stream=None):
    """Gradient of the forward into fp32 dq, dk (shape of q), dv (shape of v) and dstate
    (batch, heads, d_k, d_v) if given; dout has v's shape and q's dtype."""
    _require_cuda(q, k, v, dout, dq, dk, dv, state_in, dstate, workspace)
    b, L, h, d_k = q.shape
    d_v = v.shape[-1]
    for t, shp in ((k, q.shape), (dq, q.shape), (dk, q.shape), (v, (b, L, h, d_v)), (dout, (b, L, h, d_v)),
                   (dv, (b, L, h, d_v))):
        if tuple(t.shape) != tuple(shp):
            raise ValueError("shape mismatch between q, k, v, dout and the gradients")
    if dout.dtype != q.dtype:
        raise ValueError("dout must have the dtype of q")
    dims = (b, L, h, d_k, d_v)
    if workspace is None:
        import torch
        workspace = torch.empty(retnet_backward_workspace_size(dims), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    gm, th = _host_f32(gamma, h), _host_f32(theta, d_k // 2)
    _check(load().retnet_retention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                            Dims(*dims), _dtype_code(q), _fptr(gm), _fptr(th), int(pos0), int(flags),
                                            _ptr(state_in), _ptr(dstate), _ptr(workspace), ws_bytes,
                                            _stream(stream)))


def retnet_chunkwise_kernel(shape_qk, d_v, in_dtype, flags, chunk, gamma):
    """1 if a chunkwise call of this shape runs on the tensor-core kernel, 0 for the CUDA-core
    kernel, negative (-status) if it would be rejected.  shape_qk = (batch, L, heads, d_k)."""
    b, L, h, dk = shape_qk
    g = _host_f32(gamma, h)
    return load().retnet_chunkwise_kernel(Dims(b, L, h, dk, d_v), int(in_dtype), int(flags), int(chunk), _fptr(g))


def retnet_chunkwise_launches(shape_qk, d_v, in_dtype, flags, chunk, gamma, workspace_bytes=0):
    """Kernel launches of a chunkwise call on the current device (2 = two-pass segments),
    negative (-status) if it would be rejected.  shape_qk = (batch, L, heads, d_k)."""
    b, L, h, dk = shape_qk
    g = _host_f32(gamma, h)
    return load().retnet_chunkwise_launches(Dims(b, L, h, dk, d_v), int(in_dtype), int(flags), int(chunk), _fptr(g),
                                            int(workspace_bytes))


def retnet_debug_wait_timeouts(clear=True):
    """Bounded waits that gave up in the tensor-core kernel since the last clear (synchronises)."""
    c = ctypes.c_uint(0)
    _check(load().retnet_debug_wait_timeouts(ctypes.byref(c), 1 if clear else 0))
    return c.value


def retnet_debug_set_wait_budget(cycles=0):
    """Testing aid: pipeline-wait budget of the tensor-core kernels in SM cycles (0 = default)."""
    _check(load().retnet_debug_set_wait_budget(int(cycles)))


def retnet_fp16_range_errors(clear=True):
    """Device threads that rounded a tensor-core operand outside the fp16 range since the last
    clear (synchronises); nonzero means some output of those calls is not finite."""
    c = ctypes.c_uint(0)
    _check(load().retnet_fp16_range_errors(ctypes.byref(c), 1 if clear else 0))
    return c.value


# ---- allocating conveniences (torch.empty for the outputs, then the calls above) ----------

def retention_chunkwise(q, k, v, gamma, theta=None, chunk=64, flags=F_ALL, pos0=0, out_dtype=None,
                        state_in=None, return_state=False, z_in=None, stream=None):
    import torch
    b, L, h, dk = q.shape
    o = torch.empty(v.shape, dtype=out_dtype or v.dtype, device=v.device)
    so = torch.empty((b, h, dk, v.shape[-1]), dtype=torch.float32, device=v.device) if return_state else None
    zo = torch.empty((b, h, dk), dtype=torch.float32, device=v.device) if (return_state and flags & F_NORM_R) else None
    retnet_retention_chunkwise(q, k, v, o, gamma, theta, pos0, flags, chunk, state_in, so, z_in, zo, stream)
    return (o, so, zo) if return_state else o


def retention_parallel(q, k, v, gamma, theta=None, flags=F_ALL, pos0=0, out_dtype=None, stream=None):
    import torch
    o = torch.empty(v.shape, dtype=out_dtype or v.dtype, device=v.device)
    retnet_retention_parallel(q, k, v, o, gamma, theta, pos0, flags, stream)
    return o
