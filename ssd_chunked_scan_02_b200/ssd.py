"""Thin ctypes binding of libssd_b200.so (C ABI in include/ssd.h).

Argument marshalling only: every step of the SSD forward and of the decode
step runs in the library's CUDA kernels.  PyTorch is used for device memory
and streams.  There is no CPU fallback: if the library is missing, or a
tensor is not on a CUDA device, the call raises.

Function names match the C entry points.  Each call enqueues work on the
current torch CUDA stream (or the ``stream`` argument) and returns without
synchronising.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd_b200.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = 0, 1, 2, 3, 4
SSD_F32, SSD_BF16 = 0, 1

EXPORTED = ("ssd_status_string", "ssd_last_error_detail", "ssd_chunk_scan_fwd_workspace_size",
            "ssd_chunk_scan_fwd", "ssd_step", "ssd_chunk_state_fwd", "ssd_state_passing_fwd",
            "ssd_chunk_output_fwd", "ssd_chunk_scan_fwd_uses_tensor_cores",
            "ssd_chunk_scan_bwd_uses_tensor_cores",
            "ssd_chunk_scan_fwd_noalloc", "ssd_poll_device_status", "ssd_state_walk_fwd",
            "ssd_debug_expire_wait", "ssd_chunk_scan_bwd_workspace_size", "ssd_chunk_scan_bwd",
            "ssd_chunk_scan_fwd_data_flow", "ssd_seq_logdecay", "ssd_state_exchange_combine",
            "ssd_state_correction_workspace_size", "ssd_state_correction_fwd",
            "ssd_chunk_scan_fwd_flow_workspace_size", "ssd_chunk_scan_fwd_with_flow")

# ssd_chunk_scan_fwd_data_flow results
SSD_FLOW_SIMT, SSD_FLOW_TC_THREE_KERNEL, SSD_FLOW_WALK_OUTPUT, SSD_FLOW_WALK_OUTPUT_FUSED = 0, 1, 2, 3


class SSDError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {status_name(status)}: {detail}")
        self.status = status


class ssd_dims_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64)]


_lib = None
_vp = ctypes.c_void_p


def load(path: str = LIB_PATH):
    """Open the shared library (once).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m ssd_chunked_scan_02_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    dims_p = ctypes.POINTER(ssd_dims_t)
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_status_string.argtypes = [ctypes.c_int]
    lib.ssd_last_error_detail.restype = ctypes.c_char_p
    lib.ssd_last_error_detail.argtypes = []
    lib.ssd_chunk_scan_fwd_workspace_size.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd_workspace_size.argtypes = [dims_p, ctypes.c_int, ctypes.c_int,
                                                      ctypes.POINTER(ctypes.c_size_t)]
    lib.ssd_chunk_scan_fwd_uses_tensor_cores.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd_uses_tensor_cores.argtypes = [dims_p, ctypes.c_int, ctypes.c_int]
    lib.ssd_chunk_scan_bwd_uses_tensor_cores.restype = ctypes.c_int
    lib.ssd_chunk_scan_bwd_uses_tensor_cores.argtypes = [dims_p, ctypes.c_int]
    lib.ssd_chunk_scan_fwd_data_flow.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd_data_flow.argtypes = [dims_p, ctypes.c_int, ctypes.c_int]
    lib.ssd_chunk_scan_fwd.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd.argtypes = [_vp] * 6 + [ctypes.c_int, _vp, _vp, _vp, dims_p,
                                                   ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    lib.ssd_chunk_scan_fwd_flow_workspace_size.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd_flow_workspace_size.argtypes = [dims_p, ctypes.c_int, ctypes.c_int,
                                                           ctypes.c_int,
                                                           ctypes.POINTER(ctypes.c_size_t)]
    lib.ssd_chunk_scan_fwd_with_flow.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd_with_flow.argtypes = lib.ssd_chunk_scan_fwd.argtypes + [ctypes.c_int]
    lib.ssd_chunk_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssd_chunk_scan_fwd_noalloc.argtypes = [_vp] * 6 + [ctypes.c_int, _vp, _vp, _vp, dims_p,
                                                           ctypes.c_int, _vp]
    lib.ssd_state_walk_fwd.restype = ctypes.c_int
    lib.ssd_state_walk_fwd.argtypes = [_vp] * 7 + [ctypes.c_int, dims_p, ctypes.c_int, _vp]
    lib.ssd_debug_expire_wait.restype = ctypes.c_int
    lib.ssd_debug_expire_wait.argtypes = [ctypes.c_uint, _vp]
    lib.ssd_poll_device_status.restype = ctypes.c_int
    lib.ssd_poll_device_status.argtypes = [_vp]
    lib.ssd_step.restype = ctypes.c_int
    lib.ssd_step.argtypes = [_vp] * 8 + [dims_p, ctypes.c_int, _vp]
    lib.ssd_chunk_state_fwd.restype = ctypes.c_int
    lib.ssd_chunk_state_fwd.argtypes = [_vp] * 4 + [ctypes.c_int, _vp, _vp, dims_p,
                                                    ctypes.c_int, _vp]
    lib.ssd_state_passing_fwd.restype = ctypes.c_int
    lib.ssd_state_passing_fwd.argtypes = [_vp] * 5 + [ctypes.c_int, dims_p, ctypes.c_int, _vp]
    lib.ssd_chunk_output_fwd.restype = ctypes.c_int
    lib.ssd_chunk_output_fwd.argtypes = [_vp] * 7 + [ctypes.c_int, _vp, dims_p, ctypes.c_int, _vp]
    lib.ssd_chunk_scan_bwd_workspace_size.restype = ctypes.c_int
    lib.ssd_chunk_scan_bwd_workspace_size.argtypes = [dims_p, ctypes.c_int,
                                                      ctypes.POINTER(ctypes.c_size_t)]
    lib.ssd_chunk_scan_bwd.restype = ctypes.c_int
    lib.ssd_chunk_scan_bwd.argtypes = [_vp] * 16 + [dims_p, ctypes.c_int, _vp, ctypes.c_size_t,
                                                    _vp]
    lib.ssd_seq_logdecay.restype = ctypes.c_int
    lib.ssd_seq_logdecay.argtypes = [_vp] * 3 + [dims_p, _vp]
    lib.ssd_state_exchange_combine.restype = ctypes.c_int
    lib.ssd_state_exchange_combine.argtypes = [_vp] * 3 + [ctypes.c_int, ctypes.c_int, _vp, dims_p,
                                                           _vp]
    lib.ssd_state_correction_workspace_size.restype = ctypes.c_int
    lib.ssd_state_correction_workspace_size.argtypes = [dims_p, ctypes.c_int,
                                                        ctypes.POINTER(ctypes.c_size_t)]
    lib.ssd_state_correction_fwd.restype = ctypes.c_int
    lib.ssd_state_correction_fwd.argtypes = [_vp] * 6 + [dims_p, ctypes.c_int, _vp,
                                                         ctypes.c_size_t, _vp]
    _lib = lib
    return lib


def status_name(status: int) -> str:
    return load().ssd_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != SSD_OK:
        raise SSDError(status, where, load().ssd_last_error_detail().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return SSD_F32
    if t == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"unsupported element dtype {t} (float32 or bfloat16)")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _device_of(t):
    """The CUDA device the call runs on: the main input's.  Calls are made
    with that device current (the library looks up its per-device state for
    the current device and rejects tensors of another one)."""
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
    return t.device


def _expect(name, t, shape, dtype, device):
    """Shape, dtype and device of one argument, checked before the C call (a
    wrong shape would otherwise become an out-of-bounds access)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device} (the device of x)")


def _check_fwd_args(x, dt, A, B, C, D, init, y, final):
    """Shapes, dtypes and devices of the forward's arguments (against x and
    B), then that they are on a CUDA device.  Returns that device."""
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be (b, L, H, P) and B (b, L, G, N)")
    dev = x.device
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    f32 = torch.float32
    _expect("dt", dt, (b, L, H), f32, dev)
    _expect("A", A, (H,), f32, dev)
    _expect("D", D, (H,), f32, dev)
    _expect("B", B, (b, L, G, N), x.dtype, dev)
    _expect("C", C, (b, L, G, N), x.dtype, dev)
    _expect("init_states", init, (b, H, P, N), f32, dev)
    _expect("y", y, (b, L, H, P), x.dtype, dev)
    _expect("final_states", final, (b, H, P, N), f32, dev)
    return _device_of(x)


def make_dims(batch, seqlen, nheads, headdim, dstate, ngroups) -> ssd_dims_t:
    return ssd_dims_t(int(batch), int(seqlen), int(nheads), int(headdim), int(dstate),
                      int(ngroups))


def _fwd_dims(x, B) -> ssd_dims_t:
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return make_dims(b, L, H, P, N, G)


def ssd_chunk_scan_fwd_workspace_size(dims: ssd_dims_t, chunk_size: int, dtype: torch.dtype,
                                      flow=None) -> int:
    n = ctypes.c_size_t(0)
    fl = -1 if flow is None else int(flow)
    _check(load().ssd_chunk_scan_fwd_flow_workspace_size(ctypes.byref(dims), int(chunk_size),
                                                         _dtype_code(dtype), fl, ctypes.byref(n)),
           "ssd_chunk_scan_fwd_workspace_size")
    return int(n.value)


def ssd_chunk_scan_fwd_uses_tensor_cores(dims: ssd_dims_t, chunk_size: int,
                                         dtype: torch.dtype) -> int:
    return int(load().ssd_chunk_scan_fwd_uses_tensor_cores(ctypes.byref(dims), int(chunk_size),
                                                           _dtype_code(dtype)))


def ssd_chunk_scan_fwd_data_flow(dims: ssd_dims_t, chunk_size: int, dtype: torch.dtype) -> int:
    """SSD_FLOW_WALK_OUTPUT_FUSED, SSD_FLOW_WALK_OUTPUT, SSD_FLOW_TC_THREE_KERNEL,
    SSD_FLOW_SIMT or -1 (rejected)."""
    return int(load().ssd_chunk_scan_fwd_data_flow(ctypes.byref(dims), int(chunk_size),
                                                   _dtype_code(dtype)))


def ssd_chunk_scan_fwd(x, dt, A, B, C, D, chunk_size: int, init_states=None,
                       return_final_states: bool = False, y=None, final_states=None,
                       workspace=None, stream=None, flow=None):
    """y (b,L,H,P) [, final_states (b,H,P,N) fp32] for the whole sequences.
    ``flow``: an SSD_FLOW_* value to force that data flow (None: the
    library's choice)."""
    dev = _check_fwd_args(x, dt, A, B, C, D, init_states, y, final_states)
    dims = _fwd_dims(x, B)
    if y is None:
        y = torch.empty_like(x)
    if return_final_states and final_states is None:
        final_states = torch.empty((x.shape[0], x.shape[2], x.shape[3], B.shape[3]),
                                   device=x.device, dtype=torch.float32)
    fl = -1 if flow is None else int(flow)
    need = ssd_chunk_scan_fwd_workspace_size(dims, chunk_size, x.dtype, flow=flow)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=x.device, dtype=torch.uint8)
    with torch.cuda.device(dev):
        st = load().ssd_chunk_scan_fwd_with_flow(
            _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), int(chunk_size),
            _ptr(init_states), _ptr(y), _ptr(final_states), ctypes.byref(dims),
            _dtype_code(x.dtype), _ptr(workspace), workspace.numel(), _stream(stream, dev), fl)
    _check(st, "ssd_chunk_scan_fwd")
    return (y, final_states) if (return_final_states or final_states is not None) else y


def ssd_chunk_scan_fwd_noalloc(x, dt, A, B, C, D, chunk_size: int, init_states=None,
                               return_final_states: bool = False, y=None, final_states=None,
                               stream=None):
    """ssd_chunk_scan_fwd without a caller workspace: the library's built-in
    scratch array (SSD_NOALLOC_SCRATCH_BYTES) is used instead.  For callers
    that cannot allocate device memory; calls that overlap on the GPU race on
    that array."""
    dev = _check_fwd_args(x, dt, A, B, C, D, init_states, y, final_states)
    dims = _fwd_dims(x, B)
    if y is None:
        y = torch.empty_like(x)
    if return_final_states and final_states is None:
        final_states = torch.empty((x.shape[0], x.shape[2], x.shape[3], B.shape[3]),
                                   device=x.device, dtype=torch.float32)
    with torch.cuda.device(dev):
        st = load().ssd_chunk_scan_fwd_noalloc(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                               _ptr(D), int(chunk_size), _ptr(init_states),
                                               _ptr(y), _ptr(final_states), ctypes.byref(dims),
                                               _dtype_code(x.dtype), _stream(stream, dev))
    _check(st, "ssd_chunk_scan_fwd_noalloc")
    return (y, final_states) if (return_final_states or final_states is not None) else y


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def ssd_step(state, x, dt, A, B, C, D, y=None, stream=None):
    """One decode step; ``state`` (b,H,P,N) fp32 is updated in place.  Returns y (b,H,P)."""
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    dev = x.device
    f32 = torch.float32
    _expect("state", state, (b, H, P, N), f32, dev)
    _expect("dt", dt, (b, H), f32, dev)
    _expect("A", A, (H,), f32, dev)
    _expect("D", D, (H,), f32, dev)
    _expect("B", B, (b, G, N), x.dtype, dev)
    _expect("C", C, (b, G, N), x.dtype, dev)
    _expect("y", y, (b, H, P), x.dtype, dev)
    dev = _device_of(x)
    dims = make_dims(b, 1, H, P, N, G)
    if y is None:
        y = torch.empty_like(x)
    with torch.cuda.device(dev):
        st = load().ssd_step(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                             _ptr(y), ctypes.byref(dims), _dtype_code(x.dtype),
                             _stream(stream, dev))
    _check(st, "ssd_step")
    return y


def ssd_poll_device_status(stream=None):
    """Raise SSDError(SSD_ERR_TIMEOUT) if a bounded device-side wait gave up
    since the last poll (synchronises the stream)."""
    _check(load().ssd_poll_device_status(_stream(stream)), "ssd_poll_device_status")


def ssd_debug_expire_wait(polls: int = 4096, stream=None):
    """Launch the bounded-wait failure probe (see include/ssd.h)."""
    _check(load().ssd_debug_expire_wait(int(polls), _stream(stream)), "ssd_debug_expire_wait")


def n_chunks(seqlen: int, chunk_size: int) -> int:
    return (int(seqlen) + int(chunk_size) - 1) // int(chunk_size)


def ssd_chunk_state_fwd(x, dt, A, B, chunk_size: int, stream=None):
    """Step (2): per-chunk zero-start states (b,T,H,P,N) fp32 and log-decays (b,T,H)."""
    dims = _fwd_dims(x, B)
    b, L, H, P = x.shape
    T = n_chunks(L, chunk_size)
    dev = _check_fwd_args(x, dt, A, B, None, None, None, None, None)
    states = torch.empty((b, T, H, P, B.shape[3]), device=x.device, dtype=torch.float32)
    logdecay = torch.empty((b, T, H), device=x.device, dtype=torch.float32)
    with torch.cuda.device(dev):
        st = load().ssd_chunk_state_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), int(chunk_size),
                                        _ptr(states), _ptr(logdecay), ctypes.byref(dims),
                                        _dtype_code(x.dtype), _stream(stream, dev))
    _check(st, "ssd_chunk_state_fwd")
    return states, logdecay


def ssd_state_passing_fwd(chunk_states, chunk_logdecay, chunk_size: int, seqlen: int,
                          dtype: torch.dtype, init_states=None, want_final: bool = True,
                          stream=None):
    """Step (3): states entering each chunk (b,T,H,P,N) in ``dtype`` and the final state."""
    b, T, H, P, N = chunk_states.shape
    dims = make_dims(b, seqlen, H, P, N, 1)
    dev = _device_of(chunk_states)
    _expect("chunk_states", chunk_states, (b, T, H, P, N), torch.float32, dev)
    _expect("chunk_logdecay", chunk_logdecay, (b, T, H), torch.float32, dev)
    _expect("init_states", init_states, (b, H, P, N), torch.float32, dev)
    if n_chunks(seqlen, chunk_size) != T:
        raise ValueError(f"chunk_states has {T} chunks; seqlen {seqlen} / chunk {chunk_size} "
                         f"gives {n_chunks(seqlen, chunk_size)}")
    prev = torch.empty((b, T, H, P, N), device=chunk_states.device, dtype=dtype)
    final = (torch.empty((b, H, P, N), device=chunk_states.device, dtype=torch.float32)
             if want_final else None)
    with torch.cuda.device(dev):
        st = load().ssd_state_passing_fwd(_ptr(chunk_states), _ptr(chunk_logdecay),
                                          _ptr(init_states), _ptr(prev), _ptr(final),
                                          int(chunk_size), ctypes.byref(dims),
                                          _dtype_code(dtype), _stream(stream, dev))
    _check(st, "ssd_state_passing_fwd")
    return prev, final


def ssd_state_walk_fwd(x, dt, A, B, chunk_size: int, init_states=None, want_final: bool = True,
                       stream=None):
    """Steps (2) + (3) fused (the on-chip state walk): entering states
    (b,T,H,P,N) bf16 and the final state (b,H,P,N) fp32."""
    dims = _fwd_dims(x, B)
    b, L, H, P = x.shape
    N = B.shape[3]
    T = n_chunks(L, chunk_size)
    dev = _check_fwd_args(x, dt, A, B, None, None, init_states, None, None)
    prev = torch.empty((b, T, H, P, N), device=x.device, dtype=torch.bfloat16)
    final = torch.empty((b, H, P, N), device=x.device, dtype=torch.float32) if want_final else None
    with torch.cuda.device(dev):
        st = load().ssd_state_walk_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(init_states),
                                       _ptr(prev), _ptr(final), int(chunk_size),
                                       ctypes.byref(dims), _dtype_code(x.dtype),
                                       _stream(stream, dev))
    _check(st, "ssd_state_walk_fwd")
    return prev, final


def ssd_chunk_output_fwd(x, dt, A, B, C, D, prev_states, chunk_size: int, y=None, stream=None):
    """Steps (1) and (4): y from the inputs and the states entering each chunk."""
    dev = _check_fwd_args(x, dt, A, B, C, D, None, y, None)
    b, L, H, P = x.shape
    _expect("prev_states", prev_states, (b, n_chunks(L, chunk_size), H, P, B.shape[3]), x.dtype,
            dev)
    dims = _fwd_dims(x, B)
    if y is None:
        y = torch.empty_like(x)
    with torch.cuda.device(dev):
        st = load().ssd_chunk_output_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                         _ptr(prev_states), int(chunk_size), _ptr(y),
                                         ctypes.byref(dims), _dtype_code(x.dtype),
                                         _stream(stream, dev))
    _check(st, "ssd_chunk_output_fwd")
    return y


def ssd_chunk_scan_bwd_uses_tensor_cores(dims: ssd_dims_t, dtype: torch.dtype) -> int:
    """1: the backward runs on the tcgen05 tensor cores; 0: exact fp32 on the
    CUDA cores; -1: these sizes are rejected."""
    return int(load().ssd_chunk_scan_bwd_uses_tensor_cores(ctypes.byref(dims), _dtype_code(dtype)))


def ssd_chunk_scan_bwd_workspace_size(dims: ssd_dims_t, dtype: torch.dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(load().ssd_chunk_scan_bwd_workspace_size(ctypes.byref(dims), _dtype_code(dtype),
                                                    ctypes.byref(n)),
           "ssd_chunk_scan_bwd_workspace_size")
    return int(n.value)


def ssd_chunk_scan_bwd(x, dt, A, B, C, D, dy, init_states=None, dfinal_states=None,
                       want_dinit: bool = True, workspace=None, stream=None):
    """Gradients of ssd_chunk_scan_fwd for dL/dy = dy (b,L,H,P, x's dtype) and
    dL/dfinal_states = dfinal_states ((b,H,P,N) fp32 or None).  Returns a dict
    of fp32 tensors: dx, ddt, dA, dB, dC, dD and (if want_dinit) dinit."""
    dev = _check_fwd_args(x, dt, A, B, C, D, init_states, None, dfinal_states)
    _expect("dy", dy, tuple(x.shape), x.dtype, dev)
    dims = _fwd_dims(x, B)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    f32 = dict(device=x.device, dtype=torch.float32)
    out = {"dx": torch.empty((b, L, H, P), **f32), "ddt": torch.empty((b, L, H), **f32),
           "dA": torch.empty((H,), **f32), "dB": torch.empty((b, L, G, N), **f32),
           "dC": torch.empty((b, L, G, N), **f32), "dD": torch.empty((H,), **f32),
           "dinit": torch.empty((b, H, P, N), **f32) if want_dinit else None}
    need = ssd_chunk_scan_bwd_workspace_size(dims, x.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=x.device, dtype=torch.uint8)
    with torch.cuda.device(dev):
        st = load().ssd_chunk_scan_bwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                       _ptr(init_states), _ptr(dy), _ptr(dfinal_states),
                                       _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA"]),
                                       _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dD"]),
                                       _ptr(out["dinit"]), ctypes.byref(dims),
                                       _dtype_code(x.dtype), _ptr(workspace), workspace.numel(),
                                       _stream(stream, dev))
    _check(st, "ssd_chunk_scan_bwd")
    return out


# ---------------------------------------------------------------- sequence parallelism
def ssd_seq_logdecay(dt, A, stream=None):
    """sum_t dt[b,t,h] * A[h] over the (shard's) sequence: (b, H) fp32."""
    b, L, H = dt.shape
    _expect("dt", dt, (b, L, H), torch.float32, dt.device)
    _expect("A", A, (H,), torch.float32, dt.device)
    dev = _device_of(dt)
    out = torch.empty((b, H), device=dt.device, dtype=torch.float32)
    dims = make_dims(b, L, H, 1, 1, 1)
    with torch.cuda.device(dev):
        st = load().ssd_seq_logdecay(_ptr(dt), _ptr(A), _ptr(out), ctypes.byref(dims),
                                     _stream(stream, dev))
    _check(st, "ssd_seq_logdecay")
    return out


def ssd_state_exchange_combine(local_final, logdecay, rank: int, init_states=None, out=None,
                               stream=None):
    """The state entering rank ``rank``'s shard from the gathered local final
    states (R,b,H,P,N) and log-decays (R,b,H) of all ranks (rank order) and
    the state entering the whole sequence (None = zero).  rank = R gives the
    state after the whole sequence."""
    R, b, H, P, N = local_final.shape
    dev = local_final.device
    _expect("logdecay", logdecay, (R, b, H), torch.float32, dev)
    _expect("local_final", local_final, (R, b, H, P, N), torch.float32, dev)
    _expect("init_states", init_states, (b, H, P, N), torch.float32, dev)
    _expect("out", out, (b, H, P, N), torch.float32, dev)
    dev = _device_of(local_final)
    if out is None:
        out = torch.empty((b, H, P, N), device=local_final.device, dtype=torch.float32)
    dims = make_dims(b, 0, H, P, N, 1)
    with torch.cuda.device(dev):
        st = load().ssd_state_exchange_combine(_ptr(local_final), _ptr(logdecay), _ptr(init_states),
                                               int(rank), int(R), _ptr(out), ctypes.byref(dims),
                                               _stream(stream, dev))
    _check(st, "ssd_state_exchange_combine")
    return out


def ssd_state_correction_workspace_size(dims: ssd_dims_t, dtype: torch.dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(load().ssd_state_correction_workspace_size(ctypes.byref(dims), _dtype_code(dtype),
                                                      ctypes.byref(n)),
           "ssd_state_correction_workspace_size")
    return int(n.value)


def ssd_state_correction_fwd(h_in, dt, A, C, y, final_states=None, workspace=None, stream=None):
    """In place: y_t += exp(cs_t) h_in C_t over the shard and, if given,
    final_states += exp(cs_last) h_in.  h_in (b,H,P,N) fp32."""
    b, L, H, P = y.shape
    G, N = C.shape[2], C.shape[3]
    dev = y.device
    _expect("h_in", h_in, (b, H, P, N), torch.float32, dev)
    _expect("dt", dt, (b, L, H), torch.float32, dev)
    _expect("A", A, (H,), torch.float32, dev)
    _expect("C", C, (b, L, G, N), y.dtype, dev)
    _expect("final_states", final_states, (b, H, P, N), torch.float32, dev)
    dev = _device_of(y)
    dims = make_dims(b, L, H, P, N, G)
    need = ssd_state_correction_workspace_size(dims, y.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=y.device, dtype=torch.uint8)
    with torch.cuda.device(dev):
        st = load().ssd_state_correction_fwd(_ptr(h_in), _ptr(dt), _ptr(A), _ptr(C), _ptr(y),
                                             _ptr(final_states), ctypes.byref(dims),
                                             _dtype_code(y.dtype), _ptr(workspace),
                                             workspace.numel(), _stream(stream, dev))
    _check(st, "ssd_state_correction_fwd")
    return y
