"""Multi-scale retention on B200: thin Python binding over libretention.so.

Every function here only checks and marshals arguments: it takes torch CUDA
tensors (PyTorch supplies device memory and the current stream) and calls the
C ABI declared in include/retention.h.  All arithmetic runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback.  If the library is missing
or cannot be loaded the calls raise.

Layouts (row-major, contiguous): q, k [B,H,N,dk]; v, o [B,H,N,dv];
state [B,H,dk,dv] float32; gammas [H] float32.  q, k, v share one dtype,
torch.float32 or torch.bfloat16.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libretention.so")

RET_F32, RET_BF16 = 0, 1
RET_OK, RET_EINVAL, RET_EUNSUPPORTED, RET_ECUDA, RET_EWORKSPACE = 0, -1, -2, -3, -4

# name -> (restype, argtypes) of every symbol include/retention.h declares
_P, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "ret_parallel": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "ret_chunkwise_workspace": (_S, [_I, _I, _I, _I, _I, _I, _I]),
    "ret_chunkwise": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _S, _P]),
    "ret_chunkwise_noalloc": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F,
                                   _P]),
    "ret_chunkwise_states": (_I, [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _P, _S, _P]),
    "ret_chunkwise_output": (_I, [_P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P, _S,
                                  _P]),
    "ret_step": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "ret_parallel_gated": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "ret_chunkwise_gated": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F,
                                 _P, _S, _P]),
    "ret_chunkwise_output_gated": (_I, [_P, _P, _P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                                        _F, _P, _S, _P]),
    "ret_step_gated": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "ret_step_rotated": (_I, [_P, _P, _P, _P, _P, ctypes.c_longlong, _P, _P, _P, _I, _I, _I, _I,
                              _I, _F, _P]),
    "ret_state_combine": (_I, [_P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P]),
    "ret_chunkwise_backward_workspace": (_S, [_I, _I, _I, _I, _I, _I, _I]),
    "ret_chunkwise_backward": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I,
                                    _I, _I, _I, _P, _S, _P]),
    "ret_rotate": (_I, [_P, _P, _P, ctypes.c_longlong, _I, _I, _I, _I, _I, _P]),
    "ret_status_string": (ctypes.c_char_p, [_I]),
    "ret_last_cuda_error": (_I, []),
    "ret_version": (ctypes.c_char_p, []),
    "ret_device_error": (_I, []),
    "ret_selftest_bounded_wait": (_I, [_I, _P]),
}

_lib = None


class RetentionError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status}){detail}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libretention.so (once) and bind every exported symbol."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m linear_recurrent_sequence_scale_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().ret_status_string(status).decode()


def device_error() -> int:
    """Read and clear the tensor-core kernels' timed-out-wait flag (0 = none)."""
    return int(load_library().ret_device_error())


def version() -> str:
    return load_library().ret_version().decode()


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return RET_F32
    if t.dtype == torch.bfloat16:
        return RET_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _check(t, name, dtype=None, shape=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _raise(fn, status):
    lib = load_library()
    detail = f", cudaError {lib.ret_last_cuda_error()}" if status == RET_ECUDA else ""
    raise RetentionError(fn, status, detail)


def _seq_args(q, k, v, gammas):
    torch = _torch()
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B,H,N,d]")
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check(q, "q", device=dev)
    _check(k, "k", dtype=q.dtype, shape=(B, H, N, dk), device=dev)
    _check(v, "v", dtype=q.dtype, shape=(B, H, N, dv), device=dev)
    _check(gammas, "gammas", dtype=torch.float32, shape=(H,), device=dev)
    return B, H, N, dk, dv, dev


def _gate(gate, like, shape, dev):
    if gate is not None:
        _check(gate, "gate", dtype=like.dtype, shape=shape, device=dev)
    return gate


def parallel(q, k, v, gammas, gn_eps=None, out=None, gate=None):
    """Parallel form O = (Q K^T (.) D) V (ret_parallel); returns o.  With a
    gate (same shape as o): o = swish(gate) * O (ret_parallel_gated)."""
    torch = _torch()
    B, H, N, dk, dv, dev = _seq_args(q, k, v, gammas)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=dev)
    _check(out, "out", dtype=q.dtype, shape=(B, H, N, dv), device=dev)
    gate = _gate(gate, q, (B, H, N, dv), dev)
    eps = -1.0 if gn_eps is None else float(gn_eps)
    lib = load_library()
    if gate is None:
        s = lib.ret_parallel(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), _ptr(out),
                             B, H, N, dk, dv, _dtype_code(q), eps, _stream(dev))
    else:
        s = lib.ret_parallel_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), _ptr(gate), _ptr(out),
                                   B, H, N, dk, dv, _dtype_code(q), eps, _stream(dev))
    if s != RET_OK:
        _raise("ret_parallel", s)
    return out


def chunkwise_workspace_bytes(B, H, N, dk, dv, chunk, dtype) -> int:
    torch = _torch()
    code = RET_BF16 if dtype == torch.bfloat16 else RET_F32
    return int(load_library().ret_chunkwise_workspace(B, H, N, dk, dv, chunk, code))


def chunkwise(q, k, v, gammas, chunk, state_in=None, state_out=None, return_state=False,
              gn_eps=None, out=None, workspace=None, gate=None):
    """Chunkwise-recurrent form (ret_chunkwise; ret_chunkwise_gated with a gate).

    Returns o, or (o, state) when return_state is True or state_out is given.
    state_out may be the same tensor as state_in (updated in place).
    workspace: optional uint8 CUDA tensor of at least chunkwise_workspace_bytes().
    gate: optional tensor shaped like o; o is then multiplied by swish(gate).
    """
    torch = _torch()
    B, H, N, dk, dv, dev = _seq_args(q, k, v, gammas)
    sshape = (B, H, dk, dv)
    if state_in is not None:
        _check(state_in, "state_in", dtype=torch.float32, shape=sshape, device=dev)
    if state_out is None and return_state:
        state_out = torch.empty(sshape, dtype=torch.float32, device=dev)
    if state_out is not None:
        _check(state_out, "state_out", dtype=torch.float32, shape=sshape, device=dev)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=dev)
    _check(out, "out", dtype=q.dtype, shape=(B, H, N, dv), device=dev)
    gate = _gate(gate, q, (B, H, N, dv), dev)
    workspace, ws_bytes = _workspace(workspace, B, H, N, dk, dv, chunk, q.dtype, dev)
    eps = -1.0 if gn_eps is None else float(gn_eps)
    lib = load_library()
    if gate is None:
        s = lib.ret_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), int(chunk),
                              _ptr(state_in), _ptr(state_out), _ptr(out),
                              B, H, N, dk, dv, _dtype_code(q), eps,
                              _ptr(workspace), ws_bytes, _stream(dev))
    else:
        s = lib.ret_chunkwise_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), int(chunk),
                                    _ptr(state_in), _ptr(state_out), _ptr(gate), _ptr(out),
                                    B, H, N, dk, dv, _dtype_code(q), eps,
                                    _ptr(workspace), ws_bytes, _stream(dev))
    if s != RET_OK:
        _raise("ret_chunkwise", s)
    if state_out is not None:
        return out, state_out
    return out


def _workspace(workspace, B, H, N, dk, dv, chunk, dtype, dev):
    torch = _torch()
    need = chunkwise_workspace_bytes(B, H, N, dk, dv, chunk, dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0
    if workspace is not None:
        _check(workspace, "workspace", device=dev)
        ws_bytes = workspace.numel() * workspace.element_size()
    return workspace, ws_bytes


def chunkwise_states(k, v, gammas, chunk, workspace, state_in=None, state_out=None):
    """First phase of the chunkwise form (ret_chunkwise_states): the state
    entering every chunk into `workspace` (uint8 CUDA tensor of at least
    chunkwise_workspace_bytes()), and the final state into state_out if given."""
    torch = _torch()
    B, H, N, dk, dv, dev = _seq_args(k, k, v, gammas)
    sshape = (B, H, dk, dv)
    if state_in is not None:
        _check(state_in, "state_in", dtype=torch.float32, shape=sshape, device=dev)
    if state_out is not None:
        _check(state_out, "state_out", dtype=torch.float32, shape=sshape, device=dev)
    workspace, ws_bytes = _workspace(workspace, B, H, N, dk, dv, chunk, k.dtype, dev)
    s = load_library().ret_chunkwise_states(_ptr(k), _ptr(v), _ptr(gammas), int(chunk),
                                            _ptr(state_in), _ptr(state_out), B, H, N, dk, dv,
                                            _dtype_code(k), _ptr(workspace), ws_bytes,
                                            _stream(dev))
    if s != RET_OK:
        _raise("ret_chunkwise_states", s)
    return workspace


def chunkwise_output(q, k, v, gammas, chunk, workspace, has_state_in=False, gn_eps=None,
                     out=None, gate=None):
    """Second phase of the chunkwise form (ret_chunkwise_output, or
    ret_chunkwise_output_gated with a gate): o from the workspace that
    chunkwise_states wrote for the same sizes; returns o."""
    torch = _torch()
    B, H, N, dk, dv, dev = _seq_args(q, k, v, gammas)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=dev)
    _check(out, "out", dtype=q.dtype, shape=(B, H, N, dv), device=dev)
    gate = _gate(gate, q, (B, H, N, dv), dev)
    workspace, ws_bytes = _workspace(workspace, B, H, N, dk, dv, chunk, q.dtype, dev)
    eps = -1.0 if gn_eps is None else float(gn_eps)
    lib = load_library()
    if gate is None:
        s = lib.ret_chunkwise_output(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), int(chunk),
                                     1 if has_state_in else 0, _ptr(out), B, H, N, dk, dv,
                                     _dtype_code(q), eps, _ptr(workspace), ws_bytes,
                                     _stream(dev))
    else:
        s = lib.ret_chunkwise_output_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), int(chunk),
                                           1 if has_state_in else 0, _ptr(gate), _ptr(out),
                                           B, H, N, dk, dv, _dtype_code(q), eps,
                                           _ptr(workspace), ws_bytes, _stream(dev))
    if s != RET_OK:
        _raise("ret_chunkwise_output", s)
    return out


def chunkwise_backward(q, k, v, gammas, chunk, d_o, state_in=None, d_state_out=None,
                       workspace=None):
    """Gradients of ret_chunkwise (no GroupNorm, no gate): returns
    (dq, dk, dv, d_state_in) for the output gradient d_o [B,H,N,dv] and the
    optional final-state gradient d_state_out (ret_chunkwise_backward)."""
    torch = _torch()
    B, H, N, dk, dv, dev = _seq_args(q, k, v, gammas)
    _check(d_o, "d_o", dtype=q.dtype, shape=(B, H, N, dv), device=dev)
    sshape = (B, H, dk, dv)
    for t, name in ((state_in, "state_in"), (d_state_out, "d_state_out")):
        if t is not None:
            _check(t, name, dtype=torch.float32, shape=sshape, device=dev)
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = torch.empty(sshape, dtype=torch.float32, device=dev)
    lib = load_library()
    need = int(lib.ret_chunkwise_backward_workspace(B, H, N, dk, dv, int(chunk), _dtype_code(q)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = lib.ret_chunkwise_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), int(chunk),
                                   _ptr(state_in), _ptr(d_o), _ptr(d_state_out), _ptr(dq),
                                   _ptr(dk_), _ptr(dv_), _ptr(ds), B, H, N, dk, dv,
                                   _dtype_code(q), _ptr(workspace), wsb, _stream(dev))
    if s != RET_OK:
        _raise("ret_chunkwise_backward", s)
    return dq, dk_, dv_, ds


def state_combine(locals_, spans, r, gammas, state0=None, out=None):
    """State entering span r of a sequence split into spans (ret_state_combine).
    locals_: [R,B,H,dk,dv] float32 end states of the spans computed from a zero
    state; spans: R span lengths (host ints); state0: state entering span 0 or
    None.  r = R gives the end state of the whole sequence."""
    torch = _torch()
    R, B, H, dk, dv = locals_.shape
    dev = locals_.device
    _check(locals_, "locals", dtype=torch.float32, device=dev)
    if not 0 <= r <= R or len(spans) != R:
        raise ValueError("need 0 <= r <= number of spans and one length per span")
    _check(gammas, "gammas", dtype=torch.float32, shape=(H,), device=dev)
    if state0 is not None:
        _check(state0, "state0", dtype=torch.float32, shape=(B, H, dk, dv), device=dev)
    if out is None:
        out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _check(out, "out", dtype=torch.float32, shape=(B, H, dk, dv), device=dev)
    sp = (ctypes.c_int * max(R, 1))(*[int(n) for n in spans])
    s = load_library().ret_state_combine(_ptr(locals_), sp, int(r), _ptr(gammas), _ptr(state0),
                                         _ptr(out), B, H, dk, dv, _stream(dev))
    if s != RET_OK:
        _raise("ret_state_combine", s)
    return out


def rotate(x, theta, pos0=0, out=None):
    """xPos-style rotation of q or k rows (ret_rotate): channel pair c of the
    row at position pos0 + j turns by (pos0 + j) * theta[c].
    x [B,H,N,d] or [B,H,d] (one position, e.g. a decode step); theta [d/2]
    float32; out may be x itself (in place).  Returns out."""
    torch = _torch()
    if x.dim() not in (3, 4):
        raise ValueError("x must be [B,H,N,d] or [B,H,d]")
    B, H = x.shape[0], x.shape[1]
    N = x.shape[2] if x.dim() == 4 else 1
    d = x.shape[-1]
    dev = x.device
    _check(x, "x", device=dev)
    code = _dtype_code(x)
    _check(theta, "theta", dtype=torch.float32, shape=(d // 2,), device=dev)
    if out is None:
        out = torch.empty_like(x)
    _check(out, "out", dtype=x.dtype, shape=tuple(x.shape), device=dev)
    s = load_library().ret_rotate(_ptr(x), _ptr(out), _ptr(theta), int(pos0), B, H, N, d, code,
                                  _stream(dev))
    if s != RET_OK:
        _raise("ret_rotate", s)
    return out


def step(q, k, v, gammas, state, gn_eps=None, out=None, gate=None, theta=None, pos=0):
    """One recurrent decode step (ret_step; ret_step_gated with a gate [B,H,dv];
    ret_step_rotated with theta [dk/2], q and k then rotated by pos * theta as
    they are read): state is updated in place; returns o.
    q, k [B,H,dk]; v [B,H,dv]; state [B,H,dk,dv] float32."""
    torch = _torch()
    if q.dim() != 3:
        raise ValueError("q, k, v must be [B,H,d] for a decode step")
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check(q, "q", device=dev)
    _check(k, "k", dtype=q.dtype, shape=(B, H, dk), device=dev)
    _check(v, "v", dtype=q.dtype, shape=(B, H, dv), device=dev)
    _check(gammas, "gammas", dtype=torch.float32, shape=(H,), device=dev)
    _check(state, "state", dtype=torch.float32, shape=(B, H, dk, dv), device=dev)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=dev)
    _check(out, "out", dtype=q.dtype, shape=(B, H, dv), device=dev)
    gate = _gate(gate, q, (B, H, dv), dev)
    eps = -1.0 if gn_eps is None else float(gn_eps)
    lib = load_library()
    if theta is not None:
        _check(theta, "theta", dtype=torch.float32, shape=(dk // 2,), device=dev)
        s = lib.ret_step_rotated(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), _ptr(theta), int(pos),
                                 _ptr(state), _ptr(gate), _ptr(out), B, H, dk, dv,
                                 _dtype_code(q), eps, _stream(dev))
    elif gate is None:
        s = lib.ret_step(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), _ptr(state), _ptr(out),
                         B, H, dk, dv, _dtype_code(q), eps, _stream(dev))
    else:
        s = lib.ret_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(gammas), _ptr(state), _ptr(gate),
                               _ptr(out), B, H, dk, dv, _dtype_code(q), eps, _stream(dev))
    if s != RET_OK:
        _raise("ret_step", s)
    return out
