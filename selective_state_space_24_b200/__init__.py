"""Python binding of libssm.so, the sm_100a selective-scan library.

Argument marshalling only: every step of the scan runs in the library's
CUDA kernels.  PyTorch is used for device memory (tensors, the workspace)
and streams.  If libssm.so is missing or fails to load, every entry point
raises -- there is no fallback path.

Entry points (names as in include/ssm.h):

* ``ssm_scan_fwd(x, delta, A, B, C, ...)``  single-direction S6 scan
* ``ssm_scan_fwd_state(...)``  the same from a given initial state
* ``ssm_scan_fwd_zoh`` / ``bidir_scan_fwd_zoh``  the forward scans with the
  exact zero-order-hold input coefficient instead of dt B (N = 16)
* ``ssm_scan_bwd(x, delta, A, B, C, dout, ...)``  gradients of ssm_scan_fwd
* ``ssm_scan_fwd_ckpt`` / ``bidir_scan_fwd_ckpt``  the forward scans that also
  store the state entering every 4-step chunk, and ``ssm_scan_bwd_ckpt`` /
  ``bidir_scan_bwd_ckpt``, the backward passes that read those checkpoints
  instead of recomputing them
* ``ssm_step(x, delta, A, B, C, state, ...)``  one decode step, state in place
* ``ssm_scan_fwd_ordered`` / ``bidir_scan_fwd_ordered``  scans along a given
  order of the positions, with an optional token mask
* ``ssm_scan_fwd_conv`` / ``bidir_scan_fwd_conv``  scans of u = conv1d(x_in),
  the conv computed inside the scan
* ``bidir_scan_fwd(x, delta, fwd, bwd, ...)``  Vision-Mamba bidirectional scan
* ``ssd_chunk_fwd(x, delta, A, B, C, ...)``  Mamba2 SSD chunked scan

Each also exists in raw form in ``capi`` (ctypes functions taking plain
integers for pointers), which the tests use to check the boundary itself.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm.so")

SSM_F32, SSM_BF16 = 0, 1
STATUS = {
    0: "SSM_OK", 1: "SSM_ERR_INVALID_ARG", 2: "SSM_ERR_UNSUPPORTED_SHAPE", 3: "SSM_ERR_MISALIGNED",
    4: "SSM_ERR_UNSUPPORTED_DTYPE", 5: "SSM_ERR_WORKSPACE_TOO_SMALL", 6: "SSM_ERR_CUDA",
    7: "SSM_ERR_DEVICE_TIMEOUT",
}


class SSMError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class ssm_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("dtype", ctypes.c_int32)]


class ssd_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("chunk", ctypes.c_int64),
                ("dtype", ctypes.c_int32)]


class ssm_dir_params(ctypes.Structure):
    _fields_ = [("delta_bias", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("C", ctypes.c_void_p), ("D", ctypes.c_void_p), ("z", ctypes.c_void_p),
                ("last_state", ctypes.c_void_p)]


class ssm_dir_grads(ctypes.Structure):
    _fields_ = [("dA", ctypes.c_void_p), ("dB", ctypes.c_void_p), ("dC", ctypes.c_void_p),
                ("dD", ctypes.c_void_p), ("dz", ctypes.c_void_p), ("ddelta_bias", ctypes.c_void_p)]


class ssm_conv_params(ctypes.Structure):
    _fields_ = [("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("width", ctypes.c_int32),
                ("silu", ctypes.c_int32)]


_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_int = ctypes.c_int

# exported name -> (restype, argtypes)
SIGNATURES = {
    "ssm_debug_ssd_stall": (None, [_int, ctypes.c_uint]),
    "ssm_debug_s6_mapping": (_int, [_int]),
    "ssm_scan_workspace_size": (_sz, [ctypes.POINTER(ssm_dims)]),
    "ssm_scan_fwd": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp,
                            _int, _vp, _vp, _vp, _sz, _vp]),
    "ssm_scan_fwd_state": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                  _vp, _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "ssm_scan_fwd_zoh": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                _vp, _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "bidir_scan_fwd_zoh": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int,
                                  ctypes.POINTER(ssm_dir_params), ctypes.POINTER(ssm_dir_params), _vp,
                                  _vp, _sz, _vp]),
    "ssm_scan_fwd_ordered": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                    _vp, _int, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "bidir_scan_fwd_ordered": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int,
                                      ctypes.POINTER(ssm_dir_params), ctypes.POINTER(ssm_dir_params),
                                      _vp, _vp, _vp, _vp, _sz, _vp]),
    "ssm_scan_fwd_conv": (_int, [ctypes.POINTER(ssm_dims), _vp, ctypes.POINTER(ssm_conv_params), _vp,
                                 _vp, _int, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp, _vp, _sz, _vp]),
    "bidir_scan_fwd_conv": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int,
                                   ctypes.POINTER(ssm_dir_params), ctypes.POINTER(ssm_dir_params),
                                   ctypes.POINTER(ssm_conv_params), ctypes.POINTER(ssm_conv_params),
                                   _vp, _vp, _sz, _vp]),
    "ssm_scan_bwd_workspace_size": (_sz, [ctypes.POINTER(ssm_dims)]),
    "ssm_scan_bwd": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp, _int,
                            _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "bidir_scan_bwd": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int, ctypes.POINTER(ssm_dir_params),
                              ctypes.POINTER(ssm_dir_params), _vp, _vp, _vp, ctypes.POINTER(ssm_dir_grads),
                              ctypes.POINTER(ssm_dir_grads), _vp, _sz, _vp]),
    "ssm_scan_ckpt_size": (_sz, [ctypes.POINTER(ssm_dims)]),
    "ssm_scan_fwd_ckpt": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp,
                                 _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "bidir_scan_fwd_ckpt": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int, ctypes.POINTER(ssm_dir_params),
                                   ctypes.POINTER(ssm_dir_params), _vp, _vp, _vp, _vp, _sz, _vp]),
    "ssm_scan_bwd_ckpt": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp,
                                 _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bidir_scan_bwd_ckpt": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int, ctypes.POINTER(ssm_dir_params),
                                   ctypes.POINTER(ssm_dir_params), _vp, _vp, _vp,
                                   ctypes.POINTER(ssm_dir_grads), ctypes.POINTER(ssm_dir_grads), _vp, _vp,
                                   _vp]),
    "ssm_step": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp, _vp,
                        _vp, _vp]),
    "ssm_scan_fwd_noalloc": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                    _vp, _int, _vp, _vp, _vp]),
    "bidir_scan_workspace_size": (_sz, [ctypes.POINTER(ssm_dims)]),
    "bidir_scan_fwd": (_int, [ctypes.POINTER(ssm_dims), _vp, _vp, _int,
                              ctypes.POINTER(ssm_dir_params), ctypes.POINTER(ssm_dir_params), _vp,
                              _vp, _sz, _vp]),
    "ssd_chunk_workspace_size": (_sz, [ctypes.POINTER(ssd_dims)]),
    "ssd_chunk_fwd": (_int, [ctypes.POINTER(ssd_dims), _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                             _vp, _vp, _vp, _vp, _sz, _vp]),
    "ssm_scan_plan": (_int, [ctypes.POINTER(ssm_dims), _int, ctypes.POINTER(_int),
                             ctypes.POINTER(_int)]),
    "ssm_check_device": (_int, [_vp]),
    "ssm_status_string": (ctypes.c_char_p, [_int]),
    "ssm_version": (_int, []),
}

_capi = None


def load(path: Optional[str] = None):
    """Load libssm.so (once) and attach the signatures; raises if missing."""
    global _capi
    if _capi is not None and path is None:
        return _capi
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with "
                          "`python -m selective_state_space_24_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if path is None:
        _capi = lib
    return lib


def capi():
    return load()


def _check(status: int, what: str):
    if status != 0:
        raise SSMError(status, what)


# ------------------------------------------------------------------ tensors

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return SSM_F32
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def workspace(nbytes: int, device):
    """A device workspace of at least nbytes (None when 0)."""
    if nbytes == 0:
        return None
    torch = _torch()
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


@dataclass
class DirParams:
    """One direction's parameters for bidir_scan_fwd (tensors on the device)."""
    A: object
    B: object
    C: object
    delta_bias: object = None
    D: object = None
    z: object = None
    last_state: object = None

    def to_c(self) -> ssm_dir_params:
        return ssm_dir_params(_ptr(self.delta_bias), _ptr(self.A), _ptr(self.B), _ptr(self.C),
                              _ptr(self.D), _ptr(self.z), _ptr(self.last_state))


def s6_dims(x, dstate: int) -> ssm_dims:
    Bz, L, Dm = x.shape
    return ssm_dims(Bz, L, Dm, dstate, _dtype_code(x))


def ssm_scan_fwd(x, delta, A, B, C, *, delta_bias=None, delta_softplus=True, D=None, z=None,
                 reverse=False, out=None, last_state=None, ws=None, stream=None):
    """Single-direction S6 scan; returns out (B, L, D) in x's dtype."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    st = lib.ssm_scan_fwd(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                          int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                          int(bool(reverse)), _ptr(out), _ptr(last_state), _ptr(ws),
                          0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "ssm_scan_fwd")
    return out


def ssm_scan_fwd_state(x, delta, A, B, C, *, initial_state=None, delta_bias=None,
                       delta_softplus=True, D=None, z=None, reverse=False, out=None,
                       last_state=None, ws=None, stream=None):
    """ssm_scan_fwd from a given state (initial_state (B, D, N) float32, None
    for zero); last_state may be the same tensor as initial_state."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    st = lib.ssm_scan_fwd_state(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                                int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(z), int(bool(reverse)), _ptr(initial_state), _ptr(out),
                                _ptr(last_state), _ptr(ws), 0 if ws is None else ws.numel(),
                                _stream_handle(stream))
    _check(st, "ssm_scan_fwd_state")
    return out


def ssm_scan_fwd_zoh(x, delta, A, B, C, *, initial_state=None, delta_bias=None, delta_softplus=True,
                     D=None, z=None, reverse=False, out=None, last_state=None, ws=None, stream=None):
    """ssm_scan_fwd_state with the exact zero-order-hold input coefficient
    (exp(dt a) - 1) / a in place of dt (N = 16)."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    st = lib.ssm_scan_fwd_zoh(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                              int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                              int(bool(reverse)), _ptr(initial_state), _ptr(out), _ptr(last_state),
                              _ptr(ws), 0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "ssm_scan_fwd_zoh")
    return out


def ssm_scan_fwd_ordered(x, delta, A, B, C, *, order=None, mask=None, delta_bias=None,
                         delta_softplus=True, D=None, z=None, reverse=False, out=None,
                         last_state=None, ws=None, stream=None):
    """S6 along `order` (L) int32 (None = 0..L-1) with an optional token
    mask (B, L) uint8 (0 = bypass the token)."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    st = lib.ssm_scan_fwd_ordered(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                                  int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                  _ptr(z), int(bool(reverse)), _ptr(order), _ptr(mask), _ptr(out),
                                  _ptr(last_state), _ptr(ws), 0 if ws is None else ws.numel(),
                                  _stream_handle(stream))
    _check(st, "ssm_scan_fwd_ordered")
    return out


def bidir_scan_fwd_ordered(x, delta, fwd: DirParams, bwd: DirParams, *, order=None, mask=None,
                           delta_softplus=True, out=None, ws=None, stream=None):
    """bidir_scan_fwd along `order`, with an optional token mask."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, fwd.A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.bidir_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    f, b = fwd.to_c(), bwd.to_c()
    st = lib.bidir_scan_fwd_ordered(ctypes.byref(dims), _ptr(x), _ptr(delta), int(bool(delta_softplus)),
                                    ctypes.byref(f), ctypes.byref(b), _ptr(order), _ptr(mask),
                                    _ptr(out), _ptr(ws), 0 if ws is None else ws.numel(),
                                    _stream_handle(stream))
    _check(st, "bidir_scan_fwd_ordered")
    return out


@dataclass
class Conv:
    """The conv1d before the scan (tensors on the device): weight (D, width)
    float32, bias (D) float32 or None, SiLU after it or not."""
    weight: object
    bias: object = None
    silu: bool = True

    def to_c(self) -> ssm_conv_params:
        return ssm_conv_params(_ptr(self.weight), _ptr(self.bias), int(self.weight.shape[1]),
                               int(bool(self.silu)))


def ssm_scan_fwd_conv(x_in, conv: Conv, delta, A, B, C, *, delta_bias=None, delta_softplus=True, D=None,
                      z=None, reverse=False, out=None, last_state=None, ws=None, stream=None):
    """S6 on u = conv(x_in), computed inside the scan."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x_in, A.shape[1])
    if out is None:
        out = torch.empty_like(x_in)
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x_in.device)
    cv = conv.to_c()
    st = lib.ssm_scan_fwd_conv(ctypes.byref(dims), _ptr(x_in), ctypes.byref(cv), _ptr(delta),
                               _ptr(delta_bias), int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C),
                               _ptr(D), _ptr(z), int(bool(reverse)), _ptr(out), _ptr(last_state), _ptr(ws),
                               0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "ssm_scan_fwd_conv")
    return out


def bidir_scan_fwd_conv(x_in, delta, fwd: DirParams, bwd: DirParams, conv_fwd: Conv, conv_bwd: Conv, *,
                        delta_softplus=True, out=None, ws=None, stream=None):
    """bidir_scan_fwd on x_in, each direction with its own conv."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x_in, fwd.A.shape[1])
    if out is None:
        out = torch.empty_like(x_in)
    need = lib.bidir_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x_in.device)
    f, b = fwd.to_c(), bwd.to_c()
    cf, cb = conv_fwd.to_c(), conv_bwd.to_c()
    st = lib.bidir_scan_fwd_conv(ctypes.byref(dims), _ptr(x_in), _ptr(delta), int(bool(delta_softplus)),
                                 ctypes.byref(f), ctypes.byref(b), ctypes.byref(cf), ctypes.byref(cb),
                                 _ptr(out), _ptr(ws), 0 if ws is None else ws.numel(),
                                 _stream_handle(stream))
    _check(st, "bidir_scan_fwd_conv")
    return out


def ssm_scan_bwd(x, delta, A, B, C, dout, *, delta_bias=None, delta_softplus=True, D=None, z=None,
                 reverse=False, stream=None):
    """Gradients of ssm_scan_fwd for the incoming gradient dout: returns a
    dict of float32 tensors dx, ddelta, dA, dB, dC and, when the input was
    given, dD, dz, ddelta_bias."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    f32 = dict(dtype=torch.float32, device=x.device)
    g = {"dx": torch.empty(x.shape, **f32), "ddelta": torch.empty(x.shape, **f32),
         "dA": torch.empty(A.shape, **f32), "dB": torch.empty(B.shape, **f32),
         "dC": torch.empty(C.shape, **f32)}
    if D is not None:
        g["dD"] = torch.empty(D.shape, **f32)
    if z is not None:
        g["dz"] = torch.empty(x.shape, **f32)
    if delta_bias is not None:
        g["ddelta_bias"] = torch.empty(delta_bias.shape, **f32)
    ws = workspace(lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims)), x.device)
    st = lib.ssm_scan_bwd(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                          int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                          int(bool(reverse)), _ptr(dout), _ptr(g["dx"]), _ptr(g["ddelta"]), _ptr(g["dA"]),
                          _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g.get("dD")), _ptr(g.get("dz")),
                          _ptr(g.get("ddelta_bias")), _ptr(ws), 0 if ws is None else ws.numel(),
                          _stream_handle(stream))
    _check(st, "ssm_scan_bwd")
    return g


def bidir_scan_bwd(x, delta, fwd: DirParams, bwd: DirParams, dout, *, delta_softplus=True, stream=None):
    """Gradients of bidir_scan_fwd: returns (dx, ddelta, grads_fwd, grads_bwd)
    with float32 tensors; each grads dict holds dA, dB, dC and dD, dz,
    ddelta_bias for the inputs that direction has."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, fwd.A.shape[1])
    f32 = dict(dtype=torch.float32, device=x.device)

    def mk(p: DirParams):
        g = {"dA": torch.empty(p.A.shape, **f32), "dB": torch.empty(p.B.shape, **f32),
             "dC": torch.empty(p.C.shape, **f32)}
        if p.D is not None:
            g["dD"] = torch.empty(p.D.shape, **f32)
        if p.z is not None:
            g["dz"] = torch.empty(x.shape, **f32)
        if p.delta_bias is not None:
            g["ddelta_bias"] = torch.empty(p.delta_bias.shape, **f32)
        c = ssm_dir_grads(_ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g.get("dD")), _ptr(g.get("dz")),
                          _ptr(g.get("ddelta_bias")))
        return g, c

    gf, cf = mk(fwd)
    gb, cb = mk(bwd)
    dx, ddelta = torch.empty(x.shape, **f32), torch.empty(x.shape, **f32)
    ws = workspace(lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims)), x.device)
    f, b = fwd.to_c(), bwd.to_c()
    st = lib.bidir_scan_bwd(ctypes.byref(dims), _ptr(x), _ptr(delta), int(bool(delta_softplus)),
                            ctypes.byref(f), ctypes.byref(b), _ptr(dout), _ptr(dx), _ptr(ddelta),
                            ctypes.byref(cf), ctypes.byref(cb), _ptr(ws), 0 if ws is None else ws.numel(),
                            _stream_handle(stream))
    _check(st, "bidir_scan_bwd")
    return dx, ddelta, gf, gb


def _grads(x, p: DirParams):
    """float32 gradient tensors of one direction's parameters and their
    ssm_dir_grads."""
    torch = _torch()
    f32 = dict(dtype=torch.float32, device=x.device)
    g = {"dA": torch.empty(p.A.shape, **f32), "dB": torch.empty(p.B.shape, **f32),
         "dC": torch.empty(p.C.shape, **f32)}
    if p.D is not None:
        g["dD"] = torch.empty(p.D.shape, **f32)
    if p.z is not None:
        g["dz"] = torch.empty(x.shape, **f32)
    if p.delta_bias is not None:
        g["ddelta_bias"] = torch.empty(p.delta_bias.shape, **f32)
    c = ssm_dir_grads(_ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g.get("dD")), _ptr(g.get("dz")),
                      _ptr(g.get("ddelta_bias")))
    return g, c


def ckpt_array(x, N, device=None):
    """A checkpoint array for the checkpointing scans of x (B, L, D) with N
    states: float32, ssm_scan_ckpt_size bytes (None for an empty problem)."""
    torch = _torch()
    nbytes = capi().ssm_scan_ckpt_size(ctypes.byref(s6_dims(x, N)))
    if nbytes == 0:
        return None
    return torch.empty(nbytes // 4, dtype=torch.float32, device=device or x.device)


def ssm_scan_fwd_ckpt(x, delta, A, B, C, *, delta_bias=None, delta_softplus=True, D=None, z=None,
                      reverse=False, out=None, last_state=None, ckpt=None, ws=None, stream=None):
    """ssm_scan_fwd that also stores the state entering every 4-step chunk
    (the checkpoints ssm_scan_bwd_ckpt reads).  Returns (out, ckpt)."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    if ckpt is None:
        ckpt = ckpt_array(x, A.shape[1])
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    st = lib.ssm_scan_fwd_ckpt(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                               int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                               int(bool(reverse)), _ptr(out), _ptr(last_state), _ptr(ckpt), _ptr(ws),
                               0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "ssm_scan_fwd_ckpt")
    return out, ckpt


def bidir_scan_fwd_ckpt(x, delta, fwd: DirParams, bwd: DirParams, *, delta_softplus=True, out=None,
                        ckpt_fwd=None, ckpt_bwd=None, ws=None, stream=None):
    """bidir_scan_fwd that also stores each direction's checkpoints.
    Returns (out, ckpt_fwd, ckpt_bwd)."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, fwd.A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    if ckpt_fwd is None:
        ckpt_fwd = ckpt_array(x, fwd.A.shape[1])
    if ckpt_bwd is None:
        ckpt_bwd = ckpt_array(x, fwd.A.shape[1])
    need = lib.bidir_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    f, b = fwd.to_c(), bwd.to_c()
    st = lib.bidir_scan_fwd_ckpt(ctypes.byref(dims), _ptr(x), _ptr(delta), int(bool(delta_softplus)),
                                 ctypes.byref(f), ctypes.byref(b), _ptr(out), _ptr(ckpt_fwd), _ptr(ckpt_bwd),
                                 _ptr(ws), 0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "bidir_scan_fwd_ckpt")
    return out, ckpt_fwd, ckpt_bwd


def ssm_scan_bwd_ckpt(x, delta, A, B, C, dout, ckpt, *, delta_bias=None, delta_softplus=True, D=None, z=None,
                      reverse=False, stream=None):
    """ssm_scan_bwd from the checkpoints of ssm_scan_fwd_ckpt (same inputs):
    no recompute pass.  Returns the gradients as ssm_scan_bwd does."""
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    torch = _torch()
    f32 = dict(dtype=torch.float32, device=x.device)
    g, c = _grads(x, DirParams(A=A, B=B, C=C, delta_bias=delta_bias, D=D, z=z))
    g["dx"], g["ddelta"] = torch.empty(x.shape, **f32), torch.empty(x.shape, **f32)
    st = lib.ssm_scan_bwd_ckpt(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                               int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                               int(bool(reverse)), _ptr(dout), _ptr(g["dx"]), _ptr(g["ddelta"]), c.dA, c.dB,
                               c.dC, c.dD, c.dz, c.ddelta_bias, _ptr(ckpt), _stream_handle(stream))
    _check(st, "ssm_scan_bwd_ckpt")
    return g


def bidir_scan_bwd_ckpt(x, delta, fwd: DirParams, bwd: DirParams, dout, ckpt_fwd, ckpt_bwd, *,
                        delta_softplus=True, stream=None):
    """bidir_scan_bwd from the checkpoints of bidir_scan_fwd_ckpt.  Returns
    (dx, ddelta, grads_fwd, grads_bwd) as bidir_scan_bwd does."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, fwd.A.shape[1])
    f32 = dict(dtype=torch.float32, device=x.device)
    gf, cf = _grads(x, fwd)
    gb, cb = _grads(x, bwd)
    dx, ddelta = torch.empty(x.shape, **f32), torch.empty(x.shape, **f32)
    f, b = fwd.to_c(), bwd.to_c()
    st = lib.bidir_scan_bwd_ckpt(ctypes.byref(dims), _ptr(x), _ptr(delta), int(bool(delta_softplus)),
                                 ctypes.byref(f), ctypes.byref(b), _ptr(dout), _ptr(dx), _ptr(ddelta),
                                 ctypes.byref(cf), ctypes.byref(cb), _ptr(ckpt_fwd), _ptr(ckpt_bwd),
                                 _stream_handle(stream))
    _check(st, "bidir_scan_bwd_ckpt")
    return dx, ddelta, gf, gb


def ssm_step(x, delta, A, B, C, state, *, delta_bias=None, delta_softplus=True, D=None, z=None,
             out=None, stream=None):
    """One decode step: x, delta, z (B, D); B, C (B, N); state (B, D, N)
    float32 updated in place.  Returns out (B, D) in x's dtype."""
    torch = _torch()
    lib = capi()
    Bz, Dm = x.shape
    dims = ssm_dims(Bz, 1, Dm, A.shape[1], _dtype_code(x))
    if out is None:
        out = torch.empty_like(x)
    st = lib.ssm_step(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                      int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                      _ptr(state), _ptr(out), _stream_handle(stream))
    _check(st, "ssm_step")
    return out


def ssm_scan_fwd_noalloc(x, delta, A, B, C, *, delta_bias=None, delta_softplus=True, D=None,
                         z=None, reverse=False, out=None, last_state=None, stream=None):
    """ssm_scan_fwd without a workspace: the library's own scratch array is
    used, for callers that cannot allocate device memory when they run the
    scan.  Problems needing more than SSM_NOALLOC_SCRATCH_BYTES of scratch
    raise SSMError (SSM_ERR_WORKSPACE_TOO_SMALL)."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    st = lib.ssm_scan_fwd_noalloc(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                                  int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                  _ptr(z), int(bool(reverse)), _ptr(out), _ptr(last_state),
                                  _stream_handle(stream))
    _check(st, "ssm_scan_fwd_noalloc")
    return out


def bidir_scan_fwd(x, delta, fwd: DirParams, bwd: DirParams, *, delta_softplus=True, out=None,
                   ws=None, stream=None):
    """Vision-Mamba bidirectional scan; returns out (B, L, D) in x's dtype."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, fwd.A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.bidir_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    f, b = fwd.to_c(), bwd.to_c()
    st = lib.bidir_scan_fwd(ctypes.byref(dims), _ptr(x), _ptr(delta), int(bool(delta_softplus)),
                            ctypes.byref(f), ctypes.byref(b), _ptr(out), _ptr(ws),
                            0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "bidir_scan_fwd")
    return out


def bidir_scan_fwd_zoh(x, delta, fwd: DirParams, bwd: DirParams, *, delta_softplus=True, out=None,
                       ws=None, stream=None):
    """bidir_scan_fwd with the exact zero-order-hold input coefficient in
    both directions (N = 16)."""
    torch = _torch()
    lib = capi()
    dims = s6_dims(x, fwd.A.shape[1])
    if out is None:
        out = torch.empty_like(x)
    need = lib.bidir_scan_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    f, b = fwd.to_c(), bwd.to_c()
    st = lib.bidir_scan_fwd_zoh(ctypes.byref(dims), _ptr(x), _ptr(delta), int(bool(delta_softplus)),
                                ctypes.byref(f), ctypes.byref(b), _ptr(out), _ptr(ws),
                                0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st, "bidir_scan_fwd_zoh")
    return out


def ssd_chunk_fwd(x, delta, A, B, C, *, chunk=64, delta_bias=None, delta_softplus=True, D=None,
                  z=None, out=None, last_state=None, ws=None, stream=None):
    """Mamba2 SSD chunked scan; returns out (B, L, H, P) in x's dtype."""
    torch = _torch()
    lib = capi()
    Bz, L, H, P = x.shape
    dims = ssd_dims(Bz, L, H, P, B.shape[2], chunk, _dtype_code(x))
    if out is None:
        out = torch.empty_like(x)
    need = lib.ssd_chunk_workspace_size(ctypes.byref(dims))
    if ws is None:
        ws = workspace(need, x.device)
    st = lib.ssd_chunk_fwd(ctypes.byref(dims), _ptr(x), _ptr(delta), _ptr(delta_bias),
                           int(bool(delta_softplus)), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                           _ptr(out), _ptr(last_state), _ptr(ws), 0 if ws is None else ws.numel(),
                           _stream_handle(stream))
    _check(st, "ssd_chunk_fwd")
    return out


MAPPING_AUTO, MAPPING_WHOLE_CHANNELS, MAPPING_SPLIT_STATES, MAPPING_SPLIT_STATES_2 = 0, 1, 2, 3


class s6_mapping:
    """Context manager (tests): plain S6 calls inside it take the given
    thread layout (ssm_debug_s6_mapping); the cost model decides again on
    exit."""

    def __init__(self, mode):
        self.mode = mode

    def __enter__(self):
        _check(capi().ssm_debug_s6_mapping(int(self.mode)), "ssm_debug_s6_mapping")
        return self

    def __exit__(self, *exc):
        capi().ssm_debug_s6_mapping(MAPPING_AUTO)
        return False


def scan_plan(batch, seqlen, dim, dstate, dtype=SSM_F32, bidirectional=False):
    """(segments, channels_per_lane) the library uses for an S6 problem;
    channels_per_lane -2 or -4 means that many threads share each channel."""
    lib = capi()
    dims = ssm_dims(batch, seqlen, dim, dstate, dtype)
    seg, cpl = _int(0), _int(0)
    _check(lib.ssm_scan_plan(ctypes.byref(dims), int(bool(bidirectional)), ctypes.byref(seg),
                             ctypes.byref(cpl)), "ssm_scan_plan")
    return seg.value, cpl.value


def check_device(stream=None):
    """Synchronise and raise if a kernel reported a device-side timeout."""
    _check(capi().ssm_check_device(_stream_handle(stream)), "ssm_check_device")
