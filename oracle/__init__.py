"""Float64 CPU oracle for the selective scan -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
may import this package.  The CUDA library never calls it.  The arithmetic
lives in ``ssm_oracle.c`` (plain loops in double precision); this module only
compiles it with gcc, loads it with ctypes and converts arrays to float64.

Functions (all return float64 numpy arrays):

* ``s6(inp, reverse=False, ...)``      -- one direction (the per-step scan,
  with skip term and SiLU gate)
* ``bidir(inp, ...)``                  -- forward + reversed with separate
  parameters, summed
* ``s6_arrays(..., zoh=True)`` / ``bidir_arrays(..., zoh=True)`` -- the
  same scans with the exact zero-order-hold input coefficient instead of
  dt B
* ``ssd_seq(inp, ...)``                -- Mamba2 SSD as the sequential scan
  with a scalar A per head
* ``ssd_chunked(inp, chunk, ...)``     -- Mamba2 SSD in the chunked form
  (matrix products inside chunks, state passed between chunks)

``cols`` restricts the work to some columns (b*D + d for S6,
(b*H + h)*P + p for SSD); other outputs are left at zero.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into liboracle.so (plain -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_s6.argtypes = [_i64] * 4 + [_dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, _dp,
                                               ctypes.c_int, _dp, _dp, _ip, _i64, ctypes.c_int]
        lib.oracle_s6_state.argtypes = ([_i64] * 4 + [_dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, _dp,
                                         ctypes.c_int, _dp, _dp, _dp, _dp, _i64, ctypes.c_int])
        lib.oracle_s6_masked.argtypes = ([_i64] * 4 + [_dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, _dp,
                                          ctypes.c_int, ctypes.c_void_p, _dp, _dp, _ip, _i64,
                                          ctypes.c_int])
        lib.oracle_bidir.argtypes = ([_i64] * 4 + [_dp, _dp, ctypes.c_int] + [_dp] * 7 + [_dp] * 7
                                     + [_dp, _ip, _i64, ctypes.c_int])
        lib.oracle_s6_zoh.argtypes = lib.oracle_s6_state.argtypes
        lib.oracle_bidir_zoh.argtypes = lib.oracle_bidir.argtypes
        lib.oracle_ssd_seq.argtypes = [_i64] * 5 + [_dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp,
                                                    _dp, _dp, _dp, _ip, _i64, ctypes.c_int]
        lib.oracle_ssd_chunked.argtypes = [_i64] * 6 + [_dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp,
                                                        _dp, _dp, _dp, _dp, ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _cols(cols):
    if cols is None:
        return None, None, 0
    c = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    return c, c.ctypes.data_as(_ip), len(c)


def s6_arrays(x, delta, A, B, C, *, delta_bias=None, softplus=True, D=None, z=None,
              reverse=False, cols=None, want_state=True, nthreads=1, initial_state=None, zoh=False
              ) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """Single-direction S6 on raw arrays: returns (out (B,L,D), last_state (B,D,N)).

    initial_state (B, D, N): the state before the first step (None = zero).
    zoh: the exact zero-order-hold input coefficient (exp(dt a) - 1) / a of
    the Mamba2 page, sec. 2.2, instead of its dt B approximation."""
    x, delta, A, B, C = map(_f64, (x, delta, A, B, C))
    delta_bias, D, z, h0 = map(_f64, (delta_bias, D, z, initial_state))
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    out = np.zeros((Bsz, L, Dm))
    st = np.zeros((Bsz, Dm, N)) if want_state else None
    keep, cp, nc = _cols(cols)
    if zoh:
        if h0 is not None:
            assert h0.shape == (Bsz, Dm, N)
        _load().oracle_s6_zoh(Bsz, L, Dm, N, _ptr(x), _ptr(delta), _ptr(delta_bias),
                              int(softplus), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                              int(reverse), _ptr(h0), _ptr(out), _ptr(st), cp, nc, int(nthreads))
    elif h0 is None:
        _load().oracle_s6(Bsz, L, Dm, N, _ptr(x), _ptr(delta), _ptr(delta_bias), int(softplus),
                          _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), int(reverse), _ptr(out),
                          _ptr(st), cp, nc, int(nthreads))
    else:
        assert h0.shape == (Bsz, Dm, N)
        _load().oracle_s6_state(Bsz, L, Dm, N, _ptr(x), _ptr(delta), _ptr(delta_bias),
                                int(softplus), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                int(reverse), _ptr(h0), _ptr(out), _ptr(st), cp, nc, int(nthreads))
    return out, st


def s6_ordered_arrays(x, delta, A, B, C, *, order=None, mask=None, delta_bias=None, softplus=True,
                      D=None, z=None, reverse=False, cols=None, nthreads=1
                      ) -> Tuple[np.ndarray, np.ndarray]:
    """Single-direction S6 along a given order of the L positions, with an
    optional token mask.

    order (L,): a permutation of 0..L-1; step i visits position order[i]
    (reversed: order[L-1-i]) -- the row, column, cross and spiral scans of
    the Samba (sec. 3.1) and Mamba-YOLO (sec. 1.2, 4.4) pages.  mask (B, L),
    indexed by position: 0 bypasses the token (Samba page, sec. 2) -- the
    state passes through unchanged and its output is 0.
    Defined as the scan of the inputs gathered in that order, outputs
    scattered back to their positions."""
    x, delta, A, B, C = map(_f64, (x, delta, A, B, C))
    delta_bias, D, z = map(_f64, (delta_bias, D, z))
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    o = np.arange(L) if order is None else np.asarray(order, dtype=np.int64)
    assert sorted(o.tolist()) == list(range(L)), "order must be a permutation"
    g = lambda a: None if a is None else np.ascontiguousarray(np.take(a, o, axis=1))
    xg, dg, zg, Bg, Cg = g(x), g(delta), g(z), g(B), g(C)
    outg = np.zeros((Bsz, L, Dm))
    st = np.zeros((Bsz, Dm, N))
    keep, cp, nc = _cols(cols)
    if mask is None:
        _load().oracle_s6(Bsz, L, Dm, N, _ptr(xg), _ptr(dg), _ptr(delta_bias), int(softplus),
                          _ptr(A), _ptr(Bg), _ptr(Cg), _ptr(D), _ptr(zg), int(reverse), _ptr(outg),
                          _ptr(st), cp, nc, int(nthreads))
    else:
        mg = np.ascontiguousarray(np.take(np.asarray(mask, dtype=np.uint8), o, axis=1))
        _load().oracle_s6_masked(Bsz, L, Dm, N, _ptr(xg), _ptr(dg), _ptr(delta_bias), int(softplus),
                                 _ptr(A), _ptr(Bg), _ptr(Cg), _ptr(D), _ptr(zg), int(reverse),
                                 mg.ctypes.data_as(ctypes.c_void_p), _ptr(outg), _ptr(st), cp, nc,
                                 int(nthreads))
    out = np.zeros_like(outg)
    out[:, o] = outg
    return out, st


def bidir_ordered_arrays(x, delta, fwd: dict, bwd: dict, *, order=None, mask=None, softplus=True,
                         cols=None, nthreads=1):
    """Bidirectional scan along an order (Vim page sec. 3.2 on the ordered
    sequence): the forward parameters scan the order, the backward ones scan
    it reversed, the two outputs are summed.  Returns (out, last_f, last_b)."""
    kw = dict(order=order, mask=mask, softplus=softplus, cols=cols, nthreads=nthreads)
    of, lf = s6_ordered_arrays(x, delta, fwd["A"], fwd["B"], fwd["C"], delta_bias=fwd.get("delta_bias"),
                               D=fwd.get("D"), z=fwd.get("z"), reverse=False, **kw)
    ob, lb = s6_ordered_arrays(x, delta, bwd["A"], bwd["B"], bwd["C"], delta_bias=bwd.get("delta_bias"),
                               D=bwd.get("D"), z=bwd.get("z"), reverse=True, **kw)
    return of + ob, lf, lb


def conv_u(x, weight, bias=None, silu=True, reverse=False):
    """The depthwise causal conv1d before the scan (Mamba2 page sec. 4.4
    listing: groups = channels, padding K-1, the first L outputs kept), with
    an optional bias and SiLU after it:
        u[b,t,d] = act(bias[d] + sum_k weight[d,k] x[b, t-(K-1)+k, d]),
    x taken as 0 outside [0, L).  reverse: the conv of the flipped sequence
    (a reversed scan's own conv, as each Vim direction has), flipped back --
    the window then runs over t .. t+K-1."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    if reverse:
        return conv_u(x[:, ::-1], w, bias, silu, False)[:, ::-1].copy()
    Bsz, L, Dm = x.shape
    K = w.shape[1]
    u = np.zeros_like(x)
    for k in range(K):
        s = K - 1 - k                      # x[t - s] contributes with weight[:, k]
        if s < L:
            u[:, s:, :] += w[None, None, :, k] * x[:, :L - s, :]
    if bias is not None:
        u += np.asarray(bias, dtype=np.float64)[None, None, :]
    if silu:
        u = u / (1.0 + np.exp(-u))
    return u


def s6_conv_arrays(x_in, conv_weight, delta, A, B, C, *, conv_bias=None, conv_silu=True,
                   reverse=False, **kw):
    """S6 whose input is conv_u(x_in): the scan and its D skip both use u."""
    u = conv_u(x_in, conv_weight, conv_bias, conv_silu, reverse)
    return s6_arrays(u, delta, A, B, C, reverse=reverse, **kw)


def bidir_conv_arrays(x_in, delta, fwd: dict, bwd: dict, conv_f: dict, conv_b: dict, *, softplus=True,
                      cols=None, nthreads=1):
    """Bidirectional scan where each direction convolves x_in with its own
    conv (conv_* dicts: weight, bias, silu) along its scan direction."""
    uf = conv_u(x_in, conv_f["weight"], conv_f.get("bias"), conv_f.get("silu", True), False)
    ub = conv_u(x_in, conv_b["weight"], conv_b.get("bias"), conv_b.get("silu", True), True)
    of, lf = s6_arrays(uf, delta, fwd["A"], fwd["B"], fwd["C"], delta_bias=fwd.get("delta_bias"),
                       softplus=softplus, D=fwd.get("D"), z=fwd.get("z"), cols=cols, nthreads=nthreads)
    ob, lb = s6_arrays(ub, delta, bwd["A"], bwd["B"], bwd["C"], delta_bias=bwd.get("delta_bias"),
                       softplus=softplus, D=bwd.get("D"), z=bwd.get("z"), reverse=True, cols=cols,
                       nthreads=nthreads)
    return of + ob, lf, lb


def step_arrays(x, delta, A, B, C, state, *, delta_bias=None, softplus=True, D=None, z=None):
    """One time step of S6 for every (b, d) from a stored state -- the
    recurrent (decode) form: x, delta, z (B, D); B, C (B, N); state (B, D, N).
    Returns (y (B, D), new state (B, D, N)).  It is s6_arrays on a length-1
    sequence started from `state`."""
    add_t = lambda a: None if a is None else np.asarray(a)[:, None, ...]
    out, st = s6_arrays(add_t(x), add_t(delta), A, add_t(B), add_t(C), delta_bias=delta_bias,
                        softplus=softplus, D=D, z=add_t(z), initial_state=state)
    return out[:, 0, :], st


def s6(inp, reverse=False, cols=None, softplus=True, nthreads=1):
    """S6 on an ssm_gen.S6Inputs, forward-direction parameters."""
    return s6_arrays(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, delta_bias=inp.dt_bias_f,
                     softplus=softplus, D=inp.D_f, z=inp.z_f, reverse=reverse, cols=cols,
                     nthreads=nthreads)


def bidir_arrays(x, delta, fwd: dict, bwd: dict, *, softplus=True, cols=None, nthreads=1, zoh=False):
    """Bidirectional scan on raw arrays.

    fwd / bwd: dicts with keys delta_bias, A, B, C, D, z (delta_bias, D, z may
    be None).  zoh: the exact zero-order-hold coefficient (see s6_arrays) in
    both directions.  Returns (out, last_state_f, last_state_b).
    """
    x, delta = _f64(x), _f64(delta)
    Bsz, L, Dm = x.shape
    N = np.asarray(fwd["A"]).shape[1]
    out = np.zeros((Bsz, L, Dm))
    lf = np.zeros((Bsz, Dm, N))
    lb = np.zeros((Bsz, Dm, N))
    f = {k: _f64(fwd.get(k)) for k in ("delta_bias", "A", "B", "C", "D", "z")}
    b = {k: _f64(bwd.get(k)) for k in ("delta_bias", "A", "B", "C", "D", "z")}
    keep, cp, nc = _cols(cols)
    fn = _load().oracle_bidir_zoh if zoh else _load().oracle_bidir
    fn(Bsz, L, Dm, N, _ptr(x), _ptr(delta), int(softplus),
       _ptr(f["delta_bias"]), _ptr(f["A"]), _ptr(f["B"]), _ptr(f["C"]), _ptr(f["D"]), _ptr(f["z"]), _ptr(lf),
       _ptr(b["delta_bias"]), _ptr(b["A"]), _ptr(b["B"]), _ptr(b["C"]), _ptr(b["D"]), _ptr(b["z"]), _ptr(lb),
       _ptr(out), cp, nc, int(nthreads))
    return out, lf, lb


def bidir(inp, cols=None, softplus=True, nthreads=1):
    """Bidirectional scan on an ssm_gen.S6Inputs with bidir=True."""
    fwd = dict(delta_bias=inp.dt_bias_f, A=inp.A_f, B=inp.B_f, C=inp.C_f, D=inp.D_f, z=inp.z_f)
    bwd = dict(delta_bias=inp.dt_bias_b, A=inp.A_b, B=inp.B_b, C=inp.C_b, D=inp.D_b, z=inp.z_b)
    return bidir_arrays(inp.x, inp.delta, fwd, bwd, softplus=softplus, cols=cols, nthreads=nthreads)


def ssd_seq_arrays(x, delta, A, B, C, *, delta_bias=None, softplus=True, D=None, z=None,
                   cols=None, nthreads=1):
    """SSD by the sequential recurrence: returns (out (B,L,H,P), last_state (B,H,P,N))."""
    x, delta, A, B, C = map(_f64, (x, delta, A, B, C))
    delta_bias, D, z = map(_f64, (delta_bias, D, z))
    Bsz, L, H, P = x.shape
    N = B.shape[2]
    out = np.zeros((Bsz, L, H, P))
    st = np.zeros((Bsz, H, P, N))
    keep, cp, nc = _cols(cols)
    _load().oracle_ssd_seq(Bsz, L, H, P, N, _ptr(x), _ptr(delta), _ptr(delta_bias), int(softplus),
                           _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(out), _ptr(st),
                           cp, nc, int(nthreads))
    return out, st


def ssd_seq(inp, cols=None, softplus=True, nthreads=1):
    return ssd_seq_arrays(inp.x, inp.delta, inp.A, inp.B, inp.C, delta_bias=inp.dt_bias,
                          softplus=softplus, D=inp.D, z=inp.z, cols=cols, nthreads=nthreads)


def ssd_chunked_arrays(x, delta, A, B, C, chunk, *, delta_bias=None, softplus=True, D=None,
                       z=None, nthreads=1):
    """SSD by the chunked form: returns (out (B,L,H,P), last_state (B,H,P,N))."""
    x, delta, A, B, C = map(_f64, (x, delta, A, B, C))
    delta_bias, D, z = map(_f64, (delta_bias, D, z))
    Bsz, L, H, P = x.shape
    N = B.shape[2]
    out = np.zeros((Bsz, L, H, P))
    st = np.zeros((Bsz, H, P, N))
    _load().oracle_ssd_chunked(Bsz, L, H, P, N, int(chunk), _ptr(x), _ptr(delta),
                               _ptr(delta_bias), int(softplus), _ptr(A), _ptr(B), _ptr(C),
                               _ptr(D), _ptr(z), _ptr(out), _ptr(st), int(nthreads))
    return out, st


def ssd_chunked(inp, chunk=None, softplus=True, nthreads=1):
    return ssd_chunked_arrays(inp.x, inp.delta, inp.A, inp.B, inp.C,
                              inp.chunk if chunk is None else chunk, delta_bias=inp.dt_bias,
                              softplus=softplus, D=inp.D, z=inp.z, nthreads=nthreads)
