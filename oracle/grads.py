"""Gradients of the S6 scan -- TEST INFRASTRUCTURE ONLY (like the rest of
oracle/): the library never imports it.

The scan is written out step by step in float64 with plain PyTorch CPU
operations -- the recurrence of the Mamba2 page "手写简化版Mamba2"
sec. 4.3 with the skip term and gate of sec. 4.4, dt = softplus(delta +
bias) of sec. 4.2 -- and its gradients are taken by PyTorch's reverse-mode
automatic differentiation, i.e. by definition.  The page (sec. 5.1) trains
exactly this way: autograd through the scan loop.  No adjoint formula is
written here; the CUDA backward kernel derives its own.  Pinned against
central finite differences in tests/test_oracle_pins.py.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def _t(a, torch, grad=False):
    if a is None:
        return None
    t = torch.tensor(np.asarray(a, dtype=np.float64), dtype=torch.float64)
    if grad:
        t.requires_grad_(True)
    return t


def s6_forward_torch(x, delta, A, B, C, *, delta_bias=None, softplus=True, D=None, z=None,
                     reverse=False):
    """The scan on float64 torch tensors (autograd-friendly): returns out."""
    import torch
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    v = delta + (delta_bias[None, None, :] if delta_bias is not None else 0.0)
    dt = torch.nn.functional.softplus(v) if softplus else v
    h = torch.zeros((Bsz, Dm, N), dtype=torch.float64)
    ys = [None] * L
    steps = range(L - 1, -1, -1) if reverse else range(L)
    for t in steps:
        dA = torch.exp(dt[:, t, :, None] * A[None])                    # (B, D, N)
        dBx = dt[:, t, :, None] * B[:, t, None, :] * x[:, t, :, None]  # (B, D, N)
        h = dA * h + dBx
        y = (h * C[:, t, None, :]).sum(-1)                             # (B, D)
        if D is not None:
            y = y + D[None] * x[:, t]
        if z is not None:
            y = y * (z[:, t] * torch.sigmoid(z[:, t]))
        ys[t] = y
    return torch.stack(ys, dim=1)


def s6_grads(x, delta, A, B, C, dout, *, delta_bias=None, softplus=True, D=None, z=None,
             reverse=False) -> Dict[str, Optional[np.ndarray]]:
    """Gradients of sum(out * dout) with respect to every input (float64
    numpy arrays; None for an absent input): keys x, delta, A, B, C, D, z,
    delta_bias, and out (the forward result)."""
    import torch
    xs = {"x": x, "delta": delta, "A": A, "B": B, "C": C, "D": D, "z": z, "delta_bias": delta_bias}
    ts = {k: _t(v, torch, grad=True) for k, v in xs.items()}
    out = s6_forward_torch(ts["x"], ts["delta"], ts["A"], ts["B"], ts["C"], delta_bias=ts["delta_bias"],
                           softplus=softplus, D=ts["D"], z=ts["z"], reverse=reverse)
    (out * _t(dout, torch)).sum().backward()
    res = {k: (None if t is None else t.grad.numpy().copy()) for k, t in ts.items()}
    res["out"] = out.detach().numpy()
    return res


def bidir_grads(x, delta, fwd: dict, bwd: dict, dout, *, softplus=True) -> Dict[str, object]:
    """Gradients of sum(out * dout) for the bidirectional scan (Vim page
    sec. 3.2: forward scan + reversed scan with its own parameters, summed),
    by float64 autograd.  Returns {"x", "delta", "out", "fwd": {...},
    "bwd": {...}} with per-direction keys A, B, C, D, z, delta_bias."""
    import torch
    keys = ("A", "B", "C", "D", "z", "delta_bias")
    tx, td = _t(x, torch, grad=True), _t(delta, torch, grad=True)
    tf = {k: _t(fwd.get(k), torch, grad=True) for k in keys}
    tb = {k: _t(bwd.get(k), torch, grad=True) for k in keys}
    out = (s6_forward_torch(tx, td, tf["A"], tf["B"], tf["C"], delta_bias=tf["delta_bias"], softplus=softplus,
                            D=tf["D"], z=tf["z"], reverse=False)
           + s6_forward_torch(tx, td, tb["A"], tb["B"], tb["C"], delta_bias=tb["delta_bias"],
                              softplus=softplus, D=tb["D"], z=tb["z"], reverse=True))
    (out * _t(dout, torch)).sum().backward()
    g = lambda t: None if t is None else t.grad.numpy().copy()
    return {"x": g(tx), "delta": g(td), "out": out.detach().numpy(),
            "fwd": {k: g(v) for k, v in tf.items()}, "bwd": {k: g(v) for k, v in tb.items()}}
