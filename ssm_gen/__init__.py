"""Seeded synthetic inputs for the selective-scan workloads.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the scan's arithmetic, and it is the one piece of code that
both the float64 oracle (under ``oracle/``) and the CUDA library's tests and
bench use.

Every tensor gets its own Philox substream, keyed by (seed, tensor id), so a
tensor's values do not depend on which other tensors were drawn.

Value recipe (the shapes and distributions of the Vision-Mamba / Mamba-YOLO /
Mamba2 workloads):

* x, z ~ N(0, 1)
* raw delta = 0.5 * N(0, 1)
* delta_bias[d] = inv_softplus(dt[d]), dt log-uniform in [1e-3, 1e-1]
  (the usual dt_proj bias initialisation); the kernel then applies
  softplus(delta + delta_bias)
* S6: A[d, n] = -(n + 1) (S4D-real), or random negative values on request;
  SSD: A_h = -U[1, 16]
* B, C ~ N(0, 1) for S6, N(0, 1) / sqrt(N) for SSD, shared across channels
* D = 1, or random on request

bf16 workloads are drawn in float32 and rounded to bf16 (round to nearest
even); the arrays returned are float32 arrays whose values are exactly the
bf16 values, plus the raw uint16 bit patterns for handing to the device.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

# Tensor ids for the Philox substreams.  Changing one changes that tensor's
# values only.
_STREAM_IDS = {
    "x": 1, "delta": 2, "dt_f": 3, "dt_b": 4, "B_f": 5, "C_f": 6, "B_b": 7,
    "C_b": 8, "z_f": 9, "z_b": 10, "A_f": 11, "A_b": 12, "D_f": 13, "D_b": 14,
}


def rng_for(seed: int, name: str) -> np.random.Generator:
    """A Philox generator for one named tensor of one seed."""
    sid = _STREAM_IDS[name] if name in _STREAM_IDS else (
        1000 + sum((i + 1) * ord(c) for i, c in enumerate(name)))
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, sid])))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 arrays that already hold bf16 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _normal(seed, name, shape, scale=1.0):
    return (scale * rng_for(seed, name).standard_normal(size=shape, dtype=np.float64)).astype(np.float32)


def _dt_bias(seed, name, n):
    """inv_softplus(dt) with dt log-uniform in [1e-3, 1e-1]."""
    u = rng_for(seed, name).random(size=n)
    dt = np.exp(np.log(1e-3) + u * (np.log(1e-1) - np.log(1e-3)))
    return (dt + np.log(-np.expm1(-dt))).astype(np.float32)


@dataclasses.dataclass
class S6Inputs:
    """Host inputs of one S6 / bidirectional workload.

    Layouts (row-major, last index contiguous): x, delta, z_*: (batch, seqlen,
    dim); B_*, C_*: (batch, seqlen, dstate); A_*: (dim, dstate);
    D_*, dt_bias_*: (dim,).  Arrays of the storage dtype hold float32 values
    that are exact in that dtype.  The *_b tensors are None for a single
    direction.
    """
    batch: int
    seqlen: int
    dim: int
    dstate: int
    dtype: str            # "f32" or "bf16"
    bidir: bool
    x: np.ndarray
    delta: np.ndarray
    dt_bias_f: np.ndarray
    A_f: np.ndarray
    B_f: np.ndarray
    C_f: np.ndarray
    D_f: np.ndarray
    z_f: Optional[np.ndarray]
    dt_bias_b: Optional[np.ndarray] = None
    A_b: Optional[np.ndarray] = None
    B_b: Optional[np.ndarray] = None
    C_b: Optional[np.ndarray] = None
    D_b: Optional[np.ndarray] = None
    z_b: Optional[np.ndarray] = None

    def io_tensors(self) -> Dict[str, np.ndarray]:
        """The tensors stored in the storage dtype (x, delta, B, C, z)."""
        names = ["x", "delta", "B_f", "C_f", "z_f"]
        if self.bidir:
            names += ["B_b", "C_b", "z_b"]
        return {k: getattr(self, k) for k in names if getattr(self, k) is not None}


def make_s6_inputs(batch: int, seqlen: int, dim: int, dstate: int = 16, *,
                   dtype: str = "f32", bidir: bool = False, seed: int = 0,
                   gate: bool = True, random_A: bool = False,
                   random_D: bool = False) -> S6Inputs:
    """Draw one S6 workload.

    ``random_A`` replaces the S4D-real A = -(n+1) by A = -exp(U[-1, 2.5])
    (independent per direction), and ``random_D`` draws D ~ U[0.5, 1.5]; both
    make a parameter swap between directions visible.
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError("dtype must be 'f32' or 'bf16'")
    q = round_to_bf16 if dtype == "bf16" else (lambda a: np.ascontiguousarray(a, np.float32))
    Bz, L, Dm, N = batch, seqlen, dim, dstate

    def A_of(name):
        if random_A:
            u = rng_for(seed, name).random(size=(Dm, N))
            return (-np.exp(-1.0 + 3.5 * u)).astype(np.float32)
        return np.ascontiguousarray(np.broadcast_to(-(np.arange(N, dtype=np.float32) + 1.0), (Dm, N)))

    def D_of(name):
        if random_D:
            return (0.5 + rng_for(seed, name).random(size=Dm)).astype(np.float32)
        return np.ones(Dm, np.float32)

    out = S6Inputs(
        batch=Bz, seqlen=L, dim=Dm, dstate=N, dtype=dtype, bidir=bidir,
        x=q(_normal(seed, "x", (Bz, L, Dm))),
        delta=q(_normal(seed, "delta", (Bz, L, Dm), 0.5)),
        dt_bias_f=_dt_bias(seed, "dt_f", Dm),
        A_f=A_of("A_f"),
        B_f=q(_normal(seed, "B_f", (Bz, L, N))),
        C_f=q(_normal(seed, "C_f", (Bz, L, N))),
        D_f=D_of("D_f"),
        z_f=q(_normal(seed, "z_f", (Bz, L, Dm))) if gate else None,
    )
    if bidir:
        out.dt_bias_b = _dt_bias(seed, "dt_b", Dm)
        out.A_b = A_of("A_b")
        out.B_b = q(_normal(seed, "B_b", (Bz, L, N)))
        out.C_b = q(_normal(seed, "C_b", (Bz, L, N)))
        out.D_b = D_of("D_b")
        out.z_b = q(_normal(seed, "z_b", (Bz, L, Dm))) if gate else None
    return out


@dataclasses.dataclass
class SSDInputs:
    """Host inputs of one Mamba2 SSD workload.

    x, z: (batch, seqlen, nheads, headdim); delta: (batch, seqlen, nheads);
    B, C: (batch, seqlen, dstate) shared by all heads; A, D, dt_bias:
    (nheads,) float32.
    """
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    chunk: int
    dtype: str
    x: np.ndarray
    delta: np.ndarray
    dt_bias: np.ndarray
    A: np.ndarray
    B: np.ndarray
    C: np.ndarray
    D: np.ndarray
    z: Optional[np.ndarray]

    def io_tensors(self) -> Dict[str, np.ndarray]:
        d = {"x": self.x, "delta": self.delta, "B": self.B, "C": self.C}
        if self.z is not None:
            d["z"] = self.z
        return d


def make_ssd_inputs(batch: int, seqlen: int, nheads: int, headdim: int,
                    dstate: int, chunk: int = 64, *, dtype: str = "bf16",
                    seed: int = 0, gate: bool = True,
                    random_D: bool = False) -> SSDInputs:
    """Draw one SSD workload (A_h = -U[1, 16], B, C ~ N(0,1)/sqrt(N))."""
    q = round_to_bf16 if dtype == "bf16" else (lambda a: np.ascontiguousarray(a, np.float32))
    s = 1.0 / math.sqrt(dstate)
    A = (-(1.0 + 15.0 * rng_for(seed, "A_f").random(size=nheads))).astype(np.float32)
    D = ((0.5 + rng_for(seed, "D_f").random(size=nheads)).astype(np.float32)
         if random_D else np.ones(nheads, np.float32))
    return SSDInputs(
        batch=batch, seqlen=seqlen, nheads=nheads, headdim=headdim,
        dstate=dstate, chunk=chunk, dtype=dtype,
        x=q(_normal(seed, "x", (batch, seqlen, nheads, headdim))),
        delta=q(_normal(seed, "delta", (batch, seqlen, nheads), 0.5)),
        dt_bias=_dt_bias(seed, "dt_f", nheads),
        A=A,
        B=q(_normal(seed, "B_f", (batch, seqlen, dstate), s)),
        C=q(_normal(seed, "C_f", (batch, seqlen, dstate), s)),
        D=D,
        z=q(_normal(seed, "z_f", (batch, seqlen, nheads, headdim))) if gate else None,
    )


# The five workloads (shapes of the Vision-Mamba, high-resolution Vim,
# Mamba-YOLO stage-1 and Mamba2 cases).
WORKLOADS = {
    0: dict(kind="s6", name="vim_tiny_s6_fp32", batch=1, seqlen=196, dim=384, dstate=16,
            dtype="f32", bidir=False),
    1: dict(kind="s6", name="vim_small_bidir_fp32", batch=64, seqlen=197, dim=768, dstate=16,
            dtype="f32", bidir=True),
    2: dict(kind="s6", name="vim_hires_bidir_bf16", batch=8, seqlen=1024, dim=768, dstate=16,
            dtype="bf16", bidir=True, last_state=True),
    3: dict(kind="s6", name="mamba_yolo_rowbidir_bf16", batch=4, seqlen=16384, dim=192, dstate=16,
            dtype="bf16", bidir=True),
    4: dict(kind="ssd", name="mamba2_ssd_bf16", batch=4, seqlen=8192, nheads=32, headdim=64,
            dstate=128, chunk=64, dtype="bf16"),
}


def make_workload(idx: int, seed: int = 0, **overrides):
    """Inputs of workload ``idx`` (0..4), with optional shape overrides."""
    w = dict(WORKLOADS[idx])
    w.update(overrides)
    if w["kind"] == "s6":
        return make_s6_inputs(w["batch"], w["seqlen"], w["dim"], w["dstate"],
                              dtype=w["dtype"], bidir=w["bidir"], seed=seed)
    return make_ssd_inputs(w["batch"], w["seqlen"], w["nheads"], w["headdim"],
                           w["dstate"], w["chunk"], dtype=w["dtype"], seed=seed)


# ------------------------------------------------------------ scan orders
# Visiting orders of an H x W grid flattened row-major (position r * W + c),
# and token masks: inputs of the ordered / masked scans, no scan arithmetic.

def order_rows(H: int, W: int) -> np.ndarray:
    """Row by row, left to right (the plain flattened order)."""
    return np.arange(H * W, dtype=np.int32)


def order_cols(H: int, W: int) -> np.ndarray:
    """Column by column, top to bottom."""
    return np.array([r * W + c for c in range(W) for r in range(H)], dtype=np.int32)


def order_spiral(H: int, W: int) -> np.ndarray:
    """Square spiral from the centre cell outward, clockwise (right, down,
    left, up with run lengths 1, 1, 2, 2, 3, 3, ...), cells outside the grid
    skipped, until every cell is visited."""
    r, c = (H - 1) // 2, (W - 1) // 2
    seen = np.zeros((H, W), dtype=bool)
    out = []
    moves = [(0, 1), (1, 0), (0, -1), (-1, 0)]
    run, k = 1, 0
    if H * W:
        out.append(r * W + c)
        seen[r, c] = True
    while len(out) < H * W:
        for _ in range(2):
            dr, dc = moves[k % 4]
            for _ in range(run):
                r, c = r + dr, c + dc
                if 0 <= r < H and 0 <= c < W and not seen[r, c]:
                    seen[r, c] = True
                    out.append(r * W + c)
            k += 1
        run += 1
    return np.array(out, dtype=np.int32)


def order_random(L: int, seed: int = 0) -> np.ndarray:
    return np.random.default_rng(seed).permutation(L).astype(np.int32)


def token_mask(batch: int, L: int, keep: float, seed: int = 0) -> np.ndarray:
    """(batch, L) uint8, 1 = keep, each token kept with probability keep."""
    return (np.random.default_rng(seed).random((batch, L)) < keep).astype(np.uint8)
