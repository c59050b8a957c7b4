"""Seeded synthetic inputs for the gated delta rule workloads.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds only random draws and their shapes -- none of the rule's arithmetic:
q and k are raw (not normalised), beta is given as its logit ``b``, and the
gate is given either directly as a log-decay draw ``g`` or as the raw
``a``/``A_log``/``dt_bias`` triple of the layer.  The prologue that turns raw
draws into (q_hat, k_hat, beta, g) lives on each side separately (the oracle
in fp64, the library in its own kernels).

All draws use ``numpy.random.default_rng(seed)`` in a fixed order, in float32
(float64 for the small parity shapes), so both sides see identical bits.

The five named workloads (sizes of a Gated DeltaNet layer with 16 key heads,
32 value heads, head size 128):

  tiny      B=1,  S=64,   Nk=Nv=2,  D=32,  fp32, g = log U(0.9, 0.999), S0 = 0
  decode    B=64, S=1,    Nk=16, Nv=32, D=128, bf16, pool of 128 slots ~ N(0, 0.05^2),
            injective slot map, lengths = accepted = 1
  prefill   B=4,  S=4096, Nk=16, Nv=32, D=128, bf16, g from a ~ N(0,1),
            A_log ~ U(log 1, log 16), dt_bias ~ U(-2, 0); S0 ~ N(0, 0.05^2)
  varlen    B=8,  padded S=8192, lengths ~ U[512, 8192] with one length 0,
            otherwise as prefill; padding positions hold random values
  decode_gk B=256, S=4, pool of 512 slots, per-key gate gk = log U(0.95, 0.9999),
            lengths ~ U[1, 4], accepted ~ U[1, length], one slot per sequence
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

NAMES = ("tiny", "decode", "prefill", "varlen", "decode_gk")


@dataclass
class Workload:
    name: str
    B: int
    Nk: int
    Nv: int
    S: int
    Dk: int
    Dv: int
    dtype: str  # "f32" or "bf16": type of q, k, v, beta, state and out
    scale: float
    q: np.ndarray  # (B, Nk, S, Dk) raw
    k: np.ndarray  # (B, Nk, S, Dk) raw
    v: np.ndarray  # (B, Nv, S, Dv)
    b: np.ndarray  # (B, Nv, S) logit of beta
    lengths: np.ndarray  # (B,) int32
    g: Optional[np.ndarray] = None  # (B, Nv, S) log-decay, when drawn directly
    a: Optional[np.ndarray] = None  # (B, Nv, S) raw gate input
    A_log: Optional[np.ndarray] = None  # (Nv,)
    dt_bias: Optional[np.ndarray] = None  # (Nv,)
    gk: Optional[np.ndarray] = None  # (B, Nv, S, Dk) per-key log-decay
    initial_state: Optional[np.ndarray] = None  # (B, Nv, Dk, Dv)
    pool: Optional[np.ndarray] = None  # (slots, Nv, Dk, Dv)
    indices: Optional[np.ndarray] = None  # (B*S,) int32
    accepted: Optional[np.ndarray] = None  # (B,) int32
    meta: dict = field(default_factory=dict)

    @property
    def kind(self) -> str:
        return "decode" if self.pool is not None else "prefill"

    @property
    def valid_tokens(self) -> int:
        return int(self.lengths.sum())


def _normal(rng, shape, std=1.0, dtype=np.float32):
    x = rng.standard_normal(size=shape, dtype=np.float64 if dtype == np.float64 else np.float32)
    if std != 1.0:
        x *= std
    return x.astype(dtype, copy=False)


def _loguniform_gate(rng, shape, lo, hi, dtype):
    return np.log(rng.uniform(lo, hi, size=shape)).astype(dtype)


_SPECS = {
    "tiny": dict(B=1, S=64, Nk=2, Nv=2, D=32, seed=0, dtype="f32"),
    "decode": dict(B=64, S=1, Nk=16, Nv=32, D=128, seed=1, dtype="bf16"),
    "prefill": dict(B=4, S=4096, Nk=16, Nv=32, D=128, seed=2, dtype="bf16"),
    "varlen": dict(B=8, S=8192, Nk=16, Nv=32, D=128, seed=3, dtype="bf16"),
    "decode_gk": dict(B=256, S=4, Nk=16, Nv=32, D=128, seed=4, dtype="bf16"),
}


def spec(name: str) -> dict:
    """The sizes, seed and dtype of a named workload, without drawing it."""
    if name not in NAMES:
        raise ValueError(f"unknown workload {name!r}; choose from {NAMES}")
    return dict(_SPECS[name])


def generate(name: str, *, B=None, S=None, Nk=None, Nv=None, D=None, seed=None, fdtype=None) -> Workload:
    """Draw one of the named workloads.  Keyword overrides shrink it (for
    parity tests at small sizes) while keeping the same distributions."""
    base = spec(name)
    B = base["B"] if B is None else B
    S = base["S"] if S is None else S
    Nk = base["Nk"] if Nk is None else Nk
    Nv = base["Nv"] if Nv is None else Nv
    D = base["D"] if D is None else D
    seed = base["seed"] if seed is None else seed
    dt = base["dtype"]
    fd = fdtype if fdtype is not None else (np.float64 if B * S * Nv * D <= (1 << 22) else np.float32)
    rng = np.random.default_rng(seed)
    q = _normal(rng, (B, Nk, S, D), dtype=fd)
    k = _normal(rng, (B, Nk, S, D), dtype=fd)
    v = _normal(rng, (B, Nv, S, D), dtype=fd)
    b = _normal(rng, (B, Nv, S), dtype=fd)
    w = Workload(name=name, B=B, Nk=Nk, Nv=Nv, S=S, Dk=D, Dv=D, dtype=dt, scale=1.0 / math.sqrt(D),
                 q=q, k=k, v=v, b=b, lengths=np.full(B, S, np.int32), meta={"seed": seed, "fd": fd})
    if name in ("tiny", "decode", "decode_gk"):
        w.g = _loguniform_gate(rng, (B, Nv, S), 0.9, 0.999, np.float32 if dt == "bf16" else fd)
    else:
        w.A_log = rng.uniform(math.log(1.0), math.log(16.0), size=Nv).astype(np.float32)
        w.a = _normal(rng, (B, Nv, S), dtype=np.float32)
        w.dt_bias = rng.uniform(-2.0, 0.0, size=Nv).astype(np.float32)
    if name in ("prefill", "varlen"):
        w.initial_state = _normal(rng, (B, Nv, D, D), std=0.05, dtype=fd)
    if name == "varlen":
        lo = min(512, S)
        L = rng.integers(lo, S, size=B, endpoint=True).astype(np.int32)
        L[int(rng.integers(B))] = 0
        w.lengths = L
    if name == "decode":
        slots = 2 * B
        w.pool = _normal(rng, (slots, Nv, D, D), std=0.05, dtype=fd)
        perm = rng.permutation(slots)[:B].astype(np.int32)
        w.indices = np.repeat(perm, S).astype(np.int32)
        w.lengths = np.full(B, S, np.int32)
        w.accepted = w.lengths.copy()
    if name == "decode_gk":
        slots = 2 * B
        w.pool = _normal(rng, (slots, Nv, D, D), std=0.05, dtype=fd)
        w.gk = _loguniform_gate(rng, (B, Nv, S, D), 0.95, 0.9999, np.float32 if dt == "bf16" else fd)
        w.lengths = rng.integers(1, S, size=B, endpoint=True).astype(np.int32)
        w.accepted = np.array([rng.integers(1, L, endpoint=True) for L in w.lengths], np.int32)
        perm = rng.permutation(slots)[:B].astype(np.int32)
        w.indices = np.repeat(perm, S).astype(np.int32)
    if name == "tiny":
        w.initial_state = None
    return w


def random_case(*, B, Nk, Nv, S, Dk, Dv, seed, gate="loguniform", lengths=None, initial_state=True,
                with_gk=False, slots=None, share_slot=True, fd=np.float64) -> Workload:
    """A generic small case for parity tests (any shape).  gate is
    "loguniform" (g = log U(0.9, 0.999)), "strong" (raw a/A_log/dt_bias as in
    the prefill workload) or "none" (no gate)."""
    rng = np.random.default_rng(seed)
    q = _normal(rng, (B, Nk, S, Dk), dtype=fd)
    k = _normal(rng, (B, Nk, S, Dk), dtype=fd)
    v = _normal(rng, (B, Nv, S, Dv), dtype=fd)
    b = _normal(rng, (B, Nv, S), dtype=fd)
    w = Workload(name=f"case{seed}", B=B, Nk=Nk, Nv=Nv, S=S, Dk=Dk, Dv=Dv, dtype="f32",
                 scale=1.0 / math.sqrt(Dk), q=q, k=k, v=v, b=b, lengths=np.full(B, S, np.int32),
                 meta={"seed": seed, "fd": fd})
    if gate == "loguniform":
        w.g = _loguniform_gate(rng, (B, Nv, S), 0.9, 0.999, fd)
    elif gate == "strong":
        w.A_log = rng.uniform(0.0, math.log(16.0), size=Nv).astype(np.float32)
        w.a = _normal(rng, (B, Nv, S), dtype=np.float32)
        w.dt_bias = rng.uniform(-2.0, 0.0, size=Nv).astype(np.float32)
    elif gate != "none":
        raise ValueError(gate)
    if initial_state:
        w.initial_state = _normal(rng, (B, Nv, Dk, Dv), std=0.05, dtype=fd)
    if lengths is not None:
        w.lengths = np.asarray(lengths, np.int32)
    if with_gk:
        w.gk = _loguniform_gate(rng, (B, Nv, S, Dk), 0.95, 0.9999, fd)
    if slots is not None:
        w.pool = _normal(rng, (slots, Nv, Dk, Dv), std=0.05, dtype=fd)
        if share_slot:
            perm = rng.permutation(slots)[:B].astype(np.int32)
            w.indices = np.repeat(perm, S).astype(np.int32)
        else:
            w.indices = rng.permutation(slots)[:B * S].astype(np.int32)
        w.accepted = np.array([rng.integers(0, L, endpoint=True) if L > 0 else 0 for L in w.lengths], np.int32)
    return w


def epilogue_inputs(w: Workload):
    """The output gate branch z ~ N(0, 1), shape (B, Nv, S, Dv), and the RMSNorm weight
    norm_w ~ U(0.5, 1.5), shape (Dv,), of the layer's output epilogue.  Drawn from a stream of
    their own (seeded by the workload's seed and 1), so the workload's other draws are unchanged."""
    rng = np.random.default_rng([int(w.meta["seed"]), 1])
    z = _normal(rng, (w.B, w.Nv, w.S, w.Dv), dtype=w.meta.get("fd", np.float32))
    norm_w = rng.uniform(0.5, 1.5, size=w.Dv).astype(np.float32)
    return z, norm_w


def conv_inputs(w: Workload, K: int = 4, with_state: bool = True, with_bias: bool = True):
    """Inputs of the depthwise causal conv1d before the rule, for a workload's head layout: the fused
    projection x ~ N(0, 1) of shape (B, S, C), C = 2 Nk Dk + Nv Dv (channels last), taps ~ U(-0.5, 0.5) of
    shape (C, K), bias ~ N(0, 0.1^2) of shape (C,) and a state ~ N(0, 1) of shape (B, C, K).  Drawn from a
    stream of their own (the workload's seed and 2)."""
    rng = np.random.default_rng([int(w.meta["seed"]), 2])
    C = 2 * w.Nk * w.Dk + w.Nv * w.Dv
    fd = w.meta.get("fd", np.float32)
    x = _normal(rng, (w.B, w.S, C), dtype=fd)
    weight = rng.uniform(-0.5, 0.5, size=(C, K)).astype(fd)
    bias = _normal(rng, (C,), std=0.1, dtype=fd) if with_bias else None
    state = _normal(rng, (w.B, C, K), dtype=fd) if with_state else None
    return x, weight, bias, state
