"""Shared helpers for the parity tests: dtype rounding, tolerances, input staging.

Inputs always start from ``workloads`` draws.  For the un-fused calls the
prologue (l2norm, sigmoid, gate) is taken from the fp64 ORACLE and rounded to
the call's dtype; both the CUDA path and the oracle then read those same
rounded values.  For the fused calls both sides start from the same raw
(rounded) draws and each applies its own prologue.  Nothing the CUDA path
computes ever becomes an oracle input or an expected value.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances of the parity bar: fp32 inputs, max-abs <= 1e-4 on out and state;
# bf16 inputs and state, rel-L2 <= 2e-2 per tensor against the fp64 oracle fed the
# same bf16-rounded inputs.  fp16 (not fixed by the pages): rel-L2 <= 2e-3, derived from
# the arithmetic -- the fp16 paths compute in fp32 from the rounded inputs the oracle also
# sees; the CUDA-core kernels round each output once to fp16 (2^-11 relative) and the
# tensor-core prefill also rounds its MMA operand copies (T, W, the state, v_new, P) to fp16,
# the same number of roundings at which its bf16 (2^-9) twin stays near 3e-3, i.e. near
# 8e-4 for fp16.
F32_MAX_ABS = 1e-4
BF16_REL_L2 = 2e-2
F16_REL_L2 = 2e-3

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def rnd(x, dt: str) -> np.ndarray:
    """Round to the call dtype and return the rounded values as fp64."""
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x)).to(TORCH_DT[dt])
    return t.to(torch.float64).numpy()


def rnd32(x):
    if x is None:
        return None
    return np.asarray(x, np.float32).astype(np.float64)


def dev(x, dt: str, device="cuda"):
    """fp64 numpy (already rounded) -> device tensor of the call dtype (exact)."""
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=TORCH_DT[dt])


def dev_i32(x, device="cuda"):
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(np.asarray(x, np.int32))).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def assert_close(x, ref, dt: str, what: str):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (what, x.shape, ref.shape)
    assert np.all(np.isfinite(x)), f"{what}: non-finite values"
    if dt == "f32":
        err = float(np.abs(x - ref).max()) if x.size else 0.0
        assert err <= F32_MAX_ABS, f"{what}: max-abs {err:.3e} > {F32_MAX_ABS}"
    else:
        err = rel_l2(x, ref)
        bar = F16_REL_L2 if dt == "f16" else BF16_REL_L2
        assert err <= bar, f"{what}: rel-L2 {err:.3e} > {bar}"
    return err


def unfused_inputs(w, dt: str):
    """Prologue by the oracle (fp64), rounded to dt: returns fp64 arrays
    q_hat, k_hat, v, beta, g (fp32-rounded), gk, initial_state."""
    pro = oracle.prologue(q=w.q, k=w.k, b=w.b, a=w.a, A_log=w.A_log, dt_bias=w.dt_bias)
    g = pro["g"] if "g" in pro else w.g
    return dict(q=rnd(pro["q_hat"], dt), k=rnd(pro["k_hat"], dt), v=rnd(w.v, dt), beta=rnd(pro["beta"], dt),
                g=rnd32(g), gk=rnd32(w.gk), initial_state=rnd(w.initial_state, dt))


def fused_inputs(w, dt: str):
    """Raw draws rounded to dt (a, A_log, dt_bias in fp32), plus the oracle's
    fp64 prologue of exactly those rounded values."""
    raw = dict(q=rnd(w.q, dt), k=rnd(w.k, dt), v=rnd(w.v, dt), b=rnd(w.b, dt), initial_state=rnd(w.initial_state, dt),
               gk=rnd32(w.gk))
    if w.a is not None:
        raw.update(a=rnd32(w.a), A_log=rnd32(w.A_log), dt_bias=rnd32(w.dt_bias), g=None)
    else:
        raw.update(g=rnd32(w.g))
    pro = oracle.prologue(q=raw["q"], k=raw["k"], b=raw["b"], a=raw.get("a"), A_log=raw.get("A_log"),
                          dt_bias=raw.get("dt_bias"))
    ref = dict(q=pro["q_hat"], k=pro["k_hat"], v=raw["v"], beta=pro["beta"], g=pro.get("g", raw["g"]),
               gk=raw["gk"], initial_state=raw["initial_state"])
    return raw, ref
