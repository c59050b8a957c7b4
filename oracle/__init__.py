"""fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

This package is the reference the CUDA library is checked against.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  It shares no code with the CUDA path and never calls it.

``gdr_oracle.c`` holds the token-by-token definition (compiled here with gcc,
no fast-math); ``forms.py`` holds independent formulations from the pages
(the chunked WY form, the pseudo-value form, gated linear attention by brute
force) used to pin it.  ``gated_rmsnorm`` is the layer's output epilogue and
``causal_conv1d`` the depthwise causal convolution before the rule, each written
out from its definition and pinned by closed forms and library routines.  Every function here is pinned by
``tests/test_oracle_pins.py`` (closed forms, worked examples printed on the
pages, independent formulations, brute force, invariants); none is left
unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libgdr_oracle.so")
_lock = threading.Lock()
_lib = None

__all__ = ["build", "lib", "prologue", "chunk_fwd", "recurrent_step", "gated_rmsnorm", "causal_conv1d", "threads",
           "set_threads"]


def build(force: bool = False) -> str:
    """Compile gdr_oracle.c into oracle/_build/libgdr_oracle.so (gcc, -O2 -fopenmp)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            c_int, c_double = ctypes.c_int, ctypes.c_double
            L.gdr_oracle_prologue.restype = None
            L.gdr_oracle_prologue.argtypes = [dp, dp, dp, dp, dp, dp, c_double, c_int, c_int, c_int, c_int, c_int,
                                              dp, dp, dp, dp]
            L.gdr_oracle_chunk_fwd.restype = c_int
            L.gdr_oracle_chunk_fwd.argtypes = [dp, dp, dp, dp, dp, dp, ip, c_double, c_int, c_int, c_int, c_int,
                                               c_int, c_int, dp, dp]
            L.gdr_oracle_recurrent_step.restype = c_int
            L.gdr_oracle_recurrent_step.argtypes = [dp, dp, dp, dp, dp, dp, dp, c_int, ip, ip, ip, c_int, c_double,
                                                    c_int, c_int, c_int, c_int, c_int, c_int, dp]
            L.gdr_oracle_threads.restype = c_int
            L.gdr_oracle_threads.argtypes = []
            L.gdr_oracle_set_threads.restype = None
            L.gdr_oracle_set_threads.argtypes = [c_int]
            _lib = L
    return _lib


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x):
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _dp(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def threads() -> int:
    """OpenMP threads the C oracle runs with."""
    return int(lib().gdr_oracle_threads())


def set_threads(n: int) -> None:
    """OpenMP threads of later oracle calls (the results do not depend on it)."""
    lib().gdr_oracle_set_threads(int(n))


def prologue(q=None, k=None, b=None, a=None, A_log=None, dt_bias=None, eps: float = 1e-6):
    """fp64 prologue: l2norm(q), l2norm(k) (eps inside the sqrt), sigmoid(b),
    g = -exp(A_log) * softplus(a + dt_bias).

    q, k: (B, Nk, S, Dk); b, a: (B, Nv, S); A_log, dt_bias: (Nv).
    Returns a dict with whichever of q_hat, k_hat, beta, g could be formed.
    Follows the transformers GatedDeltaNet forward (blog page, beta and g
    lines, l2norm in torch_recurrent_gated_delta_rule) and deltanet.rs
    (module docstring, l2norm, softplus).
    """
    L = lib()
    res = {}
    qa, ka = _f64(q), _f64(k)
    if qa is not None or ka is not None:
        B, Nk, S, Dk = (qa if qa is not None else ka).shape
        qh = np.empty_like(qa) if qa is not None else None
        kh = np.empty_like(ka) if ka is not None else None
        L.gdr_oracle_prologue(_dp(qa), _dp(ka), None, None, None, None, float(eps), B, Nk, 1, S, Dk,
                              _dp(qh), _dp(kh), None, None)
        if qh is not None:
            res["q_hat"] = qh
        if kh is not None:
            res["k_hat"] = kh
    ba, aa = _f64(b), _f64(a)
    if ba is not None or aa is not None:
        B, Nv, S = (ba if ba is not None else aa).shape
        be = np.empty_like(ba) if ba is not None else None
        gg = None
        Al, dtb = _f64(A_log), _f64(dt_bias)
        if aa is not None:
            if Al is None or dtb is None or Al.shape != (Nv,) or dtb.shape != (Nv,):
                raise ValueError("a needs A_log and dt_bias of shape (Nv,)")
            gg = np.empty_like(aa)
        L.gdr_oracle_prologue(None, None, _dp(ba), _dp(aa), _dp(Al), _dp(dtb), float(eps), B, 1, Nv, S, 1,
                              None, None, _dp(be), _dp(gg))
        if be is not None:
            res["beta"] = be
        if gg is not None:
            res["g"] = gg
    return res


def chunk_fwd(q, k, v, beta, g=None, initial_state=None, actual_seq_lengths=None, scale: float = 1.0):
    """fp64 semantics of the chunked-prefill call, token by token.

    Returns (out (B,Nv,S,Dv), final_state (B,Nv,Dk,Dv)).  Raises ValueError on
    the shape errors the lite_boost chunk op defines (Nv % Nk, lengths
    outside [0, S]).
    """
    qa, ka, va, ba = _f64(q), _f64(k), _f64(v), _f64(beta)
    B, Nk, S, Dk = qa.shape
    Nv, Dv = va.shape[1], va.shape[3]
    ga, s0, L = _f64(g), _f64(initial_state), _i32(actual_seq_lengths)
    out = np.empty((B, Nv, S, Dv), np.float64)
    fin = np.empty((B, Nv, Dk, Dv), np.float64)
    rc = lib().gdr_oracle_chunk_fwd(_dp(qa), _dp(ka), _dp(va), _dp(ba), _dp(ga), _dp(s0), _ip(L), float(scale),
                                    B, Nk, Nv, S, Dk, Dv, _dp(out), _dp(fin))
    if rc != 0:
        raise ValueError(f"oracle chunk_fwd rejected the arguments (code {rc})")
    return out, fin


def recurrent_step(q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths,
                   num_accepted_tokens=None, scale: float = 1.0, per_token: bool = False):
    """fp64 semantics of the decode call over a slot pool.

    Returns (out (B,Nv,S,Dv), new_pool (slots,Nv,Dk,Dv)); the input pool is
    not modified (a copy is updated).  See gdr_oracle.c for the two readings of
    num_accepted_tokens (per_token False: commit the first A states; True: the
    speculative-decoding reading, start from the slot of token A - 1 and commit
    every token's state to its own slot).
    """
    qa, ka, va, ba = _f64(q), _f64(k), _f64(v), _f64(beta)
    B, Nk, S, Dk = qa.shape
    Nv, Dv = va.shape[1], va.shape[3]
    ga, gka = _f64(g), _f64(gk)
    pool = np.array(state_pool, dtype=np.float64, copy=True, order="C")
    slots = pool.shape[0]
    idx, L = _i32(ssm_state_indices), _i32(actual_seq_lengths)
    A = _i32(num_accepted_tokens)
    out = np.empty((B, Nv, S, Dv), np.float64)
    rc = lib().gdr_oracle_recurrent_step(_dp(qa), _dp(ka), _dp(va), _dp(ba), _dp(ga), _dp(gka), _dp(pool), slots,
                                         _ip(idx), _ip(L), _ip(A), int(bool(per_token)), float(scale), B, Nk, Nv,
                                         S, Dk, Dv, _dp(out))
    if rc != 0:
        raise ValueError(f"oracle recurrent_step rejected the arguments (code {rc})")
    return out, pool


def gated_rmsnorm(o, z, norm_w, eps: float, actual_seq_lengths=None):
    """fp64 output epilogue of the layer: per head and token, the row o (length Dv) becomes

        o / sqrt(mean_j o_j^2 + eps) * w * silu(z),   silu(z) = z / (1 + e^{-z}),

    with one weight vector w (Dv) shared by all heads.  Rows t >= L_b (padding) are returned
    unchanged (the calls leave them zero).

    Source: the gated RMSNorm applied per head after the recurrence in deltanet.rs (mean of the
    squares over the head's Dv outputs, eps inside the square root, times norm_w and silu of the
    head's z slice) and the same arithmetic in the WGSL core shader of that crate; the blog
    "gated-delta-net" page applies it as self.norm(core_attn_out, z) on rows of length d_v.  Its
    comment names the gate sigmoid(z); both code listings use silu, which is the reading taken.

    o, z: (B, Nv, S, Dv); norm_w: (Dv,); actual_seq_lengths: (B,) or None (all S).
    """
    oa, za, wa = _f64(o), _f64(z), _f64(norm_w)
    if oa.shape != za.shape or wa.shape != (oa.shape[-1],):
        raise ValueError("o and z must have the same shape and norm_w the length of their last axis")
    B, S = oa.shape[0], oa.shape[2]
    L = np.full(B, S, np.int64) if actual_seq_lengths is None else np.asarray(actual_seq_lengths, np.int64)
    inv = 1.0 / np.sqrt(np.mean(oa * oa, axis=-1, keepdims=True) + float(eps))
    y = oa * inv * wa * (za / (1.0 + np.exp(-za)))
    t = np.arange(S)[None, None, :, None]
    return np.where(t < L[:, None, None, None], y, oa)


def causal_conv1d(x, weight, bias=None, conv_state=None, actual_seq_lengths=None):
    """fp64 depthwise causal convolution with SiLU over the fused q/k/v channels, and its state.

    For sequence b with L = L_b valid positions, channel c, taps w[c, 0..K-1] oldest first:

        y[t, c] = silu(bias[c] + sum_j w[c, j] * x[t - K + 1 + j, c]),   0 <= t < L,

    where the positions before 0 are the K inputs held in the state (newest last; zeros without one).
    The state afterwards holds the last K inputs of that history (the state followed by x[0..L-1]).
    Rows t >= L are zero.

    Source: the layer's conv over mixed_qkv = cat(q, k, v) with causal_conv1d_fn / causal_conv1d_update
    and conv_state = F.pad(mixed_qkv, (K - L, 0)) (blog "gated-delta-net" page), and deltanet.rs's
    per-channel ring of the last K inputs (shift, append, dot with the taps oldest first, silu) with its
    WGSL twin.

    x: (B, S, C) channels last; weight: (C, K); bias: (C,) or None; conv_state: (B, C, K) or None;
    actual_seq_lengths: (B,) or None (all S).  Returns (y (B, S, C), new_state (B, C, K)).
    """
    xa, wa = _f64(x), _f64(weight)
    B, S, C = xa.shape
    K = wa.shape[1]
    if wa.shape != (C, K):
        raise ValueError("weight must be (C, K)")
    ba = np.zeros(C) if bias is None else _f64(bias)
    st = np.zeros((B, C, K)) if conv_state is None else _f64(conv_state)
    L = np.full(B, S, np.int64) if actual_seq_lengths is None else np.asarray(actual_seq_lengths, np.int64)
    y = np.zeros((B, S, C))
    new = np.empty((B, C, K))
    for b in range(B):
        hist = np.concatenate([st[b].T, xa[b, :L[b]]], axis=0)  # (K + L, C): the K state inputs, then x
        for t in range(L[b]):
            acc = ba + np.sum(wa.T * hist[t + 1:t + 1 + K], axis=0)
            y[b, t] = acc / (1.0 + np.exp(-acc))
        new[b] = hist[L[b]:L[b] + K].T
    return y, new
