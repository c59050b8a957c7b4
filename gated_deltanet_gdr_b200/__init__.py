"""B200 (sm_100a) gated delta rule: Python binding of libgdr.so.

The functions here only check and marshal arguments (torch tensors to device
pointers and sizes) and call the C ABI declared in ``include/gdr.h``; every
step of the computation runs in the library's CUDA kernels.  PyTorch supplies
device memory and streams.  If the compiled library is missing, importing the
binding's functions raises: there is no fallback.

    out, final_state = chunk_fwd(q, k, v, beta, g, initial_state, actual_seq_lengths, scale)
    out, state_pool  = recurrent_step(q, k, v, beta, g, gk, state_pool, ssm_state_indices,
                                      actual_seq_lengths, num_accepted_tokens, scale)

Layouts are BNSD: q, k (B, Nk, S, Dk); v (B, Nv, S, Dv); beta, g (B, Nv, S).
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr.so")

GDR_OK, GDR_ERR_SHAPE, GDR_ERR_DTYPE, GDR_ERR_NULL, GDR_ERR_ALIGN, GDR_ERR_UNSUPPORTED, GDR_ERR_DEVICE, \
    GDR_ERR_LAUNCH, GDR_ERR_WORKSPACE = range(9)
GDR_F32, GDR_BF16, GDR_F16 = 0, 1, 2
DEVERR_SLOT_INDEX, DEVERR_LENGTH, DEVERR_TIMEOUT = 0x1, 0x2, 0x4

# Every symbol the C header declares (checked by the ABI test).
EXPORTED = ("gdr_chunk_fwd_workspace", "gdr_chunk_fwd", "gdr_chunk_fwd_noalloc", "gdr_recurrent_step", "gdr_recurrent_step_spec", "gdr_conv1d",
            "gdr_prologue_apply", "gdr_get_error", "gdr_debug_set_wait_limit", "gdr_debug_timeout_site",
            "gdr_debug_set_chunk_schedule",
            "gdr_status_string", "gdr_version")


class GdrPrologueStruct(ctypes.Structure):
    _fields_ = [("l2norm_qk", ctypes.c_int), ("eps", ctypes.c_float), ("beta_logits", ctypes.c_int),
                ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p)]


class GdrEpilogueStruct(ctypes.Structure):
    _fields_ = [("z", ctypes.c_void_p), ("norm_w", ctypes.c_void_p), ("eps", ctypes.c_float)]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libgdr.so (built in-tree by ``python -m gated_deltanet_gdr_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdr.so is not built ({LIB_PATH} missing); run "
                               "`python -m gated_deltanet_gdr_b200.build` -- there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.gdr_chunk_fwd_workspace.restype = ctypes.c_size_t
        L.gdr_chunk_fwd_workspace.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        L.gdr_chunk_fwd.restype = i32
        L.gdr_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, i32, i32,
                                    ctypes.POINTER(GdrPrologueStruct), ctypes.POINTER(GdrEpilogueStruct), vp, vp, vp,
                                    ctypes.c_size_t, vp]
        L.gdr_chunk_fwd_noalloc.restype = i32
        L.gdr_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, i32, i32,
                                            ctypes.POINTER(GdrPrologueStruct), ctypes.POINTER(GdrEpilogueStruct),
                                            vp, vp, vp]
        L.gdr_recurrent_step.restype = i32
        L.gdr_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, f32, i32, i32, i32, i32, i32,
                                         i32, i32, i32, ctypes.POINTER(GdrPrologueStruct),
                                         ctypes.POINTER(GdrEpilogueStruct), vp, vp]
        L.gdr_recurrent_step_spec.restype = i32
        L.gdr_recurrent_step_spec.argtypes = L.gdr_recurrent_step.argtypes
        L.gdr_conv1d.restype = i32
        L.gdr_conv1d.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
        L.gdr_prologue_apply.restype = i32
        L.gdr_prologue_apply.argtypes = [vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                         vp]
        L.gdr_get_error.restype = i32
        L.gdr_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.gdr_debug_set_wait_limit.restype = i32
        L.gdr_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong]
        L.gdr_debug_timeout_site.restype = i32
        L.gdr_debug_timeout_site.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.gdr_debug_set_chunk_schedule.restype = i32
        L.gdr_debug_set_chunk_schedule.argtypes = [i32]
        L.gdr_status_string.restype = ctypes.c_char_p
        L.gdr_status_string.argtypes = [i32]
        L.gdr_version.restype = i32
        L.gdr_version.argtypes = []
        _lib = L
        return L


@dataclass
class Prologue:
    """Fused pre-processing (see ``gdr_prologue`` in include/gdr.h): l2norm of raw
    q/k with eps inside the sqrt, beta from logits, g from raw a via A_log/dt_bias."""
    l2norm_qk: bool = True
    eps: float = 1e-6
    beta_logits: bool = True
    A_log: Optional[torch.Tensor] = None
    dt_bias: Optional[torch.Tensor] = None

    def as_struct(self) -> GdrPrologueStruct:
        return GdrPrologueStruct(int(self.l2norm_qk), float(self.eps), int(self.beta_logits), _ptr(self.A_log),
                                 _ptr(self.dt_bias))


@dataclass
class Epilogue:
    """Fused output epilogue (see ``gdr_epilogue`` in include/gdr.h): each valid out row o
    becomes o / sqrt(mean(o^2) + eps) * norm_w * silu(z) (the layer's gated RMSNorm)."""
    z: torch.Tensor  # (B, Nv, S, Dv), the dtype of q
    norm_w: torch.Tensor  # (Dv,) fp32
    eps: float = 1e-6

    def as_struct(self) -> GdrEpilogueStruct:
        return GdrEpilogueStruct(_ptr(self.z), _ptr(self.norm_w), float(self.eps))


def _check_epilogue(epi, B, Nv, S, Dv, dt):
    if epi is None:
        return None
    _dev(epi.z, "epilogue.z", dt, (B, Nv, S, Dv))
    _dev(epi.norm_w, "epilogue.norm_w", torch.float32, (Dv,))
    return epi.as_struct()


def _check(status: int, what: str):
    if status == GDR_OK:
        return
    msg = f"{what}: {lib().gdr_status_string(status).decode()} (status {status})"
    if status == GDR_ERR_SHAPE:
        raise ValueError(msg)
    raise RuntimeError(msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return GDR_F32
    if dt == torch.bfloat16:
        return GDR_BF16
    if dt == torch.float16:
        return GDR_F16
    raise RuntimeError(f"unsupported dtype {dt}; use torch.float32, torch.bfloat16 or torch.float16")


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise RuntimeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise RuntimeError(f"{name} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:  # the kernels run on the current device and would read this pointer there
        raise RuntimeError(f"{name} is on {t.device}, but the call runs on the current device cuda:{cur}")
    if dtype is not None and t.dtype != dtype:
        raise RuntimeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise RuntimeError(f"{name} must be contiguous")
    return t


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    if s.device.index != torch.cuda.current_device():
        raise RuntimeError(f"the stream is on {s.device}, but the call runs on the current device "
                           f"cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(s.cuda_stream)


def _chunk_checked(q, k, v, beta, g, initial_state, actual_seq_lengths, prologue, out, final_state,
                   output_final_state):
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k must be (B, Nk, S, Dk) and v (B, Nv, S, Dv)")
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    dt = q.dtype
    _dtype_code(dt)
    _dev(q, "q", dt)
    _dev(k, "k", dt, (B, Nk, S, Dk))
    _dev(v, "v", dt, (B, Nv, S, Dv))
    _dev(beta, "beta", dt, (B, Nv, S))
    _dev(g, "g", torch.float32, (B, Nv, S))
    _dev(initial_state, "initial_state", dt, (B, Nv, Dk, Dv))
    _dev(actual_seq_lengths, "actual_seq_lengths", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, Nv, S, Dv), dtype=dt, device=q.device)
    _dev(out, "out", dt, (B, Nv, S, Dv))
    if output_final_state and final_state is None:
        final_state = torch.empty((B, Nv, Dk, Dv), dtype=dt, device=q.device)
    _dev(final_state, "final_state", dt, (B, Nv, Dk, Dv))
    if prologue is not None:
        _dev(prologue.A_log, "A_log", torch.float32, (Nv,))
        _dev(prologue.dt_bias, "dt_bias", torch.float32, (Nv,))
    return out, final_state


def chunk_fwd_workspace_bytes(B: int, Nk: int, Nv: int, S: int, Dk: int, Dv: int, dtype: torch.dtype) -> int:
    """Bytes of workspace the fastest schedule of ``gdr_chunk_fwd`` wants for these sizes
    (``gdr_chunk_fwd_workspace``; 0 when it wants none)."""
    return int(lib().gdr_chunk_fwd_workspace(B, Nk, Nv, S, Dk, Dv, _dtype_code(dtype)))


def _workspace(q, v, workspace):
    """The caller's workspace (a CUDA uint8 tensor), or a new one of the size the call needs."""
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    need = chunk_fwd_workspace_bytes(B, Nk, Nv, S, Dk, Dv, q.dtype)
    if workspace is None:
        return torch.empty(need, dtype=torch.uint8, device=q.device) if need else None
    _dev(workspace, "workspace", torch.uint8)
    if workspace.numel() < need:
        raise ValueError(f"workspace holds {workspace.numel()} bytes; the call needs {need}")
    return workspace


def chunk_fwd(q, k, v, beta, g=None, initial_state=None, actual_seq_lengths=None, scale: float = 1.0, *,
              prologue: Optional[Prologue] = None, epilogue: Optional[Epilogue] = None, out=None, final_state=None,
              output_final_state: bool = True, workspace=None, stream=None):
    """Chunked prefill (``gdr_chunk_fwd``).  Returns (out, final_state or None).  ``workspace`` (uint8, at least
    ``chunk_fwd_workspace_bytes`` bytes) is allocated per call when not given and the sizes ask for one."""
    out, final_state = _chunk_checked(q, k, v, beta, g, initial_state, actual_seq_lengths, prologue, out,
                                      final_state, output_final_state)
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    pro = prologue.as_struct() if prologue is not None else None
    epi = _check_epilogue(epilogue, B, Nv, S, Dv, q.dtype)
    ws = _workspace(q, v, workspace)
    st = lib().gdr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(initial_state),
                             _ptr(actual_seq_lengths), float(scale), B, Nk, Nv, S, Dk, Dv, _dtype_code(q.dtype),
                             ctypes.byref(pro) if pro is not None else None,
                             ctypes.byref(epi) if epi is not None else None, _ptr(out), _ptr(final_state),
                             _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "gdr_chunk_fwd")
    return out, final_state


def _decode_checked(q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths, num_accepted_tokens,
                    out):
    if q.dim() != 4 or v.dim() != 4 or state_pool.dim() != 4:
        raise ValueError("q, k (B, Nk, S, Dk), v (B, Nv, S, Dv), state_pool (slots, Nv, Dk, Dv)")
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    dt = q.dtype
    _dtype_code(dt)
    _dtype_code(state_pool.dtype)
    _dev(q, "q", dt)
    _dev(k, "k", dt, (B, Nk, S, Dk))
    _dev(v, "v", dt, (B, Nv, S, Dv))
    _dev(beta, "beta", dt, (B, Nv, S))
    _dev(g, "g", torch.float32, (B, Nv, S))
    _dev(gk, "gk", torch.float32, (B, Nv, S, Dk))
    _dev(state_pool, "state_pool", state_pool.dtype, (state_pool.shape[0], Nv, Dk, Dv))
    if ssm_state_indices is None or ssm_state_indices.numel() != B * S:
        raise ValueError("ssm_state_indices must hold B * S int32 slot indices, one per flattened token")
    _dev(ssm_state_indices.reshape(-1), "ssm_state_indices", torch.int32)
    _dev(actual_seq_lengths, "actual_seq_lengths", torch.int32, (B,))
    _dev(num_accepted_tokens, "num_accepted_tokens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, Nv, S, Dv), dtype=dt, device=q.device)
    _dev(out, "out", dt, (B, Nv, S, Dv))
    return out


def recurrent_step(q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths,
                   num_accepted_tokens=None, scale: float = 1.0, *, prologue: Optional[Prologue] = None,
                   epilogue: Optional[Epilogue] = None, out=None, per_token: bool = False, stream=None):
    """Recurrent decode over a slot pool (``gdr_recurrent_step``), updating
    ``state_pool`` in place.  Returns (out, state_pool).  ``per_token=True`` calls
    ``gdr_recurrent_step_spec`` (speculative decoding: start from the slot of token
    A - 1, every token's state to its own slot)."""
    out = _decode_checked(q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths,
                          num_accepted_tokens, out)
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    pro = prologue.as_struct() if prologue is not None else None
    epi = _check_epilogue(epilogue, B, Nv, S, Dv, q.dtype)
    fn = lib().gdr_recurrent_step_spec if per_token else lib().gdr_recurrent_step
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(gk), _ptr(state_pool),
                                  int(state_pool.shape[0]), _ptr(ssm_state_indices), _ptr(actual_seq_lengths),
                                  _ptr(num_accepted_tokens), float(scale), B, Nk, Nv, S, Dk, Dv,
                                  _dtype_code(q.dtype), _dtype_code(state_pool.dtype),
                                  ctypes.byref(pro) if pro is not None else None,
                                  ctypes.byref(epi) if epi is not None else None, _ptr(out), _stream(stream))
    _check(st, "gdr_recurrent_step_spec" if per_token else "gdr_recurrent_step")
    return out, state_pool


class PreparedCall:
    """A C-ABI call with its arguments checked and marshalled once.

    Calling the object launches the library's kernels again on the same buffers
    (which the caller keeps alive and may refill in place) with no Python-side
    argument work, for serving loops and for timing the kernels alone.  Raises
    like the one-shot functions if the library reports an error.
    """

    def __init__(self, fn, args, what, result):
        self._fn, self._args, self._what, self.result = fn, args, what, result

    def __call__(self):
        st = self._fn(*self._args)
        if st != GDR_OK:
            _check(st, self._what)
        return self.result


def prepare_chunk_fwd(q, k, v, beta, g=None, initial_state=None, actual_seq_lengths=None, scale: float = 1.0, *,
                      prologue: Optional[Prologue] = None, epilogue: Optional[Epilogue] = None, out=None,
                      final_state=None, workspace=None, stream=None) -> PreparedCall:
    """Check and marshal a gdr_chunk_fwd call once; see chunk_fwd for the arguments (the workspace, if not given,
    is allocated once here and kept by the prepared call)."""
    out, final_state = _chunk_checked(q, k, v, beta, g, initial_state, actual_seq_lengths, prologue, out,
                                      final_state, True)
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    pro = prologue.as_struct() if prologue is not None else None
    epi = _check_epilogue(epilogue, B, Nv, S, Dv, q.dtype)
    ws = _workspace(q, v, workspace)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(initial_state), _ptr(actual_seq_lengths),
            ctypes.c_float(scale), B, Nk, Nv, S, Dk, Dv, _dtype_code(q.dtype),
            ctypes.pointer(pro) if pro is not None else None, ctypes.pointer(epi) if epi is not None else None,
            _ptr(out), _ptr(final_state), _ptr(ws), ctypes.c_size_t(0 if ws is None else ws.numel()),
            _stream(stream))
    call = PreparedCall(lib().gdr_chunk_fwd, args, "gdr_chunk_fwd", (out, final_state))
    call._keep = (pro, prologue, epi, epilogue, ws)
    return call


def prepare_recurrent_step(q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths,
                           num_accepted_tokens=None, scale: float = 1.0, *, prologue: Optional[Prologue] = None,
                           epilogue: Optional[Epilogue] = None, out=None, per_token: bool = False,
                           stream=None) -> PreparedCall:
    """Check and marshal a gdr_recurrent_step call once; see recurrent_step for the arguments."""
    out = _decode_checked(q, k, v, beta, g, gk, state_pool, ssm_state_indices, actual_seq_lengths,
                          num_accepted_tokens, out)
    B, Nk, S, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[3]
    pro = prologue.as_struct() if prologue is not None else None
    epi = _check_epilogue(epilogue, B, Nv, S, Dv, q.dtype)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(gk), _ptr(state_pool), int(state_pool.shape[0]),
            _ptr(ssm_state_indices), _ptr(actual_seq_lengths), _ptr(num_accepted_tokens), ctypes.c_float(scale), B,
            Nk, Nv, S, Dk, Dv, _dtype_code(q.dtype), _dtype_code(state_pool.dtype),
            ctypes.pointer(pro) if pro is not None else None, ctypes.pointer(epi) if epi is not None else None,
            _ptr(out), _stream(stream))
    name = "gdr_recurrent_step_spec" if per_token else "gdr_recurrent_step"
    call = PreparedCall(getattr(lib(), name), args, name, (out, state_pool))
    call._keep = (pro, prologue, epi, epilogue)
    return call


def _conv1d_checked(x, weight, bias, conv_state, actual_seq_lengths, Nk, Nv, Dk, Dv, q, k, v, conv_state_out,
                    output_state, stream):
    if x.dim() != 3 or weight.dim() != 2:
        raise ValueError("x must be (B, S, C) and weight (C, K)")
    B, S, C = x.shape
    K = weight.shape[1]
    if C != 2 * Nk * Dk + Nv * Dv:
        raise ValueError(f"x has {C} channels; 2 * Nk * Dk + Nv * Dv = {2 * Nk * Dk + Nv * Dv}")
    dt = x.dtype
    code = _dtype_code(dt)
    _dev(x, "x", dt)
    _dev(weight, "weight", dt, (C, K))
    _dev(bias, "bias", dt, (C,))
    _dev(conv_state, "conv_state", dt, (B, C, K))
    _dev(actual_seq_lengths, "actual_seq_lengths", torch.int32, (B,))
    outs = []
    for name, t, shape in (("q", q, (B, Nk, S, Dk)), ("k", k, (B, Nk, S, Dk)), ("v", v, (B, Nv, S, Dv))):
        t = torch.empty(shape, dtype=dt, device=x.device) if t is None else t
        outs.append(_dev(t, name, dt, shape))
    if output_state and conv_state_out is None:
        conv_state_out = torch.empty((B, C, K), dtype=dt, device=x.device)
    _dev(conv_state_out, "conv_state_out", dt, (B, C, K))
    args = (_ptr(x), _ptr(weight), _ptr(bias), _ptr(conv_state), _ptr(actual_seq_lengths), B, S, Nk, Nv, Dk, Dv, K,
            code, _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), _ptr(conv_state_out), _stream(stream))
    return args, (outs[0], outs[1], outs[2], conv_state_out)


def conv1d(x, weight, bias=None, conv_state=None, actual_seq_lengths=None, *, Nk: int, Nv: int, Dk: int, Dv: int,
           q=None, k=None, v=None, conv_state_out=None, output_state: bool = True, stream=None):
    """Depthwise causal conv1d + SiLU over the fused q/k/v channels (``gdr_conv1d``).

    x (B, S, C) channels last with C = 2 * Nk * Dk + Nv * Dv, weight (C, K) taps oldest first, bias (C,) or
    None, conv_state (B, C, K) or None (zeros).  Returns (q (B, Nk, S, Dk), k, v (B, Nv, S, Dv), new state
    (B, C, K) or None).  Pass ``conv_state_out=conv_state`` to update the state in place (decode)."""
    args, res = _conv1d_checked(x, weight, bias, conv_state, actual_seq_lengths, Nk, Nv, Dk, Dv, q, k, v,
                                conv_state_out, output_state, stream)
    _check(lib().gdr_conv1d(*args), "gdr_conv1d")
    return res


def prepare_conv1d(x, weight, bias=None, conv_state=None, actual_seq_lengths=None, *, Nk: int, Nv: int, Dk: int,
                   Dv: int, q=None, k=None, v=None, conv_state_out=None, output_state: bool = True,
                   stream=None) -> "PreparedCall":
    """Check and marshal a gdr_conv1d call once; see conv1d for the arguments."""
    args, res = _conv1d_checked(x, weight, bias, conv_state, actual_seq_lengths, Nk, Nv, Dk, Dv, q, k, v,
                                conv_state_out, output_state, stream)
    return PreparedCall(lib().gdr_conv1d, args, "gdr_conv1d", res)


def prologue(q=None, k=None, b=None, a=None, A_log=None, dt_bias=None, eps: float = 1e-6, *, stream=None):
    """Stand-alone prologue (``gdr_prologue_apply``): returns a dict with q_hat,
    k_hat (l2norm, eps inside the sqrt), beta = sigmoid(b) and
    g = -exp(A_log) * softplus(a + dt_bias) for whichever inputs are given."""
    ref = next(t for t in (q, k, b) if t is not None) if any(t is not None for t in (q, k, b)) else None
    dt = ref.dtype if ref is not None else torch.float32
    code = _dtype_code(dt)
    if q is not None or k is not None:
        B, Nk, S, Dk = (q if q is not None else k).shape
    else:
        B, Nk, S, Dk = (b if b is not None else a).shape[0], 1, (b if b is not None else a).shape[2], 16
    Nv = (b if b is not None else a).shape[1] if (b is not None or a is not None) else Nk
    res = {}
    for name, t in (("q", q), ("k", k)):
        if t is not None:
            _dev(t, name, dt, (B, Nk, S, Dk))
            res[name + "_hat"] = torch.empty_like(t)
    if b is not None:
        _dev(b, "b", dt, (B, Nv, S))
        res["beta"] = torch.empty_like(b)
    if a is not None:
        _dev(a, "a", torch.float32, (B, Nv, S))
        _dev(A_log, "A_log", torch.float32, (Nv,))
        _dev(dt_bias, "dt_bias", torch.float32, (Nv,))
        res["g"] = torch.empty_like(a)
    st = lib().gdr_prologue_apply(_ptr(q), _ptr(k), _ptr(b), _ptr(a), _ptr(A_log), _ptr(dt_bias), float(eps), B, Nk,
                                  Nv, S, Dk, code, _ptr(res.get("q_hat")), _ptr(res.get("k_hat")),
                                  _ptr(res.get("beta")), _ptr(res.get("g")), _stream(stream))
    _check(st, "gdr_prologue_apply")
    return res


def get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    v = ctypes.c_int(0)
    _check(lib().gdr_get_error(_stream(stream), ctypes.byref(v)), "gdr_get_error")
    return v.value


def version() -> int:
    return int(lib().gdr_version())


def take_timeout_site() -> dict:
    """Diagnostic: the first bounded wait of the tensor-core prefill that ran out since the last read (cleared by
    the read), as {"warp", "barrier", "parity", "cta"}, or {} if none."""
    v = ctypes.c_uint(0)
    _check(lib().gdr_debug_timeout_site(ctypes.byref(v)), "gdr_debug_timeout_site")
    x = v.value
    if not x:
        return {}
    return {"warp": (x >> 24) & 0x3F, "barrier": (x >> 16) & 0xFF, "parity": (x >> 15) & 1, "cta": x & 0x7FFF}


# schedules of the tensor-core prefill for ``set_chunk_schedule``
SCHEDULE_AUTO, SCHEDULE_ONE_KERNEL, SCHEDULE_TWO_KERNELS = 0, 1, 2


def set_chunk_schedule(schedule: int) -> None:
    """Diagnostic: which schedule of the tensor-core prefill the workspace query sizes for later calls
    (``gdr_debug_set_chunk_schedule``): SCHEDULE_AUTO by shape, or one of the two always."""
    _check(lib().gdr_debug_set_chunk_schedule(int(schedule)), "gdr_debug_set_chunk_schedule")


def set_wait_limit_ns(ns: int) -> None:
    """Diagnostic: the limit of the tensor-core prefill's bounded waits for later calls (0: the default, 1 s)."""
    _check(lib().gdr_debug_set_wait_limit(int(ns)), "gdr_debug_set_wait_limit")
