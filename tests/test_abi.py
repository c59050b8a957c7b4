"""The C ABI library: it builds, loads without a GPU, exports what the header
declares, and rejects bad arguments on the host before launching anything.

Every call below that passes placeholder pointers is built so that host-side
validation must reject it; none can reach a kernel launch.
"""
import ctypes
import os
import re

import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
from gated_deltanet_gdr_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdr.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(gdr.EXPORTED), names
    for n in names:
        assert hasattr(L, n), f"libgdr.so does not export {n}"


def test_header_codes_match_the_binding():
    """The status codes, dtype codes and device error bits the header defines are the values the Python
    binding uses."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    enums = dict((n, int(v)) for n, v in re.findall(r"\b(GDR_[A-Z0-9_]+)\s*=\s*(\d+)", src))
    defines = dict((n, int(v, 16)) for n, v in re.findall(r"#define\s+(GDR_DEVERR_[A-Z_]+)\s+(0x[0-9a-fA-F]+)u", src))
    for name in ("GDR_OK", "GDR_ERR_SHAPE", "GDR_ERR_DTYPE", "GDR_ERR_NULL", "GDR_ERR_ALIGN", "GDR_ERR_UNSUPPORTED",
                 "GDR_ERR_DEVICE", "GDR_ERR_LAUNCH", "GDR_ERR_WORKSPACE", "GDR_F32", "GDR_BF16", "GDR_F16"):
        assert enums[name] == getattr(gdr, name), name
    assert defines == {"GDR_DEVERR_SLOT_INDEX": gdr.DEVERR_SLOT_INDEX, "GDR_DEVERR_LENGTH": gdr.DEVERR_LENGTH,
                       "GDR_DEVERR_TIMEOUT": gdr.DEVERR_TIMEOUT}, defines


def test_status_strings_and_version(L):
    for s in range(9):
        assert L.gdr_status_string(s) and b"unknown" not in L.gdr_status_string(s)
    assert b"unknown" in L.gdr_status_string(99)
    assert gdr.version() == 200


P = ctypes.c_void_p(4096)  # placeholder: aligned, non-NULL, never dereferenced (every call is rejected first)
NUL = None


def chunk(L, **kw):
    a = dict(q=P, k=P, v=P, beta=P, g=NUL, s0=NUL, lens=NUL, scale=1.0, B=1, Nk=2, Nv=4, S=8, Dk=128, Dv=128,
             dt=gdr.GDR_BF16, pro=None, epi=None, out=P, fin=NUL, ws=P, ws_bytes=1 << 40)
    a.update(kw)
    return L.gdr_chunk_fwd(a["q"], a["k"], a["v"], a["beta"], a["g"], a["s0"], a["lens"], a["scale"], a["B"],
                           a["Nk"], a["Nv"], a["S"], a["Dk"], a["Dv"], a["dt"], a["pro"], a["epi"], a["out"], a["fin"],
                           a["ws"], a["ws_bytes"], None)


def decode(L, **kw):
    a = dict(q=P, k=P, v=P, beta=P, g=NUL, gk=NUL, pool=P, slots=4, idx=P, lens=P, acc=NUL, scale=1.0, B=1, Nk=2,
             Nv=4, S=1, Dk=128, Dv=128, dt=gdr.GDR_BF16, sdt=gdr.GDR_BF16, pro=None, epi=None, out=P)
    a.update(kw)
    return L.gdr_recurrent_step(a["q"], a["k"], a["v"], a["beta"], a["g"], a["gk"], a["pool"], a["slots"], a["idx"],
                                a["lens"], a["acc"], a["scale"], a["B"], a["Nk"], a["Nv"], a["S"], a["Dk"], a["Dv"],
                                a["dt"], a["sdt"], a["pro"], a["epi"], a["out"], None)


def test_chunk_host_validation(L):
    assert chunk(L, Nv=3) == gdr.GDR_ERR_SHAPE  # Nv % Nk != 0
    assert chunk(L, Nk=0) == gdr.GDR_ERR_SHAPE
    assert chunk(L, B=-1) == gdr.GDR_ERR_SHAPE
    assert chunk(L, S=-5) == gdr.GDR_ERR_SHAPE
    assert chunk(L, dt=7) == gdr.GDR_ERR_DTYPE
    assert chunk(L, Dk=96) == gdr.GDR_ERR_UNSUPPORTED
    assert chunk(L, Dv=256) == gdr.GDR_ERR_UNSUPPORTED
    assert chunk(L, q=NUL) == gdr.GDR_ERR_NULL
    assert chunk(L, out=NUL) == gdr.GDR_ERR_NULL
    assert chunk(L, v=ctypes.c_void_p(4104)) == gdr.GDR_ERR_ALIGN
    assert chunk(L, fin=ctypes.c_void_p(4097)) == gdr.GDR_ERR_ALIGN
    pro = gdr.GdrPrologueStruct(1, 1e-6, 1, 4096, None)  # A_log without dt_bias
    assert chunk(L, pro=ctypes.byref(pro), g=P) == gdr.GDR_ERR_NULL
    pro = gdr.GdrPrologueStruct(1, 1e-6, 1, 4096, 8192)  # A_log without the raw a (g buffer)
    assert chunk(L, pro=ctypes.byref(pro)) == gdr.GDR_ERR_NULL
    pro = gdr.GdrPrologueStruct(1, -1.0, 0, None, None)  # negative eps
    assert chunk(L, pro=ctypes.byref(pro)) == gdr.GDR_ERR_SHAPE
    epi = gdr.GdrEpilogueStruct(4096, None, 1e-6)  # epilogue without norm_w
    assert chunk(L, epi=ctypes.byref(epi)) == gdr.GDR_ERR_NULL
    epi = gdr.GdrEpilogueStruct(None, 4096, 1e-6)  # epilogue without z
    assert chunk(L, epi=ctypes.byref(epi)) == gdr.GDR_ERR_NULL
    epi = gdr.GdrEpilogueStruct(4096, 4096, -1.0)  # negative eps
    assert chunk(L, epi=ctypes.byref(epi)) == gdr.GDR_ERR_SHAPE
    epi = gdr.GdrEpilogueStruct(4104, 4096, 1e-6)  # misaligned z
    assert chunk(L, epi=ctypes.byref(epi)) == gdr.GDR_ERR_ALIGN
    # the two-kernel schedule's workspace, when given: large enough and aligned (a NULL workspace is valid: the
    # one-kernel schedule runs, so it is not called here, where every call must be refused before a launch)
    need = L.gdr_chunk_fwd_workspace(1, 2, 4, 8, 128, 128, gdr.GDR_BF16)
    assert need > 0
    assert chunk(L, ws_bytes=need - 1) == gdr.GDR_ERR_WORKSPACE
    assert chunk(L, ws=ctypes.c_void_p(4104)) == gdr.GDR_ERR_ALIGN
    # nothing to do: B == 0 returns OK without touching a device
    assert chunk(L, B=0, q=NUL, k=NUL, v=NUL, beta=NUL, out=NUL, ws=NUL, ws_bytes=0) == gdr.GDR_OK


def test_workspace_size(L):
    """The two-kernel schedule's workspace: per (b, value head, 64-token chunk) the 64 x 64 16-bit T' and six
    vectors of 64 floats; asked for when B * Nv * 3 <= the SM count (148 where no device answers), else 0 (the
    one-kernel schedule needs none); zero for the CUDA-core path and for invalid sizes.  The schedule override
    moves the answer both ways."""
    per = 64 * 64 * 2 + 6 * 64 * 4
    assert L.gdr_chunk_fwd_workspace(1, 16, 32, 4096, 128, 128, gdr.GDR_BF16) == 32 * 64 * per  # 32 chains
    assert L.gdr_chunk_fwd_workspace(4, 16, 32, 4096, 128, 128, gdr.GDR_BF16) == 0  # 128 chains: one kernel
    assert L.gdr_chunk_fwd_workspace(1, 7, 49, 64, 128, 128, gdr.GDR_BF16) == 49 * per  # 147 <= 148
    assert L.gdr_chunk_fwd_workspace(2, 5, 25, 64, 128, 128, gdr.GDR_BF16) == 0  # 150 > 148
    assert L.gdr_chunk_fwd_workspace(2, 1, 3, 65, 128, 128, gdr.GDR_F16) == 2 * 3 * 2 * per
    assert L.gdr_chunk_fwd_workspace(2, 1, 3, 65, 128, 128, gdr.GDR_F32) == 0
    assert L.gdr_chunk_fwd_workspace(2, 1, 3, 65, 64, 64, gdr.GDR_BF16) == 0
    assert L.gdr_chunk_fwd_workspace(0, 1, 3, 65, 128, 128, gdr.GDR_BF16) == 0
    assert L.gdr_chunk_fwd_workspace(2, 2, 3, 65, 128, 128, gdr.GDR_BF16) == 0  # Nv % Nk != 0
    try:
        assert L.gdr_debug_set_chunk_schedule(2) == gdr.GDR_OK
        assert L.gdr_chunk_fwd_workspace(4, 16, 32, 4096, 128, 128, gdr.GDR_BF16) == 4 * 32 * 64 * per
        assert L.gdr_chunk_fwd_workspace(2, 1, 3, 65, 128, 128, gdr.GDR_F32) == 0
        assert L.gdr_debug_set_chunk_schedule(1) == gdr.GDR_OK
        assert L.gdr_chunk_fwd_workspace(1, 16, 32, 4096, 128, 128, gdr.GDR_BF16) == 0
        assert L.gdr_debug_set_chunk_schedule(3) == gdr.GDR_ERR_SHAPE
    finally:
        L.gdr_debug_set_chunk_schedule(0)


def test_decode_host_validation(L):
    assert decode(L, S=9) == gdr.GDR_ERR_SHAPE  # decode-only operator: S <= 8
    assert decode(L, S=0) == gdr.GDR_ERR_SHAPE
    assert decode(L, slots=0) == gdr.GDR_ERR_SHAPE
    assert decode(L, Nv=6, Nk=4) == gdr.GDR_ERR_SHAPE
    assert decode(L, sdt=3) == gdr.GDR_ERR_DTYPE
    assert decode(L, pool=NUL) == gdr.GDR_ERR_NULL
    assert decode(L, idx=NUL) == gdr.GDR_ERR_NULL
    assert decode(L, lens=NUL) == gdr.GDR_ERR_NULL
    # the pool's (slot, head) tiles are addressed in 32-bit arithmetic
    assert decode(L, slots=(1 << 31) // 4, Nv=4, Nk=2) == gdr.GDR_ERR_SHAPE
    assert decode(L, slots=(1 << 31) // 4 - 1, Nv=4, Nk=2, pool=NUL) == gdr.GDR_ERR_NULL
    assert decode(L, gk=ctypes.c_void_p(4100)) == gdr.GDR_ERR_ALIGN
    assert decode(L, Dk=48) == gdr.GDR_ERR_UNSUPPORTED
    assert decode(L, dt=gdr.GDR_F16, sdt=gdr.GDR_BF16) == gdr.GDR_ERR_DTYPE  # fp16 inputs: fp16 or fp32 state
    assert decode(L, dt=gdr.GDR_BF16, sdt=gdr.GDR_F16) == gdr.GDR_ERR_DTYPE  # an fp16 state needs fp16 inputs
    epi = gdr.GdrEpilogueStruct(4096, None, 1e-6)
    assert decode(L, epi=ctypes.byref(epi)) == gdr.GDR_ERR_NULL
    epi = gdr.GdrEpilogueStruct(4096, 4096, float("nan"))
    assert decode(L, epi=ctypes.byref(epi)) == gdr.GDR_ERR_SHAPE
    assert decode(L, B=0) == gdr.GDR_OK


def conv(L, **kw):
    a = dict(x=P, w=P, bias=NUL, s0=NUL, lens=NUL, B=1, S=8, Nk=2, Nv=4, Dk=128, Dv=128, K=4, dt=gdr.GDR_BF16,
             q=P, k=P, v=P, s1=NUL)
    a.update(kw)
    return L.gdr_conv1d(a["x"], a["w"], a["bias"], a["s0"], a["lens"], a["B"], a["S"], a["Nk"], a["Nv"], a["Dk"],
                        a["Dv"], a["K"], a["dt"], a["q"], a["k"], a["v"], a["s1"], None)


def test_conv1d_host_validation(L):
    assert conv(L, K=0) == gdr.GDR_ERR_SHAPE
    assert conv(L, K=9) == gdr.GDR_ERR_SHAPE
    assert conv(L, Nv=3) == gdr.GDR_ERR_SHAPE
    assert conv(L, B=70000) == gdr.GDR_ERR_SHAPE  # grid z limit
    assert conv(L, dt=4) == gdr.GDR_ERR_DTYPE
    assert conv(L, Dv=48) == gdr.GDR_ERR_UNSUPPORTED
    assert conv(L, x=NUL) == gdr.GDR_ERR_NULL
    assert conv(L, v=NUL) == gdr.GDR_ERR_NULL
    assert conv(L, S=0, w=NUL, s1=P) == gdr.GDR_ERR_NULL  # a state update needs the taps' shape
    assert conv(L, bias=ctypes.c_void_p(4098)) == gdr.GDR_ERR_ALIGN
    assert conv(L, B=0) == gdr.GDR_OK
    assert conv(L, S=0, x=NUL, q=NUL, k=NUL, v=NUL) == gdr.GDR_OK  # nothing to compute, no state asked for


def test_prologue_host_validation(L):
    f = L.gdr_prologue_apply
    assert f(P, NUL, NUL, NUL, NUL, NUL, 1e-6, 1, 1, 1, 4, 16, 5, P, NUL, NUL, NUL, None) == gdr.GDR_ERR_DTYPE
    assert f(P, NUL, NUL, NUL, NUL, NUL, 1e-6, 1, 1, 1, 4, 16, 0, NUL, NUL, NUL, NUL, None) == gdr.GDR_ERR_NULL
    assert f(NUL, NUL, NUL, P, NUL, P, 1e-6, 1, 1, 1, 4, 16, 0, NUL, NUL, NUL, P, None) == gdr.GDR_ERR_NULL
    assert f(P, NUL, NUL, NUL, NUL, NUL, -1.0, 1, 1, 1, 4, 16, 0, P, NUL, NUL, NUL, None) == gdr.GDR_ERR_SHAPE
    assert f(NUL, NUL, NUL, NUL, NUL, NUL, 1e-6, 1, 1, 1, 4, 16, 0, NUL, NUL, NUL, NUL, None) == gdr.GDR_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device status; on a GPU host the "
                    "placeholder pointers would be launched on")
def test_no_device_status(L):
    assert chunk(L) == gdr.GDR_ERR_DEVICE
    v = ctypes.c_int(5)
    assert L.gdr_get_error(None, ctypes.byref(v)) == gdr.GDR_ERR_DEVICE
    assert v.value == 0


def test_binding_rejects_host_tensors_and_bad_dtypes():
    q = torch.zeros(1, 1, 4, 16)
    with pytest.raises(RuntimeError):
        gdr.chunk_fwd(q, q, q, torch.zeros(1, 1, 4))
    assert gdr._dtype_code(torch.float16) == gdr.GDR_F16
    with pytest.raises(RuntimeError):
        gdr._dtype_code(torch.float64)
    with pytest.raises(ValueError):
        gdr.chunk_fwd(torch.zeros(4, 16), q, q, q)
