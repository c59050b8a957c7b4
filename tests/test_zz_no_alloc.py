"""gdr_chunk_fwd_noalloc, the prefill entry point for callers that cannot allocate device memory.

Code that only receives one operation's tensors (a framework hook or plug-in), or whose device memory is all
reserved by its own pool, cannot allocate the workspace gdr_chunk_fwd asks for.  This entry point uses a fixed
scratch array compiled into the library instead.  The test calls it through the C ABI twice in a row (the array
keeps the first call's contents) and compares each result with gdr_chunk_fwd's, within the bf16 tolerance of the
other tests; it also checks that a size beyond the array is refused before anything runs.  It lives in a file of
its own that collects last, and needs nothing from the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import workloads
from tests._helpers import BF16_REL_L2, dev, dev_i32, host, rel_l2, unfused_inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(L, t, lens, w, out, fin):
    return L.gdr_chunk_fwd_noalloc(_p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["beta"]), _p(t["g"]), _p(t["s0"]),
                                   _p(lens), ctypes.c_float(w.scale), w.B, w.Nk, w.Nv, w.S, w.Dk, w.Dv, gdr.GDR_BF16,
                                   None, None, _p(out), _p(fin), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_the_workspace_entry_point_on_two_calls():
    L = gdr.lib()
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=200, Dk=128, Dv=128, seed=500, lengths=[200, 131])
    ins = unfused_inputs(w, "bf16")
    t = dict(q=dev(ins["q"], "bf16"), k=dev(ins["k"], "bf16"), v=dev(ins["v"], "bf16"),
             beta=dev(ins["beta"], "bf16"), g=dev(ins["g"], "f32"), s0=dev(ins["initial_state"], "bf16"))
    lens = dev_i32(w.lengths)
    ref_out, ref_fin = gdr.chunk_fwd(t["q"], t["k"], t["v"], t["beta"], t["g"], t["s0"], lens, w.scale)
    assert gdr.get_error() == 0
    ro, rf = host(ref_out), host(ref_fin)
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        fin = torch.full_like(ref_fin, float("nan"))
        assert _noalloc(L, t, lens, w, out, fin) == gdr.GDR_OK
        torch.cuda.synchronize()
        assert gdr.get_error() == 0
        go, gf = host(out), host(fin)
        assert np.all(np.isfinite(go)) and np.all(np.isfinite(gf))
        assert rel_l2(go, ro) <= BF16_REL_L2 and rel_l2(gf, rf) <= BF16_REL_L2
        for b in range(w.B):
            assert np.all(go[b, :, int(w.lengths[b]):] == 0.0)


def test_noalloc_with_the_one_kernel_schedule():
    """Sizes whose workspace query is 0 (here forced to the one-kernel schedule) run without touching the array;
    the result is the same call's through gdr_chunk_fwd."""
    L = gdr.lib()
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=130, Dk=128, Dv=128, seed=501, lengths=[130, 64])
    ins = unfused_inputs(w, "bf16")
    t = dict(q=dev(ins["q"], "bf16"), k=dev(ins["k"], "bf16"), v=dev(ins["v"], "bf16"),
             beta=dev(ins["beta"], "bf16"), g=dev(ins["g"], "f32"), s0=dev(ins["initial_state"], "bf16"))
    lens = dev_i32(w.lengths)
    gdr.set_chunk_schedule(gdr.SCHEDULE_ONE_KERNEL)
    try:
        assert gdr.chunk_fwd_workspace_bytes(w.B, w.Nk, w.Nv, w.S, w.Dk, w.Dv, torch.bfloat16) == 0
        ref_out, ref_fin = gdr.chunk_fwd(t["q"], t["k"], t["v"], t["beta"], t["g"], t["s0"], lens, w.scale)
        out = torch.full_like(ref_out, float("nan"))
        fin = torch.full_like(ref_fin, float("nan"))
        assert _noalloc(L, t, lens, w, out, fin) == gdr.GDR_OK
        torch.cuda.synchronize()
    finally:
        gdr.set_chunk_schedule(gdr.SCHEDULE_AUTO)
    assert gdr.get_error() == 0
    go, gf = host(out), host(fin)
    assert rel_l2(go, host(ref_out)) <= BF16_REL_L2 and rel_l2(gf, host(ref_fin)) <= BF16_REL_L2
    for b in range(w.B):
        assert np.all(go[b, :, int(w.lengths[b]):] == 0.0)


def test_noalloc_refuses_a_size_beyond_its_array():
    """B * Nv * ceil(S / 64) > 1724 needs more than the 16 MiB array: GDR_ERR_WORKSPACE, nothing launched."""
    L = gdr.lib()
    P = ctypes.c_void_p(4096)  # never dereferenced: the call is refused before any launch
    st = L.gdr_chunk_fwd_noalloc(P, P, P, P, None, None, None, ctypes.c_float(1.0), 1, 16, 32, 64 * 54, 128, 128,
                                 gdr.GDR_BF16, None, None, P, None, None)
    assert st == gdr.GDR_ERR_WORKSPACE
