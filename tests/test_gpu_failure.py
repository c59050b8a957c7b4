"""Failure handling on the GPU without faulting it: the tensor-core prefill's bounded waits running out, and the
host-side checked mode (GDR_CHECKS=1) that rejects bad index and length arrays before anything is launched.

The recurrent_gated_delta_rule page (lite_boost) makes the slot map the caller's contract; the kernels skip a
sequence with a bad slot or length and flag the device error word, and two sequences sharing a slot would race.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, host, rnd, rnd32, unfused_inputs

pytestmark = pytest.mark.gpu


def _tiny_tc_case():
    w = workloads.random_case(B=1, Nk=1, Nv=2, S=130, Dk=128, Dv=128, seed=91)
    return w, unfused_inputs(w, "bf16")


def _call(w, ins, epi=None):
    return gdr.chunk_fwd(dev(ins["q"], "bf16"), dev(ins["k"], "bf16"), dev(ins["v"], "bf16"), dev(ins["beta"], "bf16"),
                         dev(ins["g"], "f32"), dev(ins["initial_state"], "bf16"), None, w.scale, epilogue=epi)


def test_bounded_wait_runs_out_and_the_next_call_is_clean():
    """With the wait limit cut to 1 ns every wait of the two-kernel schedule's chain kernel that is not already
    satisfied runs out: the kernel drains its own copies and MMAs, releases tensor memory, returns and sets
    GDR_DEVERR_TIMEOUT, and records which wait ran out.  The context stays usable: the next call with the default
    limit passes parity."""
    w, ins = _tiny_tc_case()
    assert gdr.get_error() == 0 and gdr.take_timeout_site() == {}
    gdr.set_chunk_schedule(gdr.SCHEDULE_TWO_KERNELS)
    gdr.set_wait_limit_ns(1)
    try:
        _call(w, ins)
        err = gdr.get_error()
        site = gdr.take_timeout_site()
    finally:
        gdr.set_wait_limit_ns(0)
        gdr.set_chunk_schedule(gdr.SCHEDULE_AUTO)
    assert err & gdr.DEVERR_TIMEOUT, err
    assert site and 0 <= site["warp"] < 20 and site["cta"] < w.B * w.Nv, site
    out, fin = _call(w, ins)
    assert gdr.get_error() == 0 and gdr.take_timeout_site() == {}
    ro, rf = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["initial_state"], None, w.scale)
    assert_close(host(out), ro, "bf16", "out")
    assert_close(host(fin), rf, "bf16", "final_state")


@pytest.mark.timeout(300)
@pytest.mark.parametrize("with_epilogue", [False, True])
def test_bounded_wait_runs_out_one_kernel_schedule(with_epilogue):
    """The same with the one-kernel schedule (the prefill workload's): with the limit at 1 ns its waits run out,
    each warp group stops at its next collective hand-off (bar.red.or, so no group splits at a named barrier),
    the issuers wait for their copies and MMAs in flight, and the call returns with GDR_DEVERR_TIMEOUT and the
    first site that ran out.  The next call with the default limit passes parity.  With the gated RMSNorm
    epilogue the helper warps that write its gate factors wait too."""
    w, ins = _tiny_tc_case()
    epi = zr = wr = None
    if with_epilogue:
        z, nw = workloads.epilogue_inputs(w)
        zr, wr = rnd(z, "bf16"), rnd32(nw)
        epi = gdr.Epilogue(z=dev(zr, "bf16"), norm_w=dev(wr, "f32"), eps=1e-6)
    assert gdr.get_error() == 0 and gdr.take_timeout_site() == {}
    gdr.set_chunk_schedule(gdr.SCHEDULE_ONE_KERNEL)
    try:
        gdr.set_wait_limit_ns(1)
        try:
            _call(w, ins, epi)
            err = gdr.get_error()
            site = gdr.take_timeout_site()
        finally:
            gdr.set_wait_limit_ns(0)
        assert err & gdr.DEVERR_TIMEOUT, err
        assert site and 0 <= site["warp"] < 20 and site["cta"] < w.B * w.Nv, site
        out, fin = _call(w, ins, epi)
        assert gdr.get_error() == 0 and gdr.take_timeout_site() == {}
    finally:
        gdr.set_chunk_schedule(gdr.SCHEDULE_AUTO)
    ro, rf = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["initial_state"], None, w.scale)
    if with_epilogue:
        ro = oracle.gated_rmsnorm(ro, zr, wr, 1e-6)
    assert_close(host(out), ro, "bf16", "out")
    assert_close(host(fin), rf, "bf16", "final_state")


def _decode_case(B=4, S=2, slots=12):
    w = workloads.random_case(B=B, Nk=1, Nv=2, S=S, Dk=128, Dv=128, seed=92, slots=slots, share_slot=True)
    ins = unfused_inputs(w, "bf16")
    return w, ins


def _decode(w, ins, idx, lengths, accepted=None, per_token=False):
    pool = dev(w.pool, "bf16")
    return gdr.recurrent_step(dev(ins["q"], "bf16"), dev(ins["k"], "bf16"), dev(ins["v"], "bf16"),
                              dev(ins["beta"], "bf16"), dev(ins["g"], "f32"), None, pool, dev_i32(idx),
                              dev_i32(lengths), dev_i32(accepted), w.scale, per_token=per_token)


def test_checked_mode_rejects_shared_slots_bad_slots_and_lengths(monkeypatch):
    w, ins = _decode_case()
    idx = np.repeat(np.array([0, 3, 5, 7], np.int32), w.S)
    L = np.full(w.B, w.S, np.int32)
    monkeypatch.setenv("GDR_CHECKS", "1")
    _decode(w, ins, idx, L)  # a valid call passes the checks
    assert gdr.get_error() == 0
    shared = idx.copy()
    shared[2 * w.S:3 * w.S] = 3  # sequence 2 commits to sequence 1's slot
    with pytest.raises(ValueError):
        _decode(w, ins, shared, L)
    out_of_range = idx.copy()
    out_of_range[0] = 12
    with pytest.raises(ValueError):
        _decode(w, ins, out_of_range, L)
    bad_len = L.copy()
    bad_len[1] = w.S + 1
    with pytest.raises(ValueError):
        _decode(w, ins, idx, bad_len)
    # speculative decoding: accepted counts must lie in [1, S]; per-token slots must not collide either
    pt = np.arange(w.B * w.S, dtype=np.int32)
    _decode(w, ins, pt, L, accepted=np.ones(w.B, np.int32), per_token=True)
    with pytest.raises(ValueError):
        _decode(w, ins, pt, L, accepted=np.zeros(w.B, np.int32), per_token=True)
    pt_shared = pt.copy()
    pt_shared[w.S] = pt[0]
    with pytest.raises(ValueError):
        _decode(w, ins, pt_shared, L, accepted=np.ones(w.B, np.int32), per_token=True)
    # prefill: lengths within [0, S]
    wc, ic = _tiny_tc_case()
    with pytest.raises(ValueError):
        gdr.chunk_fwd(dev(ic["q"], "bf16"), dev(ic["k"], "bf16"), dev(ic["v"], "bf16"), dev(ic["beta"], "bf16"),
                      dev(ic["g"], "f32"), None, dev_i32([wc.S + 1]), wc.S ** -0.5)
    assert gdr.get_error() == 0  # nothing was launched
    # without checked mode the same bad length reaches the kernel, which skips the sequence and flags it
    monkeypatch.delenv("GDR_CHECKS")
    gdr.chunk_fwd(dev(ic["q"], "bf16"), dev(ic["k"], "bf16"), dev(ic["v"], "bf16"), dev(ic["beta"], "bf16"),
                  dev(ic["g"], "f32"), None, dev_i32([wc.S + 1]), wc.S ** -0.5)
    assert gdr.get_error() & gdr.DEVERR_LENGTH
