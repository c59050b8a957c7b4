"""Decode (gdr_recurrent_step) on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import (assert_close, dev, dev_i32, fused_inputs, host, rnd, rnd32, unfused_inputs)

pytestmark = pytest.mark.gpu


def run_decode(w, dt, state_dt=None, fused=False):
    """Returns (gpu_out, gpu_pool, ref_out, ref_pool, pool0) as fp64 numpy."""
    state_dt = state_dt or dt
    pool0 = rnd(w.pool, state_dt)
    if fused:
        raw, ref = fused_inputs(w, dt)
        pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True,
                           A_log=dev(raw.get("A_log"), "f32"), dt_bias=dev(raw.get("dt_bias"), "f32"))
        gin = dict(q=dev(raw["q"], dt), k=dev(raw["k"], dt), v=dev(raw["v"], dt), beta=dev(raw["b"], dt),
                   g=dev(raw["a"] if raw.get("a") is not None else raw["g"], "f32"), gk=dev(raw["gk"], "f32"))
    else:
        ref = unfused_inputs(w, dt)
        pro = None
        gin = dict(q=dev(ref["q"], dt), k=dev(ref["k"], dt), v=dev(ref["v"], dt), beta=dev(ref["beta"], dt),
                   g=dev(ref["g"], "f32"), gk=dev(ref["gk"], "f32"))
    pool = dev(pool0, state_dt)
    out, pool = gdr.recurrent_step(gin["q"], gin["k"], gin["v"], gin["beta"], gin["g"], gin["gk"], pool,
                                   dev_i32(w.indices), dev_i32(w.lengths), dev_i32(w.accepted), w.scale,
                                   prologue=pro)
    assert gdr.get_error() == 0
    ro, rp = oracle.recurrent_step(ref["q"], ref["k"], ref["v"], ref["beta"], ref["g"], ref["gk"], pool0, w.indices,
                                   w.lengths, w.accepted, w.scale)
    return host(out), host(pool), ro, rp, pool0


def check_decode(w, go, gp, ro, rp, pool0, dt, state_dt=None):
    state_dt = state_dt or dt
    assert_close(go, ro, dt, "out")
    touched = sorted(set(int(w.indices[b * w.S + t]) for b in range(w.B)
                         for t in range(min(int(w.lengths[b]), int(w.accepted[b]) if w.accepted is not None
                                            else int(w.lengths[b])))))
    untouched = [s for s in range(w.pool.shape[0]) if s not in set(touched)]
    if touched:
        assert_close(gp[touched], rp[touched], state_dt, "state")
    # unreferenced slots: bit-exact
    assert np.array_equal(gp[untouched], pool0[untouched])
    # padding rows: exact zero
    for b in range(w.B):
        assert np.all(go[b, :, int(w.lengths[b]):] == 0.0)


def test_decode_workload_bf16():
    """64 sequences, one token each, injective slot map over a 128-slot pool."""
    w = workloads.generate("decode")
    check_decode(w, *run_decode(w, "bf16"), "bf16")


def test_decode_gk_workload_bf16():
    """256 sequences of up to 4 tokens, per-key gate, accepted < length."""
    w = workloads.generate("decode_gk")
    check_decode(w, *run_decode(w, "bf16"), "bf16")


@pytest.mark.parametrize("S,share", [(1, True), (4, False)])
def test_decode_no_gate_d128(S, share):
    """g = NULL and gk = NULL (the operator's hasGamma = 0): the D = 128 kernel's build without the decay."""
    w = workloads.random_case(B=12, Nk=2, Nv=4, S=S, Dk=128, Dv=128, seed=120 + S, gate="none", slots=64,
                              share_slot=share)
    assert w.g is None and w.gk is None
    check_decode(w, *run_decode(w, "bf16"), "bf16")


@pytest.mark.parametrize("sdt", ["f16", "f32"])
def test_decode_f16_d128_workload_and_no_gate(sdt):
    """fp16 inputs on the D = 128 kernel: the decode workload (64 sequences, one token, injective slots) with an
    fp16 or fp32 state, then the same pool stepped without a gate (its build without the decay)."""
    w = workloads.generate("decode")
    check_decode(w, *run_decode(w, "f16", sdt), "f16", sdt)
    w = workloads.random_case(B=12, Nk=2, Nv=4, S=3, Dk=128, Dv=128, seed=125, gate="none", slots=64,
                              share_slot=True)
    check_decode(w, *run_decode(w, "f16", sdt), "f16", sdt)


def test_decode_gk_workload_fused_prologue():
    w = workloads.generate("decode_gk", B=32)
    check_decode(w, *run_decode(w, "bf16", fused=True), "bf16")


@pytest.mark.parametrize("dt,sdt", [("f32", "f32"), ("bf16", "f32"), ("f32", "bf16")])
def test_decode_dtype_combinations(dt, sdt):
    w = workloads.random_case(B=5, Nk=2, Nv=4, S=3, Dk=128, Dv=128, seed=40, slots=9, with_gk=True,
                              initial_state=False, lengths=[3, 1, 2, 0, 3])
    go, gp, ro, rp, p0 = run_decode(w, dt, sdt)
    # out is held to the tolerance of its own dtype, the pool to the state dtype's
    check_decode(w, go, gp, ro, rp, p0, dt, sdt)


@pytest.mark.parametrize("Dk,Dv", [(16, 16), (32, 32), (64, 64), (128, 64), (64, 128), (32, 128), (128, 16)])
def test_decode_head_sizes_f32(Dk, Dv):
    w = workloads.random_case(B=3, Nk=1, Nv=2, S=4, Dk=Dk, Dv=Dv, seed=41 + Dk + Dv, slots=5, initial_state=False,
                              lengths=[4, 2, 3])
    go, gp, ro, rp, p0 = run_decode(w, "f32")
    check_decode(w, go, gp, ro, rp, p0, "f32")


@pytest.mark.parametrize("dt,sdt", [("bf16", "bf16"), ("bf16", "f32")])
def test_decode_max_tokens_per_key_gate(dt, sdt):
    """S = 8, the most tokens one decode call takes, with the per-key gate at D = 128: the largest stage of
    the decode kernel.  Ragged lengths (one empty), accepted counts drawn in [0, L]."""
    w = workloads.random_case(B=12, Nk=2, Nv=4, S=8, Dk=128, Dv=128, seed=44, slots=16, with_gk=True,
                              lengths=[8, 8, 7, 1, 0, 8, 5, 8, 2, 8, 8, 3])
    go, gp, ro, rp, p0 = run_decode(w, dt, sdt)
    check_decode(w, go, gp, ro, rp, p0, dt, sdt)


def test_decode_distinct_slots_per_token():
    """One slot per token: the state after token t lands in slot idx[t] for t < A."""
    w = workloads.random_case(B=4, Nk=2, Nv=4, S=4, Dk=64, Dv=64, seed=43, slots=20, share_slot=False,
                              initial_state=False)
    w.accepted = np.array([4, 2, 1, 3], np.int32)
    go, gp, ro, rp, p0 = run_decode(w, "f32")
    check_decode(w, go, gp, ro, rp, p0, "f32")


def test_tiny_decode_chain_matches_prefill_oracle():
    """The tiny fp32 workload: 8 decode calls of 8 tokens through a 1-slot pool,
    against the oracle's prefill over all 64 tokens (max-abs 1e-4)."""
    w = workloads.generate("tiny")
    ref = unfused_inputs(w, "f32")
    ro, rf = oracle.chunk_fwd(ref["q"], ref["k"], ref["v"], ref["beta"], ref["g"], None, None, w.scale)
    pool = torch.zeros((1, w.Nv, w.Dk, w.Dv), device="cuda")
    idx = torch.zeros(8, dtype=torch.int32, device="cuda")
    L = torch.full((1,), 8, dtype=torch.int32, device="cuda")
    outs = []
    for c in range(8):
        sl = slice(8 * c, 8 * c + 8)
        o, pool = gdr.recurrent_step(dev(ref["q"][:, :, sl], "f32"), dev(ref["k"][:, :, sl], "f32"),
                                     dev(ref["v"][:, :, sl], "f32"), dev(ref["beta"][:, :, sl], "f32"),
                                     dev(ref["g"][:, :, sl], "f32"), None, pool, idx, L, None, w.scale)
        outs.append(host(o))
    assert_close(np.concatenate(outs, axis=2), ro, "f32", "out")
    assert_close(host(pool)[0], rf[0], "f32", "state")


def test_decode_bad_slot_index_sets_error_and_skips():
    w = workloads.random_case(B=3, Nk=1, Nv=1, S=2, Dk=32, Dv=32, seed=44, slots=4, initial_state=False)
    w.accepted = w.lengths.copy()
    ref = unfused_inputs(w, "f32")
    bad_idx = w.indices.copy()
    bad_idx[2:4] = 7  # sequence 1 points past the pool
    pool = dev(rnd32(w.pool), "f32")
    p0 = host(pool)
    out, pool = gdr.recurrent_step(dev(ref["q"], "f32"), dev(ref["k"], "f32"), dev(ref["v"], "f32"),
                                   dev(ref["beta"], "f32"), dev(ref["g"], "f32"), None, pool, dev_i32(bad_idx),
                                   dev_i32(w.lengths), None, w.scale)
    err = gdr.get_error()
    assert err & gdr.DEVERR_SLOT_INDEX
    assert np.all(host(out)[1] == 0.0)
    assert gdr.get_error() == 0  # cleared by the read
    # the other sequences are still correct
    good = [0, 2]
    wi = w.indices.reshape(3, 2)
    ro, rp = oracle.recurrent_step(ref["q"][good], ref["k"][good], ref["v"][good], ref["beta"][good], ref["g"][good],
                                   None, p0, wi[good].ravel(), w.lengths[good], None, w.scale)
    assert_close(host(out)[good], ro, "f32", "out")


def test_decode_bad_length_sets_error():
    w = workloads.random_case(B=2, Nk=1, Nv=1, S=2, Dk=32, Dv=32, seed=45, slots=4, initial_state=False)
    ref = unfused_inputs(w, "f32")
    pool = dev(rnd32(w.pool), "f32")
    p0 = host(pool)
    out, pool = gdr.recurrent_step(dev(ref["q"], "f32"), dev(ref["k"], "f32"), dev(ref["v"], "f32"),
                                   dev(ref["beta"], "f32"), dev(ref["g"], "f32"), None, pool, dev_i32(w.indices),
                                   dev_i32([2, 5]), None, w.scale)
    assert gdr.get_error() & gdr.DEVERR_LENGTH
    assert np.all(host(out)[1] == 0.0)
    slot1 = int(w.indices[2])
    assert np.array_equal(host(pool)[slot1], p0[slot1])


def test_decode_rejects_bad_shapes_before_launch():
    q = torch.zeros((1, 1, 9, 32), device="cuda")
    v = torch.zeros((1, 1, 9, 32), device="cuda")
    pool = torch.zeros((2, 1, 32, 32), device="cuda")
    with pytest.raises(ValueError):
        gdr.recurrent_step(q, q, v, torch.zeros((1, 1, 9), device="cuda"), None, None, pool,
                           torch.zeros(9, dtype=torch.int32, device="cuda"),
                           torch.ones(1, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError):  # indices numel != B * S
        gdr.recurrent_step(q[:, :, :2], q[:, :, :2], v[:, :, :2], torch.zeros((1, 1, 2), device="cuda"), None,
                           None, pool, torch.zeros(3, dtype=torch.int32, device="cuda"),
                           torch.ones(1, dtype=torch.int32, device="cuda"))
