"""The decode call with per-token state slots (gdr_recurrent_step_spec, the speculative-decoding reading of
num_accepted_tokens) on the GPU against the fp64 oracle."""
import numpy as np
import pytest

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, host, rnd, unfused_inputs

pytestmark = pytest.mark.gpu


def run_spec(w, dt, sdt, accepted, pool0):
    ins = unfused_inputs(w, dt)
    pool = dev(pool0, sdt)
    out, pool = gdr.recurrent_step(dev(ins["q"], dt), dev(ins["k"], dt), dev(ins["v"], dt), dev(ins["beta"], dt),
                                   dev(ins["g"], "f32"), dev(ins["gk"], "f32"), pool, dev_i32(w.indices),
                                   dev_i32(w.lengths), dev_i32(accepted), w.scale, per_token=True)
    err = gdr.get_error()
    ro, rp = oracle.recurrent_step(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["gk"], pool0, w.indices,
                                   w.lengths, accepted, w.scale, per_token=True)
    return host(out), host(pool), ro, rp, err


@pytest.mark.parametrize("dt,sdt,D,S", [("bf16", "bf16", 128, 4), ("bf16", "f32", 128, 8), ("f32", "f32", 64, 3),
                                        ("f32", "bf16", 32, 5)])
def test_spec_decode_parity(dt, sdt, D, S):
    """Every token has its own slot; accepted counts in [1, S]; ragged lengths; the per-key gate."""
    B = 6
    w = workloads.random_case(B=B, Nk=2, Nv=4, S=S, Dk=D, Dv=D, seed=500 + S + D, with_gk=True, slots=B * S + 3,
                              share_slot=False, lengths=np.array([S, 1, S, max(S - 1, 1), 2, S], np.int32))
    accepted = np.array([1 + (3 * b) % S for b in range(B)], np.int32)
    pool0 = rnd(w.pool, sdt)
    go, gp, ro, rp, err = run_spec(w, dt, sdt, accepted, pool0)
    assert err == 0
    assert_close(go, ro, dt, "out")
    touched = sorted(set(int(w.indices[b * S + t]) for b in range(B) for t in range(int(w.lengths[b]))))
    untouched = [s for s in range(w.pool.shape[0]) if s not in set(touched)]
    assert_close(gp[touched], rp[touched], sdt, "state")
    assert np.array_equal(gp[untouched], pool0[untouched])
    for b in range(B):
        assert np.all(go[b, :, int(w.lengths[b]):] == 0.0)


def test_spec_decode_two_steps_on_device():
    """Step 1 from slot idx[0] (A = 1) writes each token's state to its slot; step 2 with A = 3 starts from the
    third token's state.  Both steps on the GPU against the same two oracle steps."""
    S = 4
    w1 = workloads.random_case(B=2, Nk=1, Nv=2, S=S, Dk=128, Dv=128, seed=520, with_gk=False, slots=12,
                               share_slot=False)
    w2 = workloads.random_case(B=2, Nk=1, Nv=2, S=S, Dk=128, Dv=128, seed=521, with_gk=False, slots=12,
                               share_slot=False)
    w2.indices = w1.indices  # the same per-token slots in both steps
    pool0 = rnd(w1.pool, "bf16")
    for w in (w1, w2):
        w.gk = None
    in1, in2 = unfused_inputs(w1, "bf16"), unfused_inputs(w2, "bf16")
    pool = dev(pool0, "bf16")
    outs = []
    for ins, A in ((in1, np.array([1, 1], np.int32)), (in2, np.array([3, 2], np.int32))):
        out, pool = gdr.recurrent_step(dev(ins["q"], "bf16"), dev(ins["k"], "bf16"), dev(ins["v"], "bf16"),
                                       dev(ins["beta"], "bf16"), dev(ins["g"], "f32"), None, pool,
                                       dev_i32(w1.indices), dev_i32(w1.lengths), dev_i32(A), w1.scale, per_token=True)
        outs.append(host(out))
    assert gdr.get_error() == 0
    rp = pool0
    for i, (ins, A) in enumerate(((in1, np.array([1, 1], np.int32)), (in2, np.array([3, 2], np.int32)))):
        ro, rp = oracle.recurrent_step(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], None, rp, w1.indices,
                                       w1.lengths, A, w1.scale, per_token=True)
        assert_close(outs[i], ro, "bf16", f"out step {i + 1}")
    touched = sorted(set(int(s) for s in w1.indices))
    assert_close(host(pool)[touched], rp[touched], "bf16", "state")


def test_spec_decode_accepted_out_of_range_skips_and_flags():
    S = 3
    w = workloads.random_case(B=2, Nk=1, Nv=2, S=S, Dk=64, Dv=64, seed=530, slots=8, share_slot=False)
    accepted = np.array([0, 2], np.int32)  # A = 0 is outside [1, S]
    pool0 = rnd(w.pool, "f32")
    ins = unfused_inputs(w, "f32")
    pool = dev(pool0, "f32")
    out, pool = gdr.recurrent_step(dev(ins["q"], "f32"), dev(ins["k"], "f32"), dev(ins["v"], "f32"),
                                   dev(ins["beta"], "f32"), dev(ins["g"], "f32"), None, pool, dev_i32(w.indices),
                                   dev_i32(w.lengths), dev_i32(accepted), w.scale, per_token=True)
    assert gdr.get_error() == gdr.DEVERR_LENGTH
    go, gp = host(out), host(pool)
    assert np.all(go[0] == 0.0)
    own0 = [int(s) for s in w.indices[:S]]
    assert np.array_equal(gp[own0], pool0[own0])
    sl = slice(1, 2)
    ro, rp = oracle.recurrent_step(ins["q"][sl], ins["k"][sl], ins["v"][sl], ins["beta"][sl], ins["g"][sl], None,
                                   pool0, w.indices[S:], w.lengths[sl], accepted[sl], w.scale, per_token=True)
    assert_close(go[1:], ro, "f32", "out")
