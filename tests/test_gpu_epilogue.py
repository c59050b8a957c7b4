"""The gated RMSNorm output epilogue (gdr_epilogue) on the GPU against the fp64 oracle: the oracle's
recurrence, then oracle.gated_rmsnorm of its out rows with the same (rounded) z and norm_w."""
import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, host, rnd, rnd32, unfused_inputs

pytestmark = pytest.mark.gpu

EPS = 1e-6


def epilogue_for(w, dt):
    """(z rounded to dt as fp64, norm_w rounded to fp32 as fp64, the library's Epilogue)."""
    z, nw = workloads.epilogue_inputs(w)
    zr, wr = rnd(z, dt), rnd32(nw)
    return zr, wr, gdr.Epilogue(z=dev(zr, dt), norm_w=dev(wr, "f32"), eps=EPS)


@pytest.mark.parametrize("dt,D,S", [("bf16", 128, 200), ("bf16", 128, 64), ("bf16", 128, 1), ("f32", 128, 130),
                                    ("f32", 64, 150), ("f32", 16, 40), ("bf16", 64, 100)])
@pytest.mark.usefixtures("chunk_schedule")
def test_chunk_epilogue(dt, D, S):
    """bf16 with D = 128 runs the epilogue inside the tensor-core kernel; the other cases run the CUDA-core
    kernel and the row pass.  Lengths are ragged, with one empty sequence."""
    lengths = np.array([S, max(S - 37, 1), 0], np.int32)
    w = workloads.random_case(B=3, Nk=2, Nv=4, S=S, Dk=D, Dv=D, seed=300 + S + D, gate="loguniform",
                              lengths=lengths)
    ins = unfused_inputs(w, dt)
    zr, wr, epi = epilogue_for(w, dt)
    out, fin = gdr.chunk_fwd(dev(ins["q"], dt), dev(ins["k"], dt), dev(ins["v"], dt), dev(ins["beta"], dt),
                             dev(ins["g"], "f32"), dev(ins["initial_state"], dt), dev_i32(lengths), w.scale,
                             epilogue=epi)
    assert gdr.get_error() == 0
    ro, rf = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["initial_state"], lengths,
                              w.scale)
    ref = oracle.gated_rmsnorm(ro, zr, wr, EPS, lengths)
    go = host(out)
    assert_close(go, ref, dt, "out")
    assert_close(host(fin), rf, dt, "final_state")  # the epilogue touches out only
    for b in range(w.B):
        assert np.all(go[b, :, int(lengths[b]):] == 0.0)


@pytest.mark.usefixtures("chunk_schedule")
def test_chunk_epilogue_with_fused_prologue_strong_gate():
    """bf16, D = 128, raw q/k/b/a through the fused prologue and the epilogue in the same call."""
    from tests._helpers import fused_inputs
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=190, Dk=128, Dv=128, seed=333, gate="strong",
                              lengths=np.array([190, 77], np.int32))
    raw, ref_in = fused_inputs(w, "bf16")
    zr, wr, epi = epilogue_for(w, "bf16")
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(raw["A_log"], "f32"),
                       dt_bias=dev(raw["dt_bias"], "f32"))
    out, fin = gdr.chunk_fwd(dev(raw["q"], "bf16"), dev(raw["k"], "bf16"), dev(raw["v"], "bf16"),
                             dev(raw["b"], "bf16"), dev(raw["a"], "f32"), dev(raw["initial_state"], "bf16"),
                             dev_i32(w.lengths), w.scale, prologue=pro, epilogue=epi)
    assert gdr.get_error() == 0
    ro, rf = oracle.chunk_fwd(ref_in["q"], ref_in["k"], ref_in["v"], ref_in["beta"], ref_in["g"],
                              ref_in["initial_state"], w.lengths, w.scale)
    assert_close(host(out), oracle.gated_rmsnorm(ro, zr, wr, EPS, w.lengths), "bf16", "out")
    assert_close(host(fin), rf, "bf16", "final_state")


@pytest.mark.parametrize("dt,sdt,D,S", [("bf16", "bf16", 128, 1), ("bf16", "bf16", 128, 4), ("f32", "f32", 64, 3),
                                        ("f32", "bf16", 32, 2)])
def test_decode_epilogue(dt, sdt, D, S):
    """Decode with the per-key gate, accepted counts below the lengths and the epilogue."""
    w = workloads.random_case(B=6, Nk=2, Nv=4, S=S, Dk=D, Dv=D, seed=340 + S + D, gate="loguniform",
                              lengths=np.array([S, 1, S, max(S - 1, 1), S, 1], np.int32), with_gk=True,
                              slots=9)
    ins = unfused_inputs(w, dt)
    zr, wr, epi = epilogue_for(w, dt)
    pool0 = rnd(w.pool, sdt)
    pool = dev(pool0, sdt)
    out, pool = gdr.recurrent_step(dev(ins["q"], dt), dev(ins["k"], dt), dev(ins["v"], dt), dev(ins["beta"], dt),
                                   dev(ins["g"], "f32"), dev(ins["gk"], "f32"), pool, dev_i32(w.indices),
                                   dev_i32(w.lengths), dev_i32(w.accepted), w.scale, epilogue=epi)
    assert gdr.get_error() == 0
    ro, rp = oracle.recurrent_step(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["gk"], pool0,
                                   w.indices, w.lengths, w.accepted, w.scale)
    assert_close(host(out), oracle.gated_rmsnorm(ro, zr, wr, EPS, w.lengths), dt, "out")
    touched = sorted(set(int(w.indices[b * S + t]) for b in range(w.B) for t in range(int(w.accepted[b]))))
    if touched:
        assert_close(host(pool)[touched], rp[touched], sdt, "state")


def _bf16_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to("cuda")


def test_prefill_workload_full_size_epilogue_sampled():
    """B=4, S=4096, Nk=16, Nv=32, D=128, bf16 with the fused prologue and the epilogue (the launch the
    benchmark's epilogue line times): sampled chains computed one by one by the oracle."""
    w = workloads.generate("prefill")
    z, nw = workloads.epilogue_inputs(w)
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(rnd32(w.A_log), "f32"),
                       dt_bias=dev(rnd32(w.dt_bias), "f32"))
    epi = gdr.Epilogue(z=_bf16_dev(z), norm_w=dev(rnd32(nw), "f32"), eps=EPS)
    out, fin = gdr.chunk_fwd(_bf16_dev(w.q), _bf16_dev(w.k), _bf16_dev(w.v), _bf16_dev(w.b), dev(rnd32(w.a), "f32"),
                             _bf16_dev(w.initial_state), None, w.scale, prologue=pro, epilogue=epi)
    assert gdr.get_error() == 0
    grp = w.Nv // w.Nk
    for b, h in [(0, 1), (2, 18), (3, 30)]:
        kh = h // grp
        p = oracle.prologue(q=rnd(w.q[b:b + 1, kh:kh + 1], "bf16"), k=rnd(w.k[b:b + 1, kh:kh + 1], "bf16"),
                            b=rnd(w.b[b:b + 1, h:h + 1], "bf16"), a=rnd32(w.a[b:b + 1, h:h + 1]),
                            A_log=rnd32(w.A_log[h:h + 1]), dt_bias=rnd32(w.dt_bias[h:h + 1]))
        ro, rf = oracle.chunk_fwd(p["q_hat"], p["k_hat"], rnd(w.v[b:b + 1, h:h + 1], "bf16"), p["beta"], p["g"],
                                  rnd(w.initial_state[b:b + 1, h:h + 1], "bf16"), None, w.scale)
        ref = oracle.gated_rmsnorm(ro, rnd(z[b:b + 1, h:h + 1], "bf16"), rnd32(nw), EPS)
        assert_close(host(out[b, h]), ref[0, 0], "bf16", f"out[{b},{h}]")
        assert_close(host(fin[b, h]), rf[0, 0], "bf16", f"final[{b},{h}]")
    assert bool(torch.isfinite(out).all())
