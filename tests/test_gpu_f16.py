"""fp16 inputs (GDR_F16) on every call, against the fp64 oracle fed the same fp16-rounded inputs."""
import numpy as np
import pytest

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, fused_inputs, host, rnd, rnd32, unfused_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.usefixtures("chunk_schedule")
@pytest.mark.parametrize("D,S", [(128, 200), (64, 65), (32, 40)])
def test_chunk_f16(D, S):
    """fp16 prefill (the tensor-core kernel at D = 128, the CUDA-core kernel otherwise) with ragged lengths, one
    empty sequence and an initial state."""
    lengths = np.array([S, max(S - 29, 1), 0], np.int32)
    w = workloads.random_case(B=3, Nk=2, Nv=4, S=S, Dk=D, Dv=D, seed=600 + S + D, lengths=lengths)
    ins = unfused_inputs(w, "f16")
    out, fin = gdr.chunk_fwd(dev(ins["q"], "f16"), dev(ins["k"], "f16"), dev(ins["v"], "f16"),
                             dev(ins["beta"], "f16"), dev(ins["g"], "f32"), dev(ins["initial_state"], "f16"),
                             dev_i32(lengths), w.scale)
    assert gdr.get_error() == 0
    ro, rf = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["initial_state"], lengths,
                              w.scale)
    assert_close(host(out), ro, "f16", "out")
    assert_close(host(fin), rf, "f16", "final_state")
    assert bool((out[0, :, S:] == 0).all()) and bool((out[2] == 0).all())


@pytest.mark.usefixtures("chunk_schedule")
def test_chunk_f16_fused_prologue_and_epilogue():
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=130, Dk=128, Dv=128, seed=610, gate="strong")
    raw, ref = fused_inputs(w, "f16")
    z, nw = workloads.epilogue_inputs(w)
    zr, wr = rnd(z, "f16"), rnd32(nw)
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(raw["A_log"], "f32"),
                       dt_bias=dev(raw["dt_bias"], "f32"))
    epi = gdr.Epilogue(z=dev(zr, "f16"), norm_w=dev(wr, "f32"), eps=1e-6)
    out, fin = gdr.chunk_fwd(dev(raw["q"], "f16"), dev(raw["k"], "f16"), dev(raw["v"], "f16"),
                             dev(raw["b"], "f16"), dev(raw["a"], "f32"), dev(raw["initial_state"], "f16"), None,
                             w.scale, prologue=pro, epilogue=epi)
    assert gdr.get_error() == 0
    ro, rf = oracle.chunk_fwd(ref["q"], ref["k"], ref["v"], ref["beta"], ref["g"], ref["initial_state"], None,
                              w.scale)
    # the row pass sees o already rounded to fp16: one extra 2^-11 rounding, inside the bar
    assert_close(host(out), oracle.gated_rmsnorm(ro, zr, wr, 1e-6), "f16", "out")
    assert_close(host(fin), rf, "f16", "final_state")


@pytest.mark.parametrize("sdt,D,per_token", [("f16", 128, False), ("f32", 128, False), ("f16", 128, True),
                                             ("f32", 128, True), ("f16", 64, True), ("f32", 32, True)])
def test_decode_f16(sdt, D, per_token):
    S, B = 4, 5
    w = workloads.random_case(B=B, Nk=2, Nv=4, S=S, Dk=D, Dv=D, seed=620 + D + per_token, with_gk=True,
                              slots=B * S + 2, share_slot=per_token is False,
                              lengths=np.array([S, 1, 3, S, 2], np.int32))
    if per_token:
        w.accepted = np.array([1, 4, 2, 3, 1], np.int32)
    ins = unfused_inputs(w, "f16")
    pool0 = rnd(w.pool, sdt)
    pool = dev(pool0, sdt)
    out, pool = gdr.recurrent_step(dev(ins["q"], "f16"), dev(ins["k"], "f16"), dev(ins["v"], "f16"),
                                   dev(ins["beta"], "f16"), dev(ins["g"], "f32"), dev(ins["gk"], "f32"), pool,
                                   dev_i32(w.indices), dev_i32(w.lengths), dev_i32(w.accepted), w.scale,
                                   per_token=per_token)
    assert gdr.get_error() == 0
    ro, rp = oracle.recurrent_step(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["gk"], pool0,
                                   w.indices, w.lengths, w.accepted, w.scale, per_token=per_token)
    assert_close(host(out), ro, "f16", "out")
    changed = [s for s in range(pool0.shape[0]) if not np.array_equal(rp[s], pool0[s])]
    assert_close(host(pool)[changed], rp[changed], "f16" if sdt == "f16" else "f32", "state")
    unchanged = [s for s in range(pool0.shape[0]) if s not in changed]
    assert np.array_equal(host(pool)[unchanged], pool0[unchanged])


def test_decode_rejects_f16_with_bf16_state():
    w = workloads.random_case(B=1, Nk=1, Nv=1, S=1, Dk=32, Dv=32, seed=630, slots=2)
    ins = unfused_inputs(w, "f16")
    with pytest.raises(RuntimeError):
        gdr.recurrent_step(dev(ins["q"], "f16"), dev(ins["k"], "f16"), dev(ins["v"], "f16"), dev(ins["beta"], "f16"),
                           dev(ins["g"], "f32"), None, dev(rnd(w.pool, "bf16"), "bf16"), dev_i32(w.indices),
                           dev_i32(w.lengths), None, w.scale)


def test_conv1d_f16():
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=70, Dk=64, Dv=64, seed=640)
    x, wt, bias, st = (rnd(a, "f16") for a in workloads.conv_inputs(w, 4))
    q, k, v, ns = gdr.conv1d(dev(x, "f16"), dev(wt, "f16"), dev(bias, "f16"), dev(st, "f16"), None, Nk=2, Nv=4,
                             Dk=64, Dv=64)
    assert gdr.get_error() == 0
    y, rs = oracle.causal_conv1d(x, wt, bias, st)
    qk = 2 * 64
    assert_close(host(q), y[:, :, :qk].reshape(2, 70, 2, 64).transpose(0, 2, 1, 3), "f16", "q")
    assert_close(host(v), y[:, :, 2 * qk:].reshape(2, 70, 4, 64).transpose(0, 2, 1, 3), "f16", "v")
    assert_close(host(ns), rs, "f16", "state")


@pytest.mark.usefixtures("chunk_schedule")
@pytest.mark.parametrize("gate", ["loguniform", "none"])
def test_chunk_f16_tensor_core_weak_gate(gate):
    """fp16 with D = 128 runs the tensor-core kernel (fp16 MMA operand copies); a weak or absent gate makes
    every block of the WY solve and every cross-chunk term matter."""
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=200, Dk=128, Dv=128, seed=650, gate=gate)
    ins = unfused_inputs(w, "f16")
    out, fin = gdr.chunk_fwd(dev(ins["q"], "f16"), dev(ins["k"], "f16"), dev(ins["v"], "f16"),
                             dev(ins["beta"], "f16"), dev(ins["g"], "f32"), dev(ins["initial_state"], "f16"), None,
                             w.scale)
    assert gdr.get_error() == 0
    ro, rf = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["initial_state"], None,
                              w.scale)
    assert_close(host(out), ro, "f16", "out")
    assert_close(host(fin), rf, "f16", "final_state")


@pytest.mark.usefixtures("chunk_schedule")
def test_prefill_workload_full_size_f16_sampled():
    """The prefill workload in fp16 with the fused prologue (the launch the benchmark's fp16 line times):
    sampled chains computed one by one by the oracle."""
    import torch
    w = workloads.generate("prefill")
    h = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.float16).to("cuda")
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(rnd32(w.A_log), "f32"),
                       dt_bias=dev(rnd32(w.dt_bias), "f32"))
    out, fin = gdr.chunk_fwd(h(w.q), h(w.k), h(w.v), h(w.b), dev(rnd32(w.a), "f32"), h(w.initial_state), None,
                             w.scale, prologue=pro)
    assert gdr.get_error() == 0
    grp = w.Nv // w.Nk
    for b, hh in [(0, 5), (1, 22), (3, 31)]:
        kh = hh // grp
        p = oracle.prologue(q=rnd(w.q[b:b + 1, kh:kh + 1], "f16"), k=rnd(w.k[b:b + 1, kh:kh + 1], "f16"),
                            b=rnd(w.b[b:b + 1, hh:hh + 1], "f16"), a=rnd32(w.a[b:b + 1, hh:hh + 1]),
                            A_log=rnd32(w.A_log[hh:hh + 1]), dt_bias=rnd32(w.dt_bias[hh:hh + 1]))
        ro, rf = oracle.chunk_fwd(p["q_hat"], p["k_hat"], rnd(w.v[b:b + 1, hh:hh + 1], "f16"), p["beta"], p["g"],
                                  rnd(w.initial_state[b:b + 1, hh:hh + 1], "f16"), None, w.scale)
        assert_close(host(out[b, hh]), ro[0, 0], "f16", f"out[{b},{hh}]")
        assert_close(host(fin[b, hh]), rf[0, 0], "f16", f"final[{b},{hh}]")
