"""Chunked prefill (gdr_chunk_fwd) on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import (assert_close, dev, dev_i32, fused_inputs, host, rnd, rnd32, unfused_inputs)

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("chunk_schedule")]


def gpu_chunk(ins, w, dt, lengths=None, fused_raw=None, initial=True):
    """Run gdr_chunk_fwd on already-rounded fp64 inputs; returns (out, final) fp64."""
    s0 = ins["initial_state"] if initial else None
    if fused_raw is not None:
        raw = fused_raw
        pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(raw.get("A_log"), "f32"),
                           dt_bias=dev(raw.get("dt_bias"), "f32"))
        g = raw["a"] if raw.get("a") is not None else raw["g"]
        out, fin = gdr.chunk_fwd(dev(raw["q"], dt), dev(raw["k"], dt), dev(raw["v"], dt), dev(raw["b"], dt),
                                 dev(g, "f32"), dev(s0, dt), dev_i32(lengths), w.scale, prologue=pro)
    else:
        out, fin = gdr.chunk_fwd(dev(ins["q"], dt), dev(ins["k"], dt), dev(ins["v"], dt), dev(ins["beta"], dt),
                                 dev(ins["g"], "f32"), dev(s0, dt), dev_i32(lengths), w.scale)
    assert gdr.get_error() == 0
    return host(out), host(fin)


def ref_chunk(ref, w, lengths=None, initial=True, sel=None):
    """Oracle over all chains, or over the (b, h) pairs in sel (each as its own
    one-chain problem)."""
    s0 = ref["initial_state"] if initial else None
    if sel is None:
        return oracle.chunk_fwd(ref["q"], ref["k"], ref["v"], ref["beta"], ref["g"], s0, lengths, w.scale)
    outs, fins = [], []
    grp = w.Nv // w.Nk
    for b, h in sel:
        kh = h // grp
        L = None if lengths is None else np.asarray(lengths)[b:b + 1]
        o, f = oracle.chunk_fwd(ref["q"][b:b + 1, kh:kh + 1], ref["k"][b:b + 1, kh:kh + 1],
                                ref["v"][b:b + 1, h:h + 1], ref["beta"][b:b + 1, h:h + 1],
                                None if ref["g"] is None else ref["g"][b:b + 1, h:h + 1],
                                None if s0 is None else s0[b:b + 1, h:h + 1], L, w.scale)
        outs.append(o[0, 0])
        fins.append(f[0, 0])
    return np.stack(outs), np.stack(fins)


def test_tiny_workload_f32():
    """B=1, S=64, 2 heads, D=32, fp32: max-abs <= 1e-4 on out and final state."""
    w = workloads.generate("tiny")
    ins = unfused_inputs(w, "f32")
    go, gf = gpu_chunk(ins, w, "f32", initial=False)
    ro, rf = ref_chunk(ins, w, initial=False)
    assert_close(go, ro, "f32", "out")
    assert_close(gf, rf, "f32", "final_state")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("S", [1, 63, 64, 65, 200])
def test_ragged_lengths_d128(dt, S):
    w = workloads.generate("prefill", B=2, S=S, Nk=2, Nv=4, D=128)
    ins = unfused_inputs(w, dt)
    go, gf = gpu_chunk(ins, w, dt)
    ro, rf = ref_chunk(ins, w)
    assert_close(go, ro, dt, "out")
    assert_close(gf, rf, dt, "final_state")


@pytest.mark.parametrize("gate", ["loguniform", "none"])
@pytest.mark.parametrize("S", [64, 200])
def test_weak_gate_bf16_d128(gate, S):
    """bf16, D=128 (the tensor-core path) with decay close to 1 (g = log U(0.9, 0.999)) or no gate at
    all: the WY transform T = (I + A)^{-1} then has large off-diagonal blocks, so every block of the
    solve and every cross-chunk term is exercised (a strong decay hides both)."""
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=S, Dk=128, Dv=128, seed=80 + S, gate=gate)
    ins = unfused_inputs(w, "bf16")
    go, gf = gpu_chunk(ins, w, "bf16")
    ro, rf = ref_chunk(ins, w)
    assert_close(go, ro, "bf16", "out")
    assert_close(gf, rf, "bf16", "final_state")
    # the bar is 2e-2; this path stays well inside it (about 3e-3), so a broken block of the solve
    # (which costs 1e-1 or more here) cannot hide under the tolerance
    from tests._helpers import rel_l2
    assert rel_l2(go, ro) < 1e-2 and rel_l2(gf, rf) < 1e-2


@pytest.mark.parametrize("Dk,Dv", [(16, 16), (32, 64), (64, 64), (64, 128), (128, 32), (128, 16)])
def test_head_sizes_f32(Dk, Dv):
    w = workloads.random_case(B=2, Nk=1, Nv=2, S=150, Dk=Dk, Dv=Dv, seed=50 + Dk + Dv, gate="strong")
    ins = unfused_inputs(w, "f32")
    go, gf = gpu_chunk(ins, w, "f32")
    ro, rf = ref_chunk(ins, w)
    assert_close(go, ro, "f32", "out")
    assert_close(gf, rf, "f32", "final_state")


@pytest.mark.parametrize("group", [1, 2, 4])
def test_gqa_groups(group):
    w = workloads.random_case(B=1, Nk=2, Nv=2 * group, S=130, Dk=64, Dv=64, seed=60 + group)
    ins = unfused_inputs(w, "f32")
    go, gf = gpu_chunk(ins, w, "f32")
    ro, rf = ref_chunk(ins, w)
    assert_close(go, ro, "f32", "out")
    assert_close(gf, rf, "f32", "final_state")


def test_varlen_padding_zero_and_empty_sequence():
    """Lengths 0, 1, 64, 100, S: padding rows exactly zero; L=0 returns the
    initial state bit for bit; padding contents (here NaN) never leak."""
    w = workloads.generate("varlen", B=5, S=160, Nk=2, Nv=4, D=128)
    L = np.array([0, 1, 64, 100, 160], np.int32)
    for dt in ("f32", "bf16"):
        ins = unfused_inputs(w, dt)
        dirty = {k: (v.copy() if v is not None else None) for k, v in ins.items()}
        for b in range(w.B):
            for key in ("q", "k", "v"):
                dirty[key][b, :, L[b]:] = np.nan
            dirty["beta"][b, :, L[b]:] = np.nan
            dirty["g"][b, :, L[b]:] = np.nan
        go, gf = gpu_chunk(dirty, w, dt, lengths=L)
        ro, rf = ref_chunk(ins, w, lengths=L)
        assert_close(go, ro, dt, "out")
        assert_close(gf, rf, dt, "final_state")
        for b in range(w.B):
            assert np.all(go[b, :, L[b]:] == 0.0)
        assert np.array_equal(gf[0], ins["initial_state"][0])


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_varlen_more_chains_than_sms_longest_first(dt):
    """B = 40 sequences x Nv = 4 heads = 160 chains, more than the 148 SMs hold at once, so the tensor-core
    kernel starts the longest sequences first: ragged lengths with ties, zeros and a full-length one, every
    output row and final state against the oracle (padding rows zero, L = 0 states bit for bit)."""
    B, S = 40, 130
    L = np.random.default_rng(77).integers(0, S + 1, size=B).astype(np.int32)
    L[:4] = [S, 0, 70, 70]
    w = workloads.random_case(B=B, Nk=2, Nv=4, S=S, Dk=128, Dv=128, seed=78, lengths=L)
    ins = unfused_inputs(w, dt)
    go, gf = gpu_chunk(ins, w, dt, lengths=L)
    ro, rf = ref_chunk(ins, w, lengths=L)
    assert_close(go, ro, dt, "out")
    assert_close(gf, rf, dt, "final_state")
    for b in range(B):
        assert np.all(go[b, :, L[b]:] == 0.0)
        if L[b] == 0:
            assert np.array_equal(gf[b], ins["initial_state"][b])


def test_no_gate_no_initial_state_and_empty_sequence_axis():
    w = workloads.random_case(B=2, Nk=2, Nv=2, S=70, Dk=32, Dv=32, seed=70, gate="none", initial_state=False)
    ins = unfused_inputs(w, "f32")
    go, gf = gpu_chunk(ins, w, "f32", initial=False)
    ro, rf = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], None, None, None, w.scale)
    assert_close(go, ro, "f32", "out")
    assert_close(gf, rf, "f32", "final_state")
    # S == 0: the final state is the initial state
    s0 = torch.randn((2, 2, 32, 32), device="cuda")
    z = torch.zeros((2, 2, 0, 32), device="cuda")
    out, fin = gdr.chunk_fwd(z, z, z, torch.zeros((2, 2, 0), device="cuda"), None, s0, None, 1.0)
    assert out.shape == (2, 2, 0, 32) and torch.equal(fin, s0)


def test_final_state_in_place():
    w = workloads.random_case(B=2, Nk=1, Nv=2, S=90, Dk=64, Dv=64, seed=71)
    ins = unfused_inputs(w, "f32")
    st = dev(ins["initial_state"], "f32")
    out, fin = gdr.chunk_fwd(dev(ins["q"], "f32"), dev(ins["k"], "f32"), dev(ins["v"], "f32"),
                             dev(ins["beta"], "f32"), dev(ins["g"], "f32"), st, None, w.scale, final_state=st)
    ro, rf = ref_chunk(ins, w)
    assert fin.data_ptr() == st.data_ptr()
    assert_close(host(st), rf, "f32", "final_state")


def test_split_resume_on_gpu():
    """Two calls (L1 then L2 from the returned state) match one oracle call."""
    w = workloads.random_case(B=1, Nk=1, Nv=2, S=200, Dk=64, Dv=64, seed=72)
    ins = unfused_inputs(w, "f32")
    cut = 77
    first = {k: (v[:, :, :cut] if k not in ("initial_state",) and v is not None else v) for k, v in ins.items()}
    o1, f1 = gpu_chunk(first, w, "f32")
    second = {k: (v[:, :, cut:] if k not in ("initial_state",) and v is not None else v) for k, v in ins.items()}
    second["initial_state"] = f1
    o2, f2 = gpu_chunk(second, w, "f32")
    ro, rf = ref_chunk(ins, w)
    assert_close(np.concatenate([o1, o2], axis=2), ro, "f32", "out")
    assert_close(f2, rf, "f32", "final_state")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_fused_prologue_strong_gate(dt):
    """Raw q/k, beta logits and the raw gate a with A_log/dt_bias (decay down to
    about -20 per token) through the fused prologue."""
    w = workloads.generate("prefill", B=2, S=150, Nk=2, Nv=4, D=128)
    raw, ref = fused_inputs(w, dt)
    go, gf = gpu_chunk(ref, w, dt, fused_raw=raw)
    ro, rf = ref_chunk(ref, w)
    assert_close(go, ro, dt, "out")
    assert_close(gf, rf, dt, "final_state")


def test_prefill_workload_full_size_sampled():
    """B=4, S=4096, Nk=16, Nv=32, D=128, bf16: the full-size call, checked on
    sampled chains computed one by one by the oracle."""
    w = workloads.generate("prefill")
    ins = unfused_inputs(w, "bf16")
    go, gf = gpu_chunk(ins, w, "bf16")
    sel = [(0, 0), (1, 17), (3, 31), (2, 6)]
    ro, rf = ref_chunk(ins, w, sel=sel)
    for i, (b, h) in enumerate(sel):
        assert_close(go[b, h], ro[i], "bf16", f"out[{b},{h}]")
        assert_close(gf[b, h], rf[i], "bf16", f"final[{b},{h}]")
    assert np.all(np.isfinite(go))


def _bf16_dev(x):
    """fp32 numpy -> bf16 device tensor, rounded on the CPU (the same rounding
    tests._helpers.rnd applies to the oracle's copy of a slice)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to("cuda")


def test_varlen_workload_full_size_sampled_fused():
    """B=8, padded S=8192, one empty sequence, fused prologue: sampled chains
    against the oracle, every padding row zero, empty sequence's state intact.
    The oracle's prologue runs on the sampled chains' raw (rounded) inputs only."""
    w = workloads.generate("varlen")
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(rnd32(w.A_log), "f32"),
                       dt_bias=dev(rnd32(w.dt_bias), "f32"))
    s0 = _bf16_dev(w.initial_state)
    out, fin = gdr.chunk_fwd(_bf16_dev(w.q), _bf16_dev(w.k), _bf16_dev(w.v), _bf16_dev(w.b),
                             dev(rnd32(w.a), "f32"), s0, dev_i32(w.lengths), w.scale, prologue=pro)
    assert gdr.get_error() == 0
    zero_b = int(np.flatnonzero(w.lengths == 0)[0])
    other = [b for b in range(w.B) if b != zero_b]
    grp = w.Nv // w.Nk
    for b, h in [(other[0], 3), (other[3], 20), (other[6], 31)]:
        kh = h // grp
        L = int(w.lengths[b])
        sl = (slice(b, b + 1),)
        p = oracle.prologue(q=rnd(w.q[b:b + 1, kh:kh + 1], "bf16"), k=rnd(w.k[b:b + 1, kh:kh + 1], "bf16"),
                            b=rnd(w.b[b:b + 1, h:h + 1], "bf16"), a=rnd32(w.a[b:b + 1, h:h + 1]),
                            A_log=rnd32(w.A_log[h:h + 1]), dt_bias=rnd32(w.dt_bias[h:h + 1]))
        ro, rf = oracle.chunk_fwd(p["q_hat"], p["k_hat"], rnd(w.v[b:b + 1, h:h + 1], "bf16"), p["beta"], p["g"],
                                  rnd(w.initial_state[b:b + 1, h:h + 1], "bf16"), w.lengths[sl], w.scale)
        assert_close(host(out[b, h, :L]), ro[0, 0, :L], "bf16", f"out[{b},{h}]")
        assert_close(host(fin[b, h]), rf[0, 0], "bf16", f"final[{b},{h}]")
    for b in range(w.B):
        assert bool((out[b, :, int(w.lengths[b]):] == 0).all())
    assert torch.equal(fin[zero_b], s0[zero_b])


def test_bad_length_sets_device_error():
    w = workloads.random_case(B=2, Nk=1, Nv=1, S=20, Dk=32, Dv=32, seed=73)
    ins = unfused_inputs(w, "f32")
    out, fin = gdr.chunk_fwd(dev(ins["q"], "f32"), dev(ins["k"], "f32"), dev(ins["v"], "f32"),
                             dev(ins["beta"], "f32"), dev(ins["g"], "f32"), dev(ins["initial_state"], "f32"),
                             dev_i32([20, 21]), w.scale)
    assert gdr.get_error() & gdr.DEVERR_LENGTH
    assert np.all(host(out)[1] == 0.0)
    assert np.array_equal(host(fin)[1], ins["initial_state"][1])
