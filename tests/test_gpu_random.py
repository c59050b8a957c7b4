"""Seeded random sweeps of the prefill (tensor-core path, both schedules) and of decode against the fp64 oracle.

Each case draws its own sizes and options from one seed: 1-3 sequences, 1-2 key heads with 1, 2 or 4 value heads
each (GQA), S from 1 to 300 (so partial last chunks and single-token sequences), per-sequence lengths that are
full, ragged or zero, the gate (none, log-uniform, or raw a / A_log / dt_bias through the fused prologue), bf16 or
fp16, with or without an initial state and with or without the gated RMSNorm epilogue.  The lite_boost
chunk_gated_delta_rule page fixes the layout, the optional gate and initial state, the variable lengths and the
zero padding rows checked here; the rule itself is the oracle's token loop (torch_recurrent_gated_delta_rule of
the blog "gated-delta-net" page).
"""
import numpy as np
import pytest

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, fused_inputs, host, rnd, rnd32, unfused_inputs

pytestmark = pytest.mark.gpu

CASES = 40
DCASES = 32
EPS = 1e-6


def draw(seed: int):
    rng = np.random.default_rng([2026, seed])
    B = int(rng.integers(1, 4))
    Nk = int(rng.integers(1, 3))
    Nv = Nk * int(rng.choice([1, 2, 4]))
    S = int(rng.integers(1, 301))
    lengths = []
    for _ in range(B):
        kind = rng.integers(0, 3)
        lengths.append(S if kind == 0 else (0 if kind == 1 and B > 1 else int(rng.integers(1, S + 1))))
    return dict(B=B, Nk=Nk, Nv=Nv, S=S, lengths=np.array(lengths, np.int32),
                gate=str(rng.choice(["none", "loguniform", "strong"])), dt=str(rng.choice(["bf16", "f16"])),
                init=bool(rng.random() < 0.7), epi=bool(rng.random() < 0.3))


@pytest.mark.usefixtures("chunk_schedule")
@pytest.mark.parametrize("seed", range(CASES))
def test_random_prefill_case(seed):
    c = draw(seed)
    dt = c["dt"]
    w = workloads.random_case(B=c["B"], Nk=c["Nk"], Nv=c["Nv"], S=c["S"], Dk=128, Dv=128, seed=10000 + seed,
                              gate=c["gate"], lengths=c["lengths"], initial_state=c["init"])
    epi = None
    if c["epi"]:
        z, nw = workloads.epilogue_inputs(w)
        zr, wr = rnd(z, dt), rnd32(nw)
        epi = gdr.Epilogue(z=dev(zr, dt), norm_w=dev(wr, "f32"), eps=EPS)
    lens = dev_i32(w.lengths)
    if c["gate"] == "strong":  # raw inputs through the fused prologue
        raw, ref = fused_inputs(w, dt)
        pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(raw["A_log"], "f32"),
                           dt_bias=dev(raw["dt_bias"], "f32"))
        out, fin = gdr.chunk_fwd(dev(raw["q"], dt), dev(raw["k"], dt), dev(raw["v"], dt), dev(raw["b"], dt),
                                 dev(raw["a"], "f32"), dev(raw["initial_state"], dt), lens, w.scale, prologue=pro,
                                 epilogue=epi)
    else:
        ref = unfused_inputs(w, dt)
        out, fin = gdr.chunk_fwd(dev(ref["q"], dt), dev(ref["k"], dt), dev(ref["v"], dt), dev(ref["beta"], dt),
                                 dev(ref["g"], "f32"), dev(ref["initial_state"], dt), lens, w.scale, epilogue=epi)
    assert gdr.get_error() == 0, c
    ro, rf = oracle.chunk_fwd(ref["q"], ref["k"], ref["v"], ref["beta"], ref["g"], ref["initial_state"], w.lengths,
                              w.scale)
    if c["epi"]:
        ro = oracle.gated_rmsnorm(ro, zr, wr, EPS, w.lengths)
    go, gf = host(out), host(fin)
    assert_close(go, ro, dt, f"out {c}")
    assert_close(gf, rf, dt, f"final_state {c}")
    for b in range(w.B):
        assert np.all(go[b, :, int(w.lengths[b]):] == 0.0), c
        if w.lengths[b] == 0:  # an empty sequence leaves its state as it was (zeros without an initial state)
            s0 = ref["initial_state"][b] if ref["initial_state"] is not None else np.zeros_like(gf[b])
            assert np.array_equal(gf[b], s0), c


def draw_decode(seed: int):
    rng = np.random.default_rng([2027, seed])
    B = int(rng.integers(1, 17))
    Nk = int(rng.integers(1, 3))
    Nv = Nk * int(rng.choice([1, 2, 4]))
    S = int(rng.integers(1, 9))
    spec = bool(rng.random() < 0.3)
    gate = str(rng.choice(["none", "loguniform", "strong"]))
    gk = bool(gate != "none" and rng.random() < 0.4)
    dt, sdt = [("bf16", "bf16"), ("bf16", "f32"), ("f32", "bf16"), ("f32", "f32"), ("f16", "f16"),
               ("f16", "f32")][int(rng.integers(0, 6))]
    lengths = []
    for _ in range(B):
        kind = rng.integers(0, 3)
        lengths.append(S if kind == 0 else (0 if kind == 1 and B > 1 else int(rng.integers(1, S + 1))))
    accepted = rng.integers(1, S + 1, size=B).astype(np.int32) if spec else None
    return dict(B=B, Nk=Nk, Nv=Nv, S=S, spec=spec, gate=gate, gk=gk, dt=dt, sdt=sdt,
                lengths=np.array(lengths, np.int32), accepted=accepted)


@pytest.mark.parametrize("seed", range(DCASES))
def test_random_decode_case(seed):
    """Decode over a slot pool (the lite_boost recurrent_gated_delta_rule page): shared slots with accepted counts
    in [0, L] (the committed-slot reading), or one slot per token with accepted counts in [1, S] (the
    speculative reading); slots the oracle leaves alone stay bit for bit."""
    c = draw_decode(seed)
    dt, sdt = c["dt"], c["sdt"]
    slots = c["B"] * c["S"] + 8
    w = workloads.random_case(B=c["B"], Nk=c["Nk"], Nv=c["Nv"], S=c["S"], Dk=128, Dv=128, seed=20000 + seed,
                              gate=c["gate"], lengths=c["lengths"], with_gk=c["gk"], slots=slots,
                              share_slot=not c["spec"])
    if c["spec"]:
        w.accepted = c["accepted"]
    pool0 = rnd(w.pool, sdt)
    pool = dev(pool0, sdt)
    if c["gate"] == "strong":
        raw, ref = fused_inputs(w, dt)
        pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=dev(raw["A_log"], "f32"),
                           dt_bias=dev(raw["dt_bias"], "f32"))
        out, pool = gdr.recurrent_step(dev(raw["q"], dt), dev(raw["k"], dt), dev(raw["v"], dt), dev(raw["b"], dt),
                                       dev(raw["a"], "f32"), dev(raw["gk"], "f32"), pool, dev_i32(w.indices),
                                       dev_i32(w.lengths), dev_i32(w.accepted), w.scale, prologue=pro,
                                       per_token=c["spec"])
    else:
        ref = unfused_inputs(w, dt)
        out, pool = gdr.recurrent_step(dev(ref["q"], dt), dev(ref["k"], dt), dev(ref["v"], dt), dev(ref["beta"], dt),
                                       dev(ref["g"], "f32"), dev(ref["gk"], "f32"), pool, dev_i32(w.indices),
                                       dev_i32(w.lengths), dev_i32(w.accepted), w.scale, per_token=c["spec"])
    assert gdr.get_error() == 0, c
    ro, rp = oracle.recurrent_step(ref["q"], ref["k"], ref["v"], ref["beta"], ref["g"], ref["gk"], pool0, w.indices,
                                   w.lengths, w.accepted, w.scale, per_token=c["spec"])
    go, gp = host(out), host(pool)
    assert_close(go, ro, dt, f"out {c}")
    for b in range(w.B):
        assert np.all(go[b, :, int(w.lengths[b]):] == 0.0), c
    kept = [s for s in range(slots) if np.array_equal(rp[s], pool0[s])]
    moved = [s for s in range(slots) if s not in set(kept)]
    assert np.array_equal(gp[kept], pool0[kept]), c
    if moved:
        assert_close(gp[moved], rp[moved], sdt, f"state {c}")
