"""The oracle against what the pages and the mathematics fix (CPU only)."""
import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads
from tests import _decode_pins, _pins


def chunk_impl(q, k, v, beta, g, S0, lengths, scale):
    return oracle.chunk_fwd(q, k, v, beta, g, S0, lengths, scale)


@pytest.mark.parametrize("check", _pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_chunk_oracle_pin(check):
    check(chunk_impl)


def decode_as_chunk(q, k, v, beta, g, S0, lengths, scale):
    """The decode oracle driven through a pool with one slot per chain and
    every token accepted must satisfy the same pins."""
    B, Nv = v.shape[:2]
    S = q.shape[2]
    slots = B + 3
    pool = np.zeros((slots,) + S0.shape[1:]) + 0.25
    perm = np.arange(B)[::-1] + 2
    pool[perm] = S0
    idx = np.repeat(perm, S).astype(np.int32)
    L = np.full(B, S, np.int32) if lengths is None else np.asarray(lengths, np.int32)
    out, newpool = oracle.recurrent_step(q, k, v, beta, g, None, pool, idx, L, None, scale)
    untouched = [s for s in range(slots) if s not in set(perm.tolist())]
    assert np.array_equal(newpool[untouched], pool[untouched])
    return out, newpool[perm]


@pytest.mark.parametrize("check", _pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_decode_oracle_pin(check):
    check(decode_as_chunk)


@pytest.mark.parametrize("check", _decode_pins.DECODE_CHECKS, ids=lambda c: c.__name__)
def test_decode_feature_pin(check):
    """The slot pool, the per-key gate, the accepted counts and the speculative reading (tests/_decode_pins)."""
    check(oracle.recurrent_step)


def test_prologue_values():
    with open(os.path.join(_pins.GOLDEN, "prologue_values.json")) as f:
        c = json.load(f)
    for case in c["l2norm"]:
        x = np.asarray(case["x"], np.float64)
        r = oracle.prologue(q=x[None, None, None], eps=case["eps"])["q_hat"][0, 0, 0]
        assert np.allclose(r, case["expected"], atol=1e-15, rtol=0)
    for case in c["sigmoid"]:
        r = oracle.prologue(b=np.array([[[case["b"]]]]))["beta"][0, 0, 0]
        assert abs(r - case["expected"]) < 1e-15
    for case in c["gate"]:
        r = oracle.prologue(a=np.array([[[case["a"]]]]), A_log=np.array([case["A_log"]]),
                            dt_bias=np.array([case["dt_bias"]]))["g"][0, 0, 0]
        assert abs(r - case["expected"]) <= 1e-15 * max(1.0, abs(case["expected"])), (case, r)


def test_prologue_shapes_and_heads():
    """A_log and dt_bias are per value head; l2norm acts on the last axis only."""
    rng = np.random.default_rng(3)
    a = rng.normal(size=(2, 3, 4))
    A_log = np.array([0.0, 1.0, 2.0])
    dtb = np.array([-1.0, 0.0, 0.5])
    g = oracle.prologue(a=a, A_log=A_log, dt_bias=dtb)["g"]
    z = a + dtb[None, :, None]
    ref = -np.exp(A_log)[None, :, None] * np.log1p(np.exp(z))
    assert np.allclose(g, ref, atol=1e-14, rtol=1e-14)
    q = rng.normal(size=(2, 2, 5, 7))
    qh = oracle.prologue(q=q)["q_hat"]
    assert np.allclose((qh * qh).sum(-1), (q * q).sum(-1) / ((q * q).sum(-1) + 1e-6), atol=1e-14)


def test_tiny_decode_chain_equals_prefill():
    """The tiny fp32 workload: 8 decode calls of 8 tokens through a one-slot
    pool reproduce one prefill over the 64 tokens (recurrent and chunked calls
    share one state)."""
    w = workloads.generate("tiny")
    pro = oracle.prologue(q=w.q, k=w.k, b=w.b)
    out, fin = oracle.chunk_fwd(pro["q_hat"], pro["k_hat"], w.v, pro["beta"], w.g, None, None, w.scale)
    pool = np.zeros((1, w.Nv, w.Dk, w.Dv))
    outs = []
    for c in range(8):
        sl = slice(8 * c, 8 * c + 8)
        o, pool = oracle.recurrent_step(pro["q_hat"][:, :, sl], pro["k_hat"][:, :, sl], w.v[:, :, sl],
                                        pro["beta"][:, :, sl], w.g[:, :, sl], None, pool,
                                        np.zeros(8, np.int32), np.array([8], np.int32), None, w.scale)
        outs.append(o)
    assert np.allclose(np.concatenate(outs, axis=2), out, atol=1e-13, rtol=0)
    assert np.allclose(pool[0], fin[0], atol=1e-13, rtol=0)


def test_named_workloads_chunked_form_small():
    """Each named workload shape family, shrunk, agrees with the chunked WY form
    (strong gates included: g down to about -20 per token)."""
    for name in ("tiny", "prefill", "varlen"):
        w = workloads.generate(name, B=2, S=70, Nk=2, Nv=4, D=8)
        pro = oracle.prologue(q=w.q, k=w.k, b=w.b, a=w.a, A_log=w.A_log, dt_bias=w.dt_bias)
        g = pro.get("g", w.g)
        L = w.lengths.copy()
        if name == "varlen":
            L = np.array([70, 33], np.int32)
        out, fin = oracle.chunk_fwd(pro["q_hat"], pro["k_hat"], w.v, pro["beta"], g, w.initial_state, L, w.scale)
        for b in range(w.B):
            for h in range(w.Nv):
                kh = h // (w.Nv // w.Nk)
                n = int(L[b])
                S0 = w.initial_state[b, h] if w.initial_state is not None else np.zeros((w.Dk, w.Dv))
                o2, S2 = _pins.forms.chunked_wy(w.scale * pro["q_hat"][b, kh, :n], pro["k_hat"][b, kh, :n],
                                                w.v[b, h, :n], pro["beta"][b, h, :n], g[b, h, :n], S0, 64)
                assert np.allclose(out[b, h, :n], o2, atol=1e-10, rtol=0)
                assert np.allclose(fin[b, h], S2, atol=1e-10, rtol=0)
                assert np.all(out[b, h, n:] == 0.0)


def test_oracle_rejects_bad_arguments():
    q = np.zeros((1, 2, 4, 3))
    v = np.zeros((1, 3, 4, 3))
    with pytest.raises(ValueError):
        oracle.chunk_fwd(q, q, v, np.zeros((1, 3, 4)))  # Nv % Nk != 0
    with pytest.raises(ValueError):
        oracle.chunk_fwd(q[:, :1], q[:, :1], v[:, :1], np.zeros((1, 1, 4)), actual_seq_lengths=[5])
    with pytest.raises(ValueError):
        oracle.recurrent_step(q[:, :1], q[:, :1], v[:, :1], np.zeros((1, 1, 4)), None, None,
                              np.zeros((2, 1, 3, 3)), np.array([2, 0, 0, 0], np.int32), np.array([4], np.int32))


def test_oracle_is_thread_count_independent():
    w = workloads.generate("prefill", B=2, S=33, Nk=2, Nv=4, D=8)
    pro = oracle.prologue(q=w.q, k=w.k, b=w.b, a=w.a, A_log=w.A_log, dt_bias=w.dt_bias)
    args = (pro["q_hat"], pro["k_hat"], w.v, pro["beta"], pro["g"], w.initial_state, None, w.scale)
    o1, f1 = oracle.chunk_fwd(*args)
    o2, f2 = oracle.chunk_fwd(*args)
    assert np.array_equal(o1, o2) and np.array_equal(f1, f2)
    assert oracle.threads() >= 1
    assert math.isfinite(float(np.abs(o1).max()))



@pytest.mark.parametrize("check", _pins.EPILOGUE_CHECKS, ids=lambda c: c.__name__)
def test_gated_rmsnorm_oracle_pin(check):
    check(oracle.gated_rmsnorm)


def conv_impl(x, w, bias, state, lengths):
    return oracle.causal_conv1d(x, w, bias, state, lengths)


@pytest.mark.parametrize("check", _pins.CONV_CHECKS, ids=lambda c: c.__name__)
def test_causal_conv1d_oracle_pin(check):
    check(conv_impl)


# ---- the speculative-decoding reading of num_accepted_tokens (per-token state slots) ----

def _spec_case(seed, B=3, S=4, Nk=2, Nv=4, D=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Nk, S, D))
    k = rng.standard_normal((B, Nk, S, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, Nv, S, D))
    beta = rng.uniform(0.1, 0.9, (B, Nv, S))
    g = np.log(rng.uniform(0.8, 0.99, (B, Nv, S)))
    return q, k, v, beta, g


def test_spec_reading_rejects_accepted_outside_range():
    q, k, v, beta, g = _spec_case(36, B=1)
    pool = np.zeros((4, 4, 8, 8))
    idx = np.arange(4, dtype=np.int32)
    for A in (0, 5):
        with pytest.raises(ValueError):
            oracle.recurrent_step(q, k, v, beta, g, None, pool, idx, np.array([4], np.int32),
                                  np.array([A], np.int32), 0.5, per_token=True)
