"""The oracle against what the pages and the mathematics fix (CPU only)."""
import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads
from tests import _pins


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


def test_decode_gk_closed_form():
    """beta = 0 with a per-key gate: row i of the state decays by
    exp(sum g + sum gk_i), so o_t = sum_i x_i exp(G_t + GK_t[i]) S0[i, :]
    (lite_boost recurrent op: S = S * exp(g) * exp(gk))."""
    rng = np.random.default_rng(30)
    S, Dk, Dv = 5, 4, 3
    q = rng.normal(size=(1, 1, S, Dk))
    k = rng.normal(size=(1, 1, S, Dk))
    v = rng.normal(size=(1, 1, S, Dv))
    g = np.log(rng.uniform(0.7, 0.99, size=(1, 1, S)))
    gk = np.log(rng.uniform(0.8, 0.999, size=(1, 1, S, Dk)))
    pool = rng.normal(size=(2, 1, Dk, Dv))
    idx = np.array([1] * S, np.int32)
    out, newpool = oracle.recurrent_step(q, k, v, np.zeros((1, 1, S)), g, gk, pool, idx, np.array([S], np.int32),
                                         None, 0.5)
    G = np.cumsum(g[0, 0])
    GK = np.cumsum(gk[0, 0], axis=0)
    for t in range(S):
        dec = np.exp(G[t] + GK[t])
        assert np.allclose(out[0, 0, t], (0.5 * q[0, 0, t] * dec) @ pool[1, 0], atol=1e-13, rtol=0)
    assert np.allclose(newpool[1, 0], np.exp(G[-1] + GK[-1])[:, None] * pool[1, 0], atol=1e-13, rtol=0)
    assert np.array_equal(newpool[0], pool[0])
    # a per-key gate equal on every row is the same as adding it to g
    c = np.log(rng.uniform(0.8, 0.99, size=(1, 1, S)))
    beta = rng.uniform(size=(1, 1, S))
    o1, p1 = oracle.recurrent_step(q, k, v, beta, g, np.repeat(c[..., None], Dk, -1), pool, idx,
                                   np.array([S], np.int32), None, 1.0)
    o2, p2 = oracle.recurrent_step(q, k, v, beta, g + c, None, pool, idx, np.array([S], np.int32), None, 1.0)
    assert np.allclose(o1, o2, atol=1e-13, rtol=0) and np.allclose(p1, p2, atol=1e-13, rtol=0)


def test_decode_accepted_tokens():
    """All L tokens are output; the slot receives the state after min(A, L)
    tokens (reading of num_accepted_tokens); A = 0 leaves the slot untouched."""
    w = workloads.random_case(B=4, Nk=1, Nv=2, S=4, Dk=5, Dv=3, seed=31, slots=6, initial_state=False)
    w.lengths = np.array([4, 3, 2, 4], np.int32)
    w.accepted = np.array([2, 3, 1, 0], np.int32)
    pro = oracle.prologue(q=w.q, k=w.k, b=w.b)
    args = (pro["q_hat"], pro["k_hat"], w.v, pro["beta"], w.g)
    out, pool = oracle.recurrent_step(*args, None, w.pool, w.indices, w.lengths, w.accepted, w.scale)
    for b in range(w.B):
        slot = w.indices[b * w.S]
        S0 = w.pool[slot][None]
        L, A = int(w.lengths[b]), int(w.accepted[b])
        sl = (slice(b, b + 1),)
        o_full, _ = oracle.chunk_fwd(*(x[sl][:, :, :L] for x in args), S0, None, w.scale)
        assert np.allclose(out[b, :, :L], o_full[0], atol=1e-13, rtol=0)
        assert np.all(out[b, :, L:] == 0.0)
        if A == 0:
            assert np.array_equal(pool[slot], w.pool[slot])
        else:
            _, f_acc = oracle.chunk_fwd(*(x[sl][:, :, :A] for x in args), S0, None, w.scale)
            assert np.allclose(pool[slot], f_acc[0], atol=1e-13, rtol=0)
    used = set(w.indices.tolist())
    for s in range(6):
        if s not in used:
            assert np.array_equal(pool[s], w.pool[s])


def test_decode_distinct_token_slots():
    """With one slot per token, the state after token t goes to slot
    indices[b*S + t] for t < A; the chain starts from indices[b*S]."""
    w = workloads.random_case(B=2, Nk=1, Nv=1, S=3, Dk=4, Dv=4, seed=32, slots=8, share_slot=False,
                              initial_state=False)
    w.accepted = np.array([3, 2], np.int32)
    pro = oracle.prologue(q=w.q, k=w.k, b=w.b)
    args = (pro["q_hat"], pro["k_hat"], w.v, pro["beta"], w.g)
    out, pool = oracle.recurrent_step(*args, None, w.pool, w.indices, w.lengths, w.accepted, w.scale)
    for b in range(2):
        S0 = w.pool[w.indices[b * 3]][None]
        for t in range(3):
            slot = w.indices[b * 3 + t]
            if t < w.accepted[b]:
                _, f = oracle.chunk_fwd(*(x[b:b + 1, :, :t + 1] for x in args), S0, None, w.scale)
                assert np.allclose(pool[slot], f[0], atol=1e-13, rtol=0)
            else:
                assert np.array_equal(pool[slot], w.pool[slot])


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


def test_spec_reading_with_one_accepted_equals_committing_every_token():
    """A = 1 starts from the slot of token 0, as the other reading does; with every token committed both
    write the same states to the same per-token slots."""
    q, k, v, beta, g = _spec_case(31)
    B, S = q.shape[0], q.shape[2]
    rng = np.random.default_rng(32)
    pool = rng.standard_normal((B * S + 2, 4, 8, 8))
    idx = rng.permutation(B * S + 2)[:B * S].astype(np.int32)
    L = np.array([4, 2, 3], np.int32)
    o1, p1 = oracle.recurrent_step(q, k, v, beta, g, None, pool, idx, L, np.ones(B, np.int32), 0.5, per_token=True)
    o2, p2 = oracle.recurrent_step(q, k, v, beta, g, None, pool, idx, L, L, 0.5)
    assert np.array_equal(o1, o2) and np.array_equal(p1, p2)


def test_spec_two_steps_equal_the_chain_over_accepted_tokens():
    """Step 1 verifies 4 draft tokens from slot s0 and writes each token's state to its own slot; 2 are
    accepted.  Step 2 starts from the state after the second token (slot of token A - 1) and processes 4
    new tokens: its outputs and states equal the prefill oracle's chain over x1, x2, y1..y4."""
    q1, k1, v1, b1, g1 = _spec_case(33, B=1)
    q2, k2, v2, b2, g2 = _spec_case(34, B=1)
    S = 4
    rng = np.random.default_rng(35)
    pool = rng.standard_normal((6, 4, 8, 8))
    slots = np.array([5, 1, 3, 0], np.int32)
    _, p1 = oracle.recurrent_step(q1, k1, v1, b1, g1, None, pool, slots, np.array([S], np.int32),
                                  np.array([1], np.int32), 0.5, per_token=True)
    A = 2
    o2, p2 = oracle.recurrent_step(q2, k2, v2, b2, g2, None, p1, slots, np.array([S], np.int32),
                                   np.array([A], np.int32), 0.5, per_token=True)
    cat = lambda a1, a2: np.concatenate([a1[:, :, :A], a2], axis=2)
    s0 = pool[slots[0]][None]  # the chain's state before x1
    oc, fc = oracle.chunk_fwd(cat(q1, q2), cat(k1, k2), cat(v1, v2), cat(b1, b2), cat(g1, g2), s0, None, 0.5)
    assert np.allclose(o2, oc[:, :, A:], rtol=1e-12, atol=1e-12)
    assert np.allclose(p2[slots[S - 1]], fc[0], rtol=1e-12, atol=1e-12)
    untouched = [s for s in range(6) if s not in slots]
    assert np.array_equal(p2[untouched], pool[untouched])


def test_spec_reading_rejects_accepted_outside_range():
    q, k, v, beta, g = _spec_case(36, B=1)
    pool = np.zeros((4, 4, 8, 8))
    idx = np.arange(4, dtype=np.int32)
    for A in (0, 5):
        with pytest.raises(ValueError):
            oracle.recurrent_step(q, k, v, beta, g, None, pool, idx, np.array([4], np.int32),
                                  np.array([A], np.int32), 0.5, per_token=True)
