"""Pins of the decode call's own features, as checks on any implementation.

`dec` has the signature of oracle.recurrent_step: (q, k, v, beta, g, gk, pool, indices, lengths, accepted,
scale, per_token=False) -> (out, new_pool).  The features are those of the recurrent_gated_delta_rule page
(lite_boost): a pool of state slots gathered by ssm_state_indices, the per-key gate gk (the state decays by
exp(g) * exp(gk) per key row), num_accepted_tokens, and the speculative-decoding reading of it.  The expected
values come from closed forms and from the prefill oracle, oracle.chunk_fwd, which the checks in _pins tie to
the pages on their own; none comes from `dec` itself, except where two readings must agree.
"""
import numpy as np

import oracle


def _case(seed, B, Nk, Nv, S, D, unit_k=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Nk, S, D))
    k = rng.standard_normal((B, Nk, S, D))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, Nv, S, D))
    beta = rng.uniform(0.1, 0.9, (B, Nv, S))
    g = np.log(rng.uniform(0.8, 0.99, (B, Nv, S)))
    return rng, q, k, v, beta, g


def check_dec_gk_closed_form(dec):
    """beta = 0 with a per-key gate: row i of the state decays by exp(G_t + GK_t[i]) (cumulative sums), so
    o_t = sum_i x_i exp(G_t + GK_t[i]) S0[i, :] and the slot receives exp(G_L + GK_L) * S0 row by row; the other
    slot is untouched."""
    rng = np.random.default_rng(30)
    S, Dk, Dv = 5, 4, 3
    q = rng.normal(size=(1, 1, S, Dk))
    k = rng.normal(size=(1, 1, S, Dk))
    v = rng.normal(size=(1, 1, S, Dv))
    g = np.log(rng.uniform(0.7, 0.99, size=(1, 1, S)))
    gk = np.log(rng.uniform(0.8, 0.999, size=(1, 1, S, Dk)))
    pool = rng.normal(size=(2, 1, Dk, Dv))
    idx = np.array([1] * S, np.int32)
    out, newpool = dec(q, k, v, np.zeros((1, 1, S)), g, gk, pool, idx, np.array([S], np.int32), None, 0.5)
    G = np.cumsum(g[0, 0])
    GK = np.cumsum(gk[0, 0], axis=0)
    for t in range(S):
        assert np.allclose(out[0, 0, t], (0.5 * q[0, 0, t] * np.exp(G[t] + GK[t])) @ pool[1, 0], atol=1e-13, rtol=0)
    assert np.allclose(newpool[1, 0], np.exp(G[-1] + GK[-1])[:, None] * pool[1, 0], atol=1e-13, rtol=0)
    assert np.array_equal(newpool[0], pool[0])


def check_dec_gk_uniform_equals_g(dec):
    """A per-key gate with the same value c on every key row is the scalar gate c: (g, gk = c) gives what
    (g + c, no gk) gives, with beta > 0, so the decay must come before the readout k^T S."""
    rng, q, k, v, beta, g = _case(37, 1, 1, 1, 5, 4)
    pool = rng.standard_normal((2, 1, 4, 4))
    idx = np.array([1] * 5, np.int32)
    L = np.array([5], np.int32)
    c = np.log(rng.uniform(0.8, 0.99, size=(1, 1, 5)))
    o1, p1 = dec(q, k, v, beta, g, np.repeat(c[..., None], 4, -1), pool, idx, L, None, 1.0)
    o2, p2 = dec(q, k, v, beta, g + c, None, pool, idx, L, None, 1.0)
    assert np.allclose(o1, o2, atol=1e-13, rtol=0) and np.allclose(p1, p2, atol=1e-13, rtol=0)


def check_dec_accepted(dec):
    """One slot per sequence (GQA, 2 key heads and 4 value heads): every one of the L tokens is output (the
    prefill oracle's outputs from the slot's state), rows t >= L are zero, the slot receives the state after
    min(A, L) tokens (the prefill oracle's final state over them), A = 0 leaves it untouched, and so do
    sequences of length 0 and unreferenced slots."""
    rng, q, k, v, beta, g = _case(31, 5, 2, 4, 4, 5)
    slots = 8
    pool = rng.standard_normal((slots, 4, 5, 5))
    seq_slot = np.array([6, 2, 0, 5, 3], np.int32)
    idx = np.repeat(seq_slot, 4).astype(np.int32)
    L = np.array([4, 3, 2, 4, 0], np.int32)
    A = np.array([2, 3, 1, 0, 2], np.int32)
    out, newpool = dec(q, k, v, beta, g, None, pool, idx, L, A, 0.5)
    for b in range(5):
        s, Lb, Ab = int(seq_slot[b]), int(L[b]), int(A[b])
        assert np.all(out[b, :, Lb:] == 0.0)
        sl = slice(b, b + 1)
        if Lb > 0:
            o_ref, _ = oracle.chunk_fwd(q[sl, :, :Lb], k[sl, :, :Lb], v[sl, :, :Lb], beta[sl, :, :Lb], g[sl, :, :Lb],
                                        pool[s][None], None, 0.5)
            assert np.allclose(out[b, :, :Lb], o_ref[0], atol=1e-12, rtol=0)
        n = min(Ab, Lb)
        if n == 0:
            assert np.array_equal(newpool[s], pool[s])
        else:
            _, f_ref = oracle.chunk_fwd(q[sl, :, :n], k[sl, :, :n], v[sl, :, :n], beta[sl, :, :n], g[sl, :, :n],
                                        pool[s][None], None, 0.5)
            assert np.allclose(newpool[s], f_ref[0], atol=1e-12, rtol=0)
    for s in (1, 4, 7):
        assert np.array_equal(newpool[s], pool[s])


def check_dec_token_slots(dec):
    """One slot per token, committing reading: the chain starts from slot indices[b*S]; the state after token
    t goes to slot indices[b*S + t] when t < A; the slots of tokens t >= A keep their values."""
    rng, q, k, v, beta, g = _case(32, 2, 1, 2, 3, 4)
    pool = rng.standard_normal((8, 2, 4, 4))
    idx = np.array([7, 1, 4, 2, 6, 0], np.int32)
    L = np.array([3, 3], np.int32)
    A = np.array([3, 2], np.int32)
    out, newpool = dec(q, k, v, beta, g, None, pool, idx, L, A, 0.5)
    for b in range(2):
        sl = slice(b, b + 1)
        S0 = pool[idx[3 * b]][None]
        for t in range(3):
            slot = idx[3 * b + t]
            if t < A[b]:
                _, f = oracle.chunk_fwd(q[sl, :, :t + 1], k[sl, :, :t + 1], v[sl, :, :t + 1], beta[sl, :, :t + 1],
                                        g[sl, :, :t + 1], S0, None, 0.5)
                assert np.allclose(newpool[slot], f[0], atol=1e-12, rtol=0)
            elif slot != idx[3 * b]:
                assert np.array_equal(newpool[slot], pool[slot])
    for s in (3, 5):
        assert np.array_equal(newpool[s], pool[s])


def check_dec_spec_one_accepted(dec):
    """Speculative reading with A = 1 starts from the slot of token 0, as the committing reading does; with
    every token committed both write the same states to the same per-token slots."""
    rng, q, k, v, beta, g = _case(33, 3, 2, 4, 4, 8)
    pool = rng.standard_normal((14, 4, 8, 8))
    idx = rng.permutation(14)[:12].astype(np.int32)
    L = np.array([4, 2, 3], np.int32)
    o1, p1 = dec(q, k, v, beta, g, None, pool, idx, L, np.ones(3, np.int32), 0.5, per_token=True)
    o2, p2 = dec(q, k, v, beta, g, None, pool, idx, L, L, 0.5)
    assert np.allclose(o1, o2, atol=1e-13, rtol=0) and np.allclose(p1, p2, atol=1e-13, rtol=0)


def check_dec_spec_two_steps(dec):
    """Step 1 verifies 4 draft tokens from slot s0 and writes each token's state to its own slot; 2 are
    accepted.  Step 2 starts from the state after the second token (the slot of token A - 1) and processes 4
    new tokens: its outputs and last state equal the prefill oracle's chain over x1, x2, y1..y4."""
    _, q1, k1, v1, b1, g1 = _case(34, 1, 2, 4, 4, 8)
    _, q2, k2, v2, b2, g2 = _case(35, 1, 2, 4, 4, 8)
    rng = np.random.default_rng(36)
    pool = rng.standard_normal((6, 4, 8, 8))
    slots = np.array([5, 1, 3, 0], np.int32)
    one = np.array([4], np.int32)
    _, p1 = dec(q1, k1, v1, b1, g1, None, pool, slots, one, np.array([1], np.int32), 0.5, per_token=True)
    A = 2
    o2, p2 = dec(q2, k2, v2, b2, g2, None, p1, slots, one, np.array([A], np.int32), 0.5, per_token=True)
    cat = lambda a1, a2: np.concatenate([a1[:, :, :A], a2], axis=2)
    oc, fc = oracle.chunk_fwd(cat(q1, q2), cat(k1, k2), cat(v1, v2), cat(b1, b2), cat(g1, g2), pool[slots[0]][None],
                              None, 0.5)
    assert np.allclose(o2, oc[:, :, A:], rtol=1e-12, atol=1e-12)
    assert np.allclose(p2[slots[3]], fc[0], rtol=1e-12, atol=1e-12)
    assert np.array_equal(p2[[2, 4]], pool[[2, 4]])


DECODE_CHECKS = [check_dec_gk_closed_form, check_dec_gk_uniform_equals_g, check_dec_accepted, check_dec_token_slots,
                 check_dec_spec_one_accepted, check_dec_spec_two_steps]
