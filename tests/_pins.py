"""Pins on the oracle: checks against facts the pages and the mathematics fix.

Each check takes an implementation of the chunked-prefill semantics,
``impl(q, k, v, beta, g, S0, lengths, scale) -> (out, final_state)`` over
BNSD fp64 arrays, and raises AssertionError when the implementation breaks
the fact.  ``test_oracle_pins.py`` runs every check on the C oracle;
``test_pin_sensitivity.py`` runs them on copies of the rule with a planted
mistake (on the CPU) and requires each mistake to be caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import forms

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _one(x):
    """(L, D) -> (1, 1, L, D) or (L,) -> (1, 1, L)."""
    return np.asarray(x, np.float64)[None, None]


def _rand_chain(rng, L, Dk, Dv, unit_k=True):
    q = rng.normal(size=(L, Dk))
    k = rng.normal(size=(L, Dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        q /= np.linalg.norm(q, axis=1, keepdims=True)
    v = rng.normal(size=(L, Dv))
    beta = rng.uniform(0.05, 1.0, size=L)
    g = np.log(rng.uniform(0.5, 0.999, size=L))
    S0 = rng.normal(scale=0.3, size=(Dk, Dv))
    return q, k, v, beta, g, S0


def check_worked_examples(impl):
    """deltanet.rs unit tests: the hand-computed step and decay-before-readout."""
    for name in ("hand_step.json", "decay_first.json"):
        c = _golden(name)
        out, fin = impl(_one([c["q"]]), _one([c["k"]]), _one([c["v"]]), _one([c["beta"]]), _one([c["g"]]),
                        np.asarray(c["S0"], np.float64)[None, None], None, 1.0)
        assert np.allclose(out[0, 0, 0], c["expected_out"], atol=1e-12, rtol=0), (name, out[0, 0, 0])
        assert np.allclose(fin[0, 0], c["expected_state"], atol=1e-12, rtol=0), (name, fin[0, 0])


def check_matrix_form(impl):
    """beta = 1, g = 0 gives S' = (I - k k^T) S + k v^T (deltanet.rs unit test
    beta_one_reproduces_pure_delta_rule_matrix_form); for general beta, g the
    gated matrix expression of ssm_lab.py delta_rule_recurrent holds token by
    token."""
    rng = np.random.default_rng(11)
    Dk, Dv = 4, 3
    S0 = rng.normal(size=(Dk, Dv))
    k = rng.normal(size=Dk)
    k /= np.linalg.norm(k)
    v = rng.normal(size=Dv)
    q = rng.normal(size=Dk)
    out, fin = impl(_one([q]), _one([k]), _one([v]), _one([1.0]), _one([0.0]), S0[None, None], None, 1.0)
    expect = (np.eye(Dk) - np.outer(k, k)) @ S0 + np.outer(k, v)
    assert np.allclose(fin[0, 0], expect, atol=1e-12, rtol=0)
    assert np.allclose(out[0, 0, 0], expect.T @ q, atol=1e-12, rtol=0)
    # several tokens, general beta and gate
    q, k, v, beta, g, S0 = _rand_chain(rng, 9, 5, 4)
    out, fin = impl(_one(q), _one(k), _one(v), _one(beta), _one(g), S0[None, None], None, 1.0)
    S = S0.copy()
    for t in range(9):
        S, o = forms.matrix_form_step(S, q[t], k[t], v[t], beta[t], g[t])
        assert np.allclose(out[0, 0, t], o, atol=1e-12, rtol=0), t
    assert np.allclose(fin[0, 0], S, atol=1e-12, rtol=0)


def check_readback(impl):
    """beta = 1 with an exactly unit key: the readout k^T S' equals v."""
    rng = np.random.default_rng(12)
    Dk, Dv = 8, 6
    S0 = rng.normal(size=(Dk, Dv))
    k = rng.normal(size=Dk)
    k /= np.sqrt(k @ k)
    v = rng.normal(size=Dv)
    _, fin = impl(_one([k]), _one([k]), _one([v]), _one([1.0]), _one([0.0]), S0[None, None], None, 1.0)
    assert np.allclose(k @ fin[0, 0], v, atol=1e-12, rtol=0)


def check_beta_zero(impl):
    """beta = 0 writes nothing: o_t = exp(sum_{s<=t} g_s) (scale q_t)^T S0, and
    with g = -1 the state keeps e^-1 (about 37%) per step (lite_boost
    recurrent op, description of g)."""
    rng = np.random.default_rng(13)
    L, Dk, Dv = 7, 5, 3
    q, k, v, _, g, S0 = _rand_chain(rng, L, Dk, Dv)
    scale = 0.37
    out, fin = impl(_one(q), _one(k), _one(v), _one(np.zeros(L)), _one(g), S0[None, None], None, scale)
    G = np.cumsum(g)
    for t in range(L):
        assert np.allclose(out[0, 0, t], math.exp(G[t]) * (scale * q[t]) @ S0, atol=1e-12, rtol=0), t
    assert np.allclose(fin[0, 0], math.exp(G[-1]) * S0, atol=1e-12, rtol=0)
    _, fin = impl(_one(q), _one(k), _one(v), _one(np.zeros(L)), _one(-np.ones(L)), S0[None, None], None, 1.0)
    assert np.allclose(fin[0, 0], math.exp(-L) * S0, atol=1e-14, rtol=0)
    assert abs(math.exp(-1.0) - 0.3679) < 1e-4


def check_chunked_forms(impl):
    """The chunked WY form (blog page, torch_chunk_gated_delta_rule) and the
    pseudo-value form (deltanet.rs core_chunk) reach the same values, for
    several chunk sizes and a ragged tail."""
    rng = np.random.default_rng(14)
    L, Dk, Dv = 45, 6, 5
    q, k, v, beta, g, S0 = _rand_chain(rng, L, Dk, Dv)
    scale = 0.5
    out, fin = impl(_one(q), _one(k), _one(v), _one(beta), _one(g), S0[None, None], None, scale)
    for C in (1, 4, 16, 64):
        o2, S2 = forms.chunked_wy(scale * q, k, v, beta, g, S0, C)
        assert np.allclose(out[0, 0], o2, atol=1e-11, rtol=0), C
        assert np.allclose(fin[0, 0], S2, atol=1e-11, rtol=0), C
    for C in (1, 8, 64):
        o3, S3 = forms.pseudo_value(scale * q, k, v, beta, g, S0, C)
        assert np.allclose(out[0, 0], o3, atol=1e-11, rtol=0), C
        assert np.allclose(fin[0, 0], S3, atol=1e-11, rtol=0), C


def check_gla_orthogonal(impl):
    """Mutually orthogonal unit keys and S0 = 0: the erase term vanishes, so the
    rule is gated linear attention on values beta_t v_t, which the O(L^2)
    masked sum (ssm_lab.py linear_attention_parallel with a gate) gives."""
    rng = np.random.default_rng(15)
    L, Dk, Dv = 8, 8, 4
    Qm, _ = np.linalg.qr(rng.normal(size=(Dk, Dk)))
    k = Qm[:, :L].T.copy()
    q = rng.normal(size=(L, Dk))
    v = rng.normal(size=(L, Dv))
    beta = rng.uniform(0.1, 1.0, size=L)
    g = np.log(rng.uniform(0.6, 0.99, size=L))
    out, _ = impl(_one(q), _one(k), _one(v), _one(beta), _one(g), np.zeros((1, 1, Dk, Dv)), None, 1.0)
    ref = forms.gla_parallel(q, k, beta[:, None] * v, g)
    assert np.allclose(out[0, 0], ref, atol=1e-12, rtol=0)


def check_teaching_form(impl):
    """ssm_lab.py delta_rule_recurrent's written update, token by token."""
    rng = np.random.default_rng(16)
    q, k, v, beta, g, S0 = _rand_chain(rng, 11, 4, 4)
    out, fin = impl(_one(q), _one(k), _one(v), _one(beta), _one(g), S0[None, None], None, 1.0)
    S = S0.copy()
    for t in range(11):
        S, o = forms.teaching_form_step(S, q[t], k[t], v[t], beta[t], g[t])
        assert np.allclose(out[0, 0, t], o, atol=1e-12, rtol=0), t
    assert np.allclose(fin[0, 0], S, atol=1e-12, rtol=0)


def check_split_resume(impl):
    """Running L1 tokens, then L2 tokens from the returned state, equals one
    run of L1 + L2 (deltanet.rs: sequential and chunked calls interleave on one
    sequence; the state is the whole carry)."""
    rng = np.random.default_rng(17)
    L1, L2, Dk, Dv = 13, 20, 5, 4
    q, k, v, beta, g, S0 = _rand_chain(rng, L1 + L2, Dk, Dv)
    out, fin = impl(_one(q), _one(k), _one(v), _one(beta), _one(g), S0[None, None], None, 0.7)
    s1 = slice(0, L1)
    s2 = slice(L1, L1 + L2)
    o1, f1 = impl(_one(q[s1]), _one(k[s1]), _one(v[s1]), _one(beta[s1]), _one(g[s1]), S0[None, None], None, 0.7)
    o2, f2 = impl(_one(q[s2]), _one(k[s2]), _one(v[s2]), _one(beta[s2]), _one(g[s2]), f1, None, 0.7)
    assert np.allclose(out[0, 0, :L1], o1[0, 0], atol=1e-12, rtol=0)
    assert np.allclose(out[0, 0, L1:], o2[0, 0], atol=1e-12, rtol=0)
    assert np.allclose(fin, f2, atol=1e-12, rtol=0)


def check_gqa(impl):
    """Nv = 2 Nk: value head h reads key head h // 2 (repeat_interleave in the
    transformers layer); equal to a call with the key heads repeated."""
    rng = np.random.default_rng(18)
    B, Nk, Nv, L, D = 2, 2, 4, 6, 3
    q = rng.normal(size=(B, Nk, L, D))
    k = rng.normal(size=(B, Nk, L, D))
    v = rng.normal(size=(B, Nv, L, D))
    beta = rng.uniform(size=(B, Nv, L))
    g = np.log(rng.uniform(0.7, 0.99, size=(B, Nv, L)))
    S0 = rng.normal(size=(B, Nv, D, D))
    out, fin = impl(q, k, v, beta, g, S0, None, 1.0)
    out2, fin2 = impl(np.repeat(q, 2, axis=1), np.repeat(k, 2, axis=1), v, beta, g, S0, None, 1.0)
    assert np.allclose(out, out2, atol=1e-13, rtol=0)
    assert np.allclose(fin, fin2, atol=1e-13, rtol=0)
    # and a value head must not read the neighbouring group's key head
    out3, _ = impl(q[:, ::-1].copy(), k[:, ::-1].copy(), v, beta, g, S0, None, 1.0)
    assert not np.allclose(out, out3)


def check_padding(impl):
    """Rows t >= L_b are exactly zero; L_b = 0 returns the initial state
    unchanged (lite_boost chunk op, actual_seq_lengths and the zero padding);
    padding contents never influence valid rows."""
    rng = np.random.default_rng(19)
    B, N, S, D = 3, 1, 10, 4
    q = rng.normal(size=(B, N, S, D))
    k = rng.normal(size=(B, N, S, D))
    v = rng.normal(size=(B, N, S, D))
    beta = rng.uniform(size=(B, N, S))
    g = np.log(rng.uniform(0.7, 0.99, size=(B, N, S)))
    S0 = rng.normal(size=(B, N, D, D))
    L = np.array([10, 4, 0], np.int32)
    out, fin = impl(q, k, v, beta, g, S0, L, 1.0)
    assert np.all(out[1, :, 4:] == 0.0) and np.all(out[2] == 0.0)
    assert np.array_equal(fin[2], S0[2])
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[1, :, 4:] = 1e3
    k2[1, :, 4:] = -7.0
    v2[1, :, 4:] = 5.0
    out2, fin2 = impl(q2, k2, v2, beta, g, S0, L, 1.0)
    assert np.array_equal(out2[1], out[1]) and np.array_equal(fin2[1], fin[1])
    o1, f1 = impl(q[1:2, :, :4], k[1:2, :, :4], v[1:2, :, :4], beta[1:2, :, :4], g[1:2, :, :4], S0[1:2], None, 1.0)
    assert np.allclose(out[1, :, :4], o1[0], atol=1e-13, rtol=0)
    assert np.allclose(fin[1], f1[0], atol=1e-13, rtol=0)


def check_state_bounded(impl):
    """With unit keys, beta in [0, 1] and exp(g) <= 1 the update is a
    contraction plus a bounded write, so 200 random steps keep ||S|| small
    (deltanet.rs unit test state_norm_is_contractive_under_decay_and_bounded_beta,
    dk = dv = 8, bound 20)."""
    rng = np.random.default_rng(20)
    L, D = 200, 8
    q = rng.uniform(-0.5, 0.5, size=(L, D))
    k = rng.uniform(-0.5, 0.5, size=(L, D))
    q /= np.sqrt((q * q).sum(1, keepdims=True) + 1e-6)
    k /= np.sqrt((k * k).sum(1, keepdims=True) + 1e-6)
    v = rng.uniform(-0.5, 0.5, size=(L, D))
    z = rng.uniform(-2.0, 2.0, size=L)
    g = -(np.maximum(z, 0) + np.log1p(np.exp(-np.abs(z))))
    beta = 1.0 / (1.0 + np.exp(-rng.uniform(-2.0, 2.0, size=L)))
    peak = 0.0
    S = np.zeros((1, 1, D, D))
    for t in range(L):
        sl = slice(t, t + 1)
        _, S = impl(_one(q[sl]), _one(k[sl]), _one(v[sl]), _one(beta[sl]), _one(g[sl]), S, None, 1.0)
        n = float(np.sqrt((S * S).sum()))
        assert math.isfinite(n)
        peak = max(peak, n)
    assert peak < 20.0, peak
    # the contraction itself: one step with v = 0 never grows the norm
    S1 = rng.normal(size=(1, 1, D, D))
    _, S2 = impl(_one(q[:1]), _one(k[:1]), _one(np.zeros((1, D))), _one(beta[:1]), _one([0.0]), S1, None, 1.0)
    assert np.linalg.norm(S2) <= np.linalg.norm(S1) + 1e-12


def check_store_and_recall(impl):
    """Delta rule with beta = 1 and orthonormal keys, n <= d: reading key i
    back returns exactly v_i; rewriting the first keys with new values returns
    the new values (ssm_lab.py store_and_recall, rule "delta")."""
    rng = np.random.default_rng(21)
    d, n, rw = 8, 6, 2
    Kq, _ = np.linalg.qr(rng.normal(size=(d, d)))
    K = Kq[:, :n].T.copy()
    V = rng.normal(size=(n, d))
    Vn = rng.normal(size=(rw, d))
    keys = np.concatenate([K, K[:rw]])
    vals = np.concatenate([V, Vn])
    L = n + rw
    _, fin = impl(_one(keys), _one(keys), _one(vals), _one(np.ones(L)), _one(np.zeros(L)),
                  np.zeros((1, 1, d, d)), None, 1.0)
    R = K @ fin[0, 0]
    truth = V.copy()
    truth[:rw] = Vn
    assert np.allclose(R, truth, atol=1e-12, rtol=0)


ALL_CHECKS = [check_worked_examples, check_matrix_form, check_readback, check_beta_zero, check_chunked_forms,
              check_gla_orthogonal, check_teaching_form, check_split_resume, check_gqa, check_padding,
              check_state_bounded, check_store_and_recall]


# ---- the output epilogue: rmsnorm(o) * w * silu(z) ----

def check_epi_constant_row(impl):
    """o = 3 in every entry, eps = 16: the mean square is 9, so the row factor is 3/5 exactly;
    z = ln 3 gives sigmoid(z) = 3/4 and silu(z) = (3/4) ln 3 (a gate of sigmoid(z) would give 3/4)."""
    Dv = 8
    w = np.arange(1, Dv + 1, dtype=np.float64) * 0.5
    o = np.full((1, 2, 3, Dv), 3.0)
    z = np.full_like(o, math.log(3.0))
    got = impl(o, z, w, 16.0)
    want = 0.6 * 0.75 * math.log(3.0) * w
    assert np.allclose(got, np.broadcast_to(want, got.shape), rtol=0, atol=1e-15)


def check_epi_row_mean(impl):
    """One non-zero entry 3 in a row of Dv = 4 with eps = 3/4: mean square 9/4, plus eps = 3, so the
    entry becomes 3 / sqrt(3) = sqrt(3) (a sum instead of a mean would give 3 / sqrt(9.75))."""
    o = np.zeros((1, 1, 1, 4))
    o[..., 0] = 3.0
    z = np.full_like(o, 50.0)  # silu(50) = 50 to double precision
    got = impl(o, z, np.ones(4), 0.75)
    assert abs(got[0, 0, 0, 0] - math.sqrt(3.0) * 50.0) < 1e-12
    assert np.all(got[0, 0, 0, 1:] == 0.0)


def check_epi_invariants(impl):
    """z = 0 closes the gate exactly; with eps = 0 the result does not depend on the scale of o
    and is odd in o; with w = 1 and silu(z) = 1 the output row has mean square ms / (ms + eps)."""
    rng = np.random.default_rng(7)
    o = rng.standard_normal((2, 3, 5, 16))
    w = rng.uniform(0.5, 1.5, 16)
    z = rng.standard_normal(o.shape)
    assert np.all(impl(o, np.zeros_like(o), w, 1e-6) == 0.0)
    base = impl(o, z, w, 0.0)
    assert np.allclose(impl(7.5 * o, z, w, 0.0), base, rtol=1e-13, atol=0)
    assert np.allclose(impl(-o, z, w, 0.0), -base, rtol=1e-13, atol=0)
    # silu(z1) = 1 at the root of z = 1 + e^{-z}, found by bisection
    lo, hi = 1.0, 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        lo, hi = (mid, hi) if mid / (1.0 + math.exp(-mid)) < 1.0 else (lo, mid)
    eps = 0.3
    out = impl(o, np.full_like(o, lo), np.ones(16), eps)
    ms = np.mean(o * o, axis=-1)
    assert np.allclose(np.mean(out * out, axis=-1), ms / (ms + eps), rtol=1e-12, atol=0)


def check_epi_padding(impl):
    """Rows t >= L_b are passed through untouched (the calls keep them zero)."""
    rng = np.random.default_rng(8)
    o = rng.standard_normal((2, 1, 6, 8))
    z = rng.standard_normal(o.shape)
    got = impl(o, z, np.ones(8), 1e-6, np.array([4, 0]))
    assert np.array_equal(got[0, :, 4:], o[0, :, 4:]) and np.array_equal(got[1], o[1])
    assert not np.allclose(got[0, :, :4], o[0, :, :4])


EPILOGUE_CHECKS = [check_epi_constant_row, check_epi_row_mean, check_epi_invariants, check_epi_padding]


# ---- the depthwise causal conv1d + SiLU before the rule: impl(x, w, bias, state, lengths) -> (y, state) ----

def check_conv_special_taps(impl):
    """One-hot taps with inputs whose silu is exact: 0 (silu 0), ln 3 (silu = (3/4) ln 3) and 50 (silu = 50
    to double precision).  The newest tap passes x through; the oldest delays it by K - 1 positions, with
    the zero history in front."""
    K = 4
    vals = np.array([0.0, math.log(3.0), 50.0, 0.0, 50.0, math.log(3.0), 50.0])
    silu = {0.0: 0.0, math.log(3.0): 0.75 * math.log(3.0), 50.0: 50.0}
    x = vals.reshape(1, -1, 1)
    newest = np.zeros((1, K)); newest[0, K - 1] = 1.0
    y, _ = impl(x, newest, None, None, None)
    assert np.allclose(y[0, :, 0], [silu[v] for v in vals], rtol=0, atol=1e-14)
    oldest = np.zeros((1, K)); oldest[0, 0] = 1.0
    y, _ = impl(x, oldest, None, None, None)
    want = [0.0] * (K - 1) + [silu[v] for v in vals[:len(vals) - K + 1]]
    assert np.allclose(y[0, :, 0], want, rtol=0, atol=1e-14)


def check_conv_against_library_convolution(impl):
    """The pre-activation of every channel equals numpy's full convolution of the channel with its taps in
    reverse order (taps are stored oldest first), truncated to the sequence; checked through
    silu^-1 of the output on a monotone range (|pre| < 2 keeps silu invertible by bisection)."""
    rng = np.random.default_rng(21)
    B, S, C, K = 2, 19, 5, 4
    x = rng.uniform(-0.3, 0.3, (B, S, C))
    w = rng.uniform(-0.5, 0.5, (C, K))
    bias = rng.uniform(-0.2, 0.2, C)
    y, _ = impl(x, w, bias, None, None)
    for b in range(B):
        for c in range(C):
            pre = np.convolve(x[b, :, c], w[c, ::-1])[:S] + bias[c]
            lo, hi = np.full(S, -1.2), np.full(S, 2.0)  # silu is increasing on [-1.2, inf)
            for _ in range(80):
                mid = 0.5 * (lo + hi)
                f = mid / (1.0 + np.exp(-mid))
                lo, hi = np.where(f < y[b, :, c], mid, lo), np.where(f < y[b, :, c], hi, mid)
            assert np.allclose(lo, pre, rtol=0, atol=1e-12)


def check_conv_state_handoff(impl):
    """Running [0, s) and then [s, S) with the state carried equals one run over [0, S), for every split
    (s = 1, 2 and 3 are shorter than the window: the history then comes partly from the state), and the
    final state holds the last K inputs."""
    rng = np.random.default_rng(22)
    B, S, C, K = 2, 11, 3, 4
    x = rng.standard_normal((B, S, C))
    w = rng.standard_normal((C, K))
    bias = rng.standard_normal(C)
    s0 = rng.standard_normal((B, C, K))
    y_all, st_all = impl(x, w, bias, s0, None)
    assert np.array_equal(st_all, np.transpose(x[:, S - K:], (0, 2, 1)))
    for s in range(1, S):
        y1, st1 = impl(x[:, :s], w, bias, s0, None)
        y2, st2 = impl(x[:, s:], w, bias, st1, None)
        assert np.allclose(np.concatenate([y1, y2], 1), y_all, rtol=0, atol=1e-13)
        assert np.allclose(st2, st_all, rtol=0, atol=0)


def check_conv_lengths(impl):
    """Rows t >= L are zero and do not reach the state: L = 0 keeps the state, L = 1 shifts it by one, and a
    padded batch row equals the unpadded run."""
    rng = np.random.default_rng(23)
    B, S, C, K = 3, 7, 4, 3
    x = rng.standard_normal((B, S, C))
    w = rng.standard_normal((C, K))
    s0 = rng.standard_normal((B, C, K))
    L = np.array([0, 1, 5])
    y, st = impl(x, w, None, s0, L)
    assert np.all(y[0] == 0) and np.all(y[1, 1:] == 0) and np.all(y[2, 5:] == 0)
    assert np.array_equal(st[0], s0[0])
    assert np.array_equal(st[1], np.concatenate([s0[1][:, 1:], x[1, :1].T], axis=1))
    y2, st2 = impl(x[2:, :5], w, None, s0[2:], None)
    assert np.allclose(y[2, :5], y2[0], rtol=0, atol=1e-15) and np.array_equal(st[2], st2[0])


CONV_CHECKS = [check_conv_special_taps, check_conv_against_library_convolution, check_conv_state_handoff,
               check_conv_lengths]
