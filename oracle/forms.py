"""Independent fp64 formulations of the gated delta rule -- TEST INFRASTRUCTURE.

Each function restates, in numpy, a DIFFERENT way the pages compute the same
thing as the token-by-token oracle in ``gdr_oracle.c``.  Agreement between
these and the C oracle (to ~1e-12) is one of the pins on the oracle: a dropped
term, a wrong sign, a swapped index or a transposed operand in either shows
up as a disagreement.  Only tests import this module.

Shapes follow one (batch, value-head) chain unless stated: q, k (L, Dk),
v (L, Dv), beta (L,), g (L,) log-decay, S0 (Dk, Dv).  ``q`` is the query
already multiplied by the scale.
"""
from __future__ import annotations

import numpy as np


def matrix_form_step(S, q, k, v, beta, g):
    """One token written as a single matrix expression:
    S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T,  o_t = S_t^T q.

    Source: the gated form in the docstring of ssm_lab.py delta_rule_recurrent
    (semidirectx lecture21 page, linear-attention section) and the comment
    block in torch_recurrent_gated_delta_rule (blog page).
    """
    Dk = S.shape[0]
    alpha = np.exp(g)
    S_new = alpha * (np.eye(Dk) - beta * np.outer(k, k)) @ S + beta * np.outer(k, v)
    return S_new, S_new.T @ q


def teaching_form_step(S, q, k, v, beta, g):
    """ssm_lab.py delta_rule_recurrent's update:
    S = alpha * (S - beta * k (S^T k)^T) + beta * k v^T, o = S^T q."""
    alpha = np.exp(g)
    S_new = alpha * (S - beta * np.outer(k, S.T @ k)) + beta * np.outer(k, v)
    return S_new, S_new.T @ q


def chunked_wy(q, k, v, beta, g, S0, C: int):
    """Chunked (WY / UT-transform) form of one chain, chunk size C.

    Restates the algorithm of torch_chunk_gated_delta_rule (blog page,
    steps 1-8) in fp64: pad to a multiple of C, cumulative log-gate per chunk,
    decay ratios exp(G_t - G_s) taken in log space, the strictly-lower matrix
    A = beta_t (k_t . k_s) exp(G_t - G_s), T = (I + A)^{-1} (here by a library
    inverse, the definition), U = T diag(beta) V, W = T diag(beta e^G) K, then
    the sequential inter-chunk carry
        v_new = U - W S,
        o     = (e^G * Q) S + (Q K^T * decay, causal incl. diagonal) v_new,
        S     = e^{G_last} S + (e^{G_last - G} * K)^T v_new.
    Returns (o (L, Dv), S_final).
    """
    L, Dk = k.shape
    Dv = v.shape[1]
    pad = (-L) % C
    qp = np.concatenate([q, np.zeros((pad, Dk))])
    kp = np.concatenate([k, np.zeros((pad, Dk))])
    vp = np.concatenate([v, np.zeros((pad, Dv))])
    bp = np.concatenate([beta, np.zeros(pad)])
    gp = np.concatenate([g, np.zeros(pad)])
    S = S0.copy()
    out = np.zeros((L + pad, Dv))
    lower_strict = np.tril(np.ones((C, C)), -1)
    lower_incl = np.tril(np.ones((C, C)), 0)
    for c0 in range(0, L + pad, C):
        sl = slice(c0, c0 + C)
        Q, K, V, be = qp[sl], kp[sl], vp[sl], bp[sl]
        G = np.cumsum(gp[sl])
        diff = G[:, None] - G[None, :]
        # exp only where t >= s, so that large positive differences never reach exp
        ratio = np.where(lower_incl > 0, np.exp(np.where(lower_incl > 0, diff, 0.0)), 0.0)
        A = (be[:, None] * (K @ K.T)) * ratio * lower_strict
        T = np.linalg.inv(np.eye(C) + A)
        U = T @ (be[:, None] * V)
        W = T @ ((be * np.exp(G))[:, None] * K)
        v_new = U - W @ S
        o = (np.exp(G)[:, None] * Q) @ S + ((Q @ K.T) * ratio) @ v_new
        out[sl] = o
        S = np.exp(G[-1]) * S + (np.exp(G[-1] - G)[:, None] * K).T @ v_new
    return out[:L], S


def pseudo_value(q, k, v, beta, g, S0, C: int):
    """Pseudo-value form of one chain, chunk size C.

    Restates the derivation in deltanet.rs (core_chunk docstring): with
    cumulative in-chunk decay Gamma_r, pseudo-values
        u_r = beta_r (v_r - Gamma_r S0^T k_r - sum_{i<r} (Gamma_r/Gamma_i)(k_i.k_r) u_i),
    outputs o_r = Gamma_r S0^T q_r + sum_{i<=r} (Gamma_r/Gamma_i)(k_i.q_r) u_i and the
    boundary state S_C = Gamma_C S0 + sum_i (Gamma_C/Gamma_i) k_i u_i^T, ratios taken in
    log space.  Returns (o (L, Dv), S_final).
    """
    L = k.shape[0]
    S = S0.copy()
    out = np.zeros((L, v.shape[1]))
    for c0 in range(0, L, C):
        idx = range(c0, min(c0 + C, L))
        lg = np.cumsum(g[c0:c0 + len(idx)])
        us = []
        for r_local, r in enumerate(idx):
            u = v[r] - np.exp(lg[r_local]) * (S.T @ k[r])
            for i_local in range(r_local):
                i = c0 + i_local
                u = u - np.exp(lg[r_local] - lg[i_local]) * (k[i] @ k[r]) * us[i_local]
            us.append(beta[r] * u)
        for r_local, r in enumerate(idx):
            o = np.exp(lg[r_local]) * (S.T @ q[r])
            for i_local in range(r_local + 1):
                i = c0 + i_local
                o = o + np.exp(lg[r_local] - lg[i_local]) * (k[i] @ q[r]) * us[i_local]
            out[r] = o
        last = lg[-1]
        S_new = np.exp(last) * S
        for i_local in range(len(idx)):
            i = c0 + i_local
            S_new = S_new + np.exp(last - lg[i_local]) * np.outer(k[i], us[i_local])
        S = S_new
    return out, S


def gla_parallel(q, k, v, g):
    """Gated linear attention by brute force, O(L^2):
    o_t = sum_{s<=t} exp(G_t - G_s) (q_t . k_s) v_s with G the cumulative log-gate.

    This is the masked parallel form of ssm_lab.py linear_attention_parallel
    (semidirectx lecture21 page) with an input-dependent gate; it equals the
    recurrence S_t = alpha_t S_{t-1} + k_t v_t^T, o_t = S_t^T q_t.
    """
    L = q.shape[0]
    G = np.cumsum(g)
    out = np.zeros((L, v.shape[1]))
    for t in range(L):
        for s in range(t + 1):
            out[t] += np.exp(G[t] - G[s]) * (q[t] @ k[s]) * v[s]
    return out
