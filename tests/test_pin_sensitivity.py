"""The pins catch plausible mistakes.

A plain numpy copy of the token-by-token rule is run through every pin in
``_pins``: unmodified it must pass them all (so the harness itself is sound),
and with each planted mistake (a dropped term, a wrong sign, an operation in
the wrong order, a wrong head index, padding left dirty) at least one pin
must fail.  The same is done for the output epilogue, the causal conv1d and the decode call's own
features (slot pool, per-key gate, accepted counts, the speculative reading).  Everything here runs on the
CPU; nothing touches the CUDA path.
"""
import numpy as np
import pytest

from tests import _decode_pins, _pins


def make_impl(mutation=None):
    def impl(q, k, v, beta, g, S0, lengths, scale):
        q, k, v, beta = (np.asarray(x, np.float64) for x in (q, k, v, beta))
        B, Nk, S, Dk = q.shape
        Nv, Dv = v.shape[1], v.shape[3]
        grp = Nv // Nk
        out = np.zeros((B, Nv, S, Dv))
        fin = np.zeros((B, Nv, Dk, Dv))
        for b in range(B):
            L = S if lengths is None else int(lengths[b])
            for h in range(Nv):
                kh = (h % Nk) if mutation == "gqa_modulo" else h // grp
                St = np.zeros((Dk, Dv)) if S0 is None else np.array(S0[b, h], np.float64)
                for t in range(S):
                    if t >= L:
                        if mutation == "dirty_padding":
                            out[b, h, t] = 1.0
                        continue
                    x = q[b, kh, t] * (1.0 if mutation == "no_scale" else scale)
                    y = k[b, kh, t]
                    gt = 0.0 if g is None else float(g[b, h, t])
                    a = np.exp(-gt) if mutation == "gate_sign" else np.exp(gt)
                    if mutation != "decay_after_readout":
                        St = St * a
                    m = y @ St
                    if mutation == "decay_after_readout":
                        St = St * a
                    if mutation == "beta_on_v_only":
                        d = beta[b, h, t] * v[b, h, t] - m
                    else:
                        d = beta[b, h, t] * (v[b, h, t] - m)
                    if mutation == "output_before_write":
                        out[b, h, t] = x @ St
                    if mutation == "write_sign":
                        St = St - np.outer(y, d)
                    elif mutation == "write_uses_query":
                        St = St + np.outer(x / max(scale, 1e-300), d)
                    else:
                        St = St + np.outer(y, d)
                    if mutation != "output_before_write":
                        out[b, h, t] = x @ St
                fin[b, h] = St
        return out, fin
    return impl


MUTATIONS = ["decay_after_readout", "beta_on_v_only", "output_before_write", "write_sign", "write_uses_query",
             "gqa_modulo", "no_scale", "gate_sign", "dirty_padding"]


def test_unmodified_copy_passes_every_pin():
    impl = make_impl(None)
    for check in _pins.ALL_CHECKS:
        check(impl)


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_mistake_is_caught(mutation):
    impl = make_impl(mutation)
    failed = []
    for check in _pins.ALL_CHECKS:
        try:
            check(impl)
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {mutation!r}"


def make_epilogue(mutation=None):
    """A plain copy of rmsnorm(o) * w * silu(z) per row, with planted mistakes."""
    def impl(o, z, w, eps, lengths=None):
        o, z, w = (np.asarray(x, np.float64) for x in (o, z, w))
        B, S = o.shape[0], o.shape[2]
        out = o.copy()
        for b in range(B):
            L = S if lengths is None else int(lengths[b])
            for t in range(S if mutation == "epi_pads_too" else L):
                r = o[b, :, t]
                ms = np.sum(r * r, -1, keepdims=True) if mutation == "epi_sum" else np.mean(r * r, -1, keepdims=True)
                if mutation == "epi_eps_outside":
                    inv = 1.0 / np.sqrt(ms) + eps
                else:
                    inv = 1.0 / np.sqrt(ms + eps)
                zz = z[b, :, t]
                gate = 1.0 / (1.0 + np.exp(-zz)) if mutation == "epi_sigmoid" else zz / (1.0 + np.exp(-zz))
                wv = 1.0 if mutation == "epi_no_weight" else w
                out[b, :, t] = r * inv * wv * gate
        return out
    return impl


EPI_MUTATIONS = ["epi_sum", "epi_eps_outside", "epi_sigmoid", "epi_no_weight", "epi_pads_too"]


def test_unmodified_epilogue_copy_passes_every_pin():
    for check in _pins.EPILOGUE_CHECKS:
        check(make_epilogue())


@pytest.mark.parametrize("mutation", EPI_MUTATIONS)
def test_planted_epilogue_mistake_is_caught(mutation):
    impl = make_epilogue(mutation)
    caught = 0
    for check in _pins.EPILOGUE_CHECKS:
        try:
            check(impl)
        except AssertionError:
            caught += 1
    assert caught > 0, mutation


def make_conv(mutation=None):
    """A plain copy of the depthwise causal conv + SiLU with its state, with planted mistakes."""
    def impl(x, w, bias, state, lengths):
        x, w = np.asarray(x, np.float64), np.asarray(w, np.float64)
        B, S, C = x.shape
        K = w.shape[1]
        bias = np.zeros(C) if bias is None or mutation == "conv_no_bias" else np.asarray(bias, np.float64)
        st = np.zeros((B, C, K)) if state is None or mutation == "conv_state_ignored" else np.asarray(state)
        taps = w[:, ::-1] if mutation == "conv_taps_reversed" else w
        y = np.zeros((B, S, C))
        new = np.empty((B, C, K))
        for b in range(B):
            L = S if lengths is None else int(lengths[b])
            hist = np.concatenate([st[b].T, x[b, :L]], axis=0)
            off = 0 if mutation == "conv_window_late" else 1
            for t in range(L):
                win = hist[t + off:t + off + K]
                acc = bias + np.sum(taps.T * win, axis=0)
                y[b, t] = 1.0 / (1.0 + np.exp(-acc)) if mutation == "conv_sigmoid" else acc / (1.0 + np.exp(-acc))
            keep = hist[L:L + K] if mutation != "conv_state_short" else np.concatenate([np.zeros((1, C)),
                                                                                         hist[L + 1:L + K]], 0)
            new[b] = keep.T
        return y, new
    return impl


CONV_MUTATIONS = ["conv_no_bias", "conv_state_ignored", "conv_taps_reversed", "conv_window_late", "conv_sigmoid",
                  "conv_state_short"]


def test_unmodified_conv_copy_passes_every_pin():
    for check in _pins.CONV_CHECKS:
        check(make_conv())


@pytest.mark.parametrize("mutation", CONV_MUTATIONS)
def test_planted_conv_mistake_is_caught(mutation):
    impl = make_conv(mutation)
    caught = 0
    for check in _pins.CONV_CHECKS:
        try:
            check(impl)
        except (AssertionError, IndexError, ValueError):
            caught += 1
    assert caught > 0, mutation


def make_decode(mutation=None):
    """A plain copy of the decode call over a slot pool (the recurrent_gated_delta_rule page's reading, as the
    oracle states it), with planted mistakes in the features only decode has."""
    def dec(q, k, v, beta, g, gk, pool, indices, lengths, accepted=None, scale=1.0, per_token=False):
        q, k, v, beta = (np.asarray(x, np.float64) for x in (q, k, v, beta))
        B, Nk, S, Dk = q.shape
        Nv, Dv = v.shape[1], v.shape[3]
        grp = Nv // Nk
        P = np.array(pool, np.float64, copy=True)
        out = np.zeros((B, Nv, S, Dv))
        for b in range(B):
            L = int(lengths[b])
            if L == 0:
                continue
            if per_token:
                A = 1 if accepted is None else int(accepted[b])
                if not 1 <= A <= S:
                    raise ValueError("accepted count outside [1, S]")
                start = int(indices[b * S + (0 if mutation == "spec_start_first" else A - 1)])
                ncommit = L
            else:
                A = L if accepted is None else int(accepted[b])
                start = int(indices[b * S])
                ncommit = min(A, L)
                if mutation == "commit_ignores_accepted":
                    ncommit = L
                elif mutation == "commit_one_short":
                    ncommit = max(ncommit - 1, 0)
            for h in range(Nv):
                kh = (h % Nk) if mutation == "gqa_modulo" else h // grp
                St = P[start, (Nv - 1 - h) if mutation == "pool_head_reversed" else h].copy()
                for t in range(L):
                    x = scale * q[b, kh, t]
                    y = k[b, kh, t]
                    St = St * (1.0 if g is None else np.exp(float(g[b, h, t])))
                    e = None
                    if gk is not None and mutation != "gk_ignored":
                        gkt = np.asarray(gk[b, h, t], np.float64)
                        e = np.exp(-gkt) if mutation == "gk_sign" else np.exp(gkt)
                        if mutation != "gk_after_readout":
                            St = St * e[:, None]
                    m = y @ St
                    if e is not None and mutation == "gk_after_readout":
                        St = St * e[:, None]
                    St = St + np.outer(y, beta[b, h, t] * (v[b, h, t] - m))
                    out[b, h, t] = x @ St
                    if t < ncommit and (mutation != "commit_only_last" or t == ncommit - 1):
                        slot = int(indices[b * S + (min(t + 1, S - 1) if mutation == "commit_slot_shift" else t)])
                        P[slot, h] = St
                if mutation == "dirty_padding":
                    out[b, h, L:] = 1.0
        return out, P
    return dec


DECODE_MUTATIONS = ["gk_sign", "gk_ignored", "gk_after_readout", "commit_ignores_accepted", "commit_one_short",
                    "commit_only_last", "commit_slot_shift", "spec_start_first", "pool_head_reversed", "gqa_modulo",
                    "dirty_padding"]


def test_unmodified_decode_copy_passes_every_pin():
    for check in _decode_pins.DECODE_CHECKS:
        check(make_decode())


@pytest.mark.parametrize("mutation", DECODE_MUTATIONS)
def test_planted_decode_mistake_is_caught(mutation):
    impl = make_decode(mutation)
    caught = 0
    for check in _decode_pins.DECODE_CHECKS:
        try:
            check(impl)
        except AssertionError:
            caught += 1
    assert caught > 0, mutation
