"""The depthwise causal conv1d + SiLU before the rule (gdr_conv1d) on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, host, rnd

pytestmark = pytest.mark.gpu


def split_qkv(y, Nk, Nv, Dk, Dv):
    """(B, S, C) channels last -> q, k (B, Nk, S, Dk), v (B, Nv, S, Dv), the layout the rule takes."""
    B, S, _ = y.shape
    qk = Nk * Dk
    q = y[:, :, :qk].reshape(B, S, Nk, Dk).transpose(0, 2, 1, 3)
    k = y[:, :, qk:2 * qk].reshape(B, S, Nk, Dk).transpose(0, 2, 1, 3)
    v = y[:, :, 2 * qk:].reshape(B, S, Nv, Dv).transpose(0, 2, 1, 3)
    return q, k, v


def run(w, dt, K, lengths=None, with_state=True, with_bias=True):
    x, wt, bias, st = workloads.conv_inputs(w, K, with_state, with_bias)
    xr, wr, br, sr = rnd(x, dt), rnd(wt, dt), rnd(bias, dt), rnd(st, dt)
    q, k, v, ns = gdr.conv1d(dev(xr, dt), dev(wr, dt), dev(br, dt), dev(sr, dt), dev_i32(lengths), Nk=w.Nk,
                             Nv=w.Nv, Dk=w.Dk, Dv=w.Dv)
    assert gdr.get_error() == 0
    y, rs = oracle.causal_conv1d(xr, wr, br, sr, lengths)
    return (host(q), host(k), host(v), host(ns)), split_qkv(y, w.Nk, w.Nv, w.Dk, w.Dv) + (rs,)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("S", [1, 5, 64, 65, 200])
def test_conv1d_parity(dt, K, S):
    """Ragged lengths with one empty sequence, an input state and a bias; S = 1 and 5 are single-tile
    launches (the state is written by the conv kernel itself), 64 and beyond use the state kernel."""
    w = workloads.random_case(B=3, Nk=2, Nv=4, S=S, Dk=32, Dv=64, seed=400 + S + K)
    lengths = np.array([S, max(S - 3, 1), 0], np.int32)
    got, ref = run(w, dt, K, lengths)
    for name, g, r in zip(("q", "k", "v", "state"), got, ref):
        assert_close(g, r, dt, name)
    for b in range(w.B):
        L = int(lengths[b])
        assert np.all(got[0][b, :, L:] == 0) and np.all(got[2][b, :, L:] == 0)
    assert np.array_equal(got[3][2], rnd(workloads.conv_inputs(w, K)[3], dt)[2])  # L = 0: state untouched


@pytest.mark.parametrize("Dk,Dv", [(16, 16), (64, 128), (128, 128), (128, 32)])
def test_conv1d_head_sizes_no_state_no_bias(Dk, Dv):
    w = workloads.random_case(B=2, Nk=1, Nv=2, S=70, Dk=Dk, Dv=Dv, seed=420 + Dk + Dv)
    got, ref = run(w, "f32", 4, with_state=False, with_bias=False)
    for name, g, r in zip(("q", "k", "v", "state"), got, ref):
        assert_close(g, r, "f32", name)


def test_conv1d_decode_chain_in_place():
    """Ten single-token calls that update the state in place equal one call over the ten tokens."""
    w = workloads.random_case(B=4, Nk=2, Nv=4, S=10, Dk=64, Dv=64, seed=430)
    x, wt, bias, st = workloads.conv_inputs(w, 4)
    xr, wr, br, sr = (rnd(a, "bf16") for a in (x, wt, bias, st))
    state = dev(sr, "bf16")
    outs = []
    for t in range(w.S):
        q, k, v, ns = gdr.conv1d(dev(xr[:, t:t + 1], "bf16"), dev(wr, "bf16"), dev(br, "bf16"), state, None,
                                 Nk=w.Nk, Nv=w.Nv, Dk=w.Dk, Dv=w.Dv, conv_state_out=state)
        assert ns is state
        outs.append([host(q), host(k), host(v)])
    assert gdr.get_error() == 0
    y, rs = oracle.causal_conv1d(xr, wr, br, sr)
    rq, rk, rv = split_qkv(y, w.Nk, w.Nv, w.Dk, w.Dv)
    for i, r in enumerate((rq, rk, rv)):
        assert_close(np.concatenate([o[i] for o in outs], axis=2), r, "bf16", "qkv"[i])
    assert_close(host(state), rs, "bf16", "state")


def test_conv1d_bad_length_sets_error_and_skips():
    w = workloads.random_case(B=2, Nk=1, Nv=2, S=8, Dk=16, Dv=16, seed=440)
    x, wt, bias, st = (rnd(a, "f32") for a in workloads.conv_inputs(w, 3))
    sd = dev(st, "f32")
    q, k, v, ns = gdr.conv1d(dev(x, "f32"), dev(wt, "f32"), dev(bias, "f32"), sd, dev_i32(np.array([9, 8])),
                             Nk=1, Nv=2, Dk=16, Dv=16)
    assert gdr.get_error() == gdr.DEVERR_LENGTH
    assert bool((q[0] == 0).all()) and bool((v[0] == 0).all())
    y, rs = oracle.causal_conv1d(x[1:], wt, bias, st[1:])
    assert_close(host(v[1]), split_qkv(y, 1, 2, 16, 16)[2][0], "f32", "v")


def test_conv1d_prefill_shape_full_size_sampled():
    """B=4, S=4096, Nk=16, Nv=32, D=128 (C = 8192), K = 4, bf16: the launch the benchmark's conv line times,
    checked on sampled channels of every kind (q, k and v heads) computed by the oracle."""
    w = workloads.generate("prefill")
    x, wt, bias, st = workloads.conv_inputs(w, 4)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to("cuda")
    q, k, v, ns = gdr.conv1d(to(x), to(wt), to(bias), to(st), None, Nk=w.Nk, Nv=w.Nv, Dk=w.Dk, Dv=w.Dv)
    assert gdr.get_error() == 0
    qk = w.Nk * w.Dk
    for c in (0, 517, qk + 3, qk + 2047, 2 * qk + 1, 2 * qk + 4095):
        y, rs = oracle.causal_conv1d(rnd(x[:, :, c:c + 1], "bf16"), rnd(wt[c:c + 1], "bf16"),
                                     rnd(bias[c:c + 1], "bf16"), rnd(st[:, c:c + 1], "bf16"))
        if c < qk:
            got = q[:, c // w.Dk, :, c % w.Dk]
        elif c < 2 * qk:
            got = k[:, (c - qk) // w.Dk, :, (c - qk) % w.Dk]
        else:
            got = v[:, (c - 2 * qk) // w.Dv, :, (c - 2 * qk) % w.Dv]
        assert_close(host(got), y[:, :, 0], "bf16", f"channel {c}")
        assert_close(host(ns[:, c]), rs[:, 0], "bf16", f"state {c}")
    assert bool(torch.isfinite(v).all())
