"""Stand-alone prologue (gdr_prologue_apply) on the GPU against the oracle's."""
import numpy as np
import pytest

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, host, rnd, rnd32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
def test_prologue_matches_oracle(dt):
    w = workloads.generate("prefill", B=2, S=33, Nk=2, Nv=4, D=128)
    q, k, b = rnd(w.q, dt), rnd(w.k, dt), rnd(w.b, dt)
    a, A_log, dtb = rnd32(w.a), rnd32(w.A_log), rnd32(w.dt_bias)
    res = gdr.prologue(q=dev(q, dt), k=dev(k, dt), b=dev(b, dt), a=dev(a, "f32"), A_log=dev(A_log, "f32"),
                       dt_bias=dev(dtb, "f32"), eps=1e-6)
    ref = oracle.prologue(q=q, k=k, b=b, a=a, A_log=A_log, dt_bias=dtb, eps=1e-6)
    tol = {"f32": 2e-6, "bf16": 8e-3, "f16": 1e-3}[dt]  # one rounding of values of magnitude <= 1
    for key in ("q_hat", "k_hat", "beta"):
        err = float(np.abs(host(res[key]) - ref[key]).max())
        assert err <= tol, (key, err)
    g = host(res["g"])
    assert np.allclose(g, ref["g"], rtol=2e-6, atol=1e-6)


def test_prologue_zero_row_and_extreme_gate():
    """A zero row stays zero (eps inside the sqrt); softplus stays finite for
    large |a + dt_bias|."""
    q = np.zeros((1, 1, 3, 32))
    q[0, 0, 1] = 3.0
    a = np.array([[[60.0, -60.0, 0.0]]])
    res = gdr.prologue(q=dev(q, "f32"), a=dev(a, "f32"), A_log=dev(np.zeros(1), "f32"),
                       dt_bias=dev(np.zeros(1), "f32"))
    qh = host(res["q_hat"])
    assert np.all(qh[0, 0, 0] == 0.0)
    assert np.allclose(qh[0, 0, 1], 3.0 / np.sqrt(9.0 * 32 + 1e-6), rtol=1e-6)
    g = host(res["g"])[0, 0]
    assert np.all(np.isfinite(g))
    assert abs(g[0] + 60.0) < 1e-4 and abs(g[1]) < 1e-20 and abs(g[2] + np.log(2.0)) < 1e-6
