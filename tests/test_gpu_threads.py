"""Calls from two host threads at once, each on its own stream, against the fp64 oracle: the tensor-core and the
CUDA-core prefill and two decode shapes whose shared-memory sizes differ, so that the per-device launch records
(shared-memory attribute, resident grid) are read and written concurrently."""
import threading

import numpy as np
import pytest
import torch

import gated_deltanet_gdr_b200 as gdr
import oracle
import workloads
from tests._helpers import assert_close, dev, dev_i32, host, rnd, unfused_inputs

pytestmark = pytest.mark.gpu

REPEATS = 20


def _prefill_case(dt, D, S, seed):
    w = workloads.random_case(B=2, Nk=2, Nv=4, S=S, Dk=D, Dv=D, seed=seed, lengths=np.array([S, S - 9], np.int32))
    ins = unfused_inputs(w, dt)
    args = (dev(ins["q"], dt), dev(ins["k"], dt), dev(ins["v"], dt), dev(ins["beta"], dt), dev(ins["g"], "f32"),
            dev(ins["initial_state"], dt), dev_i32(w.lengths))
    ref = oracle.chunk_fwd(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["initial_state"], w.lengths,
                           w.scale)
    return w, args, ref


def _decode_case(S, seed):
    w = workloads.random_case(B=8, Nk=2, Nv=4, S=S, Dk=128, Dv=128, seed=seed, slots=10, with_gk=True)
    ins = unfused_inputs(w, "bf16")
    pool0 = rnd(w.pool, "bf16")
    args = [dev(ins[n], "bf16") for n in ("q", "k", "v", "beta")] + [dev(ins["g"], "f32"), dev(ins["gk"], "f32")]
    ref = oracle.recurrent_step(ins["q"], ins["k"], ins["v"], ins["beta"], ins["g"], ins["gk"], pool0, w.indices,
                                w.lengths, w.accepted, w.scale)
    return w, args, pool0, ref


def test_two_host_threads_two_streams():
    pre = [_prefill_case("bf16", 128, 150, 900), _prefill_case("f32", 64, 130, 901)]
    dec = [_decode_case(1, 902), _decode_case(4, 903)]
    results = [None, None]
    errors = []
    torch.cuda.synchronize()  # the inputs are resident before either thread starts

    def work(i):
        try:
            s = torch.cuda.Stream()
            w, args, _ = pre[i]
            wd, dargs, pool0, _ = dec[i]
            with torch.cuda.stream(s):  # outputs are allocated on the stream that uses them
                pool = dev(pool0, "bf16")
                idx, lens, acc = dev_i32(wd.indices), dev_i32(wd.lengths), dev_i32(wd.accepted)
                for _ in range(REPEATS):
                    out, fin = gdr.chunk_fwd(*args, w.scale, stream=s)
                dout, pool = gdr.recurrent_step(*dargs, pool, idx, lens, acc, wd.scale, stream=s)
            s.synchronize()
            results[i] = (host(out), host(fin), host(dout), host(pool))
        except Exception as e:  # reported by the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert gdr.get_error() == 0
    for i, dt in enumerate(("bf16", "f32")):
        out, fin, dout, pool = results[i]
        ro, rf = pre[i][2]
        assert_close(out, ro, dt, f"thread {i} out")
        assert_close(fin, rf, dt, f"thread {i} final_state")
        wd, _, _, (rdo, rpool) = dec[i]
        assert_close(dout, rdo, "bf16", f"thread {i} decode out")
        touched = sorted(set(int(wd.indices[b * wd.S + t]) for b in range(wd.B) for t in range(int(wd.accepted[b]))))
        if touched:
            assert_close(pool[touched], rpool[touched], "bf16", f"thread {i} decode state")
