"""The byte accounting behind bench.py's roofline fractions, on the CPU.

The numerator of every roofline fraction is the algorithmic byte count of one launch: what the call must move
at minimum, whatever the kernel does.  These tests pin the counts of the prefill and decode workloads to sums
written out by hand from the layouts of the chunk_gated_delta_rule and recurrent_gated_delta_rule pages
(lite_boost), and check that the DRAM traffic taken from a committed ncu summary is reported only while the
kernel source it was measured on is unchanged.
"""
import hashlib
import types

import numpy as np

import bench


def _shape(B, S, Nk, Nv, D, lengths, g=True, gk=False):
    return types.SimpleNamespace(B=B, S=S, Nk=Nk, Nv=Nv, Dk=D, Dv=D, lengths=np.asarray(lengths, np.int64),
                                 g=object() if g else None, gk=object() if gk else None)


def test_prefill_bytes_of_the_prefill_workload():
    """B=4 sequences of 4096 tokens, Nk=16, Nv=32, D=128, bf16 (2 B) with the fp32 gate input.
    Per token: q and k over the key heads 2*16*128*2 = 8192, v and out over the value heads 2*32*128*2 = 16384,
    beta 32*2 = 64, the gate 32*4 = 128, in all 24768 B; 16384 tokens give 405,798,912 B.  The initial state
    read and the final state written: 2*4*32*128*128*2 = 8,388,608 B.  No padding rows."""
    w = _shape(4, 4096, 16, 32, 128, [4096] * 4)
    assert bench.algorithmic_prefill_bytes(w) == 16384 * 24768 + 8388608 == 414187520


def test_prefill_bytes_count_the_zero_padding_rows_of_out():
    """A sequence shorter than S still has its padding rows of out written (as zeros): (S - L) * Nv * Dv * 2."""
    full = _shape(2, 128, 1, 2, 16, [128, 128])
    short = _shape(2, 128, 1, 2, 16, [128, 100])
    per_token = 2 * 1 * 16 * 2 + 2 * 2 * 16 * 2 + 2 * 2 + 2 * 4
    assert bench.algorithmic_prefill_bytes(full) - bench.algorithmic_prefill_bytes(short) == \
        28 * per_token - 28 * 2 * 16 * 2


def test_decode_bytes_of_the_decode_workload():
    """64 sequences of one token, Nk=16, Nv=32, D=128: the state read and written once per (sequence, value
    head), 2*64*32*128*128*2 = 134,217,728 B; per token q, k 8192, v 8192, beta 64 and the gate 128 B
    (64 tokens: 1,060,864 B); out for every position, 64*32*128*2 = 524,288 B."""
    w = _shape(64, 1, 16, 32, 128, [1] * 64)
    nb = bench.algorithmic_decode_bytes(w)
    assert nb["state"] == 134217728
    assert nb["io"] == 64 * (8192 + 8192 + 64 + 128) + 524288
    assert nb["state"] + nb["io"] == 135802880


def test_decode_bytes_with_the_per_key_gate_and_empty_sequences():
    """gk adds Nv*Dk fp32 values per token; a sequence of length 0 moves no state (its out rows are still
    written); without g the gate input is not read."""
    base = _shape(3, 4, 1, 2, 16, [4, 0, 2], g=False)
    with_gk = _shape(3, 4, 1, 2, 16, [4, 0, 2], g=True, gk=True)
    nb0, nb1 = bench.algorithmic_decode_bytes(base), bench.algorithmic_decode_bytes(with_gk)
    assert nb0["state"] == nb1["state"] == 2 * 2 * 2 * 16 * 16 * 2  # two sequences with tokens
    assert nb1["io"] - nb0["io"] == 6 * (2 * 4 + 2 * 16 * 4)


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """The DRAM bytes of a committed capture are reported while the kernel's source hashes as recorded, and
    reported as None once the source has changed (a stale capture is not the current kernel's traffic)."""
    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\n")
    h = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(f"# kernel source hash bytes\nchunk k.cu {h} 12345\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("chunk") == 12345.0
    assert bench.profiled_traffic("decode") is None
    src.write_text("// kernel v2\n")
    assert bench.profiled_traffic("chunk") is None
