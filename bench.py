"""Benchmark of the gated delta rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the prefill hot path over the prefill workload
(B=4, S=4096, Nk=16, Nv=32, Dk=Dv=128, bf16 q/k/v/beta/state, fp32 gate):
raw q/k, beta logits and the raw gate a go through gdr_chunk_fwd with the fused
prologue (l2norm, sigmoid, softplus gate), the cumulative gate, the WY solve,
the intra-chunk products and the inter-chunk carry, writing out and the final
state.  The decode row is measured in the same run on the decode workload
(B=64, one token, 128-slot bf16 pool) and the multi-token per-key-gate decode
workload (B=256, S=4, 512 slots), reported under "decode".

Timing: W warm-up steps, then K timed steps bracketed by a barrier and
torch.cuda.synchronize(); each step is timed with CUDA events on the launching
stream, with a 256 MiB L2 flush between steps (the prefill inputs, 414 MB, are
larger than the 126 MB L2 as well).  For N > 1 (torchrun), every rank runs its
own batch (weak scaling, no data-path collective) and the max over ranks is used.

`--impl reference` times the fp64 CPU oracle (the only reference this path has)
on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "chunked GDR prefill tokens/s; decode state GB/s vs B200 HBM peak (1 GPU)"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20


def algorithmic_prefill_bytes(w) -> int:
    """HBM bytes one prefill call must move at minimum: per valid token q, k (Nk heads),
    v and out (Nv heads) in bf16, beta (bf16) and the fp32 gate input per value head;
    per (b, h) the initial state read and the final state written (bf16)."""
    e = 2  # bf16
    per_token = 2 * w.Nk * w.Dk * e + w.Nv * w.Dv * e + w.Nv * w.Dv * e + w.Nv * e + w.Nv * 4
    tokens = int(w.lengths.sum())
    state = 2 * w.B * w.Nv * w.Dk * w.Dv * e
    # padding rows of out are written as zeros too
    pad_out = (w.B * w.S - tokens) * w.Nv * w.Dv * e
    return tokens * per_token + state + pad_out


def algorithmic_decode_bytes(w) -> dict:
    """State bytes (read once and written once per referenced (slot, head)) and the
    per-token I/O bytes of one decode call."""
    e = 2
    seqs = int((w.lengths > 0).sum())
    state = 2 * seqs * w.Nv * w.Dk * w.Dv * e
    tok = int(w.lengths.sum())
    io = tok * (2 * w.Nk * w.Dk * e + w.Nv * w.Dv * e + w.Nv * e + (w.Nv * 4 if w.g is not None else 0))
    if w.gk is not None:
        io += tok * w.Nv * w.Dk * 4
    io += w.B * w.S * w.Nv * w.Dv * e  # out, all positions
    return {"state": state, "io": io}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (matching hash), else None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and parts[0] == kernel and not line.startswith("#"):
            src = os.path.join(ROOT, parts[1])
            if not os.path.exists(src):
                return None
            h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
            return float(parts[3]) if h == parts[2] else None
    return None


class ClockSampler:
    """Samples SM clock and clock-event (throttle) reasons through NVML every ~2 ms in a
    background thread while `active` is set (read-only queries; no setting is changed)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.active = False
        self._stop = False
        self.max_mhz = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                uuid = torch.cuda.get_device_properties(self.index).uuid
            except Exception:
                pass
            h = None
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.nv, self.h = pynvml, h
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.ok = True
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        while not self._stop:
            if self.active:
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((float(mhz), int(rs)))
                except Exception:
                    pass
            time.sleep(0.002)

    def __exit__(self, *exc):
        self._stop = True
        if self.ok:
            self.t.join(timeout=2)

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        sm = [m for m, _ in self.samples]
        reasons = sorted(n for n, bit in self.REASONS.items() if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "source": "NVML, 2 ms polling during the timed steps"}


def dist_setup():
    """One process per GPU (torchrun's RANK/LOCAL_RANK/WORLD_SIZE/MASTER_*): NCCL when CUDA is
    present, gloo otherwise (the CPU tests of this plumbing).  The process group carries only
    the barrier and the max-over-ranks of the timings: the ranks' batches are independent."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(x: float, world: int) -> float:
    """Max over ranks (the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank_per_step: int, steps: int, max_total_ms: float, world: int) -> float:
    """Whole-job throughput: every rank processes its own units each step; the job takes as
    long as its slowest rank."""
    return world * units_per_rank_per_step * steps / (max_total_ms / 1e3)


def timed_steps(fn, K, flush, stream):
    """Per-step CUDA-event times (ms) on `stream`, with an L2 flush before each step."""
    evs = []
    with torch.cuda.stream(stream):
        for _ in range(K):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            fn()
            e.record(stream)
            evs.append((s, e))
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in evs]


def cpu_oracle_sample(w, heads=None):
    """The fp64 oracle as it stands on one sequence of the prefill workload (all
    value heads, or the first `heads` of them, all 4096 tokens), prologue included.
    Returns (tokens/s for all the workload's value heads, seconds, threads)."""
    import oracle
    sl = slice(0, 1)
    hv = w.Nv if heads is None else heads
    hk = max(1, hv * w.Nk // w.Nv)
    to_bf16 = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()
    q, k = (to_bf16(x[sl, :hk]) for x in (w.q, w.k))
    v, b = (to_bf16(x[sl, :hv]) for x in (w.v, w.b))
    s0 = to_bf16(w.initial_state[sl, :hv])
    t0 = time.perf_counter()
    p = oracle.prologue(q=q, k=k, b=b, a=w.a[sl, :hv], A_log=w.A_log[:hv], dt_bias=w.dt_bias[:hv])
    oracle.chunk_fwd(p["q_hat"], p["k_hat"], v, p["beta"], p["g"], s0, None, w.scale)
    dt = time.perf_counter() - t0
    return w.S * hv / w.Nv / dt, dt, oracle.threads()


def cpu_model() -> str:
    """The host CPU's model name (lscpu, else /proc/cpuinfo)."""
    import subprocess
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.strip().startswith("Model name:"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def cpu_baseline_fields() -> dict:
    """The oracle on the host cores: one prefill sequence on all threads (the headline's unit), the first 4 value
    heads of it on one thread, and one call of the decode workload (B=64, one token, 32 value heads)."""
    import oracle
    wp = workloads.generate("prefill", B=1)
    tps, dt, thr = cpu_oracle_sample(wp)
    oracle.set_threads(1)
    try:
        tps1, dt1, _ = cpu_oracle_sample(wp, heads=4)
        wd = workloads.generate("decode")
        to_bf16 = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()
        q, k, v, b, pool = (to_bf16(x) for x in (wd.q, wd.k, wd.v, wd.b, wd.pool))
        g = np.asarray(wd.g, np.float32).astype(np.float64)
        t0 = time.perf_counter()
        p = oracle.prologue(q=q, k=k, b=b)
        oracle.recurrent_step(p["q_hat"], p["k_hat"], v, p["beta"], g, None, pool, wd.indices, wd.lengths,
                              wd.accepted, wd.scale)
        dtd = time.perf_counter() - t0
    finally:
        oracle.set_threads(thr)
    state = algorithmic_decode_bytes(wd)["state"]
    return {"value": tps, "unit": UNIT, "cores": thr, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"1 sequence x 4096 tokens x 32 value heads, prologue included, {dt:.1f} s on {thr} threads",
            "single_thread": {"value": tps1, "unit": UNIT, "cores": 1,
                              "sample": f"the first 4 value heads of that sequence on 1 thread, {dt1:.1f} s, "
                                        "scaled to 32 heads"},
            "decode": {"us_per_call": dtd * 1e6, "state_GBps": state / dtd / 1e9, "cores": 1,
                       "sample": "one call of the decode workload (B=64, one token, 32 value heads), 1 thread"}}


def prefill_config(world: int) -> dict:
    """The `config` of the headline line (both arms)."""
    p = workloads.spec("prefill")
    return {"workload": f"prefill B={p['B']} S={p['S']} Nk={p['Nk']} Nv={p['Nv']} Dk=Dv={p['D']} bf16, fused "
                        "prologue, equal lengths", "global_batch": p["B"] * world, "seq_len": p["S"],
            "parallelism": f"dp{world} (independent batches per GPU)",
            "l2": "inputs larger than L2, plus a 256 MiB flush before every timed step"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = workloads.generate("prefill", B=1)
    vals = []
    for i in range(args.warmup + args.steps):
        tps, dt, thr = cpu_oracle_sample(w)
        if i >= args.warmup:
            vals.append(dt)
    tot = sum(vals)
    value = w.S * len(vals) / tot
    sample = (f"1 of the workload's {workloads.spec('prefill')['B']} sequences per step (4096 tokens x 32 value "
              "heads, prologue included), on the host cores; the oracle in fp64")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(vals),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": prefill_config(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bf16_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()


def f32_dev(x):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(x, np.float32))).cuda()


def bench_prefill(gdr, args, world, rank, clk, flush, stream, peaks):
    """The headline: prefill with the fused prologue; returns (line fields, workload, tensors)."""
    w = workloads.generate("prefill", seed=2 + 1000 * rank)
    t = dict(q=bf16_dev(w.q), k=bf16_dev(w.k), v=bf16_dev(w.v), b=bf16_dev(w.b), a=f32_dev(w.a),
             s0=bf16_dev(w.initial_state))
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=f32_dev(w.A_log),
                       dt_bias=f32_dev(w.dt_bias))
    t["out"] = torch.empty((w.B, w.Nv, w.S, w.Dv), dtype=torch.bfloat16, device="cuda")
    t["fin"] = torch.empty_like(t["s0"])

    # argument checks and marshalling happen once; each step is one C-ABI call
    step = gdr.prepare_chunk_fwd(t["q"], t["k"], t["v"], t["b"], t["a"], t["s0"], None, w.scale, prologue=pro,
                                 out=t["out"], final_state=t["fin"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    clk.active = True
    times = timed_steps(step, args.steps, flush, stream)
    clk.active = False
    barrier(world)
    total_ms = all_max(sum(times), world)
    ms_per_step = total_ms / args.steps
    tokens = int(w.lengths.sum())
    alg_bytes = algorithmic_prefill_bytes(w)
    achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
    fields = {
        "value": weak_scaling_rate(tokens, args.steps, total_ms, world), "ms_per_step": ms_per_step,
        "config": prefill_config(world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic("chunk"),
                     "peak_source": peaks["source"], "algorithmic_bytes_per_launch": alg_bytes,
                     "kernel": "gdr_chunk_fwd (fused prologue)"},
        "gpu_launches": prefill_kernels(gdr, w) * args.steps,
    }
    return fields, w, t, pro, step


def bench_varlen(gdr, args, world, rank, flush, stream, peaks):
    """The variable-length prefill workload (B=8, padded S=8192, lengths ~ U[512, 8192] with one 0), fused
    prologue.  256 chains on 148 SMs: the chain kernel starts the longest sequences first."""
    w = workloads.generate("varlen", seed=3 + 1000 * rank)
    t = dict(q=bf16_dev(w.q), k=bf16_dev(w.k), v=bf16_dev(w.v), b=bf16_dev(w.b), a=f32_dev(w.a),
             s0=bf16_dev(w.initial_state))
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=f32_dev(w.A_log),
                       dt_bias=f32_dev(w.dt_bias))
    lens = torch.from_numpy(w.lengths).cuda()
    step = gdr.prepare_chunk_fwd(t["q"], t["k"], t["v"], t["b"], t["a"], t["s0"], lens, w.scale, prologue=pro)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    times = timed_steps(step, args.steps, flush, stream)
    barrier(world)
    ms = all_max(sum(times), world) / args.steps
    tokens = int(w.lengths.sum())
    nb = algorithmic_prefill_bytes(w)
    achieved = nb / (ms / 1e3) / 1e9
    return {"workload": f"varlen B={w.B} padded S={w.S} Nk={w.Nk} Nv={w.Nv} D={w.Dk} bf16, lengths "
                        f"{w.lengths.tolist()}, fused prologue", "ms_per_step": ms,
            "tokens_per_s": weak_scaling_rate(tokens, args.steps, ms * args.steps, world),
            "l2": "inputs larger than L2, plus a 256 MiB flush before every timed step",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes_per_launch": nb}}, \
        prefill_kernels(gdr, w) * args.steps


def prefill_kernels(gdr, w) -> int:
    """Kernels one prefill call launches: 2 when the sizes ask for the two-kernel schedule's workspace (the WY
    pass, then the chains), else 1 (the one-kernel schedule)."""
    return 2 if gdr.chunk_fwd_workspace_bytes(w.B, w.Nk, w.Nv, w.S, w.Dk, w.Dv, torch.bfloat16) > 0 else 1


def bench_prefill_b1(gdr, args, world, rank, flush, stream, peaks):
    """One sequence of the prefill workload (B=1, S=4096, fused prologue): 32 chains on 148 SMs, where the
    workspace query asks for the two-kernel schedule (the WY pass over every chunk on every SM, then the
    chains)."""
    w = workloads.generate("prefill", B=1, seed=12 + 1000 * rank)
    t = dict(q=bf16_dev(w.q), k=bf16_dev(w.k), v=bf16_dev(w.v), b=bf16_dev(w.b), a=f32_dev(w.a),
             s0=bf16_dev(w.initial_state))
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=f32_dev(w.A_log),
                       dt_bias=f32_dev(w.dt_bias))
    step = gdr.prepare_chunk_fwd(t["q"], t["k"], t["v"], t["b"], t["a"], t["s0"], None, w.scale, prologue=pro)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    times = timed_steps(step, args.steps, flush, stream)
    barrier(world)
    total_ms = all_max(sum(times), world)
    ms = total_ms / args.steps
    tokens = int(w.lengths.sum())
    alg = algorithmic_prefill_bytes(w)
    achieved = alg / (ms / 1e3) / 1e9
    nk = prefill_kernels(gdr, w)
    return {"workload": f"prefill B={w.B} S={w.S} Nk={w.Nk} Nv={w.Nv} Dk=Dv={w.Dk} bf16, fused prologue",
            "schedule": "two kernels (WY pass, then the chains)" if nk == 2 else "one kernel",
            "ms_per_step": ms, "tokens_per_s": weak_scaling_rate(tokens, args.steps, total_ms, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes_per_launch": alg,
                         "kernel": "gdr_chunk_fwd (fused prologue)"}}, nk * args.steps


def bench_prefill_no_gate(gdr, args, world, w, t, flush, stream, peaks):
    """The prefill workload without a gate (g = NULL, hasGamma = 0 of the chunk operator): the tensor-core
    prefill's build without the gate arithmetic; l2norm and beta logits fused."""
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True)
    step = gdr.prepare_chunk_fwd(t["q"], t["k"], t["v"], t["b"], None, t["s0"], None, w.scale, prologue=pro,
                                 out=t["out"], final_state=t["fin"])
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    times = timed_steps(step, args.steps, flush, stream)
    barrier(world)
    total_ms = all_max(sum(times), world)
    ms = total_ms / args.steps
    tokens = int(w.lengths.sum())
    alg = algorithmic_prefill_bytes(w) - tokens * w.Nv * 4  # no gate input
    achieved = alg / (ms / 1e3) / 1e9
    return {"workload": f"prefill B={w.B} S={w.S} Nk={w.Nk} Nv={w.Nv} Dk=Dv={w.Dk} bf16, no gate (g = NULL), "
                        "fused l2norm and beta", "ms_per_step": ms,
            "tokens_per_s": weak_scaling_rate(tokens, args.steps, total_ms, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes_per_launch": alg,
                         "kernel": "gdr_chunk_fwd without gate"}}, prefill_kernels(gdr, w) * args.steps


def bench_prefill_epilogue(gdr, args, world, w, t, pro, flush, stream, peaks):
    """The same prefill call with the fused gated RMSNorm output epilogue (z and norm_w of the layer's
    output gate); returns (fields, launches)."""
    z, nw = workloads.epilogue_inputs(w)
    epi = gdr.Epilogue(z=bf16_dev(z), norm_w=f32_dev(nw), eps=1e-6)
    del z
    step = gdr.prepare_chunk_fwd(t["q"], t["k"], t["v"], t["b"], t["a"], t["s0"], None, w.scale, prologue=pro,
                                 epilogue=epi, out=t["out"], final_state=t["fin"])
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    times = timed_steps(step, args.steps, flush, stream)
    barrier(world)
    total_ms = all_max(sum(times), world)
    ms_per_step = total_ms / args.steps
    tokens = int(w.lengths.sum())
    # the prefill's bytes plus z (one bf16 row per valid token and value head) and norm_w
    alg_bytes = algorithmic_prefill_bytes(w) + tokens * w.Nv * w.Dv * 2 + w.Dv * 4
    achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
    return {"workload": f"prefill B={w.B} S={w.S} Nk={w.Nk} Nv={w.Nv} Dk=Dv={w.Dk} bf16, fused prologue and "
                        "gated RMSNorm epilogue (eps 1e-6)",
            "ms_per_step": ms_per_step, "tokens_per_s": weak_scaling_rate(tokens, args.steps, total_ms, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes_per_launch":
                         alg_bytes, "kernel": "gdr_chunk_fwd (fused prologue and epilogue)"}}, \
        prefill_kernels(gdr, w) * args.steps


def bench_conv1d(gdr, args, world, rank, flush, stream, peaks):
    """The depthwise causal conv1d + SiLU before the rule on the prefill workload's layout (C = 2 Nk Dk +
    Nv Dv = 8192 channels, K = 4, bf16, with bias and input state), writing q, k, v and the new state."""
    w = workloads.generate("prefill", seed=2 + 1000 * rank)
    x, wt, bias, st = workloads.conv_inputs(w, 4)
    x, wt, bias, st = bf16_dev(x), bf16_dev(wt), bf16_dev(bias), bf16_dev(st)
    B, S, C = x.shape
    q = torch.empty((B, w.Nk, S, w.Dk), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty((B, w.Nv, S, w.Dv), dtype=torch.bfloat16, device="cuda")
    ns = torch.empty_like(st)
    step = gdr.prepare_conv1d(x, wt, bias, st, None, Nk=w.Nk, Nv=w.Nv, Dk=w.Dk, Dv=w.Dv, q=q, k=k, v=v,
                              conv_state_out=ns)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    times = timed_steps(step, args.steps, flush, stream)
    barrier(world)
    total_ms = all_max(sum(times), world)
    ms = total_ms / args.steps
    alg = 2 * B * S * C * 2 + C * 4 * 2 + C * 2 + 2 * B * C * 4 * 2  # x in, q/k/v out, taps, bias, state in/out
    achieved = alg / (ms / 1e3) / 1e9
    # one conv launch per step; with S > 64 the state is written by a second, small launch
    return {"workload": f"conv1d B={B} S={S} C={C} (Nk={w.Nk} Nv={w.Nv} D={w.Dk}) K=4 bf16, bias and state",
            "ms_per_step": ms, "tokens_per_s": weak_scaling_rate(B * S, args.steps, total_ms, world),
            "l2": "inputs larger than L2, plus a 256 MiB flush before every timed step",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic("conv1d"),
                         "algorithmic_bytes_per_launch": alg, "kernel": "gdr_conv1d"}}, 2 * args.steps


def bench_f16(gdr, args, world, rank, flush, stream, peaks):
    """fp16 inputs: the prefill workload (fused prologue; the tensor-core kernel with fp16 operands) and the decode
    workload with an fp32 state (the D = 128 decode kernel).  Returns (fields, launches)."""
    h = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.float16).cuda()
    w = workloads.generate("prefill", seed=2 + 1000 * rank)
    pro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True, A_log=f32_dev(w.A_log), dt_bias=f32_dev(w.dt_bias))
    out = torch.empty((w.B, w.Nv, w.S, w.Dv), dtype=torch.float16, device="cuda")
    s0 = h(w.initial_state)
    fin = torch.empty_like(s0)
    step = gdr.prepare_chunk_fwd(h(w.q), h(w.k), h(w.v), h(w.b), f32_dev(w.a), s0, None, w.scale, prologue=pro,
                                 out=out, final_state=fin)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    times = timed_steps(step, args.steps, flush, stream)
    barrier(world)
    p_ms = all_max(sum(times), world) / args.steps
    alg = algorithmic_prefill_bytes(w)
    wd = workloads.generate("decode", seed=1 + 1000 * rank)
    pool = f32_dev(wd.pool)
    dout = torch.empty((wd.B, wd.Nv, wd.S, wd.Dv), dtype=torch.float16, device="cuda")
    dstep = gdr.prepare_recurrent_step(h(wd.q), h(wd.k), h(wd.v), h(wd.b), f32_dev(wd.g), None, pool,
                                       torch.from_numpy(wd.indices).cuda(), torch.from_numpy(wd.lengths).cuda(),
                                       torch.from_numpy(wd.accepted).cuda(), wd.scale,
                                       prologue=gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True), out=dout)
    for _ in range(args.warmup):
        dstep()
    torch.cuda.synchronize()
    barrier(world)
    dtimes = timed_steps(dstep, args.steps, flush, stream)
    barrier(world)
    d_ms = all_max(sum(dtimes), world) / args.steps
    nb = algorithmic_decode_bytes(wd)
    nb_state = nb["state"] * 2  # the fp32 state moves twice the bytes of the bf16 one counted there
    d_gbs = (nb_state + nb["io"]) / (d_ms / 1e3) / 1e9
    return {"prefill": {"workload": "prefill B=4 S=4096 Nk=16 Nv=32 D=128 fp16, fused prologue (tensor-core kernel)",
                        "ms_per_step": p_ms, "tokens_per_s": weak_scaling_rate(int(w.lengths.sum()), args.steps,
                                                                              p_ms * args.steps, world),
                        "roofline": {"bound": "hbm", "achieved": alg / (p_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "frac": alg / (p_ms / 1e3) / 1e9 / peaks["hbm_gbs"]}},
            "decode": {"workload": "decode B=64 S=1 fp16 inputs, fp32 state, L2 flush",
                       "us_per_call": d_ms * 1e3,
                       "roofline": {"bound": "hbm", "achieved": d_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": d_gbs / peaks["hbm_gbs"]}}}, (prefill_kernels(gdr, w) + 1) * args.steps


def bench_e2e(gdr, args, world, w, t, pro, flush, stream):
    """Same metric through the public call with host buffers: every step copies its inputs from
    pinned host memory, runs the call and reads out and the final state back, all inside the
    timed region.  The steps run as a serving loop pipelines them: two device buffer sets, the
    H2D copies of a step on one stream, the call on `stream`, the D2H reads on a third, ordered
    by events, so that both PCIe directions and the GPU work at the same time.  The region runs
    from the first copy of the first step to the last read of the last one (pipeline fill and
    drain included).  Each step moves ~290 MB of fresh input, more than L2 holds, so no flush."""
    names = ("q", "k", "v", "b", "a", "s0")
    host = {n: t[n].cpu().pin_memory() for n in names}
    sets = [t, {n: torch.empty_like(t[n]) for n in names + ("out", "fin")}]
    hres = [(torch.empty(t["out"].shape, dtype=t["out"].dtype).pin_memory(),
             torch.empty(t["fin"].shape, dtype=t["fin"].dtype).pin_memory()) for _ in sets]
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = sum(x.numel() * x.element_size() for x in hres[0])
    calls = [gdr.prepare_chunk_fwd(d["q"], d["k"], d["v"], d["b"], d["a"], d["s0"], None, w.scale, prologue=pro,
                                   out=d["out"], final_state=d["fin"], stream=stream) for d in sets]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in sets]    # the set's inputs landed
    ev_done = [torch.cuda.Event() for _ in sets]  # the call on the set finished (inputs free, results ready)
    ev_out = [torch.cuda.Event() for _ in sets]   # the set's results are back in host memory

    def run(K):
        for i in range(K):
            j = i % 2
            d = sets[j]
            if i >= 2:
                s_in.wait_event(ev_done[j])  # the call two steps back has read this set's inputs
            with torch.cuda.stream(s_in):
                for n in names:
                    d[n].copy_(host[n], non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])  # this set's results of two steps back are read
            calls[j]()
            ev_done[j].record(stream)
            s_out.wait_event(ev_done[j])
            with torch.cuda.stream(s_out):
                hres[j][0].copy_(d["out"], non_blocking=True)
                hres[j][1].copy_(d["fin"], non_blocking=True)
                ev_out[j].record(s_out)

    steps = max(3, min(args.steps, 10))
    run(2)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    run(steps)
    for e in ev_out:
        stream.wait_event(e)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = all_max(t0.elapsed_time(t1), world) / steps
    tokens = int(w.lengths.sum())
    return {"value": world * tokens / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "pipeline": "2 buffer sets; H2D, call and D2H on three streams", "l2": "inputs larger than L2"}, steps


def bench_decode(gdr, name, args, world, rank, clk, flush, stream, peaks, rotate: int = 4):
    """One decode call per step.  The state a call touches (67 MB for the decode workload)
    fits in L2, so instead of a flush the steps rotate over `rotate` separate copies of the
    pool: each call reads fresh state and pays the write-back of the previous call's state,
    as a serving loop does."""
    spec = name == "decode_spec"
    if name == "decode_no_gate":
        # the decode workload with g = NULL (hasGamma = 0): the D = 128 kernel's build without the decay
        wd = workloads.generate("decode", seed=1 + 1000 * rank)
        wd.g = None
    elif spec:
        # speculative decoding: 64 sequences verify 4 draft tokens each, every token with its own slot (the
        # previous step's A of them accepted); gdr_recurrent_step_spec
        wd = workloads.random_case(B=64, Nk=16, Nv=32, S=4, Dk=128, Dv=128, seed=6 + 1000 * rank, slots=64 * 4 + 64,
                                   share_slot=False, fd=np.float32)
        wd.accepted = np.random.default_rng([6 + 1000 * rank, 3]).integers(1, 5, size=64).astype(np.int32)
    else:
        wd = workloads.generate(name, seed=(1 if name == "decode" else 4) + 1000 * rank)
    dq, dk, dv, db = bf16_dev(wd.q), bf16_dev(wd.k), bf16_dev(wd.v), bf16_dev(wd.b)
    dg = f32_dev(wd.g) if wd.g is not None else None
    dgk = f32_dev(wd.gk) if wd.gk is not None else None
    pools = [bf16_dev(wd.pool) for _ in range(rotate)]
    idx = torch.from_numpy(wd.indices).cuda()
    lens = torch.from_numpy(wd.lengths).cuda()
    acc = torch.from_numpy(wd.accepted).cuda()
    dout = torch.empty((wd.B, wd.Nv, wd.S, wd.Dv), dtype=torch.bfloat16, device="cuda")
    dpro = gdr.Prologue(l2norm_qk=True, eps=1e-6, beta_logits=True)
    calls = [gdr.prepare_recurrent_step(dq, dk, dv, db, dg, dgk, pool, idx, lens, acc, wd.scale, prologue=dpro,
                                        out=dout, per_token=spec) for pool in pools]
    for i in range(args.warmup):
        calls[i % rotate]()
    barrier(world)
    torch.cuda.synchronize()
    evs = []
    clk.active = True
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            calls[i % rotate]()
            e.record(stream)
            evs.append((s, e))
    torch.cuda.synchronize()
    barrier(world)
    times = [s.elapsed_time(e) for s, e in evs]
    single_ms = all_max(sum(times), world) / args.steps
    # the serving loop: the same calls back to back inside one event pair (no host gap inside the region)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for i in range(args.steps):
            calls[i % rotate]()
        e.record(stream)
    torch.cuda.synchronize()
    clk.active = False
    barrier(world)
    d_ms = all_max(s.elapsed_time(e), world) / args.steps
    nb = algorithmic_decode_bytes(wd)
    if spec:  # one state read per sequence and head, one state written per processed token
        nb["state"] = int((1 + wd.lengths).sum()) * wd.Nv * wd.Dk * wd.Dv * 2
    gbs = nb["state"] / (d_ms / 1e3) / 1e9
    tot = (nb["state"] + nb["io"]) / (d_ms / 1e3) / 1e9
    return {"workload": f"B={wd.B} S={wd.S} Nk={wd.Nk} Nv={wd.Nv} D={wd.Dk} bf16, pool of {wd.pool.shape[0]} slots"
                        + (", per-key gate" if wd.gk is not None else "")
                        + (", no gate (g = NULL)" if wd.g is None else "") + ", fused prologue"
                        + (", per-token slots, accepted ~ U[1, 4] (speculative decoding)" if spec else ""),
            "l2": f"{rotate} rotating pool copies (fresh state every call), no flush",
            "timing": f"{args.steps} calls back to back inside one event pair; us_per_call_single: each call inside "
                      "its own event pair",
            "us_per_call": d_ms * 1e3, "us_per_call_single": single_ms * 1e3, "steps_per_s": world * 1e3 / d_ms,
            "state_GBps": gbs, "state_frac_of_hbm": gbs / peaks["hbm_gbs"],
            "roofline": {"bound": "hbm", "achieved": tot, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": tot / peaks["hbm_gbs"], "traffic": profiled_traffic(name),
                         "algorithmic_bytes_per_launch": nb["state"] + nb["io"]}}, 2 * args.steps


def run_ours(args, world, rank, local):
    import gated_deltanet_gdr_b200 as gdr
    gdr.lib()  # fails loudly if the library is missing
    peaks = measured_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clk = ClockSampler(local).__enter__()
    line = {"metric": METRIC, "value": None, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
    launches = 0
    if args.only in ("all", "prefill"):
        fields, w, t, pro, _ = bench_prefill(gdr, args, world, rank, clk, flush, stream, peaks)
        line.update(fields)
        launches += fields.pop("gpu_launches")
        if not args.no_e2e:
            line["e2e"], n = bench_e2e(gdr, args, world, w, t, pro, flush, stream)
            launches += prefill_kernels(gdr, w) * n
        if not args.no_epilogue:
            line["prefill_epilogue"], n = bench_prefill_epilogue(gdr, args, world, w, t, pro, flush, stream, peaks)
            launches += n
        line["prefill_no_gate"], n = bench_prefill_no_gate(gdr, args, world, w, t, flush, stream, peaks)
        launches += n
        del t
    if args.only in ("all", "prefill_b1"):
        line["prefill_b1"], n = bench_prefill_b1(gdr, args, world, rank, flush, stream, peaks)
        launches += n
    if args.only in ("all", "varlen"):
        line["varlen"], n = bench_varlen(gdr, args, world, rank, flush, stream, peaks)
        launches += n
    if args.only in ("all", "conv1d"):
        line["conv1d"], n = bench_conv1d(gdr, args, world, rank, flush, stream, peaks)
        launches += n
    if args.only in ("all", "f16"):
        line["f16"], n = bench_f16(gdr, args, world, rank, flush, stream, peaks)
        launches += n
    decode = {}
    for name in ("decode", "decode_gk", "decode_spec", "decode_no_gate"):
        if args.only in ("all", name) or (name == "decode_no_gate" and args.only == "decode"):
            decode[name], n = bench_decode(gdr, name, args, world, rank, clk, flush, stream, peaks)
            launches += n
    if decode:
        line["decode"] = decode
    clk.__exit__(None, None, None)
    if gdr.get_error() != 0:
        raise RuntimeError("device error word set during the benchmark")
    line["gpu_launches"] = launches
    line["clocks"] = clk.summary()
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only in ("all", "prefill"):
        line["cpu_baseline"] = cpu_baseline_fields()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (for profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg (profiling runs)")
    ap.add_argument("--no-epilogue", action="store_true",
                    help="skip the prefill line with the fused gated RMSNorm epilogue (profiling runs)")
    ap.add_argument("--only", choices=["all", "prefill", "prefill_b1", "decode", "decode_gk", "decode_spec",
                                       "conv1d", "f16", "varlen"], default="all",
                    help="run one workload only (profiling runs); the default runs all")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup() if args.impl == "ours" or int(os.environ.get("WORLD_SIZE", "1")) > 1 \
        else (1, 0, 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
