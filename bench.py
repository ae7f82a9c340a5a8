#!/usr/bin/env python
"""Benchmark of the KDA forward hot path on B200.

A step is one ``kda_chunk_fwd`` call over the prefill workload: B=4 sequences
of T=4096 tokens, H=16 heads, dk=dv=128, bf16 q/k/v, fp32 gates and state,
S0 ~ N(0, 0.1^2). The headline value is prefill tokens/s (B*T per step over
the whole job). The decode workload (N=256 sequences, H=32, 1024 consecutive
``kda_decode_step`` calls captured in one CUDA graph) is measured in the same
run and reported under "decode".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]
For N > 1 launch with torchrun (one rank per GPU, weak scaling: every rank
runs its own batch; the only collectives are the barrier and the max-reduce
of the timings).

``--impl reference`` times the fp64 CPU oracle (the slow, obviously correct
definition of the recurrence) on the host cores, the whole prefill workload per
step (rank 0 only under torchrun).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s + decode tokens/s on 1 B200; % of tensor/HBM roofline"
PREFILL = dict(B=4, T=4096, H=16, s0_std=0.1, la_range=(0.001, 0.1), seed=20261)
DECODE = dict(N=256, H=32, steps=1024, s0_std=0.1, la_range=(0.001, 0.1), seed=20263)
VARLEN = dict(n_seqs=64, len_range=(512, 16384), H=32, la_range=(0.001, 0.1), seed=20262)
LONG = dict(T_call=65536, calls=16, H=32, la_range=(0.0001, 0.05), seed=20264)
L2_FLUSH_BYTES = 256 << 20  # larger than the 126 MB L2
D = 128
# algorithmic bytes (single pass) per token-head: q,k,v,o bf16 + log_alpha fp32 + beta fp32
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 4 + 4 + D * 2  # 1540
STATE_BYTES = D * D * 4
PAGES_FLOPS_PER_TOKEN_HEAD = 6 * D * D + 3 * 64 * D + 64 * 64  # 6Td^2 + 3TCd + TC^2 per token
DECODE_BYTES_PER_HEAD_STEP = 2 * STATE_BYTES + PREFILL_BYTES_PER_TOKEN_HEAD  # 132612
# gate bytes per token-head in each layout of the forget gate (the rest is 1028 B)
GATE_BYTES = {"channel": D * 4, "channel_bf16": D * 2, "head": 4, "none": 0}
GATE_MODELS = {"channel_bf16": "KDA with a bf16 per-channel gate",
               "head": "Gated DeltaNet (one forget rate per head)",
               "none": "DeltaNet (no forget gate)"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons while the timed region runs.

    Uses NVML from a background thread every 5 ms (the timed regions are tens
    of milliseconds); falls back to `nvidia-smi -lms 200` when NVML is absent.
    """

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index: int, period_s: float = 0.005):
        import threading

        self.samples, self.reasons, self.smax = [], set(), None
        self.proc = self.thread = None
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        try:
            import pynvml

            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
            self.stop_evt = threading.Event()

            def run():
                while not self.stop_evt.is_set():
                    self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM)))
                    mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                    for name, bit in self.REASONS.items():
                        if mask & bit:
                            self.reasons.add(name)
                    self.stop_evt.wait(period_s)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
        except Exception:  # NVML unavailable: nvidia-smi loop
            fields = "clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown," \
                     "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
                     "clocks_event_reasons.sw_power_cap"
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", uuid, "--query-gpu=" + fields, "--format=csv,noheader,nounits",
                     "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in out.strip().splitlines():
                parts = [x.strip() for x in line.split(",")]
                try:
                    self.samples.append(float(parts[0]))
                    self.smax = float(parts[1])
                except (ValueError, IndexError):
                    continue
                for name, val in zip(names, parts[2:]):
                    if val.lower() == "active":
                        self.reasons.add(name)
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.smax, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# A hardware or thermal slowdown, or an SM clock far below its maximum with no reason
# reported (a clock left locked), rejects a timed region; a power cap does not.
BAD_CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clock_rejected(clk: dict) -> bool:
    if any(r in BAD_CLOCK_REASONS for r in clk.get("reasons") or []):
        return True
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    return bool(mhz and mx and mhz < 0.8 * mx and not clk.get("reasons"))


# ------------------------------------------------------------------ ncu traffic
# DRAM bytes (read + write) per launch from one ncu capture of the B=4, T=4096,
# H=16 step and of one N=256, H=32 decode step (profiles/). Each figure is
# reported only while the sources of its kernels hash to the build it was taken
# from; otherwise the roofline's traffic is null.
TRAFFIC_SOURCES = {"prefill": ("prefill_tc.cu", "tc_ptx.cuh", "kda_internal.cuh"),
                   "decode": ("decode.cu", "kda_internal.cuh")}
TRAFFIC = {"prefill": {"source_hash": "c6cc0cd03f29ccb3", "shape": (4, 4096, 16),  # prep + chain
                       "bytes": 271514240 + 220421120 + 341894443 + 52838272},
           "decode": {"source_hash": "2f2a24e4a98dd528", "shape": (256, 32),
                      "bytes": 547406592 + 480025216}}


def source_hash(kind: str) -> str:
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_101_b200", "csrc")
    for name in TRAFFIC_SOURCES[kind]:
        h.update(name.encode())
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic(kind: str, override, shape):
    """DRAM bytes per launch: the override, else the committed capture if it was taken
    from the current sources at this shape, else None."""
    if override is not None:
        return override
    t = TRAFFIC[kind]
    return t["bytes"] if t["source_hash"] == source_hash(kind) and tuple(shape) == t["shape"] else None


# ------------------------------------------------------------------ helpers
def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_steps(fn, steps, warmup, stream, flush=None, name="kda"):
    """Runs fn warmup times, then times each of `steps` calls with CUDA events
    on `stream` (L2 flushed before each call, outside the events). Returns ms list.
    The warm-up and the timed calls sit in NVTX ranges `name`/warmup and `name`/timed
    (for `ncu --nvtx --nvtx-include`)."""
    with torch.cuda.nvtx.range(f"{name}/warmup"):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
    times = []
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with torch.cuda.nvtx.range(f"{name}/timed"), torch.cuda.stream(stream):
        for a, b in evs:
            if flush is not None:
                flush()
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize()
    for a, b in evs:
        times.append(a.elapsed_time(b))
    return times


def cpu_oracle_sample(inp, o, S_T, min_s: float = 10.0, max_reps: int = 40):
    """Times the fp64 oracle on the whole prefill batch (every sequence and head),
    repeated until at least ``min_s`` seconds of CPU time (at most ``max_reps`` passes).

    The oracle's last result is also compared with the step's own outputs ``o`` and
    ``S_T`` (the same inputs and S0), element by element over every output: relative L2
    error and max-abs error, next to the bf16 bar the parity tests hold them to."""
    import oracle

    args = [oracle._f64(t) for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)]
    threads = oracle.default_threads()
    B, T, H = inp.q.shape[:3]
    reps, total = 0, 0.0
    while total < min_s and reps < max_reps:
        t0 = time.perf_counter()
        ref = oracle.kda_fwd(*args, threads=threads)
        total += time.perf_counter() - t0
        reps += 1
    cpu = {"value": B * T * reps / total, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"the whole prefill batch ({B} sequences x {T} tokens x {H} heads, bf16 "
                     f"inputs widened to fp64) {reps} times, {total:.1f} s on {threads} threads"}
    parity = {"against": "the fp64 oracle on the same inputs, every element of o and S_T",
              "bar": {"rel_l2": 1e-2, "max_abs_over_max_ref": 2e-2}}
    for name, got, want in (("o", o, ref[0]), ("S_T", S_T, ref[1])):
        x = got.detach().to("cpu", torch.float64).numpy()
        diff = x - want
        mref = float(np.max(np.abs(want)))
        parity[name] = {"rel_l2": float(np.linalg.norm(diff) / np.linalg.norm(want)),
                        "max_abs": float(np.max(np.abs(diff))), "max_ref": mref,
                        "finite": bool(np.all(np.isfinite(x)))}
    parity["pass"] = all(parity[n]["finite"] and parity[n]["rel_l2"] <= 1e-2
                         and parity[n]["max_abs"] <= 2e-2 * parity[n]["max_ref"] for n in ("o", "S_T"))
    return cpu, parity


def prefill_config(world: int) -> dict:
    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    return {"workload": f"KDA prefill B={B} T={T} H={H} d=128 C=64, bf16 q/k/v, fp32 log_alpha/beta/"
                        "state, S0~N(0,0.1^2)",
            "global_batch": B * world, "seq_len": T, "parallelism": f"dp{world}",
            "l2": f"flushed before every step (256 MiB write); the step moves "
                  f"{(PREFILL_BYTES_PER_TOKEN_HEAD * B * T * H + 2 * STATE_BYTES * B * H) / 1e6:.0f} MB"}


# ------------------------------------------------------------------ arms
def run_reference(args, rank, world):
    """The fp64 CPU oracle timed on host cores, the whole prefill workload per step."""
    if rank != 0:
        return
    from gated_delta_rule_101_b200.inputs import prefill_inputs

    inp = prefill_inputs(B=PREFILL["B"], T=PREFILL["T"], H=PREFILL["H"], dtype=torch.bfloat16,
                         s0_std=PREFILL["s0_std"], la_range=PREFILL["la_range"],
                         seed=PREFILL["seed"], device="cpu")
    import oracle

    H = inp.q.shape[2]
    args_np = [oracle._f64(t) for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)]
    threads = oracle.default_threads()
    for _ in range(args.warmup):
        oracle.kda_fwd(*args_np, threads=threads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.kda_fwd(*args_np, threads=threads)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    tokens = PREFILL["B"] * PREFILL["T"] * args.steps
    value = tokens / total
    sample = (f"the whole prefill workload per step ({PREFILL['B']} sequences x {PREFILL['T']} "
              f"tokens x {H} heads, bf16 inputs widened to fp64), {threads} threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": prefill_config(world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def other_prefill_workloads(kda, dev, stream, flush, pk, world, rank):
    """The packed variable-length batch and the long-context sequence, each timed on
    the device (CUDA events on the launching stream, L2 flushed before the packed call;
    the long-context calls stream 3.2 GB of inputs each, far more than L2)."""
    from gated_delta_rule_101_b200.inputs import cu_from_lengths, prefill_inputs, varlen_lengths

    out = {}
    barrier(world)
    # packed: 64 sequences, lengths ~ U[512, 16384], H = 32, S0 = 0
    lengths = varlen_lengths(VARLEN["n_seqs"], *VARLEN["len_range"], seed=VARLEN["seed"] + 1000 * rank)
    cu = cu_from_lengths(lengths)
    T, H = int(cu[-1]), VARLEN["H"]
    inp = prefill_inputs(T=T, H=H, cu_seqlens=cu, dtype=torch.bfloat16, la_range=VARLEN["la_range"],
                         seed=VARLEN["seed"] + 1000 * rank, device=dev)
    o = torch.empty_like(inp.v)
    S_T = torch.empty(len(lengths), H, 128, 128, device=dev)
    ws = torch.empty(kda.workspace_size(1, T, H, len(lengths)), dtype=torch.uint8, device=dev)
    n_l = kda.chunk_fwd_launches(1, T, H, len(lengths))

    def call():
        kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, cu_seqlens=inp.cu_seqlens,
                      out=o, state_out=S_T, workspace=ws, stream=stream)

    times = time_steps(call, 3, 3, stream, flush, name="kda.varlen")
    ms = max_over_ranks(sum(times), world, dev) / len(times)
    alg = PREFILL_BYTES_PER_TOKEN_HEAD * T * H + 2 * STATE_BYTES * len(lengths) * H
    out["varlen"] = {"value": T * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_call": ms,
                     "config": {"workload": f"KDA packed prefill, {len(lengths)} sequences "
                                            f"(lengths U[{VARLEN['len_range'][0]}, "
                                            f"{VARLEN['len_range'][1]}], {T} tokens), H={H}, bf16",
                                "l2": "flushed before every call; inputs far above L2"},
                     "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9,
                                  "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                  "alg_bytes_per_launch": alg},
                     "gpu_launches": n_l * len(times)}
    del inp, o, S_T, ws
    torch.cuda.empty_cache()
    # long context: 2^20 tokens as 16 calls of 65,536 with the state carried in place
    Tc, H, calls = LONG["T_call"], LONG["H"], LONG["calls"]
    inps = [prefill_inputs(B=1, T=Tc, H=H, dtype=torch.bfloat16, la_range=LONG["la_range"],
                           seed=LONG["seed"] * 100 + c + 1000 * rank, device=dev) for c in range(2)]
    S = torch.zeros(1, H, 128, 128, device=dev)
    o = torch.empty_like(inps[0].v)
    ws = torch.empty(kda.workspace_size(1, Tc, H), dtype=torch.uint8, device=dev)
    n_l = kda.chunk_fwd_launches(1, Tc, H)

    def sequence():
        S.zero_()
        for c in range(calls):  # two input sets alternate: the data differs, the work does not
            x = inps[c % 2]
            kda.chunk_fwd(x.q, x.k, x.v, x.log_alpha, x.beta, S, out=o, state_out=S, workspace=ws,
                          stream=stream)

    times = time_steps(sequence, 2, 3, stream, name="kda.long_context")
    ms = max_over_ranks(sum(times), world, dev) / len(times)
    alg = (PREFILL_BYTES_PER_TOKEN_HEAD * Tc * H + 2 * STATE_BYTES * H) * calls
    out["long_context"] = {"value": Tc * calls * world / (ms * 1e-3), "unit": "tokens/s",
                           "ms_per_sequence": ms, "ms_per_call": ms / calls,
                           "config": {"workload": f"KDA long-context prefill, one sequence of "
                                                  f"{Tc * calls} tokens as {calls} calls of {Tc} "
                                                  f"with S_T carried as the next S0, H={H}, bf16",
                                      "l2": "not flushed; each call streams 3.2 GB of inputs"},
                           "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9,
                                        "peak": pk["hbm_gbs"], "unit": "GB/s",
                                        "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                        "alg_bytes_per_launch": alg / calls},
                           "gpu_launches": n_l * calls * len(times)}
    del inps, S, o, ws
    torch.cuda.empty_cache()
    return out


def gate_layout_workloads(kda, dev, stream, flush, pk, world, rank):
    """The step's workload with the forget gate in the other layouts (bf16 per channel,
    one rate per head, none), each call timed on the device with L2 flushed before it."""
    from gated_delta_rule_101_b200.inputs import prefill_inputs

    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    ws = torch.empty(kda.workspace_size(B, T, H), dtype=torch.uint8, device=dev)
    n_l = kda.chunk_fwd_launches(B, T, H)
    out = {}
    for gate, model in GATE_MODELS.items():
        inp = prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=PREFILL["s0_std"],
                             la_range=PREFILL["la_range"], seed=PREFILL["seed"] + 1000 * rank,
                             gate=gate, device=dev)
        o = torch.empty_like(inp.v)
        S_T = torch.empty_like(inp.S0)

        def call():
            kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, out=o, state_out=S_T,
                          workspace=ws, stream=stream)

        barrier(world)
        times = time_steps(call, 10, 3, stream, flush, name=f"kda.gate.{gate}")
        ms = max_over_ranks(sum(times), world, dev) / len(times)
        alg = (PREFILL_BYTES_PER_TOKEN_HEAD - GATE_BYTES["channel"] + GATE_BYTES[gate]) * B * T * H \
            + 2 * STATE_BYTES * B * H
        out[gate] = {"value": B * T * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_call": ms,
                     "config": {"workload": f"{model}: prefill B={B} T={T} H={H} d=128, bf16",
                                "l2": "flushed before every call"},
                     "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9,
                                  "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                  "alg_bytes_per_launch": alg},
                     "gpu_launches": n_l * len(times)}
        del inp, o, S_T
    del ws
    torch.cuda.empty_cache()
    return {"gate_layouts": out}


def chunk_size_workloads(kda, dev, stream, flush, pk, world, rank):
    """The step's workload at each chunk length the library takes (C = 32 and 64), for
    bf16 and fp32 inputs. bf16 at C = 64 is the step itself (tensor cores); the other
    three run on the CUDA-core kernel. Each call timed on the device, L2 flushed."""
    from gated_delta_rule_101_b200.inputs import prefill_inputs

    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    out = {}
    for dtype, name, esize in ((torch.bfloat16, "bf16", 2), (torch.float32, "f32", 4)):
        inp = prefill_inputs(B=B, T=T, H=H, dtype=dtype, s0_std=PREFILL["s0_std"],
                             la_range=PREFILL["la_range"], seed=PREFILL["seed"] + 1000 * rank,
                             device=dev)
        o = torch.empty_like(inp.v)
        S_T = torch.empty_like(inp.S0)
        alg = (PREFILL_BYTES_PER_TOKEN_HEAD + 4 * 128 * (esize - 2)) * B * T * H + 2 * STATE_BYTES * B * H
        for C in (32, 64):
            ws = torch.empty(max(kda.workspace_size(B, T, H, 0, dtype, C), 16), dtype=torch.uint8, device=dev)
            n_l = kda.chunk_fwd_launches(B, T, H, dtype=dtype, C=C)

            def call():
                kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, out=o, state_out=S_T,
                              workspace=ws, stream=stream, C=C)

            reps = 10 if (name == "bf16" and C == 64) else 3
            barrier(world)
            times = time_steps(call, reps, 3, stream, flush, name=f"kda.chunk{C}.{name}")
            ms = max_over_ranks(sum(times), world, dev) / len(times)
            kernel = "kda_prep_kernel + kda_chain_kernel (tensor cores)" if (name == "bf16" and C == 64) \
                else "prefill_simt_kernel (CUDA cores, fp32)"
            out[f"C{C}_{name}"] = {
                "value": B * T * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_call": ms,
                "config": {"workload": f"KDA prefill B={B} T={T} H={H} d=128, {name} inputs, chunks of {C}",
                           "l2": "flushed before every call"},
                "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                             "alg_bytes_per_launch": alg, "kernel": kernel},
                "gpu_launches": n_l * len(times)}
            del ws
        del inp, o, S_T
    torch.cuda.empty_cache()
    return {"chunk_sizes": out}


def fused_io_workload(kda, dev, stream, flush, pk, world, rank):
    """The step's shape through kda_chunk_fwd_io with every fused step of the layer:
    the gate's pre-activation z as bf16 logits (alpha = sigmoid(z)), q and k
    L2-normalised in the kernel, beta as logits, and the output RMSNorm and sigmoid
    output gate. Inputs: q, k, v, output gate ~ N(0, 1) bf16 (q, k not normalised),
    z ~ U(2, 7) bf16, beta logits ~ N(0, 1), RMSNorm weights ~ U(0.5, 1.5),
    S0 ~ N(0, 0.1^2). Timed like the step (L2 flushed before each call)."""
    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    g = torch.Generator(device=dev).manual_seed(PREFILL["seed"] + 77 + 1000 * rank)
    shape = (B, T, H, 128)
    bf = lambda: torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    q, k, v, og = bf(), bf(), bf(), bf()
    z = (torch.rand(shape, generator=g, device=dev) * 5 + 2).to(torch.bfloat16)
    b = torch.randn((B, T, H), generator=g, device=dev)
    w = torch.rand(128, generator=g, device=dev) + 0.5
    S0 = 0.1 * torch.randn((B, H, 128, 128), generator=g, device=dev)
    ws = torch.empty(kda.workspace_size(B, T, H), dtype=torch.uint8, device=dev)
    o, S_T = torch.empty_like(v), torch.empty_like(S0)

    def call():
        kda.chunk_fwd(q, k, v, z, b, S0, out=o, state_out=S_T, workspace=ws, stream=stream,
                      gate_logits=True, qk_l2norm=True, beta_logits=True, out_gate=og,
                      out_norm_weight=w)

    barrier(world)
    times = time_steps(call, 10, 3, stream, flush, name="kda.fused_io")
    ms = max_over_ranks(sum(times), world, dev) / len(times)
    # q, k, v, o, output gate and z in bf16, beta fp32; plus S0 and S_T
    per_tok = 4 * 256 + 256 + 256 + 4
    alg = per_tok * B * T * H + 2 * STATE_BYTES * B * H
    # the same layer steps as separate passes: normalise q and k (read + write), log
    # sigmoid of z (bf16 in, fp32 log_alpha out), sigmoid of beta, the KDA call with an
    # fp32 gate, then RMSNorm and the output gate (read o and the gate, write o)
    unfused = (2 * 512 + (256 + 512) + 8 + PREFILL_BYTES_PER_TOKEN_HEAD + 3 * 256) * B * T * H
    n_l = kda.chunk_fwd_launches(B, T, H, out_epilogue=True)
    del q, k, v, og, z, b, S0, ws, o, S_T
    torch.cuda.empty_cache()
    return {"fused_io": {
        "value": B * T * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_call": ms,
        "config": {"workload": f"KDA prefill B={B} T={T} H={H} d=128, bf16, with the layer's gate "
                               "pre-activation, q/k L2Norm, beta sigmoid, output RMSNorm and sigmoid "
                               "gate fused", "l2": "flushed before every call"},
        "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                     "alg_bytes_per_launch": alg},
        "bytes_per_token_head": per_tok, "unfused_bytes_per_token_head": unfused // (B * T * H),
        "gpu_launches": n_l * len(times)}}


def backward_workload(kda, dev, stream, flush, pk, world, rank):
    """kda_chunk_bwd on the step's shape (B=4, T=4096, H=16, bf16 inputs, fp32 per-channel
    gate): the gradients of sum(o * dout) + sum(S_T * dS_T), dout ~ N(0, 1) bf16, dS_T ~
    N(0, 1). Timed like the step (L2 flushed before each call)."""
    from gated_delta_rule_101_b200.inputs import prefill_inputs

    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    inp = prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=PREFILL["s0_std"],
                         la_range=PREFILL["la_range"], seed=PREFILL["seed"] + 2000 + 1000 * rank, device=dev)
    g = torch.Generator(device=dev).manual_seed(PREFILL["seed"] + 3000 + 1000 * rank)
    dout = torch.randn(inp.v.shape, generator=g, device=dev).to(torch.bfloat16)
    dS_T = torch.randn(inp.S0.shape, generator=g, device=dev)
    ws = torch.empty(kda.bwd_workspace_size(B, T, H), dtype=torch.uint8, device=dev)

    def call():
        kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T, workspace=ws,
                      stream=stream)

    barrier(world)
    times = time_steps(call, 3, 1, stream, flush, name="kda.backward")
    ms = max_over_ranks(sum(times), world, dev) / len(times)
    # inputs q, k, v, dout bf16, log_alpha fp32, beta; outputs dq, dk, dv, dlog_alpha fp32,
    # dbeta; plus S0, dS_T in and dS0 out
    per_tok = 4 * 256 + 512 + 4 + 4 * 512 + 4
    alg = per_tok * B * T * H + 3 * STATE_BYTES * B * H
    del inp, dout, dS_T, ws
    torch.cuda.empty_cache()
    return {"backward": {
        "value": B * T * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_call": ms,
        "config": {"workload": f"KDA backward (kda_chunk_bwd) B={B} T={T} H={H} d=128, bf16 inputs, "
                               "fp32 gradients", "l2": "flushed before every call"},
        "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                     "alg_bytes_per_launch": alg, "kernel": "kda_bwd_slice_kernel + kda_bwd_reduce_kernel"},
        "gpu_launches": 2 * len(times)}}


def run_kda(args, rank, world, local_rank):
    import gated_delta_rule_101_b200 as kda
    from gated_delta_rule_101_b200.inputs import decode_inputs, prefill_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    kda.lib()
    pk, pk_kind = peaks()
    stream = torch.cuda.Stream(device=dev)
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush = lambda: flush_buf.fill_(1)

    # ---------------- prefill (the step)
    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    inp = prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=PREFILL["s0_std"],
                         la_range=PREFILL["la_range"], seed=PREFILL["seed"] + 1000 * rank,
                         device=dev)
    o = torch.empty_like(inp.v)
    S_T = torch.empty_like(inp.S0)
    ws_n = kda.workspace_size(B, T, H, 0, torch.bfloat16)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, out=o, state_out=S_T,
                      workspace=ws, stream=stream)

    def timed_region():
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        clocks = ClockSampler(dev.index)
        t = time_steps(step, args.steps, args.warmup, stream, flush, name="kda.prefill")
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        return t, clocks.stop()

    times, clk = timed_region()
    # a rejected clock record on any rank re-measures once on every rank
    if max_over_ranks(float(clock_rejected(clk)), world, dev) > 0:
        first = clk
        times, clk = timed_region()
        clk["remeasured_after"] = {"sm_mhz": first.get("sm_mhz"), "reasons": first.get("reasons")}
    total_ms = max_over_ranks(sum(times), world, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * T * world
    value = tokens_per_step / (ms_per_step * 1e-3)
    launches_per_call = kda.chunk_fwd_launches(B, T, H)
    avg_kernel_s = sum(times) / len(times) * 1e-3
    alg_bytes = PREFILL_BYTES_PER_TOKEN_HEAD * B * T * H + 2 * STATE_BYTES * B * H
    achieved = alg_bytes / avg_kernel_s / 1e9
    pages_flops = PAGES_FLOPS_PER_TOKEN_HEAD * B * T * H
    tflops = pages_flops / avg_kernel_s / 1e12
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic("prefill", args.traffic, (B, T, H)),
                "peak_source": pk_kind,
                "kernel": "kda_chunk_fwd (one call, timed as a whole): "
                          + {1: "kda_fused_kernel", 2: "kda_prep_kernel + kda_chain_kernel",
                             4: "kda_prep_kernel + kda_seg_pass_kernel x2 + kda_seg_combine_kernel"}
                          .get(launches_per_call, f"{launches_per_call} kernels"),
                "alg_bytes_per_launch": alg_bytes,
                "tensor_pages_flops": {"achieved_tflops": tflops, "peak": pk["bf16_tflops"],
                                       "frac": tflops / pk["bf16_tflops"],
                                       "flops_per_launch": pages_flops}}

    # ---------------- e2e through host buffers (pinned), copies inside the timed region
    host = {n: getattr(inp, n).cpu().pin_memory() for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    dbuf = {n: torch.empty_like(getattr(inp, n)) for n in host}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    s_h = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + s_h.numel() * s_h.element_size()

    # One sequence at a time on three streams: the host-to-device copy of sequence b + 1
    # and the device-to-host copy of sequence b - 1 (separate copy engines) run while
    # sequence b is computed. Each step starts after the previous one has ended.
    copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(B)]
    ev_done = [torch.cuda.Event() for _ in range(B)]

    def e2e_step():
        copy_in.wait_stream(stream)
        copy_out.wait_stream(stream)
        for b in range(B):
            with torch.cuda.stream(copy_in):
                for n, t in host.items():
                    dbuf[n][b].copy_(t[b], non_blocking=True)
                ev_in[b].record(copy_in)
            stream.wait_event(ev_in[b])
            sl = {n: dbuf[n][b:b + 1] for n in dbuf}
            kda.chunk_fwd(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], sl["S0"],
                          out=o[b:b + 1], state_out=S_T[b:b + 1], workspace=ws, stream=stream)
            ev_done[b].record(stream)
            copy_out.wait_event(ev_done[b])
            with torch.cuda.stream(copy_out):
                o_h[b].copy_(o[b], non_blocking=True)
                s_h[b].copy_(S_T[b], non_blocking=True)
        stream.wait_stream(copy_out)

    e2e = None
    if not args.no_e2e:
        e2e_steps = max(3, min(args.steps, 10))
        barrier(world)
        e_times = time_steps(e2e_step, e2e_steps, max(3, args.warmup // 2), stream, name="kda.e2e")
        barrier(world)
        e_ms = max_over_ranks(sum(e_times), world, dev) / e2e_steps
        e2e = {"value": tokens_per_step / (e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "pipeline": "per sequence: pinned host-to-device copies, kda_chunk_fwd (B=1) and "
                           "device-to-host copies of o and S_T on three streams"}
    del host, dbuf

    # ---------------- the gate layouts, next to the step they vary and before the decode
    # graph (whose power draw would otherwise still hold the clocks down)
    extra = {}
    if not args.no_extra:
        extra.update(gate_layout_workloads(kda, dev, stream, flush, pk, world, rank))

    # ---------------- decode (N=256, H=32, 1024 steps in one CUDA graph)
    decode = None
    if not args.no_decode:
        N, Hd, nsteps = DECODE["N"], DECODE["H"], args.decode_steps
        dinp = decode_inputs(steps=nsteps, N=N, H=Hd, dtype=torch.bfloat16, s0_std=DECODE["s0_std"],
                             la_range=DECODE["la_range"], seed=DECODE["seed"] + 1000 * rank,
                             device=dev)
        S = dinp.S.clone()
        od = torch.empty_like(dinp.v)
        with torch.cuda.stream(stream):
            kda.decode_step(dinp.q[0], dinp.k[0], dinp.v[0], dinp.log_alpha[0], dinp.beta[0],
                            S.clone(), out=od[0], stream=stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for t in range(nsteps):
                kda.decode_step(dinp.q[t], dinp.k[t], dinp.v[t], dinp.log_alpha[t], dinp.beta[t], S,
                                out=od[t], stream=stream)
        barrier(world)
        dclk = ClockSampler(dev.index)
        d_times = time_steps(graph.replay, 2, 1, stream, flush, name="kda.decode")
        dclk = dclk.stop()
        barrier(world)
        d_ms = max_over_ranks(sum(d_times), world, dev) / len(d_times)
        per_launch = d_ms * 1e-3 / nsteps
        d_bytes = DECODE_BYTES_PER_HEAD_STEP * N * Hd
        d_ach = d_bytes / per_launch / 1e9
        decode = {"value": N * nsteps * world / (d_ms * 1e-3), "unit": "tokens/s",
                  "ms_per_graph": d_ms, "us_per_step": per_launch * 1e6,
                  "config": {"workload": f"KDA decode N={N} H={Hd} d=128, {nsteps} consecutive "
                                         "steps in one CUDA graph", "l2": "state 512 MiB > L2"},
                  "roofline": {"bound": "hbm", "achieved": d_ach, "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": d_ach / pk["hbm_gbs"],
                               "traffic": traffic("decode", args.decode_traffic, (N, Hd)), "peak_source": pk_kind,
                               "kernel": "kda_decode_step", "alg_bytes_per_launch": d_bytes},
                  "gpu_launches": nsteps * len(d_times), "clocks": dclk}
        del graph, dinp, S, od

    # ---------------- the other prefill workloads (reported beside the step, not the step)
    if not args.no_extra:
        extra.update(fused_io_workload(kda, dev, stream, flush, pk, world, rank))
        extra.update(chunk_size_workloads(kda, dev, stream, flush, pk, world, rank))
        extra.update(backward_workload(kda, dev, stream, flush, pk, world, rank))
        extra.update(other_prefill_workloads(kda, dev, stream, flush, pk, world, rank))

    cpu, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        torch.cuda.synchronize()
        cpu, parity = cpu_oracle_sample(inp, o, S_T)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": prefill_config(world),
                "roofline": roofline, "cpu_baseline": cpu, "parity": parity, "e2e": e2e,
                "gpu_launches": launches_per_call * args.steps, "clocks": clk, "decode": decode,
                **extra}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--decode-steps", type=int, default=DECODE["steps"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the packed, long-context and gate-layout prefill workloads")
    ap.add_argument("--shape", default=None,
                    help="B,T,H of the prefill step instead of 4,4096,16 (for profiling captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (for short profiling runs)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per prefill launch, if captured for the current sources")
    ap.add_argument("--decode-traffic", type=float, default=None,
                    help="ncu dram bytes per decode launch, if captured for the current sources")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.shape:
        try:
            B, T, H = (int(x) for x in args.shape.split(","))
        except ValueError:
            ap.error("--shape takes B,T,H")
        PREFILL.update(B=B, T=T, H=H)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "kda":
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_kda(args, rank, world, local_rank)
    finally:
        if world > 1 and args.impl == "kda":
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
