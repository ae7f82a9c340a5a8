"""Host-side rules of bench.py (no GPU needed)."""
import bench


def test_clock_record_rejection():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert not bench.clock_rejected(ok)
    # a power cap is kept; hardware and thermal slowdowns are not
    assert not bench.clock_rejected({"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clock_rejected({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [r]})
    # far below the maximum with no reason: a clock left locked
    assert bench.clock_rejected({"sm_mhz": 1100.0, "sm_max_mhz": 1965.0, "reasons": []})
    # no samples: nothing to reject on
    assert not bench.clock_rejected({"sm_mhz": None, "sm_max_mhz": None,
                                     "reasons": ["clock sampling unavailable"]})


def test_traffic_is_reported_only_for_the_captured_sources_and_shape():
    for kind in ("prefill", "decode"):
        t = bench.TRAFFIC[kind]
        same = t["source_hash"] == bench.source_hash(kind)
        assert bench.traffic(kind, None, t["shape"]) == (t["bytes"] if same else None)
        other = tuple(x + 1 for x in t["shape"])
        assert bench.traffic(kind, None, other) is None
    assert bench.traffic("prefill", 123, (1, 1, 1)) == 123  # an explicit capture overrides


def _fake_cuda(monkeypatch):
    """Runs bench.py's GPU arm on the CPU: CUDA streams, events and graphs become
    no-ops, the device becomes the CPU and libkda a stand-in that records its calls."""
    import contextlib
    import types

    import torch

    import gated_delta_rule_101_b200 as kda

    class Recorder:
        def __init__(self):
            self.calls = []

        def __getattr__(self, name):
            def call(*args):
                self.calls.append(name)
                return 0

            return call

    class Event:
        def __init__(self, **kw):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 0.25

    class Stream:
        cuda_stream = 0

        def __init__(self, *a, **kw):
            pass

        def wait_stream(self, other):
            pass

        def wait_event(self, event):
            pass

    class Graph:
        def replay(self):
            pass

    class Props:
        uuid = "00000000-0000-0000-0000-000000000000"

    cuda = types.SimpleNamespace(
        synchronize=lambda *a, **kw: None, Event=Event, Stream=Stream,
        stream=lambda s: contextlib.nullcontext(), current_stream=lambda *a, **kw: Stream(),
        set_device=lambda *a: None, get_device_properties=lambda i: Props(), CUDAGraph=Graph,
        graph=lambda g, **kw: contextlib.nullcontext(), empty_cache=lambda: None, nvtx=torch.cuda.nvtx)
    shim = types.ModuleType("torch_on_cpu")
    for k in dir(torch):
        if not k.startswith("__"):
            setattr(shim, k, getattr(torch, k))
    shim.device = lambda *a, **kw: torch.device("cpu")
    shim.cuda = cuda
    rec = Recorder()
    monkeypatch.setattr(bench, "torch", shim)
    monkeypatch.setattr(kda, "_lib", rec)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    for d, kw in ((bench.PREFILL, dict(B=2, T=130, H=2)), (bench.DECODE, dict(N=2, H=2, steps=3)),
                  (bench.VARLEN, dict(n_seqs=3, len_range=(5, 70), H=2)),
                  (bench.LONG, dict(T_call=128, calls=3, H=2))):
        for key, val in kw.items():
            monkeypatch.setitem(d, key, val)
    monkeypatch.setattr(bench, "L2_FLUSH_BYTES", 1 << 10)
    return rec


def _run_kda_line(**flags):
    import contextlib
    import io
    import json
    import types

    args = types.SimpleNamespace(steps=3, warmup=3, no_extra=False, no_cpu_baseline=True, no_e2e=False,
                                 no_decode=False, decode_steps=3, traffic=None, decode_traffic=None)
    for k, v in flags.items():
        setattr(args, k, v)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_kda(args, 0, 1, 0)
    return json.loads(out.getvalue().strip().splitlines()[-1])


def test_gpu_arm_runs_end_to_end_on_fakes(monkeypatch):
    rec = _fake_cuda(monkeypatch)
    line = _run_kda_line()
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
                "e2e", "gpu_launches", "clocks", "decode", "varlen", "long_context", "gate_layouts"):
        assert key in line, key
    assert set(line["gate_layouts"]) == {"channel_bf16", "head", "none"}
    for r in (line["roofline"], line["decode"]["roofline"]):
        assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert line["roofline"]["traffic"] is None  # captured at another shape
    assert {"kda_chunk_fwd", "kda_chunk_fwd_gated", "kda_decode_step"} <= set(rec.calls)
    # the other legs: fused layer steps, chunk lengths, backward; parity only with the oracle leg
    assert set(line["chunk_sizes"]) == {"C32_bf16", "C64_bf16", "C32_f32", "C64_f32"}
    for leg in (line["fused_io"], line["backward"], *line["chunk_sizes"].values()):
        assert {"value", "unit", "ms_per_call", "config", "roofline", "gpu_launches"} <= set(leg)
    assert {"kda_chunk_fwd_io", "kda_chunk_bwd"} <= set(rec.calls)
    assert line["parity"] is None and line["cpu_baseline"] is None
    assert {"h2d_bytes_per_step", "d2h_bytes_per_step", "pipeline"} <= set(line["e2e"])


def test_gpu_arm_remeasures_a_throttled_step(monkeypatch):
    _fake_cuda(monkeypatch)

    class Clocks:
        n = 0

        def __init__(self, index):
            pass

        def stop(self):
            Clocks.n += 1
            return {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                    "reasons": ["hw_thermal_slowdown"] if Clocks.n == 1 else []}

    monkeypatch.setattr(bench, "ClockSampler", Clocks)
    line = _run_kda_line(no_extra=True, no_decode=True, no_e2e=True)
    assert line["clocks"]["reasons"] == []
    assert line["clocks"]["remeasured_after"]["reasons"] == ["hw_thermal_slowdown"]
