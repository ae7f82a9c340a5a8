"""The Python binding's argument handling on the host (no GPU needed).

A recording stand-in replaces the loaded library: every ``kda_*`` call returns KDA_OK
and is logged, so these tests check which entry point the binding picks, what it
passes, and that malformed tensors are refused before any pointer reaches the library
(which trusts the sizes it is given). Tensors live on the CPU; nothing is launched.
"""
import pytest
import torch

import gated_delta_rule_101_b200 as kda


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            return 0

        return call


class _Stream:
    cuda_stream = 0


S = _Stream()


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(kda, "_lib", r)
    return r


def _names(rec):
    return [n for n, _ in rec.calls if n not in ("kda_chunk_fwd_workspace_size",)]


def _t(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype)


def _prefill(B=2, T=70, H=3, gate="channel", packed=False, dtype=torch.bfloat16):
    lead = (T,) if packed else (B, T)
    q = _t(*lead, H, 128, dtype=dtype)
    la = {"channel": _t(*lead, H, 128), "channel_bf16": _t(*lead, H, 128, dtype=torch.bfloat16),
          "head": _t(*lead, H), "none": None}[gate]
    return q, q.clone(), q.clone(), la, _t(*lead, H)


@pytest.mark.parametrize("gate,entry,code", [("channel", "kda_chunk_fwd", None),
                                             ("channel_bf16", "kda_chunk_fwd_gated", 1),
                                             ("head", "kda_chunk_fwd_gated", 2),
                                             ("none", "kda_chunk_fwd_gated", 3)])
def test_prefill_picks_the_entry_point_of_the_gate_layout(rec, gate, entry, code):
    q, k, v, la, b = _prefill(gate=gate)
    o, st = kda.chunk_fwd(q, k, v, la, b, stream=S)
    assert _names(rec) == [entry]
    args = rec.calls[-1][1]
    if code is not None:
        assert args[4] == code  # the kda_gate argument follows log_alpha
    assert o.shape == q.shape and st.shape == (2, 3, 128, 128)


def test_prefill_call_patterns_of_the_tests_and_the_bench(rec):
    q, k, v, la, b = _prefill()
    S0 = _t(2, 3, 128, 128)
    out = torch.empty_like(v)
    # outputs given, S0 aliased with state_out (in-place carry), no final state
    kda.chunk_fwd(q, k, v, la, b, S0, out=out, state_out=S0, stream=S)
    o, st = kda.chunk_fwd(q, k, v, la, b, S0, final_state=False, stream=S)
    assert st is None
    # packed sequences with a host copy of the offsets
    qp, kp, vp, lap, bp = _prefill(T=200, packed=True, gate="head")
    cu = torch.tensor([0, 64, 64, 200], dtype=torch.int32)
    o, st = kda.chunk_fwd(qp, kp, vp, lap, bp, None, cu_seqlens=cu, cu_seqlens_host=cu, stream=S)
    assert st.shape == (3, 3, 128, 128)
    assert _names(rec) == ["kda_chunk_fwd", "kda_chunk_fwd", "kda_chunk_fwd_gated"]


@pytest.mark.parametrize("bad", ["out", "state_out", "S0", "k", "beta", "log_alpha", "q_rank",
                                 "cu_rank"])
def test_prefill_refuses_malformed_tensors_before_calling(rec, bad):
    q, k, v, la, b = _prefill()
    kw = {}
    S0 = None
    if bad == "out":
        kw["out"] = _t(2, 69, 3, 128, dtype=torch.bfloat16)
    elif bad == "state_out":
        kw["state_out"] = _t(2, 3, 128, 64)
    elif bad == "S0":
        S0 = _t(1, 3, 128, 128)
    elif bad == "k":
        k = _t(2, 70, 2, 128, dtype=torch.bfloat16)
    elif bad == "beta":
        b = _t(2, 70)
    elif bad == "log_alpha":
        la = _t(2, 70, 3, 64)
    elif bad == "q_rank":
        q = q[0]
    elif bad == "cu_rank":
        kw["cu_seqlens"] = torch.zeros(2, 2, dtype=torch.int32)
    with pytest.raises((ValueError, TypeError)):
        kda.chunk_fwd(q, k, v, la, b, S0, stream=S, **kw)
    assert rec.calls == []


def test_noalloc_binding_checks_like_the_workspace_binding(rec):
    q, k, v, la, b = _prefill()
    out = torch.empty_like(v)
    kda.chunk_fwd_noalloc(q, k, v, la, b, out=out, stream=S)
    assert _names(rec) == ["kda_chunk_fwd_noalloc"]
    qh, kh, vh, lah, bh = _prefill(gate="head")
    with pytest.raises(ValueError):  # the noalloc entry point takes the fp32 per-channel gate
        kda.chunk_fwd_noalloc(qh, kh, vh, lah, bh, out=out, stream=S)
    with pytest.raises(ValueError):
        kda.chunk_fwd_noalloc(q, k, v, la, b, out=out[:, :10], stream=S)
    with pytest.raises(ValueError):
        kda.chunk_fwd_noalloc(q, k, v, la, b, out=None, stream=S)
    assert len(_names(rec)) == 1


@pytest.mark.parametrize("gate,entry", [("channel", "kda_decode_step"), ("head", "kda_decode_step_gated"),
                                        ("none", "kda_decode_step_gated")])
def test_decode_picks_the_entry_point_of_the_gate_layout(rec, gate, entry):
    q, k, v, la, b = _prefill(B=4, T=3, gate=gate)  # [N=4, H=3, 128] after dropping T
    q, k, v = q[:, 0], k[:, 0], v[:, 0]
    la = None if la is None else la[:, 0].contiguous()
    b = b[:, 0].contiguous()
    state = _t(4, 3, 128, 128)
    kda.decode_step(q.contiguous(), k.contiguous(), v.contiguous(), la, b, state, stream=S)
    assert _names(rec) == [entry]


@pytest.mark.parametrize("bad", ["k", "beta", "out", "S"])
def test_decode_refuses_malformed_tensors_before_calling(rec, bad):
    q = _t(4, 3, 128, dtype=torch.bfloat16)
    k, v, la, b, state, out = q.clone(), q.clone(), _t(4, 3, 128), _t(4, 3), _t(4, 3, 128, 128), None
    if bad == "k":
        k = _t(4, 2, 128, dtype=torch.bfloat16)
    elif bad == "beta":
        b = _t(4)
    elif bad == "out":
        out = _t(4, 3, 64, dtype=torch.bfloat16)
    elif bad == "S":
        state = _t(4, 3, 128, 64)
    with pytest.raises(ValueError):
        kda.decode_step(q, k, v, la, b, state, out=out, stream=S)
    assert rec.calls == []
