"""kda_decode_step on the GPU against the fp64 oracle."""
import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import decode_inputs
from parity import check, per_channel_gate

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _oracle_for(inp, n_idx, h_idx):
    """Oracle over the token sequence of each sampled (sequence, head) pair."""
    outs = []
    la_full = per_channel_gate(inp.log_alpha, inp.gate, inp.q)
    for n, h in zip(n_idx, h_idx):
        q = inp.q[:, n, h][None, :, None]  # [1, steps, 1, dk]
        k = inp.k[:, n, h][None, :, None]
        v = inp.v[:, n, h][None, :, None]
        la = la_full[:, n, h][None, :, None]
        b = inp.beta[:, n, h][None, :, None]
        S0 = inp.S[n, h][None, None]
        outs.append(oracle.kda_fwd(q, k, v, la, b, S0))
    return outs


def _gate_at(inp, t):
    return None if inp.log_alpha is None else inp.log_alpha[t]


def _run_decode(inp, graph: bool):
    S = inp.S.clone()
    steps = inp.q.shape[0]
    o = torch.empty_like(inp.v)
    if not graph:
        for t in range(steps):
            kda.decode_step(inp.q[t], inp.k[t], inp.v[t], _gate_at(inp, t), inp.beta[t], S, out=o[t])
    else:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):  # first call outside capture
            kda.decode_step(inp.q[0], inp.k[0], inp.v[0], _gate_at(inp, 0), inp.beta[0], S.clone(),
                            out=o[0])
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for t in range(steps):
                kda.decode_step(inp.q[t], inp.k[t], inp.v[t], _gate_at(inp, t), inp.beta[t], S,
                                out=o[t])
        g.replay()
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("dtype,kind", [(torch.bfloat16, "bf16"), (torch.float32, "f32")])
def test_decode_small_all_outputs(dtype, kind):
    inp = decode_inputs(steps=24, N=3, H=5, dtype=dtype, seed=4, device=DEV)
    o, S = _run_decode(inp, graph=False)
    for n in range(3):
        for h in range(5):
            (ro, rs), = _oracle_for(inp, [n], [h])
            check(o[:, n, h], ro[0, :, 0], kind, f"decode o (n={n}, h={h})")
            check(S[n, h], rs[0, 0], kind, f"decode S (n={n}, h={h})")


def test_decode_extreme_gates():
    inp = decode_inputs(steps=6, N=2, H=2, dtype=torch.float32, seed=5, device=DEV)
    inp.log_alpha[2].fill_(-1e4)  # alpha = 0 at step 2: state reset
    inp.log_alpha[4].zero_()      # alpha = 1 at step 4
    inp.beta[3].fill_(0.0)
    inp.beta[5].fill_(1.0)
    o, S = _run_decode(inp, graph=False)
    for n in range(2):
        for h in range(2):
            (ro, rs), = _oracle_for(inp, [n], [h])
            check(o[:, n, h], ro[0, :, 0], "f32", "decode o extreme gates")
            check(S[n, h], rs[0, 0], "f32", "decode S extreme gates")


def test_decode_full_workload_sampled_graph():
    """N=256 sequences, H=32, 1024 consecutive steps, captured in one CUDA graph."""
    inp = decode_inputs(steps=1024, N=256, H=32, dtype=torch.bfloat16, seed=20263, device=DEV)
    o, S = _run_decode(inp, graph=True)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    pairs = [(0, 0), (255, 31), (17, 5), (128, 16), (200, 9), (63, 30)]
    for (n, h), (ro, rs) in zip(pairs, _oracle_for(inp, [p[0] for p in pairs], [p[1] for p in pairs])):
        check(o[:, n, h], ro[0, :, 0], "bf16", f"decode o full (n={n}, h={h})")
        check(S[n, h], rs[0, 0], "bf16", f"decode S full (n={n}, h={h})")


def test_decode_deterministic():
    inp = decode_inputs(steps=8, N=4, H=4, dtype=torch.bfloat16, seed=6, device=DEV)
    o1, S1 = _run_decode(inp, graph=False)
    o2, S2 = _run_decode(inp, graph=False)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("gate", ["channel_bf16", "head", "none"])
@pytest.mark.parametrize("dtype,kind", [(torch.bfloat16, "bf16"), (torch.float32, "f32")])
def test_decode_gate_layouts(gate, dtype, kind):
    """Gated DeltaNet (one rate per head), DeltaNet (no gate) and a bf16 gate."""
    inp = decode_inputs(steps=24, N=2, H=3, dtype=dtype, seed=46, gate=gate, device=DEV)
    o, S = _run_decode(inp, graph=gate == "head")
    for n in range(2):
        for h in range(3):
            (ro, rs), = _oracle_for(inp, [n], [h])
            check(o[:, n, h], ro[0, :, 0], kind, f"decode {gate} o (n={n}, h={h})")
            check(S[n, h], rs[0, 0], kind, f"decode {gate} S (n={n}, h={h})")
