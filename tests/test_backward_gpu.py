"""kda_chunk_bwd on the GPU against the fp64 reverse-pass oracle.

The backward pass gives the gradients of sum(o * dout) + sum(S_T * dS_T) with respect
to q, k, v, the gate, beta and S0. The oracle (oracle/backward.py) differentiates the
recurrence of eq. (1) (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3) token by
token in fp64 and is pinned by autograd and finite differences. The GPU computes in
fp32 for both input dtypes, so every gradient is held to the fp32 bar: relative L2
error <= 1e-4. Inputs follow the prefill recipe; dout ~ N(0, 1) in q's dtype and
dS_T ~ N(0, 1) fp32.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_101_b200 as kda
from gated_delta_rule_101_b200.inputs import cu_from_lengths, prefill_inputs
from io_ref import f64, l2norm_rows, l2norm_rows_bwd, log_sigmoid, sigmoid
from oracle.backward import kda_bwd
from parity import check, per_channel_gate

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
EPS = 1e-6


def grads_out(inp, seed):
    """dout ~ N(0, 1) in q's dtype and dS_T ~ N(0, 1) fp32, shaped like o and S_T."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    dout = torch.randn(inp.v.shape, generator=g).to(inp.v.dtype).to(DEV)
    n_seqs = inp.q.shape[0] if inp.cu_seqlens is None else inp.cu_seqlens.numel() - 1
    dS_T = torch.randn((n_seqs, inp.q.shape[-2], 128, 128), generator=g).to(DEV)
    return dout, dS_T


def check_all(got, ref, what, gate="channel", la=None):
    for name in ("dq", "dk", "dv", "dbeta", "dS0"):
        check(got[name], ref[name], "f32", f"{what} {name}")
    if gate == "none":
        assert got["dgate"] is None
    elif gate == "head":
        check(got["dgate"], ref["dlog_alpha"].sum(axis=-1), "f32", f"{what} dgate")
    else:
        check(got["dgate"], ref["dlog_alpha"], "f32", f"{what} dgate")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 64, 200])
def test_batched_gradients(dtype, T):
    inp = prefill_inputs(B=2, T=T, H=2, dtype=dtype, s0_std=0.1, seed=100 + T, device=DEV)
    dout, dS_T = grads_out(inp, T)
    got = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    torch.cuda.synchronize()
    ref = kda_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    check_all(got, ref, f"batched T={T} {dtype}")


def test_packed_gradients_with_empty_and_ragged_sequences():
    lengths = [0, 130, 64, 1, 90, 0]
    cu = cu_from_lengths(lengths)
    inp = prefill_inputs(T=int(cu[-1]), H=2, cu_seqlens=cu, dtype=torch.bfloat16, s0_std=0.1, seed=7,
                         device=DEV)
    dout, dS_T = grads_out(inp, 8)
    got = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T,
                        cu_seqlens=inp.cu_seqlens, cu_seqlens_host=cu)
    torch.cuda.synchronize()
    ref = kda_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T,
                  cu_seqlens=inp.cu_seqlens.cpu())
    check_all(got, ref, "packed")
    for i, n in enumerate(lengths):
        if n == 0:  # an empty sequence passes dS_T straight to dS0
            assert torch.equal(got["dS0"][i], dS_T[i])


def test_no_loss_on_the_final_state_and_no_initial_state():
    inp = prefill_inputs(B=1, T=150, H=3, dtype=torch.float32, seed=9, device=DEV)
    dout, _ = grads_out(inp, 9)
    got = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, dout, None)
    torch.cuda.synchronize()
    ref = kda_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, dout, None)
    check_all(got, ref, "no S0, no dS_T")


@pytest.mark.parametrize("gate", ["channel_bf16", "head", "none"])
def test_gate_layouts(gate):
    inp = prefill_inputs(B=1, T=170, H=2, dtype=torch.bfloat16, s0_std=0.1, seed=11, gate=gate, device=DEV)
    dout, dS_T = grads_out(inp, 12)
    got = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    torch.cuda.synchronize()
    la = per_channel_gate(inp.log_alpha, inp.gate, inp.q)
    ref = kda_bwd(inp.q, inp.k, inp.v, la, inp.beta, inp.S0, dout, dS_T)
    check_all(got, ref, f"gate {gate}", gate="head" if gate == "head" else ("none" if gate == "none" else "channel"))


def test_alpha_zero_and_one_tokens_and_strong_decay():
    inp = prefill_inputs(B=1, T=160, H=2, dtype=torch.float32, s0_std=0.1, seed=13, device=DEV)
    inp.log_alpha[:, 10:12] = -30.0   # near-reset
    inp.log_alpha[:, 100:140] = 0.0   # alpha = 1
    inp.log_alpha[..., 5] = -3.0      # a fast channel
    dout, dS_T = grads_out(inp, 14)
    got = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    torch.cuda.synchronize()
    ref = kda_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    check_all(got, ref, "alpha 0/1")


def test_fused_input_steps_chain_rule():
    """Logit gate, q/k L2Norm inside the kernel and beta logits: the gradients of the raw
    inputs equal the oracle's gradients pushed back through the same steps in fp64."""
    g = torch.Generator(device="cpu").manual_seed(21)
    B, T, H = 1, 140, 2
    shape = (B, T, H, 128)
    qr, kr, v = (torch.randn(shape, generator=g).to(DEV) for _ in range(3))
    z = (torch.rand(shape, generator=g) * 5 + 2).to(DEV)
    b = torch.randn((B, T, H), generator=g).to(DEV)
    S0 = 0.1 * torch.randn((B, H, 128, 128), generator=g).to(DEV)
    dout = torch.randn(shape, generator=g).to(DEV)
    dS_T = torch.randn((B, H, 128, 128), generator=g).to(DEV)
    got = kda.chunk_bwd(qr, kr, v, z, b, S0, dout, dS_T, gate_logits=True, qk_l2norm=True, qk_eps=EPS,
                        beta_logits=True)
    torch.cuda.synchronize()
    q, k = l2norm_rows(qr, EPS), l2norm_rows(kr, EPS)
    ref = kda_bwd(q, k, f64(v), log_sigmoid(z), sigmoid(b), f64(S0), dout, dS_T)
    sb = sigmoid(b)
    check(got["dq"], l2norm_rows_bwd(qr, ref["dq"], EPS), "f32", "raw dq")
    check(got["dk"], l2norm_rows_bwd(kr, ref["dk"], EPS), "f32", "raw dk")
    check(got["dv"], ref["dv"], "f32", "dv")
    check(got["dgate"], ref["dlog_alpha"] * (1.0 - sigmoid(z)), "f32", "dz")
    check(got["dbeta"], ref["dbeta"] * sb * (1.0 - sb), "f32", "dbeta logits")
    check(got["dS0"], ref["dS0"], "f32", "dS0")


def test_deterministic_bitwise():
    inp = prefill_inputs(B=2, T=300, H=2, dtype=torch.bfloat16, s0_std=0.1, seed=15, device=DEV)
    dout, dS_T = grads_out(inp, 16)
    a = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    b = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dgate", "dbeta", "dS0"):
        assert torch.equal(a[name], b[name]), name


def test_prefill_workload_b4_t4096_h16_sampled():
    """The bench step's shape; the oracle checks two (sequence, head) pairs in full."""
    inp = prefill_inputs(B=4, T=4096, H=16, dtype=torch.bfloat16, s0_std=0.1, seed=20261, device=DEV)
    dout, dS_T = grads_out(inp, 17)
    got = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T)
    torch.cuda.synchronize()
    for s_, h in ((0, 0), (3, 15)):
        sl = lambda x: x[s_:s_ + 1, :, h:h + 1]
        ref = kda_bwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.beta),
                      inp.S0[s_:s_ + 1, h:h + 1], sl(dout), dS_T[s_:s_ + 1, h:h + 1])
        sub = {n: (got[n][s_:s_ + 1, :, h:h + 1] if n != "dS0" else got[n][s_:s_ + 1, h:h + 1])
               for n in ("dq", "dk", "dv", "dgate", "dbeta", "dS0")}
        check_all(sub, ref, f"B4 T4096 H16 (seq {s_}, head {h})")
