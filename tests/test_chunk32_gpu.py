"""Chunks of C = 32 tokens on the GPU against the fp64 oracle.

The pages name chunk lengths of 32 to 128 as the useful range and found 64 best on
their hardware (mokono.cn "Kimi Linear：高效注意力机制在长序列处理中的创新应用",
section 4.1). C = 32 runs on the CUDA-core kernel in fp32 for both input dtypes, so the
final state meets the fp32 bar (relative L2 <= 1e-4) even for bf16 inputs; o is rounded
to the input dtype and meets that dtype's bar. The chunk length changes no result
beyond rounding: the same oracle (the token recurrence of eq. (1)) decides every case.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import cu_from_lengths, prefill_inputs
from io_ref import f64, l2norm_rows, log_sigmoid, rmsnorm_gate, sigmoid
from parity import check, per_channel_gate

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KIND = {torch.bfloat16: "bf16", torch.float32: "f32"}


def run(inp, **kw):
    o, st = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                          cu_seqlens=inp.cu_seqlens, C=32, **kw)
    torch.cuda.synchronize()
    return o, st


def ref(inp):
    la = per_channel_gate(inp.log_alpha, inp.gate, inp.q)
    return oracle.kda_fwd(inp.q, inp.k, inp.v, la, inp.beta, inp.S0,
                          cu_seqlens=None if inp.cu_seqlens is None else inp.cu_seqlens.cpu())


def check_both(inp, o, st, what):
    ro, rs = ref(inp)
    check(o, ro, KIND[inp.q.dtype], f"{what} o")
    check(st, rs, "f32", f"{what} S_T")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [1, 31, 32, 33, 200])
def test_batched_ragged_with_state(dtype, T):
    inp = prefill_inputs(B=2, T=T, H=3, dtype=dtype, s0_std=0.1, seed=300 + T, device=DEV)
    assert kda.chunk_fwd_launches(2, T, 3, dtype=dtype, C=32) == 1
    o, st = run(inp)
    check_both(inp, o, st, f"C=32 T={T}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_packed_with_empty_and_ragged_sequences(dtype):
    lengths = [1, 32, 33, 0, 130, 7, 0, 65]
    cu = cu_from_lengths(lengths)
    inp = prefill_inputs(T=int(cu[-1]), H=2, cu_seqlens=cu, dtype=dtype, s0_std=0.1, seed=31, device=DEV)
    o, st = run(inp, cu_seqlens_host=cu)
    check_both(inp, o, st, "C=32 packed")
    for i, n in enumerate(lengths):
        if n == 0:
            assert torch.equal(st[i], inp.S0[i])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_strong_decay_and_alpha_zero_one_tokens(dtype):
    """Channels past the factorised range (exact pairwise path), alpha = 0 resets inside
    a chunk and at a chunk start, alpha = 1 and beta = 0 / 1 runs."""
    inp = prefill_inputs(B=2, T=190, H=2, dtype=dtype, s0_std=0.1, seed=33, device=DEV)
    inp.log_alpha[..., 5] = -3.0
    inp.log_alpha[..., 77] = -40.0
    inp.log_alpha[0, 70:80, 1, 100] = -1e4
    inp.log_alpha[:, 10:12] = -1e4
    inp.log_alpha[:, 64] = -1e4
    inp.log_alpha[:, 100:140] = 0.0
    inp.beta[:, 20:30] = 0.0
    inp.beta[:, 30:40] = 1.0
    o, st = run(inp)
    check_both(inp, o, st, "C=32 decay edge cases")


@pytest.mark.parametrize("gate", ["channel_bf16", "head", "none"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gate_layouts(gate, dtype):
    inp = prefill_inputs(B=2, T=150, H=2, dtype=dtype, s0_std=0.1, seed=35, gate=gate, device=DEV)
    o, st = run(inp)
    check_both(inp, o, st, f"C=32 gate {gate}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fused_input_steps(dtype):
    """Logit gate, q/k L2Norm and beta logits inside the kernel at C = 32."""
    g = torch.Generator(device="cpu").manual_seed(37)
    B, T, H, eps = 2, 170, 2, 1e-6
    shape = (B, T, H, 128)
    q, k, v = (torch.randn(shape, generator=g).to(dtype).to(DEV) for _ in range(3))
    z = (torch.rand(shape, generator=g) * 5 + 2).to(DEV)
    b = torch.randn((B, T, H), generator=g).to(DEV)
    S0 = 0.1 * torch.randn((B, H, 128, 128), generator=g).to(DEV)
    o, st = kda.chunk_fwd(q, k, v, z, b, S0, C=32, gate_logits=True, qk_l2norm=True, qk_eps=eps,
                          beta_logits=True)
    torch.cuda.synchronize()
    ro, rs = oracle.kda_fwd(l2norm_rows(q, eps), l2norm_rows(k, eps), f64(v), log_sigmoid(z), sigmoid(b),
                            f64(S0))
    check(o, ro, KIND[dtype], "C=32 fused inputs o")
    check(st, rs, KIND[dtype], "C=32 fused inputs S_T")


def test_state_carry_across_calls_in_place():
    inp = prefill_inputs(B=2, T=333, H=2, dtype=torch.float32, s0_std=0.1, seed=39, device=DEV)
    S = inp.S0.clone()
    outs = []
    for a, z in ((0, 32), (32, 100), (100, 101), (101, 333)):
        o, _ = kda.chunk_fwd(inp.q[:, a:z].contiguous(), inp.k[:, a:z].contiguous(),
                             inp.v[:, a:z].contiguous(), inp.log_alpha[:, a:z].contiguous(),
                             inp.beta[:, a:z].contiguous(), S, state_out=S, C=32)
        outs.append(o)
    torch.cuda.synchronize()
    ro, rs = ref(inp)
    check(torch.cat(outs, dim=1), ro, "f32", "C=32 carry o")
    check(S, rs, "f32", "C=32 carry S_T")


def test_chunk_lengths_agree():
    """fp32 inputs at C = 32 and C = 64 (both CUDA-core kernels) agree to fp32 rounding."""
    inp = prefill_inputs(B=1, T=500, H=2, dtype=torch.float32, s0_std=0.1, seed=41, device=DEV)
    o32, s32 = run(inp)
    o64, s64 = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, C=64)
    torch.cuda.synchronize()
    check(o32, o64, "f32", "C=32 vs C=64 o")
    check(s32, s64, "f32", "C=32 vs C=64 S_T")


def test_output_epilogue():
    """The output epilogue (RMSNorm, weights, sigmoid gate) after the C = 32 kernel."""
    inp = prefill_inputs(B=2, T=100, H=2, dtype=torch.bfloat16, s0_std=0.1, seed=43, device=DEV)
    og = torch.randn(inp.v.shape, generator=torch.Generator().manual_seed(44)).to(torch.bfloat16).to(DEV)
    w = torch.linspace(0.5, 1.5, 128, device=DEV)
    o, st = run(inp, out_gate=og, out_norm_weight=w, out_eps=1e-6)
    ro, rs = ref(inp)
    check(o, rmsnorm_gate(ro, og, w, 1e-6), "bf16", "C=32 epilogue o")
    check(st, rs, "f32", "C=32 epilogue S_T")


def test_prefill_workload_b4_t4096_h16_sampled():
    """The bench step's shape at C = 32 (bf16 inputs); two (sequence, head) pairs in full."""
    inp = prefill_inputs(B=4, T=4096, H=16, dtype=torch.bfloat16, s0_std=0.1, seed=20261, device=DEV)
    o, st = run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(st).all()
    for s_, h in ((0, 0), (3, 15)):
        sl = lambda x: x[s_:s_ + 1, :, h:h + 1]
        ro, rs = oracle.kda_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.beta),
                                inp.S0[s_:s_ + 1, h:h + 1])
        check(o[s_:s_ + 1, :, h:h + 1], ro, "bf16", f"C=32 B4 T4096 H16 o (seq {s_}, head {h})")
        check(st[s_:s_ + 1, h:h + 1], rs, "f32", f"C=32 B4 T4096 H16 S_T (seq {s_}, head {h})")
