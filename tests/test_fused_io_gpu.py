"""Fused input and output transformations on the GPU against the fp64 oracle.

The layer around the operator (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3)
L2-normalises q and k, takes beta through a sigmoid, parameterises the forget gate as
alpha = f(z) of a low-rank projection z (read here as f = sigmoid), and passes the
output through a head-wise RMSNorm and a sigmoid output gate. The kernels can do each
of these steps themselves (kda_chunk_fwd_io, kda_decode_step_io, and the
KDA_GATE_CHANNEL_LOGIT gate layouts). Here the oracle is fed the same steps done in
fp64 on the exact values handed to the GPU (tests/io_ref.py), and the GPU result must
match at the usual tolerances.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import cu_from_lengths
from io_ref import f64, l2norm_rows, log_sigmoid, rmsnorm_gate, sigmoid
from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KIND = {torch.bfloat16: "bf16", torch.float32: "f32"}
EPS = 1e-6


def raw_inputs(lead, H, dtype, seed, n_seqs):
    """Inputs before the layer's transformations: q, k, v ~ N(0, 1) (not normalised),
    z ~ U(2, 7) (alpha = sigmoid(z) in about [0.88, 0.999], log alpha in about
    [-0.13, -0.001], the workloads' range), beta logits ~ N(0, 1), output gate ~ N(0, 1),
    RMSNorm weights ~ U(0.5, 1.5), S0 ~ N(0, 0.1^2)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = lead + (H, 128)
    mk = lambda s, lo=None, hi=None: (torch.rand(s, generator=g) * (hi - lo) + lo) if lo is not None \
        else torch.randn(s, generator=g)
    x = dict(q=mk(shape).to(dtype), k=mk(shape).to(dtype), v=mk(shape).to(dtype),
             z=mk(shape, 2.0, 7.0), b=mk(lead + (H,)), og=mk(shape).to(dtype),
             w=mk((128,), 0.5, 1.5), S0=0.1 * mk((n_seqs, H, 128, 128)))
    return {k_: t.to(DEV) for k_, t in x.items()}


def oracle_ref(x, cu=None, out_epi=True):
    """The fp64 oracle on the transformed inputs, and its output transformed."""
    q, k = l2norm_rows(x["q"], EPS), l2norm_rows(x["k"], EPS)
    la = log_sigmoid(x["z"])
    beta = sigmoid(x["b"])
    o, st = oracle.kda_fwd(q, k, f64(x["v"]), la, beta, f64(x["S0"]), cu_seqlens=cu)
    if out_epi:
        o = rmsnorm_gate(o, x["og"], x["w"], EPS)
    return o, st


def run_fused(x, cu=None, out_epi=True, gate_dtype=torch.float32, **kw):
    return kda.chunk_fwd(x["q"], x["k"], x["v"], x["z"].to(gate_dtype).contiguous(), x["b"], x["S0"],
                         cu_seqlens=cu, gate_logits=True, qk_l2norm=True, qk_eps=EPS,
                         beta_logits=True, out_gate=x["og"] if out_epi else None,
                         out_norm_weight=x["w"] if out_epi else None, out_eps=EPS, **kw)


@pytest.mark.parametrize("T", [64, 200, 700])
def test_prefill_all_fused_steps_batched_bf16(T):
    x = raw_inputs((2, T), 3, torch.bfloat16, seed=T, n_seqs=2)
    o, st = run_fused(x)
    torch.cuda.synchronize()
    ro, rs = oracle_ref(x)
    check(o, ro, "bf16", f"fused o T={T}")
    check(st, rs, "bf16", f"fused S_T T={T}")


def test_prefill_fused_packed_with_empty_and_ragged_sequences():
    lengths = [0, 130, 64, 1, 257, 0, 65]
    cu = torch.as_tensor(cu_from_lengths(lengths), dtype=torch.int32).to(DEV)
    x = raw_inputs((int(cu[-1]),), 2, torch.bfloat16, seed=5, n_seqs=len(lengths))
    o, st = run_fused(x, cu=cu)
    torch.cuda.synchronize()
    ro, rs = oracle_ref(x, cu=cu.cpu())
    check(o, ro, "bf16", "fused packed o")
    check(st, rs, "bf16", "fused packed S_T")


@pytest.mark.parametrize("shape", [(1, 1000, 32), (1, 3000, 2)])
def test_output_epilogue_on_the_fused_grid_and_segment_scan_plans(shape):
    """The output epilogue is one kernel after whichever plan the call takes: on the
    fused grid's shape (whose L2Norm moves the call to prep and chains) and on the
    segment scan's."""
    B, T, H = shape
    base = kda.chunk_fwd_launches(B, T, H)
    assert base in (1, 4)
    assert kda.chunk_fwd_launches(B, T, H, out_epilogue=True) == base + 1
    x = raw_inputs((B, T), H, torch.bfloat16, seed=T + H, n_seqs=B)
    o, st = run_fused(x)
    torch.cuda.synchronize()
    for h in (0, H - 1):
        sub = {k_: (t[:, :, h:h + 1] if t.dim() >= 3 and k_ != "S0" else t) for k_, t in x.items()}
        sub["S0"] = x["S0"][:, h:h + 1]
        sub["w"] = x["w"]
        ro, rs = oracle_ref(sub)
        check(o[:, :, h:h + 1], ro, "bf16", f"{shape} o head {h}")
        check(st[:, h:h + 1], rs, "bf16", f"{shape} S_T head {h}")


@pytest.mark.parametrize("gate_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_input_steps_on_every_dtype(dtype, gate_dtype):
    """Logit gate (fp32 and bf16), q/k L2Norm and beta logits, without the output
    epilogue: bf16 (tensor cores) and fp32 (CUDA cores)."""
    x = raw_inputs((2, 333), 2, dtype, seed=11, n_seqs=2)
    x["z"] = x["z"].to(gate_dtype).float() if gate_dtype == torch.bfloat16 else x["z"]
    o, st = run_fused(x, out_epi=False, gate_dtype=gate_dtype)
    torch.cuda.synchronize()
    ro, rs = oracle_ref(x, out_epi=False)
    check(o, ro, KIND[dtype], "input steps o")
    check(st, rs, KIND[dtype], "input steps S_T")


@pytest.mark.parametrize("dtype,C", [(torch.float32, 64), (torch.float32, 32), (torch.bfloat16, 32)])
def test_output_epilogue_on_the_cuda_core_kernel(dtype, C):
    """fp32 inputs and chunks of 32 (the CUDA-core kernel) with every fused step."""
    x = raw_inputs((2, 150), 2, dtype, seed=3 + C, n_seqs=2)
    o, st = run_fused(x, C=C)
    torch.cuda.synchronize()
    ro, rs = oracle_ref(x)
    check(o, ro, KIND[dtype], f"cuda-core fused o C={C}")
    check(st, rs, KIND[dtype], f"cuda-core fused S_T C={C}")


def test_segment_scan_plan_with_every_fused_step():
    """The segment scan (few heads, long sequence) keeps its plan under the input steps
    and adds the epilogue kernel (no RMSNorm weights: ones)."""
    B, T, H = 1, 3000, 2
    x = raw_inputs((B, T), H, torch.bfloat16, seed=77, n_seqs=B)
    x["w"] = None
    assert kda.chunk_fwd_launches(B, T, H, out_epilogue=True) == 5
    o, st = kda.chunk_fwd(x["q"], x["k"], x["v"], x["z"], x["b"], x["S0"], gate_logits=True,
                          qk_l2norm=True, qk_eps=EPS, beta_logits=True, out_gate=x["og"], out_eps=EPS)
    torch.cuda.synchronize()
    la, beta = log_sigmoid(x["z"]), sigmoid(x["b"])
    ro, rs = oracle.kda_fwd(l2norm_rows(x["q"], EPS), l2norm_rows(x["k"], EPS), f64(x["v"]), la, beta,
                            f64(x["S0"]))
    ro = rmsnorm_gate(ro, x["og"], None, EPS)
    check(o, ro, "bf16", "segment scan fused o")
    check(st, rs, "bf16", "segment scan fused S_T")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_all_fused_steps(dtype):
    """Four decode tokens with every fused step equal the oracle over the same tokens."""
    steps, N, H = 4, 3, 2
    x = raw_inputs((N, steps), H, dtype, seed=21, n_seqs=N)
    S = x["S0"].clone()
    outs = []
    for t in range(steps):
        sl = lambda name: x[name][:, t].contiguous()
        outs.append(kda.decode_step(sl("q"), sl("k"), sl("v"), sl("z"), sl("b"), S, gate_logits=True,
                                    qk_l2norm=True, qk_eps=EPS, beta_logits=True, out_gate=sl("og"),
                                    out_norm_weight=x["w"], out_eps=EPS))
    torch.cuda.synchronize()
    ro, rs = oracle_ref(x)
    check(torch.stack(outs, dim=1), ro, KIND[dtype], "decode fused o")
    check(S, rs, KIND[dtype], "decode fused S")


def test_logit_gate_equals_the_log_gate_it_stands_for():
    """alpha = sigmoid(z) given as z, or as log sigmoid(z) in fp32: the same result to
    fp32 rounding of the gate (bf16 path)."""
    x = raw_inputs((1, 300), 2, torch.bfloat16, seed=9, n_seqs=1)
    o1, s1 = kda.chunk_fwd(x["q"], x["k"], x["v"], x["z"], torch.sigmoid(x["b"]), x["S0"],
                           gate_logits=True, qk_l2norm=True, qk_eps=EPS)
    la = torch.nn.functional.logsigmoid(x["z"])
    o2, s2 = kda.chunk_fwd(x["q"], x["k"], x["v"], la, torch.sigmoid(x["b"]), x["S0"],
                           qk_l2norm=True, qk_eps=EPS)
    torch.cuda.synchronize()
    # the two gates differ by fp32 rounding of log sigmoid(z); through the bf16 operands
    # that moves the results by far less than the bf16 bar
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2 * o2.float().abs().max().item()
    assert ((s1 - s2).norm() / s2.norm()).item() <= 1e-3
