"""kda_chunk_fwd_noalloc, the prefill entry point for callers that cannot allocate.

Some callers may not call cudaMalloc at all: a plugin whose host framework
owns every byte of GPU memory and offers no allocation hook, or a loop that
must never trigger cudaMalloc's device-wide synchronisation. For them libkda
runs the same prefill with a fixed scratch buffer that lives in its device
image instead of a caller-provided workspace.

This file checks, through the C ABI, that the allocation-free entry point
gives the same result as kda_chunk_fwd (with a workspace) on calls in a row,
bit for bit (both run the same kernels on the same inputs) and within the bf16
tolerance of the other tests against the fp64 oracle. The scratch is first
filled with junk by a larger call, so a call that read anything it had not
written itself would show. The cases cover each batched plan (prep then
chains, the fused grid, the segment scan) and packed sequences. An oversized
problem is refused. It is named so that pytest collects it after every other
test file; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import cu_from_lengths, prefill_inputs
from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_call(inp, o, S_T, cu_host=None):
    lib = kda.lib()
    packed = inp.cu_seqlens is not None
    if packed:
        T, H, _ = inp.q.shape
        B, n = 1, inp.cu_seqlens.numel() - 1
    else:
        B, T, H, _ = inp.q.shape
        n = 0
    host = None
    if cu_host is not None:
        host = (ctypes.c_int32 * len(cu_host))(*[int(x) for x in cu_host])
    return lib.kda_chunk_fwd_noalloc(
        _p(inp.q), _p(inp.k), _p(inp.v), _p(inp.log_alpha), _p(inp.beta), _p(inp.S0), _p(o),
        _p(S_T), B, T, H, 64, _p(inp.cu_seqlens), n, host, kda.KDA_BF16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _oracle(inp, heads):
    """fp64 oracle on the given heads of every sequence."""
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.cpu()
    out = []
    for h in heads:
        sl = (lambda x: x[:, h:h + 1]) if cu is not None else (lambda x: x[:, :, h:h + 1])
        S0 = None if inp.S0 is None else inp.S0[:, h:h + 1]
        out.append(oracle.kda_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha),
                                  sl(inp.beta), S0, cu_seqlens=cu))
    return out


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    # a large first call leaves junk in most of the scratch (about 58 of its 64 MiB)
    assert 48 << 20 < kda.workspace_size(1, 5500, 8) <= kda.lib().kda_noalloc_scratch_bytes()
    junk = prefill_inputs(B=1, T=5500, H=8, dtype=torch.bfloat16, s0_std=3.0, seed=100, device=DEV)
    jo, js = torch.empty_like(junk.v), torch.empty_like(junk.S0)
    assert _noalloc_call(junk, jo, js) == kda.KDA_OK
    packed = cu_from_lengths([70, 0, 129, 5])
    cases = [  # (inputs, kernels a workspace call launches: the plan it takes)
        (prefill_inputs(B=1, T=300, H=72, dtype=torch.bfloat16, s0_std=0.1, seed=101, device=DEV), 2),
        (prefill_inputs(B=2, T=300, H=3, dtype=torch.bfloat16, s0_std=0.1, seed=105, device=DEV), 1),
        (prefill_inputs(T=int(packed[-1]), H=2, cu_seqlens=packed, dtype=torch.bfloat16,
                        s0_std=0.1, seed=102, device=DEV), 3),
        (prefill_inputs(B=1, T=1000, H=32, dtype=torch.bfloat16, s0_std=0.1, seed=103, device=DEV), 1),
        (prefill_inputs(B=1, T=3000, H=2, dtype=torch.bfloat16, s0_std=0.1, seed=104, device=DEV), 4),
    ]
    for call, (inp, launches) in enumerate(cases):
        packed_in = inp.cu_seqlens is not None
        B = 1 if packed_in else inp.q.shape[0]
        T = inp.q.shape[0] if packed_in else inp.q.shape[1]
        H = inp.q.shape[-2]
        n = inp.cu_seqlens.numel() - 1 if packed_in else 0
        assert kda.chunk_fwd_launches(B, T, H, n_seqs=n) == launches
        ref_o, ref_s = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                                     cu_seqlens=inp.cu_seqlens)
        o = torch.full_like(ref_o, float("nan"))
        S_T = torch.full_like(ref_s, float("nan"))
        cu_host = None if inp.cu_seqlens is None else inp.cu_seqlens.cpu().tolist()
        assert _noalloc_call(inp, o, S_T, cu_host) == kda.KDA_OK
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o), f"no-alloc o differs from kda_chunk_fwd, call {call}"
        assert torch.equal(S_T, ref_s), f"no-alloc S_T differs from kda_chunk_fwd, call {call}"
        heads = sorted({0, H - 1})
        for h, (ro, rs) in zip(heads, _oracle(inp, heads)):
            got_o = o[:, h:h + 1] if packed_in else o[:, :, h:h + 1]
            check(got_o, ro, "bf16", f"no-alloc o vs oracle, call {call}, head {h}")
            check(S_T[:, h:h + 1], rs, "bf16", f"no-alloc S_T vs oracle, call {call}, head {h}")


def test_noalloc_refuses_problems_beyond_its_scratch():
    lib = kda.lib()
    cap = lib.kda_noalloc_scratch_bytes()
    assert cap == 64 << 20
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call is refused first
    B, T, H = 4, 4096, 16  # needs about 304 MB of workspace
    st = lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, None, B, T, H, 64,
                                   None, 0, None, kda.KDA_BF16, None)
    assert st == -6 and "scratch" in kda.strerror(st)
