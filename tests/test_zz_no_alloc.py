"""kda_chunk_fwd_noalloc, the prefill entry point for callers that cannot allocate.

Some callers may not call cudaMalloc at all: a plugin whose host framework
owns every byte of GPU memory and offers no allocation hook, or a loop that
must never trigger cudaMalloc's device-wide synchronisation. For them libkda
runs the same prefill with a fixed scratch buffer that lives in its device
image instead of a caller-provided workspace.

This file checks, through the C ABI, that the allocation-free entry point
gives the same result as kda_chunk_fwd (with a workspace) within the bf16
tolerance of the other tests, on two calls in a row (the second call reuses
the scratch the first one left behind), and that an oversized problem is
refused. It is named so that pytest collects it after every other test file;
it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_101_b200 as kda
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


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [
        prefill_inputs(B=2, T=300, H=3, dtype=torch.bfloat16, s0_std=0.1, seed=101, device=DEV),
        prefill_inputs(T=int(cu_from_lengths([70, 0, 129, 5])[-1]), H=2,
                       cu_seqlens=cu_from_lengths([70, 0, 129, 5]), dtype=torch.bfloat16,
                       s0_std=0.1, seed=102, device=DEV),
    ]
    for call, inp in enumerate(cases):
        ref_o, ref_s = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                                     cu_seqlens=inp.cu_seqlens)
        o = torch.full_like(ref_o, float("nan"))
        S_T = torch.full_like(ref_s, float("nan"))
        cu_host = None if inp.cu_seqlens is None else inp.cu_seqlens.cpu().tolist()
        assert _noalloc_call(inp, o, S_T, cu_host) == kda.KDA_OK
        torch.cuda.synchronize()
        check(o, ref_o.double(), "bf16", f"no-alloc o, call {call}")
        check(S_T, ref_s.double(), "bf16", f"no-alloc S_T, call {call}")


def test_noalloc_refuses_problems_beyond_its_scratch():
    lib = kda.lib()
    cap = lib.kda_noalloc_scratch_bytes()
    assert cap == 64 << 20
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call is refused first
    B, T, H = 4, 4096, 16  # needs about 304 MB of workspace
    st = lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, None, B, T, H, 64,
                                   None, 0, None, kda.KDA_BF16, None)
    assert st == -6 and "scratch" in kda.strerror(st)
