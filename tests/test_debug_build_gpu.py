"""The KDA_DEBUG build of libkda (libkda_debug.so) on the GPU.

That build checks, on the device, the packed-sequence offsets a caller passes
without a host copy (cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seqs] = T)
before any kernel of the call reads a sequence span; a call that fails is counted
in the device status as KDA_STATUS_BAD_INPUT and writes nothing.

The first test runs the prefill and decode parity suites in a child process with
KDA_DEBUG=1, so the debug build must meet the same oracle tolerances and finish with
a clear status; the child also runs the second test, which hands the debug build
offsets that break the contract. Those offsets stay inside the tensors' token range
(only their order or their ends are wrong), so even a build without the checks would
read and write in bounds: nothing here can fault a GPU.
"""
import os
import subprocess
import sys

import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import cu_from_lengths, prefill_inputs
from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.relpath(os.path.abspath(__file__), ROOT)


@pytest.mark.skipif(kda.DEBUG_BUILD, reason="this test starts the KDA_DEBUG run itself")
def test_debug_build_passes_the_parity_suites():
    from gated_delta_rule_101_b200 import build as kbuild

    kbuild.build(debug=True)
    env = dict(os.environ, KDA_DEBUG="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_prefill_gpu.py", "tests/test_decode_gpu.py",
           f"{HERE}::test_invalid_device_offsets_are_refused"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = r.stdout[-4000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert "skipped" not in r.stdout.strip().splitlines()[-1], tail


@pytest.mark.skipif(not kda.DEBUG_BUILD, reason="needs the KDA_DEBUG build (run by the test above)")
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_invalid_device_offsets_are_refused(dtype):
    assert os.path.basename(kda.LIB_PATH) == "libkda_debug.so"
    kda.device_status()
    good = cu_from_lengths([70, 50, 100])  # [0, 70, 120, 220]
    inp = prefill_inputs(T=220, H=2, cu_seqlens=good, dtype=dtype, s0_std=0.1, seed=55, device=DEV)
    bad_offsets = ([0, 120, 70, 220],  # not monotone
                   [0, 70, 120, 200],  # ends before T
                   [5, 70, 120, 220])  # does not start at 0
    for bad in bad_offsets:
        cu_bad = torch.tensor(bad, dtype=torch.int32, device=DEV)
        o = torch.full_like(inp.v, float("nan"))
        S_T = torch.full_like(inp.S0, float("nan"))
        kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu_seqlens=cu_bad,
                      out=o, state_out=S_T)
        torch.cuda.synchronize()
        assert torch.isnan(o.float()).all(), f"{bad}: output written"
        assert torch.isnan(S_T).all(), f"{bad}: final state written"
        assert kda.device_status() == kda.STATUS_BAD_INPUT, bad
        assert kda.device_status() == 0
    # the same call with valid offsets computes normally and records nothing
    o, st = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu_seqlens=inp.cu_seqlens)
    torch.cuda.synchronize()
    ro, rs = oracle.kda_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                            cu_seqlens=inp.cu_seqlens.cpu())
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    check(o, ro, kind, "debug build o")
    check(st, rs, kind, "debug build S_T")
    assert kda.device_status() == 0
