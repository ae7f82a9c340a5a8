"""libkda's C ABI on the host: exports and argument validation (no GPU needed).

Every rejected call below returns before any CUDA call is made, so fake
device pointers are safe: nothing dereferences them.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_101_b200 as kda
from gated_delta_rule_101_b200 import build as kbuild

BF16, F32 = kda.KDA_BF16, kda.KDA_F32
INVALID, UNSUPPORTED, WORKSPACE = -1, -2, -3
FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: every call here fails validation


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.lib()


def test_every_declared_symbol_is_exported(lib):
    names = kda.declared_symbols()
    assert {"kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size",
            "kda_strerror", "kda_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/kda.h but not exported"


def test_strerror_and_version(lib):
    for code, name in kda.STATUS.items():
        assert kda.strerror(code).startswith(name)
    assert kda.strerror(-99) == "unknown kda status"
    assert lib.kda_version() >= 100


def _chunk(lib, *, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, o=FAKE, ST=None, B=1,
           T=128, H=2, C=64, cu=None, n_seqs=0, cu_host=None, dtype=BF16, ws=None, ws_bytes=0):
    return lib.kda_chunk_fwd(q, k, v, la, beta, S0, o, ST, B, T, H, C, cu, n_seqs, cu_host, dtype,
                             ws, ws_bytes, None)


def test_chunk_fwd_rejects_bad_arguments(lib):
    for C in (0, 16, 48, 128, 256):
        assert _chunk(lib, C=C) == UNSUPPORTED, C
    assert _chunk(lib, dtype=7) == UNSUPPORTED
    assert _chunk(lib, B=0) == INVALID
    assert _chunk(lib, H=0) == INVALID
    assert _chunk(lib, T=-1) == INVALID
    assert _chunk(lib, T=0) == INVALID  # batched rows of zero tokens
    for field in ("q", "k", "v", "la", "beta", "o"):
        assert _chunk(lib, **{field: None}) == INVALID, field
    # cu_seqlens without n_seqs, n_seqs without cu_seqlens, packed with B != 1
    assert _chunk(lib, cu=FAKE) == INVALID
    assert _chunk(lib, n_seqs=2) == INVALID
    assert _chunk(lib, cu=FAKE, n_seqs=2, B=2) == INVALID


@pytest.mark.parametrize("offsets", [[0, 64, 32, 128], [1, 64, 128], [0, 64, 127], [0, 64, 129]])
def test_chunk_fwd_rejects_bad_host_offsets(lib, offsets):
    host = (ctypes.c_int32 * len(offsets))(*offsets)
    st = _chunk(lib, cu=FAKE, n_seqs=len(offsets) - 1, T=128, cu_host=host)
    assert st == INVALID


def test_workspace_size_query(lib):
    out = ctypes.c_size_t(123)
    assert lib.kda_chunk_fwd_workspace_size(1, 64, 2, 64, 0, BF16, None) == INVALID
    assert lib.kda_chunk_fwd_workspace_size(1, 64, 2, 128, 0, BF16, ctypes.byref(out)) == UNSUPPORTED
    # C = 32 runs on the CUDA-core kernel, which needs no workspace in either dtype
    for dtype in (BF16, F32):
        out.value = 123
        assert lib.kda_chunk_fwd_workspace_size(4, 4096, 16, 32, 0, dtype, ctypes.byref(out)) == 0
        assert out.value == 0
    assert lib.kda_chunk_fwd_workspace_size(4, 4096, 16, 64, 0, BF16, ctypes.byref(out)) == 0
    assert lib.kda_chunk_fwd_workspace_size(1, 4096, 16, 64, 3, F32, ctypes.byref(out)) == 0


def test_chunk_fwd_rejects_short_workspace(lib):
    need = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(4, 4096, 16, 64, 0, BF16, ctypes.byref(need)) == 0
    if need.value == 0:
        pytest.skip("the library needs no workspace for bf16 prefill")
    assert _chunk(lib, B=4, T=4096, H=16, ws=FAKE, ws_bytes=need.value - 1) == WORKSPACE
    assert _chunk(lib, B=4, T=4096, H=16, ws=None, ws_bytes=need.value) == WORKSPACE


def test_launch_count_query_follows_the_plan():
    """kda_chunk_fwd_launches reports the plan a call takes. Without a GPU the fused grid
    is unavailable (it needs a cooperative-launch check), but the rest of the planning
    is host logic: a long sequence with very few heads takes the segment scan (prep,
    two chain passes, combine), many heads take prep then chains, packed sequences add
    the offset scan, and fp32 input runs one kernel."""
    assert kda.chunk_fwd_launches(1, 3000, 2) == 4
    assert kda.chunk_fwd_launches(1, 300, 72) == 2
    assert kda.chunk_fwd_launches(4, 4096, 16) == 2
    assert kda.chunk_fwd_launches(1, 1000, 2, n_seqs=3) == 3
    assert kda.chunk_fwd_launches(1, 256, 2, dtype=torch.float32) == 1
    assert kda.chunk_fwd_launches(4, 4096, 16, C=32) == 1
    assert kda.chunk_fwd_launches(1, 1000, 2, n_seqs=3, C=32) == 1
    with pytest.raises(kda.KDAError):
        kda.chunk_fwd_launches(1, 256, 2, C=128)
    # the output epilogue is one more kernel after whichever plan the call takes
    assert kda.chunk_fwd_launches(1, 256, 2, C=32, out_epilogue=True) == 2
    assert kda.chunk_fwd_launches(1, 256, 2, dtype=torch.float32, out_epilogue=True) == 2
    assert kda.chunk_fwd_launches(1, 3000, 2, out_epilogue=True) == 5
    assert kda.chunk_fwd_launches(1, 1000, 2, n_seqs=3, out_epilogue=True) == 4


def test_decode_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S=FAKE, o=FAKE, N=4, H=2, dtype=BF16)
        a.update(kw)
        return lib.kda_decode_step(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S"], a["o"],
                                   a["N"], a["H"], a["dtype"], None)

    assert call(dtype=3) == UNSUPPORTED
    assert call(N=0) == INVALID
    assert call(H=-1) == INVALID
    for field in ("q", "k", "v", "la", "beta", "S", "o"):
        assert call(**{field: None}) == INVALID, field
    assert call(S=ctypes.c_void_p((1 << 20) + 4)) == INVALID  # state must be 16-byte aligned


def test_gated_entry_points_validate_the_gate(lib):
    G = kda

    def chunk(gate, la=FAKE, dtype=BF16):
        return lib.kda_chunk_fwd_gated(FAKE, FAKE, FAKE, la, gate, FAKE, None, FAKE, None, 1, 128, 2,
                                       64, None, 0, None, dtype, None, 0, None)

    def decode(gate, la=FAKE):
        return lib.kda_decode_step_gated(FAKE, FAKE, FAKE, la, gate, FAKE, FAKE, FAKE, 4, 2, BF16,
                                         None)

    for bad in (-1, 6, 99):
        assert chunk(bad) == UNSUPPORTED and decode(bad) == UNSUPPORTED
    for gate in (G.KDA_GATE_CHANNEL, G.KDA_GATE_CHANNEL_BF16, G.KDA_GATE_HEAD,
                 G.KDA_GATE_CHANNEL_LOGIT, G.KDA_GATE_CHANNEL_LOGIT_BF16):
        assert chunk(gate, la=None) == INVALID and decode(gate, la=None) == INVALID
    # no gate: log_alpha is not needed (validation goes on to the missing workspace)
    assert chunk(G.KDA_GATE_NONE, la=None) == WORKSPACE
    # per-channel gates are read by TMA on the bf16 path (16-byte base); head gates are fp32
    off8, off2 = ctypes.c_void_p((1 << 20) + 8), ctypes.c_void_p((1 << 20) + 2)
    assert chunk(G.KDA_GATE_CHANNEL, la=off8) == INVALID
    assert chunk(G.KDA_GATE_CHANNEL_BF16, la=off8) == INVALID
    assert chunk(G.KDA_GATE_CHANNEL_LOGIT, la=off8) == INVALID
    assert chunk(G.KDA_GATE_CHANNEL_LOGIT_BF16, la=off8) == INVALID
    assert chunk(G.KDA_GATE_HEAD, la=off8) == WORKSPACE
    assert chunk(G.KDA_GATE_HEAD, la=off2) == INVALID
    assert decode(G.KDA_GATE_HEAD, la=off2) == INVALID


def test_binding_infers_the_gate_layout():
    q = torch.zeros(2, 64, 3, 128, dtype=torch.bfloat16)
    assert kda.gate_kind(torch.zeros(2, 64, 3, 128), q) == kda.KDA_GATE_CHANNEL
    assert kda.gate_kind(torch.zeros(2, 64, 3, 128, dtype=torch.bfloat16), q) == kda.KDA_GATE_CHANNEL_BF16
    assert kda.gate_kind(torch.zeros(2, 64, 3), q) == kda.KDA_GATE_HEAD
    assert kda.gate_kind(None, q) == kda.KDA_GATE_NONE
    for bad in (torch.zeros(2, 64, 3, 1), torch.zeros(2, 64, 3, dtype=torch.bfloat16),
                torch.zeros(2, 64, 3, 128, dtype=torch.float16)):
        with pytest.raises(ValueError):
            kda.gate_kind(bad, q)


def test_binding_refuses_wrong_dtypes_before_calling():
    import torch

    q = torch.zeros(1, 64, 1, 128, dtype=torch.float16)
    with pytest.raises(TypeError):
        kda.chunk_fwd(q, q, q, q.float(), q[..., 0].float())


def test_wait_selftest_rejects_bad_pointers(lib):
    """The failure-path self-test checks its pointers before launching anything."""
    assert lib.kda_selftest_wait_timeout(None, FAKE, None) == INVALID
    assert lib.kda_selftest_wait_timeout(FAKE, None, None) == INVALID
    assert lib.kda_selftest_wait_timeout(ctypes.c_void_p((1 << 20) + 2), FAKE, None) == INVALID
    assert lib.kda_selftest_wait_timeout(FAKE, ctypes.c_void_p((1 << 20) + 1), None) == INVALID


def test_io_entry_points_validate_their_options(lib):
    """kda_chunk_fwd_io / kda_decode_step_io check the fused options before launching."""
    Io = kda.KdaIo

    def chunk(io, dtype=BF16, gate=kda.KDA_GATE_CHANNEL, C=64):
        return lib.kda_chunk_fwd_io(FAKE, FAKE, FAKE, FAKE, gate, FAKE, None, FAKE, None, 1, 128, 2, C,
                                    None, 0, None, dtype, None, 0, ctypes.byref(io), None)

    def decode(io):
        return lib.kda_decode_step_io(FAKE, FAKE, FAKE, FAKE, kda.KDA_GATE_CHANNEL, FAKE, FAKE, FAKE, 4, 2,
                                      BF16, ctypes.byref(io), None)

    gate16 = (1 << 20)
    assert chunk(Io(1, -1.0, 0, None, None, 0.0)) == INVALID            # negative eps
    assert chunk(Io(1, float("nan"), 0, None, None, 0.0)) == INVALID   # NaN eps
    assert chunk(Io(0, 0.0, 0, gate16, None, -1.0)) == INVALID          # negative output eps
    assert chunk(Io(0, 0.0, 0, gate16 + 4, None, 1e-6), dtype=F32) == INVALID  # rows read as float4
    assert chunk(Io(0, 0.0, 0, gate16 + 8, None, 1e-6)) == INVALID     # bf16 gate: 16-byte aligned
    assert chunk(Io(0, 0.0, 0, gate16, gate16 + 4, 1e-6)) == INVALID    # weights: 16-byte aligned
    assert decode(Io(1, -1.0, 0, None, None, 0.0)) == INVALID
    assert decode(Io(0, 0.0, 0, gate16 + 2, None, 1e-6)) == INVALID
    # valid options go on to the next check (the missing workspace)
    assert chunk(Io(1, 1e-6, 1, gate16, gate16, 1e-6)) == WORKSPACE
    n = ctypes.c_int(0)
    # fp32 inputs: the CUDA-core kernel, then the output epilogue
    assert lib.kda_chunk_fwd_io_launches(1, 128, 2, 64, 0, F32, ctypes.byref(Io(0, 0.0, 0, gate16, None, 0.0)),
                                         ctypes.byref(n)) == 0
    assert n.value == 2


def test_backward_validates_before_launching(lib):
    def bwd(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, gate=kda.KDA_GATE_CHANNEL, beta=FAKE, S0=None, do=FAKE,
                 dST=None, dq=FAKE, dk=FAKE, dv=FAKE, dg=FAKE, db=FAKE, dS0=None, B=1, T=128, H=2,
                 cu=None, n=0, cuh=None, dtype=BF16, io=None, ws=None, wsb=0)
        a.update(kw)
        return lib.kda_chunk_bwd(a["q"], a["k"], a["v"], a["la"], a["gate"], a["beta"], a["S0"], a["do"],
                                 a["dST"], a["dq"], a["dk"], a["dv"], a["dg"], a["db"], a["dS0"], a["B"],
                                 a["T"], a["H"], a["cu"], a["n"], a["cuh"], a["dtype"], a["io"], a["ws"],
                                 a["wsb"], None)

    for field in ("q", "k", "v", "beta", "do", "dq", "dk", "dv", "db", "dg"):
        assert bwd(**{field: None}) == INVALID, field
    assert bwd(gate=kda.KDA_GATE_NONE, dg=None) == WORKSPACE  # no gate: no gate gradient needed
    assert bwd(gate=9) == UNSUPPORTED
    assert bwd(dtype=5) == UNSUPPORTED
    assert bwd(B=0) == INVALID
    io = kda.KdaIo(0, 0.0, 0, 1 << 20, None, 1e-6)  # the output epilogue has no backward
    assert bwd(io=ctypes.byref(io)) == UNSUPPORTED
    assert bwd() == WORKSPACE
    n = ctypes.c_size_t(0)
    assert lib.kda_chunk_bwd_workspace_size(4, 4096, 16, 0, ctypes.byref(n)) == 0
    # slot words, shares 6.2 KB per token-head, 64 KB per head every 32 tokens, 256 MiB replay scratch
    assert n.value == (512 + 4 * 4096 * 16 * 4 * 385 + 4 * 128 * 16 * 4 * 4096 + 512 * 32 * 4096) * 4
