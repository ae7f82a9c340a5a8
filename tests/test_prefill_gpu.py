"""kda_chunk_fwd on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_101_b200 as kda
import oracle
from gated_delta_rule_101_b200.inputs import cu_from_lengths, prefill_inputs, varlen_lengths
from parity import check, per_channel_gate

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KIND = {torch.bfloat16: "bf16", torch.float32: "f32"}


def run(inp, **kw):
    o, st = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                          cu_seqlens=inp.cu_seqlens, **kw)
    torch.cuda.synchronize()
    return o, st


def ref(inp):
    la = per_channel_gate(inp.log_alpha, inp.gate, inp.q)
    return oracle.kda_fwd(inp.q, inp.k, inp.v, la, inp.beta, inp.S0,
                          cu_seqlens=None if inp.cu_seqlens is None else inp.cu_seqlens.cpu())


def test_tiny_fp32_config_all_outputs():
    """B=1, T=256, H=2, fp32, S0 = 0: relative L2 <= 1e-4."""
    inp = prefill_inputs(B=1, T=256, H=2, dtype=torch.float32, seed=20260, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, "f32", "o")
    check(st, rs, "f32", "S_T")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 300])
def test_batched_ragged_with_state(dtype, T):
    inp = prefill_inputs(B=2, T=T, H=3, dtype=dtype, s0_std=0.1, seed=T, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], f"o T={T}")
    check(st, rs, KIND[dtype], f"S_T T={T}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_varlen_with_empty_and_ragged_sequences(dtype):
    lengths = [1, 64, 65, 0, 130, 7, 0, 200]
    cu = cu_from_lengths(lengths)
    inp = prefill_inputs(T=int(cu[-1]), H=2, cu_seqlens=cu, dtype=dtype, s0_std=0.1, seed=9,
                         device=DEV)
    o, st = run(inp, cu_seqlens_host=cu)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], "varlen o")
    check(st, rs, KIND[dtype], "varlen S_T")
    # empty sequences keep S0 exactly
    for i, n in enumerate(lengths):
        if n == 0:
            assert torch.equal(st[i], inp.S0[i])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("la_range", [(0.5, 3.0), (5.0, 20.0)])
def test_strong_decay_uses_exact_pairwise_path(la_range, dtype):
    """Chunk log-decay far beyond 80: the factorised exp split would overflow."""
    inp = prefill_inputs(B=1, T=200, H=2, dtype=dtype, la_range=la_range, s0_std=0.1,
                         seed=11, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], "strong decay o")
    check(st, rs, KIND[dtype], "strong decay S_T")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_some_channels_strongly_decayed(dtype):
    """Only a few key channels exceed the factorised range; the rest use the MMA."""
    inp = prefill_inputs(B=2, T=190, H=2, dtype=dtype, s0_std=0.1, seed=21, device=DEV)
    inp.log_alpha[..., 5] = -3.0
    inp.log_alpha[..., 77] = -40.0
    inp.log_alpha[0, 70:80, 1, 100] = -1e4
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], "mixed decay o")
    check(st, rs, KIND[dtype], "mixed decay S_T")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_alpha_zero_and_alpha_one_tokens(dtype):
    inp = prefill_inputs(B=1, T=160, H=2, dtype=dtype, s0_std=0.1, seed=12, device=DEV)
    inp.log_alpha[:, 10:12] = -1e4   # alpha = 0: state reset inside a chunk
    inp.log_alpha[:, 64] = -1e4      # at a chunk start
    inp.log_alpha[:, 100:140] = 0.0  # alpha = 1 (DeltaNet)
    inp.beta[:, 20:30] = 0.0
    inp.beta[:, 30:40] = 1.0
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], "alpha 0/1 o")
    check(st, rs, KIND[dtype], "alpha 0/1 S_T")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_state_carry_across_calls_in_place(dtype):
    """Processing a sequence as several calls, S0 and S_T aliased, equals one call."""
    inp = prefill_inputs(B=2, T=333, H=2, dtype=dtype, s0_std=0.1, seed=13, device=DEV)
    o_full, st_full = run(inp)
    S = inp.S0.clone()
    outs = []
    for a, z in ((0, 64), (64, 100), (100, 101), (101, 333)):
        o, _ = kda.chunk_fwd(inp.q[:, a:z].contiguous(), inp.k[:, a:z].contiguous(),
                             inp.v[:, a:z].contiguous(), inp.log_alpha[:, a:z].contiguous(),
                             inp.beta[:, a:z].contiguous(), S, state_out=S)
        outs.append(o)
    torch.cuda.synchronize()
    ro, rs = ref(inp)
    check(torch.cat(outs, dim=1), ro, KIND[dtype], "carry o")
    check(S, rs, KIND[dtype], "carry S_T")
    check(o_full, ro, KIND[dtype], "single call o")


def test_decode_loop_equals_prefill():
    inp = prefill_inputs(B=2, T=70, H=2, dtype=torch.float32, s0_std=0.1, seed=14, device=DEV)
    o_p, st_p = run(inp)
    S = inp.S0.clone()
    o_d = torch.empty_like(inp.v)
    for t in range(70):
        o_d[:, t] = kda.decode_step(inp.q[:, t].contiguous(), inp.k[:, t].contiguous(),
                                    inp.v[:, t].contiguous(), inp.log_alpha[:, t].contiguous(),
                                    inp.beta[:, t].contiguous(), S)
    torch.cuda.synchronize()
    check(o_d, o_p.double(), "f32", "decode loop vs prefill o")
    check(S, st_p.double(), "f32", "decode loop vs prefill S")


def test_deterministic_bitwise():
    inp = prefill_inputs(B=2, T=500, H=3, dtype=torch.bfloat16, s0_std=0.1, seed=15, device=DEV)
    o1, s1 = run(inp)
    o2, s2 = run(inp)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_no_final_state_requested():
    inp = prefill_inputs(B=1, T=100, H=2, dtype=torch.bfloat16, seed=16, device=DEV)
    o, st = run(inp, final_state=False)
    assert st is None
    ro, _ = ref(inp)
    check(o, ro, "bf16", "o without S_T")


# ---------------------------------------------------------------- full sizes, sampled
def _sample_ref(inp, seqs, heads, cols):
    """Oracle on sampled (sequence, head) pairs and value columns, whole sequences."""
    out = []
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.cpu().tolist()
    la_full = per_channel_gate(inp.log_alpha, inp.gate, inp.q)
    for s, h in zip(seqs, heads):
        if cu is None:
            sl = (slice(s, s + 1), slice(None))
            pick = lambda x: x[sl][:, :, h:h + 1]
        else:
            a, z = cu[s], cu[s + 1]
            pick = lambda x: x[a:z, h:h + 1][None]
        q, k, la = pick(inp.q), pick(inp.k), pick(la_full)
        v = pick(inp.v)[..., cols]
        b = pick(inp.beta[..., None])[..., 0]
        S0 = None if inp.S0 is None else inp.S0[s, h][:, cols][None, None]
        out.append(oracle.kda_fwd(q, k, v, la, b, S0))
    return out


def _check_sampled(inp, o, st, seqs, heads, cols, kind, what):
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.cpu().tolist()
    for (s, h), (ro, rs) in zip(zip(seqs, heads), _sample_ref(inp, seqs, heads, cols)):
        got_o = o[s, :, h][:, cols] if cu is None else o[cu[s]:cu[s + 1], h][:, cols]
        check(got_o, ro[0, :, 0], kind, f"{what} o (seq {s}, head {h})")
        check(st[s, h][:, cols], rs[0, 0], kind, f"{what} S_T (seq {s}, head {h})")


def test_prefill_workload_b4_t4096_h16_sampled():
    inp = prefill_inputs(B=4, T=4096, H=16, dtype=torch.bfloat16, s0_std=0.1, seed=20261,
                         device=DEV)
    o, st = run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(st).all()
    cols = list(range(128))
    _check_sampled(inp, o, st, [0, 3, 1, 2], [0, 15, 7, 9], cols, "bf16", "B4 T4096 H16")


def _packed_pairs_ref(inp, pairs):
    """The oracle on several (sequence, head) pairs of a packed batch in one call: the
    pairs become the sequences of a one-head packed batch, so the oracle's threads take
    them in parallel. Returns one (o [len, 128], S_T [128, 128]) per pair."""
    cu = inp.cu_seqlens.cpu().tolist()
    la_full = per_channel_gate(inp.log_alpha, inp.gate, inp.q)
    parts = {n: [] for n in ("q", "k", "v", "la", "b")}
    lens, S0 = [], []
    for s, h in pairs:
        a, z = cu[s], cu[s + 1]
        for n, x in (("q", inp.q), ("k", inp.k), ("v", inp.v), ("la", la_full)):
            parts[n].append(x[a:z, h:h + 1].cpu())
        parts["b"].append(inp.beta[a:z, h:h + 1].cpu())
        lens.append(z - a)
        S0.append(None if inp.S0 is None else inp.S0[s, h][None].cpu())
    cat = {n: torch.cat(x) for n, x in parts.items()}
    s0 = None if inp.S0 is None else torch.stack(S0)
    ro, rs = oracle.kda_fwd(cat["q"], cat["k"], cat["v"], cat["la"], cat["b"], s0,
                            cu_seqlens=cu_from_lengths(lens))
    offs = np.concatenate([[0], np.cumsum(lens)])
    return [(ro[offs[i]:offs[i + 1], 0], rs[i, 0]) for i in range(len(pairs))]


def test_varlen_workload_64_seqs_h32_sampled():
    """Every value column of eight (sequence, head) pairs, the shortest and the longest
    sequence among them, against the oracle (run on all eight at once)."""
    lengths = varlen_lengths(64, 512, 16384, seed=20262)
    cu = cu_from_lengths(lengths)
    inp = prefill_inputs(T=int(cu[-1]), H=32, cu_seqlens=cu, dtype=torch.bfloat16, seed=20262,
                         device=DEV)
    o, st = run(inp, cu_seqlens_host=cu)
    assert torch.isfinite(o.float()).all() and torch.isfinite(st).all()
    order = np.argsort(lengths)
    seqs = [int(order[0]), int(order[-1]), int(order[1]), int(order[-2]), 0, 63, 31, int(order[32])]
    heads = [0, 31, 17, 5, 9, 24, 2, 12]
    for (s, h), (ro, rs) in zip(zip(seqs, heads), _packed_pairs_ref(inp, list(zip(seqs, heads)))):
        what = f"varlen 64 seqs (seq {s}, {lengths[s]} tokens, head {h})"
        check(o[cu[s]:cu[s + 1], h], ro, "bf16", what + " o")
        check(st[s, h], rs, "bf16", what + " S_T")


def test_long_context_1m_tokens_as_16_calls_sampled():
    """B=1, T=2^20 processed as 16 calls of 65,536 tokens with the state carried in place.
    Eight heads, every value column: o of every call and the final S_T against the
    oracle, which carries its own fp64 state through the calls."""
    H, Tc, calls = 32, 65536, 16
    heads = [0, 5, 9, 14, 18, 23, 27, 31]
    S = torch.zeros(1, H, 128, 128, dtype=torch.float32, device=DEV)
    S_ref = np.zeros((1, len(heads), 128, 128))
    for c in range(calls):
        inp = prefill_inputs(B=1, T=Tc, H=H, dtype=torch.bfloat16, la_range=(0.0001, 0.05),
                             seed=20264 * 100 + c, device=DEV)
        o, _ = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, S, state_out=S)
        torch.cuda.synchronize()
        sl = lambda x: x[:, :, heads].cpu()
        ro, S_ref = oracle.kda_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.beta), S_ref)
        for i, h in enumerate(heads):
            check(o[0, :, h], ro[0, :, i], "bf16", f"1M-token call {c} o (head {h})")
    for i, h in enumerate(heads):
        check(S[0, h], S_ref[0, i], "bf16", f"1M-token final S_T (head {h})")
    assert torch.isfinite(S).all()


def test_many_sequence_heads_take_full_width_chain():
    """100 sequence-heads: two 64-column chains each would need two waves on 148 SMs, so
    the call runs one 128-column chain CTA per (sequence, head) (chosen by wave count),
    which also issues each chunk's U product one chunk early."""
    inp = prefill_inputs(B=2, T=130, H=50, dtype=torch.bfloat16, s0_std=0.1, seed=22, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, "bf16", "128-column chain o")
    check(st, rs, "bf16", "128-column chain S_T")


# ---------------------------------------------------------------- each bf16 path
# A batched bf16 call runs one of three plans; kda_chunk_fwd_launches tells which:
# prep then chains (2 launches), the fused cooperative grid (1), or the segment scan
# for long sequences with few sequence-heads (4: prep, pass 1, combine, pass 2). Each
# gets ragged tails, strongly decayed channels, alpha = 0 / 1 tokens and a carried
# state. (B, T, H) are chosen far from the boundaries between the plans.
PATHS = {"fused_grid": (1, 1000, 32, 1), "prep_then_chain": (1, 300, 72, 2),
         "segment_scan": (1, 3000, 2, 4), "segment_scan_batched": (2, 8000, 2, 4)}


def _stress_gates(inp):
    H = inp.q.shape[2]
    hh = min(3, H - 1)
    inp.log_alpha[..., 5] = -3.0               # one channel decays fast everywhere
    inp.log_alpha[0, 100:140, hh, 77] = -40.0  # a burst beyond the factorised range
    inp.log_alpha[0, 10, hh, 100] = -1e4       # alpha = 0 for one channel of one token
    inp.log_alpha[0, 20:30, 0] = 0.0           # alpha = 1 tokens
    return inp


@pytest.mark.parametrize("path", list(PATHS))
def test_each_bf16_path_against_the_oracle(path):
    B, T, H, launches = PATHS[path]
    assert kda.chunk_fwd_launches(B, T, H) == launches
    inp = _stress_gates(prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=0.1, seed=31,
                                       device=DEV))
    o, st = run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(st).all()
    seqs = [0, 0, B - 1]
    heads = [0, min(3, H - 1), H - 1]
    _check_sampled(inp, o, st, seqs, heads, list(range(128)), "bf16", path)


def test_fused_grid_carries_state_across_calls():
    """Two fused calls of 500 tokens with the state carried in place equal the oracle
    run over all 1000 tokens."""
    H = 32
    assert kda.chunk_fwd_launches(1, 500, H) == 1
    inp = _stress_gates(prefill_inputs(B=1, T=1000, H=H, dtype=torch.bfloat16, s0_std=0.1,
                                       seed=32, device=DEV))
    S = inp.S0.clone()
    o = torch.empty_like(inp.v)
    for a in (0, 500):
        sl = lambda x: x[:, a:a + 500].contiguous()
        oc, _ = kda.chunk_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.beta), S,
                              state_out=S)
        o[:, a:a + 500] = oc
    torch.cuda.synchronize()
    _check_sampled(inp, o, S, [0, 0], [3, 17], list(range(128)), "bf16", "fused, two calls")


def test_segment_scan_carries_state_across_calls():
    """Two segment-scan calls of 3,000 tokens with the state carried in place equal the
    oracle run over all 6,000 tokens."""
    H, Tc = 2, 3000
    assert kda.chunk_fwd_launches(1, Tc, H) == 4
    inp = _stress_gates(prefill_inputs(B=1, T=2 * Tc, H=H, dtype=torch.bfloat16, s0_std=0.1,
                                       seed=33, device=DEV))
    S = inp.S0.clone()
    o = torch.empty_like(inp.v)
    for a in (0, Tc):
        sl = lambda x: x[:, a:a + Tc].contiguous()
        oc, _ = kda.chunk_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.beta), S,
                              state_out=S)
        o[:, a:a + Tc] = oc
    torch.cuda.synchronize()
    _check_sampled(inp, o, S, [0, 0], [0, 1], list(range(128)), "bf16", "segment scan, two calls")


def test_wide_chain_all_outputs():
    """One 128-column chain CTA per sequence-head (100 of them, see above), 4 chunks with a
    ragged last one, carried state, every output."""
    assert kda.chunk_fwd_launches(2, 200, 50) == 2
    inp = prefill_inputs(B=2, T=200, H=50, dtype=torch.bfloat16, s0_std=0.1, seed=48, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, "bf16", "wide chain o")
    check(st, rs, "bf16", "wide chain S_T")


def test_wide_chain_packed_with_empty_sequences():
    """8 packed sequences x 40 heads (320 sequence-heads: 128-column chains)."""
    lengths = [0, 130, 64, 1, 257, 0, 65, 190]
    cu = cu_from_lengths(lengths)
    inp = prefill_inputs(T=int(cu[-1]), H=40, cu_seqlens=cu, dtype=torch.bfloat16, s0_std=0.1,
                         seed=49, gate="head", device=DEV)
    o, st = run(inp, cu_seqlens_host=cu)
    ro, rs = ref(inp)
    check(o, ro, "bf16", "wide chain packed o")
    check(st, rs, "bf16", "wide chain packed S_T")
    for i, n in enumerate(lengths):
        if n == 0:
            assert torch.equal(st[i], inp.S0[i])


@pytest.mark.parametrize("path", ["prep_then_chain", "segment_scan"])
def test_prefill_captured_in_a_cuda_graph(path):
    """A call captured in a CUDA graph replays to the eager result bit for bit; the
    chain (or the segment scan's first pass) is launched as a dependent of the prep."""
    B, T, H, launches = PATHS[path]
    assert kda.chunk_fwd_launches(B, T, H) == launches
    inp = prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=0.1, seed=47, device=DEV)
    o_eager, s_eager = run(inp)
    ws = torch.empty(kda.workspace_size(B, T, H), dtype=torch.uint8, device=DEV)
    o, st = torch.empty_like(inp.v), torch.empty_like(inp.S0)
    call = lambda: kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, out=o,
                                 state_out=st, workspace=ws)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    o.zero_()
    st.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_eager) and torch.equal(st, s_eager)
    del graph


# ---- gate layouts: Gated DeltaNet (one rate per head), DeltaNet (no gate), bf16 gate
LAYOUTS = ["channel_bf16", "head", "none"]


@pytest.mark.parametrize("gate", LAYOUTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gate_layouts_against_the_oracle(gate, dtype):
    inp = prefill_inputs(B=2, T=300, H=3, dtype=dtype, s0_std=0.1, seed=41, gate=gate, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], f"{gate} o")
    check(st, rs, KIND[dtype], f"{gate} S_T")


@pytest.mark.parametrize("gate", ["channel_bf16", "head"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gate_layouts_strong_decay(gate, dtype):
    """Chunk log-decay beyond the factorised range in every channel (head gate) or in
    many (bf16 gate): the exact pairwise path reads the gate in its own layout."""
    inp = prefill_inputs(B=1, T=200, H=2, dtype=dtype, la_range=(0.5, 3.0), s0_std=0.1,
                         seed=42, gate=gate, device=DEV)
    o, st = run(inp)
    ro, rs = ref(inp)
    check(o, ro, KIND[dtype], f"{gate} strong decay o")
    check(st, rs, KIND[dtype], f"{gate} strong decay S_T")


@pytest.mark.parametrize("gate", LAYOUTS)
@pytest.mark.parametrize("path", ["fused_grid", "segment_scan"])
def test_gate_layouts_on_each_bf16_plan(gate, path):
    B, T, H, launches = PATHS[path]
    assert kda.chunk_fwd_launches(B, T, H) == launches
    inp = prefill_inputs(B=B, T=T, H=H, dtype=torch.bfloat16, s0_std=0.1, seed=43, gate=gate,
                         device=DEV)
    o, st = run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(st).all()
    _check_sampled(inp, o, st, [0, B - 1], [0, H - 1], list(range(128)), "bf16", f"{path} {gate}")


@pytest.mark.parametrize("gate", ["channel_bf16", "head"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gate_layout_equals_the_widened_channel_gate(gate, dtype):
    """A head-wide or bf16 gate gives bit-for-bit the result of the same gate widened to
    fp32 per channel: the layouts differ only in how the rates are read."""
    inp = prefill_inputs(B=2, T=200, H=3, dtype=dtype, s0_std=0.1, seed=44, gate=gate, device=DEV)
    o1, s1 = run(inp)
    wide = per_channel_gate(inp.log_alpha, gate, inp.q).contiguous()
    o2, s2 = kda.chunk_fwd(inp.q, inp.k, inp.v, wide, inp.beta, inp.S0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_gate_layout_none_needs_no_tensor_and_is_checked():
    """No gate: log_alpha may be None; a gate tensor of another shape is refused."""
    inp = prefill_inputs(B=1, T=70, H=2, dtype=torch.bfloat16, seed=45, gate="head", device=DEV)
    with pytest.raises(ValueError):
        kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha[..., :1], inp.beta)
    assert kda.gate_kind(None, inp.q) == kda.KDA_GATE_NONE
    assert kda.gate_kind(inp.log_alpha, inp.q) == kda.KDA_GATE_HEAD


def test_no_bounded_wait_timed_out():
    """Every tensor-core kernel run so far finished without a wait giving up."""
    import ctypes

    st = ctypes.c_int(-1)
    assert kda.lib().kda_get_device_status(ctypes.byref(st)) == 0
    assert st.value == 0
