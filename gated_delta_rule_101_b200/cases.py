"""Runs one library call on a named synthetic workload a few times: the target of a
profiler capture (``ncu -k <kernel> -s <launches to skip> -c 1 python -m
gated_delta_rule_101_b200.cases <case> ...``) and a quick timing.

Cases (sizes default to the benchmark workloads, or a smaller size where a full
capture of the benchmark's would hold too much memory):

* ``prefill``     kda_chunk_fwd, bf16, C = 64: kda_prep_kernel, then kda_chain_kernel
                  (or the fused grid / segment scan, as the planner picks for the shape)
* ``prefill_io``  kda_chunk_fwd_io with every fused step (logit gate, q/k L2Norm, beta
                  logits, output RMSNorm and sigmoid gate): prep, chains, kda_out_epilogue_kernel
* ``simt``        kda_chunk_fwd with fp32 inputs (or ``--dtype bf16 --chunk 32``):
                  prefill_simt_kernel
* ``backward``    kda_chunk_bwd: kda_bwd_slice_kernel, kda_bwd_reduce_kernel
* ``decode``      kda_decode_step, N sequences x H heads

Each run prints one JSON line: the case, its shape, the kernels per call and the
median time per call (CUDA events on the launching stream, L2 not flushed).
"""
from __future__ import annotations

import argparse
import json

import torch

import gated_delta_rule_101_b200 as kda
from gated_delta_rule_101_b200.inputs import cu_from_lengths, decode_inputs, prefill_inputs, varlen_lengths


def _shape(text: str, n: int) -> tuple[int, ...]:
    vals = tuple(int(x) for x in text.split(","))
    if len(vals) != n:
        raise SystemExit(f"expected {n} comma-separated sizes, got {text!r}")
    return vals


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("case", choices=["prefill", "prefill_io", "simt", "backward", "decode"])
    ap.add_argument("--shape", default=None, help="B,T,H (prefill cases, backward) or N,H (decode)")
    ap.add_argument("--gate", default="channel", choices=["channel", "channel_bf16", "head", "none"])
    ap.add_argument("--dtype", default=None, choices=["bf16", "f32"])
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--packed", type=int, default=0,
                    help="prefill cases: this many packed sequences of lengths U[512, 16384] "
                         "(one row, T their sum) instead of B x T")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seed", type=int, default=20261)
    args = ap.parse_args(argv)

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kda.lib()
    stream = torch.cuda.current_stream(dev)
    default_dtype = "f32" if args.case == "simt" else "bf16"
    dtype = {"bf16": torch.bfloat16, "f32": torch.float32}[args.dtype or default_dtype]

    if args.case == "decode":
        N, H = _shape(args.shape or "256,32", 2)
        inp = decode_inputs(steps=1, N=N, H=H, dtype=dtype, s0_std=0.1, seed=args.seed, gate=args.gate,
                            device=dev)
        S = inp.S.clone()
        out = torch.empty_like(inp.v[0])
        fn = lambda: kda.decode_step(inp.q[0], inp.k[0], inp.v[0], inp.log_alpha[0], inp.beta[0], S, out=out)
        shape, launches = {"N": N, "H": H}, 1
    else:
        B, T, H = _shape(args.shape or ("2,2048,16" if args.case == "backward" else "4,4096,16"), 3)
        cu, n_seqs = None, 0
        if args.packed:
            cu = cu_from_lengths(varlen_lengths(args.packed, 512, 16384, seed=args.seed))
            B, T, n_seqs = 1, int(cu[-1]), args.packed
        inp = prefill_inputs(B=B, T=T, H=H, dtype=dtype, s0_std=0.1, seed=args.seed, gate=args.gate,
                             cu_seqlens=cu, device=dev)
        shape = {"B": B, "T": T, "H": H, "n_seqs": n_seqs, "gate": args.gate, "dtype": str(dtype).split(".")[-1]}
        pk = dict(cu_seqlens=inp.cu_seqlens, cu_seqlens_host=cu) if cu is not None else {}
        o = torch.empty_like(inp.v)
        S_T = torch.empty_like(inp.S0)
        if args.case == "backward":
            g = torch.Generator(device="cpu").manual_seed(args.seed + 1)
            dout = torch.randn(inp.v.shape, generator=g).to(dtype).to(dev)
            dS_T = torch.randn(inp.S0.shape, generator=g).to(dev)
            fn = lambda: kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, dout, dS_T, **pk)
            launches = 2
        elif args.case == "prefill_io":
            if args.gate not in ("channel", "channel_bf16"):
                raise SystemExit("prefill_io takes a per-channel gate (given as logits)")
            z = (torch.rand(inp.q.shape, device=dev) * 5 + 2).to(inp.log_alpha.dtype)
            og = torch.randn_like(inp.v)
            w = torch.ones(128, device=dev)
            ws = torch.empty(kda.workspace_size(B, T, H, n_seqs), dtype=torch.uint8, device=dev)
            fn = lambda: kda.chunk_fwd(inp.q, inp.k, inp.v, z, inp.beta, inp.S0, out=o, state_out=S_T,
                                       workspace=ws, gate_logits=True, qk_l2norm=True, beta_logits=True,
                                       out_gate=og, out_norm_weight=w, **pk)
            launches = kda.chunk_fwd_launches(B, T, H, n_seqs=n_seqs, out_epilogue=True)
        else:
            C = args.chunk
            ws_n = kda.workspace_size(B, T, H, n_seqs, dtype, C)
            ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
            fn = lambda: kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, out=o,
                                       state_out=S_T, workspace=ws, C=C, **pk)
            launches = kda.chunk_fwd_launches(B, T, H, n_seqs=n_seqs, dtype=dtype, C=C)
            shape["C"] = C

    fn()  # warm-up (one call's launches before the captured ones)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    st = kda.device_status()
    if st:
        raise SystemExit(f"device status {st:#x} after the calls")
    times.sort()
    print(json.dumps({"case": args.case, "shape": shape, "kernels_per_call": launches,
                      "ms_per_call_median": times[len(times) // 2], "reps": args.reps}), flush=True)


if __name__ == "__main__":
    main()
