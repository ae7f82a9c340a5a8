"""The bf16 path's error budget, modelled on the CPU (no GPU needed).

``bf16_model`` runs the chunk algebra with the bf16 path's roundings. Its error
against the oracle is the error the GPU path is expected to show: on the bench's
prefill workload the model gives relative L2 4.1e-3 (o) and 2.9e-3 (S_T), where the
B200 measured 4.1e-3 and 3.0e-3. The tests keep the model honest and show that
operand rounding alone lands well inside the 1e-2 bar.
"""
import numpy as np
import torch

import oracle
from bf16_model import bf16, kda_bf16_model
from gated_delta_rule_101_b200.inputs import prefill_inputs


def test_rounding_is_bf16_round_to_nearest_even():
    x = np.random.default_rng(0).standard_normal(20000) * np.exp(np.random.default_rng(1).uniform(-20, 20, 20000))
    want = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(bf16(x), want)


def test_operand_rounding_alone_stays_inside_the_bar():
    inp = prefill_inputs(B=1, T=1024, H=2, dtype=torch.bfloat16, s0_std=0.1, seed=20261)
    f = lambda t: t.double().numpy()
    ro, rs = oracle.kda_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0)
    mo, ms = kda_bf16_model(f(inp.q), f(inp.k), f(inp.v), f(inp.log_alpha), f(inp.beta), f(inp.S0))
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    for name, e in (("o", rel(mo, ro)), ("S_T", rel(ms, rs))):
        assert 1e-3 < e < 6e-3, f"{name}: modelled rel-L2 {e:.3e}"
