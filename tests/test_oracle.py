"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oracle.kda_fwd)


def test_oracle_threads_do_not_change_results():
    from oracle_pins import rand_case
    import numpy as np

    c = rand_case(3, B=3, T=40, H=3, dk=16, dv=70)
    o1, s1 = oracle.kda_fwd(**c, threads=1)
    o8, s8 = oracle.kda_fwd(**c, threads=8)
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)


def test_oracle_rejects_bad_offsets():
    import numpy as np

    c = {k: v[0] for k, v in __import__("oracle_pins").rand_case(5, B=1, T=10, H=1, dk=4, dv=4).items() if k != "S0"}
    with pytest.raises(RuntimeError):
        oracle.kda_fwd(**c, cu_seqlens=np.array([0, 6, 4, 10]))


def test_io_reference_formulas():
    """The fp64 pre- and post-processing the fused-IO tests feed the oracle, on values
    with known results."""
    import numpy as np

    from io_ref import l2norm_rows, log_sigmoid, rmsnorm_gate, sigmoid

    assert np.isclose(log_sigmoid(0.0), -np.log(2.0))
    assert np.isclose(log_sigmoid(50.0), -np.exp(-50.0), rtol=1e-12)  # no cancellation
    assert np.isclose(log_sigmoid(-50.0), -50.0 - np.exp(-50.0))      # no overflow
    assert np.isclose(sigmoid(0.0), 0.5)
    v = np.array([[3.0, 4.0], [0.0, 0.0]])
    assert np.allclose(l2norm_rows(v, 0.0)[0], [0.6, 0.8])
    assert np.allclose(l2norm_rows(v, 1e-6)[1], 0.0)
    # a constant row normalises to its sign; the weight and the gate then scale it
    o = np.array([[-2.0, -2.0, -2.0, -2.0]])
    w = np.array([1.0, 2.0, 3.0, 4.0])
    assert np.allclose(rmsnorm_gate(o, np.zeros(4), w, 0.0), -0.5 * w)


def test_l2norm_backward_formula_against_finite_differences():
    import numpy as np

    from io_ref import l2norm_rows, l2norm_rows_bwd

    rng = np.random.default_rng(3)
    y, dx = rng.normal(size=(3, 8)), rng.normal(size=(3, 8))
    g = l2norm_rows_bwd(y, dx, 1e-3)
    h = 1e-6
    for i in range(3):
        for c in range(8):
            e = np.zeros_like(y)
            e[i, c] = h
            fd = np.sum((l2norm_rows(y + e, 1e-3) - l2norm_rows(y - e, 1e-3)) * dx) / (2 * h)
            assert abs(fd - g[i, c]) < 1e-7
