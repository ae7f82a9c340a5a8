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
