"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.forward)


def test_threads_do_not_change_result():
    import numpy as np
    r = np.random.default_rng(5)
    q, k, v = (r.standard_normal((2, 3, 32, 8)) for _ in range(3))
    beta = r.standard_normal(3)
    a = oracle.forward(q, k, v, beta, seg_len=8, nthreads=1)
    b = oracle.forward(q, k, v, beta, seg_len=8, nthreads=4)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_segment_sampling_matches_full_run():
    import numpy as np
    r = np.random.default_rng(6)
    q, k, v = (r.standard_normal((1, 2, 40, 4)) for _ in range(3))
    beta = r.standard_normal(2)
    full, M, z = oracle.forward(q, k, v, beta, seg_len=8)
    part, M2, z2 = oracle.forward(q, k, v, beta, seg_len=8, segments=[4, 1])
    assert np.array_equal(part[:, :, 0], full[:, :, 32:40])
    assert np.array_equal(part[:, :, 1], full[:, :, 8:16])
    assert np.array_equal(M, M2) and np.array_equal(z, z2)


def test_rejects_partial_segment():
    import numpy as np
    x = np.zeros((1, 1, 10, 4))
    with pytest.raises(ValueError):
        oracle.forward(x, x, x, [0.0], seg_len=4)
