"""The fp64 oracle against facts fixed by the pages and by mathematics.

Every pin must hold for the real operator; every planted mistake (a dropped
term, a wrong sign, a gate one token late or on the wrong channel, a readout
before the update or transposed, a missing beta, a decayed write, a readout
with the key) must break at least one pin.
"""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin_holds(pin):
    ok, detail = pin("none")
    assert ok, detail


@pytest.mark.parametrize("mutation", [m for m in oracle.MUTATIONS if m != "none"])
def test_planted_mistake_is_caught(mutation):
    failed = []
    for pin in ALL_PINS:
        ok, detail = pin(mutation)
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {mutation!r}"


def test_thread_count_does_not_change_results():
    import numpy as np
    rng = np.random.default_rng(99)
    T, H = 40, 6
    q = rng.standard_normal((T, H, 8)); k = rng.standard_normal((T, H, 8))
    v = rng.standard_normal((T, H, 4)); g = -0.2 * rng.random((T, H, 8))
    beta = rng.random((T, H)); offs = np.array([0, 13, 13, 40])
    a = oracle.gated_delta(q, k, v, g, beta, None, offs, threads=1)
    b = oracle.gated_delta(q, k, v, g, beta, None, offs, threads=5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_decode_wrapper_matches_prefill_layout():
    import numpy as np
    rng = np.random.default_rng(5)
    steps, N, H, dk, dv = 4, 3, 2, 5, 3
    q = rng.standard_normal((steps, N, H, dk)); k = rng.standard_normal((steps, N, H, dk))
    v = rng.standard_normal((steps, N, H, dv)); g = -0.3 * rng.random((steps, N, H, dk))
    beta = rng.random((steps, N, H)); s0 = rng.standard_normal((N, H, dk, dv))
    o, sT = oracle.decode_steps(q, k, v, g, beta, s0)
    for n in range(N):
        o1, s1 = oracle.gated_delta(q[:, n], k[:, n], v[:, n], g[:, n], beta[:, n], s0[n:n + 1])
        assert np.array_equal(o[:, n], o1) and np.array_equal(sT[n], s1[0])
