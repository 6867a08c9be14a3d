"""The fp64 oracle against its pins (closed forms, special cases, a hand-derived
worked example, brute force, finite differences and torch.autograd)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(check):
    check()


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(11)
    x = P.rand_inputs(rng, 3, 3, 20, 4, 5)
    o1, S1 = oracle.fwd(**x, nthreads=1)
    o4, S4 = oracle.fwd(**x, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)
    dO = rng.standard_normal(x["v"].shape)
    g1 = oracle.bwd(**x, dO=dO, nthreads=1)
    g4 = oracle.bwd(**x, dO=dO, nthreads=4)
    for n in g1:
        assert np.array_equal(g1[n], g4[n]), n


def test_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(12)
    x = P.rand_inputs(rng, 1, 2, 0, 3, 2)
    o, ST = oracle.fwd(**x)
    assert o.shape == (1, 2, 0, 2)
    assert np.array_equal(ST, x["S0"])


def test_alpha_hat_power_conventions():
    """0^0 = 1 and 0^tau = 0 for tau > 0 (C pow), seen through T = 1 outputs."""
    B, H, T, dk, dv = 1, 1, 1, 2, 1
    z = np.zeros((B, H, T, dk))
    x = dict(q=np.ones((B, H, T, dk)), k=np.ones((B, H, T, dk)), v=np.ones((B, H, T, dv)),
             g=z.copy(), tau=np.array([0.0, 0.7]).reshape(B, H, T, dk),
             beta=np.ones((B, H, T, dv)))
    o, ST = oracle.fwd(**x)
    assert ST[0, 0, 0, 0] == 1.0 and ST[0, 0, 1, 0] == 0.0
    assert o[0, 0, 0, 0] == 1.0
