"""The CPU oracle against its pins (no GPU): worked examples, library routines, closed
forms, special cases and exact-distribution enumeration."""
import pytest

import oracle
from tests import oracle_pins as P


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", [p for p in P.ALL_PINS if p is not P.pin_exact_distribution],
                         ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)


@pytest.mark.parametrize("K", [1, 2, 3])
def test_exact_distribution(o, K):
    P.pin_exact_distribution(o, K=K, V=8)


def test_threads_do_not_change_results(o):
    import numpy as np
    rng = np.random.default_rng(5)
    B, K, V = 33, 3, 64
    t = rng.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    q = (t[:, :K] + rng.normal(0, 1, size=(B, K, V))).astype(np.float32)
    d = rng.integers(0, V, size=(B, K)).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    r1 = o.verify_rejection(t, q, d, u, threads=1)
    r4 = o.verify_rejection(t, q, d, u, threads=4)
    for k in r1:
        if k != "err":
            assert np.array_equal(r1[k], r4[k]), k
    g1 = o.verify_greedy(t, d, want_lse=True, threads=1)
    g4 = o.verify_greedy(t, d, want_lse=True, threads=5)
    for k in ("out_tokens", "accepted_len", "bonus", "target_lse"):
        assert np.array_equal(g1[k], g4[k]), k
