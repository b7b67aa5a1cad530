"""Property-based pins of the fp64 oracle (CPU, hypothesis).

The deterministic pins in test_oracle_pins.py fix the oracle on chosen
shapes; these draw shapes, seeds, coefficient schedules and intervals at
random and check the facts that hold for every input:

* Newton-Schulz with per-step coefficients (a_k, b_k, c_k) is the odd matrix
  polynomial X -> composition of p_k on the singular values of the
  Frobenius-normalized X (p_k(s) = a_k s + b_k s^3 + c_k s^5), with the
  singular vectors unchanged;
* the Gram form equals the standard form (both are that polynomial);
* the linear program of the Polar Express schedule gives an error curve
  1 - p that equioscillates (Chebyshev's alternation theorem: four extrema
  of alternating sign at the minimax error).
"""
import numpy as np
from hypothesis import HealthCheck, assume, given, settings
from hypothesis import strategies as st

import oracle as orc

SETTINGS = dict(max_examples=25, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])


def _composed(sched, s):
    for a, b, c in sched:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


# Coefficients near the quintic ones, with p(1) = a + b + c in [0.7, 1.1]; the
# property checks below also assume the composed map stays bounded on [0, 1]
# (a diverging schedule overflows, and then neither side means anything).
schedules = st.lists(
    st.tuples(st.floats(1.5, 3.5), st.floats(0.3, 2.1), st.floats(0.7, 1.1)).map(
        lambda t: (t[0], t[2] - t[0] - t[1], t[1])), min_size=1, max_size=6)


def _bounded(sched):
    s = np.linspace(0.0, 1.0, 2001)
    return bool(np.all(np.abs(_composed(sched, s)) <= 10.0))


@settings(**SETTINGS)
@given(m=st.integers(1, 24), n=st.integers(1, 40), seed=st.integers(0, 2 ** 31 - 1), sched=schedules)
def test_ns_is_the_composed_polynomial_on_singular_values(m, n, seed, sched):
    assume(_bounded(sched))
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((m, n))
    steps = len(sched)
    O = orc.newton_schulz(X, steps=steps, eps=0.0, abc=sched)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    want = (U * _composed(sched, s / np.linalg.norm(X))) @ Vt
    scale = max(1.0, float(np.abs(want).max()))
    assert np.abs(O - want).max() <= 1e-9 * scale


@settings(**SETTINGS)
@given(m=st.integers(1, 24), n=st.integers(1, 40), seed=st.integers(0, 2 ** 31 - 1), sched=schedules)
def test_gram_form_equals_standard_form(m, n, seed, sched):
    assume(_bounded(sched))
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((m, n))
    steps = len(sched)
    a = orc.newton_schulz(X, steps=steps, eps=0.0, abc=sched)
    b = orc.gram_newton_schulz(X, steps=steps, eps=0.0, abc=sched)
    scale = max(1.0, float(np.abs(a).max()))
    assert np.abs(a - b).max() <= 1e-9 * scale


@settings(max_examples=12, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(lo=st.floats(1e-3, 0.6), width=st.floats(0.05, 1.0))
def test_polar_express_lp_equioscillates_on_random_intervals(lo, width):
    hi = lo + width
    coef, E = orc.minimax_quintic_lp(lo, hi)
    x = np.linspace(lo, hi, 200001)
    e = 1.0 - (coef[0] * x + coef[1] * x ** 3 + coef[2] * x ** 5)
    # the LP solver's tolerance is absolute (~1e-8), small next to E unless
    # the interval is short
    assert abs(np.abs(e).max() - E) <= 1e-5 * E + 5e-8
    d = np.diff(e)
    ext = [0] + [i + 1 for i in range(len(d) - 1) if d[i] * d[i + 1] < 0] + [len(x) - 1]
    big = e[ext][np.abs(e[ext]) >= E * (1 - 1e-3) - 5e-8]
    assert len(big) >= 4
    signs = np.sign(big)
    assert np.all(signs[1:] != signs[:-1])
