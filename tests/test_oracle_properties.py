"""Property-based checks of the oracle over randomly drawn shapes, lengths and gates
(hypothesis): the equivalent update form, split-sequence invariance, linearity in (V, S0),
the featurisation's sequence isolation, and the gradient's agreement with finite
differences. The fixed-seed pins of test_oracle_pins.py, test_oracle_featurize.py and
test_oracle_backward.py check one point each; these sweep many small ones."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from tests.test_oracle_pins import alt_form, rand_case

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.function_scoped_fixture])
shapes = st.tuples(st.lists(st.integers(0, 9), min_size=1, max_size=3), st.integers(1, 3), st.integers(1, 6),
                   st.integers(1, 6), st.integers(0, 2 ** 31 - 1))


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b)))) if b.size else 0.0


@SETTINGS
@given(shapes, st.floats(0.25, 2.0))
def test_equivalent_form_random(oracle_mod, shape, scale):
    lengths, H, dk, dv, seed = shape
    q, k, v, la, b, cu, S0 = rand_case(np.random.default_rng(seed), lengths, H, dk, dv)
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0, scale=scale)
    ya, STa = alt_form(q, k, v, la, b, cu, S0, scale)
    assert _rel(y, ya) < 1e-11 and _rel(ST, STa) < 1e-11


@SETTINGS
@given(shapes, st.integers(0, 9))
def test_split_sequence_random(oracle_mod, shape, cut):
    lengths, H, dk, dv, seed = shape
    T = max(1, sum(lengths))
    T1 = cut % (T + 1)
    q, k, v, la, b, cu, S0 = rand_case(np.random.default_rng(seed), (T,), H, dk, dv)
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0)
    ya, Sa, _ = oracle_mod.recurrent(q[:T1], k[:T1], v[:T1], la[:T1], b[:T1], np.array([0, T1]), S0=S0)
    yb, Sb, _ = oracle_mod.recurrent(q[T1:], k[T1:], v[T1:], la[T1:], b[T1:], np.array([0, T - T1]), S0=Sa)
    assert np.array_equal(np.concatenate([ya, yb]), y) and np.array_equal(Sb, ST)


@SETTINGS
@given(shapes, st.floats(-3.0, 3.0))
def test_linearity_random(oracle_mod, shape, c):
    lengths, H, dk, dv, seed = shape
    rng = np.random.default_rng(seed)
    q, k, v1, la, b, cu, S01 = rand_case(rng, lengths, H, dk, dv)
    v2, S02 = rng.standard_normal(v1.shape), rng.standard_normal(S01.shape)
    ya, Sa, _ = oracle_mod.recurrent(q, k, v1 + c * v2, la, b, cu, S0=S01 + c * S02)
    y1, S1, _ = oracle_mod.recurrent(q, k, v1, la, b, cu, S0=S01)
    y2, S2, _ = oracle_mod.recurrent(q, k, v2, la, b, cu, S0=S02)
    assert _rel(ya, y1 + c * y2) < 1e-11 and _rel(Sa, S1 + c * S2) < 1e-11


@SETTINGS
@given(st.lists(st.integers(0, 8), min_size=1, max_size=3), st.integers(1, 2), st.sampled_from([4, 8]),
       st.integers(1, 4), st.integers(0, 2 ** 31 - 1))
def test_featurize_isolation_random(oracle_mod, lengths, H, d, W, seed):
    rng = np.random.default_rng(seed)
    N = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    x = [rng.standard_normal((N, H, d)) for _ in range(3)]
    cw = [rng.standard_normal((H * d, W)) for _ in range(3)]
    g = [rng.standard_normal((N, H)), rng.standard_normal((N, H)), rng.uniform(-1, 1, H), rng.standard_normal(H)]
    packed = oracle_mod.featurize(*x, *cw, *g, cu)
    for i in range(len(lengths)):
        a, b_ = int(cu[i]), int(cu[i + 1])
        alone = oracle_mod.featurize(*[t[a:b_] for t in x], *cw, g[0][a:b_], g[1][a:b_], g[2], g[3], [0, b_ - a])
        for p, s in zip(packed, alone):
            assert np.array_equal(p[a:b_], s)


@SETTINGS
@given(shapes)
def test_backward_finite_differences_random(oracle_mod, shape):
    lengths, H, dk, dv, seed = shape
    rng = np.random.default_rng(seed)
    q, k, v, la, b, cu, S0 = rand_case(rng, lengths, H, dk, dv)
    dy = rng.standard_normal(v.shape)
    dS_T = rng.standard_normal(S0.shape)
    g = oracle_mod.backward(q, k, v, la, b, cu, dy, S0=S0, dS_T=dS_T)

    def loss(**over):
        x = dict(q=q, k=k, v=v, la=la, b=b, S0=S0)
        x.update(over)
        y, ST, _ = oracle_mod.recurrent(x["q"], x["k"], x["v"], x["la"], x["b"], cu, S0=x["S0"])
        return float(np.sum(y * dy) + np.sum(ST * dS_T))
    eps = 1e-6
    for name, arr, grad in zip(("q", "k", "v", "la", "b", "S0"), (q, k, v, la, b, S0), g):
        d = rng.standard_normal(arr.shape)
        fd = (loss(**{name: arr + eps * d}) - loss(**{name: arr - eps * d})) / (2 * eps)
        an = float(np.sum(grad * d))
        assert abs(fd - an) <= 1e-5 * max(1.0, abs(an)), (name, fd, an)
