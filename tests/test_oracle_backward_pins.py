"""Pins for the oracle's attention backward, against central finite differences
of the forward oracle (CPU only).

Loss = sum(out * W) for a fixed random W, so dO = W; every element of q, k, v
and the sink logits is perturbed by +-h and the loss difference compared with
the analytic gradient.  A backward that dropped the sink's gradient, the
D = <dO, O> term or the GQA sum over heads fails these.
"""

import numpy as np
import pytest

import oracle
from oracle.backward import prefill_backward


def _loss(q, k, v, s, W, window, cu, scale, v_scale):
    out, _ = oracle.prefill(q, k, v, s, window, cu, scale=scale, v_scale=v_scale)
    return float((out * W).sum())


def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + h
        fp = f()
        x[i] = old - h
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


@pytest.mark.parametrize("window,lengths", [(0, [7]), (3, [7]), (0, [3, 0, 5]), (2, [4, 6])])
@pytest.mark.parametrize("sinks", [True, False])
def test_gradients_match_finite_differences(window, lengths, sinks):
    rng = np.random.default_rng(sum(lengths) + window)
    Nt = sum(lengths)
    Hq, Hkv, Dqk, Dv = 4, 2, 5, 3
    q = rng.standard_normal((Nt, Hq, Dqk))
    k = rng.standard_normal((Nt, Hkv, Dqk))
    v = rng.standard_normal((Nt, Hkv, Dv))
    s = rng.standard_normal(Hq) if sinks else None
    W = rng.standard_normal((Nt, Hq, Dv))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    scale, v_scale = 0.37, 0.8
    f = lambda: _loss(q, k, v, s, W, window, cu, scale, v_scale)  # noqa: E731
    dq, dk, dv, ds = prefill_backward(q, k, v, W, s, window, cu, scale=scale, v_scale=v_scale)
    np.testing.assert_allclose(dq, _fd(f, q), atol=2e-8)
    np.testing.assert_allclose(dk, _fd(f, k), atol=2e-8)
    np.testing.assert_allclose(dv, _fd(f, v), atol=2e-8)
    if sinks:
        np.testing.assert_allclose(ds, _fd(f, s), atol=2e-8)
    else:
        assert ds is None


def test_pins_have_teeth():
    """Dropping the sink gradient or the D term changes the result."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal((6, 2, 4))
    k = rng.standard_normal((6, 1, 4))
    v = rng.standard_normal((6, 1, 3))
    s = np.array([1.5, -0.5])
    W = rng.standard_normal((6, 2, 3))
    cu = np.array([0, 6])
    dq, dk, dv, ds = prefill_backward(q, k, v, W, s, 0, cu)
    assert np.abs(ds).max() > 1e-3                     # the sink has a real gradient
    out, _ = oracle.prefill(q, k, v, s, 0, cu)
    D = (W * out).sum(axis=2)
    assert np.abs(D).max() > 1e-3                      # D matters for dS


@pytest.mark.parametrize("window", [0, 3])
@pytest.mark.parametrize("sinks", [True, False])
def test_sampled_gradients_match_finite_differences(window, sinks):
    """The sampled-position backward (used at sizes the full one cannot reach)
    against central differences of the forward, with blocks smaller than the
    sequence so that its row blocking is exercised."""
    rng = np.random.default_rng(40 + window)
    n, Hq, Hkv, Dqk, Dv = 9, 4, 2, 5, 3
    q = rng.standard_normal((n, Hq, Dqk))
    k = rng.standard_normal((n, Hkv, Dqk))
    v = rng.standard_normal((n, Hkv, Dv))
    s = rng.standard_normal(Hq) if sinks else None
    W = rng.standard_normal((n, Hq, Dv))
    cu = np.array([0, n])
    scale, v_scale = 0.41, 1.3
    f = lambda: _loss(q, k, v, s, W, window, cu, scale, v_scale)  # noqa: E731
    gq, gk, gv = _fd(f, q), _fd(f, k), _fd(f, v)
    q_rows, q_heads, k_rows, kv_heads = [0, 4, 8], [1, 3], [0, 5, 8], [0, 1]
    dq, dk, dv, ds = oracle.backward.prefill_backward_sampled(
        q, k, v, W, s, window, q_rows, q_heads, k_rows, kv_heads, sink_heads=[0, 2] if sinks else (),
        scale=scale, v_scale=v_scale, block=4)
    np.testing.assert_allclose(dq, gq[np.ix_(q_rows, q_heads)], atol=2e-8)
    np.testing.assert_allclose(dk, gk[np.ix_(k_rows, kv_heads)], atol=2e-8)
    np.testing.assert_allclose(dv, gv[np.ix_(k_rows, kv_heads)], atol=2e-8)
    if sinks:
        np.testing.assert_allclose(ds, _fd(f, s)[[0, 2]], atol=2e-8)


def test_sampled_equals_full_backward():
    rng = np.random.default_rng(7)
    n, Hq, Hkv = 40, 4, 1
    q = rng.standard_normal((n, Hq, 6))
    k = rng.standard_normal((n, Hkv, 6))
    v = rng.standard_normal((n, Hkv, 2))
    s = rng.standard_normal(Hq)
    W = rng.standard_normal((n, Hq, 2))
    for window in (0, 7):
        dq, dk, dv, ds = prefill_backward(q, k, v, W, s, window, np.array([0, n]))
        rows = list(range(n))
        sq, sk, sv, ss = oracle.backward.prefill_backward_sampled(
            q, k, v, W, s, window, rows, list(range(Hq)), rows, [0], sink_heads=list(range(Hq)), block=16)
        np.testing.assert_allclose(sq, dq, atol=1e-12)
        np.testing.assert_allclose(sk, dk, atol=1e-12)
        np.testing.assert_allclose(sv, dv, atol=1e-12)
        np.testing.assert_allclose(ss, ds, atol=1e-12)


@pytest.mark.parametrize("window", [0, 3])
def test_zero_queries_closed_forms(window):
    """q = 0: every visible score is 0, so P_ij = 1 / (n_i + e^sigma) with n_i the keys row
    i sees.  Then O_i = v_scale * mean-like sum, and in closed form
      dv_j     = v_scale * sum_{i sees j} dO_i / (n_i + e^sigma)
      dk       = 0                      (dS_ij multiplies q_i = 0)
      dq_i     = s / (n_i + e^sigma) * sum_{j seen} (v_scale <dO_i, v_j> - D_i) k_j
      dsigma_h = -sum_i e^sigma / (n_i + e^sigma) * <dO_i, O_i>."""
    rng = np.random.default_rng(60 + window)
    n, Hq, Hkv, Dqk, Dv = 7, 2, 1, 4, 3
    q = np.zeros((n, Hq, Dqk))
    k = rng.standard_normal((n, Hkv, Dqk))
    v = rng.standard_normal((n, Hkv, Dv))
    s = np.array([0.4, -1.1])
    dO = rng.standard_normal((n, Hq, Dv))
    vs = 0.8
    dq, dk, dv, ds = prefill_backward(q, k, v, dO, s, window, np.array([0, n]), scale=0.5, v_scale=vs)
    np.testing.assert_array_equal(dk, 0.0)
    want_dv = np.zeros((n, Hkv, Dv))
    want_dq = np.zeros((n, Hq, Dqk))
    want_ds = np.zeros(Hq)
    for h in range(Hq):
        for i in range(n):
            seen = [j for j in range(n) if 0 <= i - j and (window == 0 or i - j <= window - 1)]
            Z = len(seen) + np.exp(s[h])
            O_i = vs * sum(v[j, 0] for j in seen) / Z
            D_i = float(dO[i, h] @ O_i)
            for j in seen:
                want_dv[j, 0] += vs * dO[i, h] / Z
                # dq_i = s sum_j P_ij (v_scale <dO_i, v_j> - D_i) k_j
                want_dq[i, h] += 0.5 / Z * (vs * float(dO[i, h] @ v[j, 0]) - D_i) * k[j, 0]
            want_ds[h] -= np.exp(s[h]) / Z * D_i
    np.testing.assert_allclose(dv, want_dv, atol=1e-13)
    np.testing.assert_allclose(dq, want_dq, atol=1e-13)
    np.testing.assert_allclose(ds, want_ds, atol=1e-13)
