"""Pins of the DeMuon oracle (oracle/demuon.py) against what the page and
the mathematics fix, independent of the oracle's own code:

* mixing matrices: doubly stochastic; the ring's mixing rate equals the
  closed form max_k |1 + 2 cos(2 pi k / N)| / 3 of a symmetric circulant;
  the complete graph mixes in one step (rate 0);
* one agent (W = [1]): the iteration is Muon with an exponential moving
  average momentum.  It must equal the separately pinned `muon_step`,
  with beta = 1 - theta, gradient theta G and lr = eta (rows <= cols, so
  the scale is 1);
* gradient tracking: with V0 = M0 and a doubly stochastic W, the agents'
  mean of V equals their mean of M after every step;
* complete graph: after one step every agent holds the same iterate, the
  mean of X_j - eta msgn(V_j');
* scalars with a non-symmetric W: hand-written recursions with
  msgn(v) = sign(v) q(|v| / (|v| + eps)), q = the quintic map applied 5
  times.  This fixes which index of W is the receiver and the order of the
  three updates.

Each pin is chosen so that a plausible mistake fails it: a swapped W index,
a flipped tracking sign, msgn on the old V, or mixing X without the update.
"""
import numpy as np
import pytest

from oracle import demuon, gram_ns

A, B, C = gram_ns.QUINTIC


@pytest.mark.parametrize("topology", ["complete", "ring", "exponential"])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8])
def test_mixing_matrices_doubly_stochastic(topology, n):
    w = demuon.mixing_matrix(topology, n)
    assert w.shape == (n, n) and (w >= 0).all()
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-15)
    np.testing.assert_allclose(w.sum(axis=0), 1.0, atol=1e-15)


@pytest.mark.parametrize("n", [3, 4, 5, 7, 8, 16])
def test_ring_mixing_rate_closed_form(n):
    rate = demuon.mixing_rate(demuon.mixing_matrix("ring", n))
    closed = max(abs(1 + 2 * np.cos(2 * np.pi * k / n)) / 3 for k in range(1, n))
    assert rate == pytest.approx(closed, abs=1e-12)
    assert demuon.mixing_rate(demuon.mixing_matrix("complete", n)) == pytest.approx(0.0, abs=1e-12)
    assert 0 < demuon.mixing_rate(demuon.mixing_matrix("exponential", n)) < 1


def _rand(rng, shape):
    return rng.standard_normal(shape)


def test_single_agent_is_ema_muon():
    rng = np.random.default_rng(5)
    theta, eta = 0.3, 0.05
    for shape in [(8, 24), (16, 16), (4, 32)]:
        x, m, g = _rand(rng, shape), _rand(rng, shape), _rand(rng, shape)
        xn, mn, vn, o = demuon.demuon_step([[x]], [[m]], [[m]], [[g]], np.ones((1, 1)), theta=theta, eta=eta)
        m_ref, o_ref, x_ref = gram_ns.muon_step(x, m, theta * g, beta=1 - theta, lr=eta)
        np.testing.assert_allclose(mn[0][0], m_ref, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(vn[0][0], m_ref, rtol=1e-13, atol=1e-13)  # V tracks M exactly
        np.testing.assert_allclose(o[0][0], o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(xn[0][0], x_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("topology", ["ring", "exponential"])
def test_tracking_mean_invariant(topology):
    rng = np.random.default_rng(6)
    n, shapes = 5, [(6, 10), (7, 7)]
    w = demuon.mixing_matrix(topology, n)
    x = [[_rand(rng, s) for s in shapes] for _ in range(n)]
    m = [[_rand(rng, s) for s in shapes] for _ in range(n)]
    v = [[t.copy() for t in row] for row in m]
    for _ in range(4):
        g = [[_rand(rng, s) for s in shapes] for _ in range(n)]
        x, m, v, _ = demuon.demuon_step(x, m, v, g, w, theta=0.2, eta=0.01)
        for k in range(len(shapes)):
            mean_v = sum(v[i][k] for i in range(n)) / n
            mean_m = sum(m[i][k] for i in range(n)) / n
            np.testing.assert_allclose(mean_v, mean_m, rtol=0, atol=1e-12)


def test_complete_graph_reaches_consensus_in_one_step():
    rng = np.random.default_rng(7)
    n, shape, eta = 4, (5, 9), 0.1
    w = demuon.mixing_matrix("complete", n)
    x = [[_rand(rng, shape)] for _ in range(n)]
    m = [[_rand(rng, shape)] for _ in range(n)]
    g = [[_rand(rng, shape)] for _ in range(n)]
    xn, _, vn, o = demuon.demuon_step(x, m, m, g, w, theta=0.5, eta=eta)
    target = sum(x[j][0] - eta * o[j][0] for j in range(n)) / n
    for i in range(n):
        np.testing.assert_allclose(xn[i][0], target, rtol=1e-13, atol=1e-13)


def _q(t):
    for _ in range(gram_ns.K_STEPS):
        t = A * t + B * t ** 3 + C * t ** 5
    return t


def test_scalar_recursions_by_hand_with_nonsymmetric_mixing():
    w = np.array([[0.75, 0.25], [0.5, 0.5]])  # row i: weights agent i applies
    theta, eta, eps = 0.4, 0.2, 1e-7
    x = [1.5, -2.0]
    m = [0.3, -0.1]
    v = [0.2, 0.6]
    g = [1.0, -3.0]
    m1 = [(1 - theta) * m[i] + theta * g[i] for i in range(2)]
    v1 = [w[i, 0] * v[0] + w[i, 1] * v[1] + m1[i] - m[i] for i in range(2)]
    s = [np.sign(t) * _q(abs(t) / (abs(t) + eps)) for t in v1]
    x1 = [w[i, 0] * (x[0] - eta * s[0]) + w[i, 1] * (x[1] - eta * s[1]) for i in range(2)]
    xs, ms, vs, os_ = demuon.demuon_step([[np.array([[x[i]]])] for i in range(2)],
                                         [[np.array([[m[i]]])] for i in range(2)],
                                         [[np.array([[v[i]]])] for i in range(2)],
                                         [[np.array([[g[i]]])] for i in range(2)], w, theta=theta, eta=eta)
    for i in range(2):
        assert ms[i][0][0, 0] == pytest.approx(m1[i], abs=1e-15)
        assert vs[i][0][0, 0] == pytest.approx(v1[i], abs=1e-15)
        assert os_[i][0][0, 0] == pytest.approx(s[i], abs=1e-13)
        assert xs[i][0][0, 0] == pytest.approx(x1[i], abs=1e-13)


def test_unknown_topology_rejected():
    with pytest.raises(ValueError):
        demuon.mixing_matrix("torus", 4)


# ---------------------------------------------------------------- mutants
# Each mutant is the DeMuon iteration with one plausible mistake planted
# (on the CPU, in a copy of the recursions written here). Each must fail at
# least one of the pins above, or the pins would not protect the oracle.

def _step(x, m, v, g, w, theta, eta, bug=None):
    n, nm = len(x), len(x[0])
    wt = w.T if bug == "swapped W index" else w
    m1 = [[(1 - theta) * m[i][k] + theta * g[i][k] for k in range(nm)] for i in range(n)]
    sgn = -1.0 if bug == "flipped tracking sign" else 1.0
    v1 = [[sum(wt[i, j] * v[j][k] for j in range(n)) + sgn * (m1[i][k] - m[i][k]) for k in range(nm)]
          for i in range(n)]
    src = v if bug == "msgn of the old V" else v1
    o = [[demuon.msgn(src[j][k]) for k in range(nm)] for j in range(n)]
    if bug == "update not mixed":
        x1 = [[sum(wt[i, j] * x[j][k] for j in range(n)) - eta * o[i][k] for k in range(nm)] for i in range(n)]
    else:
        x1 = [[sum(wt[i, j] * (x[j][k] - eta * o[j][k]) for j in range(n)) for k in range(nm)] for i in range(n)]
    return x1, m1, v1, o


def _pins_hold(step):
    rng = np.random.default_rng(11)
    # single agent vs muon_step
    x, m, g = rng.standard_normal((6, 12)), rng.standard_normal((6, 12)), rng.standard_normal((6, 12))
    xn, mn, vn, o = step([[x]], [[m]], [[m]], [[g]], np.ones((1, 1)), 0.3, 0.05)
    m_ref, o_ref, x_ref = gram_ns.muon_step(x, m, 0.3 * g, beta=0.7, lr=0.05)
    if not (np.allclose(vn[0][0], m_ref, atol=1e-12) and np.allclose(xn[0][0], x_ref, atol=1e-12)):
        return False
    # tracking invariant
    n = 4
    w = demuon.mixing_matrix("exponential", n)
    xs = [[rng.standard_normal((5, 7))] for _ in range(n)]
    ms = [[rng.standard_normal((5, 7))] for _ in range(n)]
    vs = [[t.copy() for t in row] for row in ms]
    for _ in range(2):
        gs = [[rng.standard_normal((5, 7))] for _ in range(n)]
        xs, ms, vs, _ = step(xs, ms, vs, gs, w, 0.2, 0.01)
        if not np.allclose(sum(r[0] for r in vs) / n, sum(r[0] for r in ms) / n, atol=1e-12):
            return False
    # complete-graph consensus
    w = demuon.mixing_matrix("complete", n)
    xs = [[rng.standard_normal((5, 9))] for _ in range(n)]
    ms = [[rng.standard_normal((5, 9))] for _ in range(n)]
    gs = [[rng.standard_normal((5, 9))] for _ in range(n)]
    xn, _, _, _ = step(xs, ms, ms, gs, w, 0.5, 0.1)
    if not all(np.allclose(xn[i][0], xn[0][0], atol=1e-13) for i in range(n)):
        return False
    # scalars with a non-symmetric W, by hand
    w = np.array([[0.75, 0.25], [0.5, 0.5]])
    x, m, v, g = [1.5, -2.0], [0.3, -0.1], [0.2, 0.6], [1.0, -3.0]
    m1 = [0.6 * m[i] + 0.4 * g[i] for i in range(2)]
    v1 = [w[i, 0] * v[0] + w[i, 1] * v[1] + m1[i] - m[i] for i in range(2)]
    s = [np.sign(t) * _q(abs(t) / (abs(t) + 1e-7)) for t in v1]
    x1 = [w[i, 0] * (x[0] - 0.2 * s[0]) + w[i, 1] * (x[1] - 0.2 * s[1]) for i in range(2)]
    xs, _, _, _ = step([[np.array([[x[i]]])] for i in range(2)], [[np.array([[m[i]]])] for i in range(2)],
                       [[np.array([[v[i]]])] for i in range(2)], [[np.array([[g[i]]])] for i in range(2)],
                       w, 0.4, 0.2)
    return all(abs(xs[i][0][0, 0] - x1[i]) < 1e-12 for i in range(2))


def test_pins_accept_the_oracle_and_reject_every_mutant():
    oracle_step = lambda x, m, v, g, w, th, et: demuon.demuon_step(x, m, v, g, w, theta=th, eta=et)  # noqa: E731
    assert _pins_hold(oracle_step)
    assert _pins_hold(lambda *a: _step(*a))  # the unmutated copy passes too
    for bug in ["swapped W index", "flipped tracking sign", "msgn of the old V", "update not mixed"]:
        assert not _pins_hold(lambda *a, b=bug: _step(*a, bug=b)), bug


@pytest.mark.parametrize("n", [3, 5, 8, 13, 16])
def test_exponential_mixing_rate_closed_form(n):
    """The exponential graph's W is circulant with equal weights on the
    offsets {0} and {2^k < n}; its eigenvalues are the averages of the
    matching roots of unity, and W is normal, so its singular values are
    their moduli."""
    hops = [0] + [1 << k for k in range(n.bit_length()) if (1 << k) < n]
    eig = [abs(sum(np.exp(-2j * np.pi * h * k / n) for h in hops)) / len(hops) for k in range(1, n)]
    assert demuon.mixing_rate(demuon.mixing_matrix("exponential", n)) == pytest.approx(max(eig), abs=1e-12)
