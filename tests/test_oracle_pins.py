"""Pins for the fp64 oracle: facts fixed by the mathematics, not by the oracle.

Each pin is independent of the oracle's own arithmetic:

* polar factor: a matrix built as U diag(s) V^T from QR-orthogonalised
  random factors (so U V^T is known by construction) must come back as
  U V^T under the cubic iteration (1.5, -0.5) run to convergence;
* spectral closed form: NS acts on singular values one by one, so the
  output equals U f^K(S / ||X||_F) V^T from numpy's SVD (LAPACK), with f
  the scalar polynomial;
* exact rational special cases (row vector, diagonal matrix) against
  ``tests/golden/quintic_exact.json`` (written with Python fractions);
* Gram form == rectangular form (DMuon page, section 2.2), and every
  intermediate of the Gram trace (G_k, R_k, T_k, P_k) against products of
  the rectangular iterates X_k, X_{k+1};
* invariances: transpose, positive scale, orthogonal conjugation;
* the singular-value band of five quintic steps;
* closed-form values of the momentum and of the update scale.

``test_pins_catch_planted_mistakes`` plants plausible mistakes in copies of
the oracle (a dropped term, a flipped sign, swapped coefficients, a missing
step, a transposed iterate, a missing normalisation) and checks that a pin
fails for every one of them; ``test_gram_pin_catches_planted_mistakes`` does
the same for the Gram-space form (a one-sided G update, an unaccumulated P).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import gram_ns

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = json.load(open(os.path.join(HERE, "golden", "quintic_exact.json")))
A, B, C = oracle.QUINTIC


def _orth(n, rng):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def _scalar_iter(x, coeffs, steps):
    a, b, c = coeffs
    x = np.array(x, dtype=np.float64)
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def _rel(x, y):
    return float(np.linalg.norm(x - y) / np.linalg.norm(y))


SHAPES = [(4, 7), (6, 6), (9, 3), (1, 5), (5, 1), (16, 40), (40, 16)]


@pytest.mark.parametrize("shape", SHAPES)
def test_polar_factor_cubic(shape):
    rows, cols = shape
    k = min(rows, cols)
    rng = np.random.default_rng(rows * 100 + cols)
    u = _orth(rows, rng)[:, :k]
    v = _orth(cols, rng)[:, :k]
    s = rng.uniform(0.3, 1.0, size=k)
    x = (u * s) @ v.T
    out = oracle.orthogonalize(x, coeffs=(1.5, -0.5, 0.0), steps=60, eps=0.0)
    assert np.max(np.abs(out - u @ v.T)) < 1e-12


@pytest.mark.parametrize("shape", SHAPES + [(64, 256), (96, 33)])
@pytest.mark.parametrize("steps", [1, 5])
def test_spectral_closed_form(shape, steps):
    rng = np.random.default_rng(7 + shape[0] + 13 * shape[1])
    x = rng.standard_normal(shape)
    u, s, vt = np.linalg.svd(x, full_matrices=False)
    fs = _scalar_iter(s / np.linalg.norm(x), oracle.QUINTIC, steps)
    expect = (u * fs) @ vt
    out = oracle.orthogonalize(x, steps=steps, eps=0.0)
    assert _rel(out, expect) < 1e-11


def test_row_vector_exact():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 33))
    out = oracle.orthogonalize(x, eps=0.0)
    f5_1 = float(GOLD["quintic"]["1"][4])
    assert np.allclose(out, f5_1 * x / np.linalg.norm(x), rtol=1e-13, atol=0)
    # tall column vector: the same after the transpose
    out_t = oracle.orthogonalize(x.T, eps=0.0)
    assert np.allclose(out_t, f5_1 * x.T / np.linalg.norm(x), rtol=1e-13, atol=0)


def test_diagonal_exact_rational():
    # diag(3, 4) / 5 has Frobenius norm 1 and singular values 3/5, 4/5.
    x = np.zeros((2, 5))
    x[0, 0], x[1, 1] = 0.6, 0.8
    for steps in range(1, 6):
        out = oracle.orthogonalize(x, steps=steps, eps=0.0)
        assert out[0, 0] == pytest.approx(float(GOLD["quintic"]["3/5"][steps - 1]), rel=1e-14)
        assert out[1, 1] == pytest.approx(float(GOLD["quintic"]["4/5"][steps - 1]), rel=1e-14)
        out[0, 0] = out[1, 1] = 0.0
        assert np.max(np.abs(out)) < 1e-15


def test_golden_file_matches_fractions():
    a, b, c = (Fraction(s) for s in GOLD["coeffs"])
    assert (float(a), float(b), float(c)) == oracle.QUINTIC
    y = Fraction(1)
    for k in range(5):
        y = a * y + b * y ** 3 + c * y ** 5
        assert float(y) == float(GOLD["quintic"]["1"][k])


@pytest.mark.parametrize("shape", [(8, 8), (12, 30), (30, 12), (64, 256)])
def test_gram_equals_rectangular(shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    x = rng.standard_normal(shape)
    x0 = oracle.frobenius_normalize(x.T if shape[0] > shape[1] else x, 0.0)
    rect = oracle.ns_rectangular(x0)
    gram = oracle.ns_gram(x0)
    assert _rel(gram, rect) < 1e-12


def test_gram_trace_consistent_and_symmetric():
    rng = np.random.default_rng(11)
    x0 = oracle.frobenius_normalize(rng.standard_normal((10, 23)), 0.0)
    tr = oracle.gram_trace(x0)
    assert len(tr) == 5
    for st in tr:
        for key in ("G", "R", "T", "P"):
            mat = st[key]
            assert np.max(np.abs(mat - mat.T)) <= 1e-13 * max(1.0, np.max(np.abs(mat)))
    assert _rel(tr[-1]["P"] @ x0, oracle.ns_rectangular(x0)) < 1e-12
    np.testing.assert_allclose(tr[0]["G"], x0 @ x0.T, rtol=0, atol=1e-15)


@pytest.mark.parametrize("shape", [(7, 19), (19, 7), (12, 12)])
def test_transpose_invariance(shape):
    x = np.random.default_rng(5).standard_normal(shape)
    assert _rel(oracle.orthogonalize(x.T, eps=0.0), oracle.orthogonalize(x, eps=0.0).T) < 1e-13


@pytest.mark.parametrize("scale", [1e-6, 3.7, 1e5])
def test_scale_invariance(scale):
    x = np.random.default_rng(6).standard_normal((9, 14))
    assert _rel(oracle.orthogonalize(scale * x, eps=0.0), oracle.orthogonalize(x, eps=0.0)) < 1e-12


def test_orthogonal_invariance():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((11, 17))
    u, v = _orth(11, rng), _orth(17, rng)
    lhs = oracle.orthogonalize(u @ x @ v, eps=0.0)
    rhs = u @ oracle.orthogonalize(x, eps=0.0) @ v
    assert _rel(lhs, rhs) < 1e-12


def test_singular_value_band():
    # f^5 maps [1.5e-3, 1] into [0.6798, 1.2024] (scalar analysis of the quintic).
    rng = np.random.default_rng(9)
    rows, cols = 24, 60
    u = _orth(rows, rng)
    v = _orth(cols, rng)[:, :rows]
    s = np.geomspace(0.0016, 1.0, rows)
    x = (u * s) @ v.T
    x = x / np.linalg.norm(x)
    s_in = np.linalg.svd(x, compute_uv=False)
    s_out = np.linalg.svd(oracle.orthogonalize(x, eps=0.0), compute_uv=False)
    mask = s_in >= 1.5e-3
    assert mask.sum() >= rows - 2
    assert s_out[mask].min() >= 0.6798 and s_out[mask].max() <= 1.20237


def test_momentum_closed_forms():
    g = np.arange(6, dtype=np.float64).reshape(2, 3) - 2.5
    z = np.zeros_like(g)
    np.testing.assert_array_equal(oracle.momentum(z, g, 0.95), g)
    np.testing.assert_array_equal(oracle.momentum(g, g, 1.0), 2 * g)
    np.testing.assert_allclose(oracle.momentum(g, g, 0.5), 1.5 * g, rtol=0, atol=0)


def test_update_scale_and_step():
    assert oracle.update_scale(8, 2) == 2.0
    assert oracle.update_scale(2, 8) == 1.0
    assert oracle.update_scale(3584, 3584) == 1.0
    assert oracle.update_scale(18944, 3584) == pytest.approx(math.sqrt(18944 / 3584), rel=1e-15)
    # row vector: O = f^5(1) x / ||x||; tall 8x2 gets the factor 2.
    rng = np.random.default_rng(1)
    g = rng.standard_normal((8, 2))
    w = rng.standard_normal((8, 2))
    m_new, o, w_new = oracle.muon_step(w, np.zeros_like(g), g, beta=0.9, lr=0.1, eps=0.0)
    np.testing.assert_array_equal(m_new, g)
    u, s, vt = np.linalg.svd(g, full_matrices=False)
    expect_o = (u * _scalar_iter(s / np.linalg.norm(g), oracle.QUINTIC, 5)) @ vt
    assert _rel(o, expect_o) < 1e-12
    assert _rel(w - w_new, 0.2 * expect_o) < 1e-12


def test_bf16_bits_conversion():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F, 0x0001], dtype=np.uint16)
    vals = oracle.bf16_bits_to_f64(bits)
    assert vals[0] == 1.0 and vals[1] == -1.0
    assert vals[2] == 3.140625
    assert vals[3] == 0.0 and math.copysign(1.0, vals[4]) == -1.0
    assert vals[5] == float(np.float32(3.3895313892515355e38))
    assert vals[6] == 2.0 ** -133


# ---------------------------------------------------------------- mutations
def _pins_pass(mod):
    """Run the spectral, polar and special-case pins against a module-like
    object that provides ``orthogonalize`` with the oracle's signature.
    Diverging mutants overflow; that is their expected failure, not a warning."""
    with np.errstate(over="ignore", invalid="ignore"):
        return _pins_pass_inner(mod)


def _pins_pass_inner(mod):
    try:
        rng = np.random.default_rng(42)
        for shape in [(5, 9), (9, 5), (6, 6)]:
            x = rng.standard_normal(shape)
            u, s, vt = np.linalg.svd(x, full_matrices=False)
            expect = (u * _scalar_iter(s / np.linalg.norm(x), oracle.QUINTIC, 5)) @ vt
            if not _rel(mod.orthogonalize(x, eps=0.0), expect) <= 1e-11:
                return False
        x = np.zeros((2, 5))
        x[0, 0], x[1, 1] = 0.6, 0.8
        out = mod.orthogonalize(x, eps=0.0)
        if not abs(out[0, 0] - float(GOLD["quintic"]["3/5"][4])) <= 1e-13:
            return False
        return True
    except Exception:
        return False


class _Mutant:
    def __init__(self, rect):
        self._rect = rect

    def orthogonalize(self, m, coeffs=oracle.QUINTIC, steps=5, eps=1e-7, transpose=True,
                      normalize=True):
        m = np.asarray(m, dtype=np.float64)
        tall = m.shape[0] > m.shape[1] and transpose
        x = m.T if tall else m
        if normalize:
            x = gram_ns.frobenius_normalize(x, eps)
        o = self._rect(x, coeffs, steps)
        return o.T if tall else o


def _rect_dropped_square(x0, coeffs, steps):
    a, b, c = coeffs
    x = x0.copy()
    for _ in range(steps):
        am = x @ x.T
        x = a * x + (b * am + c * am) @ x
    return x


def _rect_flipped_sign(x0, coeffs, steps):
    a, b, c = coeffs
    x = x0.copy()
    for _ in range(steps):
        am = x @ x.T
        x = a * x - (b * am + c * am @ am) @ x
    return x


def _rect_transposed_iterate(x0, coeffs, steps):
    # the update multiplies the transposed iterate: (b A + c A^2) X^T
    a, b, c = coeffs
    x = x0.copy()
    for _ in range(steps):
        am = x @ x.T
        x = a * x + (b * am + c * am @ am) @ x.T
    return x


def _rect_right_gram(x0, coeffs, steps):
    # X (b X^T X + c (X^T X)^2) equals (b X X^T + c (X X^T)^2) X: a correct
    # alternative that the pins must accept.
    a, b, c = coeffs
    x = x0.copy()
    for _ in range(steps):
        am = x.T @ x
        x = a * x + x @ (b * am + c * am @ am)
    return x


def _rect_swapped_coeffs(x0, coeffs, steps):
    a, b, c = coeffs
    return gram_ns.ns_rectangular(x0, (a, c, b), steps)


def _rect_one_step_short(x0, coeffs, steps):
    return gram_ns.ns_rectangular(x0, coeffs, steps - 1)


def test_pins_catch_planted_mistakes():
    assert _pins_pass(oracle)
    mutants = {
        "dropped square": _Mutant(_rect_dropped_square),
        "flipped sign": _Mutant(_rect_flipped_sign),
        "swapped coefficients": _Mutant(_rect_swapped_coeffs),
        "one step short": _Mutant(_rect_one_step_short),
        "transposed iterate": _Mutant(_rect_transposed_iterate),
    }
    for name, mut in mutants.items():
        assert not _pins_pass(mut), name

    class NoNorm(_Mutant):
        def orthogonalize(self, m, **kw):
            return super().orthogonalize(m, normalize=False, **kw)

    assert not _pins_pass(NoNorm(gram_ns.ns_rectangular)), "missing normalisation"

    # Not a mistake: the Gram matrix on the other side is equivalent.
    assert _pins_pass(_Mutant(_rect_right_gram))


# Mistakes planted in the Gram-space form: the Gram == rectangular pin, with
# the rectangular form pinned to the SVD above, must reject every one.
def _gram_pin_passes(gram_fn):
    for shape in [(8, 8), (12, 30)]:
        rng = np.random.default_rng(shape[0] * 7 + shape[1])
        x0 = oracle.frobenius_normalize(rng.standard_normal(shape), 0.0)
        try:
            with np.errstate(over="ignore", invalid="ignore"):
                ok = _rel(gram_fn(x0), oracle.ns_rectangular(x0)) < 1e-12
            if not ok:
                return False
        except ValueError:
            return False
    return True


def _gram_variant(one_sided=False, p_not_accumulated=False, right_gram=False, p_right=False):
    def fn(x0, coeffs=oracle.QUINTIC, steps=5):
        a, b, c = coeffs
        g = x0.T @ x0 if right_gram else x0 @ x0.T
        eye = np.eye(g.shape[0])
        p = eye.copy()
        for _ in range(steps):
            q = a * eye + b * g + c * (g @ g)
            g = q @ g if one_sided else q @ g @ q
            p = q if p_not_accumulated else (p @ q if p_right else q @ p)
        return x0 @ p if right_gram else p @ x0
    return fn


def test_gram_pin_catches_planted_mistakes():
    assert _gram_pin_passes(oracle.ns_gram)
    assert not _gram_pin_passes(_gram_variant(one_sided=True)), "G <- Q G"
    assert not _gram_pin_passes(_gram_variant(p_not_accumulated=True)), "P <- Q"
    # Not mistakes: every Q_k is a polynomial in G_0, so P Q == Q P, and the
    # right-side Gram X0^T X0 with O = X0 P gives the same iterate.
    assert _gram_pin_passes(_gram_variant(p_right=True))
    assert _gram_pin_passes(_gram_variant(right_gram=True))


# Every intermediate of the Gram trace (which the GPU stage checks compare
# against) is fixed by the rectangular iterates X_k, themselves pinned to
# the SVD: G_k = X_k X_k^T, T_k = Q_k G_k = X_{k+1} X_k^T,
# R_k X_k = X_{k+1} - a X_k and P_{k+1} X_0 = X_{k+1}.
def _trace_pinned(trace, x0, a=A):
    xs = [oracle.ns_rectangular(x0, steps=k) for k in range(len(trace) + 1)]
    for k, st in enumerate(trace):
        checks = [
            (st["G"], xs[k] @ xs[k].T),
            (st["T"], xs[k + 1] @ xs[k].T),
            (st["R"] @ xs[k], xs[k + 1] - a * xs[k]),
            (st["P"] @ x0, xs[k + 1]),
        ]
        for got, want in checks:
            if not _rel(got, want) < 1e-11:
                return False
    return True


@pytest.mark.parametrize("shape", [(10, 23), (16, 16), (1, 9)])
def test_gram_trace_matches_rectangular_iterates(shape):
    rng = np.random.default_rng(sum(shape))
    x0 = oracle.frobenius_normalize(rng.standard_normal(shape), 0.0)
    trace = oracle.gram_trace(x0)
    assert _trace_pinned(trace, x0)
    # a T that drops its a G term, or a G advanced one-sidedly, is rejected
    bad_t = [dict(st, T=st["R"] @ st["G"]) for st in trace]
    assert not _trace_pinned(bad_t, x0)
    bad_g = [dict(st) for st in trace]
    for k in range(1, len(bad_g)):
        q = A * np.eye(shape[0]) + bad_g[k - 1]["R"]
        bad_g[k]["G"] = q @ trace[k - 1]["G"]
    assert not _trace_pinned(bad_g, x0)
