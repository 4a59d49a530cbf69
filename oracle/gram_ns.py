"""fp64 reference implementation of the Muon update (test infrastructure only).

Sources, by page title and section (the pages are technical summaries of
the papers; they print no code, no coefficients and no worked example):

* "DMuon: Efficient Distributed Muon Training with Near-Adam Overhead"
  (technical summary), section 1 "Problem definition": Muon applies a
  Newton-Schulz (NS) iteration to the momentum-accumulated gradient of each
  weight matrix; the iteration needs the full matrix product X X^T.
  Section 2.2 "Efficient Gram Newton-Schulz iteration": the recursion can be
  run in the m x m Gram space G = X X^T instead of the m x n space.
  Section 5: DMuon changes neither the update rule nor its convergence.
* "DeMuon: decentralized Muon over graphs" (technical summary), Method 1,
  "matrix orthogonalisation": the update applies the matrix sign msgn(.)
  to the tracked gradient; NS is the polynomial approximation of msgn.
* "Dion3: Full-Stack Orthogonal Updates" (review), section 1 "Key terms":
  Gram Newton-Schulz reformulates NS to iterate on the small Gram matrix.

Readings where the pages are silent (each one is listed with its reason in
the design notes):

* quintic coefficients (a, b, c) = (3.4445, -4.7750, 2.0315), K = 5 steps;
* momentum M <- beta * M + G (plain heavy-ball accumulation, no (1-beta)
  factor, no Nesterov term);
* normalisation X0 = X / (||X||_F + eps);
* a matrix with rows > cols is transposed before the iteration, so the
  iterated matrix is m x n with m = min(rows, cols) <= n;
* update W <- W - lr * sqrt(max(1, rows / cols)) * O with rows, cols of W
  as stored (out_features, in_features).

The rectangular iteration is the definition the oracle follows; the Gram
form is kept beside it only so the tests can pin the two against each
other, which is the equivalence the DMuon page's section 2.2 relies on.
"""

from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

QUINTIC: Tuple[float, float, float] = (3.4445, -4.7750, 2.0315)
K_STEPS: int = 5


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact conversion of bfloat16 bit patterns (uint16) to float64.

    A bfloat16 value is the upper half of an IEEE float32, so shifting the
    16 bits into the high half of a uint32 and reinterpreting gives the
    float32 value exactly; float32 -> float64 is exact too.
    """
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def momentum(m_prev: np.ndarray, g: np.ndarray, beta: float) -> np.ndarray:
    """Momentum accumulation M <- beta * M_prev + G, in float64.

    DMuon page, section 1: NS acts on the momentum-accumulated gradient.
    DeMuon page, Method 1 ("local momentum") keeps a running estimate per
    node; the accumulation form used here is the plain heavy-ball one.
    """
    return float(beta) * np.asarray(m_prev, dtype=np.float64) + np.asarray(g, dtype=np.float64)


def frobenius_normalize(x: np.ndarray, eps: float) -> np.ndarray:
    """X0 = X / (||X||_F + eps), which puts every singular value in [0, 1]."""
    x = np.asarray(x, dtype=np.float64)
    return x / (math.sqrt(float(np.sum(x * x))) + float(eps))


def ns_rectangular(x0: np.ndarray, coeffs: Sequence[float] = QUINTIC,
                   steps: int = K_STEPS) -> np.ndarray:
    """Rectangular Newton-Schulz: X <- a X + (b A + c A^2) X, A = X X^T.

    ``x0`` is m x n with m <= n, already normalised.  Each step applies the
    odd polynomial f(s) = a s + b s^3 + c s^5 to every singular value of X
    (DeMuon page, Method 1: the target is msgn(X) = U V^T).
    """
    a, b, c = (float(v) for v in coeffs)
    x = np.array(x0, dtype=np.float64, copy=True)
    for _ in range(int(steps)):
        amat = x @ x.T
        poly = b * amat + c * (amat @ amat)
        x = a * x + poly @ x
    return x


def ns_gram(x0: np.ndarray, coeffs: Sequence[float] = QUINTIC,
            steps: int = K_STEPS) -> np.ndarray:
    """Gram-space form of the same iteration (DMuon page, section 2.2).

    G0 = X0 X0^T, P0 = I; each step forms Q = a I + b G + c G^2, then
    G <- Q G Q and P <- Q P; the result is P X0.  Since every Q_k is a
    polynomial in G_k and X_{k+1} = Q_k X_k, this equals the rectangular
    iterate exactly in exact arithmetic.
    """
    a, b, c = (float(v) for v in coeffs)
    x0 = np.asarray(x0, dtype=np.float64)
    m = x0.shape[0]
    eye = np.eye(m)
    g = x0 @ x0.T
    p = eye.copy()
    for _ in range(int(steps)):
        q = a * eye + b * g + c * (g @ g)
        g = q @ g @ q
        p = q @ p
    return p @ x0


def gram_trace(x0: np.ndarray, coeffs: Sequence[float] = QUINTIC,
               steps: int = K_STEPS) -> List[dict]:
    """Gram-space intermediates per step, for checking stages in isolation.

    Returns one dict per step k with G_k (before the step), R_k = Q_k - aI,
    P_{k+1} = Q_k P_k and T_k = Q_k G_k.
    """
    a, b, c = (float(v) for v in coeffs)
    x0 = np.asarray(x0, dtype=np.float64)
    m = x0.shape[0]
    eye = np.eye(m)
    g = x0 @ x0.T
    p = eye.copy()
    out = []
    for _ in range(int(steps)):
        r = b * g + c * (g @ g)
        q = a * eye + r
        t = q @ g
        p = q @ p
        out.append({"G": g.copy(), "R": r, "T": t, "P": p.copy()})
        g = t @ q
    return out


def orthogonalize(m: np.ndarray, coeffs: Sequence[float] = QUINTIC,
                  steps: int = K_STEPS, eps: float = 1e-7) -> np.ndarray:
    """O = NS(M) in M's own orientation (rows x cols).

    A tall matrix (rows > cols) is transposed so that the iterated matrix
    has m = min(rows, cols) rows; the output is transposed back.  A square
    matrix is not transposed.
    """
    m = np.asarray(m, dtype=np.float64)
    tall = m.shape[0] > m.shape[1]
    x = m.T if tall else m
    o = ns_rectangular(frobenius_normalize(x, eps), coeffs, steps)
    return o.T if tall else o


def update_scale(rows: int, cols: int) -> float:
    """sqrt(max(1, rows / cols)) on W's stored shape (out, in)."""
    return math.sqrt(max(1.0, float(rows) / float(cols)))


def muon_step(w: np.ndarray, m_prev: np.ndarray, g: np.ndarray, *, beta: float,
              lr: float, eps: float = 1e-7, coeffs: Sequence[float] = QUINTIC,
              steps: int = K_STEPS) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One Muon step for one matrix: returns (M_new, O, W_new), all float64.

    M_new = beta M_prev + G; O = NS(M_new / (||M_new||_F + eps));
    W_new = W - lr * sqrt(max(1, rows/cols)) * O.
    """
    m_new = momentum(m_prev, g, beta)
    o = orthogonalize(m_new, coeffs, steps, eps)
    rows, cols = m_new.shape
    w_new = np.asarray(w, dtype=np.float64) - float(lr) * update_scale(rows, cols) * o
    return m_new, o, w_new
