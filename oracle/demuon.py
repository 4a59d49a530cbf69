"""fp64 reference of one DeMuon iteration (test infrastructure only).

Source: "DeMuon: decentralized Muon over graphs" (technical summary),
"Problem definition" and "Methodology", 1. DeMuon.  N agents on a
communication graph minimise the average of their local objectives.  Each
agent i keeps three sequences:
* a local gradient estimate M_i, an exponentially weighted moving average of
  its stochastic gradients (local momentum);
* a global gradient estimate V_i, updated from the neighbours' values
  (gradient tracking);
* its iterate X_i, updated from the neighbours' updates, each of which applies
  the matrix sign msgn to the tracked gradient.
The page prints no formulas.  The plain gradient-tracking reading, with
mixing weights w_ij (row i = the weights agent i applies to what it
receives), is:

    M_i' = (1 - theta) M_i + theta G_i
    V_i' = sum_j w_ij V_j + M_i' - M_i
    X_i' = sum_j w_ij (X_j - eta msgn(V_j'))

msgn is computed, as in Muon, by the Frobenius-normalised quintic
Newton-Schulz iteration: `gram_ns.orthogonalize`, itself pinned against the
SVD polar factor.  The tracking recursion starts from V_i = M_i.

Topologies named on the page: complete graph, ring and exponential graph.
Their mixing matrices below are the usual doubly stochastic choices:
* complete: w_ij = 1/N;
* ring: 1/3 on the agent itself and its two neighbours (N >= 3; N = 2 is
  the complete graph);
* exponential: agent i receives from itself and from i - 2^k (mod N) for
  2^k < N, with equal weights.
The mixing rate lambda is the second largest singular value of W.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np

from .gram_ns import K_STEPS, QUINTIC, orthogonalize


def mixing_matrix(topology: str, n: int) -> np.ndarray:
    """Doubly stochastic mixing weights of the named topology (float64)."""
    if n < 1:
        raise ValueError("n must be >= 1")
    if topology == "complete" or n == 1 or (topology == "ring" and n == 2):
        return np.full((n, n), 1.0 / n)
    w = np.zeros((n, n))
    if topology == "ring":
        for i in range(n):
            for d in (-1, 0, 1):
                w[i, (i + d) % n] = 1.0 / 3.0
        return w
    if topology == "exponential":
        hops = [0]
        k = 1
        while k < n:
            hops.append(k)
            k *= 2
        for i in range(n):
            for h in hops:
                w[i, (i - h) % n] = 1.0 / len(hops)
        return w
    raise ValueError(f"unknown topology {topology!r}")


def mixing_rate(w: np.ndarray) -> float:
    """lambda: the second largest singular value of W (0 for one agent)."""
    s = np.linalg.svd(np.asarray(w, dtype=np.float64), compute_uv=False)
    return float(s[1]) if len(s) > 1 else 0.0


def msgn(v: np.ndarray, coeffs: Sequence[float] = QUINTIC, steps: int = K_STEPS,
         eps: float = 1e-7) -> np.ndarray:
    """Matrix sign of v by the quintic Newton-Schulz iteration (Muon's msgn)."""
    return orthogonalize(np.asarray(v, dtype=np.float64), coeffs, steps, eps)


def demuon_step(x: List[List[np.ndarray]], m: List[List[np.ndarray]], v: List[List[np.ndarray]],
                g: List[List[np.ndarray]], w: np.ndarray, *, theta: float, eta: float,
                coeffs: Sequence[float] = QUINTIC, steps: int = K_STEPS, eps: float = 1e-7,
                msgn_input: Optional[Callable[[np.ndarray], np.ndarray]] = None
                ) -> Tuple[list, list, list, list]:
    """One DeMuon iteration for N agents, each with the same list of matrices.

    x, m, v, g: [agent][matrix] arrays.  Returns (x', m', v', o) with o the
    msgn of every agent's tracked gradient.  ``msgn_input`` maps V' to the
    value msgn is applied to; the identity by default.  A test passes the
    rounding of a lower-precision input here.
    """
    w = np.asarray(w, dtype=np.float64)
    n = len(x)
    nm = len(x[0])
    m_new = [[(1.0 - theta) * np.asarray(m[i][k], np.float64) + theta * np.asarray(g[i][k], np.float64)
              for k in range(nm)] for i in range(n)]
    v_new = []
    for i in range(n):
        row = []
        for k in range(nm):
            acc = sum(w[i, j] * np.asarray(v[j][k], np.float64) for j in range(n))
            row.append(acc + m_new[i][k] - np.asarray(m[i][k], np.float64))
        v_new.append(row)
    o = [[msgn(msgn_input(v_new[j][k]) if msgn_input else v_new[j][k], coeffs, steps, eps)
          for k in range(nm)] for j in range(n)]
    x_new = [[sum(w[i, j] * (np.asarray(x[j][k], np.float64) - eta * o[j][k]) for j in range(n))
              for k in range(nm)] for i in range(n)]
    return x_new, m_new, v_new, o
