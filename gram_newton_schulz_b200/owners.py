"""Owner assignment and cross-rank helpers for the multi-GPU step.

DMuon page, section 2.1 (owner-centric execution): every weight matrix has
exactly one owner rank, which keeps its optimizer state and runs its update
once.  Section 2.3 (computation-aware load balancing): owners are chosen to
minimise the predicted makespan -- by an MILP, with a greedy heuristic as
the fallback for large search spaces.  This module implements the greedy
fallback: longest-processing-time-first (LPT) list scheduling on a per-matrix
cost, which is within 4/3 of the optimal makespan.

The cost of a matrix is the step's algorithmic flop count (Gram SYRK, the
symmetric products of K steps and the final product) unless measured costs
are supplied.  Host logic only: no device work happens here.
"""
from __future__ import annotations

import heapq
from typing import Dict, List, Optional, Sequence, Tuple


def matrix_cost(rows: int, cols: int, steps: int = 5) -> float:
    """Algorithmic flops of one update of a rows x cols matrix:
    m^2 n (SYRK) + (4K - 3) m^3 (symmetric products) + 2 m^2 n (final)."""
    m, n = min(rows, cols), max(rows, cols)
    return 3.0 * m * m * n + (4 * steps - 3) * float(m) ** 3


def lpt_assign(costs: Sequence[float], n_ranks: int) -> List[int]:
    """Owner rank of every matrix by LPT: heaviest first, each to the rank
    with the least load so far (ties: lowest rank, then lowest index, so
    every rank computes the same answer)."""
    if n_ranks <= 0:
        raise ValueError("n_ranks must be positive")
    order = sorted(range(len(costs)), key=lambda i: (-float(costs[i]), i))
    heap: List[Tuple[float, int]] = [(0.0, r) for r in range(n_ranks)]
    owner = [0] * len(costs)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + float(costs[i]), r))
    return owner


def makespan(costs: Sequence[float], owner: Sequence[int], n_ranks: int) -> float:
    loads = [0.0] * n_ranks
    for c, r in zip(costs, owner):
        loads[r] += float(c)
    return max(loads)


def owned_indices(owner: Sequence[int], rank: int) -> List[int]:
    return [i for i, r in enumerate(owner) if r == rank]


def assign_shapes(shapes: Sequence[Tuple[int, int]], n_ranks: int, steps: int = 5,
                  measured: Optional[Dict[Tuple[int, int], float]] = None) -> List[int]:
    """Owners for a list of (rows, cols); ``measured`` maps a shape to its
    measured per-matrix cost and overrides the flop model for that shape."""
    costs = []
    for r, c in shapes:
        key = (int(r), int(c))
        costs.append(measured[key] if measured and key in measured else matrix_cost(r, c, steps))
    return lpt_assign(costs, n_ranks)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a scalar over all ranks of the default process group (the
    value itself when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
