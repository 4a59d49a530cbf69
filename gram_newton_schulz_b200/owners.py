"""Owner assignment and cross-rank helpers for the multi-GPU step.

DMuon page, section 2.1 (owner-centric execution): every weight matrix has
exactly one owner rank, which keeps its optimizer state and runs its update
once.  Section 2.3 (computation-aware load balancing): owners are chosen to
minimise the predicted makespan -- by an MILP, with a greedy heuristic as
the fallback for large search spaces.  This module implements both: the
greedy fallback, longest-processing-time-first (LPT) list scheduling on a
per-matrix cost (within 4/3 of the optimal makespan), and `milp_assign`,
an exact mixed-integer program over per-cost counts.

The cost of a matrix is the step's algorithmic flop count (Gram SYRK, the
symmetric products of K steps and the final product).  `measure_costs`
returns measured per-shape costs instead, timed through the library on the
GPU; they override the flop model.  Everything else here is host logic.
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


def milp_assign(costs: Sequence[float], n_ranks: int, time_limit: float = 5.0,
                max_vars: int = 4000) -> List[int]:
    """Owners that minimise the makespan, by a mixed-integer program (DMuon
    page, section 2.3), with LPT as the fallback for large search spaces.

    Matrices of equal cost are interchangeable, so the program has one
    integer count y[s, r] per distinct cost s and rank r:

        minimise T  subject to  sum_r y[s, r] = n_s  for every s,
                                sum_s c_s y[s, r] <= T  for every rank r,

    solved by scipy's HiGHS interface within ``time_limit`` seconds.  The
    counts are then dealt to the matrices of each cost in index order.  The
    program's answer is kept only when its makespan is not worse than
    LPT's.  With more than ``max_vars`` variables, or without a solution in
    time, the result is LPT's."""
    import numpy as np
    from scipy.optimize import Bounds, LinearConstraint, milp

    lpt = lpt_assign(costs, n_ranks)
    if n_ranks == 1 or not costs:
        return lpt
    groups: Dict[float, List[int]] = {}
    for i, c in enumerate(costs):
        groups.setdefault(float(c), []).append(i)
    keys = sorted(groups, reverse=True)
    n_s, n_r = len(keys), n_ranks
    nv = n_s * n_r + 1
    if nv > max_vars:
        return lpt
    obj = np.zeros(nv)
    obj[-1] = 1.0
    a_eq = np.zeros((n_s, nv))
    counts = np.array([len(groups[k]) for k in keys], dtype=float)
    for si in range(n_s):
        a_eq[si, si * n_r:(si + 1) * n_r] = 1.0
    a_ub = np.zeros((n_r, nv))
    for r in range(n_r):
        for si, k in enumerate(keys):
            a_ub[r, si * n_r + r] = k
        a_ub[r, -1] = -1.0
    lb = np.zeros(nv)
    ub = np.concatenate([np.repeat(counts, n_r), [np.inf]])
    integrality = np.concatenate([np.ones(nv - 1), [0]])
    res = milp(obj, constraints=[LinearConstraint(a_eq, counts, counts), LinearConstraint(a_ub, -np.inf, 0.0)],
               integrality=integrality, bounds=Bounds(lb, ub), options={"time_limit": float(time_limit)})
    if res.x is None:
        return lpt
    y = np.rint(res.x[:-1]).astype(int).reshape(n_s, n_r)
    if not all(int(y[si].sum()) == len(groups[k]) for si, k in enumerate(keys)) or (y < 0).any():
        return lpt
    owner = [0] * len(costs)
    for si, k in enumerate(keys):
        ids, pos = groups[k], 0
        for r in range(n_r):
            for _ in range(int(y[si, r])):
                owner[ids[pos]] = r
                pos += 1
    return owner if makespan(costs, owner, n_ranks) <= makespan(costs, lpt, n_ranks) else lpt


def makespan(costs: Sequence[float], owner: Sequence[int], n_ranks: int) -> float:
    loads = [0.0] * n_ranks
    for c, r in zip(costs, owner):
        loads[r] += float(c)
    return max(loads)


def owned_indices(owner: Sequence[int], rank: int) -> List[int]:
    return [i for i, r in enumerate(owner) if r == rank]


def assign_shapes(shapes: Sequence[Tuple[int, int]], n_ranks: int, steps: int = 5,
                  measured: Optional[Dict[Tuple[int, int], float]] = None, method: str = "lpt") -> List[int]:
    """Owners for a list of (rows, cols); ``measured`` maps a shape to its
    measured per-matrix cost and overrides the flop model for that shape.
    ``method``: "lpt" (greedy) or "milp" (exact program, LPT fallback)."""
    costs = []
    for r, c in shapes:
        key = (int(r), int(c))
        costs.append(measured[key] if measured and key in measured else matrix_cost(r, c, steps))
    if method == "milp":
        return milp_assign(costs, n_ranks)
    if method != "lpt":
        raise ValueError(f"unknown owner method {method!r}")
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


def measure_costs(shapes: Sequence[Tuple[int, int]], device=None, reps: int = 3,
                  batch: int = 4) -> Dict[Tuple[int, int], float]:
    """Measured cost (ms per matrix) of one full update for every distinct
    shape, timed on this GPU with CUDA events.  This is the per-shape
    profiling that the DMuon page's load balancer feeds its assignment
    with (section 2.3).

    Each shape is timed in batches of ``batch`` and ``2 * batch`` copies.
    The cost is the difference divided by ``batch``: the marginal cost of
    one more matrix in a batched step.  Fixed per-launch overheads, which a
    rank pays once whatever it owns, then cancel.  Synthetic bf16
    gradients; device work only through the library."""
    import torch
    from . import dmu, synth
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())

    def step_ms(shape, k):
        w = synth.custom("cost", [shape] * k, seed=17)
        grads = synth.gradients(w, dev)
        weights = synth.weights(w, dev)
        moms = [torch.zeros(shape, dtype=torch.float32, device=dev) for _ in range(k)]
        plan = dmu.Plan([shape] * k, device=dev)
        plan.step(grads, moms, weights, lr=0.0)  # warm-up, uploads the pointer tables
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            plan.step(grads, moms, weights, lr=0.0)
        e1.record()
        torch.cuda.synchronize(dev)
        plan.close()
        return e0.elapsed_time(e1) / reps

    out: Dict[Tuple[int, int], float] = {}
    distinct = sorted({(int(r), int(c)) for r, c in shapes})
    step_ms(distinct[0], 1)  # first-use costs (module load, clocks) outside the measurements
    for shape in distinct:
        t1 = step_ms(shape, batch)
        t2 = step_ms(shape, 2 * batch)
        out[shape] = max((t2 - t1) / batch, 1e-6)
    return out
