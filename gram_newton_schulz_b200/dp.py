"""Owner-sharded data-parallel Muon step over torch.distributed.

DMuon page, section 2.1 (owner-centric execution): in data-parallel training
every rank holds every weight matrix and a gradient for it.  Each matrix has
exactly one owner rank.  The gradients of a matrix are reduced to its owner,
the owner keeps the momentum and runs the whole update once, and the updated
matrix goes back to every rank.  Section 2.3 chooses the owners to balance
the predicted cost (`owners.assign_shapes`, LPT).

One exchange step per optimizer step, as collectives over the process group
(NCCL over NVLink on GPUs, gloo on CPU for the tests):

* **In.** One `reduce` (sum) per owner bucket to that owner. A bucket is the
  flat buffer that holds the gradients of all matrices one rank owns. The
  owner's momentum pass reads the sum scaled by 1 / world size, the mean
  gradient, with no separate pass over the bucket.
* **Compute.** The owner runs momentum, Gram Newton-Schulz and the fused
  weight update on its own matrices only.
* **Out.** One `broadcast` per owner bucket of the updated weights from
  that owner.

All collectives are issued asynchronously, every rank in the same order.  A
rank waits only for the reduce of its own bucket before it computes, so the
reduces of the other buckets run on the communicator's stream during the
compute.

Gradients and weights live as views of the per-owner flat buffers, so each
exchange is one collective per owner.  Every view starts on a 256-byte
boundary: the kernels read them with 16-byte vector loads.

Host logic only: the device work is done by the `compute` object, which is
a `dmu.Plan` over the owned shapes in production.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

from . import owners

ALIGN_ELEMS = 128  # 256 bytes of bf16; every matrix view starts on this boundary


def _align(n: int) -> int:
    return (n + ALIGN_ELEMS - 1) // ALIGN_ELEMS * ALIGN_ELEMS


class OwnerBuckets:
    """Owner of every matrix, and where each matrix lives in its owner's flat
    bucket.  The same on every rank: LPT is deterministic."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], world: int,
                 measured: Optional[Dict[Tuple[int, int], float]] = None, method: str = "lpt",
                 owner: Optional[Sequence[int]] = None):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.world = int(world)
        if owner is not None:
            if len(owner) != len(self.shapes) or any(not 0 <= int(o) < self.world for o in owner):
                raise ValueError("owner: one rank in [0, world) per matrix")
            self.owner = [int(o) for o in owner]
        else:
            self.owner = owners.assign_shapes(self.shapes, self.world, measured=measured, method=method)
        self.members: List[List[int]] = [owners.owned_indices(self.owner, r) for r in range(self.world)]
        self.offset = [0] * len(self.shapes)
        self.sizes = [0] * self.world
        for r in range(self.world):
            off = 0
            for i in self.members[r]:
                self.offset[i] = off
                rows, cols = self.shapes[i]
                off += _align(rows * cols)
            self.sizes[r] = off

    def alloc(self, dtype, device) -> list:
        """One zero-filled flat buffer per owner rank (at least 1 element)."""
        import torch
        return [torch.zeros(max(n, 1), dtype=dtype, device=device) for n in self.sizes]

    def view(self, flats: list, i: int):
        """Matrix i as a contiguous (rows, cols) view of its owner's bucket."""
        rows, cols = self.shapes[i]
        o = self.offset[i]
        return flats[self.owner[i]][o:o + rows * cols].view(rows, cols)

    def views(self, flats: list) -> list:
        return [self.view(flats, i) for i in range(len(self.shapes))]


def shared_costs(shapes, measure=None, group=None, src: int = 0) -> Dict[Tuple[int, int], float]:
    """Per-shape costs that every rank agrees on: rank ``src`` measures
    them (``owners.measure_costs`` on its GPU by default) and broadcasts the
    table, so LPT gives the same owners everywhere."""
    import torch.distributed as dist
    if measure is None:
        measure = owners.measure_costs
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return dict(measure(shapes))
    box = [dict(measure(shapes)) if dist.get_rank(group) == src else None]
    dist.broadcast_object_list(box, src=src, group=group)
    return box[0]


class PlanCompute:
    """The owned matrices' update on the GPU: one `dmu.Plan` over them."""

    def __init__(self, shapes, dtype="bf16", prec="auto", device=None):
        from . import dmu
        self.plan = dmu.Plan(shapes, dtype=dtype, prec=prec, device=device) if shapes else None
        self.launches = 0      # kernel launches of the last call
        self.tc_launches = 0   # of which tensor-core (Gram recursion + final update)

    def __call__(self, grads, momenta, weights, *, beta, lr, eps, coeffs, steps, grad_scale=1.0, out_o=None):
        self.launches = self.tc_launches = 0
        if self.plan is None:
            return
        self.plan.momentum_normalize(grads, momenta, beta, eps, grad_scale=grad_scale)
        n0 = self.plan.last_launch_count()
        self.plan.gram_ns_batched(None, coeffs, steps)
        n1 = self.plan.last_launch_count()
        self.plan.apply_update(weights, lr, out_o=out_o)
        n2 = self.plan.last_launch_count()
        self.launches, self.tc_launches = n0 + n1 + n2, n1 + n2

    def close(self):
        if self.plan is not None:
            self.plan.close()
            self.plan = None


class OwnerShardedStep:
    """One data-parallel Muon step with owner sharding.

    ``compute(grads, momenta, weights, beta=, lr=, eps=, coeffs=, steps=)``
    updates the owned matrices in place.  It defaults to a `dmu.Plan` over
    the owned shapes; tests pass their own.
    """

    def __init__(self, shapes, *, group=None, compute=None, dtype="bf16", prec="auto",
                 device=None, measured=None, method: str = "lpt"):
        import torch.distributed as dist
        self.group = group
        self.dist = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if self.dist else 1
        self.rank = dist.get_rank(group) if self.dist else 0
        owner = None
        if self.world > 1:
            # rank 0 decides and every rank takes its answer, so the owners
            # agree even if a solver's result depended on the process
            box = [owners.assign_shapes(shapes, self.world, measured=measured, method=method)
                   if self.rank == 0 else None]
            dist.broadcast_object_list(box, src=0, group=group)
            owner = box[0]
        self.buckets = OwnerBuckets(shapes, self.world, measured=measured, method=method, owner=owner)
        self.mine = self.buckets.members[self.rank]
        owned = [self.buckets.shapes[i] for i in self.mine]
        self.compute = compute if compute is not None else PlanCompute(owned, dtype, prec, device)

    def owned_shapes(self):
        return [self.buckets.shapes[i] for i in self.mine]

    def step(self, grad_flats: list, weight_flats: list, momenta: list, *, beta=0.95, lr=0.02,
             eps=1e-7, coeffs=(3.4445, -4.7750, 2.0315), steps=5, events=None, out_o=None):
        """grad_flats / weight_flats: the per-owner flat buffers of
        `OwnerBuckets.alloc`, on every rank; momenta: fp32 tensors of the owned
        matrices, in `self.mine` order.  On return every rank's weight buffers
        hold the updated weights (the broadcasts are waited on, which on GPUs
        orders the current stream after them).  ``events``: four CUDA events
        recorded on the current stream at the start, after the exchange in,
        after the compute and after the exchange out.  ``out_o``: optional
        fp32 tensors (owned matrices, `self.mine` order) that receive O."""
        import torch.distributed as dist
        if len(momenta) != len(self.mine):
            raise ValueError(f"expected {len(self.mine)} momenta, got {len(momenta)}")
        b = self.buckets
        if events is not None:
            events[0].record()
        if self.world > 1:
            works = [dist.reduce(grad_flats[r], dst=r, op=dist.ReduceOp.SUM, group=self.group, async_op=True)
                     for r in range(self.world)]
            works[self.rank].wait()
        if events is not None:
            events[1].record()
        grads = [b.view(grad_flats, i) for i in self.mine]
        weights = [b.view(weight_flats, i) for i in self.mine]
        kw = {} if out_o is None else {"out_o": out_o}
        # the owner's bucket holds the sum of the ranks' gradients; the
        # momentum pass scales it to the mean as it reads it
        self.compute(grads, momenta, weights, beta=beta, lr=lr, eps=eps, coeffs=coeffs, steps=steps,
                     grad_scale=1.0 / self.world, **kw)
        if events is not None:
            events[2].record()
        if self.world > 1:
            for r, w in enumerate(works):
                if r != self.rank:
                    w.wait()
            outs = [dist.broadcast(weight_flats[r], src=r, group=self.group, async_op=True)
                    for r in range(self.world)]
            for w in outs:
                w.wait()
        if events is not None:
            events[3].record()

    def close(self):
        if hasattr(self.compute, "close"):
            self.compute.close()
