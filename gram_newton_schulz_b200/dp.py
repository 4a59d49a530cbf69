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
  that owner.  Each owner's matrices form two publish groups of about equal
  cost; a group's broadcasts are issued as soon as its compute is enqueued,
  so they run on the communicator's stream while the next group computes
  (DMuon page, section 2.1: the publish is asynchronous and pipelined with
  the compute).

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
    """Owner of every matrix, its publish group, and where it lives in its
    (owner, group) flat bucket.  The same on every rank: LPT is
    deterministic.

    A rank's owned matrices are split into ``groups`` publish groups of
    about equal cost (LPT over the groups); bucket ``owner * groups +
    group`` holds one group's matrices.  The step computes the groups in
    order and broadcasts each group's weights as soon as it is done, so a
    group's publish overlaps the next group's compute."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], world: int,
                 measured: Optional[Dict[Tuple[int, int], float]] = None, method: str = "lpt",
                 owner: Optional[Sequence[int]] = None, groups: int = 1):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.world = int(world)
        self.groups = int(groups)
        if self.groups < 1:
            raise ValueError("groups must be >= 1")
        if owner is not None:
            if len(owner) != len(self.shapes) or any(not 0 <= int(o) < self.world for o in owner):
                raise ValueError("owner: one rank in [0, world) per matrix")
            self.owner = [int(o) for o in owner]
        else:
            self.owner = owners.assign_shapes(self.shapes, self.world, measured=measured, method=method)
        costs = [measured[s] if measured and s in measured else owners.matrix_cost(*s) for s in self.shapes]
        self.group = [0] * len(self.shapes)
        # members[r]: rank r's matrices, group 0 first; group_members[r][g]
        self.members: List[List[int]] = []
        self.group_members: List[List[List[int]]] = []
        for r in range(self.world):
            mine = owners.owned_indices(self.owner, r)
            g_of = owners.lpt_assign([costs[i] for i in mine], self.groups)
            per = [[i for i, g in zip(mine, g_of) if g == grp] for grp in range(self.groups)]
            for grp, lst in enumerate(per):
                for i in lst:
                    self.group[i] = grp
            self.group_members.append(per)
            self.members.append([i for lst in per for i in lst])
        self.offset = [0] * len(self.shapes)
        self.sizes = [0] * (self.world * self.groups)
        for r in range(self.world):
            for grp in range(self.groups):
                off = 0
                for i in self.group_members[r][grp]:
                    self.offset[i] = off
                    rows, cols = self.shapes[i]
                    off += _align(rows * cols)
                self.sizes[self.bucket(r, grp)] = off

    def bucket(self, rank: int, group: int) -> int:
        return rank * self.groups + group

    def alloc(self, dtype, device) -> list:
        """One zero-filled flat buffer per (owner rank, group) bucket (at
        least 1 element each)."""
        import torch
        return [torch.zeros(max(n, 1), dtype=dtype, device=device) for n in self.sizes]

    def view(self, flats: list, i: int):
        """Matrix i as a contiguous (rows, cols) view of its bucket."""
        rows, cols = self.shapes[i]
        o = self.offset[i]
        return flats[self.bucket(self.owner[i], self.group[i])][o:o + rows * cols].view(rows, cols)

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

    def autotune(self, cache_path=None):
        """Per-shape schedule choice for this group's plan (needs the data
        of a prior call); see `dmu.Plan.autotune`."""
        return self.plan.autotune(cache_path) if self.plan is not None else {}

    def close(self):
        if self.plan is not None:
            self.plan.close()
            self.plan = None


class OwnerShardedStep:
    """One data-parallel Muon step with owner sharding.

    Each rank's owned matrices form ``publish`` groups of about equal cost.
    ``compute(grads, momenta, weights, beta=, lr=, eps=, coeffs=, steps=,
    grad_scale=[, out_o=])`` updates one group's matrices in place; it is
    called once per group, in group order.  By default every group has its
    own `dmu.Plan` (`PlanCompute`); tests pass a stand-in.
    """

    def __init__(self, shapes, *, group=None, compute=None, dtype="bf16", prec="auto",
                 device=None, measured=None, method: str = "lpt", publish: int = 2):
        import torch.distributed as dist
        self.group = group  # the process group
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
        self.buckets = OwnerBuckets(shapes, self.world, measured=measured, method=method, owner=owner,
                                    groups=publish)
        self.mine = self.buckets.members[self.rank]
        self.publish = [self.buckets.group_members[self.rank][g] for g in range(self.buckets.groups)]
        if compute is not None:
            self.computes = [compute] * len(self.publish)
        else:
            self.computes = [PlanCompute([self.buckets.shapes[i] for i in idx], dtype, prec, device)
                             for idx in self.publish]

    def owned_shapes(self):
        return [self.buckets.shapes[i] for i in self.mine]

    @property
    def launches(self) -> int:
        """Kernel launches of the last step's compute (all groups)."""
        return sum(getattr(c, "launches", 0) for c in set(self.computes))

    @property
    def tc_launches(self) -> int:
        return sum(getattr(c, "tc_launches", 0) for c in set(self.computes))

    def autotune(self, cache_path=None):
        """Per-shape schedule choice for each publish group's plan, after a
        step has given the plans data.  Local to this rank: schedules change
        no collective, so the ranks need not agree on them."""
        return [c.autotune(cache_path) for c in self.computes if hasattr(c, "autotune")]

    def read_status(self) -> int:
        """OR of the device status words of the groups' plans."""
        st = 0
        for c in self.computes:
            plan = getattr(c, "plan", None)
            if plan is not None:
                st |= plan.read_status()
        return st

    def step(self, grad_flats: list, weight_flats: list, momenta: list, *, beta=0.95, lr=0.02,
             eps=1e-7, coeffs=(3.4445, -4.7750, 2.0315), steps=5, events=None, out_o=None):
        """grad_flats / weight_flats: the (owner, group) flat buffers of
        `OwnerBuckets.alloc`, on every rank; momenta: fp32 tensors of the
        owned matrices, in `self.mine` order.  On return every rank's weight
        buffers hold the updated weights (the broadcasts are waited on, which
        on GPUs orders the current stream after them).

        Collectives, issued in the same order on every rank: one reduce per
        bucket to its owner (all at once), then per group g, after the
        owner's compute of g is enqueued, one broadcast per rank of that
        rank's group-g bucket.  Group g's broadcasts run on the
        communicator's stream while group g+1 computes.

        ``events``: four CUDA events recorded on the current stream at the
        start, after the first group's gradients arrived, after the last
        compute was enqueued, and after the exchange out.  ``out_o``:
        optional fp32 tensors (owned matrices, `self.mine` order) that
        receive O."""
        import torch.distributed as dist
        if len(momenta) != len(self.mine):
            raise ValueError(f"expected {len(self.mine)} momenta, got {len(momenta)}")
        b = self.buckets
        pos = {i: k for k, i in enumerate(self.mine)}
        if events is not None:
            events[0].record()
        ins = {}
        if self.world > 1:
            for bid in range(len(b.sizes)):
                ins[bid] = dist.reduce(grad_flats[bid], dst=bid // b.groups, op=dist.ReduceOp.SUM,
                                       group=self.group, async_op=True)
        outs = []
        for g, idx in enumerate(self.publish):
            if self.world > 1:
                ins[b.bucket(self.rank, g)].wait()
            if g == 0 and events is not None:
                events[1].record()
            if idx:
                kw = {} if out_o is None else {"out_o": [out_o[pos[i]] for i in idx]}
                # the bucket holds the sum of the ranks' gradients; the
                # momentum pass scales it to the mean as it reads it
                self.computes[g]([b.view(grad_flats, i) for i in idx], [momenta[pos[i]] for i in idx],
                                 [b.view(weight_flats, i) for i in idx], beta=beta, lr=lr, eps=eps,
                                 coeffs=coeffs, steps=steps, grad_scale=1.0 / self.world, **kw)
            if self.world > 1:
                outs += [dist.broadcast(weight_flats[b.bucket(r, g)], src=r, group=self.group, async_op=True)
                         for r in range(self.world)]
        if events is not None:
            events[2].record()
        if self.world > 1:
            for bid, w in ins.items():
                if bid // b.groups != self.rank:
                    w.wait()
            for w in outs:
                w.wait()
        if events is not None:
            events[3].record()

    def close(self):
        for c in set(self.computes):
            if hasattr(c, "close"):
                c.close()
