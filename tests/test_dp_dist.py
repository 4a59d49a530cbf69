"""Owner-sharded data-parallel step (DMuon page, section 2.1) on CPU ranks.

The exchange logic of `gram_newton_schulz_b200.dp` runs here over gloo
(127.0.0.1) with world sizes 2 and 3. The device compute is replaced by the
fp64 oracle, since tests may import it and the product path may not. The
tests check:

* bucket layout: every matrix in exactly one owner bucket, views on
  256-byte boundaries, no overlap;
* after one step, every rank holds the weights the oracle gives for the
  mean gradient, bit for bit. The gradients are chosen so that their float32
  sums are exact in any order;
* the owner's momentum is the oracle's, and each rank computes exactly its
  owned matrices, in two publish groups;
* the collectives are issued in the same order on every rank: all reduces,
  then each group's broadcasts right after that group's compute, so a
  group's publish overlaps the next group's compute;
* a rank that dies before the exchange surfaces on the other rank as an
  error from the collective (short process-group timeout), not a hang.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gram_newton_schulz_b200 import dp
from oracle import gram_ns

SHAPES = [(8, 24), (24, 8), (16, 16), (4, 32), (12, 20), (8, 8), (32, 16)]
BETA, LR, EPS = 0.9, 0.05, 1e-7


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _grad(i, rank):
    """Per-rank gradient of matrix i: multiples of 2^-6 in [-2, 2], so float32
    sums over a few ranks are exact in any order."""
    rows, cols = SHAPES[i]
    g = np.random.default_rng(1000 * i + rank).integers(-128, 129, size=(rows, cols))
    return (g / 64.0).astype(np.float32)


def _weight(i):
    rows, cols = SHAPES[i]
    return np.random.default_rng(77 + i).standard_normal((rows, cols)).astype(np.float32)


def _momentum0(i):
    rows, cols = SHAPES[i]
    return (np.random.default_rng(300 + i).integers(-64, 65, size=(rows, cols)) / 32.0).astype(np.float32)


class OracleCompute:
    """Test stand-in for the device compute: the fp64 oracle per owned
    matrix.  ``log`` records ("compute", matrices) per call."""

    def __init__(self, log=None):
        self.log = log if log is not None else []

    @property
    def calls(self):
        return [n for kind, n in self.log if kind == "compute"]

    def __call__(self, grads, momenta, weights, *, beta, lr, eps, coeffs, steps, grad_scale=1.0):
        self.log.append(("compute", len(grads)))
        for g, m, w in zip(grads, momenta, weights):
            g = g * np.float32(grad_scale)  # fp32 product, as the momentum pass forms it
            m_new, _, w_new = gram_ns.muon_step(w.double().numpy(), m.double().numpy(), g.double().numpy(),
                                                beta=beta, lr=lr, eps=eps, coeffs=coeffs, steps=steps)
            m.copy_(torch.from_numpy(m_new))
            w.copy_(torch.from_numpy(w_new))


def _expected(world):
    """Weights and momenta after one step, from the mean gradient."""
    out_w, out_m = [], []
    for i in range(len(SHAPES)):
        s = np.zeros(SHAPES[i], dtype=np.float32)
        for r in range(world):
            s = s + _grad(i, r)
        # the mean as the owner's momentum pass forms it: the fp32 sum times 1/N in fp32
        mean = (s * np.float32(1.0 / world)).astype(np.float32)
        m_new, _, w_new = gram_ns.muon_step(_weight(i).astype(np.float64), _momentum0(i).astype(np.float64),
                                            mean.astype(np.float64), beta=BETA, lr=LR, eps=EPS)
        out_w.append(w_new.astype(np.float32))
        out_m.append(m_new.astype(np.float32))
    return out_w, out_m


def _step_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        log = []
        compute = OracleCompute(log)
        step = dp.OwnerShardedStep(SHAPES, compute=compute)
        buckets = step.buckets
        gf = buckets.alloc(torch.float32, "cpu")
        wf = buckets.alloc(torch.float32, "cpu")
        for i in range(len(SHAPES)):
            buckets.view(gf, i).copy_(torch.from_numpy(_grad(i, rank)))
            buckets.view(wf, i).copy_(torch.from_numpy(_weight(i)))
        moms = [torch.from_numpy(_momentum0(i)).clone() for i in step.mine]
        # record the order in which the step issues its collectives
        real_reduce, real_bcast = dist.reduce, dist.broadcast

        def reduce(t, dst, **kw):
            log.append(("reduce", dst))
            return real_reduce(t, dst, **kw)

        def broadcast(t, src, **kw):
            log.append(("bcast", src))
            return real_bcast(t, src, **kw)

        dist.reduce, dist.broadcast = reduce, broadcast
        try:
            step.step(gf, wf, moms, beta=BETA, lr=LR, eps=EPS)
        finally:
            dist.reduce, dist.broadcast = real_reduce, real_bcast
        q.put((rank, list(step.mine), log, [len(g) for g in step.publish],
               [buckets.view(wf, i).numpy().copy() for i in range(len(SHAPES))],
               [m.numpy().copy() for m in moms]))
    finally:
        dist.destroy_process_group()


def test_owner_buckets_layout():
    for world in (1, 2, 3, 4):
        b = dp.OwnerBuckets(SHAPES, world)
        seen = sorted(i for r in range(world) for i in b.members[r])
        assert seen == list(range(len(SHAPES)))
        for r in range(world):
            spans = sorted((b.offset[i], b.offset[i] + SHAPES[i][0] * SHAPES[i][1]) for i in b.members[r])
            for (s0, e0), (s1, _) in zip(spans, spans[1:]):
                assert e0 <= s1
            assert all(s % dp.ALIGN_ELEMS == 0 for s, _ in spans)
            assert not spans or spans[-1][1] <= b.sizes[r]
        flats = b.alloc(torch.float32, "cpu")
        for i, v in enumerate(b.views(flats)):
            assert tuple(v.shape) == SHAPES[i] and v.is_contiguous()
            assert (v.data_ptr() - flats[b.owner[i]].data_ptr()) % 256 == 0


def test_single_process_step_matches_oracle():
    compute = OracleCompute()
    step = dp.OwnerShardedStep(SHAPES, compute=compute)
    assert step.world == 1 and sorted(step.mine) == list(range(len(SHAPES)))
    assert len(compute.calls) == 0 and [len(g) for g in step.publish] != [len(SHAPES), 0]
    b = step.buckets
    gf, wf = b.alloc(torch.float32, "cpu"), b.alloc(torch.float32, "cpu")
    for i in range(len(SHAPES)):
        b.view(gf, i).copy_(torch.from_numpy(_grad(i, 0)))
        b.view(wf, i).copy_(torch.from_numpy(_weight(i)))
    moms = [torch.from_numpy(_momentum0(i)).clone() for i in step.mine]
    step.step(gf, wf, moms, beta=BETA, lr=LR, eps=EPS)
    assert compute.calls == [len(g) for g in step.publish]  # one call per publish group
    # a stand-in compute has no schedules to tune: autotune is a no-op
    assert step.autotune() == []
    ew, em = _expected(1)
    for i in range(len(SHAPES)):
        assert np.array_equal(b.view(wf, i).numpy(), ew[i])
    for k, i in enumerate(step.mine):
        assert np.array_equal(moms[k].numpy(), em[i])


def test_publish_groups_balance_cost():
    """Each rank's owned matrices split into two publish groups of about
    equal flop cost (LPT over the groups), each in its own bucket."""
    from gram_newton_schulz_b200 import owners
    for world in (1, 2, 3):
        b = dp.OwnerBuckets(SHAPES, world, groups=2)
        assert len(b.sizes) == 2 * world
        for r in range(world):
            g0, g1 = b.group_members[r]
            assert sorted(g0 + g1) == sorted(b.members[r]) and b.members[r] == g0 + g1
            c0 = sum(owners.matrix_cost(*SHAPES[i]) for i in g0)
            c1 = sum(owners.matrix_cost(*SHAPES[i]) for i in g1)
            if g0 and g1:
                assert max(c0, c1) <= min(c0, c1) + max(owners.matrix_cost(*SHAPES[i]) for i in g0 + g1)
        flats = b.alloc(torch.float32, "cpu")
        seen = set()
        for i, v in enumerate(b.views(flats)):
            assert tuple(v.shape) == SHAPES[i]
            k = b.bucket(b.owner[i], b.group[i])
            assert (v.data_ptr() - flats[k].data_ptr()) % 256 == 0
            seen.add((k, b.offset[i]))
        assert len(seen) == len(SHAPES)


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_owner_step_matches_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_step_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    ew, em = _expected(world)
    owned = []
    for rank, mine, log, groups, weights, moms in results:
        # reduces of all 2 * world buckets first; then per publish group: its
        # compute (if the group has matrices), then one broadcast per rank
        expect = [("reduce", b // 2) for b in range(2 * world)]
        for g in range(2):
            if groups[g]:
                expect.append(("compute", groups[g]))
            expect += [("bcast", r) for r in range(world)]
        assert log == expect, (rank, log)
        assert sum(groups) == len(mine)
        owned += mine
        for i in range(len(SHAPES)):
            assert np.array_equal(weights[i], ew[i]), (rank, i)
        for k, i in enumerate(mine):
            assert np.array_equal(moms[k], em[i]), (rank, i)
    assert sorted(owned) == list(range(len(SHAPES)))


def _dying_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()
        os._exit(0)  # leaves between steps, before the exchange
    try:
        # the owner table is broadcast from rank 0 when the step is built,
        # and the exchange follows: either collective reports the missing peer
        step = dp.OwnerShardedStep(SHAPES, compute=OracleCompute())
        buckets = step.buckets
        gf, wf = buckets.alloc(torch.float32, "cpu"), buckets.alloc(torch.float32, "cpu")
        moms = [torch.zeros(SHAPES[i]) for i in step.mine]
        step.step(gf, wf, moms)
        q.put((rank, "no error"))
    except Exception as e:
        q.put((rank, "error: " + type(e).__name__))
    q.close()
    q.join_thread()
    os._exit(0)


def test_gloo_missing_rank_is_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = dict(q.get(timeout=120) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert got[1] == "left"
    assert got[0].startswith("error"), got[0]


def _cost_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # every rank "measures" something different; only rank 0's table counts
        fake = lambda shapes: {tuple(s): float(s[0] * s[1]) * (1.0 + rank) for s in shapes}  # noqa: E731
        costs = dp.shared_costs(SHAPES, measure=fake)
        step = dp.OwnerShardedStep(SHAPES, compute=OracleCompute(), measured=costs)
        q.put((rank, sorted(costs.items()), list(step.buckets.owner)))
    finally:
        dist.destroy_process_group()


def test_measured_costs_are_shared_so_owners_agree():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cost_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    try:
        res = [q.get(timeout=180) for _ in range(3)]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    costs = {r: c for r, c, _ in res}
    owners_ = {r: o for r, _, o in res}
    assert costs[0] == costs[1] == costs[2]
    assert dict(costs[0])[(8, 24)] == 8 * 24 * 1.0  # rank 0's measurement
    assert owners_[0] == owners_[1] == owners_[2]


def _sparse_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shapes = SHAPES[:3]  # fewer matrices than ranks: some ranks own nothing
        step = dp.OwnerShardedStep(shapes, compute=OracleCompute())
        b = step.buckets
        gf, wf = b.alloc(torch.float32, "cpu"), b.alloc(torch.float32, "cpu")
        for i in range(len(shapes)):
            b.view(gf, i).copy_(torch.from_numpy(_grad(i, rank)))
            b.view(wf, i).copy_(torch.from_numpy(_weight(i)))
        moms = [torch.from_numpy(_momentum0(i)).clone() for i in step.mine]
        step.step(gf, wf, moms, beta=BETA, lr=LR, eps=EPS)
        q.put((rank, list(step.mine), [b.view(wf, i).numpy().copy() for i in range(len(shapes))]))
    finally:
        dist.destroy_process_group()


def test_more_ranks_than_matrices():
    world = 5
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sparse_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = [q.get(timeout=180) for _ in range(world)]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    ew, _ = _expected(world)
    owned = sorted(i for _, mine, _ in res for i in mine)
    assert owned == [0, 1, 2]
    assert sum(1 for _, mine, _ in res if not mine) == world - 3
    for rank, mine, weights in res:
        for i in range(3):
            assert np.array_equal(weights[i], ew[i]), (rank, i)
