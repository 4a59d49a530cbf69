"""Owner assignment (DMuon page, sections 2.1 and 2.3: one owner per matrix,
greedy makespan fallback) and the cross-rank helpers, on CPU.

* LPT against brute force on tiny instances: within 4/3 of the optimum;
* every matrix owned exactly once, deterministic across calls;
* two gloo ranks (world size 2, 127.0.0.1) compute identical assignments,
  cover every matrix exactly once between them, and agree on the max over
  ranks.
"""
import itertools
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gram_newton_schulz_b200 import owners, synth


def _opt_makespan(costs, n):
    best = float("inf")
    for assign in itertools.product(range(n), repeat=len(costs)):
        best = min(best, owners.makespan(costs, assign, n))
    return best


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("n", [2, 3])
def test_lpt_within_four_thirds_of_optimum(seed, n):
    g = torch.Generator().manual_seed(seed)
    costs = (torch.rand(7, generator=g) * 10 + 1).tolist()
    own = owners.lpt_assign(costs, n)
    assert sorted(set(own)) <= list(range(n))
    ms = owners.makespan(costs, own, n)
    opt = _opt_makespan(costs, n)
    assert ms <= 4.0 / 3.0 * opt + 1e-9
    assert own == owners.lpt_assign(costs, n)  # deterministic


def test_layer_set_assignment_balanced():
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    for n in (1, 2, 4, 8):
        own = owners.assign_shapes(w.shapes, n)
        costs = [owners.matrix_cost(r, c) for r, c in w.shapes]
        loads = [sum(c for c, o in zip(costs, own) if o == r) for r in range(n)]
        assert abs(sum(loads) - sum(costs)) < 1e-6 * sum(costs)
        # the largest matrix bounds the imbalance
        assert max(loads) - min(loads) <= max(costs) + 1e-9
        idx = [i for r in range(n) for i in owners.owned_indices(own, r)]
        assert sorted(idx) == list(range(w.count))


def test_measured_costs_override_model():
    shapes = [(4, 8), (8, 4), (16, 16)]
    own = owners.assign_shapes(shapes, 2, measured={(16, 16): 0.0, (4, 8): 100.0})
    assert own[0] != own[1] or own[0] != own[2]
    assert owners.matrix_cost(3584, 18944) == owners.matrix_cost(18944, 3584)


def test_max_over_ranks_without_process_group():
    assert owners.max_over_ranks(3.5) == 3.5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.workload("qwen2.5-7b-layer-set-x28")
        own = owners.assign_shapes(w.shapes, world)
        mine = owners.owned_indices(own, rank)
        counts = torch.zeros(w.count, dtype=torch.int64)
        counts[mine] = 1
        dist.all_reduce(counts)
        sig = torch.tensor([hash(tuple(own)) % (2 ** 31)], dtype=torch.int64)
        sigs = [torch.zeros_like(sig) for _ in range(world)]
        dist.all_gather(sigs, sig)
        mx = owners.max_over_ranks(10.0 + rank)
        out_q.put((rank, bool(torch.all(counts == 1)), len({int(s) for s in sigs}) == 1, mx))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_cover_every_matrix_once():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, covered, same, mx in results:
        assert covered and same
        assert mx == 11.0


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("n", [2, 3])
def test_milp_reaches_the_optimum_on_small_instances(seed, n):
    g = torch.Generator().manual_seed(100 + seed)
    base = (torch.rand(3, generator=g) * 10 + 1).tolist()
    costs = [base[int(i)] for i in torch.randint(0, 3, (7,), generator=g)]  # repeated costs, as shapes repeat
    own = owners.milp_assign(costs, n)
    assert sorted(set(own)) <= list(range(n)) and len(own) == len(costs)
    assert owners.makespan(costs, own, n) == pytest.approx(_opt_makespan(costs, n), rel=1e-9)
    assert owners.makespan(costs, own, n) <= owners.makespan(costs, owners.lpt_assign(costs, n), n) + 1e-9
    assert own == owners.milp_assign(costs, n)


def test_milp_on_the_layer_set_is_valid_and_no_worse_than_lpt():
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    costs = [owners.matrix_cost(r, c) for r, c in w.shapes]
    for n in (2, 3, 5, 8):
        own = owners.assign_shapes(w.shapes, n, method="milp")
        assert len(own) == w.count and sorted(set(own)) == list(range(n))
        assert owners.makespan(costs, own, n) <= owners.makespan(costs, owners.lpt_assign(costs, n), n) + 1e-6
    with pytest.raises(ValueError):
        owners.assign_shapes(w.shapes, 2, method="annealing")
    # too many variables: the greedy fallback
    assert owners.milp_assign(costs, 8, max_vars=10) == owners.lpt_assign(costs, 8)
