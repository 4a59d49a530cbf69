"""The owner-sharded step's device path on one GPU (world size 1, so there
are no collectives): the compute must run on views of the per-owner flat
buffers; its O must match the fp64 oracle's Muon step (2e-2 relative
Frobenius error) and its W write must be within one bf16 ulp of
bf16(W - lr * scale * O); and it must agree bit for bit with the same
update through `dmu.Plan.step` on separate tensors.  (DMuon page, section
2.1: the owner runs the whole update of the matrices it owns.)"""
import numpy as np
import pytest
import torch

import oracle
from gram_newton_schulz_b200 import dmu, dp, synth
from gpu_util import check_update_within_ulp, f64, rel

pytestmark = pytest.mark.gpu


def test_owner_step_on_flat_buffers_matches_plan_step():
    shapes = [(512, 2048), (2048, 512), (384, 384), (256, 1024), (1024, 1024)]
    w = synth.custom("dp-check", shapes, seed=11)
    dev = torch.device("cuda", 0)
    grads = synth.gradients(w, dev)
    weights = synth.weights(w, dev)

    osd = dp.OwnerShardedStep(shapes, device=dev)
    assert osd.world == 1 and sorted(osd.mine) == list(range(len(shapes)))
    b = osd.buckets
    gflat, wflat = b.alloc(torch.bfloat16, dev), b.alloc(torch.bfloat16, dev)
    for i in range(len(shapes)):
        b.view(gflat, i).copy_(grads[i])
        b.view(wflat, i).copy_(weights[i])
    moms_a = [torch.zeros(shapes[i], dtype=torch.float32, device=dev) for i in osd.mine]
    moms_b = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
    plan = dmu.Plan(shapes, device=dev)
    w_ref = [x.clone() for x in weights]
    for k in range(2):
        osd.step(gflat, wflat, moms_a, beta=0.95, lr=0.02)
        plan.step(grads, moms_b, w_ref, beta=0.95, lr=0.02)
        if k == 0:
            # the owner plans pick schedules per shape on their own data;
            # every schedule gives the same bits, so the comparison stands
            choices = osd.autotune()
            assert len(choices) == len(osd.computes) and all("gram" in c for c in choices if c)
    torch.cuda.synchronize()
    assert osd.launches > 0 and osd.tc_launches > 0
    for i in range(len(shapes)):
        assert torch.equal(b.view(wflat, i), w_ref[i]), i
    for k, i in enumerate(osd.mine):
        assert torch.equal(moms_a[k], moms_b[i]), i
    assert osd.read_status() == 0
    osd.close()
    plan.close()


def test_owner_step_matches_oracle():
    """Two owner-sharded steps on flat buffers; after the second, O of every
    matrix against the oracle on the accumulated momentum, W against O."""
    shapes = [(512, 2048), (2048, 512), (384, 384), (1024, 4096), (4096, 1024), (300, 700)]
    w = synth.custom("dp-oracle", shapes, seed=12)
    dev = torch.device("cuda", 0)
    grads = synth.gradients(w, dev)
    weights = synth.weights(w, dev)
    osd = dp.OwnerShardedStep(shapes, device=dev)
    b = osd.buckets
    gflat, wflat = b.alloc(torch.bfloat16, dev), b.alloc(torch.bfloat16, dev)
    for i in range(len(shapes)):
        b.view(gflat, i).copy_(grads[i])
        b.view(wflat, i).copy_(weights[i])
    # momenta and O in the step's owned order
    moms = [torch.zeros(shapes[i], dtype=torch.float32, device=dev) for i in osd.mine]
    outs_m = [torch.empty(shapes[i], dtype=torch.float32, device=dev) for i in osd.mine]
    osd.step(gflat, wflat, moms, beta=0.95, lr=0.02)
    w_mid = [b.view(wflat, i).clone() for i in range(len(shapes))]
    osd.step(gflat, wflat, moms, beta=0.95, lr=0.02, out_o=outs_m)
    torch.cuda.synchronize()
    assert osd.read_status() == 0
    pos = {i: k for k, i in enumerate(osd.mine)}
    outs = [outs_m[pos[i]] for i in range(len(shapes))]
    for i, (r, c) in enumerate(shapes):
        g = f64(grads[i])
        m_ref = oracle.momentum(oracle.momentum(np.zeros_like(g), g, 0.95), g, 0.95)
        np.testing.assert_allclose(f64(moms[pos[i]]), m_ref, rtol=2.0 ** -22, atol=0)
        # the oracle's Muon step on the momentum the device holds
        _, o_ref, _ = oracle.muon_step(f64(w_mid[i]), 0.95 * g, g, beta=1.0, lr=0.02)
        e = rel(f64(outs[i]), o_ref)
        assert e < 2e-2, (r, c, e)
        u = check_update_within_ulp(w_mid[i], b.view(wflat, i), outs[i], r, c, 0.02)
        assert u <= 1.0, (r, c, u)
    osd.close()


def test_measured_costs_order_shapes_by_work():
    from gram_newton_schulz_b200 import owners
    shapes = [(256, 1024), (1024, 4096), (1024, 4096), (512, 512)]
    costs = owners.measure_costs(shapes)
    assert set(costs) == {(256, 1024), (1024, 4096), (512, 512)}
    assert all(c > 0 for c in costs.values())
    assert costs[(1024, 4096)] > costs[(256, 1024)]
    own = owners.assign_shapes(shapes, 2, measured=costs)
    assert sorted(set(own)) == [0, 1]
