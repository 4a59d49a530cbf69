"""The on-chip Gram recursion for small matrices (m <= 128, split-bf16
precision) and the per-shape schedule cache (needs an sm_100a GPU).

DMuon page, section 2.2: the recursion runs in the m x m Gram space and
similar shapes are batched; for m <= 128 the whole recursion of a matrix
runs in one CTA, with G/T, R and P in shared memory, and only the final P
goes back to HBM.  It issues the same MMAs in the same order and applies
the same epilogue arithmetic as the staged path, so the two must agree bit
for bit; both must match the fp64 oracle.  DMuon page, section 2.4:
kernel configurations are tuned per shape and cached -- here per Gram class
and per bucket's final GEMM.
"""
import numpy as np
import pytest
import torch

import oracle
from gram_newton_schulz_b200 import dmu, synth
from gpu_util import EPS, check_update_within_ulp, f64, oracle_o, rel

pytestmark = pytest.mark.gpu

SMALL = [(128, 512), (512, 128), (100, 700), (700, 100), (64, 256), (8, 8), (1, 300), (128, 128), (33, 65)]


def _run(shapes, seed, monkeypatch, onchip, steps=5, coeffs=dmu.QUINTIC, prec="auto", dist="spiked"):
    monkeypatch.setenv("DMU_ONCHIP", "1" if onchip else "0")
    w = synth.custom("onchip", shapes, seed=seed, dist=dist, var=1e-3 if dist == "spiked" else 1.0)
    grads = synth.gradients(w, "cuda")
    weights = synth.weights(w, "cuda")
    w0 = [x.clone() for x in weights]
    moms = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    plan = dmu.Plan(shapes, prec=prec)
    plan.momentum_normalize(grads, moms, beta=w.beta, eps=EPS)
    plan.gram_ns_batched(None, coeffs, steps)
    plan.apply_update(weights, lr=w.lr, out_o=outs)
    torch.cuda.synchronize()
    assert plan.read_status() == 0
    return plan, grads, w0, weights, outs


def test_onchip_schedule_is_selected(monkeypatch):
    monkeypatch.setenv("DMU_ONCHIP", "1")
    plan = dmu.Plan([(128, 512), (256, 1024), (64, 64)])
    assert [plan.lib.dmu_get_gram_schedule(plan.handle, i) for i in range(3)] == [3, 1, 3]
    plan.close()
    plan = dmu.Plan([(128, 512)], prec="fast")  # only the split-bf16 class runs on chip
    assert plan.lib.dmu_get_gram_schedule(plan.handle, 0) == 1
    plan.close()


@pytest.mark.parametrize("steps", [1, 2, 5])
def test_onchip_equals_staged_bitwise(steps, monkeypatch):
    shapes = SMALL + [(256, 1024)]  # one class stays on the staged path
    _, _, _, w_a, o_a = _run(shapes, 71, monkeypatch, onchip=True, steps=steps)
    _, _, _, w_b, o_b = _run(shapes, 71, monkeypatch, onchip=False, steps=steps)
    for i, s in enumerate(shapes):
        assert torch.equal(o_a[i], o_b[i]), (s, steps)
        assert torch.equal(w_a[i], w_b[i]), (s, steps)


@pytest.mark.parametrize("dist", ["spiked", "normal"])
def test_onchip_matches_oracle(dist, monkeypatch):
    plan, grads, w0, w1, outs = _run(SMALL, 72, monkeypatch, onchip=True, dist=dist)
    for i, (r, c) in enumerate(SMALL):
        o_ref = oracle_o(grads[i], torch.zeros(r, c), 0.95)
        e = rel(f64(outs[i]), o_ref)
        assert e < 5e-3, (r, c, e)  # split-bf16 precision class
        assert check_update_within_ulp(w0[i], w1[i], outs[i], r, c, 0.02) <= 1.0, (r, c)
    # the final P left on chip is exactly symmetric and matches the Gram trace
    for i, (r, c) in enumerate(SMALL[:4]):
        x = f64(grads[i])
        x = x.T if r > c else x
        x0 = x / (np.linalg.norm(x) + EPS)
        p_ref = oracle.gram_trace(x0)[-1]["P"]
        p = plan.debug(7, i).cpu().numpy().astype(np.float64)
        assert np.array_equal(p, p.T)
        assert rel(p, p_ref) < 5e-3, (r, c, rel(p, p_ref))
    with pytest.raises(dmu.DmuError, match="on chip"):
        plan.debug(0, 0)


def test_onchip_many_matrices_per_cta(monkeypatch):
    """More matrices than SMs, mixed m: every CTA runs several matrices in
    turn, with buffers reused from a larger m to a smaller one."""
    shapes = [(128, 384), (48, 96), (96, 200)] * 110
    _, grads, _, _, o_a = _run(shapes, 73, monkeypatch, onchip=True)
    _, _, _, _, o_b = _run(shapes, 73, monkeypatch, onchip=False)
    for i in range(len(shapes)):
        assert torch.equal(o_a[i], o_b[i]), i
    for i in (0, 1, 2, 200, 328, 329):
        r, c = shapes[i]
        assert rel(f64(o_a[i]), oracle_o(grads[i], torch.zeros(r, c), 0.95)) < 5e-3


def test_onchip_cubic_coefficients(monkeypatch):
    cubic = (1.5, -0.5, 0.0)
    shapes = [(128, 512), (512, 128), (64, 200)]
    _, grads, _, _, outs = _run(shapes, 74, monkeypatch, onchip=True, steps=8, coeffs=cubic)
    for i, (r, c) in enumerate(shapes):
        g = f64(grads[i])
        o_ref = oracle.orthogonalize(g, cubic, 8, EPS)
        assert rel(f64(outs[i]), o_ref) < 5e-3, (r, c)


def test_autotune_per_class_and_bucket(tmp_path, monkeypatch):
    monkeypatch.delenv("DMU_ONCHIP", raising=False)
    shapes = [(128, 512)] * 40 + [(256, 1024)] * 20 + [(1024, 512)] * 3
    w = synth.custom("tune", shapes, seed=75)
    grads = synth.gradients(w, "cuda")
    weights = synth.weights(w, "cuda")
    w_ref = [x.clone() for x in weights]
    cache = str(tmp_path / "sched.txt")
    plan = dmu.Plan(shapes)
    plan.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    sch = plan.autotune(cache)
    assert set(sch["gram"]) == {128, 256, 512}
    assert set(sch["final"]) == {(128, 512), (256, 1024), (1024, 512)}
    lines = open(cache).read().splitlines()
    assert sum("/gram/" in l for l in lines) == 3 and sum("/final/" in l for l in lines) == 3
    # autotune leaves the caller's weights alone
    for a, b in zip(weights, w_ref):
        assert torch.equal(a, b)
    plan.step(grads, None, weights, beta=0.0, lr=0.02)
    ref = dmu.Plan(shapes)  # default schedules
    ref.step(grads, None, w_ref, beta=0.0, lr=0.02)
    torch.cuda.synchronize()
    for a, b in zip(weights, w_ref):
        assert torch.equal(a, b)  # every schedule gives the same bits
    # a second plan with the same shapes takes the cached choices untimed
    plan2 = dmu.Plan(shapes)
    plan2.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    assert plan2.autotune(cache) == sch
    assert open(cache).read().splitlines() == lines
    for p in (plan, ref, plan2):
        p.close()
