"""The seeded synthetic inputs (gram_newton_schulz_b200/synth.py) follow
their stated recipes: shapes and counts of every workload, dtypes,
determinism per matrix index, the spike's rank and scale, the per-matrix
log-uniform scale of the small-matrix swarm, and the weight distribution.
CPU only, on small draws."""
import math

import numpy as np
import pytest
import torch

from gram_newton_schulz_b200 import synth


def test_workload_shapes_and_counts():
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    assert w.count == 196 and w.dtype == "bf16" and w.dist == "spiked" and w.rank == 8
    per_layer = [(3584, 3584), (512, 3584), (512, 3584), (3584, 3584), (18944, 3584), (18944, 3584),
                 (3584, 18944)]
    assert list(w.shapes) == per_layer * 28
    assert w.elements() == 28 * sum(r * c for r, c in per_layer)
    assert synth.workload("qwen2.5-7b-layer-set-x4").count == 28
    u = synth.workload("uniform-64x512x2048")
    assert u.shapes == ((512, 2048),) * 64 and u.dist == "spiked" and u.var == pytest.approx(1e-3)
    s = synth.workload("small-swarm-4096")
    assert s.shapes == ((128, 512),) * 2048 + ((256, 1024),) * 2048 and s.dist == "logscaled"
    big = synth.workload("large-dense-24")
    assert big.shapes == ((8192, 8192),) * 16 + ((8192, 28672),) * 8 and big.rank == 32
    one = synth.workload("single-64x256-fp32")
    assert one.shapes == ((64, 256),) and one.dtype == "f32" and one.dist == "normal"
    for name in synth.WORKLOADS:
        assert synth.workload(name).name == name
    with pytest.raises(KeyError):
        synth.workload("no-such-workload")


def test_draws_are_deterministic_per_matrix():
    w = synth.custom("det", [(32, 64), (32, 64), (16, 48)], seed=9)
    a = synth.gradients(w)
    b = synth.gradients(w, indices=[2, 0])
    assert torch.equal(a[2], b[0]) and torch.equal(a[0], b[1])
    assert not torch.equal(a[0], a[1])  # same shape, different index, different draw
    assert a[0].dtype == torch.bfloat16
    wa, wb = synth.weights(w), synth.weights(w, indices=[1])
    assert torch.equal(wa[1], wb[0])
    assert not torch.equal(wa[0].float(), a[0].float())  # weights use their own streams


def test_spike_has_the_stated_rank_and_scale():
    rows, cols, rank, var = 256, 1024, 8, 1e-3
    w = synth.custom("spk", [(rows, cols)], seed=3, dist="spiked", var=var, rank=rank)
    x = synth.gradient(w, 0).double().numpy()
    s = np.linalg.svd(x, compute_uv=False)
    std = math.sqrt(var)
    # noise bulk: singular values of an N(0, std^2) matrix, at most std (sqrt(m) + sqrt(n))
    bulk = std * (math.sqrt(rows) + math.sqrt(cols))
    assert s[rank] < 1.2 * bulk
    # the spike's singular values: about 10 std sqrt(m n / r) each, far above the bulk
    spike = 10 * std * math.sqrt(rows * cols / rank)
    assert s[rank - 1] > 0.3 * spike > 3 * bulk
    # every entry of the spike has std 10 * std, so the total std is about sqrt(101) * std
    assert x.std() == pytest.approx(math.sqrt(101.0) * std, rel=0.15)


def test_logscaled_swarm_spans_three_decades():
    w = synth.custom("swarm", [(16, 32)] * 200, seed=4, dist="logscaled")
    scales = np.array([synth.gradient(w, i).float().std().item() for i in range(w.count)])
    assert scales.min() >= 1e-4 * 0.5 and scales.max() <= 1e-1 * 1.5
    logs = np.log10(scales)
    assert logs.max() - logs.min() > 2.5  # U(-4, -1) over 200 draws covers nearly 3 decades


def test_weights_are_n0_002():
    w = synth.custom("wt", [(512, 512)], seed=6)
    x = synth.weight(w, 0).float()
    assert x.mean().abs().item() < 1e-3
    assert x.std().item() == pytest.approx(0.02, rel=0.02)


def test_sample_indices_cover_every_bucket():
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    idx = synth.sample_indices(w)
    shapes = {w.shapes[i] for i in idx}
    assert shapes == set(w.shapes)
    by = {}
    for i, s in enumerate(w.shapes):
        by.setdefault(s, []).append(i)
    for s, ids in by.items():
        assert ids[0] in idx and ids[-1] in idx
    assert idx == synth.sample_indices(w)  # deterministic
