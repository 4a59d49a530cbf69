"""The orthogonalisation entry point on caller-supplied device matrices, and
coefficients other than the quintic ones (needs an sm_100a GPU).

`dmu_gram_ns_batched(plan, ptrs, ...)` with `ptrs != NULL` normalises the
given matrices itself (beta = 0, no momentum state) before the Gram
recursion; nothing from `dmu_momentum_normalize` is used.  Its input path
chooses 16-byte vector loads when every pointer is 16-byte aligned and every
row length is a multiple of 8, and scalar loads otherwise, so both are run
here: aligned tensors, the same values at a 2-byte offset, and ragged
shapes.  The result O (via `dmu_apply_update`'s out_o) must match the fp64
oracle's rectangular Newton-Schulz iteration on the same bf16 values
(DMuon page, section 2.2: the Gram-space recursion equals the rectangular
one; DeMuon page, Method 1: NS approximates msgn).

The `coeffs` argument is exercised with the cubic iteration
(a, b, c) = (1.5, -0.5, 0) over K = 8 steps, through both precision classes
(split bf16 for m < 1024, scaled fp16 at m = 1024).
"""
import numpy as np
import pytest
import torch

import oracle
from gram_newton_schulz_b200 import dmu, synth
from gpu_util import EPS, f64, rel

pytestmark = pytest.mark.gpu

ALIGNED = [(256, 1024), (1024, 256), (384, 384), (1024, 2048), (2048, 1024)]
RAGGED = [(300, 700), (700, 300), (130, 130), (1, 300)]
CUBIC = (1.5, -0.5, 0.0)


def _inputs(shapes, seed, offset_elems=0):
    """bf16 device matrices (spiked, like the layer-set recipe); with
    ``offset_elems`` > 0 each one is a view that starts that many elements
    into its own buffer, so its address is not 16-byte aligned."""
    w = synth.custom("inputs", shapes, seed=seed)
    src = synth.gradients(w, "cuda")
    if offset_elems == 0:
        return src
    out = []
    for x in src:
        buf = torch.zeros(x.numel() + 16, dtype=x.dtype, device=x.device)
        v = buf[offset_elems:offset_elems + x.numel()].view(x.shape)
        v.copy_(x)
        out.append(v)
    return out


def _orthogonalize_on_gpu(shapes, xs, coeffs=dmu.QUINTIC, steps=5):
    plan = dmu.Plan(shapes)
    plan.gram_ns_batched(xs, coeffs=coeffs, steps=steps)
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    plan.apply_update(None, lr=0.02, out_o=outs)
    torch.cuda.synchronize()
    assert plan.read_status() == 0
    return plan, outs


@pytest.mark.parametrize("shapes,offset", [(ALIGNED, 0), (ALIGNED, 1), (RAGGED, 0)],
                         ids=["aligned-vector", "misaligned-scalar", "ragged-scalar"])
def test_gram_ns_batched_on_device_matrices(shapes, offset):
    xs = _inputs(shapes, seed=61, offset_elems=offset)
    if offset:
        assert all(x.data_ptr() % 16 != 0 for x in xs)
    plan, outs = _orthogonalize_on_gpu(shapes, xs)
    inv = plan.debug(6).cpu().numpy().astype(np.float64)
    for i, (r, c) in enumerate(shapes):
        x = f64(xs[i])
        # the input path normalises with eps = 1e-7 (no momentum call made)
        assert inv[i] == pytest.approx(1.0 / (np.linalg.norm(x) + EPS), rel=2e-6), (r, c)
        o_ref = oracle.orthogonalize(x, oracle.QUINTIC, 5, EPS)
        e = rel(f64(outs[i]), o_ref)
        assert e < 2e-2, (r, c, e)
    plan.close()


def test_device_matrices_do_not_touch_momentum_state():
    """ptrs != NULL after a momentum call: the recursion runs on the given
    matrices, not on the image the momentum call left."""
    shapes = [(256, 1024), (512, 512)]
    grads = _inputs(shapes, seed=62)
    xs = _inputs(shapes, seed=63)
    plan = dmu.Plan(shapes)
    plan.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    plan.gram_ns_batched(xs, coeffs=dmu.QUINTIC, steps=5)
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    plan.apply_update(None, lr=0.02, out_o=outs)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        o_ref = oracle.orthogonalize(f64(xs[i]), oracle.QUINTIC, 5, EPS)
        assert rel(f64(outs[i]), o_ref) < 2e-2
    plan.close()


@pytest.mark.parametrize("prec", ["auto", "split3"])
def test_cubic_coefficients_eight_steps(prec):
    shapes = [(256, 1024), (1024, 256), (384, 384), (1024, 2048)]
    xs = _inputs(shapes, seed=64)
    plan = dmu.Plan(shapes, prec=prec)
    plan.gram_ns_batched(xs, coeffs=CUBIC, steps=8)
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    plan.apply_update(None, lr=0.02, out_o=outs)
    torch.cuda.synchronize()
    assert plan.read_status() == 0
    for i, (r, c) in enumerate(shapes):
        x = f64(xs[i])
        o_ref = oracle.orthogonalize(x, CUBIC, 8, EPS)
        e = rel(f64(outs[i]), o_ref)
        assert e < 2e-2, (prec, r, c, e)
        # the cubic and the quintic maps differ: the kernels used `coeffs`
        o_q = oracle.orthogonalize(x, oracle.QUINTIC, 5, EPS)
        assert rel(o_ref, o_q) > 5 * e, (r, c)
    plan.close()
