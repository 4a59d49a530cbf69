"""Helpers shared by the GPU tests: run the CUDA path through the C ABI and
bring sampled results back to the host for the fp64 oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from gram_newton_schulz_b200 import dmu, synth

LR = 0.02
BETA = 0.95
EPS = 1e-7


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp32 tensor."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def rel(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def run_step(w: synth.Workload, prec="auto", steps=5, dev="cuda", keep=None):
    """Run one full Muon step (momentum from zero) on the GPU for ``w``.

    Returns a dict with the plan, the gradients, W after the step, momenta
    after, and -- for the matrices in ``keep`` (default: all) -- W before
    the step and O (fp32, W's orientation); other entries are None.
    """
    grads = synth.gradients(w, dev)
    wdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    weights = synth.weights(w, dev)
    keep = set(range(w.count)) if keep is None else set(keep)
    w_before = [x.clone() if i in keep else None for i, x in enumerate(weights)]
    moms = [torch.zeros(s, dtype=torch.float32, device=dev) for s in w.shapes]
    m_before = [torch.zeros(s, dtype=torch.float32) if i in keep else None for i, s in enumerate(w.shapes)]
    outs = [torch.empty(s, dtype=torch.float32, device=dev) if i in keep else None
            for i, s in enumerate(w.shapes)]
    plan = dmu.Plan(w.shapes, dtype=w.dtype, prec=prec)
    plan.momentum_normalize(grads, moms, beta=w.beta, eps=EPS)
    plan.gram_ns_batched(None, dmu.QUINTIC, steps)
    plan.apply_update(weights, lr=w.lr, out_o=outs)
    torch.cuda.synchronize()
    assert weights[0].dtype == wdt
    return dict(plan=plan, grads=grads, w_before=w_before, w_after=weights, m_before=m_before,
                m_after=moms, o=outs)


def oracle_o(grad: torch.Tensor, m_prev: torch.Tensor, beta: float, steps: int = 5) -> np.ndarray:
    m = oracle.momentum(f64(m_prev), f64(grad), beta)
    return oracle.orthogonalize(m, oracle.QUINTIC, steps, EPS)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_update_within_ulp(w_before, w_after, o, rows, cols, lr):
    """W_new must equal bf16(W_old - lr * scale * O_gpu) to within one bf16
    ulp of the result, plus the fp32 rounding of the two terms (which is
    what remains when W_old and lr*scale*O nearly cancel).  Returns the
    worst ratio of the difference to that bound (<= 1 passes)."""
    scale = math.sqrt(max(1.0, rows / cols))
    delta = (-lr * scale) * o
    expect = (w_before.float() + delta).to(torch.bfloat16)
    got = f64(w_after)
    exp = f64(expect)
    diff = np.abs(got - exp)
    bound = bf16_ulp(exp) + 2.0 ** -22 * (np.abs(f64(w_before)) + np.abs(f64(delta)))
    return float(np.max(diff / bound))
