"""DeMuon on the GPU (N simulated agents) against the fp64 oracle
(oracle/demuon.py).

Each step is checked one step at a time from the device's own previous
state, so errors do not compound between steps:

* M' and V': fp32 against fp64, relative Frobenius error <= 1e-6;
* O = msgn(V'), with the oracle applied to the same bf16 rounding of V' that
  the device feeds its Gram Newton-Schulz path: <= 2e-2, the bound of the
  Muon step;
* X' = sum_j w_ij (X_j - eta O_j): within eta * 2e-2 * max_j ||O_j||_F
  (the O error, mixed by weights that sum to 1), plus fp32 rounding.

The elementwise kernels are also checked on their own, with a ragged
element count (4k + 3) so the scalar tail runs. Two identical runs must be
bitwise equal.
"""
import numpy as np
import pytest
import torch

from gram_newton_schulz_b200 import demuon, dmu
from oracle import demuon as odm

pytestmark = pytest.mark.gpu

SHAPES = [(64, 256), (96, 96), (200, 72)]


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def _grads(seed, n):
    g = torch.Generator().manual_seed(seed)
    out = []
    for a in range(n):
        row = []
        for r, c in SHAPES:
            noise = torch.randn(r, c, generator=g) * 1e-2
            u, v = torch.randn(r, 4, generator=g), torch.randn(4, c, generator=g)
            row.append((noise + 0.05 * (u @ v) / 2.0).to(torch.bfloat16))
        out.append(row)
    return out


def _state(dm, getter):
    return [[getter(a, k).detach().double().cpu().numpy() for k in range(len(SHAPES))] for a in range(dm.n)]


@pytest.mark.parametrize("n,topology", [(4, "ring"), (4, "exponential"), (5, "complete"), (1, "ring")])
def test_demuon_steps_match_oracle(n, topology):
    theta, eta = 0.1, 0.02
    dm = demuon.DeMuon(SHAPES, n, topology=topology, theta=theta, eta=eta, device="cuda")
    w = np.array(dm.mix, dtype=np.float64)
    g0 = torch.Generator().manual_seed(100 + n)
    for a in range(n):
        for k, (r, c) in enumerate(SHAPES):
            dm.iterate(a, k).copy_(torch.randn(r, c, generator=g0) * 0.02)
    for step in range(3):
        grads = _grads(1000 * n + step, n)
        for a in range(n):
            for k in range(len(SHAPES)):
                dm.grad(a, k).copy_(grads[a][k])
        x0, m0, v0 = _state(dm, dm.iterate), _state(dm, dm.momentum), _state(dm, dm.tracked)
        g64 = [[grads[a][k].double().numpy() for k in range(len(SHAPES))] for a in range(n)]
        dm.step()
        torch.cuda.synchronize()
        x1, m1, v1 = _state(dm, dm.iterate), _state(dm, dm.momentum), _state(dm, dm.tracked)
        o1 = _state(dm, dm.msgn_out)
        xr, mr, vr, orf = odm.demuon_step(x0, m0, v0, g64, w, theta=theta, eta=eta, msgn_input=bf16_round)
        for a in range(n):
            for k in range(len(SHAPES)):
                what = (step, a, SHAPES[k])
                assert rel(m1[a][k], mr[a][k]) <= 1e-6, what
                assert rel(v1[a][k], vr[a][k]) <= 1e-6, what
                assert rel(o1[a][k], orf[a][k]) <= 2e-2, (what, rel(o1[a][k], orf[a][k]))
        for k in range(len(SHAPES)):
            o_max = max(np.linalg.norm(orf[j][k]) for j in range(n))
            for a in range(n):
                err = np.linalg.norm(x1[a][k] - xr[a][k])
                assert err <= 2e-2 * eta * o_max + 1e-6 * np.linalg.norm(xr[a][k]), (step, a, k, err)
    assert dm.plan.read_status() == 0
    dm.close()


def test_demuon_is_deterministic():
    outs = []
    for _ in range(2):
        dm = demuon.DeMuon(SHAPES, 3, topology="ring", device="cuda")
        grads = _grads(7, 3)
        for step in range(2):
            for a in range(3):
                for k in range(len(SHAPES)):
                    dm.grad(a, k).copy_(grads[a][k])
            dm.step()
        torch.cuda.synchronize()
        outs.append([t.clone() for t in dm.x[dm.cur]] + [t.clone() for t in dm.v[dm.cur]])
        dm.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_elementwise_kernels_with_ragged_tail():
    n, numel, theta, eta = 3, 4 * 1000 + 3, 0.25, 0.1
    w = odm.mixing_matrix("exponential", n)
    g = torch.Generator().manual_seed(9)
    dev = "cuda"
    grads = [torch.randn(numel, generator=g).to(torch.bfloat16).to(dev) for _ in range(n)]
    m = [torch.randn(numel, generator=g).to(dev) for _ in range(n)]
    v = [torch.randn(numel, generator=g).to(dev) for _ in range(n)]
    x = [torch.randn(numel, generator=g).to(dev) for _ in range(n)]
    m0 = [t.double().cpu().numpy()[None, :] for t in m]
    v0 = [t.double().cpu().numpy()[None, :] for t in v]
    x0 = [t.double().cpu().numpy()[None, :] for t in x]
    g64 = [t.double().cpu().numpy()[None, :] for t in grads]
    v_out = [torch.empty(numel, device=dev) for _ in range(n)]
    vb = [torch.empty(numel, dtype=torch.bfloat16, device=dev) for _ in range(n)]
    dmu.demuon_track(w.tolist(), theta, grads, m, v, v_out, vb)
    xr, mr, vr, orf = odm.demuon_step([[t] for t in x0], [[t] for t in m0], [[t] for t in v0],
                                      [[t] for t in g64], w, theta=theta, eta=eta)
    o_dev = [torch.from_numpy(orf[j][0][0]).float().to(dev) for j in range(n)]
    x_out = [torch.empty(numel, device=dev) for _ in range(n)]
    dmu.demuon_mix(w.tolist(), eta, x, o_dev, x_out)
    torch.cuda.synchronize()
    for i in range(n):
        assert rel(m[i].double().cpu().numpy(), mr[i][0][0]) <= 1e-6
        assert rel(v_out[i].double().cpu().numpy(), vr[i][0][0]) <= 1e-6
        assert torch.equal(vb[i], v_out[i].to(torch.bfloat16))  # the msgn input is bf16(V') exactly
        assert rel(x_out[i].double().cpu().numpy(), xr[i][0][0]) <= 1e-6
        # the last three elements come from the scalar tail
        tail = slice(numel - 3, numel)
        np.testing.assert_allclose(v_out[i].double().cpu().numpy()[tail], vr[i][0][0][tail], rtol=1e-5, atol=1e-6)
