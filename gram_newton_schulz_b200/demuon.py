"""DeMuon: decentralised Muon over a communication graph, with N agents
simulated on one GPU.

Source: DeMuon technical summary, "Methodology", 1. DeMuon.  Each agent i
keeps, per weight matrix:
* a local momentum estimate M_i, an exponential moving average of its
  stochastic gradients;
* a tracked global-gradient estimate V_i, mixed from its neighbours;
* an iterate X_i, mixed from its neighbours' updates, each of which applies
  msgn to the tracked gradient.

With mixing weights w_ij (row i = the weights agent i applies), one
iteration is:

    M_i' = (1 - theta) M_i + theta G_i
    V_i' = sum_j w_ij V_j + M_i' - M_i
    X_i' = sum_j w_ij (X_j - eta msgn(V_j'))

One iteration is five launch groups on the current stream:
1. `dmu_demuon_track`: momentum, tracking, and the bf16 msgn input.
2.–4. One `dmu.Plan` over all agents' matrices: `momentum_normalize` (no
   momentum, beta 0), `gram_ns_batched`, and `apply_update` writing only O.
   msgn is thus the same batched Gram Newton-Schulz path as the Muon step.
5. `dmu_demuon_mix`: the gossip mixing of X - eta O.

Host-simulated agents: the "communication"
is the mixing kernel reading every agent's arrays on one GPU.  On a real
graph each agent would receive only its neighbours' V and X - eta O.

State layout: per agent, one flat array per quantity with every matrix at a
256-byte-aligned offset (the same offsets in every agent), so the
elementwise kernels see each agent's state as one vector.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

from . import dmu

ALIGN = 128  # elements; every matrix view starts on a 256-byte boundary (bf16) / 512 (fp32)


def mixing_matrix(topology: str, n: int) -> List[List[float]]:
    """Doubly stochastic mixing weights (row i: what agent i applies).

    * complete: w_ij = 1/n;
    * ring: 1/3 on i-1, i, i+1 (n >= 3; n <= 2 is the complete graph);
    * exponential: i receives from itself and from i - 2^k (mod n) for every
      2^k < n, with equal weights.
    """
    if n < 1:
        raise ValueError("n must be >= 1")
    if topology == "complete" or n == 1 or (topology == "ring" and n == 2):
        return [[1.0 / n] * n for _ in range(n)]
    rows = [[0.0] * n for _ in range(n)]
    if topology == "ring":
        for i in range(n):
            for j in ((i - 1) % n, i, (i + 1) % n):
                rows[i][j] = 1.0 / 3.0
        return rows
    if topology == "exponential":
        offsets, h = [0], 1
        while h < n:
            offsets.append(h)
            h *= 2
        for i in range(n):
            for h in offsets:
                rows[i][(i - h) % n] += 1.0 / len(offsets)
        return rows
    raise ValueError(f"unknown topology {topology!r}")


class DeMuon:
    """N simulated agents, each with the same list of matrix shapes."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], n_agents: int, *, topology: str = "ring",
                 mix: Optional[Sequence[Sequence[float]]] = None, theta: float = 0.1, eta: float = 0.02,
                 coeffs=dmu.QUINTIC, steps: int = 5, eps: float = 1e-7, device=None):
        import torch
        if not 1 <= n_agents <= dmu.DEMUON_MAX_AGENTS:
            raise ValueError(f"n_agents must be in [1, {dmu.DEMUON_MAX_AGENTS}]")
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.n = int(n_agents)
        self.mix = [list(map(float, row)) for row in (mix if mix is not None else mixing_matrix(topology, self.n))]
        self.theta, self.eta, self.coeffs, self.steps, self.eps = float(theta), float(eta), coeffs, steps, eps
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.offset = []
        off = 0
        for r, c in self.shapes:
            self.offset.append(off)
            off += (r * c + ALIGN - 1) // ALIGN * ALIGN
        self.numel = max(off, ALIGN)
        z32 = lambda: [torch.zeros(self.numel, dtype=torch.float32, device=self.device) for _ in range(self.n)]  # noqa: E731
        z16 = lambda: [torch.zeros(self.numel, dtype=torch.bfloat16, device=self.device) for _ in range(self.n)]  # noqa: E731
        self.g = z16()
        self.m = z32()
        self.v = [z32(), z32()]
        self.vb = z16()
        self.x = [z32(), z32()]
        self.o = z32()
        self.cur = 0
        self.plan = dmu.Plan(self.shapes * self.n, dtype="bf16", device=self.device)
        self._vb_views = [self.view(self.vb, a, k) for a in range(self.n) for k in range(len(self.shapes))]
        self._o_views = [self.view(self.o, a, k) for a in range(self.n) for k in range(len(self.shapes))]

    def view(self, flats, agent: int, k: int):
        r, c = self.shapes[k]
        o = self.offset[k]
        return flats[agent][o:o + r * c].view(r, c)

    # user-facing views of the current state
    def grad(self, agent: int, k: int):
        """Agent's gradient buffer for matrix k (bf16): write G_i here before step()."""
        return self.view(self.g, agent, k)

    def iterate(self, agent: int, k: int):
        return self.view(self.x[self.cur], agent, k)

    def momentum(self, agent: int, k: int):
        return self.view(self.m, agent, k)

    def tracked(self, agent: int, k: int):
        return self.view(self.v[self.cur], agent, k)

    def msgn_out(self, agent: int, k: int):
        """O_j = msgn(V_j') of the last step (fp32)."""
        return self.view(self.o, agent, k)

    def reset_tracking(self):
        """V_i = M_i, the start of the tracking recursion."""
        for a in range(self.n):
            self.v[self.cur][a].copy_(self.m[a])

    def step(self, events=None):
        """One iteration on the current stream.  ``events``: optional four CUDA
        events recorded before tracking, before msgn, before mixing and at the
        end."""
        nxt = 1 - self.cur
        if events is not None:
            events[0].record()
        dmu.demuon_track(self.mix, self.theta, self.g, self.m, self.v[self.cur], self.v[nxt], self.vb)
        if events is not None:
            events[1].record()
        self.plan.momentum_normalize(self._vb_views, None, beta=0.0, eps=self.eps)
        self.plan.gram_ns_batched(None, self.coeffs, self.steps)
        self.plan.apply_update(None, lr=0.0, out_o=self._o_views)
        if events is not None:
            events[2].record()
        dmu.demuon_mix(self.mix, self.eta, self.x[self.cur], self.o, self.x[nxt])
        if events is not None:
            events[3].record()
        self.cur = nxt

    def close(self):
        if self.plan is not None:
            self.plan.close()
            self.plan = None
