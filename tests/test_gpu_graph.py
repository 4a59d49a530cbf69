"""A steady-state step (momentum, Gram recursion, fused update) is
capturable into a CUDA graph. Its replay gives the same bits as eager
launches: the library only enqueues kernels once its pointer tables are
uploaded."""
import pytest
import torch

from gram_newton_schulz_b200 import dmu, synth

pytestmark = pytest.mark.gpu


def _state(w, dev):
    grads = synth.gradients(w, dev)
    weights = synth.weights(w, dev)
    moms = [torch.zeros(s, dtype=torch.float32, device=dev) for s in w.shapes]
    return grads, moms, weights


def test_graph_replay_matches_eager_bitwise():
    shapes = [(512, 2048), (2048, 512), (300, 300), (1024, 4096), (128, 512)]
    w = synth.custom("graph-check", shapes, seed=21)
    dev = torch.device("cuda", 0)
    ga, ma, wa = _state(w, dev)
    gb, mb, wb = _state(w, dev)
    pa = dmu.Plan(shapes, device=dev)
    pb = dmu.Plan(shapes, device=dev)
    for _ in range(2):
        pa.step(ga, ma, wa, beta=0.9, lr=0.02)
    pb.step(gb, mb, wb, beta=0.9, lr=0.02)  # uploads the pointer tables outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pb.step(gb, mb, wb, beta=0.9, lr=0.02)
    g.replay()
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        assert torch.equal(wa[i], wb[i]), i
        assert torch.equal(ma[i], mb[i]), i
    assert pa.read_status() == 0 and pb.read_status() == 0
    del g
    pa.close()
    pb.close()
