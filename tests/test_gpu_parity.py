"""CUDA path vs the fp64 oracle, through the C ABI (needs an sm_100a GPU).

Stage checks isolate each kernel:
  * K = 0: G0 = s^2 X X^T (SYRK, wide = K-major, tall = MN-major operands)
    and O = I X0 (final GEMM, wide = MN-major B, tall = K-major B);
  * K = 1, 2: R, T, G, P after one and two steps against the oracle's
    Gram-space trace (DMuon page, section 2.2);
  * full steps: O against the rectangular oracle within 2e-2 relative
    Frobenius error (bf16 path; tighter for SPLIT3), the fused W update
    within one bf16 ulp of bf16(W - lr*scale*O), momentum state, exact
    symmetry of every Gram-space output, determinism, edge cases.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gram_newton_schulz_b200 import dmu, synth
from gpu_util import BETA, EPS, LR, check_update_within_ulp, f64, oracle_o, rel, run_step

pytestmark = pytest.mark.gpu

MIXED = [(128, 512), (512, 128), (256, 256), (200, 520), (520, 200), (64, 300), (300, 64),
         (130, 1030), (1030, 130), (384, 384), (136, 1000)]


def _plan_inputs(shapes, seed, dist="spiked", dtype="bf16", prec="split3"):
    w = synth.custom("t", shapes, seed=seed, dist=dist, dtype=dtype)
    grads = synth.gradients(w, "cuda")
    plan = dmu.Plan(w.shapes, dtype=dtype, prec=prec)
    return w, grads, plan


@pytest.mark.parametrize("prec", ["fast", "split3"])
def test_syrk_and_final_gemm_k0(prec):
    w, grads, plan = _plan_inputs(MIXED, 11, prec=prec)
    plan.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    plan.gram_ns_batched(None, dmu.QUINTIC, 0)
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in w.shapes]
    plan.apply_update(None, lr=LR, out_o=outs)
    inv = plan.debug(6).cpu().numpy().astype(np.float64)
    isc = plan.debug(9).cpu().numpy().astype(np.float64)
    for i, (r, c) in enumerate(w.shapes):
        x = f64(grads[i])
        nrm = np.linalg.norm(x)
        assert inv[i] == pytest.approx(1.0 / (nrm + EPS), rel=2e-6)
        # the image is M = G in fp16 at scale 2^e; a plan's first call picks
        # 2^e ||M|| in (2^11, 2^12]
        assert np.log2(isc[i]) == np.round(np.log2(isc[i])) and 2 ** 11 < isc[i] * nrm <= 2 ** 12
        mb = plan.debug(5, i).cpu().numpy()
        np.testing.assert_array_equal(mb, (x * isc[i]).astype(np.float16).astype(np.float64) / isc[i])
        xo = x.T if r > c else x
        g_ref = (xo @ xo.T) * float(inv[i]) ** 2
        g = plan.debug(0, i).cpu().numpy().astype(np.float64)
        assert np.array_equal(g, g.T), f"G0 not exactly symmetric for {r}x{c}"
        assert rel(g, g_ref) < 2e-5, (r, c, rel(g, g_ref))
        # K = 0: P = I, so O = X0 in W's orientation
        o = f64(outs[i])
        assert rel(o, x * float(inv[i])) < 1e-5, (r, c, rel(o, x * float(inv[i])))


@pytest.mark.parametrize("prec,tol", [("split3", 2e-4), ("split2", 2e-2), ("fast", 3e-2)])
def test_gram_intermediates_k1_k2(prec, tol):
    shapes = [(128, 512), (512, 128), (256, 700), (300, 300)]
    w, grads, plan = _plan_inputs(shapes, 12, prec=prec)
    plan.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    inv = plan.debug(6).cpu().numpy().astype(np.float64)
    traces = []
    for i, (r, c) in enumerate(shapes):
        x = f64(grads[i])
        xo = x.T if r > c else x
        traces.append(oracle.gram_trace(xo * float(inv[i])))
    # one step: R_0 and P_1 = a I + R_0 (buffer A)
    plan.gram_ns_batched(None, dmu.QUINTIC, 1)
    for i in range(len(shapes)):
        r0 = plan.debug(1, i).cpu().numpy()
        p1 = plan.debug(7, i).cpu().numpy()
        _assert_symmetric(p1)
        assert rel(r0, traces[i][0]["R"]) < tol, ("R0", shapes[i], rel(r0, traces[i][0]["R"]))
        assert rel(p1, traces[i][0]["P"]) < tol, ("P1", shapes[i], rel(p1, traces[i][0]["P"]))
    # two steps: G_1, T_0, R_1, P_2
    plan.gram_ns_batched(None, dmu.QUINTIC, 2)
    for i in range(len(shapes)):
        tr = traces[i]
        got = {k: plan.debug(j, i).cpu().numpy() for k, j in (("G", 0), ("R", 1), ("T", 2), ("P", 7))}
        for k in got:
            _assert_symmetric(got[k], (k, shapes[i]))
        assert rel(got["T"], tr[0]["T"]) < tol, ("T0", shapes[i], rel(got["T"], tr[0]["T"]))
        assert rel(got["G"], tr[1]["G"]) < tol, ("G1", shapes[i], rel(got["G"], tr[1]["G"]))
        assert rel(got["R"], tr[1]["R"]) < tol, ("R1", shapes[i], rel(got["R"], tr[1]["R"]))
        assert rel(got["P"], tr[1]["P"]) < tol, ("P2", shapes[i], rel(got["P"], tr[1]["P"]))


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _mirrored(d):
    """A symmetric product as the kernels store it: the upper triangle, and
    its mirror image below (whether the lower blocks are written or read
    back as transposed upper blocks)."""
    return np.triu(d) + np.triu(d, 1).T


def _assert_symmetric(x, what=None):
    assert np.array_equal(x, x.T), what


def _emul_product(a, b, prec):
    """The half-stored bf16 product each precision mode issues, in fp64 from
    the GPU's own operands (hi + lo pairs)."""
    ah, bh = _bf16(a), _bf16(b)
    al, bl = _bf16(a - ah), _bf16(b - bh)
    d = ah @ bh
    if prec in ("split2",):
        d = d + al @ bh
    if prec in ("split3",):
        d = d + ah @ bl + al @ bh
    return _mirrored(d)


@pytest.mark.parametrize("prec", ["fast", "split2", "split3"])
def test_products_match_emulation(prec):
    """Each Gram-space product against an fp64 emulation of exactly the MMA
    terms the mode issues, on the operands read back from the GPU: checks
    the kernel, not the method's conditioning."""
    a, b, c = dmu.QUINTIC
    shapes = [(128, 512), (384, 384), (520, 200), (300, 700)]
    w, grads, plan = _plan_inputs(shapes, 13, prec=prec)
    plan.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    plan.gram_ns_batched(None, dmu.QUINTIC, 2)
    for i in range(len(shapes)):
        d = {k: plan.debug(j, i).cpu().numpy().astype(np.float64) for k, j in
             (("G", 0), ("R", 1), ("PA", 3), ("PB", 7))}  # P_2, the final P (fp16 pair)
        r_ref = b * d["G"] + c * _emul_product(d["G"], d["G"], prec)
        # fp32 accumulation and hi/lo storage leave ~1e-5; a wrong term is >= 1e-3
        tol = 1e-4
        if prec == "fast":  # R is stored as hi only: a few elements may round the other way
            r_ref = _bf16(r_ref)
            tol = 1e-3
        assert rel(d["R"], r_ref) < tol, ("R", shapes[i], rel(d["R"], r_ref))
        rp = _emul_product(d["PA"], d["R"], prec) if prec == "split2" else _emul_product(d["R"], d["PA"], prec)
        p_ref = a * d["PA"] + rp
        assert rel(d["PB"], p_ref) < 1e-4, ("P", shapes[i], rel(d["PB"], p_ref))


@pytest.mark.parametrize("prec", ["tf32", "f16"])
def test_tf32_f16_products_accuracy(prec):
    """TF32 and scaled-fp16 modes: each product within their 10-bit operand
    precision of the exact product of the GPU's own operands (a bf16
    product would be ~8x further off)."""
    a, b, c = dmu.QUINTIC
    shapes = [(256, 1024), (300, 300), (1100, 200)]
    w, grads, plan = _plan_inputs(shapes, 14, prec=prec)
    plan.momentum_normalize(grads, None, beta=0.0, eps=EPS)
    plan.gram_ns_batched(None, dmu.QUINTIC, 2)
    for i in range(len(shapes)):
        d = {k: plan.debug(j, i).cpu().numpy().astype(np.float64) for k, j in
             (("G", 0), ("R", 1), ("PA", 3), ("P", 7))}
        store = _mirrored
        gg = d["G"] @ d["G"]
        r_ref = b * d["G"] + c * store(gg)
        assert rel(d["R"], r_ref) < 1e-3, ("R", shapes[i], rel(d["R"], r_ref))
        rp = d["R"] @ d["PA"]
        p_ref = a * d["PA"] + store(rp)
        assert rel(d["P"], p_ref) < 1e-3, ("P", shapes[i], rel(d["P"], p_ref))
        _assert_symmetric(d["P"])


@pytest.mark.parametrize("prec", ["tf32", "f16", "auto"])
def test_full_step_large_m(prec):
    shapes = [(1024, 4096), (4096, 1024), (1536, 1536), (1024, 1024), (512, 2048)]
    w = synth.custom("large", shapes, seed=23)
    res = run_step(w, prec=prec)
    for i, (r, c) in enumerate(w.shapes):
        o_ref = oracle_o(res["grads"][i], res["m_before"][i], w.beta)
        e = rel(f64(res["o"][i]), o_ref)
        assert e < (2e-2 if min(r, c) < 1024 else 1e-2), (r, c, e)
        u = check_update_within_ulp(res["w_before"][i], res["w_after"][i], res["o"][i], r, c, w.lr)
        assert u <= 1.0, (r, c, u)


@pytest.mark.parametrize("prec,tol", [("auto", 2e-2), ("split3", 5e-3)])
@pytest.mark.parametrize("dist", ["spiked", "normal"])
def test_full_step_mixed_shapes(prec, tol, dist):
    w = synth.custom("mixed", MIXED, seed=21, dist=dist, var=1e-3 if dist == "spiked" else 1.0)
    res = run_step(w, prec=prec)
    worst = 0.0
    for i, (r, c) in enumerate(w.shapes):
        o_ref = oracle_o(res["grads"][i], res["m_before"][i], w.beta)
        e = rel(f64(res["o"][i]), o_ref)
        worst = max(worst, e)
        assert e < tol, (r, c, e)
        u = check_update_within_ulp(res["w_before"][i], res["w_after"][i], res["o"][i], r, c, w.lr)
        assert u <= 1.0, (r, c, u)
        np.testing.assert_array_equal(res["m_after"][i].cpu().numpy(), res["grads"][i].float().cpu().numpy())
    assert worst < tol


def test_momentum_two_steps():
    shapes = [(256, 1024), (1024, 256)]
    w = synth.custom("mom", shapes, seed=31)
    dev = "cuda"
    g1 = synth.gradients(w, dev)
    w2 = synth.custom("mom2", shapes, seed=32)
    g2 = synth.gradients(w2, dev)
    moms = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
    weights = synth.weights(w, dev)
    outs = [torch.empty(s, dtype=torch.float32, device=dev) for s in shapes]
    plan = dmu.Plan(shapes)
    plan.step(g1, moms, weights, beta=BETA, lr=LR)
    plan.step(g2, moms, weights, beta=BETA, lr=LR, out_o=outs)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        m_ref = BETA * f64(g1[i]) + f64(g2[i])
        # one fp32 multiply-add: error within 2^-23 of the terms' magnitudes
        bound = 2.0 ** -23 * (BETA * np.abs(f64(g1[i])) + np.abs(f64(g2[i]))) + 1e-30
        assert np.all(np.abs(moms[i].cpu().numpy() - m_ref) <= bound)
        o_ref = oracle.orthogonalize(f64(moms[i]), oracle.QUINTIC, 5, EPS)
        # M is no longer bf16-exact; its bf16 image feeds the Gram kernels
        assert rel(f64(outs[i]), o_ref) < 2e-2


def test_fp32_path_single_64x256():
    w = synth.workload("single-64x256-fp32")
    res = run_step(w)
    o_ref = oracle_o(res["grads"][0], res["m_before"][0], w.beta)
    assert rel(f64(res["o"][0]), o_ref) < 1e-4
    d = f64(res["w_after"][0]) - (f64(res["w_before"][0]) - w.lr * f64(res["o"][0]))
    assert np.max(np.abs(d)) < 1e-6


@pytest.mark.parametrize("shapes", [[(64, 256), (256, 64), (100, 333), (333, 100), (1, 300), (300, 1), (7, 7)]])
def test_fp32_path_shapes(shapes):
    w = synth.custom("f32", shapes, seed=41, dtype="f32", dist="normal", var=1.0)
    res = run_step(w)
    for i, (r, c) in enumerate(shapes):
        o_ref = oracle_o(res["grads"][i], res["m_before"][i], w.beta)
        assert rel(f64(res["o"][i]), o_ref) < 1e-4, (r, c)


def test_edge_shapes_bf16():
    shapes = [(1, 300), (300, 1), (1, 1), (3, 5), (129, 1001), (1001, 129), (8, 8), (257, 257)]
    w = synth.custom("edge", shapes, seed=51, dist="normal", var=1.0)
    res = run_step(w, prec="split3")
    for i, (r, c) in enumerate(shapes):
        o_ref = oracle_o(res["grads"][i], res["m_before"][i], w.beta)
        assert rel(f64(res["o"][i]), o_ref) < 2e-2, (r, c)
        assert check_update_within_ulp(res["w_before"][i], res["w_after"][i], res["o"][i], r, c, w.lr) <= 1.0


def test_zero_gradient_gives_zero_update():
    shapes = [(128, 512), (512, 128)]
    grads = [torch.zeros(s, dtype=torch.bfloat16, device="cuda") for s in shapes]
    weights = [torch.ones(s, dtype=torch.bfloat16, device="cuda") for s in shapes]
    outs = [torch.full(s, 7.0, dtype=torch.float32, device="cuda") for s in shapes]
    plan = dmu.Plan(shapes)
    plan.step(grads, None, weights, out_o=outs)
    torch.cuda.synchronize()
    assert plan.read_status() == 0
    for i in range(2):
        assert torch.all(outs[i] == 0)
        assert torch.all(weights[i] == 1)


def test_nonfinite_gradient_sets_status():
    shapes = [(128, 512), (256, 256)]
    w = synth.custom("nan", shapes, seed=61)
    grads = synth.gradients(w, "cuda")
    grads[1][3, 5] = float("nan")
    plan = dmu.Plan(shapes)
    plan.momentum_normalize(grads, None, beta=0.0)
    assert plan.read_status() & dmu.FLAG_NONFINITE
    assert plan.read_status() == 0  # cleared by the read
    grads[1][3, 5] = 0.0
    plan.momentum_normalize(grads, None, beta=0.0)
    plan.gram_ns_batched(None)
    assert plan.read_status() == 0


def test_bounded_wait_selftest_reports_timeout():
    plan = dmu.Plan([(128, 128)])
    plan.debug(8, 2000)  # a kernel waits 2 ms on a barrier nothing completes
    assert plan.read_status() & dmu.FLAG_TIMEOUT
    # the context stays usable
    w = synth.custom("after", [(128, 128)], seed=71)
    g = synth.gradients(w, "cuda")
    plan.momentum_normalize(g, None, beta=0.0)
    plan.gram_ns_batched(None)
    outs = [torch.empty((128, 128), dtype=torch.float32, device="cuda")]
    plan.apply_update(None, out_o=outs)
    assert plan.read_status() == 0
    assert rel(f64(outs[0]), oracle_o(g[0], torch.zeros(128, 128), 0.0)) < 2e-2


def test_deterministic():
    w = synth.custom("det", MIXED[:6], seed=81)
    a = run_step(w)
    b = run_step(w)
    for i in range(w.count):
        assert torch.equal(a["o"][i], b["o"][i])
        assert torch.equal(a["w_after"][i], b["w_after"][i])


def test_plan_errors_on_gpu():
    shapes = [(128, 256)]
    plan = dmu.Plan(shapes)
    with pytest.raises(dmu.DmuError) as ei:
        plan.apply_update(None, out_o=[torch.empty((128, 256), device="cuda")])
    assert ei.value.status == dmu.ERR_NOT_PLANNED
    with pytest.raises(dmu.DmuError) as ei:
        plan.gram_ns_batched(None)
    assert ei.value.status == dmu.ERR_NOT_PLANNED
    lib = dmu.load()
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    import ctypes
    st = lib.dmu_set_workspace(plan.handle, ctypes.c_void_p(small.data_ptr()), 256)
    assert st == dmu.ERR_WORKSPACE
    other = dmu.Shape * 1
    bad = other(dmu.Shape(128, 257))
    co = (ctypes.c_float * 3)(*dmu.QUINTIC)
    st = lib.dmu_gram_ns_batched(plan.handle, None, ctypes.cast(bad, ctypes.c_void_p), 1,
                                 ctypes.cast(co, ctypes.c_void_p), 5, None)
    assert st == dmu.ERR_NOT_PLANNED


@pytest.mark.parametrize("prec", ["auto", "split3"])
def test_half_and_full_storage_agree(prec, monkeypatch):
    """Half-stored symmetric matrices (upper blocks only, lower blocks read
    transposed) must give bitwise the results of fully mirrored storage."""
    shapes = [(1100, 3000), (3000, 1100), (520, 200), (700, 700)]
    w = synth.custom("half", shapes, seed=31)
    monkeypatch.setenv("DMU_HALF", "1")
    a = run_step(w, prec=prec)
    monkeypatch.setenv("DMU_HALF", "0")
    b = run_step(w, prec=prec)
    for i in range(w.count):
        assert torch.equal(a["o"][i], b["o"][i]), shapes[i]
        assert torch.equal(a["w_after"][i], b["w_after"][i]), shapes[i]


@pytest.mark.parametrize("prec", ["auto", "split3", "tf32"])
def test_cta_pair_and_single_cta_agree(prec, monkeypatch):
    """The CTA-pair kernels (256 x 256 tiles, cta_group::2, with 3, 2 or 1 K
    atoms per stage; 256 x 512 tiles), and the single-CTA kernels (128 x 256
    and 128 x 128 tiles) accumulate every element over K in the same order,
    so they must give bitwise-equal results."""
    shapes = [(1100, 3000), (3000, 1100), (512, 2048), (520, 200), (384, 384), (128, 512), (100, 300)]
    w = synth.custom("pair", shapes, seed=29)
    monkeypatch.setenv("DMU_SCHEDULE", "1")
    a = run_step(w, prec=prec)
    # 4 and 5: CTA pairs staging 2 and 1 K atoms per stage (fp16 kernels);
    # 6: 256 x 512 CTA-pair tiles (fp16 launches; the others run as 1)
    for sched in ("0", "2", "4", "5", "6"):
        monkeypatch.setenv("DMU_SCHEDULE", sched)
        b = run_step(w, prec=prec)
        for i in range(w.count):
            assert torch.equal(a["o"][i], b["o"][i]), (sched, shapes[i])
            assert torch.equal(a["w_after"][i], b["w_after"][i]), (sched, shapes[i])


def test_autotune_picks_and_caches_schedule(tmp_path):
    """Per-shape choices: one per Gram class, one per final bucket, each
    with the times of its candidates in the cache file; a second plan with
    the same shapes reuses them untimed; the tuned plan then matches the
    oracle."""
    shapes = [(1024, 4096), (4096, 1024), (512, 2048)]
    w = synth.custom("tune", shapes, seed=33)
    grads = synth.gradients(w, "cuda")
    cache = str(tmp_path / "dmu_schedule.txt")
    plan = dmu.Plan(shapes)
    plan.momentum_normalize(grads, None, beta=0.0)
    choice = plan.autotune(cache)
    names = set(dmu.SCHEDULES.values())
    assert set(choice["gram"]) == {1024, 512} and set(choice["final"]) == set(shapes)
    assert set(choice["syrk"]) == set(shapes)
    assert all(v in names and v != "onchip" for part in choice.values() for v in part.values())
    text = open(cache).read()
    assert "s1_ms=" in text and "s0_ms=" in text and "s2_ms=" in text
    assert "s3_ms=" not in text  # no class here has m <= 128
    assert "s6_ms=" in text  # 256 x 512 CTA-pair tiles: a candidate for every bucket's SYRK
    assert sum("/syrk/" in line for line in text.splitlines()) == len(shapes)
    # a second plan with the same shapes reuses the cached choices
    plan2 = dmu.Plan(shapes)
    plan2.momentum_normalize(grads, None, beta=0.0)
    assert plan2.autotune(cache) == choice
    assert open(cache).read() == text
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    plan2.gram_ns_batched(None)
    plan2.apply_update(None, out_o=outs)
    for i in range(len(shapes)):
        assert rel(f64(outs[i]), oracle_o(grads[i], torch.zeros(shapes[i]), 0.0)) < 2e-2
