"""Host-side checks of the C ABI (no GPU needed).

* libdmu.so loads and exports every function include/dmu.h declares;
* argument errors come back as status codes before any CUDA call;
* planning (bucketing, Gram classes, workspace layout) works without a
  device, and compute calls then fail cleanly.
"""
import ctypes
import os
import re

import pytest
import torch

from gram_newton_schulz_b200 import dmu, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dmu.h")
NO_GPU = not torch.cuda.is_available()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"DMU_API\s+[\w\s\*]+?\b(dmu_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("dmu_momentum_normalize", "dmu_gram_ns_batched", "dmu_apply_update", "dmu_plan_create",
              "dmu_set_workspace", "dmu_workspace_bytes", "dmu_read_status", "dmu_plan_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = dmu.load()
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) <= set(dmu.SIGNATURES)
    assert lib.dmu_version() == 100


def _shapes(pairs):
    arr = (dmu.Shape * max(len(pairs), 1))(*[dmu.Shape(r, c) for r, c in pairs])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def _create(pairs, dtype=0, prec=0, count=None):
    lib = dmu.load()
    p, keep = _shapes(pairs)
    h = ctypes.c_void_p()
    st = lib.dmu_plan_create(p, len(pairs) if count is None else count, dtype, prec, 0, ctypes.byref(h))
    return st, h, keep


def test_argument_errors():
    lib = dmu.load()
    h = ctypes.c_void_p()
    assert lib.dmu_plan_create(None, 1, 0, 0, 0, ctypes.byref(h)) == dmu.ERR_INVALID_ARG
    assert b"NULL" in lib.dmu_last_error()
    assert _create([(4, 4)], count=0)[0] == dmu.ERR_INVALID_ARG
    assert _create([(0, 4)])[0] == dmu.ERR_INVALID_ARG
    assert _create([(4, -1)])[0] == dmu.ERR_INVALID_ARG
    assert _create([(4, 4)], dtype=7)[0] == dmu.ERR_INVALID_ARG
    assert _create([(4, 4)], prec=9)[0] == dmu.ERR_INVALID_ARG
    assert _create([(4, 1 << 21)])[0] == dmu.ERR_UNSUPPORTED
    p, keep = _shapes([(4, 4)])
    assert lib.dmu_plan_create(p, 1, 0, 0, 0, None) == dmu.ERR_INVALID_ARG
    # calls on a NULL plan
    assert lib.dmu_set_workspace(None, None, 0) == dmu.ERR_INVALID_ARG
    assert lib.dmu_momentum_normalize(None, None, None, 0.9, 1.0, 1e-7, None) == dmu.ERR_INVALID_ARG
    co = (ctypes.c_float * 3)(*dmu.QUINTIC)
    assert lib.dmu_gram_ns_batched(None, None, p, 1, ctypes.cast(co, ctypes.c_void_p), 5, None) == dmu.ERR_INVALID_ARG
    assert lib.dmu_apply_update(None, None, 0.02, None, None) == dmu.ERR_INVALID_ARG
    assert lib.dmu_workspace_bytes(None) == 0
    lib.dmu_plan_destroy(None)


def _ws_expected(shapes, nslots, esize=2, auto_tf32=True):
    mb = 0
    buckets = {}
    for r, c in shapes:
        buckets.setdefault((r, c), 0)
        buckets[(r, c)] += 1
    for (r, c), n in buckets.items():
        ldc = -(-c // 8) * 8
        mb += n * r * ldc
    gram = 0
    classes = {}
    for r, c in shapes:
        m = min(r, c)
        classes[m] = classes.get(m, 0) + 1
    for m, n in classes.items():
        ldg = -(-m // 8) * 8 if esize == 2 else m
        if esize == 2 and auto_tf32 and m < 1024:
            # split-bf16 classes: 10 slots + the final P as an fp16 pair
            gram += (nslots + 2) * n * m * ldg
        else:
            # scaled-fp16 classes (m >= 1024) keep their final P in their own
            # fp16 P slots; fp32 plans have 5 fp32 slots
            gram += nslots * n * m * ldg
    return esize * (mb + gram)


@pytest.mark.skipif(not NO_GPU, reason="host-only planning is checked where no device exists")
def test_host_only_plan_layout_qwen7b():
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    st, h, keep = _create(w.shapes)
    assert st == dmu.OK
    lib = dmu.load()
    total = lib.dmu_workspace_bytes(h)
    expect = _ws_expected(w.shapes, 10)
    # tables, per-chunk partial sums and alignment add a little on top
    assert expect <= total <= expect * 1.002
    assert 45e9 < total < 52e9
    # no device: setting a workspace or computing fails cleanly
    assert lib.dmu_set_workspace(h, ctypes.c_void_p(256), total) == dmu.ERR_CUDA
    assert lib.dmu_momentum_normalize(h, None, None, 0.9, 1.0, 1e-7, None) == dmu.ERR_WORKSPACE
    lib.dmu_plan_destroy(h)


@pytest.mark.skipif(not NO_GPU, reason="host-only planning is checked where no device exists")
@pytest.mark.parametrize("name", ["single-64x256-fp32", "uniform-64x512x2048", "small-swarm-4096",
                                  "large-dense-24"])
def test_host_only_plan_sizes(name):
    w = synth.workload(name)
    st, h, keep = _create(w.shapes, dtype=0 if w.dtype == "bf16" else 1)
    assert st == dmu.OK
    total = dmu.load().dmu_workspace_bytes(h)
    expect = _ws_expected(w.shapes, 10 if w.dtype == "bf16" else 5, 2 if w.dtype == "bf16" else 4)
    assert expect <= total <= expect * 1.01 + (1 << 20)
    dmu.load().dmu_plan_destroy(h)


def test_binding_rejects_mismatched_tensors():
    # shape/dtype validation happens in the binding before the C call
    class Fake:
        shape = (3, 3)
        dtype = torch.bfloat16
        device = torch.device("cpu")

        def is_contiguous(self):
            return True

    p = dmu.Plan.__new__(dmu.Plan)
    p.count = 1
    p.shapes = [(4, 4)]
    p.device = torch.device("cuda", 0)
    with pytest.raises(ValueError):
        p._check_tensors([Fake()], "grads", torch.bfloat16)
    with pytest.raises(ValueError):
        p._check_tensors([], "grads", torch.bfloat16)


def test_demuon_argument_errors_before_any_launch():
    """dmu_demuon_track / dmu_demuon_mix validate everything on the host;
    these calls return before any CUDA call, so they need no GPU.  The fake
    device pointers are never dereferenced."""
    lib = dmu.load()
    vp = ctypes.c_void_p

    def ptrs(*vals):
        arr = (ctypes.c_void_p * len(vals))(*vals)
        return ctypes.cast(arr, vp), arr

    mix2 = (ctypes.c_float * 4)(0.5, 0.5, 0.5, 0.5)
    m2 = ctypes.cast(mix2, vp)
    a, ka = ptrs(0x1000, 0x2000)
    b, kb = ptrs(0x3000, 0x4000)
    c, kc = ptrs(0x5000, 0x6000)
    d, kd = ptrs(0x7000, 0x8000)
    e, ke = ptrs(0x9000, 0xa000)
    track = lib.dmu_demuon_track
    mixf = lib.dmu_demuon_mix
    assert track(0, 16, m2, 0.1, a, b, c, d, e, None) == dmu.ERR_INVALID_ARG      # no agents
    assert track(17, 16, m2, 0.1, a, b, c, d, e, None) == dmu.ERR_INVALID_ARG     # too many agents
    assert track(2, -1, m2, 0.1, a, b, c, d, e, None) == dmu.ERR_INVALID_ARG      # negative size
    assert track(2, 16, None, 0.1, a, b, c, d, e, None) == dmu.ERR_INVALID_ARG    # no weights
    assert track(2, 16, m2, 1.5, a, b, c, d, e, None) == dmu.ERR_INVALID_ARG      # theta > 1
    assert track(2, 16, m2, float("nan"), a, b, c, d, e, None) == dmu.ERR_INVALID_ARG
    assert track(2, 16, m2, 0.1, a, b, c, c, e, None) == dmu.ERR_INVALID_ARG      # v_out aliases v_in
    assert b"alias" in lib.dmu_last_error()
    assert track(2, 16, m2, 0.1, a, b, c, b, e, None) == dmu.ERR_INVALID_ARG      # v_out aliases momenta
    assert track(2, 16, m2, 0.1, a, b, c, d, a, None) == dmu.ERR_INVALID_ARG      # v_bf16 aliases grads
    assert track(2, 16, m2, 0.1, a, b, c, d, d, None) == dmu.ERR_INVALID_ARG      # v_bf16 aliases v_out
    odd, ko = ptrs(0x1004, 0x2000)
    assert track(2, 16, m2, 0.1, odd, b, c, d, e, None) == dmu.ERR_INVALID_ARG    # misaligned
    assert b"16-byte" in lib.dmu_last_error()
    nul, kn = ptrs(0x1000, 0)
    assert track(2, 16, m2, 0.1, nul, b, c, d, e, None) == dmu.ERR_INVALID_ARG    # null pointer
    bad = (ctypes.c_float * 4)(0.5, float("inf"), 0.5, 0.5)
    assert track(2, 16, ctypes.cast(bad, vp), 0.1, a, b, c, d, e, None) == dmu.ERR_INVALID_ARG
    assert mixf(2, 16, m2, float("inf"), a, b, c, None) == dmu.ERR_INVALID_ARG    # eta not finite
    assert mixf(2, 16, m2, 0.1, a, b, a, None) == dmu.ERR_INVALID_ARG             # x_out aliases x_in
    assert mixf(2, 16, m2, 0.1, a, b, b, None) == dmu.ERR_INVALID_ARG             # x_out aliases o
    assert mixf(2, 16, m2, 0.1, odd, b, c, None) == dmu.ERR_INVALID_ARG
    assert mixf(0, 16, m2, 0.1, a, b, c, None) == dmu.ERR_INVALID_ARG
    # zero elements is valid and launches nothing
    assert track(2, 0, m2, 0.1, a, b, c, d, e, None) == dmu.OK
    assert mixf(2, 0, m2, 0.1, a, b, c, None) == dmu.OK


def test_demuon_mixing_matrices_match_the_oracle():
    import numpy as np
    from gram_newton_schulz_b200 import demuon
    from oracle import demuon as odm
    for topo in ("complete", "ring", "exponential"):
        for n in (1, 2, 3, 4, 6, 8, 16):
            np.testing.assert_allclose(np.array(demuon.mixing_matrix(topo, n)), odm.mixing_matrix(topo, n),
                                       rtol=0, atol=1e-15)


def test_per_class_schedule_queries(monkeypatch):
    """Planning alone (no device needed): with DMU_ONCHIP=1 the split-bf16
    classes with m <= 128 start on the on-chip schedule (3), the others and
    every final GEMM on the plan default (CTA pairs, 1)."""
    lib = dmu.load()
    monkeypatch.setenv("DMU_ONCHIP", "1")
    monkeypatch.delenv("DMU_SCHEDULE", raising=False)
    monkeypatch.delenv("DMU_CTA_PAIR", raising=False)
    pairs = [(128, 512), (512, 128), (256, 1024), (64, 64), (2048, 1024)]
    st, h, keep = _create(pairs)
    assert st == dmu.OK
    assert [lib.dmu_get_gram_schedule(h, i) for i in range(5)] == [3, 3, 1, 3, 1]
    assert [lib.dmu_get_final_schedule(h, i) for i in range(5)] == [1] * 5
    assert [lib.dmu_get_syrk_schedule(h, i) for i in range(5)] == [3, 3, 1, 3, 1]
    assert lib.dmu_get_syrk_schedule(h, 5) == -1 and lib.dmu_get_syrk_schedule(None, 0) == -1
    assert lib.dmu_get_gram_schedule(h, 5) == -1 and lib.dmu_get_final_schedule(h, -1) == -1
    assert lib.dmu_get_gram_schedule(None, 0) == -1
    lib.dmu_plan_destroy(h)
    st, h, keep = _create(pairs, prec=1)  # FAST precision: nothing runs on chip
    assert st == dmu.OK and lib.dmu_get_gram_schedule(h, 0) == 1
    lib.dmu_plan_destroy(h)
    monkeypatch.setenv("DMU_ONCHIP", "0")
    st, h, keep = _create(pairs)
    assert st == dmu.OK and lib.dmu_get_gram_schedule(h, 0) == 1
    lib.dmu_plan_destroy(h)
    # DMU_SCHEDULE takes the tile schedules (6: 256 x 512 CTA-pair tiles);
    # 3 (on chip) and values outside 0..6 leave the default
    for env, want in (("6", 6), ("4", 4), ("3", 1), ("7", 1), ("-1", 1)):
        monkeypatch.setenv("DMU_SCHEDULE", env)
        st, h, keep = _create(pairs)
        assert st == dmu.OK
        assert lib.dmu_get_schedule(h) == want, env
        assert lib.dmu_get_final_schedule(h, 4) == want, env
        lib.dmu_plan_destroy(h)
