"""The allocation-free momentum/norm entry point (dmu_momentum_norm_static).

Callers that cannot allocate device memory -- a host process whose device
memory belongs to another framework's pool, a plugin forbidden to call the
CUDA allocator, or a hot loop where cudaMalloc would synchronise -- use this
entry point, which keeps its scratch in a fixed array inside the library.
This test calls it through the C ABI twice in a row (two matrices of
different sizes, so the shared scratch is reused with stale contents) and
checks each result against the plan-based dmu_momentum_normalize on the same
inputs.  The file sorts last so that a failure here never hides another
test's result.
"""
import ctypes

import numpy as np
import pytest
import torch

from gram_newton_schulz_b200 import dmu, synth

pytestmark = pytest.mark.gpu

BETA, EPS = 0.95, 1e-7


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _plan_image(m, sc, dtype):
    """The image the plan path holds for fp32 values m: fp16 at the power-of
    -two scale sc, read back in m's units (fp32 plans keep m itself)."""
    if dtype == "f32":
        return m
    return (m * sc).half().float() / sc


def _static_call(lib, g, mom, img, inv, dtype_code, beta=BETA):
    r, c = g.shape
    return lib.dmu_momentum_norm_static(
        _ptr(g), _ptr(mom), _ptr(img), r, c, dtype_code, beta, EPS, _ptr(inv),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_static_scratch_matches_plan_path_two_calls(dtype):
    lib = dmu.load()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    # second call is smaller: the scratch still holds the first call's sums
    for call, shape in enumerate([(3584, 3584), (512, 2048), (300, 77)]):
        w = synth.custom("noalloc", [shape], seed=90 + call, dtype=dtype)
        g = synth.gradients(w, "cuda")[0]
        m0 = torch.randn(shape, generator=torch.Generator("cuda").manual_seed(call), device="cuda")

        plan = dmu.Plan([shape], dtype=dtype)
        mom_a = m0.clone()
        plan.momentum_normalize([g], [mom_a], beta=BETA, eps=EPS)
        inv_a = plan.debug(6)
        img_a = plan.debug(5, 0)
        sc = float(plan.debug(9)[0]) if dtype == "bf16" else 1.0

        mom_b = m0.clone()
        img_b = torch.empty(shape, dtype=tdt, device="cuda")
        inv_b = torch.full((1,), -1.0, device="cuda")
        st = _static_call(lib, g, mom_b, img_b, inv_b, dmu.DTYPES[dtype])
        assert st == dmu.OK, lib.dmu_last_error()
        torch.cuda.synchronize()
        assert torch.equal(mom_a, mom_b)
        # this entry point writes M rounded to the dtype; the plan keeps M in
        # fp16 at its power-of-two scale 2^e (fp32 plans: M itself)
        assert torch.equal(img_b, mom_b.to(tdt))
        assert torch.equal(img_a, _plan_image(mom_a, sc, dtype))
        assert float(inv_b[0]) == pytest.approx(float(inv_a[0]), rel=1e-6)
        x = mom_b.double().cpu().numpy()
        assert float(inv_b[0]) == pytest.approx(1.0 / (np.linalg.norm(x) + EPS), rel=2e-6)


@pytest.mark.parametrize("drop", ["momentum", "image"])
def test_static_scratch_optional_outputs(drop):
    """momentum = NULL: M = G and no state is written; image_out = NULL: only
    the norm is produced.  Compared with the plan path at beta = 0 (M = G)."""
    lib = dmu.load()
    shape = (1024, 768)
    w = synth.custom("noalloc-opt", [shape], seed=97)
    g = synth.gradients(w, "cuda")[0]
    plan = dmu.Plan([shape])
    plan.momentum_normalize([g], None, beta=0.0, eps=EPS)
    inv_a = plan.debug(6)
    img_a = plan.debug(5, 0)
    sc = float(plan.debug(9)[0])
    for _ in range(2):
        if drop == "momentum":
            img_b = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
            st = _static_call(lib, g, None, img_b, inv_b := torch.full((1,), -1.0, device="cuda"), 0)
        else:
            mom = torch.zeros(shape, device="cuda")
            img_b = None
            st = _static_call(lib, g, mom, None, inv_b := torch.full((1,), -1.0, device="cuda"), 0)
        assert st == dmu.OK, lib.dmu_last_error()
        torch.cuda.synchronize()
        if img_b is not None:
            assert torch.equal(img_b, g)
            assert torch.equal(img_a, _plan_image(g.float(), sc, "bf16"))
        else:
            assert torch.equal(mom, g.float())  # beta * 0 + G
        assert float(inv_b[0]) == pytest.approx(float(inv_a[0]), rel=1e-6)


def test_static_call_allocates_no_device_memory():
    """Free device memory is the same before and after a warmed-up call."""
    lib = dmu.load()
    shape = (2048, 2048)
    w = synth.custom("noalloc-mem", [shape], seed=98)
    g = synth.gradients(w, "cuda")[0]
    mom = torch.zeros(shape, device="cuda")
    img = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    inv = torch.empty(1, device="cuda")
    assert _static_call(lib, g, mom, img, inv, 0) == dmu.OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _static_call(lib, g, mom, img, inv, 0) == dmu.OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_static_scratch_rejects_oversize_and_bad_args():
    lib = dmu.load()
    dummy = torch.empty(16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = lib.dmu_momentum_norm_static(p, None, p, 1 << 15, 1 << 14, 0, BETA, EPS, p, None)
    assert st == dmu.ERR_UNSUPPORTED
    assert b"2^28" in lib.dmu_last_error()
    assert lib.dmu_momentum_norm_static(None, None, p, 4, 4, 0, BETA, EPS, p, None) == dmu.ERR_INVALID_ARG
    assert lib.dmu_momentum_norm_static(p, None, p, 0, 4, 0, BETA, EPS, p, None) == dmu.ERR_INVALID_ARG
