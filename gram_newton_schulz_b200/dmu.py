"""ctypes binding for libdmu (include/dmu.h): argument marshalling only.

Every step of the update runs in the library's CUDA kernels; this module
passes device pointers (``tensor.data_ptr()``), sizes and the current torch
stream across the C ABI and turns status codes into exceptions.  It has no
compute fallback: when ``_lib/libdmu.so`` is missing, ``load()`` raises.

Typical use::

    plan = Plan([(w.shape[0], w.shape[1]) for w in weights], dtype="bf16")
    plan.momentum_normalize(grads, momenta, beta=0.95, eps=1e-7)
    plan.gram_ns_batched(coeffs=QUINTIC, steps=5)
    plan.apply_update(weights, lr=0.02)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

QUINTIC = (3.4445, -4.7750, 2.0315)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libdmu.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_NONFINITE, ERR_NOT_PLANNED, ERR_TIMEOUT = range(8)
STATUS_NAMES = ["OK", "INVALID_ARG", "UNSUPPORTED", "WORKSPACE", "CUDA", "NONFINITE", "NOT_PLANNED", "TIMEOUT"]
DTYPES = {"bf16": 0, "f32": 1}
PRECS = {"auto": 0, "fast": 1, "split2": 2, "split3": 3, "tf32": 4, "f16": 5}
FLAG_NONFINITE, FLAG_TIMEOUT = 1, 2
SCHEDULES = {0: "single_cta", 1: "cta_pair", 2: "single_cta_n128", 3: "onchip", 4: "cta_pair_k2",
             5: "cta_pair_k1", 6: "cta_pair_n512"}

# name -> (restype, argtypes); every symbol of include/dmu.h
_VP = ctypes.c_void_p
SIGNATURES = {
    "dmu_plan_create": (ctypes.c_int, [_VP, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_VP)]),
    "dmu_workspace_bytes": (ctypes.c_size_t, [_VP]),
    "dmu_set_workspace": (ctypes.c_int, [_VP, _VP, ctypes.c_size_t]),
    "dmu_momentum_normalize": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_float, ctypes.c_float, ctypes.c_float, _VP]),
    "dmu_gram_ns_batched": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int, _VP, ctypes.c_int, _VP]),
    "dmu_apply_update": (ctypes.c_int, [_VP, _VP, ctypes.c_float, _VP, _VP]),
    "dmu_read_status": (ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_uint32)]),
    "dmu_debug_gram": (ctypes.c_int, [_VP, ctypes.c_int, ctypes.c_int, _VP, _VP]),
    "dmu_last_launch_count": (ctypes.c_int, [_VP]),
    "dmu_last_error": (ctypes.c_char_p, []),
    "dmu_version": (ctypes.c_int, []),
    "dmu_plan_destroy": (None, [_VP]),
    "dmu_autotune": (ctypes.c_int, [_VP, ctypes.c_char_p, _VP]),
    "dmu_get_schedule": (ctypes.c_int, [_VP]),
    "dmu_get_gram_schedule": (ctypes.c_int, [_VP, ctypes.c_int]),
    "dmu_get_final_schedule": (ctypes.c_int, [_VP, ctypes.c_int]),
    "dmu_get_syrk_schedule": (ctypes.c_int, [_VP, ctypes.c_int]),
    "dmu_momentum_norm_static": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                                ctypes.c_float, ctypes.c_float, _VP, _VP]),
    "dmu_demuon_track": (ctypes.c_int, [ctypes.c_int, ctypes.c_int64, _VP, ctypes.c_float, _VP, _VP, _VP, _VP,
                                        _VP, _VP]),
    "dmu_demuon_mix": (ctypes.c_int, [ctypes.c_int, ctypes.c_int64, _VP, ctypes.c_float, _VP, _VP, _VP, _VP]),
}
DEMUON_MAX_AGENTS = 16


class Shape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class DmuError(RuntimeError):
    def __init__(self, status: int, msg: str):
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"dmu error {name}: {msg}")
        self.status = status


_lib = None


def load(path: Optional[str] = None):
    """Load libdmu.so once; raise if it is missing (there is no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libdmu.so not found at {p}; build it with "
                           "python gram_newton_schulz_b200/csrc/build.py")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _check(st: int):
    if st != OK:
        raise DmuError(st, load().dmu_last_error().decode())


def _ptr_array(ptrs):
    return (ctypes.c_void_p * len(ptrs))(*ptrs)


def _stream_handle(stream, device):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """A plan plus the workspace torch allocates for it (caller-owned memory)."""

    def __init__(self, shapes: Sequence[Sequence[int]], dtype: str = "bf16", prec: str = "auto",
                 device=None, allocate: bool = True):
        import torch
        self.lib = load()
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.count = len(self.shapes)
        self._sizes = [torch.Size(sh) for sh in self.shapes]
        self._shape_arr = (Shape * self.count)(*[Shape(r, c) for r, c in self.shapes])
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None else
                                   torch.device(device).index or 0)
        self.dtype = dtype
        h = ctypes.c_void_p()
        _check(self.lib.dmu_plan_create(ctypes.cast(self._shape_arr, _VP), self.count, DTYPES[dtype],
                                        PRECS[prec], self.device.index, ctypes.byref(h)))
        self.handle = h
        self.workspace_bytes = int(self.lib.dmu_workspace_bytes(h))
        self.workspace = None
        if allocate:
            self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
            _check(self.lib.dmu_set_workspace(h, ctypes.c_void_p(self.workspace.data_ptr()),
                                              self.workspace_bytes))
        self._keep = []

    def close(self):
        if getattr(self, "handle", None):
            self.lib.dmu_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check_tensors(self, ts, what, dtype):
        # one pass of cheap comparisons (torch.Size equality, dtype identity,
        # integer device index): thousands of matrices per call
        if len(ts) != self.count:
            raise ValueError(f"{what}: expected {self.count} tensors, got {len(ts)}")
        sizes = getattr(self, "_sizes", None)
        if sizes is None:
            import torch
            sizes = self._sizes = [torch.Size(sh) for sh in self.shapes]
        dev = self.device.index
        for k, t in enumerate(ts):
            if t.shape != sizes[k] or t.dtype is not dtype or not t.is_contiguous() or t.get_device() != dev:
                r, c = self.shapes[k]
                raise ValueError(f"{what}: tensor {tuple(t.shape)} {t.dtype} {t.device} does not match "
                                 f"({r}, {c}) {dtype} contiguous on {self.device}")

    def _wdtype(self):
        import torch
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def momentum_normalize(self, grads, momenta=None, beta: float = 0.95, eps: float = 1e-7, stream=None,
                           grad_scale: float = 1.0):
        import torch
        self._check_tensors(grads, "grads", self._wdtype())
        g = _ptr_array([t.data_ptr() for t in grads])
        m = None
        if momenta is not None:
            self._check_tensors(momenta, "momenta", torch.float32)
            m = _ptr_array([t.data_ptr() for t in momenta])
        _check(self.lib.dmu_momentum_normalize(self.handle, ctypes.cast(g, _VP),
                                               ctypes.cast(m, _VP) if m is not None else None,
                                               float(beta), float(grad_scale), float(eps),
                                               _stream_handle(stream, self.device)))

    def gram_ns_batched(self, ptrs=None, coeffs=QUINTIC, steps: int = 5, stream=None):
        arr = None
        if ptrs is not None:
            self._check_tensors(ptrs, "ptrs", self._wdtype())
            arr = _ptr_array([t.data_ptr() for t in ptrs])
        co = (ctypes.c_float * 3)(*[float(c) for c in coeffs])
        _check(self.lib.dmu_gram_ns_batched(self.handle, ctypes.cast(arr, _VP) if arr is not None else None,
                                            ctypes.cast(self._shape_arr, _VP), self.count, ctypes.cast(co, _VP),
                                            int(steps), _stream_handle(stream, self.device)))

    def apply_update(self, weights=None, lr: float = 0.02, out_o=None, stream=None):
        import torch
        w = o = None
        if weights is not None:
            self._check_tensors(weights, "weights", self._wdtype())
            w = _ptr_array([t.data_ptr() for t in weights])
        if out_o is not None:
            present = [t for t in out_o if t is not None]
            if len(out_o) != self.count:
                raise ValueError(f"out_o: expected {self.count} entries, got {len(out_o)}")
            for t, (r, c) in zip(out_o, self.shapes):
                if t is not None and (tuple(t.shape) != (r, c) or t.dtype != torch.float32
                                      or not t.is_contiguous() or t.device != self.device):
                    raise ValueError(f"out_o: tensor {tuple(t.shape)} {t.dtype} does not match ({r}, {c}) float32")
            del present
            o = _ptr_array([t.data_ptr() if t is not None else 0 for t in out_o])
        _check(self.lib.dmu_apply_update(self.handle, ctypes.cast(w, _VP) if w is not None else None, float(lr),
                                         ctypes.cast(o, _VP) if o is not None else None,
                                         _stream_handle(stream, self.device)))

    def step(self, grads, momenta, weights, *, beta=0.95, lr=0.02, eps=1e-7, coeffs=QUINTIC, steps=5,
             out_o=None, stream=None):
        """The whole update: momentum, Gram NS, fused weight update."""
        self.momentum_normalize(grads, momenta, beta, eps, stream)
        self.gram_ns_batched(None, coeffs, steps, stream)
        self.apply_update(weights, lr, out_o, stream)

    def autotune(self, cache_path: Optional[str] = None, stream=None) -> dict:
        """Choose, by measurement, the schedule of every Gram class and of
        every bucket's final GEMM (needs a prior momentum_normalize); returns
        `schedules()`."""
        _check(self.lib.dmu_autotune(self.handle, cache_path.encode() if cache_path else None,
                                     _stream_handle(stream, self.device)))
        return self.schedules()

    def schedules(self) -> dict:
        """{"gram": {m: name}, "syrk": {(rows, cols): name}, "final":
        {(rows, cols): name}} with the schedule names of SCHEDULES."""
        gram, syrk, final = {}, {}, {}
        for i, (r, c) in enumerate(self.shapes):
            gram[min(r, c)] = SCHEDULES.get(int(self.lib.dmu_get_gram_schedule(self.handle, i)), "?")
            syrk[(r, c)] = SCHEDULES.get(int(self.lib.dmu_get_syrk_schedule(self.handle, i)), "?")
            final[(r, c)] = SCHEDULES.get(int(self.lib.dmu_get_final_schedule(self.handle, i)), "?")
        return {"gram": gram, "syrk": syrk, "final": final}

    def read_status(self) -> int:
        flags = ctypes.c_uint32(0)
        st = self.lib.dmu_read_status(self.handle, ctypes.byref(flags))
        if st not in (OK, ERR_NONFINITE, ERR_TIMEOUT):
            _check(st)
        return int(flags.value)

    def debug(self, which: int, index: int = 0):
        """Test hook: fetch a workspace quantity as an fp32 torch tensor."""
        import torch
        if which == 8:
            out = torch.empty(1, dtype=torch.float32, device=self.device)
        elif which in (6, 9):
            out = torch.empty(self.count, dtype=torch.float32, device=self.device)
        elif which == 5:
            out = torch.empty(self.shapes[index], dtype=torch.float32, device=self.device)
        else:
            m = min(self.shapes[index])
            out = torch.empty((m, m), dtype=torch.float32, device=self.device)
        _check(self.lib.dmu_debug_gram(self.handle, int(which), int(index), ctypes.c_void_p(out.data_ptr()),
                                       _stream_handle(None, self.device)))
        return out

    def last_launch_count(self) -> int:
        return int(self.lib.dmu_last_launch_count(self.handle))


# ---------------------------------------------------------------- DeMuon
def _mix_array(mix, n: int):
    flat = [float(x) for row in mix for x in row]
    if len(flat) != n * n:
        raise ValueError(f"mix must be {n} x {n}")
    return (ctypes.c_float * (n * n))(*flat)


def _flat_args(tensors, what: str, dtype, numel: int):
    import torch
    for t in tensors:
        if t.dtype != dtype or not t.is_contiguous() or t.numel() < numel or not t.is_cuda:
            raise ValueError(f"{what}: expected contiguous CUDA {dtype} tensors of at least {numel} elements")
    return _ptr_array([t.data_ptr() for t in tensors])


def demuon_track(mix, theta: float, grads, momenta, v_in, v_out, v_bf16, numel: Optional[int] = None,
                 stream=None):
    """dmu_demuon_track on per-agent flat tensors: M and V fp32, grads and
    the msgn input bf16; ``mix`` is n x n (row i: what agent i applies)."""
    import torch
    lib = load()
    n = len(grads)
    numel = grads[0].numel() if numel is None else int(numel)
    args = [_flat_args(grads, "grads", torch.bfloat16, numel), _flat_args(momenta, "momenta", torch.float32, numel),
            _flat_args(v_in, "v_in", torch.float32, numel), _flat_args(v_out, "v_out", torch.float32, numel),
            _flat_args(v_bf16, "v_bf16", torch.bfloat16, numel)]
    _check(lib.dmu_demuon_track(n, numel, ctypes.cast(_mix_array(mix, n), _VP), float(theta),
                                *[ctypes.cast(a, _VP) for a in args], _stream_handle(stream, grads[0].device)))


def demuon_mix(mix, eta: float, x_in, o, x_out, numel: Optional[int] = None, stream=None):
    """dmu_demuon_mix on per-agent flat fp32 tensors: X_i' = sum_j w_ij (X_j - eta O_j)."""
    import torch
    lib = load()
    n = len(x_in)
    numel = x_in[0].numel() if numel is None else int(numel)
    args = [_flat_args(x_in, "x_in", torch.float32, numel), _flat_args(o, "o", torch.float32, numel),
            _flat_args(x_out, "x_out", torch.float32, numel)]
    _check(lib.dmu_demuon_mix(n, numel, ctypes.cast(_mix_array(mix, n), _VP), float(eta),
                              *[ctypes.cast(a, _VP) for a in args], _stream_handle(stream, x_in[0].device)))
