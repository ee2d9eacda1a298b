"""ctypes binding of libmuon (include/muon.h): argument marshalling only.

Every step of the Muon update runs in the CUDA kernels of libmuon.so; this
module turns torch tensors into raw device pointers and the current CUDA
stream into a cudaStream_t, and raises on any non-OK status.  There is no
CPU fallback: without the built library, or without an sm_100 device, every
call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmuon.so")

MUON_OK = 0
STATUS_NAMES = {
    0: "MUON_OK", 1: "MUON_ERR_INVALID_ARG", 2: "MUON_ERR_UNSUPPORTED_SHAPE", 3: "MUON_ERR_DTYPE",
    4: "MUON_ERR_CUDA", 5: "MUON_ERR_NONFINITE", 6: "MUON_ERR_TIMEOUT", 7: "MUON_ERR_NO_DEVICE",
    8: "MUON_ERR_ALLOC",
}
MUON_BF16, MUON_F32 = 0, 1
SCALE_SQRT_RATIO, SCALE_NONE, SCALE_RMS_MATCH = 0, 1, 2
FLAG_NONFINITE = 1
MAX_BATCH = 256
MAX_ITERS = 32
MAX_GROUPS = 8
QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)

# Every symbol include/muon.h declares.
EXPORTS = (
    "muon_abi_version", "muon_status_string", "muon_last_cuda_error", "muon_create", "muon_destroy",
    "muon_set_coeffs", "muon_get_coeffs", "muon_step", "muon_step_groups", "muon_step_groups_host",
    "muon_ns_orthogonalize", "muon_get_status", "muon_get_norms", "muon_workspace_bytes",
    "muon_profile_enable", "muon_profile_read", "muon_momentum_norm_noalloc", "muon_adamw_step",
    "muon_power_iteration", "muon_min_singular", "muon_step_capped",
)
KERNEL_KINDS = ("momentum", "gram", "poly", "update", "apply", "ns_fused")


class MuonError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class Hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("eps", ctypes.c_float), ("nesterov", ctypes.c_int), ("scale_mode", ctypes.c_int),
                ("grad_scale", ctypes.c_float)]


class Profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int * 6), ("ms", ctypes.c_double * 6)]


class AdamWHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int)]


class Group(ctypes.Structure):
    _fields_ = [("W", ctypes.POINTER(ctypes.c_void_p)), ("G", ctypes.POINTER(ctypes.c_void_p)),
                ("M", ctypes.POINTER(ctypes.c_void_p)), ("batch", ctypes.c_int),
                ("rows", ctypes.c_int), ("cols", ctypes.c_int), ("dtype", ctypes.c_int)]


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libmuon.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libmuon.so not built at {p}: run `python -m spectral_optimizer_state_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    pvp = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "muon_abi_version": (i, []),
        "muon_status_string": (ctypes.c_char_p, [i]),
        "muon_last_cuda_error": (ctypes.c_char_p, []),
        "muon_create": (i, [ctypes.POINTER(vp), i]),
        "muon_destroy": (i, [vp]),
        "muon_set_coeffs": (i, [vp, ctypes.POINTER(f), i]),
        "muon_get_coeffs": (i, [vp, ctypes.POINTER(f), ctypes.POINTER(i)]),
        "muon_step": (i, [vp, pvp, pvp, pvp, i, i, i, i, ctypes.POINTER(Hparams), vp]),
        "muon_step_groups": (i, [vp, ctypes.POINTER(Group), i, ctypes.POINTER(Hparams), vp]),
        "muon_step_groups_host": (i, [vp, ctypes.POINTER(Group), i, ctypes.POINTER(Hparams),
                                      ctypes.POINTER(f), ctypes.POINTER(i), vp]),
        "muon_ns_orthogonalize": (i, [vp, pvp, pvp, i, i, i, i, f, vp]),
        "muon_get_status": (i, [vp, ctypes.POINTER(i), i, ctypes.POINTER(i)]),
        "muon_get_norms": (i, [vp, ctypes.POINTER(f), i, ctypes.POINTER(i)]),
        "muon_workspace_bytes": (sz, [vp]),
        "muon_profile_enable": (i, [vp, i]),
        "muon_profile_read": (i, [vp, ctypes.POINTER(Profile), i]),
        "muon_momentum_norm_noalloc": (i, [pvp, pvp, vp, i, i, i, i, f, i, vp]),
        "muon_adamw_step": (i, [pvp, pvp, pvp, pvp, ctypes.POINTER(ctypes.c_longlong), i, i,
                                ctypes.POINTER(AdamWHparams), vp]),
        "muon_power_iteration": (i, [vp, pvp, pvp, pvp, vp, i, i, i, i, i, vp]),
        "muon_min_singular": (i, [vp, pvp, pvp, vp, vp, i, i, i, i, i, vp]),
        "muon_step_capped": (i, [vp, pvp, pvp, pvp, pvp, pvp, i, i, i, i, ctypes.POINTER(Hparams), vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _ptrs(tensors: Sequence) -> ctypes.Array:
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    if t.dtype == torch.float32:
        return MUON_F32
    raise TypeError(f"unsupported dtype {t.dtype}; libmuon takes bfloat16 or float32")


def _check_same(ts: Sequence, shape, dtype, device_type: str, what: str):
    if len(ts) == 0:
        raise ValueError(f"{what}: empty list")
    for t in ts:
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            raise ValueError(f"{what}: every matrix must be {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")
        if t.device.type != device_type:
            raise ValueError(f"{what}: expected {device_type} tensors, got {t.device}")
        if not t.is_contiguous():
            raise ValueError(f"{what}: tensors must be contiguous (row-major)")


def _stream_handle(stream) -> ctypes.c_void_p:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(int(s.cuda_stream))


class Muon:
    """A libmuon context on one CUDA device (owns the workspace and the coefficient table)."""

    def __init__(self, device: int = 0, coeffs: Iterable | None = None):
        self.lib = load_library()
        self.device = device
        h = ctypes.c_void_p()
        st = self.lib.muon_create(ctypes.byref(h), device)
        self._check(st, "muon_create")
        self.handle = h
        self._keep = []
        if coeffs is not None:
            self.set_coeffs(coeffs)

    # -------------------------------------------------------------- helpers
    def _check(self, st: int, what: str):
        if st != MUON_OK:
            detail = ""
            if st in (4, 8):
                detail = self.lib.muon_last_cuda_error().decode()
            raise MuonError(st, what, detail)

    def close(self):
        if getattr(self, "handle", None):
            self.lib.muon_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -------------------------------------------------------------- coefficients
    def set_coeffs(self, coeffs: Iterable):
        flat = [float(v) for abc in coeffs for v in abc]
        k = len(flat) // 3
        arr = (ctypes.c_float * len(flat))(*flat)
        self._check(self.lib.muon_set_coeffs(self.handle, arr, k), "muon_set_coeffs")

    def get_coeffs(self):
        arr = (ctypes.c_float * (3 * MAX_ITERS))()
        k = ctypes.c_int()
        self._check(self.lib.muon_get_coeffs(self.handle, arr, ctypes.byref(k)), "muon_get_coeffs")
        return [tuple(arr[3 * i:3 * i + 3]) for i in range(k.value)]

    # -------------------------------------------------------------- steps
    @staticmethod
    def hparams(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True, scale_mode=SCALE_SQRT_RATIO,
                grad_scale=1.0):
        return Hparams(float(lr), float(beta), float(weight_decay), float(eps), int(bool(nesterov)), int(scale_mode),
                       float(grad_scale))

    def _group(self, W, G, M, g_device_type="cuda"):
        import torch
        shape, dt = tuple(W[0].shape), W[0].dtype
        if len(shape) != 2:
            raise ValueError("matrices must be 2-D")
        if not (len(W) == len(G) == len(M)):
            raise ValueError("W, G and M must have the same length")
        _check_same(W, shape, dt, "cuda", "W")
        _check_same(G, shape, dt, g_device_type, "G")
        _check_same(M, shape, torch.float32, "cuda", "M")
        pw, pg, pm = _ptrs(W), _ptrs(G), _ptrs(M)
        self._keep = [pw, pg, pm]
        return Group(pw, pg, pm, len(W), shape[0], shape[1], _dtype_code(W[0])), (pw, pg, pm)

    def step(self, W, G, M, stream=None, **hp):
        """One Muon step on same-shape matrices W[l] (updated), G[l], M[l] (fp32, updated)."""
        self.step_groups([(W, G, M)], stream=stream, **hp)

    def step_groups(self, groups, stream=None, **hp):
        """groups: list of (W list, G list, M list), one entry per shape."""
        gs, keep = [], []
        for (W, G, M) in groups:
            g, k = self._group(W, G, M)
            gs.append(g)
            keep.append(k)
        arr = (Group * len(gs))(*gs)
        h = self.hparams(**hp)
        st = self.lib.muon_step_groups(self.handle, arr, len(gs), ctypes.byref(h), _stream_handle(stream))
        self._check(st, "muon_step_groups")

    def step_groups_host(self, groups, stream=None, **hp):
        """Like step_groups, but every G is a (pinned) CPU tensor; copies happen inside the call.

        Returns (nu, flags) per matrix in group order, after the stream has completed.
        """
        gs, keep = [], []
        for (W, G, M) in groups:
            g, k = self._group(W, G, M, g_device_type="cpu")
            gs.append(g)
            keep.append(k)
        n = sum(g.batch for g in gs)
        nu = (ctypes.c_float * n)()
        flags = (ctypes.c_int * n)()
        arr = (Group * len(gs))(*gs)
        h = self.hparams(**hp)
        st = self.lib.muon_step_groups_host(self.handle, arr, len(gs), ctypes.byref(h), nu, flags,
                                            _stream_handle(stream))
        if st not in (MUON_OK, 5):
            self._check(st, "muon_step_groups_host")
        return list(nu), list(flags)

    def ns_orthogonalize(self, X, Out, eps=1e-7, stream=None):
        """Out[l] = NS_k(X[l] / (||X[l]||_F + eps)) for same-shape matrices (bf16 or fp32)."""
        shape, dt = tuple(X[0].shape), X[0].dtype
        _check_same(X, shape, dt, "cuda", "X")
        _check_same(Out, shape, dt, "cuda", "Out")
        if len(X) != len(Out):
            raise ValueError("X and Out must have the same length")
        px, po = _ptrs(X), _ptrs(Out)
        st = self.lib.muon_ns_orthogonalize(self.handle, px, po, len(X), shape[0], shape[1],
                                            _dtype_code(X[0]), float(eps), _stream_handle(stream))
        self._check(st, "muon_ns_orthogonalize")

    # -------------------------------------------------------------- spectral
    def power_iteration(self, W, u, v, sigma, iters=8, stream=None):
        """Top singular triplet of each W[l] by `iters` power iterations.

        v[l] (fp32, cols) holds the start vector and receives the right vector;
        u[l] (fp32, rows) receives the left vector; sigma (fp32 CUDA, len(W))
        the top singular value.
        """
        import torch
        shape, dt = tuple(W[0].shape), W[0].dtype
        _check_same(W, shape, dt, "cuda", "W")
        _check_same(u, (shape[0],), torch.float32, "cuda", "u")
        _check_same(v, (shape[1],), torch.float32, "cuda", "v")
        if not (len(W) == len(u) == len(v)) or sigma.numel() < len(W) or sigma.dtype != torch.float32:
            raise ValueError("W, u, v need one entry per matrix and sigma len(W) fp32 slots")
        pw, pu, pv = _ptrs(W), _ptrs(u), _ptrs(v)
        st = self.lib.muon_power_iteration(self.handle, pw, pu, pv, ctypes.c_void_p(sigma.data_ptr()), len(W),
                                           shape[0], shape[1], _dtype_code(W[0]), int(iters),
                                           _stream_handle(stream))
        self._check(st, "muon_power_iteration")

    def min_singular(self, W, y, sigma_max, sigma_min, iters=32, stream=None):
        """Smallest singular value of each W[l] by `iters` shifted power iterations.

        y[l] (fp32 CUDA, min(rows, cols)) is the start vector and receives the
        iterate; sigma_max (fp32 CUDA, len(W)) the top singular values, e.g.
        from power_iteration; sigma_min (fp32 CUDA, len(W)) receives the estimate.
        """
        import torch
        shape, dt = tuple(W[0].shape), W[0].dtype
        _check_same(W, shape, dt, "cuda", "W")
        _check_same(y, (min(shape),), torch.float32, "cuda", "y")
        for t, what in ((sigma_max, "sigma_max"), (sigma_min, "sigma_min")):
            if t.dtype != torch.float32 or t.numel() < len(W) or t.device.type != "cuda":
                raise ValueError(f"{what}: needs len(W) fp32 CUDA slots")
        if len(y) != len(W):
            raise ValueError("y needs one entry per matrix")
        pw, py = _ptrs(W), _ptrs(y)
        st = self.lib.muon_min_singular(self.handle, pw, py, ctypes.c_void_p(sigma_max.data_ptr()),
                                        ctypes.c_void_p(sigma_min.data_ptr()), len(W), shape[0], shape[1],
                                        _dtype_code(W[0]), int(iters), _stream_handle(stream))
        self._check(st, "muon_min_singular")

    def step_capped(self, W, G, M, u, v, alpha, stream=None, **hp):
        """step() with the update's component along u[l] v[l]^T removed; alpha[l] receives u^T O v."""
        import torch
        g, (pw, pg, pm) = self._group(W, G, M)
        _check_same(u, (g.rows,), torch.float32, "cuda", "u")
        _check_same(v, (g.cols,), torch.float32, "cuda", "v")
        if not (len(u) == len(v) == len(W)) or alpha.numel() < len(W) or alpha.dtype != torch.float32:
            raise ValueError("u, v need one entry per matrix and alpha len(W) fp32 slots")
        pu, pv = _ptrs(u), _ptrs(v)
        h = self.hparams(**hp)
        st = self.lib.muon_step_capped(self.handle, pw, pg, pm, pu, pv, g.batch, g.rows, g.cols, g.dtype,
                                       ctypes.byref(h), ctypes.c_void_p(alpha.data_ptr()), _stream_handle(stream))
        self._check(st, "muon_step_capped")

    # -------------------------------------------------------------- plans (checked and marshalled once)
    def step_plan(self, groups, **hp):
        """A StepPlan for a fixed set of groups [(W list, G list, M list), ...]: the tensors are
        checked and their pointers marshalled once, so each step is one C call (the tensors must
        stay alive and in place; G is read afresh every step)."""
        return StepPlan(self, groups, **hp)

    def spectral_plan(self, W, u, v, sigma, y=None, sigma_min=None):
        """A SpectralPlan for fixed tensors: power_iteration(iters) and min_singular(iters) as one
        C call each (same arguments as the methods of the same names)."""
        return SpectralPlan(self, W, u, v, sigma, y, sigma_min)

    # -------------------------------------------------------------- status
    def status(self):
        """(status code, per-matrix flags) of the last call; synchronises its stream."""
        cap = 8 * MAX_BATCH * MAX_GROUPS
        flags = (ctypes.c_int * cap)()
        cnt = ctypes.c_int()
        st = self.lib.muon_get_status(self.handle, flags, cap, ctypes.byref(cnt))
        if st not in (MUON_OK, 5, 6):
            self._check(st, "muon_get_status")
        return st, list(flags[:cnt.value])

    def norms(self):
        cap = 8 * MAX_BATCH * MAX_GROUPS
        nu = (ctypes.c_float * cap)()
        cnt = ctypes.c_int()
        self._check(self.lib.muon_get_norms(self.handle, nu, cap, ctypes.byref(cnt)), "muon_get_norms")
        return list(nu[:cnt.value])

    def workspace_bytes(self) -> int:
        return int(self.lib.muon_workspace_bytes(self.handle))

    def profile_enable(self, on: bool = True):
        self._check(self.lib.muon_profile_enable(self.handle, int(bool(on))), "muon_profile_enable")

    def profile_read(self, reset: bool = True):
        """{kind: (launches, total device ms)} since the last reset; synchronises on the events."""
        p = Profile()
        self._check(self.lib.muon_profile_read(self.handle, ctypes.byref(p), int(bool(reset))), "muon_profile_read")
        return {k: (p.launches[i], p.ms[i]) for i, k in enumerate(KERNEL_KINDS)}


class StepPlan:
    """muon_step_groups over a fixed list of groups, validated and marshalled once."""

    def __init__(self, muon: "Muon", groups, **hp):
        self.muon = muon
        gs, self._keep = [], []
        for (W, G, M) in groups:
            g, k = muon._group(W, G, M)
            gs.append(g)
            self._keep.append((k, list(W), list(G), list(M)))  # pointer arrays and the tensors
        self._arr = (Group * len(gs))(*gs)
        self._n = len(gs)
        self._hp = Muon.hparams(**hp)

    def __call__(self, stream=None):
        st = self.muon.lib.muon_step_groups(self.muon.handle, self._arr, self._n, ctypes.byref(self._hp),
                                            _stream_handle(stream))
        self.muon._check(st, "muon_step_groups")


class SpectralPlan:
    """muon_power_iteration / muon_min_singular over fixed tensors, validated and marshalled once."""

    def __init__(self, muon: "Muon", W, u, v, sigma, y=None, sigma_min=None):
        import torch
        self.muon = muon
        shape, dt = tuple(W[0].shape), W[0].dtype
        _check_same(W, shape, dt, "cuda", "W")
        _check_same(u, (shape[0],), torch.float32, "cuda", "u")
        _check_same(v, (shape[1],), torch.float32, "cuda", "v")
        if not (len(W) == len(u) == len(v)) or sigma.numel() < len(W) or sigma.dtype != torch.float32:
            raise ValueError("W, u, v need one entry per matrix and sigma len(W) fp32 slots")
        if y is not None:
            _check_same(y, (min(shape),), torch.float32, "cuda", "y")
            if len(y) != len(W) or sigma_min is None or sigma_min.numel() < len(W) \
                    or sigma_min.dtype != torch.float32:
                raise ValueError("y needs one entry per matrix and sigma_min len(W) fp32 slots")
        self._tensors = (list(W), list(u), list(v), sigma, None if y is None else list(y), sigma_min)
        self._pw, self._pu, self._pv = _ptrs(W), _ptrs(u), _ptrs(v)
        self._py = _ptrs(y) if y is not None else None
        self._args = (len(W), shape[0], shape[1], _dtype_code(W[0]))

    def power_iteration(self, iters=8, stream=None):
        n, r, c, dt = self._args
        st = self.muon.lib.muon_power_iteration(self.muon.handle, self._pw, self._pu, self._pv,
                                                ctypes.c_void_p(self._tensors[3].data_ptr()), n, r, c, dt,
                                                int(iters), _stream_handle(stream))
        self.muon._check(st, "muon_power_iteration")

    def min_singular(self, iters=32, stream=None):
        if self._py is None:
            raise ValueError("plan built without y / sigma_min")
        n, r, c, dt = self._args
        st = self.muon.lib.muon_min_singular(self.muon.handle, self._pw, self._py,
                                             ctypes.c_void_p(self._tensors[3].data_ptr()),
                                             ctypes.c_void_p(self._tensors[5].data_ptr()), n, r, c, dt, int(iters),
                                             _stream_handle(stream))
        self.muon._check(st, "muon_min_singular")


def momentum_norm_noalloc(G, M, nu, beta=0.95, nesterov=True, stream=None):
    """M <- beta M + G in place and nu[l] = ||G + beta M||_F (or ||M||_F), without allocating.

    For callers that cannot allocate device memory: no context is created and
    the library's fixed static scratch is used (see include/muon.h).  `nu` is
    a float32 CUDA tensor with one entry per matrix.
    """
    import torch
    lib = load_library()
    shape, dt = tuple(G[0].shape), G[0].dtype
    _check_same(G, shape, dt, "cuda", "G")
    _check_same(M, shape, torch.float32, "cuda", "M")
    if len(G) != len(M) or nu.dtype != torch.float32 or not nu.is_cuda or nu.numel() < len(G):
        raise ValueError("G, M and nu do not match")
    st = lib.muon_momentum_norm_noalloc(_ptrs(G), _ptrs(M), ctypes.c_void_p(nu.data_ptr()), len(G), shape[0],
                                        shape[1], _dtype_code(G[0]), float(beta), int(bool(nesterov)),
                                        _stream_handle(stream))
    if st != MUON_OK:
        raise MuonError(st, "muon_momentum_norm_noalloc")


def _check_adamw(W, G, m, v):
    import torch
    if not (len(W) == len(G) == len(m) == len(v)) or len(W) == 0:
        raise ValueError("W, G, m and v must be non-empty lists of equal length")
    dt = W[0].dtype
    for w, g, a, b in zip(W, G, m, v):
        if w.dtype != dt or g.dtype != dt or a.dtype != torch.float32 or b.dtype != torch.float32:
            raise ValueError("W and G share one dtype; m and v are float32")
        if not (w.is_cuda and g.is_cuda and a.is_cuda and b.is_cuda):
            raise ValueError("all tensors must be on the GPU")
        if not (w.is_contiguous() and g.is_contiguous() and a.is_contiguous() and b.is_contiguous()):
            raise ValueError("tensors must be contiguous")
        if not (w.numel() == g.numel() == a.numel() == b.numel()):
            raise ValueError("W, G, m and v must match in size")


class AdamWGroup:
    """AdamW over a fixed list of tensors: validated and marshalled once, so a step costs
    one C call per MAX_BATCH tensors (the tensors must stay alive and in place)."""

    def __init__(self, W, G, m, v):
        _check_adamw(W, G, m, v)
        self.lib = load_library()
        self._tensors = (list(W), list(G), list(m), list(v))  # keep the storage alive
        self._calls = []
        for c0 in range(0, len(W), MAX_BATCH):
            sl = slice(c0, c0 + MAX_BATCH)
            ws = W[sl]
            numel = (ctypes.c_longlong * len(ws))(*[t.numel() for t in ws])
            self._calls.append((_ptrs(ws), _ptrs(G[sl]), _ptrs(m[sl]), _ptrs(v[sl]), numel, len(ws),
                                _dtype_code(ws[0])))

    def step(self, step, lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, stream=None):
        hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay), int(step))
        sh = _stream_handle(stream)
        for pw, pg, pm, pv, numel, n, dt in self._calls:
            st = self.lib.muon_adamw_step(pw, pg, pm, pv, numel, n, dt, ctypes.byref(hp), sh)
            if st != MUON_OK:
                raise MuonError(st, "muon_adamw_step")


def adamw_step(W, G, m, v, step, lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, stream=None):
    """AdamW on tensors of any shapes (one dtype, bf16 or fp32; fp32 moments), one launch per
    MAX_BATCH tensors.  For a fixed set of tensors stepped repeatedly, AdamWGroup does the
    checks once."""
    AdamWGroup(W, G, m, v).step(step, lr=lr, beta1=beta1, beta2=beta2, eps=eps, weight_decay=weight_decay,
                                stream=stream)

