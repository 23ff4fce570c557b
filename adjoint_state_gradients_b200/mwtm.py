"""ctypes binding of libmwtm.so (declared in include/mw_tm.h).

Argument marshalling only: torch tensors become device pointers, the current
torch stream becomes the cudaStream_t.  Every step of the computation runs in
the library's CUDA kernels.  Loading fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

MW_OK = 0
MW_ERR_ARG = -1
MW_ERR_CFL = -2
MW_ERR_WORKSPACE = -3
MW_ERR_CUDA = -4
MW_ERR_NONFINITE = -5
MW_ERR_TIMEOUT = -6
MW_ERR_UNSUPPORTED = -7

SNAP_NONE, SNAP_FP32, SNAP_BF16, SNAP_CKPT, SNAP_FP8, SNAP_CKPT_EY = 0, 1, 2, 3, 4, 5
SNAP_MODES = {"none": SNAP_NONE, "fp32": SNAP_FP32, "bf16": SNAP_BF16, "ckpt": SNAP_CKPT,
              "fp8": SNAP_FP8, "ckpt_ey": SNAP_CKPT_EY}


class Params(ctypes.Structure):
    _fields_ = [("ny", ctypes.c_int32), ("nx", ctypes.c_int32), ("order", ctypes.c_int32),
                ("n_shots", ctypes.c_int32), ("n_src", ctypes.c_int32), ("n_rec", ctypes.c_int32),
                ("nt", ctypes.c_int32), ("dt", ctypes.c_double), ("dy", ctypes.c_double),
                ("dx", ctypes.c_double), ("n_pml", ctypes.c_int32), ("model_batched", ctypes.c_int32),
                ("cq_is_scalar", ctypes.c_int32), ("snap_mode", ctypes.c_int32),
                ("ckpt_every", ctypes.c_int32), ("grad_mask_pml", ctypes.c_int32),
                ("vmax", ctypes.c_double), ("allow_unstable", ctypes.c_int32),
                ("check_finite", ctypes.c_int32), ("snap_host", ctypes.c_int32),
                ("snap_host_ptr", ctypes.c_void_p), ("ckpt_tail", ctypes.c_int32)]


class MWError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"mw_tm error {code}: {msg}")
        self.code = code


_lib = None
_VP = ctypes.c_void_p
_P = ctypes.POINTER(Params)

# (name, restype, argtypes) of every exported entry point
SIGNATURES = [
    ("mw_params_init", None, [_P]),
    ("mw_state_floats", ctypes.c_size_t, [_P]),
    ("mw_snap_host_bytes", ctypes.c_size_t, [_P]),
    ("mw_workspace_bytes", ctypes.c_size_t, [_P]),
    ("mw_cfl_dt", ctypes.c_double, [ctypes.c_int32, ctypes.c_double, ctypes.c_double, ctypes.c_double]),
    ("mw_validate", ctypes.c_int, [_P]),
    ("mw_model_from_eps_sigma", ctypes.c_int, [_P, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("mw_cpml_profiles", ctypes.c_int, [_P, ctypes.c_double, ctypes.c_double, _VP, _VP]),
    ("mw_tm_forward", ctypes.c_int, [_P, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                     ctypes.c_size_t, _VP]),
    ("mw_tm_adjoint_grad", ctypes.c_int, [_P, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                          _VP, _VP, ctypes.c_size_t, _VP]),
    ("mw_combine_grad", ctypes.c_int, [_P, _VP, _VP, ctypes.c_int32, _VP]),
    ("mw_grad_eps_sigma", ctypes.c_int, [ctypes.c_int64, ctypes.c_double, _VP, _VP, _VP, _VP, _VP, _VP,
                                         _VP]),
    ("mw_residual", ctypes.c_int, [ctypes.c_int64, _VP, _VP, _VP, _VP, _VP]),
    ("mw_sync_status", ctypes.c_int, [_VP, _VP]),
    ("mw_last_error", ctypes.c_char_p, []),
    ("mw_profile_enable", ctypes.c_int, [ctypes.c_int32]),
    ("mw_profile_read", ctypes.c_int, [ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double),
                                       ctypes.c_int32]),
    ("mw_launch_count", ctypes.c_int64, []),
    ("mw_tm_born", ctypes.c_int, [_P] + [ctypes.c_void_p] * 10 + [ctypes.c_size_t, ctypes.c_void_p]),
    ("mw_selftest_wait_timeout", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    ("mw_snapshot_encode", ctypes.c_int, [ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p]),
    ("mw_workspace_init", ctypes.c_int, [_VP, ctypes.c_size_t, _VP]),
    ("mw_tm_forward_noalloc", ctypes.c_int, [_P, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
]

NOALLOC_SCRATCH_BYTES = 64 << 20


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libmwtm.so (building it first if the sources are newer)."""
    global _lib
    if _lib is None:
        if not _build.up_to_date():
            _build.build()
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"CUDA library missing: {_build.LIB}")
        L = ctypes.CDLL(_build.LIB)
        for name, res, args in SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def last_error() -> str:
    return lib().mw_last_error().decode()


def check(rc: int):
    if rc != MW_OK:
        raise MWError(rc, last_error())
    return rc


def ptr(t):
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_params(**kw) -> Params:
    p = Params()
    lib().mw_params_init(ctypes.byref(p))
    for k, v in kw.items():
        if not hasattr(p, k):
            raise KeyError(k)
        setattr(p, k, v)
    return p


def state_floats(p: Params) -> int:
    n = lib().mw_state_floats(ctypes.byref(p))
    if n == 0:
        raise MWError(MW_ERR_ARG, last_error())
    return n


def snap_host_bytes(p: Params) -> int:
    """Pinned host bytes of the snapshots when p.snap_host = 1."""
    return lib().mw_snap_host_bytes(ctypes.byref(p))


def workspace_bytes(p: Params) -> int:
    n = lib().mw_workspace_bytes(ctypes.byref(p))
    if n == 0:
        raise MWError(MW_ERR_ARG, last_error())
    return n


def cfl_dt(order, dy, dx, vmax) -> float:
    return lib().mw_cfl_dt(order, dy, dx, vmax)


def validate(p: Params) -> int:
    return lib().mw_validate(ctypes.byref(p))


def model_from_eps_sigma(p, eps_r, sigma, mu_r, ca, cb, cq, stream=None):
    return check(lib().mw_model_from_eps_sigma(ctypes.byref(p), ptr(eps_r), ptr(sigma), ptr(mu_r),
                                               ptr(ca), ptr(cb), ptr(cq), stream_ptr(stream)))


def cpml_profiles(p, f0, R, cpml, stream=None):
    return check(lib().mw_cpml_profiles(ctypes.byref(p), f0, R, ptr(cpml), stream_ptr(stream)))


def workspace_init(workspace, stream=None):
    return check(lib().mw_workspace_init(ptr(workspace), workspace.numel() * workspace.element_size(),
                                         stream_ptr(stream)))


def tm_forward(p, ca, cb, cq, cpml, f, src_idx, rec_idx, state, rec, workspace, stream=None):
    return check(lib().mw_tm_forward(ctypes.byref(p), ptr(ca), ptr(cb), ptr(cq), ptr(cpml), ptr(f),
                                     ptr(src_idx), ptr(rec_idx), ptr(state), ptr(rec), ptr(workspace),
                                     workspace.numel() * workspace.element_size(), stream_ptr(stream)))


def tm_forward_noalloc(p, ca, cb, cq, cpml, f, src_idx, rec_idx, state, rec, stream=None) -> int:
    """Scratch-free forward (records only); returns the status code."""
    return lib().mw_tm_forward_noalloc(ctypes.byref(p), ptr(ca), ptr(cb), ptr(cq), ptr(cpml), ptr(f),
                                       ptr(src_idx), ptr(rec_idx), ptr(state), ptr(rec),
                                       stream_ptr(stream))


def tm_adjoint_grad(p, ca, cb, cq, cpml, f, src_idx, rec_idx, res, gca_shot, gcb_shot, grad_f,
                    adj_state, workspace, stream=None):
    return check(lib().mw_tm_adjoint_grad(ctypes.byref(p), ptr(ca), ptr(cb), ptr(cq), ptr(cpml), ptr(f),
                                          ptr(src_idx), ptr(rec_idx), ptr(res), ptr(gca_shot),
                                          ptr(gcb_shot), ptr(grad_f), ptr(adj_state), ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          stream_ptr(stream)))


def combine_grad(p, grad_shot, grad, accumulate=False, stream=None):
    return check(lib().mw_combine_grad(ctypes.byref(p), ptr(grad_shot), ptr(grad), int(accumulate),
                                       stream_ptr(stream)))


def grad_eps_sigma(n, dt, ca, cb, gca, gcb, g_eps, g_sigma, stream=None):
    return check(lib().mw_grad_eps_sigma(n, dt, ptr(ca), ptr(cb), ptr(gca), ptr(gcb), ptr(g_eps),
                                         ptr(g_sigma), stream_ptr(stream)))


def residual(n, d, d_obs, res, J=None, stream=None):
    return check(lib().mw_residual(n, ptr(d), ptr(d_obs), ptr(res), ptr(J), stream_ptr(stream)))


def sync_status(workspace, stream=None) -> int:
    return lib().mw_sync_status(ptr(workspace), stream_ptr(stream))


def profile_enable(on: bool):
    return check(lib().mw_profile_enable(1 if on else 0))


def launch_count() -> int:
    return lib().mw_launch_count()


def profile_read(n_classes: int = 3):
    counts = (ctypes.c_int64 * n_classes)()
    ms = (ctypes.c_double * n_classes)()
    check(lib().mw_profile_read(counts, ms, n_classes))
    return list(counts), list(ms)


def snapshot_encode(snap_mode, x, out, stream=None):
    """Round float32 `x` to the storage format of snap_mode (SNAP_BF16 or
    SNAP_FP8) into `out` (2 or 1 bytes per value) on the device."""
    return check(lib().mw_snapshot_encode(int(snap_mode), x.numel(), ptr(x), ptr(out),
                                          stream_ptr(stream)))


def selftest_wait_timeout(workspace, stream=None):
    """Run the bounded-wait self-test kernel on `workspace` (see mw_tm.h)."""
    return check(lib().mw_selftest_wait_timeout(ptr(workspace), stream_ptr(stream)))


def tm_born(p, ca, cb, cq, cpml, dca, dcb, f, src_idx, rec_idx, rec, workspace, stream=None):
    """Born (linearised) forward records of (dca, dcb) about the last forward's
    background on this workspace (see mw_tm.h)."""
    return check(lib().mw_tm_born(ctypes.byref(p), ptr(ca), ptr(cb), ptr(cq), ptr(cpml), ptr(dca),
                                  ptr(dcb), ptr(f), ptr(src_idx), ptr(rec_idx), ptr(rec),
                                  ptr(workspace), workspace.numel() * workspace.element_size(),
                                  stream_ptr(stream)))
