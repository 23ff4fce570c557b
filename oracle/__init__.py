"""fp64 CPU oracle for the 2-D TM Maxwell FDTD forward / exact adjoint / gradients.

TEST INFRASTRUCTURE ONLY: the checker that the CUDA library is compared
against.  Only the test suite, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the library never does, and this
package imports nothing from the library.

The arithmetic lives in ``mw_oracle.c`` (plain C, fp64, OpenMP over shots and
rows); this module compiles it with gcc and marshals numpy arrays.  Method
source: the page "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu" (header comment on
the exact discrete adjoint-state method, forward H/E kernels, source/receiver
kernels, combine and epsilon/sigma chain-rule kernels).

Parity pins are in ``tests/test_oracle_*.py``.  Parity unpinned: the CPML
profile's reflection quality (only its absorption is checked).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mw_oracle.c")
_LIB = os.path.join(_HERE, "libmworacle.so")
_lib = None

NFIELD = 7
FIELDS = ("ey", "hx", "hz", "m_ey_x", "m_ey_z", "m_hz_x", "m_hx_z")


def build(force: bool = False) -> str:
    """Compile mw_oracle.c into libmworacle.so next to it (gcc, -O3, OpenMP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=gnu11", "-O3", "-march=native", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


class _Sim(ctypes.Structure):
    _fields_ = [("ny", ctypes.c_int), ("nx", ctypes.c_int), ("order", ctypes.c_int),
                ("n_shots", ctypes.c_int), ("n_src", ctypes.c_int), ("n_rec", ctypes.c_int),
                ("dy", ctypes.c_double), ("dx", ctypes.c_double),
                ("model_batched", ctypes.c_int), ("cq_is_array", ctypes.c_int),
                ("ca", _D), ("cb", _D), ("cq", _D),
                ("ay", _D), ("ayh", _D), ("by", _D), ("byh", _D), ("ky", _D), ("kyh", _D),
                ("ax", _D), ("axh", _D), ("bx", _D), ("bxh", _D), ("kx", _D), ("kxh", _D),
                ("src_idx", _I64), ("rec_idx", _I64)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.orc_coeffs.argtypes = [ctypes.c_int, _D]
        L.orc_coeffs.restype = ctypes.c_int
        L.orc_model.argtypes = [ctypes.c_int64, _D, _D, _D, ctypes.c_double, _D, _D, _D]
        L.orc_eps_sigma_grad.argtypes = [ctypes.c_int64, _D, _D, ctypes.c_double, _D, _D, _D, _D]
        L.orc_cfl_dt.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_double]
        L.orc_cfl_dt.restype = ctypes.c_double
        L.orc_c0.restype = ctypes.c_double
        L.orc_cpml.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                               ctypes.c_double, ctypes.c_double, ctypes.c_double] + [_D] * 6
        L.orc_forward.argtypes = [ctypes.POINTER(_Sim), ctypes.c_int, _D, _D, _D, _D, _D]
        L.orc_forward.restype = ctypes.c_int
        L.orc_adjoint.argtypes = [ctypes.POINTER(_Sim), ctypes.c_int, _D, _D, _D, _D, _D, _D, _D]
        L.orc_adjoint.restype = ctypes.c_int
        L.orc_fwd_adj_ckpt.argtypes = [ctypes.POINTER(_Sim), ctypes.c_int, ctypes.c_int, _D, _D,
                                       _D, _D, _D, _D, _D]
        L.orc_fwd_adj_ckpt.restype = ctypes.c_int
        L.orc_combine.argtypes = [ctypes.c_int, ctypes.c_int64, _D, _D]
        L.orc_residual.argtypes = [ctypes.c_int64, _D, _D, _D]
        L.orc_residual.restype = ctypes.c_double
        L.orc_num_threads.restype = ctypes.c_int
        _U8 = ctypes.POINTER(ctypes.c_uint8)
        L.orc_born.argtypes = [ctypes.POINTER(_Sim), ctypes.c_int, _D, _D, _D, _D, _D, _D]
        L.orc_born.restype = ctypes.c_int
        L.orc_quant_bf16.argtypes = [ctypes.c_int64, _D, _D]
        L.orc_fp8_encode.argtypes = [ctypes.c_int64, _D, _U8]
        L.orc_fp8_decode.argtypes = [ctypes.c_int64, _U8, _D]
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous, (a.dtype, a.flags)
    return a.ctypes.data_as(_D)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# small helpers (each a direct call into the C oracle)

def coeffs(order: int) -> np.ndarray:
    c = np.zeros(4)
    P = lib().orc_coeffs(order, _p(c))
    if P == 0:
        raise ValueError(f"unsupported order {order}")
    return c[:P].copy()


def c0() -> float:
    return lib().orc_c0()


def cfl_dt(order: int, dy: float, dx: float, vmax: float) -> float:
    return lib().orc_cfl_dt(order, dy, dx, vmax)


def model(eps_r, sigma, mu_r, dt):
    """(Ca, Cb, Cq) in fp64 from eps_r, sigma (S/m), mu_r (None = 1)."""
    eps_r = _f64(eps_r)
    shape = eps_r.shape
    n = eps_r.size
    sigma = _f64(sigma) if sigma is not None else None
    mu_r = _f64(mu_r) if mu_r is not None else None
    ca, cb, cq = np.empty(n), np.empty(n), np.empty(n)
    lib().orc_model(n, _p(eps_r.reshape(-1)), _p(None if sigma is None else sigma.reshape(-1)),
                    _p(None if mu_r is None else mu_r.reshape(-1)), dt, _p(ca), _p(cb), _p(cq))
    return ca.reshape(shape), cb.reshape(shape), cq.reshape(shape)


def eps_sigma_grad(ca, cb, dt, gca, gcb):
    ca, cb, gca, gcb = map(_f64, (ca, cb, gca, gcb))
    ge, gs = np.empty(ca.size), np.empty(ca.size)
    lib().orc_eps_sigma_grad(ca.size, _p(ca.reshape(-1)), _p(cb.reshape(-1)), dt,
                             _p(gca.reshape(-1)), _p(gcb.reshape(-1)), _p(ge), _p(gs))
    return ge.reshape(ca.shape), gs.reshape(ca.shape)


def cpml(n: int, n_pml: int, h: float, dt: float, vmax: float, f0: float, R: float = 1e-3):
    """(a, ah, b, bh, k, kh) along one axis, fp64."""
    out = [np.empty(n) for _ in range(6)]
    lib().orc_cpml(n, n_pml, h, dt, vmax, f0, R, *[_p(o) for o in out])
    return tuple(out)


def combine(g_shot):
    g_shot = _f64(g_shot)
    S = g_shot.shape[0]
    g = np.empty(g_shot.shape[1:])
    lib().orc_combine(S, g.size, _p(g_shot.reshape(S, -1)), _p(g.reshape(-1)))
    return g


def quant_bf16(x):
    """Snapshot storage in bfloat16: x rounded to fp32, then to bf16
    (nearest, ties to even); returned as fp64 values."""
    x = _f64(x)
    out = np.empty_like(x)
    lib().orc_quant_bf16(x.size, _p(x.reshape(-1)), _p(out.reshape(-1)))
    return out


def fp8_encode(x):
    """E4M3 codes (uint8) of x rounded to fp32: nearest, ties to even,
    saturating to +-448."""
    x = _f64(x)
    codes = np.empty(x.shape, dtype=np.uint8)
    lib().orc_fp8_encode(x.size, _p(x.reshape(-1)),
                         codes.reshape(-1).ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return codes


def fp8_decode(codes):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    lib().orc_fp8_decode(codes.size, codes.reshape(-1).ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                         _p(out.reshape(-1)))
    return out


def quant_fp8(x):
    """Snapshot storage in FP8 E4M3: decode(encode(x))."""
    return fp8_decode(fp8_encode(x))


def residual(d, d_obs):
    d, d_obs = _f64(d), _f64(d_obs)
    res = np.empty_like(d)
    J = lib().orc_residual(d.size, _p(d.reshape(-1)), _p(d_obs.reshape(-1)), _p(res.reshape(-1)))
    return res, J


# --------------------------------------------------------------------------

@dataclass
class Sim:
    """One simulation setup.  Arrays are converted to fp64 C-contiguous.

    ca, cb: [ny, nx] shared or [S, ny, nx] batched.  cq: scalar or an array
    shaped like ca.  prof_y / prof_x: (a, ah, b, bh, k, kh) tuples.
    src_idx [S, n_src], rec_idx [S, n_rec]: flat cell indices y*nx + x, -1 off.
    """
    ny: int
    nx: int
    order: int
    dy: float
    dx: float
    ca: np.ndarray
    cb: np.ndarray
    cq: object
    prof_y: tuple
    prof_x: tuple
    src_idx: np.ndarray
    rec_idx: np.ndarray
    _keep: list = field(default_factory=list, repr=False)

    def __post_init__(self):
        self.ca = _f64(self.ca)
        self.cb = _f64(self.cb)
        self.model_batched = int(self.ca.ndim == 3)
        cq = np.asarray(self.cq, dtype=np.float64)
        self.cq_is_array = int(cq.ndim > 0 and cq.size > 1)
        self.cq = np.ascontiguousarray(cq.reshape(-1) if self.cq_is_array else cq.reshape(1))
        self.prof_y = tuple(_f64(v) for v in self.prof_y)
        self.prof_x = tuple(_f64(v) for v in self.prof_x)
        self.src_idx = np.ascontiguousarray(self.src_idx, dtype=np.int64)
        self.rec_idx = np.ascontiguousarray(self.rec_idx, dtype=np.int64)
        assert self.src_idx.ndim == 2 and self.rec_idx.ndim == 2
        assert self.src_idx.shape[0] == self.rec_idx.shape[0]
        self.n_shots = self.src_idx.shape[0]
        if self.model_batched:
            assert self.ca.shape == (self.n_shots, self.ny, self.nx)
        else:
            assert self.ca.shape == (self.ny, self.nx)
        assert self.cb.shape == self.ca.shape

    @property
    def n_src(self):
        return self.src_idx.shape[1]

    @property
    def n_rec(self):
        return self.rec_idx.shape[1]

    def _struct(self):
        ay, ayh, by, byh, ky, kyh = self.prof_y
        ax, axh, bx, bxh, kx, kxh = self.prof_x
        s = _Sim(self.ny, self.nx, self.order, self.n_shots, self.n_src, self.n_rec,
                 self.dy, self.dx, self.model_batched, self.cq_is_array,
                 _p(self.ca), _p(self.cb), _p(self.cq),
                 _p(ay), _p(ayh), _p(by), _p(byh), _p(ky), _p(kyh),
                 _p(ax), _p(axh), _p(bx), _p(bxh), _p(kx), _p(kxh),
                 self.src_idx.ctypes.data_as(_I64), self.rec_idx.ctypes.data_as(_I64))
        return s

    def zero_state(self):
        return np.zeros((NFIELD, self.n_shots, self.ny, self.nx))

    def forward(self, f, nt=None, state=None, snapshots=False, records=True):
        """Run nt steps.  Returns dict(rec, state, snap_ey, snap_curl)."""
        f = _f64(f)
        nt = f.shape[0] if nt is None else nt
        if f.size == 0:
            f = np.zeros((max(nt, 1), self.n_shots, max(self.n_src, 1)))
        state = self.zero_state() if state is None else _f64(state).copy()
        rec = np.zeros((nt, self.n_shots, self.n_rec)) if records else None
        sey = np.zeros((nt, self.n_shots, self.ny, self.nx)) if snapshots else None
        scu = np.zeros((nt, self.n_shots, self.ny, self.nx)) if snapshots else None
        st = self._struct()
        rc = lib().orc_forward(ctypes.byref(st), nt, _p(f), _p(state), _p(rec), _p(sey), _p(scu))
        if rc != 0:
            raise RuntimeError(f"orc_forward failed: {rc}")
        return dict(rec=rec, state=state, snap_ey=sey, snap_curl=scu)

    def adjoint(self, res, snap_ey=None, snap_curl=None, adj=None, grad_f=True):
        """Reverse sweep.  Returns dict(gca, gcb, grad_f, adj) with per-shot gradients."""
        res = _f64(res)
        nt = res.shape[0]
        if res.size == 0:
            res = np.zeros((max(nt, 1), self.n_shots, max(self.n_rec, 1)))
        adj = self.zero_state() if adj is None else _f64(adj).copy()
        gca = np.zeros((self.n_shots, self.ny, self.nx))
        gcb = np.zeros((self.n_shots, self.ny, self.nx))
        gf = np.zeros((nt, self.n_shots, self.n_src)) if grad_f else None
        st = self._struct()
        rc = lib().orc_adjoint(ctypes.byref(st), nt, _p(res), _p(_f64(snap_ey)),
                               _p(_f64(snap_curl)), _p(adj), _p(gca), _p(gcb), _p(gf))
        if rc != 0:
            raise RuntimeError(f"orc_adjoint failed: {rc}")
        return dict(gca=gca, gcb=gcb, grad_f=gf, adj=adj)

    def born(self, snap_ey, snap_curl, dca, dcb, nt=None, state=None):
        """Born (linearised) forward: records [nt, S, n_rec] of the derivative
        of the forward's records in the direction (dCa, dCb), given the
        background's snapshots (forward(..., snapshots=True)).  The
        transpose of this map is the adjoint's (shot-summed) gradient."""
        snap_ey, snap_curl = _f64(snap_ey), _f64(snap_curl)
        nt = snap_ey.shape[0] if nt is None else nt
        dca = _f64(np.broadcast_to(dca, self.ca.shape))
        dcb = _f64(np.broadcast_to(dcb, self.ca.shape))
        state = self.zero_state() if state is None else _f64(state).copy()
        rec = np.zeros((nt, self.n_shots, self.n_rec))
        st = self._struct()
        rc = lib().orc_born(ctypes.byref(st), nt, _p(snap_ey), _p(snap_curl), _p(dca), _p(dcb),
                            _p(state), _p(rec))
        if rc != 0:
            raise RuntimeError(f"orc_born failed: {rc}")
        return rec

    def fwd_adj_ckpt(self, f, res, C, nt=None, state0=None, records=True, grad_f=True):
        """Checkpointed forward + replayed adjoint (memory O(nt/C state + C snapshots))."""
        f = _f64(f)
        nt = f.shape[0] if nt is None else nt
        res = None if res is None else _f64(res)
        rec = np.zeros((nt, self.n_shots, self.n_rec)) if records else None
        gca = np.zeros((self.n_shots, self.ny, self.nx))
        gcb = np.zeros((self.n_shots, self.ny, self.nx))
        gf = np.zeros((nt, self.n_shots, self.n_src)) if (grad_f and res is not None) else None
        st = self._struct()
        rc = lib().orc_fwd_adj_ckpt(ctypes.byref(st), nt, C, _p(f), _p(_f64(state0)), _p(rec),
                                    _p(res), _p(gca), _p(gcb), _p(gf))
        if rc != 0:
            raise RuntimeError(f"orc_fwd_adj_ckpt failed: {rc}")
        return dict(rec=rec, gca=gca, gcb=gcb, grad_f=gf)


def num_threads() -> int:
    return lib().orc_num_threads()
