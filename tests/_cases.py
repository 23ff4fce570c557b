"""Shared test set-up: builds oracle simulations from the seeded inputs.

Only the oracle's own functions are used here (model coefficients, CPML
profiles, CFL bound); the CUDA library is never called from this module.
"""
from __future__ import annotations

import numpy as np

import oracle
from adjoint_state_gradients_b200 import synth


def profiles(ny, nx, n_pml, dy, dx, dt, vmax, f0, R=1e-3):
    py = oracle.cpml(ny, n_pml, dy, dt, vmax, f0, R)
    px = oracle.cpml(nx, n_pml, dx, dt, vmax, f0, R)
    return py, px


def oracle_sim(eps_r, sigma, src_idx, rec_idx, order, h, dt, n_pml, f0, mu_r=None, vmax=None,
               cq_array=False, round_f32=True):
    """Oracle Sim for a model.  With round_f32 the coefficient arrays are
    rounded to fp32 first (the values the CUDA path consumes), then used in
    fp64 arithmetic."""
    eps_r = np.asarray(eps_r, dtype=np.float64)
    ny, nx = eps_r.shape[-2:]
    ca, cb, cq = oracle.model(eps_r, sigma, mu_r, dt)
    if vmax is None:
        vmax = oracle.c0() / np.sqrt(eps_r.min())
    py, px = profiles(ny, nx, n_pml, h, h, dt, vmax, f0)
    cqv = cq if (cq_array or mu_r is not None) else cq.reshape(-1)[0]
    if round_f32:
        r = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
        ca, cb = r(ca), r(cb)
        cqv = r(cqv) if np.ndim(cqv) else float(np.float32(cqv))
        py = tuple(r(v) for v in py)
        px = tuple(r(v) for v in px)
    return oracle.Sim(ny=ny, nx=nx, order=order, dy=h, dx=h, ca=ca, cb=cb, cq=cqv,
                      prof_y=py, prof_x=px, src_idx=src_idx, rec_idx=rec_idx)


def workload_sim(number, n_shots=None, nt=None, round_f32=True, true_model=False):
    """(sim, inputs, dt, f) for one of the five workloads (first n_shots)."""
    inp = synth.make_inputs(number, n_shots)
    wl = inp.wl
    vmax = oracle.c0() / np.sqrt(inp.eps_min)
    dt = wl.cfl_fraction * oracle.cfl_dt(wl.order, wl.h, wl.h, vmax)
    eps = inp.eps_r_true if true_model else inp.eps_r
    sim = oracle_sim(eps, inp.sigma, inp.src_idx, inp.rec_idx, wl.order, wl.h, dt, wl.n_pml,
                     wl.f0, vmax=vmax, round_f32=round_f32)
    f = inp.wavelet(dt, wl.nt if nt is None else nt)
    if round_f32:
        f = f.astype(np.float32).astype(np.float64)
    return sim, inp, dt, f


def small_sim(seed, ny, nx, S, ns, nr, order, n_pml, h=0.02, f0=400e6, frac=0.6, sigma_max=0.01,
              batched=False, cq_array=False, round_f32=False, eps_lo=2.0, eps_hi=6.0):
    eps, sig, src, rec = synth.small_case(seed, ny, nx, S, ns, nr, eps_lo=eps_lo, eps_hi=eps_hi,
                                          sigma_max=sigma_max, batched=batched)
    vmax = oracle.c0() / np.sqrt(eps.min())
    dt = frac * oracle.cfl_dt(order, h, h, vmax)
    mu = None
    if cq_array:
        g = synth.rng(seed + 77)
        mu = g.uniform(1.0, 2.0, size=eps.shape)
    sim = oracle_sim(eps, sig, src, rec, order, h, dt, n_pml, f0, mu_r=mu, vmax=vmax,
                     cq_array=cq_array, round_f32=round_f32)
    return sim, dt, (eps, sig, mu)


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))
