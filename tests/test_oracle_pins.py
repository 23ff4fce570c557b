"""Pins of the fp64 oracle against mathematics (no GPU, no CUDA library).

Each test checks the oracle against something other than itself: exact
rational Taylor conditions, order of accuracy, an exact discrete invariant,
the adjoint (dot-product) identity, central finite differences, the von
Neumann bound measured by power iteration, reciprocity, the physical wave
speed, and the constant printed on the maxwell.cu page.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from adjoint_state_gradients_b200 import synth
from tests._cases import oracle_sim, profiles, rel_l2, small_sim

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    return vals


# ----------------------------------------------------------------------------
# stencil coefficients


def _taylor_staggered(P):
    """Solve sum_k c_k (2k-1)^(2m+1) = [m == 0], m = 0..P-1, in exact rationals."""
    A = [[Fraction((2 * k - 1) ** (2 * m + 1)) for k in range(1, P + 1)] for m in range(P)]
    b = [Fraction(1 if m == 0 else 0) for m in range(P)]
    n = P
    for i in range(n):  # Gauss-Jordan
        piv = next(r for r in range(i, n) if A[r][i] != 0)
        A[i], A[piv] = A[piv], A[i]
        b[i], b[piv] = b[piv], b[i]
        for r in range(n):
            if r != i and A[r][i] != 0:
                f = A[r][i] / A[i][i]
                A[r] = [x - f * y for x, y in zip(A[r], A[i])]
                b[r] -= f * b[i]
    return [b[i] / A[i][i] for i in range(n)]


@pytest.mark.parametrize("order", [2, 4, 6, 8])
def test_stencil_coefficients_solve_taylor_conditions(order):
    exact = _taylor_staggered(order // 2)
    got = oracle.coeffs(order)
    assert len(got) == order // 2
    for g, e in zip(got, exact):
        assert g == float(e)


def _one_step(sim, state):
    return sim.forward(np.zeros((1, sim.n_shots, sim.n_src)), nt=1, state=state, records=False)["state"]


def _deriv_sim(n, order, h):
    """Uniform medium, no PML, Ca = 1, Cb = Cq = 1 so one step exposes the difference operators."""
    ca = np.ones((n, n))
    cb = np.ones((n, n))
    z = np.zeros(n)
    one = np.ones(n)
    prof = (z, z, z, z, one, one)
    idx = np.zeros((1, 0), dtype=np.int64)
    return oracle.Sim(ny=n, nx=n, order=order, dy=h, dx=h, ca=ca, cb=cb, cq=1.0, prof_y=prof, prof_x=prof,
                      src_idx=idx, rec_idx=idx)


@pytest.mark.parametrize("order", [2, 4, 6, 8])
def test_difference_operators_converge_at_their_order(order):
    """D^h applied to a smooth field matches d/dx at the half node with error
    O(h^order); D from half nodes matches at the integer node.  A wrong
    coefficient, stagger offset, sign or axis breaks the rate."""
    k = 12.0  # wavenumber (rad / unit length); domain [0, 1]
    errs_h, errs_i = [], []
    hs = [1.0 / 40, 1.0 / 80]
    for h in hs:
        n = int(round(1.0 / h))
        sim = _deriv_sim(n, order, h)
        y = np.arange(n)[:, None] * h
        x = np.arange(n)[None, :] * h
        st = sim.zero_state()
        st[0, 0] = np.sin(k * x + 0.3) * np.cos(k * y + 0.7)
        sim.ca[:] = 0.0  # keep E out of the E update so it only shows D of H
        sim.cb[:] = 0.0
        out = _one_step(sim, st)
        hz, hx = out[2, 0], out[1, 0]
        ex_hz = k * np.cos(k * (x + 0.5 * h) + 0.3) * np.cos(k * y + 0.7)  # +dE/dx at x+1/2
        ex_hx = -(-k * np.sin(k * x + 0.3) * np.sin(k * (y + 0.5 * h) + 0.7))  # -dE/dz at y+1/2
        m = order  # stay away from the zero-extended edges
        errs_h.append(max(np.abs(hz - ex_hz)[m:-m, m:-m].max(), np.abs(hx - ex_hx)[m:-m, m:-m].max()))
        # integer-node operator: H fields given at half nodes, E = D_x Hz - D_z Hx
        sim.cb[:] = 1.0
        st = sim.zero_state()
        st[2, 0] = np.sin(k * (x + 0.5 * h) + 0.3) * np.cos(k * y)
        st[1, 0] = np.cos(k * x) * np.sin(k * (y + 0.5 * h) + 0.2)
        out = _one_step(sim, st)
        ex_e = k * np.cos(k * x + 0.3) * np.cos(k * y) - k * np.cos(k * x) * np.cos(k * y + 0.2)
        errs_i.append(np.abs(out[0, 0] - ex_e)[m:-m, m:-m].max())
    for errs in (errs_h, errs_i):
        rate = math.log(errs[0] / errs[1], 2.0)
        assert rate > order - 0.6, (order, errs, rate)


# ----------------------------------------------------------------------------
# model coefficients and constants


def test_eps0_matches_page_constant():
    """The eps_r gradient carries the eps0 printed on the page (EP0)."""
    g = _read_golden("page_constants.txt")
    eps0 = float(g["EP0"])
    # with Ca = 0, Cb = dt, dJ/dCa = 1, dJ/dCb = 0: dJ/deps_r = eps0 * (1 - 0) * dt / dt
    ge, gs = oracle.eps_sigma_grad(np.zeros(1), np.full(1, 1e-9), 1e-9, np.ones(1), np.zeros(1))
    assert ge[0] == pytest.approx(eps0, rel=1e-15)
    # sigma derivative of Ca at Ca = 0: -1/2 (1 + 0) Cb
    assert gs[0] == pytest.approx(-0.5e-9, rel=1e-15)


def test_model_lossless_limit_and_light_speed():
    dt = 1e-11
    ca, cb, cq = oracle.model(np.array([1.0, 4.0]), np.zeros(2), None, dt)
    assert np.all(ca == 1.0)
    # Cb Cq = dt^2 / (eps mu) = (c dt)^2 / eps_r
    c = 299792458.0
    assert cb[0] * cq[0] == pytest.approx((c * dt) ** 2, rel=1e-9)
    assert cb[1] * cq[1] == pytest.approx((c * dt) ** 2 / 4.0, rel=1e-9)
    assert oracle.c0() == pytest.approx(c, rel=1e-9)


def test_model_conductive_decay_is_crank_nicolson():
    """Ca approximates the exact decay exp(-sigma dt / eps) of eps dE/dt = -sigma E
    to third order in sigma dt / eps; Cb is the trapezoidal source weight."""
    eps0 = float(_read_golden("page_constants.txt")["EP0"])
    dt, er = 1e-11, 5.0
    for sig in (1e-3, 1e-2, 1e-1):
        ca, cb, _ = oracle.model(np.array([er]), np.array([sig]), None, dt)
        x = sig * dt / (eps0 * er)
        assert abs(ca[0] - math.exp(-x)) <= 0.1 * x ** 3 + 1e-16
        # integral of exp(-x s) over one step, trapezoid-consistent
        assert cb[0] == pytest.approx(dt / (eps0 * er) * (1 + ca[0]) / 2.0, rel=1e-12)


def test_chain_rule_matches_finite_differences_of_model():
    g = synth.rng(3)
    er = g.uniform(2, 9, size=20)
    sg = g.uniform(0, 0.05, size=20)
    dt = 3e-11
    w_ca, w_cb = g.normal(size=20), g.normal(size=20)

    def J(e, s):
        ca, cb, _ = oracle.model(e, s, None, dt)
        return float(np.dot(w_ca, ca) + np.dot(w_cb, cb))

    ca, cb, _ = oracle.model(er, sg, None, dt)
    ge, gs = oracle.eps_sigma_grad(ca, cb, dt, w_ca, w_cb)
    eps0 = float(_read_golden("page_constants.txt")["EP0"])
    for i in range(0, 20, 3):
        h = 1e-6 * er[i]
        e1, e2 = er.copy(), er.copy()
        e1[i] += h
        e2[i] -= h
        fd = (J(e1, sg) - J(e2, sg)) / (2 * h)
        # dJ/deps_r = eps0 dJ/deps
        assert ge[i] == pytest.approx(fd, rel=1e-6, abs=1e-12 * abs(ge).max())
        hs = 1e-6 * max(sg[i], 1e-3)
        s1, s2 = sg.copy(), sg.copy()
        s1[i] += hs
        s2[i] -= hs
        fd = (J(er, s1) - J(er, s2)) / (2 * hs)
        assert gs[i] == pytest.approx(fd, rel=1e-6, abs=1e-12 * abs(gs).max())
    assert eps0 > 0


# ----------------------------------------------------------------------------
# invariants of the time stepping


def _lossless_sim(n, order, h=0.01, frac=0.9, eps_field=True, seed=0):
    g = synth.rng(seed)
    eps = synth.smooth_field(g, (n, n), 3.0, 1.5, 5.0) if eps_field else np.full((n, n), 3.0)
    mu = synth.smooth_field(g, (n, n), 3.0, 1.0, 2.0)
    vmax = oracle.c0() / math.sqrt((eps * mu).min())
    dt = frac * oracle.cfl_dt(order, h, h, vmax)
    idx = np.zeros((1, 0), dtype=np.int64)
    sim = oracle_sim(eps, np.zeros_like(eps), idx, idx, order, h, dt, 0, 1e8, mu_r=mu, vmax=vmax,
                     round_f32=False)
    return sim, dt, eps, mu


def _energy(sim, st_before, st_after, eps, mu):
    """W^n = sum eps (E^n)^2 + sum mu H^{n-1/2} . H^{n+1/2}, with the absolute
    eps = dt / Cb and mu = dt / Cq of the lossless scheme (dt factored out)."""
    e = st_before[0, 0]
    hb = st_before[1:3, 0]
    ha = st_after[1:3, 0]
    w_e = 1.0 / sim.cb
    w_h = 1.0 / sim.cq.reshape(sim.ny, sim.nx) if sim.cq_is_array else 1.0 / sim.cq[0]
    return float(np.sum(w_e * e * e) + np.sum(w_h * hb * ha))


@pytest.mark.parametrize("order", [2, 4, 8])
def test_energy_is_conserved_without_loss(order):
    n = 40
    sim, dt, eps, mu = _lossless_sim(n, order, seed=order)
    g = synth.rng(10 + order)
    st = sim.zero_state()
    st[0, 0] = synth.smooth_field(g, (n, n), 2.0, -1.0, 1.0)
    st[1, 0] = 1e-3 * synth.smooth_field(g, (n, n), 2.0, -1.0, 1.0)
    st[2, 0] = 1e-3 * synth.smooth_field(g, (n, n), 2.0, -1.0, 1.0)
    nxt = _one_step(sim, st)
    W0 = _energy(sim, st, nxt, eps, mu)
    assert W0 > 0
    worst = 0.0
    for _ in range(300):
        st, nxt = nxt, _one_step(sim, nxt)
        worst = max(worst, abs(_energy(sim, st, nxt, eps, mu) - W0) / W0)
    assert worst < 1e-12, worst


def test_energy_decreases_with_conductivity():
    n = 32
    sim, dt, eps, mu = _lossless_sim(n, 4, seed=5)
    ca, cb, _ = oracle.model(eps, np.full_like(eps, 0.05), mu, dt)
    sim.ca[:] = ca
    sim.cb[:] = cb
    g = synth.rng(99)
    st = sim.zero_state()
    st[0, 0] = synth.smooth_field(g, (n, n), 2.0, -1.0, 1.0)
    nxt = _one_step(sim, st)
    W = _energy(sim, st, nxt, eps, mu)
    for _ in range(100):
        st, nxt = nxt, _one_step(sim, nxt)
        W2 = _energy(sim, st, nxt, eps, mu)
        assert W2 <= W * (1 + 1e-13)
        W = W2


@pytest.mark.parametrize("order", [2, 4, 6, 8])
def test_cfl_bound_matches_operator_spectrum(order):
    """Power iteration of M = (E - step(E, H=0)) / dt^2 gives the largest
    eigenvalue of the spatial operator; the leapfrog is stable iff
    dt^2 lambda_max <= 4, and the closed-form dt_max must sit just above
    the exact limit (within a few % on a 48x48 homogeneous grid)."""
    n, h = 48, 0.01
    eps = np.full((n, n), 2.0)
    vmax = oracle.c0() / math.sqrt(2.0)
    dt_max = oracle.cfl_dt(order, h, h, vmax)
    dt = 0.5 * dt_max
    idx = np.zeros((1, 0), dtype=np.int64)
    sim = oracle_sim(eps, np.zeros_like(eps), idx, idx, order, h, dt, 0, 1e8, vmax=vmax, round_f32=False)
    g = synth.rng(order)
    v = g.normal(size=(n, n))
    lam = 0.0
    for _ in range(400):
        v /= np.linalg.norm(v)
        st = sim.zero_state()
        st[0, 0] = v
        out = _one_step(sim, st)
        w = (v - out[0, 0]) / dt ** 2
        lam = float(np.dot(w.ravel(), v.ravel()))
        v = w
    dt_exact = 2.0 / math.sqrt(lam)
    assert dt_exact >= dt_max * (1 - 1e-9)
    assert dt_exact <= dt_max * 1.05


@pytest.mark.parametrize("order", [2, 4])
def test_cfl_growth_threshold(order):
    n, h = 24, 0.01
    eps = np.full((n, n), 2.0)
    vmax = oracle.c0() / math.sqrt(2.0)
    dt_max = oracle.cfl_dt(order, h, h, vmax)
    idx = np.zeros((1, 0), dtype=np.int64)
    g = synth.rng(1)
    init = g.normal(size=(n, n))
    out = {}
    for frac in (0.99, 1.10):
        sim = oracle_sim(eps, np.zeros_like(eps), idx, idx, order, h, frac * dt_max, 0, 1e8, vmax=vmax,
                         round_f32=False)
        st = sim.zero_state()
        st[0, 0] = init
        st = sim.forward(np.zeros((3000, 1, 0)), nt=3000, state=st, records=False)["state"]
        out[frac] = np.abs(st[0, 0]).max()
    assert out[0.99] < 10 * np.abs(init).max()
    # unstable run: grows without bound (may overflow to inf / nan)
    assert not (out[1.10] <= 1e6 * np.abs(init).max())


# ----------------------------------------------------------------------------
# adjoint identities


@pytest.mark.parametrize("order,batched,cq_array", [(2, False, False), (4, True, False), (6, False, True),
                                                     (8, False, False)])
def test_dot_product_record_map(order, batched, cq_array):
    """<A f, y> = <f, A^T y> with A: wavelet -> records, CPML on, sigma > 0."""
    sim, dt, _ = small_sim(11 + order, 23, 29, 2, 3, 5, order, 6, batched=batched, cq_array=cq_array)
    nt = 60
    g = synth.rng(100 + order)
    f = g.normal(size=(nt, sim.n_shots, sim.n_src))
    y = g.normal(size=(nt, sim.n_shots, sim.n_rec))
    r = sim.forward(f)["rec"]
    gf = sim.adjoint(y)["grad_f"]
    lhs, rhs = float(np.sum(r * y)), float(np.sum(f * gf))
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), abs(rhs)), (lhs, rhs)


@pytest.mark.parametrize("order", [2, 4, 6, 8])
def test_dot_product_state_map(order):
    """<A x0, y> = <x0, A^T y> on the full 7-field state (fields and CPML
    memories), with sources and receivers inactive."""
    sim, dt, _ = small_sim(21 + order, 22, 19, 2, 1, 1, order, 5)
    sim.src_idx[:] = -1
    sim.rec_idx[:] = -1
    nt = 40
    g = synth.rng(200 + order)
    x0 = g.normal(size=sim.zero_state().shape)
    yT = g.normal(size=sim.zero_state().shape)
    xT = sim.forward(np.zeros((nt, sim.n_shots, sim.n_src)), state=x0, records=False)["state"]
    a0 = sim.adjoint(np.zeros((nt, sim.n_shots, sim.n_rec)), adj=yT, grad_f=False)["adj"]
    lhs, rhs = float(np.sum(xT * yT)), float(np.sum(x0 * a0))
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), abs(rhs)), (lhs, rhs)


def _misfit(sim, f, d_obs):
    """J = 1/2 ||d - d_obs||^2 as the oracle's residual routine returns it."""
    return oracle.residual(sim.forward(f)["rec"], d_obs)[1]


@pytest.mark.parametrize("order,n_pml", [(2, 3), (4, 3), (4, 0)])
def test_model_gradient_matches_central_differences_16x16(order, n_pml):
    """dJ/dCa and dJ/dCb on every cell of a 16x16 grid (10x10 interior + 3-cell
    CPML, and a no-PML variant), J = 1/2 ||d - d_obs||^2, two shots summed.

    Both the misfit J the differences are taken of and the residual the
    adjoint is driven by come from the oracle's residual routine, so a wrong
    factor or sign in it (J without the 1/2, res = d_obs - d) breaks the
    agreement."""
    n = 16
    sim, dt, (eps, sig, _) = small_sim(31 + order, n, n, 2, 1, 4, order, n_pml, sigma_max=0.02)
    nt = 80
    f = np.broadcast_to(synth.ricker(nt, dt, 400e6)[:, None, None], (nt, 2, 1)).copy()
    g = synth.rng(5)
    d_obs = sim.forward(f)["rec"] * (1 + 0.1 * g.normal(size=(nt, 2, sim.n_rec)))
    fw = sim.forward(f, snapshots=True)
    res, _ = oracle.residual(fw["rec"], d_obs)
    adj = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"])
    gca = oracle.combine(adj["gca"])
    gcb = oracle.combine(adj["gcb"])
    fd_ca = np.zeros((n, n))
    fd_cb = np.zeros((n, n))
    ca0, cb0 = sim.ca.copy(), sim.cb.copy()
    for arr, base, out in ((sim.ca, ca0, fd_ca), (sim.cb, cb0, fd_cb)):
        for j in range(n * n):
            y, x = divmod(j, n)
            h = 1e-6 * abs(base[y, x])
            arr[y, x] = base[y, x] + h
            jp = _misfit(sim, f, d_obs)
            arr[y, x] = base[y, x] - h
            jm = _misfit(sim, f, d_obs)
            arr[y, x] = base[y, x]
            out[y, x] = (jp - jm) / (2 * h)
    assert rel_l2(gca, fd_ca) <= 1e-6, rel_l2(gca, fd_ca)
    assert rel_l2(gcb, fd_cb) <= 1e-6, rel_l2(gcb, fd_cb)


def test_eps_sigma_gradient_matches_central_differences():
    n, order, nt = 16, 4, 60
    sim, dt, (eps, sig, _) = small_sim(41, n, n, 1, 1, 4, order, 3, sigma_max=0.02)
    f = synth.ricker(nt, dt, 400e6)[:, None, None].copy()
    d_obs = 0.9 * sim.forward(f)["rec"]

    def J(e, s):
        ca, cb, _ = oracle.model(e, s, None, dt)
        sim.ca[:] = ca
        sim.cb[:] = cb
        return _misfit(sim, f, d_obs)

    ca, cb, _ = oracle.model(eps, sig, None, dt)
    sim.ca[:] = ca
    sim.cb[:] = cb
    fw = sim.forward(f, snapshots=True)
    adj = sim.adjoint(fw["rec"] - d_obs, fw["snap_ey"], fw["snap_curl"])
    ge, gs = oracle.eps_sigma_grad(ca, cb, dt, adj["gca"][0], adj["gcb"][0])
    g = synth.rng(7)
    for _ in range(6):
        y, x = g.integers(3, 13, size=2)
        h = 1e-6 * eps[y, x]
        e1, e2 = eps.copy(), eps.copy()
        e1[y, x] += h
        e2[y, x] -= h
        fd = (J(e1, sig) - J(e2, sig)) / (2 * h)
        assert ge[y, x] == pytest.approx(fd, rel=1e-5, abs=1e-8 * np.abs(ge).max())
        hs = 1e-4 * max(sig[y, x], 1e-3)
        s1, s2 = sig.copy(), sig.copy()
        s1[y, x] += hs
        s2[y, x] -= hs
        fd = (J(eps, s1) - J(eps, s2)) / (2 * hs)
        assert gs[y, x] == pytest.approx(fd, rel=1e-5, abs=1e-8 * np.abs(gs).max())


def test_source_gradient_matches_central_differences():
    sim, dt, _ = small_sim(51, 18, 18, 1, 2, 3, 4, 4)
    nt = 50
    g = synth.rng(8)
    f = g.normal(size=(nt, 1, 2))
    d_obs = g.normal(size=(nt, 1, 3))
    res = sim.forward(f)["rec"] - d_obs
    gf = sim.adjoint(res)["grad_f"]
    for (t, k) in ((0, 0), (10, 1), (49, 0)):
        h = 1e-5
        f1, f2 = f.copy(), f.copy()
        f1[t, 0, k] += h
        f2[t, 0, k] -= h
        fd = (_misfit(sim, f1, d_obs) - _misfit(sim, f2, d_obs)) / (2 * h)
        assert gf[t, 0, k] == pytest.approx(fd, rel=1e-7, abs=1e-10)


def test_reciprocity_without_pml():
    """Cb(s) d(r <- s) = Cb(r) d(s <- r) for raw injection into Ey (lossy,
    heterogeneous medium, no PML)."""
    n, order = 30, 4
    g = synth.rng(61)
    eps = synth.smooth_field(g, (n, n), 3.0, 2.0, 6.0)
    sig = g.uniform(0.0, 0.02, size=(n, n))
    a, b = 7 * n + 9, 21 * n + 18
    vmax = oracle.c0() / math.sqrt(eps.min())
    dt = 0.6 * oracle.cfl_dt(order, 0.02, 0.02, vmax)
    nt = 150
    f = synth.ricker(nt, dt, 400e6)[:, None, None].copy()

    def run(s, r):
        sim = oracle_sim(eps, sig, np.array([[s]]), np.array([[r]]), order, 0.02, dt, 0, 4e8, vmax=vmax,
                         round_f32=False)
        return sim.forward(f)["rec"][:, 0, 0], sim.cb.reshape(-1)

    d_ab, cbv = run(a, b)
    d_ba, _ = run(b, a)
    lhs = cbv[a] * d_ab
    rhs = cbv[b] * d_ba
    assert np.abs(lhs).max() > 0
    assert np.abs(lhs - rhs).max() <= 1e-10 * np.abs(lhs).max()


def test_linearity_duplicate_and_inactive_sources():
    sim, dt, _ = small_sim(71, 20, 20, 1, 3, 4, 4, 4)
    sim.src_idx[0] = [55, 55, -1]
    nt = 40
    g = synth.rng(9)
    f = g.normal(size=(nt, 1, 3))
    r = sim.forward(f)["rec"]
    sim2, _, _ = small_sim(71, 20, 20, 1, 1, 4, 4, 4)
    sim2.src_idx[0] = [55]
    sim2.rec_idx[:] = sim.rec_idx
    r2 = sim2.forward((f[:, :, 0] + f[:, :, 1])[:, :, None])["rec"]
    assert rel_l2(r, r2) < 1e-14


# ----------------------------------------------------------------------------
# physics: wave speed and absorbing boundary


def test_plane_wave_speed():
    """Delay between two far-field receivers on one ray equals the distance
    over c0 / sqrt(eps_r) within numerical dispersion (well-resolved pulse)."""
    n, h, er, order = 220, 0.01, 4.0, 4
    eps = np.full((n, n), er)
    c = oracle.c0() / math.sqrt(er)
    f0 = c / (30 * h)  # ~30 cells per peak wavelength
    dt = 0.5 * oracle.cfl_dt(order, h, h, c)
    s = 110 * n + 40
    rec = np.array([[110 * n + 100, 110 * n + 160]])
    sim = oracle_sim(eps, np.zeros_like(eps), np.array([[s]]), rec, order, h, dt, 0, f0, vmax=c,
                     round_f32=False)
    nt = int(2.6 * (120 * h / c) / dt)
    f = synth.ricker(nt, dt, f0)[:, None, None].copy()
    r = sim.forward(f)["rec"][:, 0, :]
    a, b = r[:, 0], r[:, 1]
    xc = np.correlate(b, a, mode="full")
    k = int(np.argmax(xc))
    y0, y1, y2 = xc[k - 1], xc[k], xc[k + 1]
    frac = 0.5 * (y0 - y2) / (y0 - 2 * y1 + y2)
    lag = (k - (len(a) - 1) + frac) * dt
    expected = 60 * h / c
    assert lag == pytest.approx(expected, rel=0.01)


def test_cpml_absorbs_outgoing_waves():
    """With the CPML band the field energy left after the pulse has crossed
    the domain is a small fraction of its peak; with a bare (lossless) edge
    it stays."""
    n, h, order = 80, 0.02, 4
    eps = np.full((n, n), 4.0)
    c = oracle.c0() / 2.0
    f0 = 400e6
    dt = 0.6 * oracle.cfl_dt(order, h, h, c)
    src = np.array([[40 * n + 40]])
    rec = np.zeros((1, 0), dtype=np.int64)
    nt = int(4.0 * (n * h / c) / dt)
    f = synth.ricker(nt, dt, f0)[:, None, None].copy()
    energy = {}
    for npml in (0, 15):
        sim = oracle_sim(eps, np.zeros_like(eps), src, rec, order, h, dt, npml, f0, vmax=c, round_f32=False)
        st = sim.zero_state()
        peak = 0.0
        chunk = nt // 8
        for i in range(8):
            st = sim.forward(f[i * chunk:(i + 1) * chunk], state=st, records=False)["state"]
            e = float(np.sum(st[0, 0, 15:-15, 15:-15] ** 2))
            peak = max(peak, e)
        energy[npml] = (e, peak)
    assert energy[0][0] > 0.1 * energy[0][1]
    assert energy[15][0] < 1e-3 * energy[15][1]


def test_cpml_profile_shape():
    n, npml, h, dt = 50, 10, 0.02, 4e-11
    a, ah, b, bh, k, kh = oracle.cpml(n, npml, h, dt, 1.5e8, 4e8)
    inner = slice(npml + 1, n - npml - 1)
    assert np.all(a[inner] == 0) and np.all(b[inner] == 0) and np.all(k == 1)
    band = np.r_[0:npml, n - npml:n]
    assert np.all(a[band] < 0) and np.all((b[band] > 0) & (b[band] < 1))
    hband = np.r_[0:npml, n - npml - 1:n]
    assert np.all(ah[hband] < 0) and np.all((bh[hband] > 0) & (bh[hband] < 1))
    # zero outside the half band too
    hin = np.setdiff1d(np.arange(n), hband)
    assert np.all(ah[hin] == 0) and np.all(bh[hin] == 0)
    # symmetric: left integer node i mirrors right integer node n-1-i
    assert np.allclose(a[:npml], a[::-1][:npml], rtol=1e-14)


# ----------------------------------------------------------------------------
# checkpoint replay


@pytest.mark.parametrize("C", [1, 7, 16, 64])
def test_checkpoint_replay_equals_full_storage(C):
    sim, dt, _ = small_sim(81, 21, 27, 2, 1, 6, 4, 4)
    nt = 45  # not a multiple of 7 / 16; shorter than 64
    g = synth.rng(10)
    f = g.normal(size=(nt, 2, 1))
    res = g.normal(size=(nt, 2, 6))
    fw = sim.forward(f, snapshots=True)
    adj = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"])
    ck = sim.fwd_adj_ckpt(f, res, C)
    assert np.array_equal(ck["rec"], fw["rec"])
    assert np.array_equal(ck["gca"], adj["gca"])
    assert np.array_equal(ck["gcb"], adj["gcb"])
    assert np.array_equal(ck["grad_f"], adj["grad_f"])


def test_combine_is_fixed_order_shot_sum():
    g = synth.rng(12)
    gs = g.normal(size=(5, 7, 9))
    out = oracle.combine(gs)
    ref = gs[0] + gs[1] + gs[2] + gs[3] + gs[4]
    assert np.array_equal(out, ref)


def test_residual_worked_example():
    """d = (3, 1, -2), d_obs = (1, 2, -2): residual (2, -1, 0), J = (4 + 1) / 2."""
    res, J = oracle.residual(np.array([3.0, 1.0, -2.0]), np.array([1.0, 2.0, -2.0]))
    assert list(res) == [2.0, -1.0, 0.0]
    assert J == 2.5


def test_residual_and_misfit():
    g = synth.rng(13)
    d, o = g.normal(size=100), g.normal(size=100)
    res, J = oracle.residual(d, o)
    assert np.allclose(res, d - o, rtol=0, atol=0)
    assert J == pytest.approx(0.5 * np.sum((d - o) ** 2), rel=1e-14)


def test_workload_configs_are_stable_and_shaped():
    for num in (1, 2, 4):
        inp = synth.make_inputs(num, n_shots=1)
        wl = inp.wl
        assert inp.eps_r.shape == (wl.ny, wl.nx)
        assert inp.rec_idx.shape == (1, wl.n_rec)
        assert np.all((inp.src_idx >= 0) & (inp.src_idx < wl.ny * wl.nx))
        assert inp.eps_r.min() >= 2.99
    # published time steps (0.5 / 0.6 of the CFL bound of the smallest eps_r)
    inp = synth.make_inputs(4, n_shots=1)
    dt = 0.6 * oracle.cfl_dt(4, 0.02, 0.02, oracle.c0() / math.sqrt(inp.eps_min))
    assert dt == pytest.approx(4.20e-11, rel=0.01)


# ----------------------------------------------------------------------------
# snapshot storage formats (bfloat16, FP8 E4M3 with saturation)


def test_fp8_e4m3_code_table_follows_the_format_definition():
    """1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent field 0 holds
    subnormals m * 2^-9; S.1111.111 is NaN, so 448 is the largest value."""
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.fp8_decode(codes)
    assert v[0x00] == 0.0 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x08] == 2.0 ** -6 and v[0x38] == 1.0 and v[0x39] == 1.125
    assert v[0x7E] == 448.0 and np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.all(v[0x80:0xFF] == -v[0x00:0x7F])
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)
    # encoding a representable value gives its code back
    assert np.all(oracle.fp8_encode(pos) == codes[:0x7F])
    assert np.all(oracle.fp8_encode(-pos[1:]) == codes[0x81:0xFF])


def test_fp8_e4m3_rounds_to_nearest_even_and_saturates():
    v = oracle.fp8_decode(np.arange(0x7F, dtype=np.uint8))
    mid = (v[:-1] + v[1:]) / 2          # exact ties between neighbouring codes
    got = oracle.fp8_encode(mid)
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)  # the even code wins a tie
    assert np.all(got == want)
    # just off the tie goes to the nearer code
    assert np.all(oracle.fp8_encode(mid * (1 - 1e-6)) == lo)
    assert np.all(oracle.fp8_encode(mid * (1 + 1e-6)) == lo + 1)
    # saturation to the largest finite value, both signs
    assert list(oracle.fp8_encode(np.array([448.0, 464.0, 1e6, -1e30]))) == [0x7E, 0x7E, 0x7E, 0xFE]
    # underflow: half the smallest subnormal is a tie to zero (even)
    assert list(oracle.fp8_encode(np.array([2.0 ** -10, 1.5 * 2.0 ** -10, 1e-30]))) == [0, 1, 0]


def test_bf16_rounds_to_nearest_even():
    one = 1.0
    x = np.array([one + 2.0 ** -8, one + 3 * 2.0 ** -8, one + 2.0 ** -8 + 2.0 ** -20, -(one + 2.0 ** -8)])
    assert list(oracle.quant_bf16(x)) == [1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7, -1.0]
    # the value is first rounded to fp32
    assert oracle.quant_bf16(np.array([1.0 + 2.0 ** -30]))[0] == 1.0


def test_storage_formats_match_torch_casts():
    """Against an independent implementation: torch's float32 -> bfloat16 and
    float32 -> float8_e4m3fn casts (both nearest-even) inside the range."""
    g = np.random.default_rng(5)
    x = g.normal(size=50000) * 10.0 ** g.uniform(-5, 2.6, size=50000)
    x = x[np.abs(x) < 448].astype(np.float32).astype(np.float64)
    t = torch.tensor(x, dtype=torch.float32)
    assert np.array_equal(oracle.quant_fp8(x), t.to(torch.float8_e4m3fn).double().numpy())
    assert np.array_equal(oracle.quant_bf16(x), t.to(torch.bfloat16).double().numpy())


# ----------------------------------------------------------------------------
# Born (linearised) forward


def _born_case(batched=False):
    sim, dt, _ = small_sim(321, 24, 28, 2, 1, 5, 4, 4, batched=batched, round_f32=False,
                           sigma_max=0.02)
    nt = 40
    g = synth.rng(3210)
    f = g.normal(size=(nt, 2, 1))
    dca = 0.01 * g.normal(size=sim.ca.shape)
    dcb = 0.01 * float(np.mean(sim.cb)) * g.normal(size=sim.ca.shape)
    return sim, f, dca, dcb, g


def _with_model(sim, ca, cb):
    return oracle.Sim(ny=sim.ny, nx=sim.nx, order=sim.order, dy=sim.dy, dx=sim.dx, ca=ca, cb=cb,
                      cq=sim.cq if sim.cq_is_array else float(sim.cq[0]), prof_y=sim.prof_y,
                      prof_x=sim.prof_x, src_idx=sim.src_idx, rec_idx=sim.rec_idx)


def test_born_forward_is_the_derivative_of_the_records():
    """Central difference of the forward's records along (dCa, dCb) against
    the Born map (error O(h^2)), with the CPML band on."""
    sim, f, dca, dcb, _ = _born_case()
    fw = sim.forward(f, snapshots=True)
    b = sim.born(fw["snap_ey"], fw["snap_curl"], dca, dcb)
    h = 1e-4
    rp = _with_model(sim, sim.ca + h * dca, sim.cb + h * dcb).forward(f)["rec"]
    rm = _with_model(sim, sim.ca - h * dca, sim.cb - h * dcb).forward(f)["rec"]
    fd = (rp - rm) / (2 * h)
    assert np.abs(b).max() > 0
    assert rel_l2(b, fd) <= 1e-6


@pytest.mark.parametrize("batched", [False, True])
def test_born_forward_is_the_transpose_of_the_gradient(batched):
    """<B dm, r> = <dm, B^T r>, B^T r being the adjoint's gradient (summed
    over shots for a shared model, per shot for a batched one)."""
    sim, f, dca, dcb, g = _born_case(batched)
    fw = sim.forward(f, snapshots=True)
    res = g.normal(size=fw["rec"].shape)
    b = sim.born(fw["snap_ey"], fw["snap_curl"], dca, dcb)
    adj = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"])
    gca, gcb = adj["gca"], adj["gcb"]
    if not batched:
        gca, gcb = gca.sum(axis=0), gcb.sum(axis=0)
    lhs = float(np.sum(b * res))
    rhs = float(np.sum(dca * gca) + np.sum(dcb * gcb))
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), abs(rhs))


@pytest.mark.parametrize("order,n_pml", [(2, 3), (4, 4), (8, 0)])
def test_cb_gradient_regroups_by_summation_by_parts(order, n_pml):
    """The identity the E-alone checkpoint mode evaluates, in fp64: with the
    forward E^{t+1} = Ca E^t + Cb curl^t + s^t and the adjoint's E update
    lam~^t = Ca lam^{t+1} + G^t (lam^{t+1} = lam~^{t+1} + the residual injected
    at step t),
        Cb sum_t curl^t lam^{t+1} = sum_{t>=1} G^t E^t - Ca lam^1 E^0
            + lam~^{nt} E^{nt} + sum_t res[t] rec[t] (receiver cells)
            - sum_t f[t] lam^{t+1} (source cells),
    every end term live: given initial and adjoint states, duplicate and
    inactive indices, a source on a receiver.  The left side is the oracle's
    own gradient; the right side steps the oracle's adjoint one step at a time
    to read lam~^t."""
    S, ny, nx, nt = 2, 20, 24, 30
    sim, dt, _ = small_sim(950 + order, ny, nx, S, 3, 4, order, n_pml, sigma_max=0.02)
    sim.src_idx[0] = [50, 50, -1]
    sim.rec_idx[0, :3] = [50, 77, 77]
    sim.rec_idx[1, 1] = -1
    g = synth.rng(951 + order)
    st0 = np.zeros(sim.zero_state().shape)
    st0[:3] = 0.1 * g.normal(size=st0[:3].shape)
    ad0 = np.zeros_like(st0)
    ad0[:3] = g.normal(size=ad0[:3].shape)
    f = g.normal(size=(nt, S, 3))
    res = g.normal(size=(nt, S, 4))
    fw = sim.forward(f, state=st0, snapshots=True)
    full = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"], adj=ad0)
    ca = np.broadcast_to(sim.ca, (S, ny, nx))
    cb = np.broadcast_to(sim.cb, (S, ny, nx))

    def scatter(idx, vals):  # per-entry values onto their cells; duplicates add
        out = np.zeros((S, ny * nx))
        for s in range(S):
            for k, i in enumerate(idx[s]):
                if i >= 0:
                    out[s, i] += vals[s, k]
        return out.reshape(S, ny, nx)

    def gather(idx, field):
        flat = field.reshape(S, -1)
        return np.array([[flat[s, i] if i >= 0 else 0.0 for i in idx[s]] for s in range(S)])

    rhs = ad0[0] * fw["state"][0]                      # lam~^{nt} E^{nt}
    adj = ad0.copy()
    for t in range(nt - 1, -1, -1):
        lam = adj[0] + scatter(sim.rec_idx, res[t])   # lam^{t+1}
        adj = sim.adjoint(res[t:t + 1], fw["snap_ey"][t:t + 1], fw["snap_curl"][t:t + 1],
                          adj=adj, grad_f=False)["adj"]   # lam~^t
        e_t = fw["snap_ey"][t]
        rhs += (adj[0] - ca * lam) * e_t if t >= 1 else -ca * lam * e_t
        rhs += scatter(sim.rec_idx, res[t] * fw["rec"][t])
        rhs -= scatter(sim.src_idx, f[t] * gather(sim.src_idx, lam))
    lhs = cb * full["gcb"]
    assert np.abs(lhs).max() > 0
    assert rel_l2(rhs, lhs) <= 1e-12
