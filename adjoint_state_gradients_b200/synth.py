"""Seeded synthetic inputs for the 2-D TM Maxwell FDTD workloads.

This module generates inputs only -- relative permittivity and conductivity
fields, source wavelets, source / receiver positions -- and holds none of the
method's arithmetic (no stencils, no coefficients, no CFL bound, no physical
constants).  Both the CUDA path (benchmark, tests) and the fp64 oracle (tests)
consume its arrays, so both sides see identical inputs.  The time step is an
input too: callers compute dt = cfl_fraction * dt_max with their own CFL
function and pass it in.

Recipe (numpy PCG64, seed 1000 + workload number; per-shot models of the
batched workload use seed 5000 + shot):
  * smooth field: iid uniform noise, separable Gaussian filter (reflect
    edges), min-max rescaled to [lo, hi];
  * layered overlay: n sorted random depths, each layer adds an offset drawn
    uniformly in +-15 % of (hi - lo), result clipped to [lo, hi];
  * blob: Gaussian bump of given amplitude and width at the array centre;
  * conductivity: iid uniform in [0, sigma_max] (not smoothed);
  * sources / receivers on interior row 2 (row n_pml + 2), columns given in
    interior coordinates (offset by n_pml);
  * wavelet: Ricker, w(n) = (1 - 2 pi^2 f0^2 tau^2) exp(-pi^2 f0^2 tau^2),
    tau = n dt - 1.5 / f0 (unit peak);
  * "observed" model: the background plus a positive Gaussian perturbation,
    from which each side simulates its own d_obs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
from scipy.ndimage import gaussian_filter


@dataclass(frozen=True)
class Workload:
    name: str
    number: int
    n_interior: int
    n_pml: int
    order: int
    n_shots: int
    nt: int
    n_rec: int
    h: float           # grid spacing dx = dz (m)
    f0: float          # Ricker peak frequency (Hz)
    cfl_fraction: float
    snapshot: str      # "fp32" | "bf16" | "ckpt" | "ckpt_ey" | "none"
    ckpt_every: int = 0
    ckpt_tail: int = 0  # checkpoint modes: last steps whose snapshots the forward keeps
    batched: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return self.n_interior + 2 * self.n_pml

    @property
    def ny(self) -> int:
        return self.n

    @property
    def nx(self) -> int:
        return self.n

    @property
    def cells_per_shot(self) -> int:
        return self.n * self.n

    @property
    def cell_updates(self) -> int:
        return self.n * self.n * self.nt * self.n_shots


WORKLOADS = {
    1: Workload("tm2d-84sq-o2-s1-nt300-fp32snap", 1, 64, 10, 2, 1, 300, 32, 0.02, 400e6, 0.5, "fp32"),
    2: Workload("tm2d-296sq-o4-s4-nt1000-fp32snap", 2, 256, 20, 4, 4, 1000, 128, 0.02, 400e6, 0.6, "fp32"),
    3: Workload("tm2d-1064sq-o8-s16-nt2000-bf16snap", 3, 1000, 32, 8, 16, 2000, 256, 0.01, 200e6, 0.6, "bf16"),
    # the last 768 steps' E snapshots (111.3 GB) kept from the forward: about
    # 162 GB of the 180 GB HBM in all
    4: Workload("tm2d-2128sq-o4-s8-nt4000-ckpt64", 4, 2048, 40, 4, 8, 4000, 512, 0.02, 200e6, 0.6,
                "ckpt_ey", ckpt_every=64, ckpt_tail=768),
    5: Workload("tm2d-552sq-o8-s256-nt2000-fwd", 5, 512, 20, 8, 256, 2000, 128, 0.02, 200e6, 0.6, "none",
                batched=True),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def smooth_field(g: np.random.Generator, shape, sigma_cells: float, lo: float, hi: float) -> np.ndarray:
    a = g.uniform(0.0, 1.0, size=shape)
    if sigma_cells > 0:
        a = gaussian_filter(a, sigma=sigma_cells, mode="reflect")
    amin, amax = a.min(), a.max()
    a = (a - amin) / (amax - amin) if amax > amin else np.zeros_like(a)
    return lo + (hi - lo) * a


def layered_overlay(g: np.random.Generator, base: np.ndarray, n_layers: int, lo: float, hi: float,
                    rel: float = 0.15) -> np.ndarray:
    ny = base.shape[0]
    depths = np.sort(g.integers(1, ny - 1, size=n_layers))
    out = base.copy()
    for d in depths:
        out[d:, :] += g.uniform(-rel, rel) * (hi - lo)
    return np.clip(out, lo, hi)


def gaussian_blob(shape, amp: float, sigma_cells: float, centre=None) -> np.ndarray:
    ny, nx = shape
    cy, cx = ((ny - 1) / 2.0, (nx - 1) / 2.0) if centre is None else centre
    y = np.arange(ny)[:, None] - cy
    x = np.arange(nx)[None, :] - cx
    return amp * np.exp(-(y * y + x * x) / (2.0 * sigma_cells * sigma_cells))


def ricker(nt: int, dt: float, f0: float) -> np.ndarray:
    tau = np.arange(nt) * dt - 1.5 / f0
    a = (math.pi * f0 * tau) ** 2
    return (1.0 - 2.0 * a) * np.exp(-a)


def line_indices(nx: int, row: int, cols) -> np.ndarray:
    cols = np.asarray(cols, dtype=np.int64)
    return row * nx + cols


@dataclass
class Inputs:
    """One workload's inputs (fp64 numpy; callers cast to the dtype they need)."""
    wl: Workload
    eps_r: np.ndarray          # [ny, nx] or [S, ny, nx]
    sigma: np.ndarray          # same shape
    eps_r_true: np.ndarray     # model the "observed" data come from
    src_idx: np.ndarray        # [S, n_src] int64
    rec_idx: np.ndarray        # [S, n_rec] int64
    eps_min: float             # smallest eps_r over every model used (for vmax)

    def wavelet(self, dt: float, nt: int | None = None) -> np.ndarray:
        """Source time functions f [nt, S, n_src] (Ricker at f0)."""
        nt = self.wl.nt if nt is None else nt
        w = ricker(nt, dt, self.wl.f0)
        S, ns = self.src_idx.shape
        return np.ascontiguousarray(np.broadcast_to(w[:, None, None], (nt, S, ns)))


def make_inputs(number: int, n_shots: int | None = None, survey_shots: int | None = None,
                first_shot: int = 0) -> Inputs:
    """Inputs of workload `number` (1..5).  n_shots < S keeps the first shots.

    Workload 4 only: `survey_shots` spreads that many sources evenly over the
    interior (default: the workload's 8) and the inputs hold shots
    first_shot .. first_shot + n_shots - 1 of that survey, so that ranks of a
    multi-GPU run each simulate their own block of one larger survey."""
    wl = WORKLOADS[number]
    S = wl.n_shots if n_shots is None else n_shots
    n, p = wl.n, wl.n_pml
    g = rng(1000 + number)
    row = p + 2
    N = wl.n_interior
    if number == 1:
        eps = smooth_field(g, (n, n), 4.0, 4.0, 9.0)
        sig = g.uniform(0.0, 0.01, size=(n, n))
        eps_true = eps + gaussian_blob((n, n), 0.5, 6.0)
        src_cols = [[32]]
        rec_cols = np.arange(1, 64, 2)
    elif number == 2:
        eps = layered_overlay(g, smooth_field(g, (n, n), 8.0, 3.0, 12.0), 6, 3.0, 12.0)
        sig = g.uniform(0.0, 0.02, size=(n, n))
        eps_true = eps + gaussian_blob((n, n), 1.0, N / 10.0)
        src_cols = [[c] for c in (32, 96, 160, 224)]
        rec_cols = 2 * np.arange(128) + 1
    elif number == 3:
        base = np.full((n, n), 0.0)
        depths = np.sort(g.integers(1, n - 1, size=8))
        vals = g.uniform(3.0, 20.0, size=9)
        base[:, :] = vals[0]
        for d, v in zip(depths, vals[1:]):
            base[d:, :] = v
        eps = np.clip(base + gaussian_blob((n, n), 5.0, 40.0), 3.0, 25.0)
        sig = g.uniform(0.0, 0.05, size=(n, n))
        eps_true = eps + gaussian_blob((n, n), 1.0, N / 10.0)
        src_cols = [[int(round((k + 0.5) * 1000 / 16))] for k in range(16)]
        rec_cols = np.array([int(round((k + 0.5) * 1000 / 256)) for k in range(256)])
    elif number == 4:
        eps = smooth_field(g, (n, n), 16.0, 3.0, 20.0)
        sig = np.zeros((n, n))
        eps_true = eps + gaussian_blob((n, n), 1.0, N / 10.0)
        n_survey = wl.n_shots if survey_shots is None else survey_shots
        if first_shot < 0 or first_shot + S > n_survey:
            raise ValueError("shot block outside the survey")
        src_cols = [[int((k + 0.5) * N / n_survey)] for k in range(first_shot, first_shot + S)]
        rec_cols = 4 * np.arange(512) + 2
    elif number == 5:
        eps = np.empty((S, n, n))
        sig = np.empty((S, n, n))
        for s in range(S):
            gs = rng(5000 + s)
            eps[s] = smooth_field(gs, (n, n), 8.0, 3.0, 15.0)
            sig[s] = gs.uniform(0.0, 0.02, size=(n, n))
        eps_true = eps
        src_cols = [[256] for _ in range(wl.n_shots)]
        rec_cols = 4 * np.arange(128) + 2
    else:
        raise ValueError(number)
    src_idx = np.array([line_indices(n, row, np.asarray(c) + p) for c in src_cols], dtype=np.int64)[:S]
    rec_idx = np.tile(line_indices(n, row, rec_cols + p)[None, :], (S, 1))
    eps_min = float(min(eps.min(), eps_true.min()))
    return Inputs(wl, eps, sig, eps_true, src_idx, rec_idx, eps_min)


def small_case(seed: int, ny: int, nx: int, n_shots: int, n_src: int, n_rec: int,
               eps_lo: float = 2.0, eps_hi: float = 6.0, sigma_max: float = 0.01,
               smooth: float = 2.0, batched: bool = False):
    """A small random setup for parity / edge tests.

    Returns (eps_r, sigma, src_idx, rec_idx) with sources and receivers at
    random distinct-or-not cells anywhere in the array.
    """
    g = rng(seed)
    shape = (n_shots, ny, nx) if batched else (ny, nx)
    if batched:
        eps = np.stack([smooth_field(g, (ny, nx), smooth, eps_lo, eps_hi) for _ in range(n_shots)])
    else:
        eps = smooth_field(g, shape, smooth, eps_lo, eps_hi)
    sig = g.uniform(0.0, sigma_max, size=shape)
    src = g.integers(0, ny * nx, size=(n_shots, n_src)).astype(np.int64)
    rec = g.integers(0, ny * nx, size=(n_shots, n_rec)).astype(np.int64)
    return eps, sig, src, rec
