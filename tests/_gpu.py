"""GPU-side helpers for the parity tests: run the CUDA library on the same
fp32 coefficient arrays an oracle Sim holds.  Inputs flow oracle -> GPU only
(coefficients, wavelets, residuals); nothing computed on the GPU is ever fed
to the oracle."""
from __future__ import annotations

import numpy as np
import torch

from adjoint_state_gradients_b200 import api, mwtm


def problem_from_sim(sim, nt, dt, n_pml, snapshot="fp32", ckpt_every=64, grad_mask=False,
                     check_finite=False, vmax=None, ckpt_tail=0):
    kw = dict(vmax=vmax if vmax is not None else 1.0, allow_unstable=vmax is None)
    prob = api.Problem(sim.ny, sim.nx, sim.order, sim.dy, sim.dx, dt, nt, n_pml, sim.src_idx,
                       sim.rec_idx, snapshot=snapshot, ckpt_every=ckpt_every,
                       batched=bool(sim.model_batched), cq_scalar=not sim.cq_is_array,
                       grad_mask_pml=grad_mask, check_finite=check_finite,
                       ckpt_tail=ckpt_tail, **kw)
    cpml = np.concatenate(list(sim.prof_y) + list(sim.prof_x))
    prob.set_coefficients(sim.ca, sim.cb, sim.cq, cpml)
    return prob


def run_forward(prob, f, state=None):
    rec = prob.forward(torch.as_tensor(np.asarray(f, dtype=np.float32)).cuda(), state=state)
    torch.cuda.synchronize()
    return rec.cpu().numpy().astype(np.float64)


def run_adjoint(prob, res, grad_f=True, adj_state=None):
    gca, gcb, gf = prob.adjoint(torch.as_tensor(np.asarray(res, dtype=np.float32)).cuda(),
                                grad_f=grad_f, adj_state=adj_state)
    torch.cuda.synchronize()
    to = lambda t: None if t is None else t.cpu().numpy().astype(np.float64)
    return to(gca), to(gcb), to(gf)


def f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)
