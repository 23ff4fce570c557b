"""The two-step forward kernel (steps t and t + 1 in one launch, temporal
blocking) against the one-step kernel, bit for bit.

Both kernels make the same floating-point operations in the same order for
every update, source injection and receiver sample, so every output --
records, the final state with its CPML memories, stored snapshots (seen
through the adjoint gradients that read them) -- must be identical.  The
environment switch MW_NO_TWO_STEP=1 makes the library run every step with
the one-step kernel.  Sources and receivers sit on and around the two-step
strips' boundaries (columns 112 k, where the step-t values of one strip are
recomputed in its neighbour's halo), in the CPML bands, duplicated, and
inactive; odd step counts leave a single step at the end; checkpoints every
6 steps (and a forward-stored tail) force single steps where a checkpoint
falls after the first step of a pair.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from adjoint_state_gradients_b200 import api, mwtm, synth
from tests._cases import small_sim
from tests._gpu import f32, problem_from_sim

pytestmark = pytest.mark.gpu


def _indices(seed, ny, nx, S, n_pml, n):
    """Cells around the strip boundaries x = 112 k (and 104 k), in the bands,
    one duplicate and one inactive entry per shot."""
    g = synth.rng(seed)
    cols = [c for k in range(1, nx // 104 + 1) for c in (104 * k - 2, 104 * k, 112 * k - 1, 112 * k,
                                                       112 * k + 3) if c < nx]
    cols += [1, n_pml // 2, nx - 2, nx - 1 - n_pml // 2]
    out = np.empty((S, n), np.int64)
    for s in range(S):
        ys = g.integers(0, ny, size=n)
        xs = g.choice(cols, size=n)
        out[s] = ys * nx + xs
        out[s, 1] = out[s, 0]        # a duplicate
        out[s, n - 1] = -1           # an inactive entry
    return out


def _run(prob, f, res, one_step, monkeypatch):
    monkeypatch.setenv("MW_NO_SMALL", "1")  # the step-by-step launches on every grid
    if one_step:
        monkeypatch.setenv("MW_NO_TWO_STEP", "1")
    else:
        monkeypatch.delenv("MW_NO_TWO_STEP", raising=False)
    state = prob.new_state()
    rec = prob.forward(torch.as_tensor(f, dtype=torch.float32).cuda(), state=state).clone()
    out = [rec.cpu().numpy(), state.cpu().numpy()]
    if prob.p.snap_mode != mwtm.SNAP_NONE:
        gca, gcb, gf = prob.adjoint(torch.as_tensor(res, dtype=torch.float32).cuda(), grad_f=True)
        out += [gca.cpu().numpy(), gcb.cpu().numpy(), gf.cpu().numpy()]
    torch.cuda.synchronize()
    assert prob.status() == mwtm.MW_OK, mwtm.last_error()
    return out


@pytest.mark.parametrize("order,ny,nx,S,n_pml,batched,nt", [
    (2, 70, 232, 2, 5, False, 33),
    (4, 150, 344, 3, 8, True, 41),
    (4, 61, 120, 1, 0, False, 20),
    (6, 90, 240, 2, 6, False, 27),
])
@pytest.mark.parametrize("snapshot", ["none", "fp32", "bf16", "ckpt", "ckpt_ey"])
def test_two_step_forward_is_bitwise_one_step(order, ny, nx, S, n_pml, batched, nt, snapshot,
                                              monkeypatch):
    sim, dt, _ = small_sim(700 + order + nx, ny, nx, S, 3, 9, order, n_pml, batched=batched,
                           round_f32=True, sigma_max=0.02)
    sim.src_idx = _indices(11 + order, ny, nx, S, n_pml, 3)
    sim.rec_idx = _indices(23 + order, ny, nx, S, n_pml, 9)
    g = synth.rng(order + nt)
    f = f32(g.normal(size=(nt, S, 3)))
    res = f32(g.normal(size=(nt, S, 9)))
    tail = 7 if snapshot == "ckpt_ey" else 0
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot=snapshot, ckpt_every=6, ckpt_tail=tail)
    one = _run(prob, f, res, True, monkeypatch)
    two = _run(prob, f, res, False, monkeypatch)
    names = ["records", "state", "dJ/dCa", "dJ/dCb", "dJ/df"]
    for nm, x, y in zip(names, one, two):
        assert np.array_equal(x, y), nm
    st = api.unpack_state(prob.p, torch.as_tensor(two[1]))
    assert np.abs(st["ey"]).max() > 0  # the sources reached the field
