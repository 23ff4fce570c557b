"""The whole-sweep launch of small grids (every step of the forward, or of
the adjoint, in one cooperative launch) against the step-by-step launches,
bit for bit, in both variants: the resident one (each block's rows in shared
memory, halo rows read from the neighbouring blocks), with the library's
cluster, group width and chunks of global traffic, with at most 4 blocks a
shot, with groups of 4 cells only, and with chunks of 2 steps, and the one
whose state stays in global memory (MW_SMALL_L2=1).

Both paths make the same floating-point operations in the same order for
every update, source sum, receiver sample and gradient term, so records,
final states (CPML memories included), per-shot gradients and the source
gradient must be identical.  MW_NO_SMALL=1 makes the library take the
step-by-step launches.  The cases cover every stencil order, the snapshot
formats, batched models, a Cq array, the interior-only gradient mask, grids
without a CPML band, duplicate and inactive sources and receivers, a given
initial state and a given adjoint start state.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from adjoint_state_gradients_b200 import mwtm, synth
from tests._cases import small_sim
from tests._gpu import f32, problem_from_sim

pytestmark = pytest.mark.gpu


VARIANTS = {"resident": {}, "resident-4": {"MW_SMALL_CLUSTER": "4"},
            "resident-w4": {"MW_SMALL_WIDTH": "4"},
            "resident-chunk2": {"MW_SMALL_CHUNK": "2"}, "l2": {"MW_SMALL_L2": "1"}}


def _run(prob, f, res, state0, adj0, small, monkeypatch, variant="resident"):
    for k in ("MW_SMALL_CLUSTER", "MW_SMALL_CHUNK", "MW_SMALL_WIDTH", "MW_SMALL_L2"):
        monkeypatch.delenv(k, raising=False)
    if small:
        monkeypatch.delenv("MW_NO_SMALL", raising=False)
        for k, v in VARIANTS[variant].items():
            monkeypatch.setenv(k, v)
    else:
        monkeypatch.setenv("MW_NO_SMALL", "1")
    state = state0.clone()
    rec = prob.forward(torch.as_tensor(f, dtype=torch.float32).cuda(), state=state).clone()
    out = [rec.cpu().numpy(), state.cpu().numpy()]
    if prob.p.snap_mode != mwtm.SNAP_NONE:
        adj = adj0.clone()
        gca, gcb, gf = prob.adjoint(torch.as_tensor(res, dtype=torch.float32).cuda(), grad_f=True,
                                    adj_state=adj)
        out += [gca.cpu().numpy(), gcb.cpu().numpy(), gf.cpu().numpy(), adj.cpu().numpy()]
    torch.cuda.synchronize()
    assert prob.status() == mwtm.MW_OK, mwtm.last_error()
    return out


@pytest.mark.parametrize("order,ny,nx,S,n_pml,batched,cq_array,snapshot,mask", [
    (2, 37, 44, 1, 4, False, False, "fp32", False),
    (4, 61, 140, 2, 6, False, False, "bf16", False),
    (6, 50, 132, 3, 5, True, False, "fp8", False),
    (8, 70, 264, 2, 7, False, True, "fp32", False),
    (4, 150, 20, 2, 3, True, True, "fp32", True),
    (4, 33, 40, 1, 0, False, False, "none", False),
    (4, 84, 84, 1, 10, False, False, "fp32", True),
    (8, 64, 96, 2, 5, False, False, "fp32", False),    # 4 rows a block: the halo is a whole block
    (8, 61, 40, 1, 3, False, False, "bf16", False),    # a last block of one row
    (4, 200, 264, 2, 8, False, False, "fp32", False),  # up to 2 groups a thread
])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_whole_sweep_is_bitwise_step_by_step(order, ny, nx, S, n_pml, batched, cq_array,
                                             snapshot, mask, variant, monkeypatch):
    sim, dt, _ = small_sim(900 + order + ny, ny, nx, S, 3, 7, order, n_pml, batched=batched,
                           cq_array=cq_array, round_f32=True, sigma_max=0.02)
    src, rec = sim.src_idx.copy(), sim.rec_idx.copy()
    src[:, 1] = src[:, 0]     # a duplicate source
    rec[:, 2] = -1            # an inactive receiver
    rec[:, 4] = rec[:, 3]     # a duplicate receiver
    sim.src_idx, sim.rec_idx = src, rec
    nt = 45
    g = synth.rng(order + nx)
    f = f32(g.normal(size=(nt, S, 3)))
    res = f32(g.normal(size=(nt, S, 7)))
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot=snapshot, grad_mask=mask)
    n = mwtm.state_floats(prob.p)
    state0 = torch.as_tensor(f32(1e-3 * g.normal(size=n)), dtype=torch.float32).cuda()
    adj0 = torch.as_tensor(f32(1e-3 * g.normal(size=n)), dtype=torch.float32).cuda()
    step = _run(prob, f, res, state0, adj0, False, monkeypatch)
    whole = _run(prob, f, res, state0, adj0, True, monkeypatch, variant)
    names = ["records", "state", "dJ/dCa", "dJ/dCb", "dJ/df", "adjoint state"]
    for nm, x, y in zip(names, step, whole):
        assert np.array_equal(x, y), nm
    assert np.abs(step[0]).max() > 0
