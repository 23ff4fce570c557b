"""A whole misfit-gradient sweep captured as one CUDA graph (api.SweepGraph):
replays give, bit for bit, what the eager calls give, for the full-storage
and the E-alone checkpoint modes (forward-stored tail included), and new
inputs copied into the graph's buffers take effect."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from adjoint_state_gradients_b200 import api, mwtm, synth
from tests._cases import small_sim
from tests._gpu import f32, problem_from_sim

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,tail", [("fp32", 0), ("ckpt_ey", 12), ("ckpt", 0)])
def test_graph_replay_is_bitwise_the_eager_sweep(mode, tail):
    S, ny, nx, n_pml, nt = 2, 40, 56, 5, 50
    sim, dt, _ = small_sim(1200, ny, nx, S, 1, 6, 4, n_pml, round_f32=True, sigma_max=0.02)
    g = synth.rng(1201)
    f1 = torch.as_tensor(f32(g.normal(size=(nt, S, 1))), dtype=torch.float32).cuda()
    f2 = torch.as_tensor(f32(g.normal(size=(nt, S, 1))), dtype=torch.float32).cuda()
    d_obs = torch.as_tensor(f32(0.1 * g.normal(size=(nt, S, 6))), dtype=torch.float32).cuda()
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot=mode, ckpt_every=16, ckpt_tail=tail)

    def eager(f):
        J, rec, gca, gcb = prob.misfit_gradient(f, d_obs)
        torch.cuda.synchronize()
        return [t.detach().cpu().numpy().copy() for t in (J, rec, gca, gcb)]

    want1, want2 = eager(f1), eager(f2)
    sg = api.SweepGraph(prob, f1, d_obs)
    for _ in range(2):
        got = [t.cpu().numpy() for t in sg.replay()]
        torch.cuda.synchronize()
        for a, b, nm in zip(got, want1, ("J", "rec", "gca", "gcb")):
            assert np.array_equal(a, b), nm
    sg.f.copy_(f2)
    got = [t.cpu().numpy() for t in sg.replay()]
    torch.cuda.synchronize()
    for a, b, nm in zip(got, want2, ("J", "rec", "gca", "gcb")):
        assert np.array_equal(a, b), nm
    assert prob.status() == mwtm.MW_OK
    assert np.abs(want1[2]).max() > 0 and not np.array_equal(want1[2], want2[2])
