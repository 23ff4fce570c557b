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


def test_graph_follows_model_updates_and_refuses_replaced_buffers():
    """The problem's model setters write into the buffers the graph baked in,
    so a replay after set_model_eps_sigma computes the new model's sweep (bit
    for bit the eager one); a buffer replaced behind the problem's back stops
    the replay instead of reading stale memory."""
    S, ny, nx, n_pml, nt = 2, 40, 56, 5, 40
    eps, sig, src, rec = synth.small_case(1210, ny, nx, S, 1, 5, sigma_max=0.02)
    vmax = 299792458.0 / np.sqrt(eps.min())
    dt = 0.6 * mwtm.cfl_dt(4, 0.02, 0.02, vmax)
    prob = api.Problem(ny, nx, 4, 0.02, 0.02, dt, nt, n_pml, src, rec, vmax=vmax, snapshot="fp32")
    prob.set_model_eps_sigma(eps.astype(np.float32), sig.astype(np.float32), f0=4e8)
    g = synth.rng(1211)
    f = torch.as_tensor(f32(g.normal(size=(nt, S, 1))), dtype=torch.float32).cuda()
    d_obs = torch.as_tensor(f32(0.1 * g.normal(size=(nt, S, 5))), dtype=torch.float32).cuda()
    sg = api.SweepGraph(prob, f, d_obs)
    eps2 = (eps * 1.1).astype(np.float32)
    prob.set_model_eps_sigma(eps2, sig.astype(np.float32), f0=4e8)
    got = [t.cpu().numpy().copy() for t in sg.replay()]
    torch.cuda.synchronize()
    J, r, gca, gcb = prob.misfit_gradient(f, d_obs)
    torch.cuda.synchronize()
    for a, b, nm in zip(got, (J, r, gca, gcb), ("J", "rec", "gca", "gcb")):
        assert np.array_equal(a, b.cpu().numpy()), nm
    prob.ca = prob.ca.clone()
    with pytest.raises(RuntimeError, match="replaced after capture"):
        sg.replay()
