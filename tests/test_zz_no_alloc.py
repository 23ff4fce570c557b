"""The scratch-free forward (mw_tm_forward_noalloc), for callers that cannot
allocate device memory: it keeps its scratch in an array the library defines
in device memory instead of a caller-provided workspace.  Called through the
C ABI twice in a row, it must reproduce the workspace forward (mw_tm_forward)
within the records tolerance, and a problem too large for its scratch must be
refused before any work runs.  It reports the device status of its own call:
an out-of-range receiver index (which the kernels flag and skip, never
access) gives MW_ERR_ARG, and the next valid call starts from clean status
words and returns MW_OK.  Collected last on purpose; runs alone too.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from adjoint_state_gradients_b200 import api, mwtm, synth
from tests._cases import rel_l2, small_sim
from tests._gpu import f32, problem_from_sim, run_forward

pytestmark = pytest.mark.gpu

REC_TOL = 1e-5


def test_noalloc_forward_matches_workspace_forward_on_two_calls():
    n_pml, nt = 8, 70
    sim, dt, _ = small_sim(909, 96, 136, 2, 2, 6, 4, n_pml, round_f32=True, sigma_max=0.02)
    g = synth.rng(9)
    f = f32(g.normal(size=(nt, 2, 2)))
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="none")
    state_ref = prob.new_state()
    rec_ref = run_forward(prob, f, state=state_ref)
    st_ref = api.unpack_state(prob.p, state_ref)
    f_dev = torch.as_tensor(np.asarray(f, dtype=np.float32)).cuda()
    for call in range(2):
        state = prob.new_state()
        rec = torch.full((nt, 2, 6), float("nan"), device="cuda")
        rc = mwtm.tm_forward_noalloc(prob.p, prob.ca, prob.cb, prob.cq, prob.cpml, f_dev,
                                     prob.src_idx, prob.rec_idx, state, rec)
        assert rc == mwtm.MW_OK, mwtm.last_error()
        got = rec.cpu().numpy().astype(np.float64)
        assert rel_l2(got, rec_ref) <= REC_TOL, call
        st = api.unpack_state(prob.p, state)
        for name in st_ref:
            if np.abs(st_ref[name]).max() > 0:
                assert rel_l2(st[name], st_ref[name]) <= REC_TOL, (call, name)


def test_noalloc_forward_refuses_a_problem_larger_than_its_scratch():
    ny = nx = 1024
    S = 8  # 3 fields x 8 shots x 1024^2 x 4 B = 96 MiB > 64 MiB of scratch
    p = mwtm.make_params(ny=ny, nx=nx, order=4, n_shots=S, nt=1, dt=1e-12, dy=0.01, dx=0.01,
                         n_pml=0, vmax=1.5e8)
    dummy = torch.zeros(4, device="cuda")
    idx = torch.zeros((S, 1), dtype=torch.int64, device="cuda")
    rc = mwtm.tm_forward_noalloc(p, dummy, dummy, dummy, dummy, None, idx, idx, dummy, None)
    assert rc == mwtm.MW_ERR_WORKSPACE
    assert "built-in scratch" in mwtm.last_error()


def test_noalloc_forward_reports_its_own_status_and_clears_it():
    n_pml, nt = 8, 40
    sim, dt, _ = small_sim(919, 64, 96, 1, 1, 4, 4, n_pml, round_f32=True)
    g = synth.rng(19)
    f = f32(g.normal(size=(nt, 1, 1)))
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="none")
    rec_ref = run_forward(prob, f)
    f_dev = torch.as_tensor(np.asarray(f, dtype=np.float32)).cuda()
    bad_idx = prob.rec_idx.clone()
    bad_idx[0, 2] = sim.ny * sim.nx + 5  # one receiver past the last cell
    state = prob.new_state()
    rec = torch.zeros((nt, 1, 4), device="cuda")
    rc = mwtm.tm_forward_noalloc(prob.p, prob.ca, prob.cb, prob.cq, prob.cpml, f_dev,
                                 prob.src_idx, bad_idx, state, rec)
    assert rc == mwtm.MW_ERR_ARG
    assert "out of range" in mwtm.last_error()
    state = prob.new_state()
    rec = torch.zeros((nt, 1, 4), device="cuda")
    rc = mwtm.tm_forward_noalloc(prob.p, prob.ca, prob.cb, prob.cq, prob.cpml, f_dev,
                                 prob.src_idx, prob.rec_idx, state, rec)
    assert rc == mwtm.MW_OK, mwtm.last_error()
    assert rel_l2(rec.cpu().numpy().astype(np.float64), rec_ref) <= REC_TOL
