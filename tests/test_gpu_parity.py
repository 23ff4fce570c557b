"""CUDA library vs the fp64 oracle, element by element on identical seeded
inputs (tolerances: fp32 records rel-L2 <= 1e-5, fp32 gradients <= 1e-4,
bf16-snapshot gradients <= 2e-2, GPU dot test <= 1e-5).

Both sides consume the same fp32 coefficient arrays (the oracle's, rounded to
fp32, evaluated in fp64 on the oracle side), so the comparison measures the
time stepping alone; model preparation is compared separately.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from adjoint_state_gradients_b200 import api, mwtm, synth
from tests._cases import oracle_sim, rel_l2, small_sim, workload_sim
from tests._gpu import f32, problem_from_sim, run_adjoint, run_forward

pytestmark = pytest.mark.gpu

REC_TOL = 1e-5
GRAD_TOL = 1e-4


def _oracle_pair(sim, f, res, snapshots=True):
    fw = sim.forward(f, snapshots=snapshots)
    adj = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"])
    return fw, adj


# ----------------------------------------------------------------------------
# small grids: every order, ragged strips, several chunks, bands, batching


@pytest.mark.parametrize("order,ny,nx,S,n_pml,batched,cq_array", [
    (2, 37, 44, 1, 4, False, False),
    (4, 61, 140, 2, 6, False, False),
    (6, 50, 132, 3, 5, True, False),
    (8, 70, 264, 2, 7, False, True),
    (8, 33, 40, 1, 0, False, False),
    (4, 150, 20, 2, 3, True, True),
])
@pytest.mark.parametrize("path", ["whole_sweep", "step_by_step"])
def test_small_forward_adjoint_parity(order, ny, nx, S, n_pml, batched, cq_array, path,
                                      monkeypatch):
    """Both the whole-sweep launch small grids take and the step-by-step
    launches (MW_NO_SMALL=1) against the oracle."""
    if path == "step_by_step":
        monkeypatch.setenv("MW_NO_SMALL", "1")
    else:
        monkeypatch.delenv("MW_NO_SMALL", raising=False)
    sim, dt, _ = small_sim(100 + order + ny, ny, nx, S, 2, 5, order, n_pml, batched=batched,
                           cq_array=cq_array, round_f32=True, sigma_max=0.02)
    nt = 57
    g = synth.rng(7 + order)
    f = f32(g.normal(size=(nt, S, 2)))
    res = f32(g.normal(size=(nt, S, 5)))
    fw, adj = _oracle_pair(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, n_pml)
    state = prob.new_state()
    rec = run_forward(prob, f, state=state)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    st = api.unpack_state(prob.p, state)
    for i, nm in enumerate(oracle.FIELDS):
        assert rel_l2(st[nm], fw["state"][i]) <= REC_TOL, nm
    adj_state = prob.new_state()
    gca, gcb, gf = run_adjoint(prob, res, adj_state=adj_state)
    assert rel_l2(gca, adj["gca"]) <= GRAD_TOL
    assert rel_l2(gcb, adj["gcb"]) <= GRAD_TOL
    assert rel_l2(gf, adj["grad_f"]) <= GRAD_TOL
    ast = api.unpack_state(prob.p, adj_state)
    for i, nm in enumerate(oracle.FIELDS):
        if np.abs(adj["adj"][i]).max() > 0:
            assert rel_l2(ast[nm], adj["adj"][i]) <= GRAD_TOL, nm
    assert prob.status() == mwtm.MW_OK


@pytest.mark.parametrize("placement", ["ca_then_cb", "cb_then_ca", "same_array"])
def test_model_array_placement(placement):
    """Ca and Cb reach the forward stencil as one two-row box when their
    distance in memory allows it (in either order) and as two boxes otherwise
    (here: both arguments are the same array).  Records and states must match
    the oracle in every placement."""
    ny, nx, S, n_pml, nt = 64, 264, 2, 6, 50
    sim, dt, _ = small_sim(515, ny, nx, S, 2, 5, 4, n_pml, round_f32=True, sigma_max=0.02)
    if placement == "same_array":
        # Ca = Cb = 1 with Cq scaled by max(Cb): a lossless medium inside the
        # stability bound (the scheme couples Cb and Cq only through their product)
        one = np.ones_like(sim.ca)
        sim = oracle.Sim(ny=ny, nx=nx, order=4, dy=sim.dy, dx=sim.dx, ca=one, cb=one,
                         cq=float(np.float32(sim.cq[0] * sim.cb.max())), prof_y=sim.prof_y,
                         prof_x=sim.prof_x, src_idx=sim.src_idx, rec_idx=sim.rec_idx)
    g = synth.rng(51)
    f = f32(g.normal(size=(nt, S, 2)))
    fw = sim.forward(f, snapshots=False)
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="none")
    ca = torch.as_tensor(sim.ca, dtype=torch.float32, device="cuda")
    cb = torch.as_tensor(sim.cb, dtype=torch.float32, device="cuda")
    if placement == "same_array":
        prob.ca = prob.cb = ca
    else:
        buf = torch.empty((2, ny, nx), dtype=torch.float32, device="cuda")
        first, second = (0, 1) if placement == "ca_then_cb" else (1, 0)
        buf[first] = ca
        buf[second] = cb
        prob.ca, prob.cb = buf[first], buf[second]
    state = prob.new_state()
    rec = run_forward(prob, f, state=state)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    st = api.unpack_state(prob.p, state)
    for i, nm in enumerate(oracle.FIELDS):
        assert rel_l2(st[nm], fw["state"][i]) <= REC_TOL, nm
    assert prob.status() == mwtm.MW_OK


@pytest.mark.parametrize("placement", ["first_then_second", "second_then_first", "same_model"])
def test_adjoint_array_placement(placement):
    """The adjoint fetches Ca / Cb and the per-shot gradients gCa / gCb as
    pair boxes when their distance allows it (either order) and as single
    boxes otherwise (Ca and Cb given as one array).  Gradients must match the
    oracle in every placement."""
    ny, nx, S, n_pml, nt = 60, 240, 2, 5, 40
    sim, dt, _ = small_sim(616, ny, nx, S, 2, 5, 4, n_pml, round_f32=True, sigma_max=0.02)
    if placement == "same_model":
        one = np.ones_like(sim.ca)
        sim = oracle.Sim(ny=ny, nx=nx, order=4, dy=sim.dy, dx=sim.dx, ca=one, cb=one,
                         cq=float(np.float32(sim.cq[0] * sim.cb.max())), prof_y=sim.prof_y,
                         prof_x=sim.prof_x, src_idx=sim.src_idx, rec_idx=sim.rec_idx)
    g = synth.rng(61)
    f = f32(g.normal(size=(nt, S, 2)))
    res = f32(g.normal(size=(nt, S, 5)))
    fw, adj = _oracle_pair(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, n_pml)
    ca = torch.as_tensor(sim.ca, dtype=torch.float32, device="cuda")
    cb = torch.as_tensor(sim.cb, dtype=torch.float32, device="cuda")
    gbuf = torch.zeros((2, S, ny, nx), dtype=torch.float32, device="cuda")
    if placement == "same_model":
        prob.ca = prob.cb = ca
        gca, gcb = gbuf[0], gbuf[1]
    else:
        mbuf = torch.empty((2, ny, nx), dtype=torch.float32, device="cuda")
        k = (0, 1) if placement == "first_then_second" else (1, 0)
        mbuf[k[0]] = ca
        mbuf[k[1]] = cb
        prob.ca, prob.cb = mbuf[k[0]], mbuf[k[1]]
        gca, gcb = gbuf[k[0]], gbuf[k[1]]
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    prob.adjoint(torch.as_tensor(np.asarray(res, dtype=np.float32)).cuda(), gca=gca, gcb=gcb)
    torch.cuda.synchronize()
    assert rel_l2(gca.cpu().numpy().astype(np.float64), adj["gca"]) <= GRAD_TOL
    assert rel_l2(gcb.cpu().numpy().astype(np.float64), adj["gcb"]) <= GRAD_TOL
    assert prob.status() == mwtm.MW_OK


@pytest.mark.parametrize("nt", [0, 1, 2, 3, 64, 65])
def test_step_counts_and_checkpoint_partial_segments(nt):
    sim, dt, _ = small_sim(300 + nt, 40, 48, 2, 1, 3, 4, 5, round_f32=True)
    g = synth.rng(nt)
    f = f32(g.normal(size=(max(nt, 1), 2, 1)))[:nt]
    res = f32(g.normal(size=(max(nt, 1), 2, 3)))[:nt]
    if nt == 0:
        prob = problem_from_sim(sim, 0, dt, 5)
        state = prob.new_state()
        prob.forward(torch.zeros((1, 2, 1), device="cuda"), state=state)
        torch.cuda.synchronize()
        assert float(state.abs().max()) == 0.0
        return
    fw, adj = _oracle_pair(sim, f, res)
    for mode, C in (("fp32", 64), ("ckpt", 16), ("ckpt", 64)):
        prob = problem_from_sim(sim, nt, dt, 5, snapshot=mode, ckpt_every=C)
        rec = run_forward(prob, f)
        assert rel_l2(rec, fw["rec"]) <= REC_TOL
        gca, gcb, gf = run_adjoint(prob, res)
        assert rel_l2(gca, adj["gca"]) <= GRAD_TOL, mode
        assert rel_l2(gcb, adj["gcb"]) <= GRAD_TOL, mode
        assert rel_l2(gf, adj["grad_f"]) <= GRAD_TOL, mode


def test_duplicate_and_inactive_indices():
    sim, dt, _ = small_sim(401, 30, 36, 2, 4, 6, 4, 4, round_f32=True)
    sim.src_idx[0] = [100, 100, -1, 333]
    sim.src_idx[1] = [-1, -1, -1, 7]
    sim.rec_idx[0, :3] = [100, 100, -1]
    nt = 40
    g = synth.rng(5)
    f = f32(g.normal(size=(nt, 2, 4)))
    res = f32(g.normal(size=(nt, 2, 6)))
    fw, adj = _oracle_pair(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, 4)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    assert np.all(rec[:, 0, 2] == 0.0)
    gca, gcb, gf = run_adjoint(prob, res)
    assert rel_l2(gca, adj["gca"]) <= GRAD_TOL
    assert rel_l2(gf, adj["grad_f"]) <= GRAD_TOL
    assert np.all(gf[:, 1, :3] == 0.0)


def test_gradient_mask_matches_masked_oracle():
    n_pml = 6
    sim, dt, _ = small_sim(402, 44, 52, 1, 1, 4, 4, n_pml, round_f32=True)
    nt = 50
    g = synth.rng(6)
    f = f32(g.normal(size=(nt, 1, 1)))
    res = f32(g.normal(size=(nt, 1, 4)))
    fw, adj = _oracle_pair(sim, f, res)
    mask = np.zeros((44, 52))
    mask[n_pml:44 - n_pml, n_pml:52 - n_pml] = 1.0
    prob = problem_from_sim(sim, nt, dt, n_pml, grad_mask=True)
    run_forward(prob, f)
    gca, gcb, _ = run_adjoint(prob, res)
    assert rel_l2(gca, adj["gca"] * mask) <= GRAD_TOL
    assert np.all(gca[0][mask == 0] == 0.0)


# ----------------------------------------------------------------------------
# the five workloads (shot subsets / reduced nt where the oracle would take
# minutes; full grids and the launch configuration the benchmark uses)


def _workload_case(num, n_shots, nt, snapshot, C=64):
    sim, inp, dt, f = workload_sim(num, n_shots=n_shots, nt=nt)
    sim_true, _, _, _ = workload_sim(num, n_shots=n_shots, nt=nt, true_model=True)
    d_obs = f32(sim_true.forward(f)["rec"])
    return sim, inp, dt, f, d_obs


def test_workload1_full():
    """84x84 order 2, nt 300, fp32 snapshots, misfit 1/2||d - d_obs||^2.

    (a) adjoint parity on identical inputs: both sides get the oracle's
    residual (rounded to fp32);  (b) end to end, each side computing its own
    residual d - d_obs.  In (b) the residual is a cancelling difference, so
    its fp32 error is the record error times ||d|| / ||d - d_obs||; the
    gradient is linear in the residual, so its tolerance is the measured
    relative residual error plus the same-input bound."""
    sim, inp, dt, f, d_obs = _workload_case(1, 1, 300, "fp32")
    fw = sim.forward(f, snapshots=True)
    res_o, J_o = oracle.residual(fw["rec"], d_obs)
    res32 = f32(res_o)
    adj = sim.adjoint(res32, fw["snap_ey"], fw["snap_curl"])
    prob = problem_from_sim(sim, 300, dt, inp.wl.n_pml)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    gca, gcb, _ = run_adjoint(prob, res32)
    assert rel_l2(gca, adj["gca"]) <= GRAD_TOL
    assert rel_l2(gcb, adj["gcb"]) <= GRAD_TOL
    # (b) end to end through the public API
    prob = problem_from_sim(sim, 300, dt, inp.wl.n_pml)
    J, rec, gca, gcb = prob.misfit_gradient(torch.as_tensor(f, dtype=torch.float32).cuda(),
                                            torch.as_tensor(d_obs, dtype=torch.float32).cuda())
    torch.cuda.synchronize()
    res_gpu = rec.cpu().numpy().astype(np.float64) - d_obs
    e_res = rel_l2(res_gpu, res_o)
    tol = GRAD_TOL + 2.0 * e_res
    adj_o = sim.adjoint(res_o, fw["snap_ey"], fw["snap_curl"])
    assert float(J.cpu()[0]) == pytest.approx(J_o, rel=2.0 * e_res + 1e-6)
    assert rel_l2(gca.cpu().numpy(), oracle.combine(adj_o["gca"])) <= tol
    assert rel_l2(gcb.cpu().numpy(), oracle.combine(adj_o["gcb"])) <= tol


def test_workload2_full():
    """296x296 order 4, 4 shots, nt 1000, fp32 snapshots."""
    sim, inp, dt, f, d_obs = _workload_case(2, 4, 1000, "fp32")
    fw = sim.forward(f, snapshots=True)
    res_o, _ = oracle.residual(fw["rec"], d_obs)
    res = f32(res_o)
    adj = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"])
    prob = problem_from_sim(sim, 1000, dt, inp.wl.n_pml)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    gca, gcb, gf = run_adjoint(prob, res)
    assert rel_l2(gca, adj["gca"]) <= GRAD_TOL
    assert rel_l2(gcb, adj["gcb"]) <= GRAD_TOL
    g_gpu = prob.combine(torch.as_tensor(gca, dtype=torch.float32).cuda()).cpu().numpy()
    assert rel_l2(g_gpu, oracle.combine(adj["gca"])) <= GRAD_TOL


def test_workload3_bf16_snapshots():
    """1064x1064 order 8, bf16 snapshots: the full 16-shot sweep on the GPU;
    the fp32-storage gradient and the oracle on a 2-shot subset, nt 300."""
    nt = 300
    sim, inp, dt, f = workload_sim(3, n_shots=2, nt=nt)
    g = synth.rng(33)
    res = f32(g.normal(size=(nt, 2, inp.wl.n_rec)))
    ck = sim.fwd_adj_ckpt(f, res, 32)
    p32 = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot="fp32")
    rec = run_forward(p32, f)
    assert rel_l2(rec, ck["rec"]) <= REC_TOL
    gca32, gcb32, _ = run_adjoint(p32, res)
    assert rel_l2(gca32, ck["gca"]) <= GRAD_TOL
    assert rel_l2(gcb32, ck["gcb"]) <= GRAD_TOL
    del p32
    p16 = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot="bf16")
    run_forward(p16, f)
    gca16, gcb16, _ = run_adjoint(p16, res)
    e_ca, e_cb = rel_l2(gca16, gca32), rel_l2(gcb16, gcb32)
    print(f"bf16-snapshot gradient error vs fp32 storage: Ca {e_ca:.3e} Cb {e_cb:.3e}")
    assert e_ca <= 2e-2 and e_cb <= 2e-2


@pytest.mark.parametrize("snapshot", ["ckpt", "ckpt_ey"])
def test_workload4_checkpoint_replay(snapshot):
    """2128x2128 order 4, checkpoints every 64 steps: one shot, nt 200
    (3 full segments + a partial one) against the oracle's own replay, with
    the pair segment and with the E-alone segment."""
    nt = 200
    sim, inp, dt, f = workload_sim(4, n_shots=1, nt=nt)
    g = synth.rng(44)
    res = f32(g.normal(size=(nt, 1, inp.wl.n_rec)))
    ck = sim.fwd_adj_ckpt(f, res, 50)
    prob = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot=snapshot, ckpt_every=64)
    rec = run_forward(prob, f)
    assert rel_l2(rec, ck["rec"]) <= REC_TOL
    gca, gcb, gf = run_adjoint(prob, res)
    assert rel_l2(gca, ck["gca"]) <= GRAD_TOL
    assert rel_l2(gcb, ck["gcb"]) <= GRAD_TOL
    assert rel_l2(gf, ck["grad_f"]) <= GRAD_TOL


def test_workload5_batched_records():
    """552x552 order 8 with per-shot models: 2 shots, nt 600, records only."""
    nt = 600
    sim, inp, dt, f = workload_sim(5, n_shots=2, nt=nt)
    fw = sim.forward(f)
    prob = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot="none")
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL


# ----------------------------------------------------------------------------
# full shot batches in the launch configuration the benchmark times; shots
# are independent, so the oracle checks sampled shots one by one


def _subset_sim(inp, sel, dt, batched=False):
    wl = inp.wl
    vmax = oracle.c0() / np.sqrt(inp.eps_min)
    eps = inp.eps_r[sel] if batched else inp.eps_r
    sig = inp.sigma[sel] if batched else inp.sigma
    return oracle_sim(eps, sig, inp.src_idx[sel], inp.rec_idx[sel], wl.order, wl.h, dt, wl.n_pml,
                      wl.f0, vmax=vmax, round_f32=True)


@pytest.mark.parametrize("snapshot", ["ckpt", "ckpt_ey"])
def test_workload4_all_shots_sampled(snapshot):
    """2128x2128 order 4, all 8 shots, checkpoints every 64 steps (the
    benchmark's launch plan with "ckpt_ey"), nt 137 = two full segments + a
    partial one; records and per-shot gradients of shots 0 and 7 against the
    oracle."""
    nt, sel = 137, [0, 7]
    sim, inp, dt, f = workload_sim(4, n_shots=8, nt=nt)
    g = synth.rng(404)
    res = f32(g.normal(size=(nt, 8, inp.wl.n_rec)))
    prob = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot=snapshot, ckpt_every=64)
    rec = run_forward(prob, f)
    gca, gcb, gf = run_adjoint(prob, res)
    assert prob.status() == mwtm.MW_OK
    del prob
    sub = _subset_sim(inp, sel, dt)
    ck = sub.fwd_adj_ckpt(f[:, sel], res[:, sel], 64)
    assert rel_l2(rec[:, sel], ck["rec"]) <= REC_TOL
    assert rel_l2(gca[sel], ck["gca"]) <= GRAD_TOL
    assert rel_l2(gcb[sel], ck["gcb"]) <= GRAD_TOL
    assert rel_l2(gf[:, sel], ck["grad_f"]) <= GRAD_TOL


def test_workload5_all_shots_sampled():
    """552x552 order 8, all 256 shots with per-shot models, records only,
    nt 300; shots 0, 131 and 255 against the oracle."""
    nt, sel = 300, [0, 131, 255]
    inp = synth.make_inputs(5)
    wl = inp.wl
    vmax = oracle.c0() / np.sqrt(inp.eps_min)
    dt = wl.cfl_fraction * oracle.cfl_dt(wl.order, wl.h, wl.h, vmax)
    f = f32(inp.wavelet(dt, nt))
    sim = oracle_sim(inp.eps_r, inp.sigma, inp.src_idx, inp.rec_idx, wl.order, wl.h, dt, wl.n_pml,
                     wl.f0, vmax=vmax, round_f32=True)
    prob = problem_from_sim(sim, nt, dt, wl.n_pml, snapshot="none")
    rec = run_forward(prob, f)
    assert prob.status() == mwtm.MW_OK
    del prob
    sub = _subset_sim(inp, sel, dt, batched=True)
    fw = sub.forward(f[:, sel])
    assert rel_l2(rec[:, sel], fw["rec"]) <= REC_TOL


def test_workload5_per_shot_model_gradients_sampled():
    """Per-shot models (552x552 order 8, all 256 shots): the adjoint keeps one
    gradient per shot and the chain rule runs per shot (no shot sum).
    Checkpoints every 64 steps, nt 130; shots 0 and 255 against the oracle."""
    nt, sel = 130, [0, 255]
    inp = synth.make_inputs(5)
    wl = inp.wl
    vmax = oracle.c0() / np.sqrt(inp.eps_min)
    dt = wl.cfl_fraction * oracle.cfl_dt(wl.order, wl.h, wl.h, vmax)
    f = f32(inp.wavelet(dt, nt))
    g = synth.rng(505)
    res = f32(g.normal(size=(nt, wl.n_shots, wl.n_rec)))
    sim = oracle_sim(inp.eps_r, inp.sigma, inp.src_idx, inp.rec_idx, wl.order, wl.h, dt, wl.n_pml,
                     wl.f0, vmax=vmax, round_f32=True)
    prob = problem_from_sim(sim, nt, dt, wl.n_pml, snapshot="ckpt", ckpt_every=64)
    run_forward(prob, f)
    gca_t, gcb_t, _ = prob.adjoint(torch.as_tensor(res, dtype=torch.float32).cuda())
    ge_t, gs_t = prob.eps_sigma_gradient(gca_t, gcb_t)
    torch.cuda.synchronize()
    assert prob.status() == mwtm.MW_OK
    gca, gcb = gca_t.cpu().numpy(), gcb_t.cpu().numpy()
    ge, gs = ge_t.cpu().numpy(), gs_t.cpu().numpy()
    del prob, gca_t, gcb_t, ge_t, gs_t
    sub = _subset_sim(inp, sel, dt, batched=True)
    ck = sub.fwd_adj_ckpt(f[:, sel], res[:, sel], 64)
    assert rel_l2(gca[sel], ck["gca"]) <= GRAD_TOL
    assert rel_l2(gcb[sel], ck["gcb"]) <= GRAD_TOL
    ge_o, gs_o = oracle.eps_sigma_grad(sub.ca, sub.cb, dt, ck["gca"], ck["gcb"])
    assert rel_l2(ge[sel], ge_o) <= GRAD_TOL
    assert rel_l2(gs[sel], gs_o) <= GRAD_TOL


def test_workload3_all_shots_sampled_bf16():
    """1064x1064 order 8, all 16 shots, nt 150: fp32-storage gradients of
    shots 0 and 15 against the oracle, and the bf16-storage gradient error
    against fp32 storage on every shot (reported, <= 2e-2)."""
    nt, sel = 150, [0, 15]
    sim, inp, dt, f = workload_sim(3, n_shots=16, nt=nt)
    g = synth.rng(303)
    res = f32(g.normal(size=(nt, 16, inp.wl.n_rec)))
    p32 = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot="fp32")
    rec = run_forward(p32, f)
    gca32, gcb32, _ = run_adjoint(p32, res)
    del p32
    p16 = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot="bf16")
    run_forward(p16, f)
    gca16, gcb16, _ = run_adjoint(p16, res)
    del p16
    sub = _subset_sim(inp, sel, dt)
    ck = sub.fwd_adj_ckpt(f[:, sel], res[:, sel], 32)
    assert rel_l2(rec[:, sel], ck["rec"]) <= REC_TOL
    assert rel_l2(gca32[sel], ck["gca"]) <= GRAD_TOL
    assert rel_l2(gcb32[sel], ck["gcb"]) <= GRAD_TOL
    e_ca, e_cb = rel_l2(gca16, gca32), rel_l2(gcb16, gcb32)
    print(f"bf16-snapshot gradient error vs fp32 storage (16 shots): Ca {e_ca:.3e} Cb {e_cb:.3e}")
    assert e_ca <= 2e-2 and e_cb <= 2e-2


# ----------------------------------------------------------------------------
# properties of the GPU path itself


@pytest.mark.parametrize("order", [2, 4, 8])
def test_gpu_dot_product(order):
    """<A f, y> = <f, A^T y> in fp32 on the GPU (CPML on), <= 1e-5."""
    sim, dt, _ = small_sim(500 + order, 96, 136, 3, 2, 7, order, 8, round_f32=True)
    nt = 200
    g = synth.rng(order)
    f = f32(g.normal(size=(nt, 3, 2)))
    y = f32(g.normal(size=(nt, 3, 7)))
    prob = problem_from_sim(sim, nt, dt, 8)
    r = run_forward(prob, f)
    _, _, gf = run_adjoint(prob, y)
    lhs, rhs = float(np.sum(r * y)), float(np.sum(f * gf))
    assert abs(lhs - rhs) <= 1e-5 * max(abs(lhs), abs(rhs))


def test_checkpoint_gradient_equals_full_storage_bitwise():
    sim, dt, _ = small_sim(601, 80, 100, 2, 1, 6, 4, 6, round_f32=True)
    nt = 150
    g = synth.rng(9)
    f = f32(g.normal(size=(nt, 2, 1)))
    res = f32(g.normal(size=(nt, 2, 6)))
    out = {}
    for mode, C in (("fp32", 1), ("ckpt", 64), ("ckpt", 7)):
        prob = problem_from_sim(sim, nt, dt, 6, snapshot=mode, ckpt_every=C)
        rec = run_forward(prob, f)
        out[(mode, C)] = (rec,) + run_adjoint(prob, res)
    a = out[("fp32", 1)]
    for key in (("ckpt", 64), ("ckpt", 7)):
        b = out[key]
        for x, y in zip(a, b):
            assert np.array_equal(x, y), key


def test_run_to_run_bitwise_determinism():
    sim, dt, _ = small_sim(602, 64, 128, 2, 3, 6, 8, 6, round_f32=True)
    sim.src_idx[0, 1] = sim.src_idx[0, 0]
    nt = 80
    g = synth.rng(10)
    f = f32(g.normal(size=(nt, 2, 3)))
    res = f32(g.normal(size=(nt, 2, 6)))
    runs = []
    for _ in range(2):
        prob = problem_from_sim(sim, nt, dt, 6)
        runs.append((run_forward(prob, f),) + run_adjoint(prob, res))
    for x, y in zip(*runs):
        assert np.array_equal(x, y)


def test_model_prep_matches_oracle():
    eps, sig, _, _ = synth.small_case(7, 40, 64, 1, 1, 1, sigma_max=0.05)
    mu = synth.rng(8).uniform(1.0, 3.0, size=eps.shape)
    dt = 2e-11
    ca_o, cb_o, cq_o = oracle.model(f32(eps), f32(sig), f32(mu), dt)
    p = mwtm.make_params(ny=40, nx=64, order=4, n_shots=1, nt=1, dt=dt, dy=0.01, dx=0.01,
                         n_pml=0, cq_is_scalar=0, allow_unstable=1)
    dev = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float32)).cuda()
    ca, cb, cq = (torch.empty((40, 64), device="cuda") for _ in range(3))
    mwtm.model_from_eps_sigma(p, dev(eps), dev(sig), dev(mu), ca, cb, cq)
    torch.cuda.synchronize()
    for gpu, ref in ((ca, ca_o), (cb, cb_o), (cq, cq_o)):
        assert np.max(np.abs(gpu.cpu().numpy() - ref) / np.abs(ref)) <= 1e-6


def test_cpml_profiles_match_oracle():
    ny, nx, n_pml, h, dt, vmax, f0 = 60, 72, 9, 0.02, 4e-11, 1.5e8, 3e8
    p = mwtm.make_params(ny=ny, nx=nx, order=4, n_shots=1, nt=1, dt=dt, dy=h, dx=h, n_pml=n_pml,
                         vmax=vmax)
    out = torch.empty(6 * (ny + nx), device="cuda")
    mwtm.cpml_profiles(p, f0, 1e-3, out)
    torch.cuda.synchronize()
    ref = np.concatenate(list(oracle.cpml(ny, n_pml, h, dt, vmax, f0)) +
                         list(oracle.cpml(nx, n_pml, h, dt, vmax, f0)))
    got = out.cpu().numpy()
    assert np.allclose(got, ref, rtol=1e-6, atol=1e-30)


def test_combine_and_chain_rule_match_oracle():
    g = synth.rng(11)
    S, ny, nx = 5, 24, 32
    gs = f32(g.normal(size=(S, ny, nx)))
    p = mwtm.make_params(ny=ny, nx=nx, order=2, n_shots=S, nt=1, dt=1e-11, dy=0.01, dx=0.01,
                         allow_unstable=1)
    t = torch.as_tensor(gs, dtype=torch.float32).cuda()
    out = torch.full((ny, nx), 2.0, device="cuda")
    mwtm.combine_grad(p, t, out, accumulate=True)
    torch.cuda.synchronize()
    assert rel_l2(out.cpu().numpy(), oracle.combine(gs) + 2.0) <= 1e-6
    eps = g.uniform(2, 9, size=(ny, nx))
    sig = g.uniform(0, 0.05, size=(ny, nx))
    dt = 3e-11
    ca, cb, _ = oracle.model(eps, sig, None, dt)
    ca, cb = f32(ca), f32(cb)
    gca, gcb = f32(g.normal(size=(ny, nx))), f32(g.normal(size=(ny, nx)))
    ge_o, gs_o = oracle.eps_sigma_grad(ca, cb, dt, gca, gcb)
    d = lambda a: torch.as_tensor(a, dtype=torch.float32).cuda()
    ge, gsg = torch.empty((ny, nx), device="cuda"), torch.empty((ny, nx), device="cuda")
    mwtm.grad_eps_sigma(ny * nx, dt, d(ca), d(cb), d(gca), d(gcb), ge, gsg)
    torch.cuda.synchronize()
    assert rel_l2(ge.cpu().numpy(), ge_o) <= 1e-5
    assert rel_l2(gsg.cpu().numpy(), gs_o) <= 1e-5


def test_residual_and_misfit():
    g = synth.rng(12)
    d, o = f32(g.normal(size=10007)), f32(g.normal(size=10007))
    res_o, J_o = oracle.residual(d, o)
    dt = lambda a: torch.as_tensor(a, dtype=torch.float32).cuda()
    res = torch.empty(10007, device="cuda")
    J = torch.zeros(1, dtype=torch.float64, device="cuda")
    mwtm.residual(10007, dt(d), dt(o), res, J)
    torch.cuda.synchronize()
    r32 = res.cpu().numpy().astype(np.float64)
    assert np.array_equal(r32, f32(res_o))
    # the library's J is 1/2 sum of the fp32 residual squared (fp64 sum)
    assert float(J.cpu()[0]) == pytest.approx(0.5 * float(np.sum(r32 * r32)), rel=1e-12)
    assert float(J.cpu()[0]) == pytest.approx(J_o, rel=1e-6)


# ----------------------------------------------------------------------------
# error reporting (host-side checks and device status words; nothing faults)


def test_nonfinite_model_is_reported():
    sim, dt, _ = small_sim(701, 20, 24, 1, 1, 2, 4, 3, round_f32=True)
    sim.cb[5, 5] = np.nan
    prob = problem_from_sim(sim, 10, dt, 3, check_finite=True)
    run_forward(prob, np.ones((10, 1, 1)))
    assert prob.status() == mwtm.MW_ERR_NONFINITE
    assert prob.status() == mwtm.MW_OK  # cleared


def test_out_of_range_index_is_reported_not_faulted():
    sim, dt, _ = small_sim(702, 20, 24, 1, 1, 2, 4, 3, round_f32=True)
    sim.src_idx[0, 0] = 20 * 24 + 5
    prob = problem_from_sim(sim, 5, dt, 3)
    run_forward(prob, np.ones((5, 1, 1)))
    assert prob.status() == mwtm.MW_ERR_ARG


def test_host_side_argument_errors():
    base = dict(ny=32, nx=32, order=4, n_shots=1, n_src=1, n_rec=1, nt=4, dt=1e-11, dy=0.01,
                dx=0.01, n_pml=4, vmax=1.5e8)
    assert mwtm.validate(mwtm.make_params(**base)) == mwtm.MW_OK
    assert mwtm.validate(mwtm.make_params(**{**base, "nx": 30})) == mwtm.MW_ERR_ARG
    assert mwtm.validate(mwtm.make_params(**{**base, "order": 5})) == mwtm.MW_ERR_ARG
    assert mwtm.validate(mwtm.make_params(**{**base, "n_pml": 20})) == mwtm.MW_ERR_ARG
    assert mwtm.validate(mwtm.make_params(**{**base, "dt": 1e-9})) == mwtm.MW_ERR_CFL
    p = mwtm.make_params(**{**base, "snap_mode": 1})
    ws = torch.empty(16, device="cuda")
    dummy = torch.zeros(64 * 64, device="cuda")
    idx = torch.zeros((1, 1), dtype=torch.int64, device="cuda")
    with pytest.raises(mwtm.MWError) as e:
        mwtm.tm_forward(p, dummy, dummy, dummy, dummy, dummy, idx, idx, None, dummy, ws)
    assert e.value.code == mwtm.MW_ERR_WORKSPACE


def test_no_sources_and_no_receivers():
    """A problem with receivers but no sources (the field comes from a given
    initial state), and one with sources but no receivers (the adjoint then
    has no residual to inject, so its gradients vanish)."""
    S, ny, nx, nt = 2, 44, 64, 40
    sim0, dt, _ = small_sim(930, ny, nx, S, 0, 5, 4, 5, round_f32=True)
    st0 = np.zeros((7, S, ny, nx))
    st0[:3] = f32(synth.rng(931).normal(size=(3, S, ny, nx)))  # Ey, Hx, Hz; memories zero
    fw = sim0.forward(np.zeros((nt, S, 0)), state=st0)
    prob = problem_from_sim(sim0, nt, dt, 5)
    state = prob.new_state()
    SN = S * ny * nx
    state[:3 * SN] = torch.as_tensor(st0[:3].reshape(-1), dtype=torch.float32)
    rec = run_forward(prob, np.zeros((nt, S, 1)), state=state)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    assert prob.status() == mwtm.MW_OK

    sim1, dt1, _ = small_sim(932, ny, nx, S, 2, 0, 4, 5, round_f32=True)
    f = f32(synth.rng(933).normal(size=(nt, S, 2)))
    prob1 = problem_from_sim(sim1, nt, dt1, 5)
    run_forward(prob1, f)
    gca, gcb, gf = run_adjoint(prob1, np.zeros((nt, S, 1)))
    assert np.all(gca == 0) and np.all(gcb == 0) and np.all(gf == 0)
    assert prob1.status() == mwtm.MW_OK
