"""Checkpoint mode with the E snapshot alone (snapshot "ckpt_ey"): the replay
keeps E^t only and the Cb gradient is formed by summation by parts from the
adjoint's E-update term, with the end terms at t = 0, t = nt, the receivers
and the sources added at the end of the sweep.

The oracle computes the gradient from its definition (curl^t lambda^{t+1});
these tests hold the regrouped sum to it, to the fp32 gradient tolerance, in
every case where one of the end terms is live: partial segments, nt = 1,
a given initial forward state (E^0 != 0), a given adjoint start state,
duplicate and inactive indices, sources on receivers, the PML mask, no
grad_f requested.  grad_ca, grad_f and the adjoint state must equal those of
the pair-store checkpoint mode bit for bit (same arithmetic, same order)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from adjoint_state_gradients_b200 import api, mwtm, synth
from tests._cases import rel_l2, small_sim, workload_sim
from tests._gpu import f32, problem_from_sim, run_adjoint, run_forward

pytestmark = pytest.mark.gpu

REC_TOL = 1e-5
GRAD_TOL = 1e-4


def _oracle(sim, f, res, state=None, adj=None):
    fw = sim.forward(f, snapshots=True, state=state)
    ad = sim.adjoint(res, fw["snap_ey"], fw["snap_curl"], adj=adj)
    return fw, ad


def _check_grads(gca, gcb, gf, ad, gf_tol=GRAD_TOL):
    assert rel_l2(gca, ad["gca"]) <= GRAD_TOL
    assert rel_l2(gcb, ad["gcb"]) <= GRAD_TOL
    if gf is not None and ad["grad_f"] is not None and ad["grad_f"].size:
        assert rel_l2(gf, ad["grad_f"]) <= gf_tol


@pytest.mark.parametrize("order,ny,nx,S,n_pml,batched,cq_array,C", [
    (2, 37, 44, 1, 4, False, False, 16),
    (4, 61, 140, 2, 6, False, False, 20),
    (6, 50, 132, 3, 5, True, False, 64),
    (8, 70, 264, 2, 7, False, True, 13),
    (8, 33, 40, 1, 0, False, False, 57),
    (4, 150, 20, 2, 3, True, True, 7),
])
def test_ckpt_ey_matches_oracle(order, ny, nx, S, n_pml, batched, cq_array, C):
    sim, dt, _ = small_sim(100 + order + ny, ny, nx, S, 2, 5, order, n_pml, batched=batched,
                           cq_array=cq_array, round_f32=True, sigma_max=0.02)
    nt = 57
    g = synth.rng(7 + order)
    f = f32(g.normal(size=(nt, S, 2)))
    res = f32(g.normal(size=(nt, S, 5)))
    fw, ad = _oracle(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="ckpt_ey", ckpt_every=C)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    adj_state = prob.new_state()
    gca, gcb, gf = run_adjoint(prob, res, adj_state=adj_state)
    _check_grads(gca, gcb, gf, ad)
    ast = api.unpack_state(prob.p, adj_state)
    for i, nm in enumerate(oracle.FIELDS):
        if np.abs(ad["adj"][i]).max() > 0:
            assert rel_l2(ast[nm], ad["adj"][i]) <= GRAD_TOL, nm
    assert prob.status() == mwtm.MW_OK


@pytest.mark.parametrize("order", [2, 4, 8])
def test_ckpt_ey_bitwise_against_pair_checkpoints(order):
    """Same lambda, same gCa, same grad_f as the pair-store checkpoint mode."""
    S, ny, nx, n_pml, nt, C = 2, 58, 152, 5, 70, 16
    sim, dt, _ = small_sim(710 + order, ny, nx, S, 2, 6, order, n_pml, round_f32=True,
                           sigma_max=0.02)
    g = synth.rng(711 + order)
    f = torch.as_tensor(f32(g.normal(size=(nt, S, 2))), dtype=torch.float32).cuda()
    res = torch.as_tensor(f32(g.normal(size=(nt, S, 6))), dtype=torch.float32).cuda()
    out = {}
    for mode in ("ckpt", "ckpt_ey"):
        prob = problem_from_sim(sim, nt, dt, n_pml, snapshot=mode, ckpt_every=C)
        rec = prob.forward(f)
        adj_state = prob.new_state()
        gca, gcb, gf = prob.adjoint(res, grad_f=True, adj_state=adj_state)
        torch.cuda.synchronize()
        assert prob.status() == mwtm.MW_OK
        out[mode] = [t.cpu().numpy() for t in (rec, gca, gcb, gf, adj_state)]
    a, b = out["ckpt"], out["ckpt_ey"]
    for k, nm in ((0, "rec"), (1, "gca"), (3, "grad_f"), (4, "adj_state")):
        assert np.array_equal(a[k], b[k]), nm
    assert rel_l2(b[2], a[2]) <= GRAD_TOL


@pytest.mark.parametrize("nt,C", [(1, 64), (2, 1), (3, 2), (64, 64), (65, 64), (40, 7)])
def test_ckpt_ey_step_counts(nt, C):
    """nt = 1 (only the t = 0 and t = nt end terms), one-step segments, a
    ragged last segment."""
    sim, dt, _ = small_sim(300 + nt, 40, 48, 2, 1, 3, 4, 5, round_f32=True)
    g = synth.rng(nt + 1000)
    f = f32(g.normal(size=(nt, 2, 1)))
    res = f32(g.normal(size=(nt, 2, 3)))
    fw, ad = _oracle(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, 5, snapshot="ckpt_ey", ckpt_every=C)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    gca, gcb, gf = run_adjoint(prob, res)
    _check_grads(gca, gcb, gf, ad)


def test_ckpt_ey_given_initial_and_adjoint_states():
    """E^0 != 0 (the -Ca lam^1 E^0 term) and a nonzero adjoint start state
    (the lam~^{nt} E^{nt} term, E^{nt} from the last replayed segment)."""
    S, ny, nx, n_pml, nt, C = 2, 44, 64, 5, 45, 16
    sim, dt, _ = small_sim(820, ny, nx, S, 2, 4, 4, n_pml, round_f32=True, sigma_max=0.02)
    g = synth.rng(821)
    st0 = np.zeros((7, S, ny, nx))
    st0[:3] = f32(0.1 * g.normal(size=(3, S, ny, nx)))
    ad0 = np.zeros((7, S, ny, nx))
    ad0[:3] = f32(g.normal(size=(3, S, ny, nx)))
    f = f32(g.normal(size=(nt, S, 2)))
    res = f32(g.normal(size=(nt, S, 4)))
    fw, ad = _oracle(sim, f, res, state=st0, adj=ad0)
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="ckpt_ey", ckpt_every=C)
    SN = S * ny * nx
    state = prob.new_state()
    state[:3 * SN] = torch.as_tensor(st0[:3].reshape(-1), dtype=torch.float32)
    rec = run_forward(prob, f, state=state)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    adj_state = prob.new_state()
    adj_state[:3 * SN] = torch.as_tensor(ad0[:3].reshape(-1), dtype=torch.float32)
    gca, gcb, gf = run_adjoint(prob, res, adj_state=adj_state)
    _check_grads(gca, gcb, gf, ad)
    assert prob.status() == mwtm.MW_OK


def test_ckpt_ey_duplicates_inactive_and_shared_cells():
    """Duplicate sources and receivers, inactive entries, a source on a
    receiver: the end-term sums follow each entry."""
    sim, dt, _ = small_sim(401, 30, 36, 2, 4, 6, 4, 4, round_f32=True)
    sim.src_idx[0] = [100, 100, -1, 333]
    sim.src_idx[1] = [-1, -1, -1, 7]
    sim.rec_idx[0, :3] = [100, 100, -1]
    sim.rec_idx[1, 0] = 7
    nt = 40
    g = synth.rng(5)
    f = f32(g.normal(size=(nt, 2, 4)))
    res = f32(g.normal(size=(nt, 2, 6)))
    fw, ad = _oracle(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, 4, snapshot="ckpt_ey", ckpt_every=8)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    gca, gcb, gf = run_adjoint(prob, res)
    _check_grads(gca, gcb, gf, ad)
    assert np.all(gf[:, 1, :3] == 0.0)


def test_ckpt_ey_without_grad_f_and_with_mask():
    """No grad_f buffer (lambda at the sources still feeds the source term),
    and the PML mask on both gradients."""
    n_pml = 6
    sim, dt, _ = small_sim(402, 44, 52, 1, 1, 4, 4, n_pml, round_f32=True)
    nt = 50
    g = synth.rng(6)
    f = f32(g.normal(size=(nt, 1, 1)))
    res = f32(g.normal(size=(nt, 1, 4)))
    fw, ad = _oracle(sim, f, res)
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="ckpt_ey", ckpt_every=16)
    run_forward(prob, f)
    gca, gcb, _ = run_adjoint(prob, res, grad_f=False)
    _check_grads(gca, gcb, None, ad)
    mask = np.zeros((44, 52))
    mask[n_pml:44 - n_pml, n_pml:52 - n_pml] = 1.0
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="ckpt_ey", ckpt_every=16,
                            grad_mask=True)
    run_forward(prob, f)
    gca, gcb, _ = run_adjoint(prob, res)
    assert rel_l2(gca, ad["gca"] * mask) <= GRAD_TOL
    assert rel_l2(gcb, ad["gcb"] * mask) <= GRAD_TOL
    assert np.all(gcb[0][mask == 0] == 0.0)


def test_ckpt_ey_no_sources_no_receivers():
    S, ny, nx, nt = 2, 44, 64, 30
    sim, dt, _ = small_sim(932, ny, nx, S, 2, 0, 4, 5, round_f32=True)
    f = f32(synth.rng(933).normal(size=(nt, S, 2)))
    prob = problem_from_sim(sim, nt, dt, 5, snapshot="ckpt_ey", ckpt_every=8)
    run_forward(prob, f)
    gca, gcb, gf = run_adjoint(prob, np.zeros((nt, S, 1)))
    assert np.all(gca == 0) and np.all(gcb == 0) and np.all(gf == 0)
    sim, dt, _ = small_sim(934, ny, nx, S, 0, 4, 4, 5, round_f32=True)
    res = f32(synth.rng(935).normal(size=(nt, S, 4)))
    fw, ad = _oracle(sim, np.zeros((nt, S, 0)), res)
    prob = problem_from_sim(sim, nt, dt, 5, snapshot="ckpt_ey", ckpt_every=8)
    rec = run_forward(prob, np.zeros((nt, S, 1)))
    assert np.all(rec == 0)
    gca, gcb, _ = run_adjoint(prob, res)
    assert np.all(gca == 0) and np.all(gcb == 0)
    assert prob.status() == mwtm.MW_OK


@pytest.mark.parametrize("mode", ["ckpt", "ckpt_ey"])
def test_forward_stored_tail_is_bitwise_the_replay(mode):
    """ckpt_tail: the forward stores the last steps' snapshots itself and the
    adjoint replays only the steps before them.  The replay recomputes the
    same values, so every output equals the tail-free run bit for bit, for
    tails inside a segment, on a segment boundary, of the whole run and
    longer than it; with a given adjoint start state (the final E then comes
    from the tail store)."""
    S, ny, nx, n_pml, nt, C = 2, 46, 72, 5, 40, 8
    sim, dt, _ = small_sim(900, ny, nx, S, 2, 4, 4, n_pml, round_f32=True, sigma_max=0.02)
    g = synth.rng(901)
    f = torch.as_tensor(f32(g.normal(size=(nt, S, 2))), dtype=torch.float32).cuda()
    res = torch.as_tensor(f32(g.normal(size=(nt, S, 4))), dtype=torch.float32).cuda()
    ad0 = torch.as_tensor(f32(g.normal(size=(3 * S * ny * nx,))), dtype=torch.float32).cuda()
    out = {}
    for tail in (0, 3, 8, 21, 40, 100):
        prob = problem_from_sim(sim, nt, dt, n_pml, snapshot=mode, ckpt_every=C, ckpt_tail=tail)
        rec = prob.forward(f)
        adj_state = prob.new_state()
        adj_state[:ad0.numel()] = ad0
        gca, gcb, gf = prob.adjoint(res, grad_f=True, adj_state=adj_state)
        torch.cuda.synchronize()
        assert prob.status() == mwtm.MW_OK
        out[tail] = [t.cpu().numpy() for t in (rec, gca, gcb, gf, adj_state)]
    for tail in (3, 8, 21, 40, 100):
        for k, nm in enumerate(("rec", "gca", "gcb", "grad_f", "adj_state")):
            assert np.array_equal(out[tail][k], out[0][k]), (tail, nm)


def test_forward_stored_tail_matches_oracle_and_born():
    S, ny, nx, n_pml, nt, C = 2, 46, 72, 5, 45, 16
    sim, dt, _ = small_sim(902, ny, nx, S, 2, 4, 4, n_pml, round_f32=True, sigma_max=0.02)
    g = synth.rng(903)
    f = f32(g.normal(size=(nt, S, 2)))
    res = f32(g.normal(size=(nt, S, 4)))
    fw, ad = _oracle(sim, f, res)
    dca = f32(1e-3 * g.normal(size=(ny, nx)))
    dcb = f32(1e-3 * g.normal(size=(ny, nx)))
    want_born = sim.born(fw["snap_ey"], fw["snap_curl"], dca, dcb)
    prob = problem_from_sim(sim, nt, dt, n_pml, snapshot="ckpt_ey", ckpt_every=C, ckpt_tail=20)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    born = prob.born(torch.as_tensor(dca, dtype=torch.float32),
                     torch.as_tensor(dcb, dtype=torch.float32)).cpu().numpy().astype(np.float64)
    assert rel_l2(born, want_born) <= REC_TOL
    gca, gcb, gf = run_adjoint(prob, res)
    _check_grads(gca, gcb, gf, ad)
    assert prob.status() == mwtm.MW_OK


def test_full_length_sweep_matches_pair_checkpoints():
    """The 2128^2 order-4 workload over its full 4000 steps (2 of its 8 shots):
    the summation-by-parts dJ/dCb of the E-alone checkpoints, with and without
    the forward-stored tail, against the direct sum of the pair checkpoints
    (both fp32); dJ/dCa and dJ/df bitwise."""
    nt = 4000
    sim, inp, dt, f = workload_sim(4, n_shots=2, nt=nt)
    g = synth.rng(4004)
    res = torch.as_tensor(f32(g.normal(size=(nt, 2, inp.wl.n_rec))), dtype=torch.float32).cuda()
    f_d = torch.as_tensor(np.asarray(f, dtype=np.float32)).cuda()
    out = {}
    for mode, tail in (("ckpt", 0), ("ckpt_ey", 0), ("ckpt_ey", 320)):
        prob = problem_from_sim(sim, nt, dt, inp.wl.n_pml, snapshot=mode, ckpt_every=64,
                                ckpt_tail=tail)
        prob.forward(f_d)
        gca, gcb, gf = prob.adjoint(res, grad_f=True)
        torch.cuda.synchronize()
        assert prob.status() == mwtm.MW_OK
        out[(mode, tail)] = [t.cpu().numpy().astype(np.float64) for t in (gca, gcb, gf)]
        del prob
    ref = out[("ckpt", 0)]
    for key in (("ckpt_ey", 0), ("ckpt_ey", 320)):
        assert np.array_equal(out[key][0], ref[0]) and np.array_equal(out[key][2], ref[2])
        err = rel_l2(out[key][1], ref[1])
        print(f"{key}: rel-L2 of dJ/dCb against the direct sum {err:.2e}")
        assert err <= GRAD_TOL
    assert np.array_equal(out[("ckpt_ey", 0)][1], out[("ckpt_ey", 320)][1])
