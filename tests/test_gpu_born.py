"""Born (linearised) forward on the GPU against the oracle, and the GPU's
own Born / adjoint-gradient pair checked by a dot test.

The background snapshots are those the forward stored (fp32, bf16 or FP8, in
device or pinned host memory) or a checkpoint replay; the oracle applies the
same rounding to its own snapshots before its Born map."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from adjoint_state_gradients_b200 import api, synth
from tests._cases import rel_l2, small_sim
from tests._gpu import f32, problem_from_sim, run_forward

pytestmark = pytest.mark.gpu

REC_TOL = 1e-5


def _case(order, batched, seed):
    sim, dt, _ = small_sim(seed, 56, 152, 2, 2, 6, order, 6, round_f32=True, sigma_max=0.02,
                           batched=batched)
    nt = 70
    g = synth.rng(seed + 1)
    f = f32(g.normal(size=(nt, 2, 2)))
    dca = f32(0.01 * g.normal(size=sim.ca.shape))
    dcb = f32(0.01 * float(np.mean(sim.cb)) * g.normal(size=sim.ca.shape))
    return sim, dt, nt, f, dca, dcb, g


def _problem(sim, nt, dt, mode):
    if mode == "fp32-host":
        kw = dict(vmax=1.0, allow_unstable=True, snapshot="fp32", snapshot_host=True,
                  batched=bool(sim.model_batched))
        prob = api.Problem(sim.ny, sim.nx, sim.order, sim.dy, sim.dx, dt, nt, 6, sim.src_idx,
                           sim.rec_idx, **kw)
        prob.set_coefficients(sim.ca, sim.cb, sim.cq,
                              np.concatenate(list(sim.prof_y) + list(sim.prof_x)))
        return prob
    return problem_from_sim(sim, nt, dt, 6, snapshot=mode, ckpt_every=32)


@pytest.mark.parametrize("mode,order,batched", [
    ("fp32", 4, False), ("bf16", 4, False), ("fp8", 4, False), ("ckpt", 4, False),
    ("fp32-host", 4, False), ("fp32", 8, True), ("ckpt", 8, False), ("ckpt_ey", 4, False)])
def test_born_forward_matches_oracle(mode, order, batched):
    sim, dt, nt, f, dca, dcb, _ = _case(order, batched, 800 + order)
    fw = sim.forward(f, snapshots=True)
    quant = {"bf16": oracle.quant_bf16, "fp8": oracle.quant_fp8}.get(mode, lambda x: x)
    want = sim.born(quant(fw["snap_ey"]), quant(fw["snap_curl"]), dca, dcb)
    prob = _problem(sim, nt, dt, mode)
    rec = run_forward(prob, f)
    assert rel_l2(rec, fw["rec"]) <= REC_TOL
    got = prob.born(torch.as_tensor(dca, dtype=torch.float32), torch.as_tensor(dcb, dtype=torch.float32))
    torch.cuda.synchronize()
    assert prob.status() == 0
    got = got.cpu().numpy().astype(np.float64)
    assert np.abs(want).max() > 0
    assert rel_l2(got, want) <= REC_TOL


@pytest.mark.parametrize("order", [4, 8])
def test_gpu_born_is_the_transpose_of_the_gpu_gradient(order):
    """<B dm, r> = <dm, sum_s grad_s(r)> with both maps run on the GPU (fp32)."""
    sim, dt, nt, f, dca, dcb, g = _case(order, False, 820 + order)
    prob = problem_from_sim(sim, nt, dt, 6, snapshot="fp32")
    run_forward(prob, f)
    born = prob.born(torch.as_tensor(dca, dtype=torch.float32),
                     torch.as_tensor(dcb, dtype=torch.float32)).cpu().numpy().astype(np.float64)
    r = f32(g.normal(size=born.shape))
    gca, gcb, _ = prob.adjoint(torch.as_tensor(r, dtype=torch.float32).cuda())
    torch.cuda.synchronize()
    assert prob.status() == 0
    lhs = float(np.sum(born * r))
    rhs = float(np.sum(dca * gca.sum(0).cpu().numpy()) + np.sum(dcb * gcb.sum(0).cpu().numpy()))
    assert abs(lhs - rhs) <= 1e-5 * max(abs(lhs), abs(rhs))


@pytest.mark.parametrize("mode", ["ckpt", "fp32", "fp8"])
def test_workspace_reuse_adjoint_twice_and_born_around_it(mode):
    """One forward, then adjoint, Born, adjoint, Born on the same workspace:
    each repeated call returns bit-identical results (the checkpoint replays
    and the Born state never disturb what a later call needs)."""
    sim, dt, nt, f, dca, dcb, g = _case(4, False, 840)
    prob = _problem(sim, nt, dt, mode)
    run_forward(prob, f)
    r = torch.as_tensor(f32(g.normal(size=(nt, 2, 6))), dtype=torch.float32).cuda()
    dca_t = torch.as_tensor(dca, dtype=torch.float32)
    dcb_t = torch.as_tensor(dcb, dtype=torch.float32)
    g1 = [t.clone() for t in prob.adjoint(r)[:2]]
    b1 = prob.born(dca_t, dcb_t).clone()
    g2 = [t.clone() for t in prob.adjoint(r)[:2]]
    b2 = prob.born(dca_t, dcb_t).clone()
    torch.cuda.synchronize()
    assert prob.status() == 0
    assert torch.equal(g1[0], g2[0]) and torch.equal(g1[1], g2[1])
    assert torch.equal(b1, b2)


def test_born_with_no_steps_is_a_no_op():
    sim, dt, _, f, dca, dcb, _ = _case(4, False, 850)
    prob = problem_from_sim(sim, 0, dt, 6, snapshot="fp32")
    rec = torch.full((1, 2, 6), 7.0, device="cuda")
    prob.born(torch.as_tensor(dca, dtype=torch.float32), torch.as_tensor(dcb, dtype=torch.float32),
              rec=rec)
    torch.cuda.synchronize()
    assert prob.status() == 0
    assert float(rec.min()) == 7.0 and float(rec.max()) == 7.0
