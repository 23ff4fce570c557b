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
    ("fp32-host", 4, False), ("fp32", 8, True), ("ckpt", 8, False)])
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
