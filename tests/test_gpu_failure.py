"""Failure detection on the GPU without a fault: a stage wait that nothing
completes gives up after its bounded poll count, the host reads
MW_ERR_TIMEOUT from the workspace's status words, the stencil kernels stand
down while that status is set, and once it has been reported the same
workspace and context compute correct results again."""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

from adjoint_state_gradients_b200 import mwtm, synth
from tests._cases import small_sim
from tests._gpu import f32, problem_from_sim, run_forward

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    sim, dt, _ = small_sim(31, 40, 88, 2, 1, 4, 4, 5, round_f32=True)
    nt = 30
    f = f32(synth.rng(3).normal(size=(nt, 2, 1)))
    prob = problem_from_sim(sim, nt, dt, 5, snapshot="none")
    rec_ok = run_forward(prob, f)
    assert prob.status() == mwtm.MW_OK
    assert np.abs(rec_ok).max() > 0

    t0 = time.perf_counter()
    mwtm.selftest_wait_timeout(prob.workspace)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert 0.05 < waited < 30.0, waited   # bounded: the wait gave up by itself

    # while the timeout is unreported, stencil launches on this workspace stand down
    rec_skipped = run_forward(prob, f)
    assert prob.status() == mwtm.MW_ERR_TIMEOUT
    assert "timed out" in mwtm.last_error()
    assert not np.array_equal(rec_skipped, rec_ok)

    # reported and cleared: the same workspace gives the same records again
    rec_again = run_forward(prob, f)
    assert prob.status() == mwtm.MW_OK
    assert np.array_equal(rec_again, rec_ok)
