"""bench.py on the host: the algorithmic byte model per pass, the sample
sizing of the oracle baseline, and the reference arm's JSON line (the fp64
oracle timed on host cores), run as the driver runs it."""
from __future__ import annotations

import dataclasses
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from adjoint_state_gradients_b200 import synth  # noqa: E402


def test_byte_model_of_the_headline_sweep():
    """Checkpoints every 64 steps with the E-alone segment: the replay writes
    and the adjoint reads 4 B of snapshot per cell-update; with the pair
    segment 8 B.  Checkpoints add no bytes (written and read in place).  One
    step per forward launch (MW_NO_TWO_STEP=1 / one_pass)."""
    wl = synth.WORKLOADS[4]
    assert wl.snapshot == "ckpt_ey"
    b = bench.alg_bytes(wl, wl.n_shots, one_pass=True)
    band = 16.0 * (2 * 40 / 2128 + 2 * 40 / 2128)
    assert b["forward"] == pytest.approx(24 + 1 + band)
    assert b["replay"] == pytest.approx(24 + 1 + band + 4)
    assert b["adjoint"] == pytest.approx(24 + 1 + band + 4 + 16)
    assert sum(b.values()) == pytest.approx(102.61, abs=0.01)
    assert bench.pass_classes(wl) == {"forward": (0, 4, ()), "replay": (1, 5, ()),
                                      "adjoint": (2, None, ())}
    bp = bench.alg_bytes(dataclasses.replace(wl, snapshot="ckpt"), wl.n_shots, one_pass=True)
    assert bp["replay"] - b["replay"] == pytest.approx(4.0)
    assert bp["adjoint"] - b["adjoint"] == pytest.approx(4.0)
    assert sum(bp.values()) == pytest.approx(110.61, abs=0.01)
    # the forward-stored tail: those steps write E (4 B) and skip the replay
    assert wl.ckpt_tail == 768
    want = b["forward"] + 0.192 * 4 + 0.808 * b["replay"] + b["adjoint"]
    assert bench.sweep_bytes_per_cell(wl, wl.n_shots, one_pass=True) == pytest.approx(want)
    assert bench.sweep_bytes_per_cell(dataclasses.replace(wl, ckpt_tail=0), wl.n_shots,
                                      one_pass=True) == pytest.approx(102.61, abs=0.01)


def test_byte_model_of_two_step_forward_passes():
    """Two steps per forward launch: the state (24 B) and the band memories
    move once per two steps, Ca / Cb and the snapshots once per step; the
    adjoint is unchanged."""
    wl = synth.WORKLOADS[4]
    one, two = bench.alg_bytes(wl, 8, one_pass=True), bench.alg_bytes(wl, 8)
    band = 16.0 * (2 * 40 / 2128 + 2 * 40 / 2128)
    assert bench.two_step(wl) and not bench.two_step(synth.WORKLOADS[5])
    assert two["forward"] == pytest.approx(12 + 1 + band / 2)
    assert two["replay"] == pytest.approx(12 + 1 + band / 2 + 4)
    assert two["adjoint"] == one["adjoint"]
    assert bench.alg_bytes(synth.WORKLOADS[5], 256) == bench.alg_bytes(synth.WORKLOADS[5], 256,
                                                                       one_pass=True)


def test_byte_model_of_the_other_storage_modes():
    w3, w5 = synth.WORKLOADS[3], synth.WORKLOADS[5]
    b3, b5 = bench.alg_bytes(w3, w3.n_shots), bench.alg_bytes(w5, w5.n_shots)
    assert b3["adjoint"] - b3["forward"] == pytest.approx(16.0)   # gradient read + write
    assert set(b5) == {"forward"}
    assert b5["forward"] > 24 + 8                                  # per-shot model: 8 B per cell
    assert bench.pass_classes(w5) == {"forward": (0, 4, (6, 9))}


def test_per_step_time_of_each_launch_kind():
    """One-step launches count one step, two-step launches two, whole-sweep
    launches nt."""
    counts = [10, 0, 0, 0, 5, 0, 0, 0, 0, 0, 0, 0]
    ms = [1.0, 0, 0, 0, 2.0, 0, 0, 0, 0, 0, 0, 0]
    assert bench.per_step_ms(counts, ms, (0, 4, (6, 9)), 300) == pytest.approx(3.0 / 20)
    counts[8], ms[8] = 2, 6.0
    assert bench.per_step_ms(counts, ms, (2, None, (8, 11)), 300) == pytest.approx(6.0 / 600)
    assert bench.N_CLASSES == 12


def test_steps_per_launch():
    counts = [0] * 12
    assert bench.steps_per_launch(counts, (2, None, (8, 11)), 300) == 1.0  # nothing ran
    counts[0], counts[4] = 2, 98   # a pass of two one-step and 98 two-step launches
    assert bench.steps_per_launch(counts, (0, 4, ()), 4000) == pytest.approx(198 / 100)
    counts[8] = 3                  # three whole-sweep adjoint launches
    assert bench.steps_per_launch(counts, (2, None, (8, 11)), 300) == 300.0


def test_oracle_sample_is_bounded():
    for n in range(1, 6):
        wl = synth.WORKLOADS[n]
        k = bench.sample_steps(wl, 1.2e9)
        assert 16 <= k <= wl.nt
        assert k * wl.ny * wl.nx <= max(1.2e9, 16 * wl.ny * wl.nx)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "1", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == synth.WORKLOADS[1].name


def test_tail_fits_free_memory():
    """The forward-stored tail shrinks, by whole segments, to what the free
    device memory holds beside the reserve, and vanishes when nothing fits."""
    from adjoint_state_gradients_b200 import mwtm
    wl = synth.WORKLOADS[4]
    kw = dict(ny=wl.ny, nx=wl.nx, order=4, n_shots=8, n_src=1, n_rec=512, nt=4000, dt=4.2e-11,
              dy=0.02, dx=0.02, n_pml=40, snap_mode=mwtm.SNAP_CKPT_EY, ckpt_every=64, vmax=1.7e8)
    w = {k: mwtm.workspace_bytes(mwtm.make_params(ckpt_tail=k, **kw)) for k in (1, 2, 640)}
    step = w[2] - w[1]
    base = w[1] - step
    assert base + 640 * step == pytest.approx(w[640], abs=4096)
    gb = 1e9
    assert bench.fit_tail(640, base, step, 192 * gb) == 640            # a whole B200
    assert bench.fit_tail(768, base, step, 190 * gb) == 768
    k = bench.fit_tail(640, base, step, 120 * gb)                      # less free memory
    assert k % 64 == 0 and 0 < k < 640
    assert base + k * step <= 120 * gb - bench.TAIL_RESERVE
    assert base + (k + 64) * step > 120 * gb - bench.TAIL_RESERVE
    assert bench.fit_tail(640, base, step, 40 * gb) == 0                # not even the checkpoints
    assert bench.fit_tail(0, base, step, 192 * gb) == 0
