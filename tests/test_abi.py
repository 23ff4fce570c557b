"""The C-ABI library loads without a GPU and exports every entry point that
include/mw_tm.h declares; host-only entry points behave as documented."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from adjoint_state_gradients_b200 import build, mwtm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mw_tm.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(mw_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_path_entry_points():
    names = declared_functions()
    for n in ("mw_tm_forward", "mw_tm_adjoint_grad", "mw_combine_grad", "mw_workspace_bytes",
              "mw_last_error", "mw_grad_eps_sigma", "mw_model_from_eps_sigma"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(build.build())
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_constants_match_the_header():
    """Status codes and snapshot modes: the binding's values are the
    header's, and every mode the header defines is reachable by name."""
    text = open(HEADER).read()
    defs = {k: int(v) for k, v in re.findall(r"#define\s+(MW_(?:ERR_[A-Z]+|OK|SNAP_[A-Z0-9_]+))\s+"
                                              r"\(?(-?\d+)\)?", text)}
    assert defs["MW_OK"] == mwtm.MW_OK
    errs = {k: v for k, v in defs.items() if k.startswith("MW_ERR_")}
    assert len(errs) >= 7
    for k, v in errs.items():
        assert getattr(mwtm, k) == v, k
    modes = {k[len("MW_SNAP_"):].lower(): v for k, v in defs.items() if k.startswith("MW_SNAP_")}
    assert modes == {"none": 0, "fp32": 1, "bf16": 2, "ckpt": 3, "fp8": 4, "ckpt_ey": 5}
    assert mwtm.SNAP_MODES == modes


def test_binding_scratch_size_matches_the_header():
    """The scratch-free forward's built-in scratch size: the binding's copy
    is the header's MW_NOALLOC_SCRATCH_BYTES."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+MW_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "MW_NOALLOC_SCRATCH_BYTES not found in the header"
    assert mwtm.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_binding_covers_every_declared_symbol():
    bound = {name for name, _, _ in mwtm.SIGNATURES}
    missing = [n for n in declared_functions() if n not in bound]
    assert not missing, missing


def test_host_only_entry_points():
    p = mwtm.make_params(ny=84, nx=84, order=2, n_shots=1, n_src=1, n_rec=32, nt=300, dt=4.7e-11,
                         dy=0.02, dx=0.02, n_pml=10, snap_mode=mwtm.SNAP_FP32, vmax=1.5e8)
    assert mwtm.validate(p) == mwtm.MW_OK
    # state: 3 fields + 2 x-band (Wx = 12) + 2 z-band (Wz = 11) memories
    assert mwtm.state_floats(p) == 3 * 84 * 84 + 2 * 84 * 24 + 2 * 22 * 84
    ws = mwtm.workspace_bytes(p)
    assert ws >= 2 * 300 * 84 * 84 * 4
    bad = mwtm.make_params(ny=84, nx=82, order=2, n_shots=1, nt=1, dt=1e-12, dy=0.02, dx=0.02,
                           vmax=1.5e8)
    assert mwtm.validate(bad) == mwtm.MW_ERR_ARG
    assert "multiple of 4" in mwtm.last_error()
    big_pml = mwtm.make_params(ny=600, nx=600, order=2, n_shots=1, nt=1, dt=1e-12, dy=0.02,
                               dx=0.02, n_pml=130, vmax=1.5e8)
    assert mwtm.validate(big_pml) == mwtm.MW_ERR_UNSUPPORTED
    assert mwtm.workspace_bytes(p) == ws


def test_checkpoint_modes_workspace_and_tail():
    """The E-alone checkpoint mode adds its Cb accumulator, record copy and
    end-term sums; a forward-stored tail adds its snapshot slots (pairs, or E
    alone plus the final E); ckpt_tail needs a checkpoint mode."""
    kw = dict(ny=84, nx=84, order=2, n_shots=2, n_src=1, n_rec=32, nt=300, dt=4.7e-11, dy=0.02,
              dx=0.02, n_pml=10, vmax=1.5e8, ckpt_every=64)
    step = 2 * 84 * 84 * 4
    pair = mwtm.workspace_bytes(mwtm.make_params(snap_mode=mwtm.SNAP_CKPT, **kw))
    ey = mwtm.workspace_bytes(mwtm.make_params(snap_mode=mwtm.SNAP_CKPT_EY, **kw))
    assert ey >= pair + step + 300 * 2 * 32 * 4
    for tail, slots_pair, slots_ey in ((10, 20, 11), (300, 600, 301), (1000, 600, 301)):
        pt = mwtm.workspace_bytes(mwtm.make_params(snap_mode=mwtm.SNAP_CKPT, ckpt_tail=tail, **kw))
        et = mwtm.workspace_bytes(mwtm.make_params(snap_mode=mwtm.SNAP_CKPT_EY, ckpt_tail=tail, **kw))
        assert slots_pair * step <= pt - pair < slots_pair * step + 256
        assert slots_ey * step <= et - ey < slots_ey * step + 256
    for mode, tail in ((mwtm.SNAP_FP32, 5), (mwtm.SNAP_CKPT, -1)):
        assert mwtm.validate(mwtm.make_params(snap_mode=mode, ckpt_tail=tail, **kw)) == mwtm.MW_ERR_ARG
        assert "ckpt_tail" in mwtm.last_error()


@pytest.mark.parametrize("order,s", [(2, 1.0), (4, 7 / 6), (6, 1.2416666666666667),
                                     (8, 1.2863095238095237)])
def test_cfl_dt_matches_oracle(order, s):
    import oracle
    for h, v in ((0.02, 1.5e8), (0.01, 2.9e8)):
        assert mwtm.cfl_dt(order, h, h, v) == pytest.approx(oracle.cfl_dt(order, h, h, v), rel=1e-15)
        assert mwtm.cfl_dt(order, h, h, v) == pytest.approx(1 / (v * s * (2 / h ** 2) ** 0.5), rel=1e-12)
