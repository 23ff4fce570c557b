"""One forward + adjoint sweep of a reduced 2128^2 order-4 case, for profilers.

    python -m adjoint_state_gradients_b200.profile_case [--shots 4] [--nt 8] [--mode fp32] [--born]

Same grid, stencil, CPML band and launch configuration as the benchmark
workload, with fewer shots and steps so that an ncu capture of a single
kernel launch holds only a few GB on the device (4 shots: 217 MB per state
buffer, larger than L2).
"""
from __future__ import annotations

import argparse
import math

import numpy as np
import torch

from . import api, mwtm, synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--shots", type=int, default=4)
    ap.add_argument("--nt", type=int, default=8)
    ap.add_argument("--mode", default="fp32", choices=["fp32", "bf16", "fp8", "ckpt", "ckpt_ey", "none"])
    ap.add_argument("--born", action="store_true",
                    help="after the forward, the Born forward about it (instead of the adjoint)")
    args = ap.parse_args()
    inp = synth.make_inputs(args.workload, n_shots=args.shots)
    wl = inp.wl
    vmax = 299792458.0 / math.sqrt(inp.eps_min)
    dt = wl.cfl_fraction * mwtm.cfl_dt(wl.order, wl.h, wl.h, vmax)
    prob = api.Problem(wl.ny, wl.nx, wl.order, wl.h, wl.h, dt, args.nt, wl.n_pml, inp.src_idx,
                       inp.rec_idx, vmax=vmax, snapshot=args.mode, batched=wl.batched)
    prob.set_model_eps_sigma(inp.eps_r.astype(np.float32), inp.sigma.astype(np.float32), f0=wl.f0)
    f = torch.as_tensor(inp.wavelet(dt, args.nt).astype(np.float32)).cuda()
    rec = prob.forward(f)
    if args.born and args.mode != "none":
        g = torch.Generator(device="cuda").manual_seed(1)
        shape = prob.model_shape
        prob.born(1e-3 * torch.randn(shape, device="cuda", generator=g) * prob.ca,
                  1e-3 * torch.randn(shape, device="cuda", generator=g) * prob.cb)
    elif args.mode != "none":
        prob.adjoint(rec.contiguous())
    torch.cuda.synchronize()
    rc = prob.status()
    print(f"profile_case: workload {args.workload}, {args.shots} shots, nt {args.nt}, mode {args.mode}, "
          f"status {rc}, launches {mwtm.launch_count()}")
    if rc != mwtm.MW_OK:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
