"""Public Python API over the C-ABI library (device tensors in, device tensors out).

`Problem` owns the device buffers of one setup (model coefficients, CPML
profiles, source / receiver indices, workspace) and runs the library's
forward, adjoint-gradient, shot-reduction and chain-rule entry points on the
current torch stream.  `misfit_gradient_host` is the end-to-end call on host
arrays: it copies the inputs in, runs the whole sweep and copies the results
out.  All arithmetic happens in the library's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import mwtm

F32 = torch.float32


def _dev(x, dtype=F32, device="cuda"):
    if isinstance(x, torch.Tensor):
        return x.to(device=device, dtype=dtype).contiguous()
    return torch.as_tensor(np.ascontiguousarray(x), dtype=dtype, device=device)


class Problem:
    """One 2-D TM setup: grid, stencil order, time step, shots, storage mode.

    src_idx [S, n_src] / rec_idx [S, n_rec] are flat cell indices y*nx + x
    (-1 = inactive).  snapshot: "none" | "fp32" | "bf16" | "fp8" | "ckpt" |
    "ckpt_ey" (checkpoints whose replay keeps E alone; the Cb gradient by
    summation by parts).
    snapshot_host: keep the fp32 / bf16 / fp8 snapshots in page-locked host
    memory (staged through a 3-step device ring) instead of the workspace.
    ckpt_tail: checkpoint modes, the forward stores the snapshots of the last
    ckpt_tail steps itself (HBM for replay work).
    """

    def __init__(self, ny, nx, order, dy, dx, dt, nt, n_pml, src_idx, rec_idx, *, vmax,
                 snapshot="fp32", ckpt_every=64, batched=False, cq_scalar=True,
                 grad_mask_pml=False, allow_unstable=False, check_finite=False, device="cuda",
                 snapshot_host=False, ckpt_tail=0):
        src_idx = np.asarray(src_idx, dtype=np.int64)
        rec_idx = np.asarray(rec_idx, dtype=np.int64)
        self.S = src_idx.shape[0]
        self.device = device
        self.p = mwtm.make_params(
            ny=ny, nx=nx, order=order, n_shots=self.S, n_src=src_idx.shape[1], n_rec=rec_idx.shape[1],
            nt=nt, dt=dt, dy=dy, dx=dx, n_pml=n_pml, model_batched=int(batched),
            cq_is_scalar=int(cq_scalar), snap_mode=mwtm.SNAP_MODES[snapshot], ckpt_every=ckpt_every,
            grad_mask_pml=int(grad_mask_pml), vmax=vmax, allow_unstable=int(allow_unstable),
            check_finite=int(check_finite), snap_host=int(bool(snapshot_host)),
            ckpt_tail=int(ckpt_tail))
        mwtm.check(mwtm.validate(self.p))
        self.host_snapshots = None
        if snapshot_host:
            n = mwtm.snap_host_bytes(self.p)
            self.host_snapshots = torch.empty(max(n, 1), dtype=torch.uint8, pin_memory=True)
            self.p.snap_host_ptr = self.host_snapshots.data_ptr()
        self.src_idx = _dev(src_idx if src_idx.size else np.zeros((self.S, 1), np.int64),
                            torch.int64, device)
        self.rec_idx = _dev(rec_idx if rec_idx.size else np.zeros((self.S, 1), np.int64),
                            torch.int64, device)
        self.workspace = torch.empty(mwtm.workspace_bytes(self.p) // 4 + 64, dtype=F32, device=device)
        mwtm.workspace_init(self.workspace)
        self.cpml = torch.empty(6 * (ny + nx), dtype=F32, device=device)
        self.ca = self.cb = self.cq = None
        self.state = None

    # ---- model -------------------------------------------------------------
    @property
    def model_shape(self):
        p = self.p
        return (self.S, p.ny, p.nx) if p.model_batched else (p.ny, p.nx)

    def _model_buffers(self):
        """Ca, Cb, Cq buffers, allocated once: later model updates write into
        them, so a captured SweepGraph sees the new model."""
        d = self.device
        cq_shape = (1,) if self.p.cq_is_scalar else self.model_shape
        for name, shape in (("ca", self.model_shape), ("cb", self.model_shape), ("cq", cq_shape)):
            t = getattr(self, name)
            if t is None or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
                setattr(self, name, torch.empty(shape, dtype=F32, device=d))

    def set_model_eps_sigma(self, eps_r, sigma=None, mu_r=None, f0=0.0, R=1e-3):
        """Ca, Cb, Cq from eps_r, sigma, mu_r (library kernel) and CPML profiles,
        written into the problem's model buffers."""
        d = self.device
        eps_r = _dev(eps_r, device=d).reshape(self.model_shape)
        sigma = None if sigma is None else _dev(sigma, device=d).reshape(self.model_shape)
        mu_r = None if mu_r is None else _dev(mu_r, device=d).reshape(self.model_shape)
        self._model_buffers()
        mwtm.model_from_eps_sigma(self.p, eps_r, sigma, mu_r, self.ca, self.cb, self.cq)
        mwtm.cpml_profiles(self.p, f0, R, self.cpml)
        return self

    def set_coefficients(self, ca, cb, cq, cpml):
        """Copy Ca, Cb, Cq and the 12 CPML profiles into the model buffers."""
        d = self.device
        self._model_buffers()
        self.ca.copy_(_dev(ca, device=d).reshape(self.model_shape))
        self.cb.copy_(_dev(cb, device=d).reshape(self.model_shape))
        self.cq.copy_(_dev(cq, device=d).reshape(self.cq.shape))
        self.cpml.copy_(_dev(cpml, device=d).reshape(-1))
        return self

    # ---- sweeps ------------------------------------------------------------
    def new_state(self):
        return torch.zeros(mwtm.state_floats(self.p), dtype=F32, device=self.device)

    def forward(self, f, state=None, rec=None):
        """Run nt steps; returns records [nt, S, n_rec].  `state` (flat) is in/out."""
        p = self.p
        f = _dev(f, device=self.device) if p.n_src > 0 else None
        if rec is None:
            rec = torch.empty((p.nt, self.S, max(p.n_rec, 1)), dtype=F32, device=self.device)
        mwtm.tm_forward(p, self.ca, self.cb, self.cq, self.cpml, f, self.src_idx, self.rec_idx, state,
                        rec if p.n_rec > 0 else None, self.workspace)
        self._f = f
        return rec[:, :, :p.n_rec]

    def adjoint(self, res, grad_f=False, gca=None, gcb=None, adj_state=None):
        """Adjoint sweep; returns (grad_ca_shot, grad_cb_shot, grad_f or None)."""
        p = self.p
        shp = (self.S, p.ny, p.nx)
        gca = torch.zeros(shp, dtype=F32, device=self.device) if gca is None else gca
        gcb = torch.zeros(shp, dtype=F32, device=self.device) if gcb is None else gcb
        gf = torch.zeros((p.nt, self.S, p.n_src), dtype=F32, device=self.device) if (
            grad_f and p.n_src > 0) else None
        res = _dev(res, device=self.device) if p.n_rec > 0 else None
        mwtm.tm_adjoint_grad(p, self.ca, self.cb, self.cq, self.cpml, getattr(self, "_f", None),
                             self.src_idx, self.rec_idx, res, gca, gcb, gf, adj_state, self.workspace)
        return gca, gcb, gf

    def born(self, dca, dcb, rec=None):
        """Born (linearised) forward about the last forward's background:
        records [nt, S, n_rec] of the perturbation (dca, dcb) of (Ca, Cb)."""
        p = self.p
        d = self.device
        dca = _dev(dca, device=d).reshape(self.model_shape)
        dcb = _dev(dcb, device=d).reshape(self.model_shape)
        rec = torch.zeros((p.nt, self.S, max(p.n_rec, 1)), dtype=F32, device=d) if rec is None else rec
        mwtm.tm_born(p, self.ca, self.cb, self.cq, self.cpml, dca, dcb, getattr(self, "_f", None),
                     self.src_idx, self.rec_idx, rec, self.workspace)
        return rec

    def combine(self, g_shot, out=None, accumulate=False):
        p = self.p
        out = torch.empty((p.ny, p.nx), dtype=F32, device=self.device) if out is None else out
        mwtm.combine_grad(p, g_shot, out, accumulate)
        return out

    def eps_sigma_gradient(self, gca, gcb):
        """Chain rule to (eps_r, sigma), cell by cell: gca / gcb shaped like the
        model (the shot sum for a shared model, per-shot gradients for a
        batched one)."""
        if gca.numel() != self.ca.numel() or gcb.numel() != self.ca.numel():
            raise ValueError(f"gradients of {gca.numel()} cells for a model of {self.ca.numel()}")
        n = gca.numel()
        ge = torch.empty_like(gca)
        gs = torch.empty_like(gca)
        mwtm.grad_eps_sigma(n, self.p.dt, self.ca, self.cb, gca, gcb, ge, gs)
        return ge, gs

    def residual(self, d, d_obs, res=None, J=None):
        res = torch.empty_like(d) if res is None else res
        J = torch.zeros(1, dtype=torch.float64, device=self.device) if J is None else J
        mwtm.residual(d.numel(), d, d_obs, res, J)
        return res, J

    def status(self):
        return mwtm.sync_status(self.workspace)

    def misfit_gradient(self, f, d_obs):
        """Forward, residual, adjoint, shot sum: (J [1] f64, rec, grad_Ca, grad_Cb)."""
        rec = self.forward(f)
        res, J = self.residual(rec.contiguous(), d_obs)
        gca_s, gcb_s, _ = self.adjoint(res)
        if self.p.model_batched:
            return J, rec, gca_s, gcb_s
        return J, rec, self.combine(gca_s), self.combine(gcb_s)


class SweepGraph:
    """One misfit-gradient sweep of `prob` (forward, residual, adjoint, shot
    sums) captured once as a CUDA graph and replayed.  Every launch of the
    sweep is recorded (programmatic dependent launches keep their overlap as
    graph edges), so a replay costs one host call: small, launch-bound
    problems lose the host cost of their ~3 nt launches per pass.

    The sweep reads `self.f` and `self.d_obs` and writes `self.J`, `self.rec`,
    `self.gca`, `self.gcb` (per-shot gradients for a batched model): copy new
    inputs into the former before `replay()`.  The model and the problem's
    workspace are those of `prob` at capture time; the pinned-host snapshot
    store (a second stream of host copies) is not captured."""

    def __init__(self, prob: Problem, f, d_obs):
        p = prob.p
        if p.snap_host:
            raise ValueError("SweepGraph: the pinned-host snapshot store is not captured")
        if p.snap_mode == mwtm.SNAP_NONE:
            raise ValueError("SweepGraph: snap_mode 'none' has no adjoint")
        dev = prob.device
        S, shp = prob.S, (prob.S, p.ny, p.nx)
        self.prob = prob
        self.f = torch.as_tensor(f, dtype=F32, device=dev).clone().contiguous()
        self.d_obs = torch.as_tensor(d_obs, dtype=F32, device=dev).clone().contiguous()
        self._rec = torch.zeros((p.nt, S, max(p.n_rec, 1)), dtype=F32, device=dev)
        self.rec = self._rec[:, :, :p.n_rec]
        self.res = torch.zeros_like(self.rec)
        self.J = torch.zeros(1, dtype=torch.float64, device=dev)
        self.gca_s = torch.zeros(shp, dtype=F32, device=dev)
        self.gcb_s = torch.zeros(shp, dtype=F32, device=dev)
        if p.model_batched:
            self.gca, self.gcb = self.gca_s, self.gcb_s
        else:
            self.gca = torch.zeros((p.ny, p.nx), dtype=F32, device=dev)
            self.gcb = torch.zeros((p.ny, p.nx), dtype=F32, device=dev)
        # the buffers the capture bakes in (kept alive; replay() checks that
        # the problem still uses them)
        self._baked = (prob.ca, prob.cb, prob.cq, prob.cpml, prob.workspace, prob.src_idx,
                       prob.rec_idx)
        # one eager sweep first: kernel attributes are set and the work
        # counters settle outside the capture
        self._body()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        n0 = mwtm.launch_count()
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            self._body()
        self.launches = mwtm.launch_count() - n0  # library kernels per replay

    def _body(self):
        prob = self.prob
        prob.forward(self.f, rec=self._rec)
        if prob.p.n_rec > 0:
            prob.residual(self.rec, self.d_obs, res=self.res, J=self.J)
        self.gca_s.zero_()
        self.gcb_s.zero_()
        prob.adjoint(self.res, gca=self.gca_s, gcb=self.gcb_s)
        if not prob.p.model_batched:
            prob.combine(self.gca_s, out=self.gca)
            prob.combine(self.gcb_s, out=self.gcb)

    def replay(self):
        """Run the captured sweep on the current stream's device; returns
        (J, rec, grad_Ca, grad_Cb) (the buffers above).  Model updates must go
        through the problem's setters, which write in place."""
        prob = self.prob
        now = (prob.ca, prob.cb, prob.cq, prob.cpml, prob.workspace, prob.src_idx, prob.rec_idx)
        if any(a is not b for a, b in zip(now, self._baked)):
            raise RuntimeError("SweepGraph: a buffer of the problem was replaced after capture "
                               "(update the model through set_model_eps_sigma / set_coefficients)")
        self.graph.replay()
        return self.J, self.rec, self.gca, self.gcb


def unpack_state(p, flat):
    """Split a flat state into full [S, ny, nx] arrays (memories expanded; numpy fp64)."""
    a = flat.detach().cpu().numpy().astype(np.float64) if isinstance(flat, torch.Tensor) else flat
    S, ny, nx, n_pml = p.n_shots, p.ny, p.nx, p.n_pml
    Wx = ((n_pml + 1 + 3) // 4) * 4 if n_pml > 0 else 0
    Wz = n_pml + 1 if n_pml > 0 else 0
    SN = S * ny * nx
    out = {"ey": a[:SN].reshape(S, ny, nx), "hx": a[SN:2 * SN].reshape(S, ny, nx),
           "hz": a[2 * SN:3 * SN].reshape(S, ny, nx)}
    off = 3 * SN
    xb = S * ny * 2 * Wx
    zb = S * 2 * Wz * nx
    names_x = ("m_ey_x", "m_hz_x")
    names_z = ("m_ey_z", "m_hx_z")
    for nm in names_x:
        full = np.zeros((S, ny, nx))
        if Wx:
            band = a[off:off + xb].reshape(S, ny, 2 * Wx)
            full[:, :, :Wx] = band[:, :, :Wx]
            full[:, :, nx - Wx:] = band[:, :, Wx:]
        out[nm] = full
        off += xb
    for nm in names_z:
        full = np.zeros((S, ny, nx))
        if Wz:
            band = a[off:off + zb].reshape(S, 2 * Wz, nx)
            full[:, :Wz, :] = band[:, :Wz, :]
            full[:, ny - Wz:, :] = band[:, Wz:, :]
        out[nm] = full
        off += zb
    return out


def misfit_gradient_host(prob: Problem, f_host, d_obs_host, eps_r_host=None, sigma_host=None,
                         f0=0.0, pinned_out=None):
    """End-to-end on host arrays: H2D of the inputs, the whole sweep, D2H of
    J, records and the combined gradients.  Returns numpy arrays."""
    dev = prob.device
    if eps_r_host is not None:
        prob.set_model_eps_sigma(torch.as_tensor(eps_r_host).to(dev, non_blocking=True),
                                 None if sigma_host is None else
                                 torch.as_tensor(sigma_host).to(dev, non_blocking=True), f0=f0)
    f = torch.as_tensor(f_host).to(dev, non_blocking=True)
    d_obs = torch.as_tensor(d_obs_host).to(dev, non_blocking=True)
    J, rec, gca, gcb = prob.misfit_gradient(f, d_obs)
    if pinned_out is None:
        return J.cpu().numpy(), rec.cpu().numpy(), gca.cpu().numpy(), gcb.cpu().numpy()
    outs = []
    for t, h in zip((J, rec, gca, gcb), pinned_out):
        h.copy_(t.reshape(h.shape), non_blocking=True)
        outs.append(h)
    torch.cuda.current_stream().synchronize()
    return outs
