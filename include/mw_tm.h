/*
 * mw_tm.h -- C ABI of the B200 (sm_100a) 2-D TM Maxwell FDTD library:
 * forward time stepping, exact discrete adjoint and adjoint-state model
 * gradients, batched over shots.
 *
 * The method is the one stated in the header comment of the page
 * "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu" ("EXACT DISCRETE Adjoint State
 * Method for Maxwell TM equations"):
 *   forward   H^{n+1/2} = H^{n-1/2} -/+ Cq psi(D^h E^n)          (Hx: -, Hz: +)
 *             E^{n+1}   = Ca E^n + Cb (psi(D_x Hz) - psi(D_z Hx))
 *   adjoint   the same step transposed, run backwards in time
 *   gradients dJ/dCa = sum_n E^n lambda^{n+1},  dJ/dCb = sum_n curlH^n lambda^{n+1}
 * psi is the CPML operator of the page's H / E kernels: memory m <- b m + a d,
 * output d / k + m.
 *
 * Conventions used by every entry point
 * -------------------------------------
 *  - Grid: ny rows (y = depth z) by nx columns (x), row-major; cell index
 *    j = y * nx + x.  Ey at (y, x), Hx at (y + 1/2, x), Hz at (y, x + 1/2).
 *    Every array cell of every field is updated; fields are zero outside the
 *    array.  nx must be a multiple of 4 (rows are read as float4) and n_pml
 *    at most 123 (a CPML band row is one TMA box of at most 256 floats).
 *  - Per-shot arrays are [S][ny][nx] float32, time series are time-major
 *    [nt][S][n] float32 (the page's source / receiver kernels).
 *  - Source / receiver positions are flat per-shot cell indices int64
 *    [S][n_src] / [S][n_rec]; -1 marks an inactive entry.  Duplicate source
 *    cells add up (applied in index order); inactive receivers record 0.
 *  - Pointers named *_dev are device memory; *_host are host memory.  The
 *    caller owns every buffer.  Nothing allocates device memory per call.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Compute calls are asynchronous and stream-ordered; they
 *    return after enqueueing.  Errors found on the host return at once;
 *    device-side status (an out-of-range index, a non-finite field with
 *    check_finite, a stage wait that ran out) is recorded in the workspace
 *    and reported by mw_sync_status.
 *  - Return codes: MW_OK (0) or a negative MW_ERR_*; mw_last_error() gives a
 *    thread-local message.  No entry point aborts the process.
 *
 * State layout (one buffer, float32, mw_state_floats() floats), used for the
 * forward state (Ey, Hx, Hz, CPML memories) and the adjoint state (their
 * adjoints):
 *    [0] Ey    [S][ny][nx]
 *    [1] Hx    [S][ny][nx]
 *    [2] Hz    [S][ny][nx]
 *    [3] m_ey_x  x-band memory at Hz nodes     [S][ny][2*Wx]
 *    [4] m_hz_x  x-band memory at Ey nodes     [S][ny][2*Wx]
 *    [5] m_ey_z  z-band memory at Hx nodes     [S][2*Wz][nx]
 *    [6] m_hx_z  z-band memory at Ey nodes     [S][2*Wz][nx]
 *  Wx = round_up(n_pml + 1, 4), Wz = n_pml + 1 (0 when n_pml == 0).  The
 *  x band holds columns [0, Wx) then [nx - Wx, nx); the z band rows
 *  [0, Wz) then [ny - Wz, ny).  CPML coefficients a and b must vanish, and
 *  k must equal 1, outside those bands (the memories exist only there).
 */
#ifndef MW_TM_H
#define MW_TM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define MW_OK 0
#define MW_ERR_ARG (-1)         /* invalid argument, shape or index        */
#define MW_ERR_CFL (-2)         /* dt above the stability bound             */
#define MW_ERR_WORKSPACE (-3)   /* workspace missing or too small           */
#define MW_ERR_CUDA (-4)        /* a CUDA runtime call failed               */
#define MW_ERR_NONFINITE (-5)   /* NaN / Inf found in a field (device flag) */
#define MW_ERR_TIMEOUT (-6)     /* a kernel gave up waiting for its own copies
                                   (device flag; results of that call invalid) */
#define MW_ERR_UNSUPPORTED (-7) /* valid request the library does not serve */

/* forward snapshot storage for the gradient */
#define MW_SNAP_NONE 0 /* records only; mw_tm_adjoint_grad unavailable       */
#define MW_SNAP_FP32 1 /* Ey^n and curl^n of every step, float32, on the GPU */
#define MW_SNAP_BF16 2 /* same, rounded to bfloat16 (round to nearest even)  */
#define MW_SNAP_CKPT 3 /* full state every ckpt_every steps; the adjoint
                          replays each segment into an fp32 segment buffer  */
#define MW_SNAP_FP8 4  /* Ey^n and curl^n rounded to FP8 E4M3 (nearest even,
                          saturating to +-448, no scaling), as the
                          maxwell.cu page's forward_kernel_e_with_storage_fp8
                          stores them                                        */
#define MW_SNAP_CKPT_EY 5 /* checkpoints as MW_SNAP_CKPT, but the replayed
                          segment keeps Ey^n alone and the adjoint forms the
                          Cb gradient by summation by parts (below), which
                          halves the segment's snapshot traffic; the forward
                          keeps a copy of the records in the workspace (it
                          then needs rec_idx when n_rec > 0), and Cb must be
                          nonzero everywhere                                 */

typedef struct mw_params {
  int32_t ny, nx;        /* array size incl. the CPML band                 */
  int32_t order;         /* stencil order: 2, 4, 6 or 8                      */
  int32_t n_shots;       /* S                                                */
  int32_t n_src, n_rec;  /* sources / receivers per shot (may be 0)          */
  int32_t nt;            /* time steps of this call                          */
  double dt, dy, dx;     /* s, m, m                                          */
  int32_t n_pml;         /* CPML band width in cells, all four sides         */
  int32_t model_batched; /* 0: Ca, Cb (and Cq array) [ny][nx] shared;
                            1: [S][ny][nx] per shot                          */
  int32_t cq_is_scalar;  /* 1: cq points to one float (mu_r constant)        */
  int32_t snap_mode;     /* MW_SNAP_*                                        */
  int32_t ckpt_every;    /* C for MW_SNAP_CKPT                               */
  int32_t grad_mask_pml; /* 1: accumulate gradients only at cells outside the
                            CPML band (the page's masking); 0: everywhere    */
  double vmax;           /* fastest wave speed in the model, m/s (CFL check) */
  int32_t allow_unstable;/* 1: skip the CFL check                            */
  int32_t check_finite;  /* 1: flag NaN / Inf in the final state             */
  int32_t snap_host;     /* 1 (with MW_SNAP_FP32 / BF16 / FP8): keep the
                            snapshots in pinned host memory (snap_host_ptr,
                            mw_snap_host_bytes(p) bytes, caller-owned) and
                            stage them through a 3-step ring in the
                            workspace, copied on a stream of the library's
                            own (the page's CPU snapshot storage with its
                            ring of device buffers and prefetch)           */
  void *snap_host_ptr;   /* page-locked host buffer for snap_host = 1        */
  int32_t ckpt_tail;     /* checkpoint modes: the forward itself stores the
                            snapshots of the last min(ckpt_tail, nt) steps (E
                            and curl, or E alone for MW_SNAP_CKPT_EY) in the
                            workspace, and the adjoint replays only the steps
                            before them; it trades HBM for replay work (each
                            tail step takes ny*nx*S*4 bytes per stored field).
                            0: replay every step                            */
} mw_params;

/* Fill *p with defaults (zeros, cq_is_scalar = 1, snap_mode NONE). */
void mw_params_init(mw_params *p);

/* Bytes of pinned host memory the snapshots of p take when p->snap_host = 1
 * (both fields of every step; rows padded to 16 bytes).  0 otherwise or on
 * invalid params. */
size_t mw_snap_host_bytes(const mw_params *p);

/* Floats in one state buffer (layout above). 0 on invalid params. */
size_t mw_state_floats(const mw_params *p);

/* Bytes of workspace mw_tm_forward / mw_tm_adjoint_grad need for p (ping-pong
 * state buffers, adjoint state, snapshots or checkpoints + segment buffer).
 * The same workspace carries the forward's snapshots to the adjoint.  0 on
 * invalid params. */
size_t mw_workspace_bytes(const mw_params *p);

/* Largest stable dt for stencil `order` and wave speed vmax:
 * 1 / (vmax * sum_k |c_k| * sqrt(1/dx^2 + 1/dy^2)).  Negative on bad input. */
double mw_cfl_dt(int32_t order, double dy, double dx, double vmax);

/* Check p (sizes, order, band fits, CFL unless allow_unstable).  Host only. */
int mw_validate(const mw_params *p);

/* Model coefficients from relative permittivity, conductivity (S/m) and
 * relative permeability, float32 device arrays of the model's shape
 * ([ny][nx] or [S][ny][nx] when model_batched):
 *   Ca = (1 - s dt / (2 eps)) / (1 + s dt / (2 eps)),  Cb = dt / (eps + s dt / 2),
 *   Cq = dt / (mu0 mu_r),  eps = eps0 eps_r
 * (the forms whose derivatives the page's epsilon / sigma conversion kernel
 * uses).  Computed in fp64, stored as float32.  sigma_dev may be NULL (0);
 * mu_r_dev may be NULL (1): then cq_dev receives one float when
 * p->cq_is_scalar, else a full array. */
int mw_model_from_eps_sigma(const mw_params *p, const float *eps_r_dev,
                            const float *sigma_dev, const float *mu_r_dev,
                            float *ca_dev, float *cb_dev, float *cq_dev,
                            void *stream);

/* CPML profiles, float32 device array of 6*(ny + nx) floats:
 *   [ay, ayh, by, byh, ky, kyh] (ny each) then [ax, axh, bx, bxh, kx, kxh]
 *   (nx each); "h" = half node (i + 1/2).  Quadratic damping
 *   d = d_max s^2, d_max = -3 vmax ln(R) / (2 n_pml h), kappa = 1,
 *   alpha = pi f0 (1 - s), b = exp(-(d + alpha) dt), a = d (b - 1) / (d + alpha),
 *   s = distance into the band / band width.  Any profile obeying the band
 *   rule in the layout note may be passed instead. */
int mw_cpml_profiles(const mw_params *p, double f0, double R, float *cpml_dev,
                     void *stream);

/* Prepare a workspace for first use: zero its status words (the first 256
 * bytes).  Call once after allocating it; mw_sync_status clears them again
 * after reporting. */
int mw_workspace_init(void *workspace_dev, size_t workspace_bytes, void *stream);

/* Forward: nt steps of H update, E update (+ snapshot / checkpoint store),
 * source injection f[t], receiver sampling rec[t] = Ey after injection
 * (order of the page's forward host loop).
 *   ca, cb     model [ny][nx] or [S][ny][nx]
 *   cq         one float or an array shaped like ca (p->cq_is_scalar)
 *   cpml       6*(ny+nx) profile floats (mw_cpml_profiles layout)
 *   f          [nt][S][n_src] source amplitudes added to Ey (may be NULL if n_src == 0)
 *   state      in/out state buffer (layout above), or NULL to start from rest
 *              (the final state then stays in the workspace)
 *   rec        [nt][S][n_rec] out (may be NULL)
 *   workspace  mw_workspace_bytes(p) bytes of device memory, 256-byte
 *              aligned, prepared once with mw_workspace_init
 * Sources / receivers of step t use time index t of this call. */
int mw_tm_forward(const mw_params *p, const float *ca_dev, const float *cb_dev,
                  const float *cq_dev, const float *cpml_dev, const float *f_dev,
                  const int64_t *src_idx_dev, const int64_t *rec_idx_dev,
                  float *state_dev, float *rec_dev, void *workspace_dev,
                  size_t workspace_bytes, void *stream);

/* Forward sweep that allocates nothing and needs no workspace (this entry
 * point has no counterpart on the reference pages; it exists for callers that
 * cannot allocate device memory, for instance a library embedded in an
 * application whose device memory all belongs to another allocator, or a
 * service that may allocate only at start-up).  Same arguments and results
 * as mw_tm_forward with snap_mode MW_SNAP_NONE (records only), except:
 *   - `state` is required (in/out; zero it for a run from rest);
 *   - the scratch it needs (status words, duplicate chains, CPML band table,
 *     the second ping-pong state buffer) lives in one array of
 *     MW_NOALLOC_SCRATCH_BYTES bytes that the library defines in device
 *     memory; every GPU that loads the library holds that array until the
 *     process exits.  A problem needing more than that is rejected with
 *     MW_ERR_WORKSPACE before any work is queued;
 *   - the call is synchronous: it waits for its work on `stream` to finish
 *     (cudaStreamSynchronize) and reads back the device status of this call
 *     (MW_ERR_ARG for an out-of-range index, MW_ERR_TIMEOUT,
 *     MW_ERR_NONFINITE with check_finite), so no mw_sync_status call is
 *     needed; the status words are cleared at the start of every call, so a
 *     failed call leaves nothing behind for the next one;
 *   - every call looks up the array's device address (cudaGetSymbolAddress)
 *     with the calling thread's current device, so the address stays valid
 *     after a context teardown such as cudaDeviceReset;
 *   - every call shares the one array: calls that overlap on the GPU (other
 *     threads, other streams) race and corrupt each other's results. */
#define MW_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int mw_tm_forward_noalloc(const mw_params *p, const float *ca_dev,
                          const float *cb_dev, const float *cq_dev,
                          const float *cpml_dev, const float *f_dev,
                          const int64_t *src_idx_dev,
                          const int64_t *rec_idx_dev, float *state_dev,
                          float *rec_dev, void *stream);

/* Adjoint sweep t = nt-1 .. 0 and per-shot gradients, after mw_tm_forward
 * with the same p, model, sources and workspace (snap_mode != NONE).  Per
 * step: lambda_E[rec] += res[t]; grad_f[t] = lambda_E[src];
 * grad_ca_shot += Ey^t lambda_E; grad_cb_shot += curl^t lambda_E; then the
 * transposed E and H updates, CPML band included.
 *   res            [nt][S][n_rec] adjoint source (d - d_obs for 1/2||d - d_obs||^2)
 *   grad_*_shot    [S][ny][nx] accumulated (+=): zero them for a fresh gradient
 *   grad_f         [nt][S][n_src] out, or NULL
 *   adj_state      in/out adjoint state, or NULL (start from zero)
 * In MW_SNAP_CKPT mode the forward is replayed segment by segment from the
 * checkpoints, which needs f and src_idx again. */
/* MW_SNAP_CKPT_EY: the same gradient (the maxwell.cu page's header comment:
 * grad_cb = sum_t curl^t lambda_E^{t+1}), regrouped.  With
 * E^{t+1} = Ca E^t + Cb curl^t + s^t (s the source injection; the page's
 * forward equations) and the adjoint's E update lam~^t = Ca lam^{t+1} + G^t
 * (lam^{t+1} = lam~^{t+1} + the residual injected at step t), the sum
 * Cb * grad_cb = sum_t curl^t lam^{t+1} * Cb regroups, exactly, into
 *     sum_{t>=1} G^t E^t  -  Ca lam^1 E^0  +  lam~^{nt} E^{nt}
 *   + sum_t res[t] rec[t]  (at the receiver cells)
 *   - sum_t f[t] lam^{t+1} (at the source cells),
 * which needs only E^t from the replay.  The kernel accumulates the first two
 * terms row by row, at each row's E update, into a workspace array that
 * starts at the third (zero unless adj_state is given; E^{nt} comes from the
 * last replayed segment or the forward-stored tail), the injection launches
 * gather the last two, and the end of the call adds them and divides by
 * Cb.  grad_ca_shot, grad_f and the adjoint state are
 * bitwise those of MW_SNAP_CKPT; grad_cb_shot agrees to rounding. */
int mw_tm_adjoint_grad(const mw_params *p, const float *ca_dev,
                       const float *cb_dev, const float *cq_dev,
                       const float *cpml_dev, const float *f_dev,
                       const int64_t *src_idx_dev, const int64_t *rec_idx_dev,
                       const float *res_dev, float *grad_ca_shot_dev,
                       float *grad_cb_shot_dev, float *grad_f_dev,
                       float *adj_state_dev, void *workspace_dev,
                       size_t workspace_bytes, void *stream);

/* Born (linearised) forward: the derivative of the records with respect to
 * (Ca, Cb) in the direction (dCa, dCb), the transpose of mw_tm_adjoint_grad's
 * gradient map (LSRTM-style modelling / migration pairs; the PR page
 * "DeepWave-KAUST/sweep #125", commits 1-2, describes such Born / adjoint
 * pairs, checked by a dot test, for its acoustic and qP operators).  A perturbation state starts at zero and takes the
 * forward step without sources, plus dCa E^t + dCb curl^t from the
 * background's snapshots of that step; rec_dev [nt][S][n_rec] receives its
 * records.  The background is the last mw_tm_forward on this workspace with
 * the same p, ca, cb, cq, cpml: its stored snapshots (FP32, BF16 or FP8, on
 * the device or in pinned host memory with snap_host, used exactly as
 * stored) or, with MW_SNAP_CKPT, its checkpoints replayed segment by segment
 * (which needs f and src_idx again).  dca_dev / dcb_dev are model-shaped
 * float32.  The workspace's adjoint state buffers are overwritten; the
 * snapshots and checkpoints are kept, so mw_tm_adjoint_grad may follow. */
int mw_tm_born(const mw_params *p, const float *ca_dev, const float *cb_dev, const float *cq_dev,
               const float *cpml_dev, const float *dca_dev, const float *dcb_dev,
               const float *f_dev, const int64_t *src_idx_dev, const int64_t *rec_idx_dev,
               float *rec_dev, void *workspace_dev, size_t workspace_bytes, void *stream);

/* Shot reduction (the page's combine_grad, over every cell):
 * grad[j] (+)= sum_{s=0..S-1} grad_shot[s][j], shots summed in order in
 * float32.  accumulate = 0 overwrites, 1 adds. */
int mw_combine_grad(const mw_params *p, const float *grad_shot_dev,
                    float *grad_dev, int32_t accumulate, void *stream);

/* Chain rule to relative permittivity and conductivity (the page's
 * convert_grad_ca_cb_to_eps_sigma): with dCa/deps = (1-Ca)Cb/dt,
 * dCb/deps = -Cb^2/dt, dCa/dsigma = -(1+Ca)Cb/2, dCb/dsigma = -Cb^2/2,
 *   grad_eps_r = eps0 (gCa dCa/deps + gCb dCb/deps),
 *   grad_sigma = gCa dCa/dsigma + gCb dCb/dsigma.
 * n cells; either output may be NULL. */
int mw_grad_eps_sigma(int64_t n, double dt, const float *ca_dev,
                      const float *cb_dev, const float *grad_ca_dev,
                      const float *grad_cb_dev, float *grad_eps_r_dev,
                      float *grad_sigma_dev, void *stream);

/* Residual res = d - d_obs over n values and, when J_dev is not NULL, the
 * misfit J = 1/2 sum res^2 (one double, fixed summation order). */
int mw_residual(int64_t n, const float *d_dev, const float *d_obs_dev,
                float *res_dev, double *J_dev, void *stream);

/* Wait for `stream` and report device-side status recorded in the workspace
 * by earlier calls (MW_ERR_NONFINITE), then clear it. */
int mw_sync_status(void *workspace_dev, void *stream);

/* Thread-local message of the last failing call ("" if none). */
const char *mw_last_error(void);

/* Per-kernel timing (CUDA events around each launch of the stencil kernels,
 * by class: 0 forward, 1 forward with snapshot store, 2 adjoint, 3 Born
 * forward, 4 / 5 two-step forward without / with snapshot store; whole-sweep
 * launches of small grids, each covering all nt steps: 6 / 7 / 8 with the
 * state in shared memory, 9 / 10 / 11 with the state in global memory
 * (forward, forward with snapshot store, adjoint)).  enable = 1 clears and
 * starts recording; mw_profile_read synchronizes the recorded events and
 * returns, per class, the launch count and total milliseconds. */
int mw_profile_enable(int32_t enable);
int mw_profile_read(int64_t *counts, double *total_ms, int32_t n_classes);

/* Number of CUDA kernels this library has launched in this process (all
 * entry points, all devices).  Host counter; no synchronization. */
int64_t mw_launch_count(void);

/* Failure-detection self-test (no counterpart on the pages): launches one
 * kernel whose stage wait nothing completes (an expected byte count no copy
 * delivers).  The wait gives up after its bounded poll count (about half a
 * second), records the timeout in the workspace's status words and returns,
 * exactly as a stencil kernel does when one of its copies never lands.  The
 * next mw_sync_status reports MW_ERR_TIMEOUT and clears it; until then the
 * stencil kernels launched on this workspace return at once.  No copy is in
 * flight when the kernel ends and the context stays usable. */
int mw_selftest_wait_timeout(void *workspace_dev, void *stream);

/* Snapshot storage encoding (page: maxwell.cu, the bf16 / "FP8 E4M3"
 * storage helpers used by forward_kernel_e_with_storage_bf16 / _fp8).
 * Rounds n float32 values x_dev[0..n) to the storage format of snap_mode
 * (MW_SNAP_BF16: bfloat16, 2 bytes each; MW_SNAP_FP8: E4M3, 1 byte each)
 * into out_dev, with the same device conversion the forward kernel applies
 * when it stores snapshots.  n % 4 == 0; x_dev 16-byte aligned, out_dev
 * 8-byte (bf16) or 4-byte (fp8) aligned; device pointers owned by the
 * caller.  Asynchronous on `stream`.  MW_ERR_ARG for another snap_mode, a
 * bad n or misaligned pointers. */
int mw_snapshot_encode(int32_t snap_mode, int64_t n, const float *x_dev, void *out_dev,
                       void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MW_TM_H */
