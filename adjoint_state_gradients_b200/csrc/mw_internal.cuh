// Internal declarations of the mw_tm library (CUDA, sm_100a).
//
// Data layout in HBM (float32 unless noted):
//   fields       [S][ny][nx]           Ey, Hx, Hz (or their adjoints)
//   x-band mem   [S][ny][2*Wx]         columns [0,Wx) then [nx-Wx,nx)
//   z-band mem   [S][2*Wz][nx]         rows    [0,Wz) then [ny-Wz,ny)
//   model        [ny][nx] or [S][ny][nx]
//   snapshots    [n][S][ny][nx]        float32 or bf16
// Stencil kernels are "marching strips": one warp owns a 128-column strip of
// one shot over a chunk of rows and walks down it, keeping the y-direction
// stencil operands in registers and the x-direction ones in a per-warp
// shared-memory row, so each cell's state is read and written once per step.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mw_tm.h"

namespace mw {

constexpr int kStripCols = 128;    // columns per warp (32 lanes x float4)
constexpr int kWarpsPerCta = 4;
constexpr int kEySlots = 36;       // 2 left halo + 32 own + 2 right halo float4
constexpr int kHzSlots = 34;       // 1 left halo + 32 own + 1 right halo float4

struct Geom {
  int ny, nx, S;
  int Wx, Wz;         // band widths (0: no CPML band)
  int n_strips, n_chunks, chunk_h;
  int n_pml;
  int grad_mask;      // adjoint: accumulate gradients outside the band only
  int64_t numel;      // ny * nx
};

// Staggered first-derivative weights times 1/dx (cx) and 1/dy (cy).
struct Coef {
  float cx[4], cy[4];
};

// CPML profiles (device): y axis then x axis; "h" = half node.
struct Prof {
  const float *ay, *ayh, *by, *byh, *ky, *kyh;
  const float *ax, *axh, *bx, *bxh, *kx, *kxh;
};

// One state buffer (forward fields or their adjoints).
struct Fields {
  float *ey, *hx, *hz;
  float *mxh_node;  // x-band memory at the H (Hz) nodes
  float *mxe_node;  // x-band memory at the E nodes
  float *mzh_node;  // z-band memory at the H (Hx) nodes
  float *mze_node;  // z-band memory at the E nodes
};

struct StepArgs {
  Geom g;
  Coef c;
  Prof pr;
  Fields in, out;
  const float *ca, *cb, *cq;
  float cq_scalar;
  // snapshots of this step ([S][ny][nx]; float or bf16), may be null
  void *snap_e, *snap_c;
  // adjoint only: per-shot gradients [S][ny][nx]
  float *gca, *gcb;
};

// Workspace layout (byte offsets, 256-aligned).
struct Layout {
  size_t flags;       // 256 B of device status words
  size_t stA, stB;    // forward ping-pong state buffers (stA used when state==NULL)
  size_t adA, adB;    // adjoint ping-pong state buffers
  size_t rpA, rpB;    // replay ping-pong state buffers (checkpoint mode)
  size_t snap;        // snapshots / checkpoints
  size_t seg;         // checkpoint mode: fp32 segment snapshot buffer
  size_t total;
  size_t state_bytes;
  size_t snap_step_bytes;  // one step of one snapshot field ([S][ny][nx])
  int n_seg;
};

enum StoreKind { kStoreNone = 0, kStoreF32 = 1, kStoreBF16 = 2 };

// device status word indices in the flags area
enum { kFlagNonFinite = 0, kFlagBadIndex = 1 };

// count of kernel launches made by the library (mw_host.cu)
void count_launches(int n);

// stencil launchers (mw_stencil.cu); return a cudaError_t
cudaError_t launch_forward(const StepArgs &a, int order, int store, bool batched,
                           bool cq_array, int grid, cudaStream_t st);
cudaError_t launch_adjoint(const StepArgs &a, int order, int snap_bf16,
                           bool batched, bool cq_array, int grid,
                           cudaStream_t st);
int stencil_slots_per_sm(int order, bool adjoint);

// small kernels (mw_aux.cu)
cudaError_t launch_src_rec(float *ey, int64_t numel, int S, const float *f_t,
                           const int64_t *src, int ns, const int64_t *rec,
                           int nr, float *r_t, int *flags, cudaStream_t st);
cudaError_t launch_adj_src_rec(float *lam, int64_t numel, int S,
                               const float *res_t, const int64_t *rec, int nr,
                               const int64_t *src, int ns, float *gf_t,
                               int *flags, cudaStream_t st);
cudaError_t launch_check_finite(const float *x, int64_t n, int *flags,
                                cudaStream_t st);
cudaError_t launch_model(int64_t n, const float *eps_r, const float *sigma,
                         const float *mu_r, double dt, float *ca, float *cb,
                         float *cq, int cq_full, cudaStream_t st);
cudaError_t launch_cpml(int ny, int nx, int n_pml, double dy, double dx,
                        double dt, double vmax, double f0, double R, float *out,
                        cudaStream_t st);
cudaError_t launch_combine(const float *gs, float *g, int S, int64_t n,
                           int accumulate, cudaStream_t st);
cudaError_t launch_eps_sigma(int64_t n, double dt, const float *ca,
                             const float *cb, const float *gca,
                             const float *gcb, float *ge, float *gs,
                             cudaStream_t st);
cudaError_t launch_residual(int64_t n, const float *d, const float *o,
                            float *res, double *J, cudaStream_t st);

}  // namespace mw
