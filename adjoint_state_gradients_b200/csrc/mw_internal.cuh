// Internal declarations of the mw_tm library (CUDA, sm_100a).
//
// Data layout in HBM (float32 unless noted):
//   fields       [S][ny][nx]           Ey, Hx, Hz (or their adjoints)
//   x-band mem   [S][ny][2*Wx]         columns [0,Wx) then [nx-Wx,nx)
//   z-band mem   [S][2*Wz][nx]         rows    [0,Wz) then [ny-Wz,ny)
//   model        [ny][nx] or [S][ny][nx]
//   snapshots    [2][n][S][ny][pitch]  float32, bf16 or E4M3 (rows padded
//                                      to 16 bytes)
// Stencil kernels are "marching strips": one warp owns a 120- (forward) or
// 112-column (adjoint) strip of one shot over a chunk of rows and walks down
// it, keeping the y-direction stencil operands in registers and the
// x-direction ones in per-warp shared-memory rows, so each cell's state is
// read and written once per step.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/mw_tm.h"

namespace mw {

constexpr int kFwdStripCols = 120;  // forward: columns owned per warp (30 float4)
constexpr int kAdjStripCols = 112;  // adjoint: columns owned per warp (28 float4)
constexpr int kWarpsPerCta = 4;    // forward CTA: 4 warps
constexpr int kAdjWarpsPerCta = 5; // adjoint CTA: 5 warps (at most)
// warps of an adjoint CTA: 4 at order 8, whose larger stages then fit three
// CTAs an SM, else 5
__host__ __device__ constexpr int adj_warps_per_cta(int P) { return P == 4 ? 4 : kAdjWarpsPerCta; }

struct Geom {
  int ny, nx, S;
  int Wx, Wz;         // band widths (0: no CPML band)
  int strip_cols, n_strips, n_chunks;
  // row chunks: n_big chunks of chunk_h rows, then chunks of chunk_h2 rows
  // (the last one ragged); the short chunks are claimed last
  int chunk_h, chunk_h2, n_big;
  // strips [is_lo, is_hi) and chunks [ic_lo, ic_hi) form the interior
  // rectangle (items whose walk touches no band and no array edge)
  int is_lo, is_hi, ic_lo, ic_hi;
  int n_pml;
  int grad_mask;      // adjoint: accumulate gradients outside the band only
  int64_t numel;      // ny * nx
};

// Staggered first-derivative weights times 1/dx (cx) and 1/dy (cy).
struct Coef {
  float cx[4], cy[4];
};

// One state buffer (forward fields or their adjoints).
struct Fields {
  float *ey, *hx, *hz;
  float *mxh_node;  // x-band memory at the H (Hz) nodes
  float *mxe_node;  // x-band memory at the E nodes
  float *mzh_node;  // z-band memory at the H (Hx) nodes
  float *mze_node;  // z-band memory at the E nodes
};

// Sorted source or receiver entries of one index set idx [S][n] (built once
// per call by launch_entry_table), so that the stencil kernels inject and
// sample them in the rows they compute:
//   ent  [S][n]    the valid entries of each shot sorted by (cell, k):
//                  {row, column, k, run}; run = the number of consecutive
//                  entries with this cell when this is the first of them,
//                  else 0 (duplicates add up in index order)
//   arow [S][n+1]  the distinct rows holding entries, ascending, then INT_MAX
//   abeg [S][n+1]  the first sorted position of each of those rows, then the
//                  number of valid entries
//   rcur [S][ny+1] for each row y: {a, arow[a]} with a the first active row
//                  at or after y (where a walk starting at row y begins)
// An empty set has n == 0 and null pointers.
struct EntrySet {
  const int4 *ent;
  const int *arow, *abeg;
  const int2 *rcur;
  int n, ny;
};

// Forward stage slots placed by the host (float offsets within a stage).
enum { kFoCqH = 0, kFoCqX, kFoMzh, kFoMze, kFoMxh, kFoMxe, kFoBd, kFoBs, kFoCount };
// Adjoint stage slots placed by the host.
enum { kAoCqR = 0, kAoCqH, kAoMx, kAoMze, kAoMzh, kAoCount };

struct StepArgs {
  Geom g;
  Coef c;
  Fields in, out;
  const float *ca, *cb, *cq;
  float cq_scalar;
  // forward: snapshots of this step ([S][ny][snap_pitch]; float32, bf16 or
  // E4M3 bytes), may be null
  void *snap_e, *snap_c;
  int snap_pitch;     // snapshot row pitch in elements (>= nx, 16-byte rows)
  // adjoint only: per-shot gradients [S][ny][nx]; time index of the
  // snapshot tensor maps
  float *gca, *gcb;
  int snap_t;
  int tzero;          // adjoint, kStoreEy: this launch is step t = 0
  int *flags;         // device status words (wait timeouts, work counters)
  int ctr_slot;       // work counter of this launch (flags[kCtrBase + ctr_slot])
  // CPML band coefficients (BandTab layout), float4-aligned, 1/k precomputed
  const float *bt;
  // shared-memory layout of one warp (floats): stage size, warp area, band
  // row width (the x-band memory TMA box, 2*Wx)
  int stage_floats, warp_floats, band_box_floats;
  int band_ring;  // two-step forward: floats per band row of the x-band carry rings
  // forward only: optional stage slots (kFo*), Ca / Cb pair fetch and order
  int fo[kFoCount];
  int md_pair, md_swap;
  int bd_pair, bd_swap;  // Born forward: dCa / dCb pair fetch and order
  // adjoint only: optional stage slots (kAo*), gCa / gCb pair fetch and order
  int ao[kAoCount];
  int gg_pair, gg_swap;
  // sources / receivers of this step: set `ea` is injected (forward: the
  // sources, vals_t = f[t]; adjoint: the receivers, vals_t = res[t]), set
  // `eb` is sampled after the injection (forward: the receivers, out_t =
  // rec[t]; adjoint: the sources, out_t = grad_f[t]); vals_t / out_t are
  // [S][n] slices, null when there is nothing to inject / record
  EntrySet ea, eb;
  const float *vals_t;
  float *out_t;
  // two-step forward launches (k_forward2): the second step's snapshots,
  // source values and records (the first step's are snap_e / snap_c,
  // vals_t, out_t)
  void *snap_e2, *snap_c2;
  const float *vals_t2;
  float *out_t2;
};

// TMA tensor maps of one forward launch (the input buffer set and model).
// Boxes are one row high:
//   kMapEH  Ey and Hz of one row as one 4-D box (x, y, shot, field) with the
//           field stride Hz - Ey: 136 wide from x0 - 8, 2 fields
//   kMapHX  Hx, 120 wide from x0
//   kMapMD  Ca and Cb as one pair box (x, y, shot, field; field stride
//           |Cb - Ca|, the lower address first) when md_pair, else Ca alone
//           with kMapCB beside it; 120 wide from x0
//   kMapCQ  Cq when it is an array: 128 wide from x0 - 4
//   kMapMXH / kMapMXE  x-band memories, a whole band row (2*Wx)
//   kMapMZH / kMapMZE  z-band memories, 120 wide from x0
//   kMapBD / kMapBDB  Born forward: dCa and dCb (like kMapMD / kMapCB)
//   kMapBS  Born forward: the background's E and curl snapshots of the step
//           as one 5-D box, 144 wide from a 16-element boundary
enum FwdMap {
  kMapEH = 0, kMapHX, kMapMD, kMapCB, kMapCQ, kMapMXH, kMapMXE, kMapMZH, kMapMZE, kMapBD,
  kMapBDB, kMapBS, kFwdMaps
};
struct FwdMaps {
  CUtensorMap map[kFwdMaps];
};
// TMA tensor maps of one adjoint launch.  Boxes are one row high:
//   kAMapEH  lambda_E and lambda_Hz of one row as one 4-D box (field stride
//            lambda_Hz - lambda_E): 128 wide from x0 - 8, 2 fields
//   kAMapMD  Ca and Cb of one row as one pair box when md_pair (else Ca, with
//            kAMapCB beside it): 128 wide from x0 - 8
//   kAMapHX  lambda_Hx, 112 wide from x0
//   kAMapSS  the E and curl snapshots as one 5-D box (x, y, shot, step,
//            field): 112 wide from x0
//   kAMapGG  the per-shot gradients gCa, gCb as one pair box when gg_pair
//            (else gCa, with kAMapGB beside it): 112 wide from x0
//   kAMapCQ  Cq when it is an array: 128 wide from x0 - 8
//   kAMapMX  the x-band memories at the H and E nodes (adjacent arrays) as
//            one pair box of whole band rows
//   kAMapMZE / kAMapMZH  z-band memories, 112 wide from x0
//   kAMapCA  Ca alone, 112 wide from x0 (kStoreEy: a row's E update and its
//            gradients come 2P - 1 rows after its first fetch, which then
//            needs Cb alone, kAMapCB; the walk carries lambda_E to the E
//            update and kAMapSS is the E snapshot alone, 4-D)
enum AdjMap {
  kAMapEH = 0, kAMapMD, kAMapCB, kAMapHX, kAMapSS, kAMapGG, kAMapGB, kAMapCQ, kAMapMX,
  kAMapMZE, kAMapMZH, kAMapCA, kAdjMaps
};
struct AdjMaps {
  CUtensorMap map[kAdjMaps];
};

// TMA tensor maps of one two-step forward launch (k_forward2).  Boxes are one
// row high and 128 wide from the walk's first column x0 - H (H the x halo):
//   kM2E, kM2HZ, kM2HX  Ey (row r), Hz (row r - 2P + 1), Hx (row r - P)
//   kM2MD / kM2CB  Ca and Cb as one pair box when md_pair, else two boxes
//   kM2MXH / kM2MXE  x-band memories, a whole band row (2*Wx)
//   kM2MZH / kM2MZE  z-band memories
enum Fwd2Map { kM2E = 0, kM2HZ, kM2HX, kM2MD, kM2CB, kM2MXH, kM2MXE, kM2MZH, kM2MZE, kFwd2Maps };
struct Fwd2Maps {
  CUtensorMap map[kFwd2Maps];
};
// Two-step forward: columns of x halo on each side of the owned strip, and
// the owned strip width (the walk covers 128 columns).  The halo holds the
// 4P - 2 columns two steps consume, rounded up to whole float4s.
__host__ __device__ constexpr int fwd2_halo(int P) { return P <= 2 ? 8 : P == 3 ? 12 : 16; }
__host__ __device__ constexpr int fwd2_width(int P) { return 128 - 2 * fwd2_halo(P); }

// Rows [ya, yb) of row chunk k.
__host__ __device__ inline void chunk_rows(const Geom &g, int k, int *ya, int *yb) {
  const bool big = k < g.n_big;
  const int a = big ? k * g.chunk_h : g.n_big * g.chunk_h + (k - g.n_big) * g.chunk_h2;
  const int h = big ? g.chunk_h : g.chunk_h2;
  *ya = a;
  *yb = a + h < g.ny ? a + h : g.ny;
}

// Claim order of the work items: items touching a band or an array edge
// first, then the interior rectangle; the shot index runs fastest, then the
// strip, then the chunk.  A bijection of [0, S * n_strips * n_chunks).
__host__ __device__ inline void item_coords(const Geom &g, int item, int *s, int *strip,
                                            int *chunk) {
  const int ns = g.n_strips, nc = g.n_chunks;
  const int n_is = g.is_hi > g.is_lo ? g.is_hi - g.is_lo : 0;
  const int n_ic = g.ic_hi > g.ic_lo ? g.ic_hi - g.ic_lo : 0;
  const int n_int = g.S * n_is * n_ic;
  const int n_band = g.S * ns * nc - n_int;
  *s = item % g.S;
  if (item < n_band) {
    const int jj = item / g.S;
    const int n_ec = nc - n_ic;  // chunks touching a z edge: all their strips
    if (jj < n_ec * ns) {
      const int ci = jj / ns;
      *strip = jj % ns;
      *chunk = ci < g.ic_lo ? ci : g.ic_hi + (ci - g.ic_lo);
    } else {  // interior chunks: only the edge strips
      const int k = jj - n_ec * ns;
      const int n_es = ns - n_is;
      const int e = k % n_es;
      *chunk = g.ic_lo + k / n_es;
      *strip = e < g.is_lo ? e : g.is_hi + (e - g.is_lo);
    }
  } else {
    const int jj = (item - n_band) / g.S;
    *strip = g.is_lo + jj % n_is;
    *chunk = g.ic_lo + jj / n_is;
  }
}

// Workspace layout (byte offsets, 256-aligned).
struct Layout {
  size_t flags;       // 256 B of device status words
  size_t stA, stB;    // forward ping-pong state buffers (stA used when state==NULL)
  size_t adA, adB;    // adjoint ping-pong state buffers
  size_t rpA, rpB;    // replay ping-pong state buffers (checkpoint mode)
  size_t snap;        // snapshots / checkpoints
  size_t seg;         // checkpoint mode: fp32 segment snapshot buffer
  size_t tab_src, tab_rec;  // entry tables of the sources and of the receivers
  size_t bandtab;     // CPML band coefficient table (BandTab)
  // MW_SNAP_CKPT_EY: the Cb-gradient accumulator [S][ny][nx], the record copy
  // [nt][S][n_rec], the receiver / source end-term sums [S][n_rec + n_src] and
  // lambda_E sampled at the sources [nt][S][n_src] (when the caller asks for
  // no grad_f)
  size_t sbp, rcopy, acc, gfbuf;
  // checkpoint modes: snapshots of the last n_tail steps, stored by the forward
  size_t tail;
  int n_tail;
  size_t total;
  size_t state_bytes;
  size_t snap_step_bytes;  // one step of one snapshot field ([S][ny][snap_pitch])
  int snap_pitch;          // snapshot row pitch (elements): rows start 16-byte aligned
  int n_seg;
};

// kStoreEy: the E snapshot alone, float32 (the summation-by-parts Cb
// gradient needs no curl snapshot)
enum StoreKind { kStoreNone = 0, kStoreF32 = 1, kStoreBF16 = 2, kStoreFP8 = 3, kStoreEy = 4 };

// device status word indices in the flags area; kCtrBase, kCtrBase + 1: the
// work-item counters that consecutive stencil launches alternate between
enum { kFlagNonFinite = 0, kFlagBadIndex = 1, kFlagTimeout = 2, kCtrBase = 32 };

// CPML band coefficient table (floats; Wx, Wz as in Geom): x band per band
// column j (array column j < Wx ? j : nx - 2*Wx + j), z band per band row.
//   [0]   a_x   [1] b_x   [2] 1/k_x     (integer nodes)
//   [3]   a_xh  [4] b_xh  [5] 1/k_xh    (half nodes)          2*Wx each
//   [6..11] the same along z                                  2*Wz each
struct BandTab {
  int Wx, Wz;
  __host__ __device__ int x(int k) const { return k * 2 * Wx; }
  __host__ __device__ int z(int k) const { return 12 * Wx + k * 2 * Wz; }
  __host__ __device__ int floats() const { return 12 * Wx + 12 * Wz; }
};

// count of kernel launches made by the library (mw_host.cu)
void count_launches(int n);

// Launch with programmatic stream serialization: the kernel may begin
// launching while the previous kernel in the stream finishes; it must wait
// (griddepcontrol.wait) before reading that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), int grid, int block, size_t smem,
                             cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// two-step forward (steps t and t + 1 in one launch): scalar Cq, orders 2-6,
// no Born term; store as in launch_forward (both steps' snapshots)
cudaError_t launch_forward2(const Fwd2Maps &m, const StepArgs &a, int order, int store,
                            bool batched, int grid, cudaStream_t st);
void forward2_layout(int order, int Wx, StepArgs *a, size_t *smem_bytes);
int forward2_slots_per_sm(int order, int Wx);
bool forward2_supported(int order);
// stencil launchers (mw_stencil.cu); return a cudaError_t
// born: kStoreNone, or the background snapshots' kind for the Born forward
// (then store must be kStoreNone)
cudaError_t launch_forward(const FwdMaps &m, const StepArgs &a, int order, int store, int born,
                           bool batched, bool cq_array, int grid, cudaStream_t st);
// snap: the snapshot storage (kStoreF32, kStoreBF16 or kStoreFP8)
cudaError_t launch_adjoint(const AdjMaps &m, const StepArgs &a, int order, int snap,
                           bool batched, bool cq_array, int grid, cudaStream_t st);
// snapshot storage encoding of n floats (n % 4 == 0) with the forward's
// conversion (kStoreBF16 or kStoreFP8)
cudaError_t launch_snap_encode(int store, int64_t n, const float *x, void *out, cudaStream_t st);
// a stage wait that nothing completes (bounded; sets the timeout flag)
cudaError_t launch_wait_selftest(int *flags, cudaStream_t st);
// forward / adjoint: the full stage layout (optional slots for a Cq array and
// bands)
void forward_layout(int order, int Wx, bool cq_array, bool born, StepArgs *a, size_t *smem_bytes);
void adjoint_layout(int order, int Wx, bool cq_array, bool bf16, StepArgs *a, size_t *smem_bytes);
int stencil_slots_per_sm(int order, bool adjoint, int Wx, bool cq_array);

// Whole-sweep launches for small grids (mw_small.cu): one cooperative launch
// runs every step of the forward or the adjoint, the state updated in place.
struct SmallArgs {
  int S, ny, nx, Wx, Wz, n_pml, grad_mask, batched, cq_arr, nt;
  // resident variant (set by launch_small): rows a block; steps a chunk of
  // the global traffic; ring entries a step for sources and receivers
  int rows, kchunk, csrc, crec;
  int64_t numel;
  Coef c;
  Fields st;                 // the state, updated in place
  const float *ca, *cb, *cq;
  const float *bt;           // CPML band table (BandTab)
  void *snap_e, *snap_c;     // snapshots [nt][S][ny][pitch]: step t at t * step_elems
  int64_t step_elems;
  int snap_pitch;
  EntrySet src, rec;
  const float *f;            // forward: [nt][S][n_src] or null
  float *rec_out;            // forward: [nt][S][n_rec] or null
  const float *res;          // adjoint: [nt][S][n_rec] or null
  float *grad_f;             // adjoint: [nt][S][n_src] or null
  float *gca, *gcb;          // adjoint: per-shot gradients (+=)
  float *px, *pz, *qx, *qz;  // adjoint: scratch [S][ny][nx] each
  int *flags;                // status words
};
// Shape of a whole-sweep launch: the resident variant (each block's rows in
// shared memory, `rows` rows a block) or the L2 variant (the state in global
// memory); `cluster` blocks per shot, `block` threads a block.
struct SmallPlan {
  bool resident;
  int block, cluster, rows, kchunk, csrc, crec, width;  // width: cells a thread's group
  size_t smem;
};
// The shape for one direction (store: the forward's snapshot kind, or the
// adjoint's) of a shot of ny x nx cells; false when no cluster fits.
bool small_plan(int order, bool adjoint, int store, int ny, int nx, int Wx, int Wz, int n_src,
                int n_rec, SmallPlan *pl);
// store: the forward's snapshot kind (kStoreNone / F32 / BF16 / FP8), or the
// adjoint's (kStoreF32 / BF16 / FP8); one cluster per shot
cudaError_t launch_small(const SmallArgs &a, bool adjoint, int order, int store,
                         const SmallPlan &pl, cudaStream_t st);

// small kernels (mw_aux.cu)
// Bytes of the entry table of an index set [S][n] on ny rows (EntrySet layout).
size_t entry_table_bytes(int S, int n, int ny);
// The EntrySet of an index set whose table starts at `base`.
EntrySet entry_set_at(void *base, int S, int n, int ny);
// Build the entry table of idx [S][n] (cells y * nx + x, -1 inactive) into
// the table at `base`; out-of-range entries set the bad-index flag.  Entries
// that are not valid record nothing: with `out` ([nt][S][n]) their outputs
// are zeroed for every step.
cudaError_t launch_entry_table(const int64_t *idx, int S, int n, int ny, int nx, void *base,
                               int *flags, float *out, int nt, cudaStream_t st);
// Add vals [S][ea.n] at the cells of set `ea` of the E field [S][ny][nx]
// (duplicates added up in index order first), then read the field at the
// cells of set `eb` into out [S][eb.n]; either part is skipped when its
// pointer is null.
cudaError_t launch_fix_field(float *field, int S, int ny, int nx, const EntrySet &ea,
                             const float *vals, const EntrySet &eb, float *out, cudaStream_t st);
// End-term sums of the summation-by-parts Cb gradient, in the adjoint's
// order t = nt - 1 .. 0: acc_rec[s][k] = sum_t res[t][s][k] rec[t][s][k] (the
// residual times the record it answers) and acc_src[s][k] = sum_t
// f[t][s][k] lam[t][s][k] (the source wavelet times lambda_E sampled at the
// source).  A null pair skips that sum.
cudaError_t launch_sbp_sums(int nt, int S, const float *res, const float *rec, int n_rec,
                            float *acc_rec, const float *f, const float *lam, int n_src,
                            float *acc_src, cudaStream_t st);
// summation-by-parts Cb gradient: P = lambda_E * E (the end term of a given
// adjoint start state), the scatter of the end-term sums into P (sequential
// per shot: duplicates add in index order), and grad_cb_shot += P / Cb at
// the cells the gradient mask keeps
cudaError_t launch_sbp_init(float *P, const float *lam, const float *e, int64_t n,
                            cudaStream_t st);
cudaError_t launch_sbp_scatter(float *P, int64_t numel, int S, const int64_t *rec_idx,
                               const float *acc_rec, int n_rec, const int64_t *src_idx,
                               const float *acc_src, int n_src, cudaStream_t st);
cudaError_t launch_sbp_finish(const float *P, const float *cb, float *gcb, int S, int ny, int nx,
                              int batched, int mask_pml, cudaStream_t st);
cudaError_t launch_check_finite(const float *x, int64_t n, int *flags,
                                cudaStream_t st);
cudaError_t launch_model(int64_t n, const float *eps_r, const float *sigma,
                         const float *mu_r, double dt, float *ca, float *cb,
                         float *cq, int cq_full, cudaStream_t st);
cudaError_t launch_band_table(const float *cpml, int ny, int nx, int Wx, int Wz, float *out,
                              cudaStream_t st);
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
