// Stencil kernels of the 2-D TM Maxwell FDTD step and its exact adjoint.
//
// Method: page "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu" -- header comment
// (discrete forward / adjoint equations, gradient formulas) and its
// forward_kernel_h / forward_kernel_e / backward kernels, which this file
// replaces with one fused kernel per step in each direction:
//
//   forward step (k_forward), per cell:
//     Hz' = Hz + Cq psi_x^h(D_x^h Ey),   Hx' = Hx - Cq psi_z^h(D_z^h Ey)
//     curl = psi_x(D_x Hz') - psi_z(D_z Hx')
//     [store Ey, curl]   Ey' = Ca Ey + Cb curl
//   adjoint step (k_adjoint), the literal transpose, per cell:
//     gCa += Ey^t lam, gCb += curl^t lam            (lam = lambda_E^{t+1})
//     g = Cb lam; px = psi^T_x(g), pz = psi^T_z(-g) at E nodes (integer grid)
//     lamHz' = lamHz - D_x^h px,  lamHx' = lamHx - D_z^h pz
//     qx = psi^T_x^h(Cq lamHz'), qz = psi^T_z^h(-Cq lamHx')      (H nodes)
//     lam' = Ca lam - D_x qx - D_z qz
//   psi(d) = d/k + m with m <- b m + a d;  psi^T(v) = v/k + a M with
//   M = m_adj + v, m_adj <- b M (the transposed recursion at the same node).
//
// Work decomposition ("marching strips"): one warp owns a strip of columns
// (forward 120 = 30 float4, adjoint 112 = 28 float4) of one shot over a chunk
// of rows and walks it top to bottom; lane l works on the float4 at column
// x0 - 4 + 4l (forward) or x0 - 8 + 4l (adjoint), so the halo columns the
// x-stencils need are computed in the same SIMD pass as the owned ones.
// Input rows arrive by TMA (cp.async.bulk.tensor, one-row boxes, zero fill
// outside the array) into a ring of L+1 shared-memory stages, L rows ahead
// of the row being computed, each tracked by an mbarrier with a bounded
// wait.  Lane 0 issues all of a row's loads; fields that share a row and a
// column range come as one multi-field box (Ey with Hz, Ca with Cb, the two
// snapshots, the two gradients).  The y-stencil operands live in register
// queues; the x-stencil operands come from the staged row and from a ring of
// 2P computed rows.  States are ping-ponged between two buffers so halo
// recompute never races with a neighbour's writes.  Items whose walk touches
// neither a CPML band nor the array's side edges take a lean path with no
// band code; CPML memories exist only in the bands.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <atomic>

#include "mw_device.cuh"
#include "mw_internal.cuh"

namespace mw {
namespace {
using namespace dev;

// Stage layouts (float offsets, 128-byte aligned slots).
// forward: Ey and Hz of row r (one pair box), Hx of row r - P, Ca / Cb of
// row r - 2P + 1 (one pair box); optional slots follow at host-given offsets
constexpr int kF_EY = 0, kF_HZ = 136, kF_HX = 288, kF_MD = 416, kF_FIXED = 672;
static_assert(kF_MD + 128 + 120 <= kF_FIXED, "Ca / Cb slots overflow");
// adjoint: lambda_E and lambda_Hz of row r (one pair box), Ca / Cb of row r
// (one pair box), lambda_Hx of row r - P, the two snapshots of row r (one
// box), the per-shot gradients of row r (one pair box); optional slots follow
constexpr int kA_EH = 0, kA_MD = 256, kA_HX = 512, kA_SS = 640, kA_GG = 896, kA_FIXED = 1152;
static_assert(kA_GG + 128 + 112 <= kA_FIXED, "gradient slots overflow");
constexpr int kFRing = 128;  // forward Hz ring row: 32 float4
constexpr int kAPx = 128;    // adjoint px row: 32 float4
constexpr int kARing = 120;  // adjoint qx ring row: 30 float4

template <int L>
struct Stages {
  static_assert(kWarpsPerCta * (L + 1) * 8 <= 128, "barrier area too small");
  static_assert(kAdjWarpsPerCta * (L + 1) * 8 <= 128, "barrier area too small");
};

// D_x^h at half node xb+q+1/2 from integer-node values w[col - xb + 4].
template <int P>
__device__ __forceinline__ float d_half(const float w[12], int q, const float c[4]) {
  float d = 0.f;
#pragma unroll
  for (int k = 1; k <= P; ++k) d = fmaf(c[k - 1], w[q + k + 4] - w[q - k + 5], d);
  return d;
}
// D_x at integer node xb+q from half-node values w[col - xb + 4].
template <int P>
__device__ __forceinline__ float d_int(const float w[12], int q, const float c[4]) {
  float d = 0.f;
#pragma unroll
  for (int k = 1; k <= P; ++k) d = fmaf(c[k - 1], w[q + k + 3] - w[q - k + 4], d);
  return d;
}

__device__ __forceinline__ int xband_col(int c, int nx, int Wx) {
  if (c < 0 || c >= nx) return -1;
  if (c < Wx) return c;
  if (c >= nx - Wx) return c - nx + 2 * Wx;
  return -1;
}
__device__ __forceinline__ int zband_row(int r, int ny, int Wz) {
  if (r < 0 || r >= ny) return -1;
  if (r < Wz) return r;
  if (r >= ny - Wz) return r - ny + 2 * Wz;
  return -1;
}

// Ring position of the running iteration counter.
struct Ring {
  int slot;
  uint32_t phase;
  __device__ __forceinline__ void next(int nslots) {
    if (++slot == nslots) {
      slot = 0;
      phase ^= 1u;
    }
  }
};


// Register queues of the z-stencils: the last 2P rows of a quantity.  The
// walk's loop body is unrolled over a group of M iterations.  With M == 2P a
// queue is a ring indexed modulo 2P (no moves); with a smaller M (long
// stencils, to keep the unrolled body small enough for the instruction
// cache) it is a window of 2P + M - 1 entries, written at 2P - 1 + t in step
// t of a group and shifted down by M after each group.
template <int NQ, int M>
struct Queue {
  static constexpr int kSize = M == NQ ? NQ : NQ + M - 1;
  // entry holding the row j rows older than the one written in step t
  __host__ __device__ static constexpr int at(int t, int j) {
    return M == NQ ? (t - j + 2 * NQ) % NQ : NQ - 1 + t - j;
  }
};
template <int NQ, int M, int N>
__device__ __forceinline__ void shift_queue(F4 (&q)[N]) {
  if constexpr (M != NQ) {
#pragma unroll
    for (int k = 0; k < NQ - 1; ++k) q[k] = q[k + M];
  }
}
// iterations per unrolled group of a walk: 1 for the adjoint (but at order
// 6, where one iteration a group spills) and for the forward at order 8,
// else 2 (measured on B200: order 8 runs 1.3-1.6x
// faster with groups of 2 than with the full ring of 8, and one iteration a
// group -- half the loop's code, more queue moves -- takes its bf16-snapshot
// forward and adjoint launches from 0.147 / 0.226 to 0.139 / 0.217 ms at
// 1064^2 x 16 shots; the order-4 E-alone adjoint, unrolled over its full
// ring of 4 before, from 0.308 to 0.303 ms at 2128^2 x 8 shots, with 88
// registers instead of 123; the order-4 one-step forward gained 3 % with
// groups of 2 over the full ring)
template <int P, bool ADJ>
__host__ __device__ constexpr int walk_group() {
  return ADJ ? (P == 3 ? 2 : 1) : (P == 4 ? 1 : 2);
}

// ---- sources and receivers in the rows a walk computes -------------------
// A walk meets the rows of an EntrySet in ascending order: `Cursor` is the
// next active row at or after the walk's position (INT_MAX when none).
struct Cursor {
  int a, row;
};
__device__ __forceinline__ Cursor cursor_at(const EntrySet &e, int s, int y0) {
  if (e.n == 0) return Cursor{0, 0x7fffffff};
  const int y = y0 < 0 ? 0 : y0 > e.ny ? e.ny : y0;
  const int2 c = __ldg(e.rcur + (int64_t)s * (e.ny + 1) + y);
  return Cursor{c.x, c.y};
}
__device__ __forceinline__ void cursor_next(const EntrySet &e, int s, Cursor &c) {
  ++c.a;
  c.row = __ldg(e.arow + (int64_t)s * (e.n + 1) + c.a);
}

// Fix-ups of one E row that the warp has just stored (row base `row`, the
// warp's stores made visible by __syncwarp): add vals_t[s][k] into the cells
// of the entries of active row c.a whose column lies in [lo, hi) -- the
// entries of one cell add up first, in index order, then join the field,
// like a serial loop over the duplicates -- or read those cells into
// out_t[s][k].  One lane per entry; every cell is owned by exactly one warp.
__device__ __forceinline__ void fix_inject(const EntrySet &e, int s, const Cursor &c,
                                           const float *vals_t, int lo, int hi, float *row,
                                           int lane) {
  const int *ab = e.abeg + (int64_t)s * (e.n + 1);
  const int j0 = __ldg(ab + c.a), j1 = __ldg(ab + c.a + 1);
  const int4 *en = e.ent + (int64_t)s * e.n;
  const float *vs = vals_t + (int64_t)s * e.n;
  for (int j = j0 + lane; j < j1; j += 32) {
    const int4 q = __ldg(en + j);
    if (q.w > 0 && q.y >= lo && q.y < hi) {
      float v = __ldg(vs + q.z);
      for (int u = 1; u < q.w; ++u) v += __ldg(vs + __ldg(en + j + u).z);
      row[q.y] += v;
    }
  }
}
__device__ __forceinline__ void fix_sample(const EntrySet &e, int s, const Cursor &c, float *out_t,
                                           int lo, int hi, const float *row, int lane) {
  const int *ab = e.abeg + (int64_t)s * (e.n + 1);
  const int j0 = __ldg(ab + c.a), j1 = __ldg(ab + c.a + 1);
  const int4 *en = e.ent + (int64_t)s * e.n;
  for (int j = j0 + lane; j < j1; j += 32) {
    const int4 q = __ldg(en + j);
    if (q.y >= lo && q.y < hi) out_t[(int64_t)s * e.n + q.z] = row[q.y];
  }
}
// The fix-ups of the E rows [ya, yb) of one item once its walk has stored
// them all (sources first, then receivers, row by row), in the columns
// [lo, hi) the item owns.  Outside the walk loop, so the walk's code is
// untouched by them.
__device__ __forceinline__ void fix_item(const StepArgs &a, int s, int ya, int yb, int lo, int hi,
                                         float *field, int nx, int lane, const float *vals_t,
                                         float *out_t) {
  Cursor ca = cursor_at(a.ea, s, ya), cb = cursor_at(a.eb, s, ya);
  while (ca.row < yb || cb.row < yb) {
    const int y = ca.row < cb.row ? ca.row : cb.row;
    float *row = field + (int64_t)y * nx;
    __syncwarp();
    if (y == ca.row) {
      if (vals_t) fix_inject(a.ea, s, ca, vals_t, lo, hi, row, lane);
      cursor_next(a.ea, s, ca);
      __syncwarp();
    }
    if (y == cb.row) {
      if (out_t) fix_sample(a.eb, s, cb, out_t, lo, hi, row, lane);
      cursor_next(a.eb, s, cb);
    }
  }
}

// Strip / chunk of one work item.
struct Item {
  int s, sm, x0, ya, yb, r0, n_it;
  int hx_lo, hx_hi;  // iterations whose H row r - P lies in the array and is needed
  bool xb;    // the strip (with its halo) touches an x band
  bool edge;  // the walk touches a band or the array's side edges
};

template <int P>
__device__ __forceinline__ bool make_item(const Geom &g, int item, bool batched, Item &it) {
  int strip, chunk;
  item_coords(g, item, &it.s, &strip, &chunk);
  it.sm = batched ? it.s : 0;
  it.x0 = strip * g.strip_cols;
  chunk_rows(g, chunk, &it.ya, &it.yb);
  it.r0 = it.ya - (2 * P - 1);
  it.n_it = (it.yb - it.ya) + 4 * P - 2;
  const bool near_x = it.x0 - 8 < g.Wx || it.x0 + g.strip_cols + 8 > g.nx - g.Wx;
  it.xb = g.Wx > 0 && near_x;
  it.edge = near_x || (g.Wz > 0 && (it.r0 < g.Wz || it.r0 + it.n_it > g.ny - g.Wz));
  it.hx_lo = max(it.ya - P, 0) - (it.r0 - P);
  it.hx_hi = min(it.yb + P - 2, g.ny - 1) - (it.r0 - P);
  return it.ya < it.yb;
}

// ---------------------------------------------------------------------------
// forward

// One warp's shared memory: stage barriers, the stage ring, the Hz ring.
struct FwdWarp {
  uint32_t bars, stage0, hring;
  uint32_t stage_bytes;
  uint32_t ca_o, cb_o;  // byte offsets of the Ca / Cb rows in a stage
  uint32_t dca_o, dcb_o;  // Born forward: byte offsets of the dCa / dCb rows
  int lane;
  Ring ring;
};

// Issue the loads of walk iteration i into stage `st` (lane 0 only): the
// rows are r (Ey, Hz; Cq), r - P (Hx; Cq, z-band memory of Hx) and
// y = r - 2P + 1 (Ca, Cb; band memories of E); the x-band memory of Hz is
// that of row r.  Rows outside the array read as zeros.
template <int P, bool BAND, int BORN>
__device__ __forceinline__ void fwd_issue(const FwdMaps &m, const StepArgs &a, const Item &it,
                                          int i, uint32_t st, uint32_t bar, int cq_arr) {
  const int r = it.r0 + i;
  const bool hx_in = i >= it.hx_lo && i <= it.hx_hi;
  const bool e_row = (unsigned)(i - (4 * P - 2)) < (unsigned)(it.yb - it.ya);
  uint32_t bytes = 2 * 136 * 4;
  if (hx_in) bytes += 120 * 4;
  if (e_row) bytes += 2 * 120 * 4;
  if (cq_arr) bytes += hx_in ? 2 * 128 * 4 : 128 * 4;
  int zh = -1, ze = -1;
  if constexpr (BAND) {
    if (hx_in) zh = zband_row(r - P, a.g.ny, a.g.Wz);
    if (e_row) ze = zband_row(r - 2 * P + 1, a.g.ny, a.g.Wz);
    if (zh >= 0) bytes += 120 * 4;
    if (ze >= 0) bytes += 120 * 4;
    if (it.xb) bytes += (uint32_t)a.band_box_floats * 4 * (e_row ? 2 : 1);
  }
  if constexpr (BORN != kStoreNone) {
    constexpr uint32_t be = BORN == kStoreF32 ? 4 : BORN == kStoreBF16 ? 2 : 1;
    if (e_row) bytes += 2 * 120 * 4 + 2 * 144 * be;
  }
  expect_tx_s(bar, bytes);
  fence_proxy_async();
  tma4s(st + kF_EY * 4, &m.map[kMapEH], it.x0 - 8, r, it.s, 0, bar);
  if constexpr (BORN != kStoreNone) {
    if (e_row) {  // dCa, dCb and the background's E, curl of row y at this step
      const int y = r - 2 * P + 1;
      if (a.bd_pair) {
        tma4s(st + a.fo[kFoBd] * 4, &m.map[kMapBD], it.x0, y, it.sm, 0, bar);
      } else {
        tma3s(st + a.fo[kFoBd] * 4, &m.map[kMapBD], it.x0, y, it.sm, bar);
        tma3s(st + (a.fo[kFoBd] + 128) * 4, &m.map[kMapBDB], it.x0, y, it.sm, bar);
      }
      // a 16-element boundary, so that a byte-sized row stays TMA-aligned
      const int xs = ((it.x0 - 4) >> 4) << 4;
      tma5s(st + a.fo[kFoBs] * 4, &m.map[kMapBS], xs, y, it.s, a.snap_t, 0, bar);
    }
  }
  if (hx_in) tma3s(st + kF_HX * 4, &m.map[kMapHX], it.x0, r - P, it.s, bar);
  if (e_row) {
    if (a.md_pair) {
      tma4s(st + kF_MD * 4, &m.map[kMapMD], it.x0, r - 2 * P + 1, it.sm, 0, bar);
    } else {
      tma3s(st + kF_MD * 4, &m.map[kMapMD], it.x0, r - 2 * P + 1, it.sm, bar);
      tma3s(st + (kF_MD + 128) * 4, &m.map[kMapCB], it.x0, r - 2 * P + 1, it.sm, bar);
    }
  }
  if (cq_arr) {
    tma3s(st + a.fo[kFoCqH] * 4, &m.map[kMapCQ], it.x0 - 4, r, it.sm, bar);
    if (hx_in) tma3s(st + a.fo[kFoCqX] * 4, &m.map[kMapCQ], it.x0 - 4, r - P, it.sm, bar);
  }
  if constexpr (BAND) {
    if (zh >= 0) tma3s(st + a.fo[kFoMzh] * 4, &m.map[kMapMZH], it.x0, zh, it.s, bar);
    if (ze >= 0) tma3s(st + a.fo[kFoMze] * 4, &m.map[kMapMZE], it.x0, ze, it.s, bar);
    if (it.xb) {
      tma3s(st + a.fo[kFoMxh] * 4, &m.map[kMapMXH], 0, r, it.s, bar);
      if (e_row) tma3s(st + a.fo[kFoMxe] * 4, &m.map[kMapMXE], 0, r - 2 * P + 1, it.s, bar);
    }
  }
}

// Give up after a wait timed out: flag it, let the copies in flight land.
template <int L>
__device__ __noinline__ void give_up_s(int *flags, uint32_t bars, Ring ring, int i, int n_it,
                                       int lane) {
  if (lane == 0) atomicOr(flags + kFlagTimeout, 1);
  for (int j = i; j < n_it && j <= i + L; ++j) {
    mbar_wait_s(bars + 8 * ring.slot, ring.phase);
    ring.next(L + 1);
  }
}

// Walk one item.  Per iteration: Hz of row r (owned rows), Hx of row r - P
// (every row, queued for the E update's z-stencil), E of row y = r - 2P + 1
// (owned rows); the row-range tests are warp-uniform, the per-lane ones only
// predicate stores.  BAND adds the CPML recursions and the array-edge masks
// that interior items do not need.
template <int P, int STORE, int L, bool BAND, int BORN>
__device__ __forceinline__ bool fwd_walk(const FwdMaps &m, const StepArgs &a, const Item &it,
                                         FwdWarp &w, int cq_arr, float cqs) {
  constexpr int NQ = 2 * P;
  constexpr int NS = L + 1;
  const int lane = w.lane;
  const int nx = a.g.nx;
  const int c = it.x0 - 4 + 4 * lane;
  const bool c_ok = !BAND || (c >= 0 && c < nx);
  const bool own_lane = lane >= 1 && lane <= 30;
  const bool own = own_lane && c_ok;
  const int wl = own_lane ? lane : 1;  // window base for the E update
  const int rows = it.yb - it.ya;
  const int64_t pb = (int64_t)it.s * a.g.numel + c;
  float *const hz_o = a.out.hz + pb;
  float *const hx_o = a.out.hx + pb;
  float *const ey_o = a.out.ey + pb;
  int ro = it.r0 * nx;  // r * nx of the running iteration
  // CPML band state of this lane / item
  const BandTab T{a.g.Wx, a.g.Wz};
  const int bcol = BAND ? xband_col(c, nx, a.g.Wx) : -1;
  const int64_t xbw = BAND ? (int64_t)it.s * a.g.ny * 2 * a.g.Wx + bcol : 0;
  const int64_t zbw = BAND ? (int64_t)it.s * 2 * a.g.Wz * nx + c : 0;

  {
    Ring pr = w.ring;
    for (int j = 0; j < L && j < it.n_it; ++j) {
      if (lane == 0)
        fwd_issue<P, BAND, BORN>(m, a, it, j, w.stage0 + pr.slot * w.stage_bytes, w.bars + 8 * pr.slot,
                           cq_arr);
      pr.next(NS);
    }
  }
  constexpr int M = walk_group<P, false>();
  using Q = Queue<NQ, M>;
  F4 eq[Q::kSize], hq[Q::kSize];
#pragma unroll
  for (int k = 0; k < Q::kSize; ++k) eq[k] = hq[k] = zero4();
  int ring0 = 0;  // Hz ring slot of the group's first iteration

  for (int i0 = 0; i0 < it.n_it; i0 += M) {
#pragma unroll
    for (int u = 0; u < M; ++u) {
      const int i = i0 + u;
      if (i < it.n_it) {
        if (i + L < it.n_it && lane == 0) {
          const int ps = w.ring.slot == 0 ? NS - 1 : w.ring.slot - 1;
          fwd_issue<P, BAND, BORN>(m, a, it, i + L, w.stage0 + ps * w.stage_bytes, w.bars + 8 * ps,
                             cq_arr);
        }
        if (!mbar_wait_s(w.bars + 8 * w.ring.slot, w.ring.phase)) {
          give_up_s<L>(a.flags, w.bars, w.ring, i, it.n_it, lane);
          return false;
        }
        const uint32_t st = w.stage0 + w.ring.slot * w.stage_bytes;
        const bool own_r = (unsigned)(i - (2 * P - 1)) < (unsigned)rows;
        const bool hx_own = (unsigned)(i - (3 * P - 1)) < (unsigned)rows;  // r - P in [ya, yb)
        const bool e_row = (unsigned)(i - (4 * P - 2)) < (unsigned)rows;
        const bool hx_in = i >= it.hx_lo && i <= it.hx_hi;

        // Ey of row r at this lane's column: the z-stencil queue (every row)
        eq[Q::at(u, 0)] = lds4s(st + (kF_EY + 4) * 4 + 16 * lane);
        // Hz ring slots: this row's, and that of row y = r - 2P + 1
        const int slot_w = M == NQ ? u : (ring0 + u < NQ ? ring0 + u : ring0 + u - NQ);
        const int slot_r = M == NQ ? (u + 1) % NQ
                                   : (ring0 + u + 1 < NQ ? ring0 + u + 1 : ring0 + u + 1 - NQ);

        // ---- Hz, row r: every lane, float4 at column c (owned rows only; the
        // E update reads the Hz of its own row)
        if (own_r) {
          float wv[12];
          {
            const F4 lo = lds4s(st + kF_EY * 4 + 16 * lane);
            const F4 hi = lds4s(st + (kF_EY + 8) * 4 + 16 * lane);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              wv[q] = lo.v[q];
              wv[q + 4] = eq[Q::at(u, 0)].v[q];
              wv[q + 8] = hi.v[q];
            }
          }
          const F4 hz_old = lds4s(st + (kF_HZ + 4) * 4 + 16 * lane);
          const F4 cq = cq_arr ? lds4s(st + a.fo[kFoCqH] * 4 + 16 * lane) : splat4(cqs);
          F4 hn;
          if (!BAND || bcol < 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(cq.v[q], d_half<P>(wv, q, a.c.cx), hz_old.v[q]);
          } else {
            F4 mn = lds4s(st + (a.fo[kFoMxh] + bcol) * 4);
            const F4 ah = ld4(a.bt + T.x(3) + bcol), bh = ld4(a.bt + T.x(4) + bcol);
            const F4 rk = ld4(a.bt + T.x(5) + bcol);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float d = d_half<P>(wv, q, a.c.cx);
              mn.v[q] = fmaf(bh.v[q], mn.v[q], ah.v[q] * d);
              hn.v[q] = fmaf(cq.v[q], fmaf(d, rk.v[q], mn.v[q]), hz_old.v[q]);
            }
            st4p(own, a.out.mxh_node + xbw + (int64_t)(it.r0 + i) * 2 * a.g.Wx, mn);
          }
          sts4s(w.hring + slot_w * kFRing * 4 + 16 * lane, c_ok ? hn : zero4());
          st4p(own, hz_o + ro, hn);
        }

        // ---- Hx, row r - P (z-stencil from the Ey queue)
        {
          const F4 hx_old = lds4s(st + (kF_HX - 4) * 4 + 16 * lane);
          const F4 cq = cq_arr ? lds4s(st + a.fo[kFoCqX] * 4 + 16 * lane) : splat4(cqs);
          F4 d;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float s = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              s = fmaf(a.c.cy[k - 1],
                       eq[Q::at(u, P - k)].v[q] - eq[Q::at(u, P + k - 1)].v[q], s);
            d.v[q] = s;
          }
          if constexpr (BAND) {
            const int zr = hx_in ? zband_row(it.r0 + i - P, a.g.ny, a.g.Wz) : -1;
            if (zr >= 0) {
              F4 mz = lds4s(st + (a.fo[kFoMzh] - 4) * 4 + 16 * lane);
              const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
              const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(byh, mz.v[q], ayh * d.v[q]);
                d.v[q] = fmaf(d.v[q], rkyh, mz.v[q]);
              }
              st4p(own && hx_own, a.out.mzh_node + zbw + (int64_t)zr * nx, mz);
            }
          }
          F4 hn;
#pragma unroll
          for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(-cq.v[q], d.v[q], hx_old.v[q]);
          hq[Q::at(u, 0)] = hx_in ? hn : zero4();
          st4p(own && hx_own, hx_o + (ro - P * nx), hn);
        }

        // ---- E, row y = r - 2P + 1
        if (e_row) {
          float wv[12];
          win12s(w.hring + slot_r * kFRing * 4 + 16 * wl - 16, wv);
          const F4 ca4 = lds4s(st + w.ca_o + 16 * lane - 16);
          const F4 cb4 = lds4s(st + w.cb_o + 16 * lane - 16);
          const F4 &e_old = eq[Q::at(u, NQ - 1)];
          F4 cx, cz;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            cx.v[q] = d_int<P>(wv, q, a.c.cx);
            float s = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              s = fmaf(a.c.cy[k - 1], hq[Q::at(u, P - k)].v[q] - hq[Q::at(u, P - 1 + k)].v[q], s);
            cz.v[q] = s;
          }
          if constexpr (BAND) {
            const int y = it.r0 + i - 2 * P + 1;
            if (bcol >= 0) {
              F4 mx = lds4s(st + (a.fo[kFoMxe] + bcol) * 4);
              const F4 ax = ld4(a.bt + T.x(0) + bcol), bx = ld4(a.bt + T.x(1) + bcol);
              const F4 rk = ld4(a.bt + T.x(2) + bcol);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mx.v[q] = fmaf(bx.v[q], mx.v[q], ax.v[q] * cx.v[q]);
                cx.v[q] = fmaf(cx.v[q], rk.v[q], mx.v[q]);
              }
              st4p(own, a.out.mxe_node + xbw + (int64_t)y * 2 * a.g.Wx, mx);
            }
            const int zr = e_row ? zband_row(y, a.g.ny, a.g.Wz) : -1;
            if (zr >= 0) {
              F4 mz = lds4s(st + (a.fo[kFoMze] - 4) * 4 + 16 * lane);
              const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
              const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(by, mz.v[q], ay * cz.v[q]);
                cz.v[q] = fmaf(cz.v[q], rky, mz.v[q]);
              }
              st4p(own, a.out.mze_node + zbw + (int64_t)zr * nx, mz);
            }
          }
          F4 curl, en;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            curl.v[q] = cx.v[q] - cz.v[q];
            en.v[q] = fmaf(ca4.v[q], e_old.v[q], cb4.v[q] * curl.v[q]);
          }
          if constexpr (BORN != kStoreNone) {
            // linearised step: + dCa E0 + dCb curl0 (the background's values)
            constexpr uint32_t be = BORN == kStoreF32 ? 4 : BORN == kStoreBF16 ? 2 : 1;
            const F4 dca4 = lds4s(st + w.dca_o + 16 * lane - 16);
            const F4 dcb4 = lds4s(st + w.dcb_o + 16 * lane - 16);
            const uint32_t sb = st + a.fo[kFoBs] * 4 + (((it.x0 - 4) & 15) + 4 * lane) * be;
            const F4 e0 = snap_lds_s<BORN>(sb), c0 = snap_lds_s<BORN>(sb + 144 * be);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              en.v[q] += fmaf(dcb4.v[q], c0.v[q], dca4.v[q] * e0.v[q]);
          }
          {
            const int off = ro - (2 * P - 1) * nx;
            if constexpr (STORE != kStoreNone) {
              const int64_t so = ((int64_t)it.s * a.g.ny + (it.r0 + i - 2 * P + 1)) * a.snap_pitch + c;
              snap_store_p<STORE>(own, a.snap_e, so, e_old);
              if constexpr (STORE != kStoreEy) snap_store_p<STORE>(own, a.snap_c, so, curl);
            }
            st4p(own, ey_o + off, en);
          }
        }
        __syncwarp();
        w.ring.next(NS);
        ro += nx;
      }
    }
    shift_queue<NQ, M>(eq);
    shift_queue<NQ, M>(hq);
    if constexpr (M != NQ) ring0 = ring0 + M < NQ ? ring0 + M : ring0 + M - NQ;
  }
  return true;
}

template <int P, int STORE, int L, int BORN>
__global__ void __launch_bounds__(128, BORN != kStoreNone ? 3 : (P <= 3 ? 5 : 4))
    k_forward(const __grid_constant__ FwdMaps m,
                                                 const StepArgs a, const int batched,
                                                 const int cq_arr) {
  constexpr int NS = L + 1;
  (void)sizeof(Stages<L>);
  extern __shared__ __align__(128) float smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 127u) & ~127u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  FwdWarp w;
  w.lane = lane;
  w.bars = base + warp * NS * 8;
  w.stage_bytes = (uint32_t)a.stage_floats * 4;
  w.stage0 = base + 128 + warp * a.warp_floats * 4;
  w.hring = w.stage0 + NS * w.stage_bytes;  // Hz ring: 2P rows of 32 float4
  // pair box: [Ca][Cb] (or [Cb][Ca] when Cb lies first), 120 floats each;
  // two boxes: Ca at kF_MD, Cb at kF_MD + 128 (every box starts 128-aligned)
  w.ca_o = (kF_MD + (a.md_pair && a.md_swap ? 120 : 0)) * 4;
  w.cb_o = (kF_MD + (a.md_pair ? (a.md_swap ? 0 : 120) : 128)) * 4;
  w.dca_o = w.dcb_o = 0;
  if constexpr (BORN != kStoreNone) {
    w.dca_o = (a.fo[kFoBd] + (a.bd_pair && a.bd_swap ? 120 : 0)) * 4;
    w.dcb_o = (a.fo[kFoBd] + (a.bd_pair ? (a.bd_swap ? 0 : 120) : 128)) * 4;
  }
  w.ring = Ring{0, 0u};
  const Geom &g = a.g;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  grid_dep_launch();
  if (lane == 0) {
    for (int k = 0; k < NS; ++k)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(w.bars + 8 * k), "r"(1)
                   : "memory");
    fence_mbar_init();
  }
  __syncwarp();
  grid_dep_wait();  // everything below reads what earlier kernels wrote
  if (__any_sync(kFull, *reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0)) return;
  const float cqs = cq_arr ? 0.f : __ldg(a.cq);
  // work items are claimed dynamically; the counter of the next launch is
  // reset here (the previous launch that used it has completed)
  int *ctr = a.flags + kCtrBase + a.ctr_slot;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.flags[kCtrBase + (a.ctr_slot ^ 1)] = 0;

  for (;;) {
    int item = 0;
    if (lane == 0) item = atomicAdd(ctr, 1);
    item = __shfl_sync(kFull, item, 0);
    if (item >= n_items) break;
    Item it;
    if (!make_item<P>(g, item, batched != 0, it)) continue;
    const bool ok = it.edge ? fwd_walk<P, STORE, L, true, BORN>(m, a, it, w, cq_arr, cqs)
                            : fwd_walk<P, STORE, L, false, BORN>(m, a, it, w, cq_arr, cqs);
    if (!ok) return;
    // this step's sources, then its receivers, in the item's cells
    fix_item(a, it.s, it.ya, it.yb, it.x0, min(it.x0 + g.strip_cols, g.nx),
             a.out.ey + (int64_t)it.s * g.numel, g.nx, lane, a.vals_t, a.out_t);
  }
}

// ---------------------------------------------------------------------------
// adjoint

struct AdjWarp {
  uint32_t bars, stage0, prow, qring;
  uint32_t stage_bytes;
  uint32_t ca_o, cb_o, gca_o, gcb_o;  // byte offsets within a stage
  int lane;
  Ring ring;
};

// Issue the loads of walk iteration i (lane 0 only): row r = r0 + i for
// lambda_E / lambda_Hz, Ca / Cb, Cq, the snapshots, the gradients and the
// band memories of the E nodes and (x band) H nodes; row r - P for
// lambda_Hx, its Cq and its z-band memory.  With the E snapshot alone
// (kStoreEy) row r brings Cb only, and Ca, the E snapshot and the gradients
// come for row r - 2P + 1, whose E update this iteration makes.  Rows
// outside the array read as zeros.
template <int P, int SNAP, bool BAND>
__device__ __forceinline__ void adj_issue(const AdjMaps &m, const StepArgs &a, const Item &it,
                                          int i, uint32_t st, uint32_t bar, int cq_arr) {
  const int r = it.r0 + i;
  const bool own_r = (unsigned)(i - (2 * P - 1)) < (unsigned)(it.yb - it.ya);
  const bool hx_in = i >= it.hx_lo && i <= it.hx_hi;
  constexpr bool EY = SNAP == kStoreEy;
  constexpr uint32_t snap_elem = SNAP == kStoreF32 || EY ? 4 : SNAP == kStoreBF16 ? 2 : 1;
  constexpr uint32_t snap_bytes = EY ? 2 * 112 * 4 : 2 * 112 * snap_elem;
  // the gradient rows: this row's (snapshot pair), or with the E snapshot
  // alone that of row r - 2P + 1, whose E update this iteration makes
  // (lambda_E and the E snapshot)
  const bool g_r = EY ? (unsigned)(i - (4 * P - 2)) < (unsigned)(it.yb - it.ya) : own_r;
  const int rg = EY ? r - 2 * P + 1 : r;
  uint32_t bytes = 2 * 128 * 4 + (EY ? 128 * 4 : 2 * 128 * 4);
  if (hx_in) bytes += 112 * 4;
  if (g_r) bytes += snap_bytes + 2 * 112 * 4;
  if (cq_arr) bytes += hx_in ? 2 * 128 * 4 : 128 * 4;
  int ze = -1, zh = -1;
  if constexpr (BAND) {
    ze = zband_row(r, a.g.ny, a.g.Wz);
    if (hx_in) zh = zband_row(r - P, a.g.ny, a.g.Wz);
    if (ze >= 0) bytes += 112 * 4;
    if (zh >= 0) bytes += 112 * 4;
    if (own_r && it.xb) bytes += 2 * (uint32_t)a.band_box_floats * 4;
  }
  expect_tx_s(bar, bytes);
  fence_proxy_async();
  tma4s(st + kA_EH * 4, &m.map[kAMapEH], it.x0 - 8, r, it.s, 0, bar);
  if constexpr (EY) {
    tma3s(st + kA_MD * 4, &m.map[kAMapCB], it.x0 - 8, r, it.sm, bar);
  } else if (a.md_pair) {
    tma4s(st + kA_MD * 4, &m.map[kAMapMD], it.x0 - 8, r, it.sm, 0, bar);
  } else {
    tma3s(st + kA_MD * 4, &m.map[kAMapMD], it.x0 - 8, r, it.sm, bar);
    tma3s(st + (kA_MD + 128) * 4, &m.map[kAMapCB], it.x0 - 8, r, it.sm, bar);
  }
  if (hx_in) tma3s(st + kA_HX * 4, &m.map[kAMapHX], it.x0, r - P, it.s, bar);
  if (g_r) {
    if constexpr (EY) {
      tma3s(st + kA_SS * 4, &m.map[kAMapCA], it.x0, rg, it.sm, bar);
      tma4s(st + (kA_SS + 128) * 4, &m.map[kAMapSS], it.x0, rg, it.s, a.snap_t, bar);
    } else {
      tma5s(st + kA_SS * 4, &m.map[kAMapSS], it.x0, rg, it.s, a.snap_t, 0, bar);
    }
    if (a.gg_pair) {
      tma4s(st + kA_GG * 4, &m.map[kAMapGG], it.x0, rg, it.s, 0, bar);
    } else {
      tma3s(st + kA_GG * 4, &m.map[kAMapGG], it.x0, rg, it.s, bar);
      tma3s(st + (kA_GG + 128) * 4, &m.map[kAMapGB], it.x0, rg, it.s, bar);
    }
  }
  if (cq_arr) {
    tma3s(st + a.ao[kAoCqR] * 4, &m.map[kAMapCQ], it.x0 - 8, r, it.sm, bar);
    if (hx_in) tma3s(st + a.ao[kAoCqH] * 4, &m.map[kAMapCQ], it.x0 - 8, r - P, it.sm, bar);
  }
  if constexpr (BAND) {
    if (ze >= 0) tma3s(st + a.ao[kAoMze] * 4, &m.map[kAMapMZE], it.x0, ze, it.s, bar);
    if (zh >= 0) tma3s(st + a.ao[kAoMzh] * 4, &m.map[kAMapMZH], it.x0, zh, it.s, bar);
    if (own_r && it.xb) tma4s(st + a.ao[kAoMx] * 4, &m.map[kAMapMX], 0, r, it.s, 0, bar);
  }
}

// Walk one item of the adjoint.  Per iteration (row r = r0 + i):
//   g = Cb lam, Ca lam (queued for the E update of this row), pz (every
//   row, queued for the z-stencil); on owned rows the gradients, px and then
//   lamHz and qx; lamHx and qz of row r - P; lamE of row r - 2P + 1.
// Lanes: 0..31 hold the float4 at x0 - 8 + 4 lane (g, px, pz; lanes 2..29
// own theirs), lanes 0..29 the qx float4 at x0 - 4 + 4 lane.
template <int P, int SNAP, int L, bool BAND>
__device__ __forceinline__ bool adj_walk(const AdjMaps &m, const StepArgs &a, const Item &it,
                                         AdjWarp &w, int cq_arr, float cqs) {
  constexpr int NQ = 2 * P;
  constexpr int NS = L + 1;
  const int lane = w.lane;
  const int nx = a.g.nx, ny = a.g.ny;
  const bool own_lane = lane >= 2 && lane <= 29;  // owned float4 o = lane - 2
  const bool q_lane = lane <= 29;
  const int wq = q_lane ? lane : 0;        // px window base (lanes 30, 31 idle)
  const int wo = own_lane ? lane - 2 : 0;  // qx window base of the E update
  const int pc = it.x0 - 8 + 4 * lane;
  const int qc = it.x0 - 4 + 4 * lane;
  const bool pc_ok = !BAND || (pc >= 0 && pc < nx);
  const bool qc_ok = q_lane && (!BAND || (qc >= 0 && qc < nx));
  const bool own = own_lane && pc_ok;
  const bool q_own = lane >= 1 && lane <= 28 && qc_ok;
  const int rows = it.yb - it.ya;
  const int64_t sp = (int64_t)it.s * a.g.numel + pc;
  float *const hz_o = a.out.hz + (sp + 4);
  float *const hx_o = a.out.hx + sp;
  float *const ey_o = a.out.ey + sp;
  float *const gca_o = a.gca + sp;
  float *const gcb_o = a.gcb + sp;
  int ro = it.r0 * nx;
  const BandTab T{a.g.Wx, a.g.Wz};
  const int pb = BAND ? xband_col(pc, nx, a.g.Wx) : -1;
  const int qb = BAND && q_lane ? xband_col(qc, nx, a.g.Wx) : -1;
  const int64_t xw = BAND ? (int64_t)it.s * ny * 2 * a.g.Wx : 0;
  const int64_t zbw = BAND ? (int64_t)it.s * 2 * a.g.Wz * nx + pc : 0;
  bool colmask[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    colmask[q] = !BAND || !a.g.grad_mask || (pc + q >= a.g.n_pml && pc + q < nx - a.g.n_pml);

  {
    Ring pr = w.ring;
    for (int j = 0; j < L && j < it.n_it; ++j) {
      if (lane == 0)
        adj_issue<P, SNAP, BAND>(m, a, it, j, w.stage0 + pr.slot * w.stage_bytes,
                                 w.bars + 8 * pr.slot, cq_arr);
      pr.next(NS);
    }
  }
  constexpr int M = walk_group<P, true>();
  using Q = Queue<NQ, M>;
  F4 pq[Q::kSize], qq[Q::kSize], cl[Q::kSize];
#pragma unroll
  for (int k = 0; k < Q::kSize; ++k) pq[k] = qq[k] = cl[k] = zero4();
  int ring0 = 0;  // qx ring slot of the group's first iteration

  for (int i0 = 0; i0 < it.n_it; i0 += M) {
#pragma unroll
    for (int u = 0; u < M; ++u) {
      const int i = i0 + u;
      if (i < it.n_it) {
        if (i + L < it.n_it && lane == 0) {
          const int ps = w.ring.slot == 0 ? NS - 1 : w.ring.slot - 1;
          adj_issue<P, SNAP, BAND>(m, a, it, i + L, w.stage0 + ps * w.stage_bytes,
                                   w.bars + 8 * ps, cq_arr);
        }
        if (!mbar_wait_s(w.bars + 8 * w.ring.slot, w.ring.phase)) {
          give_up_s<L>(a.flags, w.bars, w.ring, i, it.n_it, lane);
          return false;
        }
        const uint32_t st = w.stage0 + w.ring.slot * w.stage_bytes;
        // qx ring slots: this row's, and that of row r - 2P + 1
        const int slot_w = M == NQ ? u : (ring0 + u < NQ ? ring0 + u : ring0 + u - NQ);
        const int slot_r = M == NQ ? (u + 1) % NQ
                                   : (ring0 + u + 1 < NQ ? ring0 + u + 1 : ring0 + u + 1 - NQ);
        const int r = it.r0 + i;
        const bool own_r = (unsigned)(i - (2 * P - 1)) < (unsigned)rows;
        const bool hx_own = (unsigned)(i - (3 * P - 1)) < (unsigned)rows;  // r - P in [ya, yb)
        const bool e_row = (unsigned)(i - (4 * P - 2)) < (unsigned)rows;
        const bool hx_in = i >= it.hx_lo && i <= it.hx_hi;

        const F4 lam = lds4s(st + kA_EH * 4 + 16 * lane);
        const F4 cbv = lds4s(st + w.cb_o + 16 * lane);
        F4 gv;
        if constexpr (SNAP == kStoreEy) {  // lambda_E itself goes to the E update
#pragma unroll
          for (int q = 0; q < 4; ++q) gv.v[q] = cbv.v[q] * lam.v[q];
          cl[Q::at(u, 0)] = lam;
        } else {
          const F4 cav = lds4s(st + w.ca_o + 16 * lane);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            gv.v[q] = cbv.v[q] * lam.v[q];
            cl[Q::at(u, 0)].v[q] = cav.v[q] * lam.v[q];
          }
        }
        // ---- pz at E nodes (every row; owned lanes matter)
        {
          F4 pz;
#pragma unroll
          for (int q = 0; q < 4; ++q) pz.v[q] = -gv.v[q];
          if constexpr (BAND) {
            const int zr = zband_row(r, ny, a.g.Wz);
            if (zr >= 0) {
              F4 M = lds4s(st + (a.ao[kAoMze] - 8) * 4 + 16 * lane);
              const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
              const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                M.v[q] -= gv.v[q];
                pz.v[q] = fmaf(ay, M.v[q], -gv.v[q] * rky);
                M.v[q] *= by;
              }
              st4p(own && own_r, a.out.mze_node + zbw + (int64_t)zr * nx, M);
            }
          }
          pq[Q::at(u, 0)] = pz;
        }
        // ---- owned rows: gradients (lam = lambda_E^{t+1}) and px
        if (own_r) {
          if constexpr (SNAP != kStoreEy) {  // every lane computes; owned lanes store
            const uint32_t sbase = st + kA_SS * 4;
            constexpr uint32_t selem = SNAP == kStoreF32 ? 4 : SNAP == kStoreBF16 ? 2 : 1;
            constexpr uint32_t sfield = 112 * selem, sstep = 4 * selem;
            const F4 se = snap_lds_s<SNAP>(sbase + sstep * wo);
            const F4 sc = snap_lds_s<SNAP>(sbase + sfield + sstep * wo);
            F4 gca = lds4s(st + w.gca_o + 16 * wo), gcb = lds4s(st + w.gcb_o + 16 * wo);
            const bool rowmask = !BAND || !a.g.grad_mask || (r >= a.g.n_pml && r < ny - a.g.n_pml);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (rowmask && colmask[q]) {
                gca.v[q] = fmaf(se.v[q], lam.v[q], gca.v[q]);
                gcb.v[q] = fmaf(sc.v[q], lam.v[q], gcb.v[q]);
              }
            }
            st4p(own, gca_o + ro, gca);
            st4p(own, gcb_o + ro, gcb);
          }
          F4 px = gv;
          if constexpr (BAND) {
            if (pb >= 0) {
              F4 M = lds4s(st + (a.ao[kAoMx] + a.band_box_floats + pb) * 4);
              const F4 ax = ld4(a.bt + T.x(0) + pb), bx = ld4(a.bt + T.x(1) + pb);
              const F4 rk = ld4(a.bt + T.x(2) + pb);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                M.v[q] += gv.v[q];
                px.v[q] = fmaf(ax.v[q], M.v[q], gv.v[q] * rk.v[q]);
                M.v[q] *= bx.v[q];
              }
              st4p(own, a.out.mxe_node + xw + (int64_t)r * 2 * a.g.Wx + pb, M);
            }
          }
          sts4s(w.prow + 16 * lane, pc_ok ? px : zero4());
        }
        __syncwarp();

        // ---- owned rows: lamHz and qx (lanes 0..29)
        if (own_r) {
          float wv[12];
          win12s(w.prow + 16 * wq, wv);
          const F4 lhz_old = lds4s(st + (kA_EH + 128 + 4) * 4 + 16 * wq);
          const F4 cq = cq_arr ? lds4s(st + (a.ao[kAoCqR] + 4) * 4 + 16 * wq) : splat4(cqs);
          F4 lhz, v;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            lhz.v[q] = lhz_old.v[q] - d_half<P>(wv, q, a.c.cx);
            v.v[q] = cq.v[q] * lhz.v[q];
          }
          st4p(q_own, hz_o + ro, lhz);
          if constexpr (BAND) {
            if (qb >= 0) {
              F4 M = lds4s(st + (a.ao[kAoMx] + qb) * 4);
              const F4 ah = ld4(a.bt + T.x(3) + qb), bh = ld4(a.bt + T.x(4) + qb);
              const F4 rk = ld4(a.bt + T.x(5) + qb);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                M.v[q] += v.v[q];
                const float vq = v.v[q];
                v.v[q] = fmaf(ah.v[q], M.v[q], vq * rk.v[q]);
                M.v[q] *= bh.v[q];
              }
              st4p(q_own, a.out.mxh_node + xw + (int64_t)r * 2 * a.g.Wx + qb, M);
            }
          }
          sts4p(q_lane, w.qring + slot_w * kARing * 4 + 16 * lane, qc_ok ? v : zero4());
        }

        // ---- lamHx and qz of row r - P (owned lanes)
        {
          const F4 lhx = lds4s(st + (kA_HX - 8) * 4 + 16 * lane);
          const F4 cq = cq_arr ? lds4s(st + a.ao[kAoCqH] * 4 + 16 * lane) : splat4(cqs);
          F4 lh, qz;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float d = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              d = fmaf(a.c.cy[k - 1],
                       pq[Q::at(u, P - k)].v[q] - pq[Q::at(u, P + k - 1)].v[q], d);
            lh.v[q] = lhx.v[q] - d;
            qz.v[q] = -cq.v[q] * lh.v[q];
          }
          st4p(own && hx_own, hx_o + (ro - P * nx), lh);
          if constexpr (BAND) {
            const int zr = hx_in ? zband_row(r - P, ny, a.g.Wz) : -1;
            if (zr >= 0) {
              F4 M = lds4s(st + (a.ao[kAoMzh] - 8) * 4 + 16 * lane);
              const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
              const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float vq = qz.v[q];
                M.v[q] += vq;
                qz.v[q] = fmaf(ayh, M.v[q], vq * rkyh);
                M.v[q] *= byh;
              }
              st4p(own && hx_own, a.out.mzh_node + zbw + (int64_t)zr * nx, M);
            }
          }
          qq[Q::at(u, 0)] = hx_in ? qz : zero4();
        }

        // ---- lamE of row r - 2P + 1 (owned lanes)
        if (e_row) {
          float wv[12];
          win12s(w.qring + slot_r * kARing * 4 + 16 * wo, wv);
          // Ca lam^{t+1} of this row: queued, or (kStoreEy) formed here from
          // the queued lambda_E and the row's Ca
          F4 cla = cl[Q::at(u, NQ - 1)];
          if constexpr (SNAP == kStoreEy) {
            const F4 ca_e = lds4s(st + kA_SS * 4 + 16 * wo);
#pragma unroll
            for (int q = 0; q < 4; ++q) cla.v[q] = ca_e.v[q] * cla.v[q];
          }
          F4 en;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float dz = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              dz = fmaf(a.c.cy[k - 1], qq[Q::at(u, P - k)].v[q] - qq[Q::at(u, P - 1 + k)].v[q],
                        dz);
            en.v[q] = cla.v[q] - d_int<P>(wv, q, a.c.cx) - dz;
          }
          st4p(own, ey_o + (ro - (2 * P - 1) * nx), en);
          if constexpr (SNAP == kStoreEy) {
            // gradients of this row by summation by parts: gCa += E^t lam^{t+1};
            // the Cb accumulator takes E^t times the E-update term
            // G^t = lam~^t - Ca lam^{t+1} (at t = 0: E^0 times -Ca lam^1)
            const int re = r - 2 * P + 1;
            const F4 lv = cl[Q::at(u, NQ - 1)];
            const F4 se = lds4s(st + (kA_SS + 128) * 4 + 16 * wo);
            F4 gca = lds4s(st + w.gca_o + 16 * wo), gcb = lds4s(st + w.gcb_o + 16 * wo);
            const bool rowmask =
                !BAND || !a.g.grad_mask || (re >= a.g.n_pml && re < ny - a.g.n_pml);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (rowmask && colmask[q]) {
                const float c = cla.v[q];
                gca.v[q] = fmaf(se.v[q], lv.v[q], gca.v[q]);
                gcb.v[q] = fmaf(se.v[q], a.tzero ? -c : en.v[q] - c, gcb.v[q]);
              }
            }
            const int go = ro - (2 * P - 1) * nx;
            st4p(own, gca_o + go, gca);
            st4p(own, gcb_o + go, gcb);
          }
        }
        __syncwarp();
        w.ring.next(NS);
        ro += nx;
      }
    }
    shift_queue<NQ, M>(pq);
    shift_queue<NQ, M>(qq);
    shift_queue<NQ, M>(cl);
    if constexpr (M != NQ) ring0 = ring0 + M < NQ ? ring0 + M : ring0 + M - NQ;
  }
  return true;
}

template <int P, int SNAP, int L>
__global__ void __launch_bounds__(32 * adj_warps_per_cta(P)) k_adjoint(const __grid_constant__ AdjMaps m,
                                                                  const StepArgs a,
                                                                  const int batched,
                                                                  const int cq_arr) {
  constexpr int NS = L + 1;
  (void)sizeof(Stages<L>);
  extern __shared__ __align__(128) float smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 127u) & ~127u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AdjWarp w;
  w.lane = lane;
  w.bars = base + warp * NS * 8;
  w.stage_bytes = (uint32_t)a.stage_floats * 4;
  w.stage0 = base + 128 + warp * a.warp_floats * 4;
  w.prow = w.stage0 + NS * w.stage_bytes;  // px row: 32 float4
  w.qring = w.prow + kAPx * 4;             // qx ring: 2P rows of 30 float4
  // pair boxes: [Ca][Cb] / [gCa][gCb], or the other order when the second
  // array lies first; single boxes at 128-float slots
  w.ca_o = (kA_MD + (a.md_pair && a.md_swap ? 128 : 0)) * 4;
  w.cb_o = (kA_MD + (a.md_pair && a.md_swap ? 0 : 128)) * 4;
  if constexpr (SNAP == kStoreEy) w.cb_o = kA_MD * 4;  // Cb alone
  w.gca_o = (kA_GG + (a.gg_pair && a.gg_swap ? 112 : 0)) * 4;
  w.gcb_o = (kA_GG + (a.gg_pair ? (a.gg_swap ? 0 : 112) : 128)) * 4;
  w.ring = Ring{0, 0u};
  const Geom &g = a.g;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  grid_dep_launch();
  if (lane == 0) {
    for (int k = 0; k < NS; ++k)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(w.bars + 8 * k), "r"(1)
                   : "memory");
    fence_mbar_init();
  }
  __syncwarp();
  grid_dep_wait();  // everything below reads what earlier kernels wrote
  if (__any_sync(kFull, *reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0)) return;
  const float cqs = cq_arr ? 0.f : __ldg(a.cq);
  int *ctr = a.flags + kCtrBase + a.ctr_slot;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.flags[kCtrBase + (a.ctr_slot ^ 1)] = 0;

  for (;;) {
    int item = 0;
    if (lane == 0) item = atomicAdd(ctr, 1);
    item = __shfl_sync(kFull, item, 0);
    if (item >= n_items) break;
    Item it;
    if (!make_item<P>(g, item, batched != 0, it)) continue;
    const bool ok = it.edge ? adj_walk<P, SNAP, L, true>(m, a, it, w, cq_arr, cqs)
                            : adj_walk<P, SNAP, L, false>(m, a, it, w, cq_arr, cqs);
    if (!ok) return;
    // the next step's residuals, then its source gradient, in the item's cells
    fix_item(a, it.s, it.ya, it.yb, it.x0, min(it.x0 + g.strip_cols, g.nx),
             a.out.ey + (int64_t)it.s * g.numel, g.nx, lane, a.vals_t, a.out_t);
  }
}

// ---------------------------------------------------------------------------
// two-step forward (temporal blocking): steps t and t + 1 in one walk, so the
// state is read and written once per two steps.
//
// Iteration i of an item's walk (row r = r0 + i) stages row r of Ey (step-t
// input), row y1 = r - 2P + 1 of Hz, row h1 = r - P of Hx and the Ca / Cb rows
// of the two E updates, and computes
//   step t:      Hx1(h1), then Hz1(y1) and E1(y1)
//   step t + 1:  Hx2(y1 - P), then Hz2(y2) and E2(y2), y2 = y1 - 2P + 1.
// Lane l holds the float4 at column xb + 4l, xb = x0 - H; every x window comes
// from the neighbouring lanes (shuffles), so each level loses a few columns
// at the warp's edges and the halo H covers the 4P - 2 columns that two
// steps consume on each side.  Register queues of 2P rows hold Ey, Hx1, E1,
// Hx2 (the z-stencils) and Hz1 (Hz2 starts from it 2P - 1 rows later); band
// items carry the step-t CPML memories to step t + 1 in per-warp shared
// rings.  Every update is that of k_forward, operation for operation, so the
// two steps give the bits two k_forward launches give.

// stage slots (floats): Ey row r, Hz row y1, Hx row h1, Ca / Cb rows y1 and
// y2 (pairs of 128); the band slots follow at host-given offsets
constexpr int kF2_E = 0, kF2_HZ = 128, kF2_HX = 256, kF2_MD1 = 384, kF2_MD2 = 640,
              kF2_FIXED = 896;

// x window w[0..12) of columns c - 4 .. c + 8 (c this lane's first column)
// from lanes l - 1, l, l + 1; only the entries [LO, HI] the stencil reads.
template <int LO, int HI>
__device__ __forceinline__ void win_lanes(const F4 &v, float w[12]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[4 + j] = v.v[j];
    w[j] = j >= LO ? __shfl_up_sync(kFull, v.v[j], 1) : 0.f;
    w[8 + j] = 8 + j <= HI ? __shfl_down_sync(kFull, v.v[j], 1) : 0.f;
  }
}

// Sources of active row c.a added into the float4 v of every lane whose
// columns [xb + 4l, xb + 4l + 4) hold one (entries of one cell added up first,
// in index order).  A serial loop: source rows hold few entries.
__device__ __forceinline__ void inject_lanes(const EntrySet &e, int s, const Cursor &c,
                                             const float *vals_t, int xb, int lane, F4 &v) {
  const int *ab = e.abeg + (int64_t)s * (e.n + 1);
  const int j0 = __ldg(ab + c.a), j1 = __ldg(ab + c.a + 1);
  const int4 *en = e.ent + (int64_t)s * e.n;
  const float *vs = vals_t + (int64_t)s * e.n;
  for (int j = j0; j < j1; ++j) {
    const int4 q = __ldg(en + j);
    const int d = q.y - xb;
    if (q.w == 0 || d < 0 || d >= 128) continue;
    float val = __ldg(vs + q.z);
    for (int u = 1; u < q.w; ++u) val += __ldg(vs + __ldg(en + j + u).z);
    if (lane == (d >> 2)) {
      const int k = d & 3;
      if (k == 0) v.v[0] += val;
      else if (k == 1) v.v[1] += val;
      else if (k == 2) v.v[2] += val;
      else v.v[3] += val;
    }
  }
}
// Receivers of active row c.a in the columns [lo, hi): the warp's row v goes
// to the shared row `buf` (xb at offset 0), then one lane per entry reads it.
__device__ __forceinline__ void sample_lanes(const EntrySet &e, int s, const Cursor &c,
                                             float *out_t, int xb, int lo, int hi, uint32_t buf,
                                             int lane, const F4 &v) {
  sts4s(buf + 16 * lane, v);
  __syncwarp();
  const int *ab = e.abeg + (int64_t)s * (e.n + 1);
  const int j0 = __ldg(ab + c.a), j1 = __ldg(ab + c.a + 1);
  const int4 *en = e.ent + (int64_t)s * e.n;
  for (int j = j0 + lane; j < j1; j += 32) {
    const int4 q = __ldg(en + j);
    if (q.y >= lo && q.y < hi) {
      float x;
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(x) : "r"(buf + 4u * (uint32_t)(q.y - xb)) : "memory");
      out_t[(int64_t)s * e.n + q.z] = x;
    }
  }
  __syncwarp();
}

template <int P>
__device__ __forceinline__ bool make_item2(const Geom &g, int item, bool batched, Item &it) {
  constexpr int H = fwd2_halo(P), W = fwd2_width(P);
  int strip, chunk;
  item_coords(g, item, &it.s, &strip, &chunk);
  it.sm = batched ? it.s : 0;
  it.x0 = strip * W;
  chunk_rows(g, chunk, &it.ya, &it.yb);
  it.r0 = it.ya - (4 * P - 2);
  it.n_it = (it.yb - it.ya) + 8 * P - 4;
  const bool near_x = it.x0 - H - 4 < g.Wx || it.x0 + W + H + 4 > g.nx - g.Wx;
  it.xb = g.Wx > 0 && near_x;
  it.edge = near_x || (g.Wz > 0 && (it.r0 < g.Wz || it.r0 + it.n_it > g.ny - g.Wz));
  it.hx_lo = it.hx_hi = 0;
  return it.ya < it.yb;
}

struct Fwd2Warp {
  uint32_t bars, stage0, carry;
  uint32_t stage_bytes;
  uint32_t ca_o, cb_o;  // byte offsets of Ca / Cb within a stage's Ca / Cb slot
  int lane;
  Ring ring;
};

template <int P, bool BAND>
__device__ __forceinline__ void md2_issue(const Fwd2Maps &m, const StepArgs &a, const Item &it,
                                          int x, int y, uint32_t dst, uint32_t bar) {
  if (a.md_pair) {
    tma4s(dst, &m.map[kM2MD], x, y, it.sm, 0, bar);
  } else {
    tma3s(dst, &m.map[kM2MD], x, y, it.sm, bar);
    tma3s(dst + 128 * 4, &m.map[kM2CB], x, y, it.sm, bar);
  }
}

// Loads of iteration i (lane 0): Ey row r; Hx row h1 (from iteration 2P - 1);
// Hz row y1 and Ca / Cb row y1 (from 4P - 2, rows inside the array); Ca / Cb
// row y2 (from 8P - 4); band items add the memories the step-t updates read
// (z band: Hx nodes row h1, E nodes row y1; x band: rows y1).
template <int P, bool BAND>
__device__ __forceinline__ void fwd2_issue(const Fwd2Maps &m, const StepArgs &a, const Item &it,
                                           int i, uint32_t st, uint32_t bar) {
  constexpr int H = fwd2_halo(P);
  const int xb = it.x0 - H, ny = a.g.ny;
  const int r = it.r0 + i, y1 = r - 2 * P + 1, y2 = y1 - 2 * P + 1, h1 = r - P;
  const bool hx1 = i >= 2 * P - 1 && h1 >= 0 && h1 < ny;
  const bool e1 = i >= 4 * P - 2 && y1 >= 0 && y1 < ny;
  const bool e2 = i >= 8 * P - 4;
  uint32_t bytes = 128 * 4;
  if (hx1) bytes += 128 * 4;
  if (e1) bytes += 3 * 128 * 4;
  if (e2) bytes += 2 * 128 * 4;
  int zh = -1, ze = -1;
  if constexpr (BAND) {
    if (hx1) zh = zband_row(h1, ny, a.g.Wz);
    if (e1) ze = zband_row(y1, ny, a.g.Wz);
    if (zh >= 0) bytes += 128 * 4;
    if (ze >= 0) bytes += 128 * 4;
    if (it.xb && e1) bytes += 2 * (uint32_t)a.band_box_floats * 4;
  }
  expect_tx_s(bar, bytes);
  fence_proxy_async();
  tma3s(st + kF2_E * 4, &m.map[kM2E], xb, r, it.s, bar);
  if (hx1) tma3s(st + kF2_HX * 4, &m.map[kM2HX], xb, h1, it.s, bar);
  if (e1) {
    tma3s(st + kF2_HZ * 4, &m.map[kM2HZ], xb, y1, it.s, bar);
    md2_issue<P, BAND>(m, a, it, xb, y1, st + kF2_MD1 * 4, bar);
  }
  if (e2) md2_issue<P, BAND>(m, a, it, xb, y2, st + kF2_MD2 * 4, bar);
  if constexpr (BAND) {
    if (zh >= 0) tma3s(st + a.fo[kFoMzh] * 4, &m.map[kM2MZH], xb, zh, it.s, bar);
    if (ze >= 0) tma3s(st + a.fo[kFoMze] * 4, &m.map[kM2MZE], xb, ze, it.s, bar);
    if (it.xb && e1) {
      tma3s(st + a.fo[kFoMxh] * 4, &m.map[kM2MXH], 0, y1, it.s, bar);
      tma3s(st + a.fo[kFoMxe] * 4, &m.map[kM2MXE], 0, y1, it.s, bar);
    }
  }
}

template <int P, int STORE, bool BAND>
__device__ __forceinline__ bool fwd2_walk(const Fwd2Maps &m, const StepArgs &a, const Item &it,
                                          Fwd2Warp &w, float cqs) {
  constexpr int NQ = 2 * P;
  constexpr int NS = 2;
  constexpr int H = fwd2_halo(P), W = fwd2_width(P);
  // one iteration per loop trip (a longer unrolled body overflows the
  // instruction cache): the register queues shift once per iteration and the
  // carry rings rotate by a running slot
  constexpr int M = 1;
  using Q = Queue<NQ, M>;
  const int lane = w.lane;
  const int nx = a.g.nx, ny = a.g.ny;
  const int xb = it.x0 - H;
  const int c = xb + 4 * lane;
  const bool c_ok = !BAND || (c >= 0 && c < nx);
  const bool own = lane >= H / 4 && lane < H / 4 + W / 4 && c_ok;
  const int64_t pb = (int64_t)it.s * a.g.numel + c;
  float *const hz_o = a.out.hz + pb;
  float *const hx_o = a.out.hx + pb;
  float *const ey_o = a.out.ey + pb;
  const BandTab T{a.g.Wx, a.g.Wz};
  const int bcol = BAND ? xband_col(c, nx, a.g.Wx) : -1;
  const int64_t xbw = BAND ? (int64_t)it.s * ny * 2 * a.g.Wx + bcol : 0;
  const int64_t zbw = BAND ? (int64_t)it.s * 2 * a.g.Wz * nx + c : 0;
  // carry rings: x band at the H and E nodes (NQ band rows each), z band at
  // the H and E nodes (NQ rows of 32 float4 each)
  const uint32_t rxh = w.carry, rxe = rxh + NQ * a.band_ring * 4;
  const uint32_t rzh = rxe + NQ * a.band_ring * 4, rze = rzh + NQ * 128 * 4;
  // step-t sources into every E1 row computed, receivers of the owned rows
  Cursor c1a = cursor_at(a.ea, it.s, it.ya - 2 * P + 1), c1b = cursor_at(a.eb, it.s, it.ya);

  if (lane == 0) fwd2_issue<P, BAND>(m, a, it, 0, w.stage0 + w.ring.slot * w.stage_bytes,
                                     w.bars + 8 * w.ring.slot);
  F4 eq[Q::kSize], hq[Q::kSize], e1q[Q::kSize], h2q[Q::kSize], z1q[Q::kSize];
#pragma unroll
  for (int k = 0; k < Q::kSize; ++k) eq[k] = hq[k] = e1q[k] = h2q[k] = z1q[k] = zero4();
  // carry ring slots: written this iteration, written 2P - 1 iterations ago
  int cw = 0, cr = 1;

  for (int i0 = 0; i0 < it.n_it; i0 += M) {
#pragma unroll
    for (int u = 0; u < M; ++u) {
      const int i = i0 + u;
      if (i < it.n_it) {
        if (i + 1 < it.n_it && lane == 0) {
          const int ps = w.ring.slot ^ 1;
          fwd2_issue<P, BAND>(m, a, it, i + 1, w.stage0 + ps * w.stage_bytes, w.bars + 8 * ps);
        }
        if (!mbar_wait_s(w.bars + 8 * w.ring.slot, w.ring.phase)) {
          give_up_s<1>(a.flags, w.bars, w.ring, i, it.n_it, lane);
          return false;
        }
        const uint32_t st = w.stage0 + w.ring.slot * w.stage_bytes;
        const int r = it.r0 + i, y1 = r - 2 * P + 1, y2 = y1 - 2 * P + 1;
        const int h1 = r - P, h2 = y1 - P;
        const bool hx1 = i >= 2 * P - 1 && h1 >= 0 && h1 < ny;
        const bool e1 = i >= 4 * P - 2 && y1 >= 0 && y1 < ny;
        const bool e1_own = y1 >= it.ya && y1 < it.yb;
        const bool hx2 = i >= 6 * P - 3 && h2 >= 0 && h2 < ny;
        const bool hx2_own = h2 >= it.ya && h2 < it.yb;
        const bool e2 = i >= 8 * P - 4;

        eq[Q::at(u, 0)] = lds4s(st + kF2_E * 4 + 16 * lane);

        // ---- step t: Hx1, row h1 (z-stencil of the Ey queue)
        {
          const F4 hx_old = lds4s(st + kF2_HX * 4 + 16 * lane);
          F4 d;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float s = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              s = fmaf(a.c.cy[k - 1], eq[Q::at(u, P - k)].v[q] - eq[Q::at(u, P + k - 1)].v[q], s);
            d.v[q] = s;
          }
          if constexpr (BAND) {
            const int zr = hx1 ? zband_row(h1, ny, a.g.Wz) : -1;
            if (zr >= 0) {
              F4 mz = lds4s(st + a.fo[kFoMzh] * 4 + 16 * lane);
              const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
              const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(byh, mz.v[q], ayh * d.v[q]);
                d.v[q] = fmaf(d.v[q], rkyh, mz.v[q]);
              }
              sts4s(rzh + cw * 512 + 16 * lane, mz);
            }
          }
          F4 hn;
#pragma unroll
          for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(-cqs, d.v[q], hx_old.v[q]);
          hq[Q::at(u, 0)] = hx1 ? hn : zero4();
        }

        // ---- step t: Hz1 and E1, row y1
        F4 hz1 = zero4(), e1v = zero4();
        if (e1) {
          const F4 &e0 = eq[Q::at(u, NQ - 1)];
          {
            float wv[12];
            win_lanes<5 - P, 7 + P>(e0, wv);
            const F4 hz_old = lds4s(st + kF2_HZ * 4 + 16 * lane);
            if (!BAND || bcol < 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                hz1.v[q] = fmaf(cqs, d_half<P>(wv, q, a.c.cx), hz_old.v[q]);
            } else {
              F4 mn = lds4s(st + (a.fo[kFoMxh] + bcol) * 4);
              const F4 ah = ld4(a.bt + T.x(3) + bcol), bh = ld4(a.bt + T.x(4) + bcol);
              const F4 rk = ld4(a.bt + T.x(5) + bcol);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float d = d_half<P>(wv, q, a.c.cx);
                mn.v[q] = fmaf(bh.v[q], mn.v[q], ah.v[q] * d);
                hz1.v[q] = fmaf(cqs, fmaf(d, rk.v[q], mn.v[q]), hz_old.v[q]);
              }
              sts4s(rxh + (cw * a.band_ring + bcol) * 4, mn);
            }
            if (!c_ok) hz1 = zero4();
          }
          float wh[12];
          win_lanes<4 - P, 6 + P>(hz1, wh);
          const F4 ca4 = lds4s(st + kF2_MD1 * 4 + w.ca_o + 16 * lane);
          const F4 cb4 = lds4s(st + kF2_MD1 * 4 + w.cb_o + 16 * lane);
          F4 cx, cz;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            cx.v[q] = d_int<P>(wh, q, a.c.cx);
            float s = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              s = fmaf(a.c.cy[k - 1], hq[Q::at(u, P - k)].v[q] - hq[Q::at(u, P - 1 + k)].v[q], s);
            cz.v[q] = s;
          }
          if constexpr (BAND) {
            if (bcol >= 0) {
              F4 mx = lds4s(st + (a.fo[kFoMxe] + bcol) * 4);
              const F4 ax = ld4(a.bt + T.x(0) + bcol), bx = ld4(a.bt + T.x(1) + bcol);
              const F4 rk = ld4(a.bt + T.x(2) + bcol);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mx.v[q] = fmaf(bx.v[q], mx.v[q], ax.v[q] * cx.v[q]);
                cx.v[q] = fmaf(cx.v[q], rk.v[q], mx.v[q]);
              }
              sts4s(rxe + (cw * a.band_ring + bcol) * 4, mx);
            }
            const int zr = zband_row(y1, ny, a.g.Wz);
            if (zr >= 0) {
              F4 mz = lds4s(st + a.fo[kFoMze] * 4 + 16 * lane);
              const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
              const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(by, mz.v[q], ay * cz.v[q]);
                cz.v[q] = fmaf(cz.v[q], rky, mz.v[q]);
              }
              sts4s(rze + cw * 512 + 16 * lane, mz);
            }
          }
          F4 curl, en;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            curl.v[q] = cx.v[q] - cz.v[q];
            en.v[q] = fmaf(ca4.v[q], e0.v[q], cb4.v[q] * curl.v[q]);
          }
          if constexpr (STORE != kStoreNone) {  // step t's snapshots
            const int64_t so = ((int64_t)it.s * ny + y1) * a.snap_pitch + c;
            snap_store_p<STORE>(own && e1_own, a.snap_e, so, e0);
            if constexpr (STORE != kStoreEy) snap_store_p<STORE>(own && e1_own, a.snap_c, so, curl);
          }
          // step t's sources (every lane holding the cell), then its receivers
          if (y1 == c1a.row) {
            if (a.vals_t) inject_lanes(a.ea, it.s, c1a, a.vals_t, xb, lane, en);
            cursor_next(a.ea, it.s, c1a);
          }
          if (y1 == c1b.row) {
            if (a.out_t && y1 < it.yb)
              sample_lanes(a.eb, it.s, c1b, a.out_t, xb, it.x0, min(it.x0 + W, nx),
                           st + kF2_E * 4, lane, en);
            cursor_next(a.eb, it.s, c1b);
          }
          e1v = c_ok ? en : zero4();
        }
        z1q[Q::at(u, 0)] = hz1;
        e1q[Q::at(u, 0)] = e1v;

        // ---- step t + 1: Hx2, row h2 (z-stencil of the E1 queue)
        {
          const F4 &hx_old = hq[Q::at(u, NQ - 1)];
          F4 d;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float s = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              s = fmaf(a.c.cy[k - 1], e1q[Q::at(u, P - k)].v[q] - e1q[Q::at(u, P + k - 1)].v[q],
                       s);
            d.v[q] = s;
          }
          if constexpr (BAND) {
            const int zr = hx2 ? zband_row(h2, ny, a.g.Wz) : -1;
            if (zr >= 0) {
              F4 mz = lds4s(rzh + cr * 512 + 16 * lane);
              const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
              const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(byh, mz.v[q], ayh * d.v[q]);
                d.v[q] = fmaf(d.v[q], rkyh, mz.v[q]);
              }
              st4p(own && hx2_own, a.out.mzh_node + zbw + (int64_t)zr * nx, mz);
            }
          }
          F4 hn;
#pragma unroll
          for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(-cqs, d.v[q], hx_old.v[q]);
          h2q[Q::at(u, 0)] = hx2 ? hn : zero4();
          st4p(own && hx2_own, hx_o + (int64_t)h2 * nx, hn);
        }

        // ---- step t + 1: Hz2 and E2, row y2
        if (e2) {
          const F4 &e1o = e1q[Q::at(u, NQ - 1)];
          const F4 &hz1o = z1q[Q::at(u, NQ - 1)];
          F4 hz2;
          {
            float wv[12];
            win_lanes<5 - P, 7 + P>(e1o, wv);
            if (!BAND || bcol < 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q) hz2.v[q] = fmaf(cqs, d_half<P>(wv, q, a.c.cx), hz1o.v[q]);
            } else {
              F4 mn = lds4s(rxh + (cr * a.band_ring + bcol) * 4);
              const F4 ah = ld4(a.bt + T.x(3) + bcol), bh = ld4(a.bt + T.x(4) + bcol);
              const F4 rk = ld4(a.bt + T.x(5) + bcol);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float d = d_half<P>(wv, q, a.c.cx);
                mn.v[q] = fmaf(bh.v[q], mn.v[q], ah.v[q] * d);
                hz2.v[q] = fmaf(cqs, fmaf(d, rk.v[q], mn.v[q]), hz1o.v[q]);
              }
              st4p(own, a.out.mxh_node + xbw + (int64_t)y2 * 2 * a.g.Wx, mn);
            }
            st4p(own, hz_o + (int64_t)y2 * nx, hz2);
            if (!c_ok) hz2 = zero4();
          }
          float wh[12];
          win_lanes<4 - P, 6 + P>(hz2, wh);
          const F4 ca4 = lds4s(st + kF2_MD2 * 4 + w.ca_o + 16 * lane);
          const F4 cb4 = lds4s(st + kF2_MD2 * 4 + w.cb_o + 16 * lane);
          F4 cx, cz;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            cx.v[q] = d_int<P>(wh, q, a.c.cx);
            float s = 0.f;
#pragma unroll
            for (int k = 1; k <= P; ++k)
              s = fmaf(a.c.cy[k - 1], h2q[Q::at(u, P - k)].v[q] - h2q[Q::at(u, P - 1 + k)].v[q], s);
            cz.v[q] = s;
          }
          if constexpr (BAND) {
            if (bcol >= 0) {
              F4 mx = lds4s(rxe + (cr * a.band_ring + bcol) * 4);
              const F4 ax = ld4(a.bt + T.x(0) + bcol), bx = ld4(a.bt + T.x(1) + bcol);
              const F4 rk = ld4(a.bt + T.x(2) + bcol);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mx.v[q] = fmaf(bx.v[q], mx.v[q], ax.v[q] * cx.v[q]);
                cx.v[q] = fmaf(cx.v[q], rk.v[q], mx.v[q]);
              }
              st4p(own, a.out.mxe_node + xbw + (int64_t)y2 * 2 * a.g.Wx, mx);
            }
            const int zr = zband_row(y2, ny, a.g.Wz);
            if (zr >= 0) {
              F4 mz = lds4s(rze + cr * 512 + 16 * lane);
              const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
              const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(by, mz.v[q], ay * cz.v[q]);
                cz.v[q] = fmaf(cz.v[q], rky, mz.v[q]);
              }
              st4p(own, a.out.mze_node + zbw + (int64_t)zr * nx, mz);
            }
          }
          F4 curl, en;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            curl.v[q] = cx.v[q] - cz.v[q];
            en.v[q] = fmaf(ca4.v[q], e1o.v[q], cb4.v[q] * curl.v[q]);
          }
          if constexpr (STORE != kStoreNone) {  // step t + 1's snapshots
            const int64_t so = ((int64_t)it.s * ny + y2) * a.snap_pitch + c;
            snap_store_p<STORE>(own, a.snap_e2, so, e1o);
            if constexpr (STORE != kStoreEy) snap_store_p<STORE>(own, a.snap_c2, so, curl);
          }
          st4p(own, ey_o + (int64_t)y2 * nx, en);
        }
        __syncwarp();
        w.ring.next(NS);
        if constexpr (BAND) {
          cw = cw + 1 == NQ ? 0 : cw + 1;
          cr = cr + 1 == NQ ? 0 : cr + 1;
        }
      }
    }
    shift_queue<NQ, M>(eq);
    shift_queue<NQ, M>(hq);
    shift_queue<NQ, M>(e1q);
    shift_queue<NQ, M>(h2q);
    shift_queue<NQ, M>(z1q);
  }
  return true;
}

template <int P, int STORE>
__global__ void __launch_bounds__(128, 3)
    k_forward2(const __grid_constant__ Fwd2Maps m, const StepArgs a, const int batched) {
  constexpr int NS = 2;
  extern __shared__ __align__(128) float smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 127u) & ~127u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  Fwd2Warp w;
  w.lane = lane;
  w.bars = base + warp * NS * 8;
  w.stage_bytes = (uint32_t)a.stage_floats * 4;
  w.stage0 = base + 128 + warp * a.warp_floats * 4;
  w.carry = w.stage0 + NS * w.stage_bytes;
  // a pair box is [Ca][Cb] (or [Cb][Ca] when Cb lies first); two boxes put
  // Ca first, each 128 wide
  w.ca_o = a.md_pair && a.md_swap ? 512 : 0;
  w.cb_o = a.md_pair && a.md_swap ? 0 : 512;
  w.ring = Ring{0, 0u};
  const Geom &g = a.g;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  grid_dep_launch();
  if (lane == 0) {
    for (int k = 0; k < NS; ++k)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(w.bars + 8 * k), "r"(1)
                   : "memory");
    fence_mbar_init();
  }
  __syncwarp();
  grid_dep_wait();  // everything below reads what earlier kernels wrote
  if (__any_sync(kFull, *reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0)) return;
  const float cqs = __ldg(a.cq);
  int *ctr = a.flags + kCtrBase + a.ctr_slot;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.flags[kCtrBase + (a.ctr_slot ^ 1)] = 0;

  for (;;) {
    int item = 0;
    if (lane == 0) item = atomicAdd(ctr, 1);
    item = __shfl_sync(kFull, item, 0);
    if (item >= n_items) break;
    Item it;
    if (!make_item2<P>(g, item, batched != 0, it)) continue;
    const bool ok = it.edge ? fwd2_walk<P, STORE, true>(m, a, it, w, cqs)
                            : fwd2_walk<P, STORE, false>(m, a, it, w, cqs);
    if (!ok) return;
    // step t + 1's sources, then its receivers, in the item's cells
    fix_item(a, it.s, it.ya, it.yb, it.x0, min(it.x0 + fwd2_width(P), g.nx),
             a.out.ey + (int64_t)it.s * g.numel, g.nx, lane, a.vals_t2, a.out_t2);
  }
}

// ---------------------------------------------------------------------------

constexpr int kFwdL = 1;  // forward lookahead (rows in flight)
constexpr int kAdjL = 1;  // adjoint lookahead

// Forward stage: the fixed slots, then a Cq array's rows r and r - P, then
// the z-band memory rows and the two x-band memory rows, each only if used.
template <int P>
void fwd_layout_t(int Wx, bool cq_arr, bool born, StepArgs *a, size_t *smem) {
  const int bw = Wx > 0 ? ((2 * Wx + 31) / 32) * 32 : 0;
  int o = kF_FIXED;
  for (int k = 0; k < kFoCount; ++k) a->fo[k] = 0;
  if (cq_arr) {
    a->fo[kFoCqH] = o;
    a->fo[kFoCqX] = o + 128;
    o += 256;
  }
  if (Wx > 0) {
    a->fo[kFoMzh] = o;
    a->fo[kFoMze] = o + 128;
    a->fo[kFoMxh] = o + 256;
    a->fo[kFoMxe] = o + 256 + bw;
    o += 256 + 2 * bw;
  }
  if (born) {  // dCa / dCb (pair, or two 128-aligned boxes) and the snapshots
    a->fo[kFoBd] = o;
    a->fo[kFoBs] = o + 256;
    o += 256 + 288;
  }
  int wf = (kFwdL + 1) * o + 2 * P * kFRing;
  wf = ((wf + 31) / 32) * 32;
  a->stage_floats = o;
  a->warp_floats = wf;
  a->band_box_floats = 2 * Wx;
  *smem = (size_t)(32 + kWarpsPerCta * wf) * sizeof(float) + 128;
}

// Adjoint stage: the fixed slots, then a Cq array's rows r and r - P, then
// the x-band memory pair row and the two z-band memory rows, each only if
// used.  The warp area adds the px row and the qx ring.
template <int P>
void adj_layout_t(int Wx, bool cq_arr, StepArgs *a, size_t *smem) {
  int o = kA_FIXED;
  for (int k = 0; k < kAoCount; ++k) a->ao[k] = 0;
  if (cq_arr) {
    a->ao[kAoCqR] = o;
    a->ao[kAoCqH] = o + 128;
    o += 256;
  }
  if (Wx > 0) {
    a->ao[kAoMx] = o;
    o += ((4 * Wx + 31) / 32) * 32;
    a->ao[kAoMze] = o;
    a->ao[kAoMzh] = o + 128;
    o += 256;
  }
  int wf = (kAdjL + 1) * o + kAPx + 2 * P * kARing;
  wf = ((wf + 31) / 32) * 32;
  a->stage_floats = o;
  a->warp_floats = wf;
  a->band_box_floats = 2 * Wx;
  *smem = (size_t)(32 + adj_warps_per_cta(P) * wf) * sizeof(float) + 128;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per
// device.  `done` is a per-kernel bitmask of devices already configured.
template <typename K>
void allow_big_smem(K kern, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(done.load(std::memory_order_relaxed) & bit)) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    done.fetch_or(bit);
  }
}
template <int P, int STORE, int BORN = kStoreNone>
std::atomic<uint64_t> &fwd_smem_flag() {
  static std::atomic<uint64_t> f{0};
  return f;
}
template <int P, int SNAP>
std::atomic<uint64_t> &adj_smem_flag() {
  static std::atomic<uint64_t> f{0};
  return f;
}

template <int P, int STORE, int BORN = kStoreNone>
cudaError_t fwd_t(const FwdMaps &m, const StepArgs &a, bool batched, bool cq_arr, int grid,
                  cudaStream_t st) {
  const size_t smem = (size_t)(32 + kWarpsPerCta * a.warp_floats) * sizeof(float) + 128;
  allow_big_smem(k_forward<P, STORE, kFwdL, BORN>, fwd_smem_flag<P, STORE, BORN>());
  const cudaError_t e = launch_dependent(k_forward<P, STORE, kFwdL, BORN>, grid, 128, smem, st, m, a,
                                         batched ? 1 : 0, cq_arr ? 1 : 0);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}
template <int P, int SNAP>
cudaError_t adj_t(const AdjMaps &m, const StepArgs &a, bool batched, bool cq_arr, int grid,
                  cudaStream_t st) {
  const size_t smem = (size_t)(32 + adj_warps_per_cta(P) * a.warp_floats) * sizeof(float) + 128;
  allow_big_smem(k_adjoint<P, SNAP, kAdjL>, adj_smem_flag<P, SNAP>());
  const cudaError_t e = launch_dependent(k_adjoint<P, SNAP, kAdjL>, grid, 32 * adj_warps_per_cta(P),
                                         smem, st, m, a, batched ? 1 : 0, cq_arr ? 1 : 0);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

// Two-step forward stage: the fixed slots, then (with a band) the z-band
// memory rows of the H and E nodes and the two x-band memory rows.  The warp
// area adds the band items' carry rings: NQ x-band rows at each node, NQ
// rows of 128 floats at each z-band node.
template <int P>
void fwd2_layout_t(int Wx, StepArgs *a, size_t *smem) {
  const int bw = Wx > 0 ? ((2 * Wx + 31) / 32) * 32 : 0;
  int o = kF2_FIXED;
  for (int k = 0; k < kFoCount; ++k) a->fo[k] = 0;
  if (Wx > 0) {
    a->fo[kFoMzh] = o;
    a->fo[kFoMze] = o + 128;
    a->fo[kFoMxh] = o + 256;
    a->fo[kFoMxe] = o + 256 + bw;
    o += 256 + 2 * bw;
  }
  const int carry = Wx > 0 ? 2 * (2 * P) * bw + 2 * (2 * P) * 128 : 0;
  int wf = 2 * o + carry;
  wf = ((wf + 31) / 32) * 32;
  a->stage_floats = o;
  a->warp_floats = wf;
  a->band_box_floats = 2 * Wx;
  a->band_ring = bw;
  *smem = (size_t)(32 + kWarpsPerCta * wf) * sizeof(float) + 128;
}

template <int P, int STORE>
std::atomic<uint64_t> &fwd2_smem_flag() {
  static std::atomic<uint64_t> f{0};
  return f;
}

template <int P, int STORE>
cudaError_t fwd2_t(const Fwd2Maps &m, const StepArgs &a, bool batched, int grid, cudaStream_t st) {
  const size_t smem = (size_t)(32 + kWarpsPerCta * a.warp_floats) * sizeof(float) + 128;
  allow_big_smem(k_forward2<P, STORE>, fwd2_smem_flag<P, STORE>());
  const cudaError_t e = launch_dependent(k_forward2<P, STORE>, grid, 128, smem, st, m, a,
                                         batched ? 1 : 0);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

template <int P>
cudaError_t fwd2_store(const Fwd2Maps &m, const StepArgs &a, int store, bool batched, int grid,
                       cudaStream_t st) {
  switch (store) {
    case kStoreNone: return fwd2_t<P, kStoreNone>(m, a, batched, grid, st);
    case kStoreF32: return fwd2_t<P, kStoreF32>(m, a, batched, grid, st);
    case kStoreBF16: return fwd2_t<P, kStoreBF16>(m, a, batched, grid, st);
    case kStoreFP8: return fwd2_t<P, kStoreFP8>(m, a, batched, grid, st);
    case kStoreEy: return fwd2_t<P, kStoreEy>(m, a, batched, grid, st);
  }
  return cudaErrorInvalidValue;
}

template <int P>
cudaError_t fwd_store(const FwdMaps &m, const StepArgs &a, int store, int born, bool batched,
                      bool cq_arr, int grid, cudaStream_t st) {
  if (born != kStoreNone) {
    if (store != kStoreNone) return cudaErrorInvalidValue;
    switch (born) {
      case kStoreF32: return fwd_t<P, kStoreNone, kStoreF32>(m, a, batched, cq_arr, grid, st);
      case kStoreBF16: return fwd_t<P, kStoreNone, kStoreBF16>(m, a, batched, cq_arr, grid, st);
      case kStoreFP8: return fwd_t<P, kStoreNone, kStoreFP8>(m, a, batched, cq_arr, grid, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (store) {
    case kStoreNone: return fwd_t<P, kStoreNone>(m, a, batched, cq_arr, grid, st);
    case kStoreF32: return fwd_t<P, kStoreF32>(m, a, batched, cq_arr, grid, st);
    case kStoreBF16: return fwd_t<P, kStoreBF16>(m, a, batched, cq_arr, grid, st);
    case kStoreFP8: return fwd_t<P, kStoreFP8>(m, a, batched, cq_arr, grid, st);
    case kStoreEy: return fwd_t<P, kStoreEy>(m, a, batched, cq_arr, grid, st);
  }
  return cudaErrorInvalidValue;
}

template <int P>
cudaError_t adj_snap(const AdjMaps &m, const StepArgs &a, int snap, bool batched, bool cq_arr,
                     int grid, cudaStream_t st) {
  switch (snap) {
    case kStoreF32: return adj_t<P, kStoreF32>(m, a, batched, cq_arr, grid, st);
    case kStoreBF16: return adj_t<P, kStoreBF16>(m, a, batched, cq_arr, grid, st);
    case kStoreFP8: return adj_t<P, kStoreFP8>(m, a, batched, cq_arr, grid, st);
    case kStoreEy: return adj_t<P, kStoreEy>(m, a, batched, cq_arr, grid, st);
  }
  return cudaErrorInvalidValue;
}

template <typename K>
int occupancy(K kern, int threads, size_t smem, std::atomic<uint64_t> &flag) {
  allow_big_smem(kern, flag);
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

template <int P>
int slots_t(bool adjoint, int Wx, bool cq_arr) {
  size_t smem;
  StepArgs a{};
  if (adjoint) {
    adj_layout_t<P>(Wx, cq_arr, &a, &smem);
    return occupancy(k_adjoint<P, kStoreF32, kAdjL>, 32 * adj_warps_per_cta(P), smem,
                     adj_smem_flag<P, kStoreF32>()) *
           adj_warps_per_cta(P);
  }
  fwd_layout_t<P>(Wx, cq_arr, false, &a, &smem);
  return occupancy(k_forward<P, kStoreF32, kFwdL, kStoreNone>, 32 * kWarpsPerCta, smem,
                   fwd_smem_flag<P, kStoreF32>()) *
         kWarpsPerCta;
}

template <int P>
int fwd2_slots_t(int Wx) {
  size_t smem;
  StepArgs a{};
  fwd2_layout_t<P>(Wx, &a, &smem);
  return occupancy(k_forward2<P, kStoreF32>, 128, smem, fwd2_smem_flag<P, kStoreF32>()) *
         kWarpsPerCta;
}

}  // namespace

cudaError_t launch_forward(const FwdMaps &m, const StepArgs &a, int order, int store, int born,
                           bool batched, bool cq_array, int grid, cudaStream_t st) {
  switch (order) {
    case 2: return fwd_store<1>(m, a, store, born, batched, cq_array, grid, st);
    case 4: return fwd_store<2>(m, a, store, born, batched, cq_array, grid, st);
    case 6: return fwd_store<3>(m, a, store, born, batched, cq_array, grid, st);
    case 8: return fwd_store<4>(m, a, store, born, batched, cq_array, grid, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_adjoint(const AdjMaps &m, const StepArgs &a, int order, int snap,
                           bool batched, bool cq_array, int grid, cudaStream_t st) {
  switch (order) {
    case 2: return adj_snap<1>(m, a, snap, batched, cq_array, grid, st);
    case 4: return adj_snap<2>(m, a, snap, batched, cq_array, grid, st);
    case 6: return adj_snap<3>(m, a, snap, batched, cq_array, grid, st);
    case 8: return adj_snap<4>(m, a, snap, batched, cq_array, grid, st);
  }
  return cudaErrorInvalidValue;
}

bool forward2_supported(int order) { return order >= 2 && order <= 6; }

cudaError_t launch_forward2(const Fwd2Maps &m, const StepArgs &a, int order, int store,
                            bool batched, int grid, cudaStream_t st) {
  switch (order) {
    case 2: return fwd2_store<1>(m, a, store, batched, grid, st);
    case 4: return fwd2_store<2>(m, a, store, batched, grid, st);
    case 6: return fwd2_store<3>(m, a, store, batched, grid, st);
  }
  return cudaErrorInvalidValue;
}

void forward2_layout(int order, int Wx, StepArgs *a, size_t *smem) {
  switch (order) {
    case 2: fwd2_layout_t<1>(Wx, a, smem); return;
    case 4: fwd2_layout_t<2>(Wx, a, smem); return;
    default: fwd2_layout_t<3>(Wx, a, smem); return;
  }
}

int forward2_slots_per_sm(int order, int Wx) {
  switch (order) {
    case 2: return fwd2_slots_t<1>(Wx);
    case 4: return fwd2_slots_t<2>(Wx);
    default: return fwd2_slots_t<3>(Wx);
  }
}

int stencil_slots_per_sm(int order, bool adjoint, int Wx, bool cq_array) {
  switch (order) {
    case 2: return slots_t<1>(adjoint, Wx, cq_array);
    case 4: return slots_t<2>(adjoint, Wx, cq_array);
    case 6: return slots_t<3>(adjoint, Wx, cq_array);
    default: return slots_t<4>(adjoint, Wx, cq_array);
  }
}

void adjoint_layout(int order, int Wx, bool cq_array, bool bf16, StepArgs *a, size_t *smem) {
  (void)bf16;  // the snapshot slot is sized for float32 either way
  switch (order) {
    case 2: adj_layout_t<1>(Wx, cq_array, a, smem); return;
    case 4: adj_layout_t<2>(Wx, cq_array, a, smem); return;
    case 6: adj_layout_t<3>(Wx, cq_array, a, smem); return;
    default: adj_layout_t<4>(Wx, cq_array, a, smem); return;
  }
}

void forward_layout(int order, int Wx, bool cq_array, bool born, StepArgs *a, size_t *smem) {
  switch (order) {
    case 2: fwd_layout_t<1>(Wx, cq_array, born, a, smem); return;
    case 4: fwd_layout_t<2>(Wx, cq_array, born, a, smem); return;
    case 6: fwd_layout_t<3>(Wx, cq_array, born, a, smem); return;
    default: fwd_layout_t<4>(Wx, cq_array, born, a, smem); return;
  }
}

}  // namespace mw
