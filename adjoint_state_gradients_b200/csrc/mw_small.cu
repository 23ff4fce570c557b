// Small grids: a whole forward or adjoint sweep in one cooperative launch.
//
// Method: page "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu" -- the forward and
// adjoint steps of its header comment, in the order of the host drivers
// `forward` (H, E, sources, receivers) and `backward` (adjoint sources,
// source gradient, adjoint H, adjoint E with gradient).
//
// On a few thousand to a few hundred thousand cells the marching-strip
// kernels are bound by launch and row latency: a launch walks a handful of
// rows per warp, each waiting for its TMA copy.  Here one launch runs every
// step: each shot gets a thread-block cluster (up to 16 blocks), whose
// threads own groups of cells (a row's 4, or 2, consecutive columns), and
// the steps' phases are separated by the cluster's hardware barrier.  Two
// variants: the resident one (further below), whose blocks keep their rows
// of every field in shared memory, and, for grids too large for that, the
// one here, whose state stays in place in global memory (it fits in L2;
// reads of anything the launch writes bypass L1 (ld.global.cg), since L1 is
// not coherent between blocks).  Every update, source sum and receiver
// sample is the stencil kernels' operation for operation, so the results
// are bitwise those of the step-by-step launches.
//
// Forward step t:  H phase (Hz, Hx and their band memories; the receivers of
//   step t - 1, read from E) | E phase (snapshots of E^t and curl^t, the E
//   update and its band memories, then f[t] added in the source cells,
//   duplicates of a cell summed first).  After the last step, the receivers
//   of step nt - 1.
// Adjoint (res[nt - 1] added to the start state first), step t = nt - 1 .. 0:
//   E-node phase (gradients gCa += E^t lam, gCb += curl^t lam; lambda_E
//   sampled at the sources; g = Cb lam and its transposed band terms px,
//   pz) | H-node phase (lambda_Hz, lambda_Hx from px, pz; their transposed
//   band terms qx, qz) | E phase (lambda_E = Ca lam - D_x qx - D_z qz, then
//   res[t - 1] added in the receiver cells).  px, pz, qx, qz live in
//   workspace arrays (resident: shared memory) between the phases; the
//   resident adjoint accumulates the gradients in its lambda_E phase.
#include <cooperative_groups.h>
#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "mw_device.cuh"
#include "mw_internal.cuh"

namespace mw {
namespace {
using namespace dev;
namespace cg = cooperative_groups;

__device__ __forceinline__ F4 ldcg4(const float *p) {
  const float4 t = __ldcg(reinterpret_cast<const float4 *>(p));
  return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ void stg4(float *p, const F4 &v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v.v[0], v.v[1], v.v[2], v.v[3]);
}
// float4 of a written-in-this-launch field at (row y, column c) of one shot,
// zero outside the array (c is a multiple of 4 and nx % 4 == 0)
__device__ __forceinline__ F4 fld4(const float *base, int y, int c, int ny, int nx) {
  // an unconditional load (clamped address) and a select, so that a group's
  // loads issue back to back instead of one per branch
  const bool ok = y >= 0 && y < ny && c >= 0 && c < nx;
  const F4 v = ldcg4(base + (ok ? (int64_t)y * nx + c : 0));
  return ok ? v : zero4();
}
// x window w[0..12) = columns c - 4 .. c + 8 of row y
__device__ __forceinline__ void win_row(const float *base, int y, int c, int ny, int nx,
                                        float w[12]) {
  const F4 a = fld4(base, y, c - 4, ny, nx), b = fld4(base, y, c, ny, nx),
           d = fld4(base, y, c + 4, ny, nx);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    w[q] = a.v[q];
    w[q + 4] = b.v[q];
    w[q + 8] = d.v[q];
  }
}

template <int P>
__device__ __forceinline__ float dh(const float w[12], int q, const float c[4]) {
  float d = 0.f;
#pragma unroll
  for (int k = 1; k <= P; ++k) d = fmaf(c[k - 1], w[q + k + 4] - w[q - k + 5], d);
  return d;
}
template <int P>
__device__ __forceinline__ float di(const float w[12], int q, const float c[4]) {
  float d = 0.f;
#pragma unroll
  for (int k = 1; k <= P; ++k) d = fmaf(c[k - 1], w[q + k + 3] - w[q - k + 4], d);
  return d;
}

__device__ __forceinline__ int xband(int c, int nx, int Wx) {
  if (Wx == 0) return -1;
  if (c < Wx) return c;
  if (c >= nx - Wx) return c - nx + 2 * Wx;
  return -1;
}
__device__ __forceinline__ int zband(int r, int ny, int Wz) {
  if (Wz == 0 || r < 0 || r >= ny) return -1;
  if (r < Wz) return r;
  if (r >= ny - Wz) return r - ny + 2 * Wz;
  return -1;
}

// The barrier between phases: every thread of the shot's cluster arrives
// (release) and waits (acquire) -- a hardware barrier, so every block of the
// cluster runs the same sequence of phases (the loops' trip counts are the
// same for all of them).  The non-.aligned form: a warp may reach it
// diverged after the per-group branches.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ int cluster_rank() {
  int r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ int cluster_size() {
  int n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}

// The cluster of shot s = blockIdx.x / cluster size walks the shot's float4
// groups (row, column / 4); thread k of the cluster takes k, k + threads, ...
#define MW_FOR_GROUPS(a, s, y, c)                                                   \
  for (int64_t g_ = (int64_t)cluster_rank() * blockDim.x + threadIdx.x,             \
               ng_ = (int64_t)(a).ny * ((a).nx / 4);                                \
       g_ < ng_; g_ += (int64_t)cluster_size() * blockDim.x)                        \
    if (const int s = (int)(blockIdx.x / cluster_size()); true)                    \
      if (const int y = (int)(g_ / ((a).nx / 4)); true)                             \
        if (const int c = (int)(g_ % ((a).nx / 4)) * 4; true)

// Add vals[s][k] at the cells of `es` (run heads add their duplicates'
// values first, in index order); one thread per sorted entry.
__device__ __forceinline__ void inject_all(const EntrySet &es, const float *vals, float *field,
                                           int64_t numel, int nx, int S) {
  if (vals == nullptr || es.n == 0) return;
  const int s = blockIdx.x / cluster_size();
  for (int j = cluster_rank() * blockDim.x + threadIdx.x; j < es.n;
       j += cluster_size() * blockDim.x) {
    const int nv = __ldg(es.abeg + (int64_t)s * (es.n + 1) + es.n);
    if (j >= nv) continue;
    const int4 *en = es.ent + (int64_t)s * es.n;
    const int4 q = __ldg(en + j);
    if (q.w == 0) continue;
    const float *vs = vals + (int64_t)s * es.n;
    float v = __ldg(vs + q.z);
    for (int u = 1; u < q.w; ++u) v += __ldg(vs + __ldg(en + j + u).z);
    float *p = field + (int64_t)s * numel + (int64_t)q.x * nx + q.y;
    *p = __ldcg(p) + v;
  }
}
// out[s][k] = field at the cell of entry k of `es`
__device__ __forceinline__ void sample_all(const EntrySet &es, float *out, const float *field,
                                           int64_t numel, int nx, int S) {
  if (out == nullptr || es.n == 0) return;
  const int s = blockIdx.x / cluster_size();
  for (int j = cluster_rank() * blockDim.x + threadIdx.x; j < es.n;
       j += cluster_size() * blockDim.x) {
    const int nv = __ldg(es.abeg + (int64_t)s * (es.n + 1) + es.n);
    if (j >= nv) continue;
    const int4 q = __ldg(es.ent + (int64_t)s * es.n + j);
    out[(int64_t)s * es.n + q.z] = __ldcg(field + (int64_t)s * numel + (int64_t)q.x * nx + q.y);
  }
}

// Add vals[s][k] into the float4 v of group (s, y, c) for the entries of
// `es` in those four cells (run heads add their duplicates first, in index
// order): the same sum, added the same way, as the stencil kernels' fix-ups.
__device__ __forceinline__ void inject_group(const EntrySet &es, const float *vals, int s, int y,
                                             int c, int ny, F4 &v) {
  if (vals == nullptr || es.n == 0) return;
  const int2 rc = __ldg(es.rcur + (int64_t)s * (ny + 1) + y);
  if (rc.y != y) return;
  const int *ab = es.abeg + (int64_t)s * (es.n + 1);
  int j = __ldg(ab + rc.x);
  const int j1 = __ldg(ab + rc.x + 1);
  const int4 *en = es.ent + (int64_t)s * es.n;
  const float *vs = vals + (int64_t)s * es.n;
  // the row's entries are sorted by column: the first one at column >= c
  for (int hi = j1; j < hi;) {
    const int mid = (j + hi) >> 1;
    if (__ldg(&en[mid].y) < c) j = mid + 1;
    else hi = mid;
  }
  for (; j < j1; ++j) {
    const int4 q = __ldg(en + j);
    const int d = q.y - c;
    if (d >= 4) break;
    if (q.w == 0) continue;
    float val = __ldg(vs + q.z);
    for (int u = 1; u < q.w; ++u) val += __ldg(vs + __ldg(en + j + u).z);
    if (d == 0) v.v[0] += val;
    else if (d == 1) v.v[1] += val;
    else if (d == 2) v.v[2] += val;
    else v.v[3] += val;
  }
}

// ---------------------------------------------------------------------------
// forward

template <int P, int STORE, int NT>
__global__ void __launch_bounds__(NT) k_small_fwd(const SmallArgs a) {
  // a wait timed out earlier on this workspace and is not reported yet: stand
  // down like the stencil kernels (every block reads the same word, so the
  // whole cluster leaves before its first barrier)
  if (*reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0) return;
  const int ny = a.ny, nx = a.nx;
  const BandTab T{a.Wx, a.Wz};
  const float cqs = a.cq_arr ? 0.f : __ldg(a.cq);
  for (int t = 0; t < a.nt; ++t) {
    // ---- H phase (and the receivers of step t - 1)
    if (t > 0)
      sample_all(a.rec, a.rec_out ? a.rec_out + (int64_t)(t - 1) * a.S * a.rec.n : nullptr,
                 a.st.ey, a.numel, nx, a.S);
    MW_FOR_GROUPS(a, s, y, c) {
      const int64_t sb = (int64_t)s * a.numel, cell = sb + (int64_t)y * nx + c;
      const int64_t mb = a.batched ? cell : (int64_t)y * nx + c;
      const F4 cq = a.cq_arr ? ld4(a.cq + mb) : splat4(cqs);
      const float *ey = a.st.ey + sb;
      // Hz(y, c..c+3) at the half nodes
      {
        float w[12];
        win_row(ey, y, c, ny, nx, w);
        const F4 hz_old = ldcg4(a.st.hz + cell);
        F4 hn;
        const int bc = xband(c, nx, a.Wx);
        if (bc < 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(cq.v[q], dh<P>(w, q, a.c.cx), hz_old.v[q]);
        } else {
          float *mp = a.st.mxh_node + ((int64_t)s * ny + y) * 2 * a.Wx + bc;
          F4 mn = ldcg4(mp);
          const F4 ah = ld4(a.bt + T.x(3) + bc), bh = ld4(a.bt + T.x(4) + bc);
          const F4 rk = ld4(a.bt + T.x(5) + bc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float d = dh<P>(w, q, a.c.cx);
            mn.v[q] = fmaf(bh.v[q], mn.v[q], ah.v[q] * d);
            hn.v[q] = fmaf(cq.v[q], fmaf(d, rk.v[q], mn.v[q]), hz_old.v[q]);
          }
          stg4(mp, mn);
        }
        stg4(a.st.hz + cell, hn);
      }
      // Hx(y + 1/2, c..c+3): z window of E rows y - P + 1 .. y + P
      {
        F4 e[2 * P];
#pragma unroll
        for (int j = 0; j < 2 * P; ++j) e[j] = fld4(ey, y + P - j, c, ny, nx);  // e[j] = E(y + P - j)
        const F4 hx_old = ldcg4(a.st.hx + cell);
        F4 d;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float sacc = 0.f;
#pragma unroll
          for (int k = 1; k <= P; ++k)  // E(y + k) - E(y - k + 1)
            sacc = fmaf(a.c.cy[k - 1], e[P - k].v[q] - e[P + k - 1].v[q], sacc);
          d.v[q] = sacc;
        }
        const int zr = zband(y, ny, a.Wz);
        if (zr >= 0) {
          float *mp = a.st.mzh_node + ((int64_t)s * 2 * a.Wz + zr) * nx + c;
          F4 mz = ldcg4(mp);
          const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
          const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            mz.v[q] = fmaf(byh, mz.v[q], ayh * d.v[q]);
            d.v[q] = fmaf(d.v[q], rkyh, mz.v[q]);
          }
          stg4(mp, mz);
        }
        F4 hn;
#pragma unroll
        for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(-cq.v[q], d.v[q], hx_old.v[q]);
        stg4(a.st.hx + cell, hn);
      }
    }
    cluster_sync();
    // ---- E phase
    MW_FOR_GROUPS(a, s, y, c) {
      const int64_t sb = (int64_t)s * a.numel, cell = sb + (int64_t)y * nx + c;
      const int64_t mb = a.batched ? cell : (int64_t)y * nx + c;
      float w[12];
      win_row(a.st.hz + sb, y, c, ny, nx, w);
      F4 h[2 * P];
#pragma unroll
      for (int j = 0; j < 2 * P; ++j) h[j] = fld4(a.st.hx + sb, y + P - 1 - j, c, ny, nx);  // Hx(y+P-1-j)
      const F4 ca4 = ld4(a.ca + mb), cb4 = ld4(a.cb + mb);
      const F4 e_old = ldcg4(a.st.ey + cell);
      F4 cx, cz;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        cx.v[q] = di<P>(w, q, a.c.cx);
        float sacc = 0.f;
#pragma unroll
        for (int k = 1; k <= P; ++k)  // Hx(y + k - 1) - Hx(y - k)
          sacc = fmaf(a.c.cy[k - 1], h[P - k].v[q] - h[P - 1 + k].v[q], sacc);
        cz.v[q] = sacc;
      }
      const int bc = xband(c, nx, a.Wx);
      if (bc >= 0) {
        float *mp = a.st.mxe_node + ((int64_t)s * ny + y) * 2 * a.Wx + bc;
        F4 mx = ldcg4(mp);
        const F4 ax = ld4(a.bt + T.x(0) + bc), bx = ld4(a.bt + T.x(1) + bc);
        const F4 rk = ld4(a.bt + T.x(2) + bc);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mx.v[q] = fmaf(bx.v[q], mx.v[q], ax.v[q] * cx.v[q]);
          cx.v[q] = fmaf(cx.v[q], rk.v[q], mx.v[q]);
        }
        stg4(mp, mx);
      }
      const int zr = zband(y, ny, a.Wz);
      if (zr >= 0) {
        float *mp = a.st.mze_node + ((int64_t)s * 2 * a.Wz + zr) * nx + c;
        F4 mz = ldcg4(mp);
        const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
        const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mz.v[q] = fmaf(by, mz.v[q], ay * cz.v[q]);
          cz.v[q] = fmaf(cz.v[q], rky, mz.v[q]);
        }
        stg4(mp, mz);
      }
      F4 curl, en;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        curl.v[q] = cx.v[q] - cz.v[q];
        en.v[q] = fmaf(ca4.v[q], e_old.v[q], cb4.v[q] * curl.v[q]);
      }
      if constexpr (STORE != kStoreNone) {
        const int64_t so = (int64_t)t * a.step_elems + ((int64_t)s * ny + y) * a.snap_pitch + c;
        snap_store<STORE>(a.snap_e, so, e_old);
        snap_store<STORE>(a.snap_c, so, curl);
      }
      // the sources of step t in these cells
      inject_group(a.src, a.f ? a.f + (int64_t)t * a.S * a.src.n : nullptr, s, y, c, ny, en);
      stg4(a.st.ey + cell, en);
    }
    cluster_sync();
  }
  sample_all(a.rec, a.rec_out ? a.rec_out + (int64_t)(a.nt - 1) * a.S * a.rec.n : nullptr,
             a.st.ey, a.numel, nx, a.S);
}

// ---------------------------------------------------------------------------
// adjoint

template <int P, int SNAP, int NT>
__global__ void __launch_bounds__(NT) k_small_adj(const SmallArgs a) {
  // a wait timed out earlier on this workspace and is not reported yet: stand
  // down like the stencil kernels (every block reads the same word, so the
  // whole cluster leaves before its first barrier)
  if (*reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0) return;
  const int ny = a.ny, nx = a.nx;
  const BandTab T{a.Wx, a.Wz};
  const float cqs = a.cq_arr ? 0.f : __ldg(a.cq);
  constexpr int64_t kElem = SNAP == kStoreF32 ? 4 : SNAP == kStoreBF16 ? 2 : 1;
  // the residuals of the last step enter the start state; each later step's
  // are added by the E phase of the step before it in adjoint order
  inject_all(a.rec, a.res ? a.res + (int64_t)(a.nt - 1) * a.S * a.rec.n : nullptr, a.st.ey,
             a.numel, nx, a.S);
  cluster_sync();
  for (int t = a.nt - 1; t >= 0; --t) {
    // ---- E nodes: gradients, the source gradient, px and pz
    sample_all(a.src, a.grad_f ? a.grad_f + (int64_t)t * a.S * a.src.n : nullptr, a.st.ey,
               a.numel, nx, a.S);
    MW_FOR_GROUPS(a, s, y, c) {
      const int64_t sb = (int64_t)s * a.numel, cell = sb + (int64_t)y * nx + c;
      const int64_t mb = a.batched ? cell : (int64_t)y * nx + c;
      const F4 lam = ldcg4(a.st.ey + cell);
      const F4 cbv = ld4(a.cb + mb);
      F4 gv;
#pragma unroll
      for (int q = 0; q < 4; ++q) gv.v[q] = cbv.v[q] * lam.v[q];
      // gradients (lam = lambda_E^{t+1})
      {
        const int64_t so = (int64_t)t * a.step_elems + ((int64_t)s * ny + y) * a.snap_pitch + c;
        const char *se = reinterpret_cast<const char *>(a.snap_e) + so * kElem;
        const char *sc = reinterpret_cast<const char *>(a.snap_c) + so * kElem;
        F4 ev, cv;
        if constexpr (SNAP == kStoreF32) {
          ev = ld4(reinterpret_cast<const float *>(se));
          cv = ld4(reinterpret_cast<const float *>(sc));
        } else if constexpr (SNAP == kStoreBF16) {
          const uint2 ue = __ldg(reinterpret_cast<const uint2 *>(se));
          const uint2 uc = __ldg(reinterpret_cast<const uint2 *>(sc));
          const float2 e0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ue.x));
          const float2 e1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ue.y));
          const float2 c0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&uc.x));
          const float2 c1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&uc.y));
          ev = F4{{e0.x, e0.y, e1.x, e1.y}};
          cv = F4{{c0.x, c0.y, c1.x, c1.y}};
        } else {
          const uint32_t ue = __ldg(reinterpret_cast<const uint32_t *>(se));
          const uint32_t uc = __ldg(reinterpret_cast<const uint32_t *>(sc));
          auto dec = [](uint32_t w) {
            const __half2_raw lo =
                __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xffffu), __NV_E4M3);
            const __half2_raw hi =
                __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
            const float2 fa = __half22float2(__half2(lo)), fb = __half22float2(__half2(hi));
            return F4{{fa.x, fa.y, fb.x, fb.y}};
          };
          ev = dec(ue);
          cv = dec(uc);
        }
        F4 gca = ldcg4(a.gca + cell), gcb = ldcg4(a.gcb + cell);
        const bool rowmask = !a.grad_mask || (y >= a.n_pml && y < ny - a.n_pml);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool colmask = !a.grad_mask || (c + q >= a.n_pml && c + q < nx - a.n_pml);
          if (rowmask && colmask) {
            gca.v[q] = fmaf(ev.v[q], lam.v[q], gca.v[q]);
            gcb.v[q] = fmaf(cv.v[q], lam.v[q], gcb.v[q]);
          }
        }
        stg4(a.gca + cell, gca);
        stg4(a.gcb + cell, gcb);
      }
      // pz (z band at the E nodes) and px (x band at the E nodes)
      F4 pz, px = gv;
#pragma unroll
      for (int q = 0; q < 4; ++q) pz.v[q] = -gv.v[q];
      const int zr = zband(y, ny, a.Wz);
      if (zr >= 0) {
        float *mp = a.st.mze_node + ((int64_t)s * 2 * a.Wz + zr) * nx + c;
        F4 M = ldcg4(mp);
        const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
        const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          M.v[q] -= gv.v[q];
          pz.v[q] = fmaf(ay, M.v[q], -gv.v[q] * rky);
          M.v[q] *= by;
        }
        stg4(mp, M);
      }
      const int bc = xband(c, nx, a.Wx);
      if (bc >= 0) {
        float *mp = a.st.mxe_node + ((int64_t)s * ny + y) * 2 * a.Wx + bc;
        F4 M = ldcg4(mp);
        const F4 ax = ld4(a.bt + T.x(0) + bc), bx = ld4(a.bt + T.x(1) + bc);
        const F4 rk = ld4(a.bt + T.x(2) + bc);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          M.v[q] += gv.v[q];
          px.v[q] = fmaf(ax.v[q], M.v[q], gv.v[q] * rk.v[q]);
          M.v[q] *= bx.v[q];
        }
        stg4(mp, M);
      }
      stg4(a.px + cell, px);
      stg4(a.pz + cell, pz);
    }
    cluster_sync();
    // ---- H nodes: lambda_Hz, qx; lambda_Hx, qz
    MW_FOR_GROUPS(a, s, y, c) {
      const int64_t sb = (int64_t)s * a.numel, cell = sb + (int64_t)y * nx + c;
      const int64_t mb = a.batched ? cell : (int64_t)y * nx + c;
      const F4 cq = a.cq_arr ? ld4(a.cq + mb) : splat4(cqs);
      {
        float w[12];
        win_row(a.px + sb, y, c, ny, nx, w);
        const F4 lhz_old = ldcg4(a.st.hz + cell);
        F4 lhz, v;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          lhz.v[q] = lhz_old.v[q] - dh<P>(w, q, a.c.cx);
          v.v[q] = cq.v[q] * lhz.v[q];
        }
        stg4(a.st.hz + cell, lhz);
        const int bc = xband(c, nx, a.Wx);
        if (bc >= 0) {
          float *mp = a.st.mxh_node + ((int64_t)s * ny + y) * 2 * a.Wx + bc;
          F4 M = ldcg4(mp);
          const F4 ah = ld4(a.bt + T.x(3) + bc), bh = ld4(a.bt + T.x(4) + bc);
          const F4 rk = ld4(a.bt + T.x(5) + bc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            M.v[q] += v.v[q];
            const float vq = v.v[q];
            v.v[q] = fmaf(ah.v[q], M.v[q], vq * rk.v[q]);
            M.v[q] *= bh.v[q];
          }
          stg4(mp, M);
        }
        stg4(a.qx + cell, v);
      }
      {
        F4 p[2 * P];
#pragma unroll
        for (int j = 0; j < 2 * P; ++j) p[j] = fld4(a.pz + sb, y + P - j, c, ny, nx);  // pz(y + P - j)
        const F4 lhx = ldcg4(a.st.hx + cell);
        F4 lh, qz;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float d = 0.f;
#pragma unroll
          for (int k = 1; k <= P; ++k)  // pz(y + k) - pz(y - k + 1)
            d = fmaf(a.c.cy[k - 1], p[P - k].v[q] - p[P + k - 1].v[q], d);
          lh.v[q] = lhx.v[q] - d;
          qz.v[q] = -cq.v[q] * lh.v[q];
        }
        stg4(a.st.hx + cell, lh);
        const int zr = zband(y, ny, a.Wz);
        if (zr >= 0) {
          float *mp = a.st.mzh_node + ((int64_t)s * 2 * a.Wz + zr) * nx + c;
          F4 M = ldcg4(mp);
          const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
          const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float vq = qz.v[q];
            M.v[q] += vq;
            qz.v[q] = fmaf(ayh, M.v[q], vq * rkyh);
            M.v[q] *= byh;
          }
          stg4(mp, M);
        }
        stg4(a.qz + cell, qz);
      }
    }
    cluster_sync();
    // ---- lambda_E
    MW_FOR_GROUPS(a, s, y, c) {
      const int64_t sb = (int64_t)s * a.numel, cell = sb + (int64_t)y * nx + c;
      const int64_t mb = a.batched ? cell : (int64_t)y * nx + c;
      float w[12];
      win_row(a.qx + sb, y, c, ny, nx, w);
      F4 qv[2 * P];
#pragma unroll
      for (int j = 0; j < 2 * P; ++j) qv[j] = fld4(a.qz + sb, y + P - 1 - j, c, ny, nx);  // qz(y+P-1-j)
      const F4 lam = ldcg4(a.st.ey + cell);
      const F4 cav = ld4(a.ca + mb);
      F4 en;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // Ca lam rounded on its own (never fused with the subtraction below),
        // as the stencil kernel queues it for 2P - 1 rows
        const float cla = __fmul_rn(cav.v[q], lam.v[q]);
        float dz = 0.f;
#pragma unroll
        for (int k = 1; k <= P; ++k)  // qz(y + k - 1) - qz(y - k)
          dz = fmaf(a.c.cy[k - 1], qv[P - k].v[q] - qv[P - 1 + k].v[q], dz);
        en.v[q] = cla - di<P>(w, q, a.c.cx) - dz;
      }
      // the residuals of step t - 1 in these cells
      if (t > 0)
        inject_group(a.rec, a.res ? a.res + (int64_t)(t - 1) * a.S * a.rec.n : nullptr, s, y, c,
                     ny, en);
      stg4(a.st.ey + cell, en);
    }
    cluster_sync();
  }
}

// x unchanged, but opaque to the compiler: what is derived from a group's
// coordinates is recomputed in every phase instead of being held in
// registers across the whole sweep
__device__ __forceinline__ int opaque(int x) {
  asm volatile("" : "+r"(x));
  return x;
}
// a group coordinate for the phase: opaque with several groups a thread
// (registers are scarce), else as is (its addresses are kept across steps)
template <int G>
__device__ __forceinline__ int gco(int x) {
  if constexpr (G > 1) return opaque(x);
  else return x;
}

// ---------------------------------------------------------------------------
// Resident variants: every block keeps its rows of the state -- and, in the
// adjoint, of the transposed band terms px, pz, qx, qz -- in shared memory
// for the whole sweep.  Block b of a shot's cluster owns rows [b R, b R + R);
// a z stencil reads the up to P rows beyond its block's edges from the
// neighbouring blocks' shared memory (the cluster's distributed shared
// memory), so every stencil load is an on-chip load.  The model and the
// per-shot gradients sit in registers: thread i owns the float4 groups i,
// i + NT, ... (at most G) of its block's rows.  Updates, source sums,
// receiver samples and gradient terms are the same operations as above, so
// the results are bitwise those of the step-by-step launches.
//
// The cluster barrier releases the thread's memory operations: it waits for
// every global load or store it still has in flight (asynchronous copies
// included), a few hundred ns each time.  So global traffic is issued at
// the start of a phase, and on small blocks (one group a thread) it moves
// in chunks of K steps through rings in shared memory: the forward stages
// the snapshots and receiver samples of K steps and writes them out at the
// start of the next chunk, and loads K steps of source values at once; the
// adjoint likewise with its source-gradient samples and residual values.
// The adjoint loads a step's snapshots into registers at the end of the
// lambda_E phase before it (the next cluster barrier is a phase away) and
// accumulates the gradients in its own lambda_E phase.

// Shared-memory layout of a resident block (floats): nf fields of R rows of
// nx + 8 floats (the row's cells from offset 4, four zero columns on each
// side, so that an x window needs no bounds checks), the two x-band
// memories (R x 2 Wx each), the two z-band memories (R x nx each, at the
// block's row; only band rows are used), the CPML band table, ring A (K x
// Cs: forward source values, adjoint source-gradient samples), ring B (K x
// Cr: forward receiver samples, adjoint residual values), and `ns` snapshot
// staging slots of E then curl of the block's cells (forward; `eb` bytes a
// cell).
struct ResLayout {
  int R, nx, Wx, Wz, nf, K, Cs, Cr, eb, ns;
  __host__ __device__ static int64_t up4(int64_t n) { return (n + 3) / 4 * 4; }
  __host__ __device__ int pitch() const { return nx + 8; }
  __host__ __device__ int64_t field(int k) const { return (int64_t)k * R * pitch(); }
  __host__ __device__ int64_t xmem(int k) const { return field(nf) + (int64_t)k * R * 2 * Wx; }
  __host__ __device__ int64_t zmem(int k) const {
    return xmem(2) + (int64_t)k * (Wz > 0 ? R : 0) * nx;
  }
  __host__ __device__ int64_t btab() const { return zmem(2); }
  __host__ __device__ int64_t ring_a() const { return btab() + up4(12 * Wx + 12 * Wz); }
  __host__ __device__ int64_t ring_b() const { return ring_a() + up4((int64_t)K * Cs); }
  __host__ __device__ int64_t slots() const { return ring_b() + up4((int64_t)K * Cr); }
  __host__ __device__ int64_t slot_bytes() const { return (int64_t)2 * R * nx * eb; }
  __host__ __device__ int64_t floats() const { return slots() + up4(ns * slot_bytes() / 4); }
};
constexpr int kResFieldsFwd = 3;  // E, Hx, Hz
constexpr int kResFieldsAdj = 7;  // lambda_E, lambda_Hx, lambda_Hz, px, pz, qx, qz
// steps a chunk at most (a power of two): 8 with one group a thread, else 1
__host__ __device__ constexpr int res_kmax(int G) { return G == 1 ? 8 : 1; }

// One field of the cluster: this block's rows in its own shared memory, and
// the generic addresses of the same array in the blocks above and below.
struct CRows {
  float *loc;
  const float *up, *dn;
};
__device__ __forceinline__ CRows crows(const cg::cluster_group &cl, float *loc, int rank, int cs) {
  CRows r;
  r.loc = loc;
  r.up = rank > 0 ? cl.map_shared_rank(loc, rank - 1) : loc;
  r.dn = rank + 1 < cs ? cl.map_shared_rank(loc, rank + 1) : loc;
  return r;
}
__device__ __forceinline__ F4 lds4(const float *p) {
  const float4 t = *reinterpret_cast<const float4 *>(p);
  return F4{{t.x, t.y, t.z, t.w}};
}
// W consecutive cells (a group of 4, or of 2 on small blocks, where twice
// the threads each take half a float4's work)
template <int W>
struct VW {
  float v[W];
};
template <int W>
__device__ __forceinline__ VW<W> ldv(const float *p) {
  VW<W> r;
  if constexpr (W == 4) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    r.v[0] = t.x, r.v[1] = t.y, r.v[2] = t.z, r.v[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2 *>(p);
    r.v[0] = t.x, r.v[1] = t.y;
  }
  return r;
}
template <int W>
__device__ __forceinline__ VW<W> ldgv(const float *p) {  // read-only global data
  VW<W> r;
  if constexpr (W == 4) {
    const float4 t = __ldg(reinterpret_cast<const float4 *>(p));
    r.v[0] = t.x, r.v[1] = t.y, r.v[2] = t.z, r.v[3] = t.w;
  } else {
    const float2 t = __ldg(reinterpret_cast<const float2 *>(p));
    r.v[0] = t.x, r.v[1] = t.y;
  }
  return r;
}
template <int W>
__device__ __forceinline__ void stv(float *p, const VW<W> &a) {
  if constexpr (W == 4)
    *reinterpret_cast<float4 *>(p) = make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
  else
    *reinterpret_cast<float2 *>(p) = make_float2(a.v[0], a.v[1]);
}
template <int W>
__device__ __forceinline__ VW<W> zerov() {
  VW<W> r;
#pragma unroll
  for (int q = 0; q < W; ++q) r.v[q] = 0.f;
  return r;
}
template <int W>
__device__ __forceinline__ VW<W> splatv(float x) {
  VW<W> r;
#pragma unroll
  for (int q = 0; q < W; ++q) r.v[q] = x;
  return r;
}

// The rows [r0, r1) of one block (R rows per block; block b - 1 holds
// [r0 - R, r0), block b + 1 starts at r1) of a shot with ny rows; rows of
// `np` floats, cells from offset 4.
struct RBlk {
  int r0, r1, R, ny, np;
  // the W cells at (y, c) of a cluster field, zero outside the array
  // (column c is a group's own column; |y - row| <= P <= R)
  template <int W>
  __device__ __forceinline__ VW<W> zrow(const CRows &f, int y, int c) const {
    const bool in = y >= 0 && y < ny;
    const float *p = f.loc + 4 + c;
    if (in)
      p = (y < r0 ? f.up + (y - r0 + R) * np : y < r1 ? f.loc + (y - r0) * np : f.dn + (y - r1) * np) +
          4 + c;
    const VW<W> v = ldv<W>(p);
    return in ? v : zerov<W>();
  }
  // out[j] = field at row y + D0 - j, j < N, of the group at (y, c): from
  // this block's rows at constant offsets when all of them are here
  template <int W, int N, int D0>
  __device__ __forceinline__ void zwin(const CRows &f, int y, int c, VW<W> out[N]) const {
    if (y - r0 + D0 - (N - 1) >= 0 && y - r0 + D0 < r1 - r0) {
      const float *p = f.loc + (y - r0 + D0) * np + 4 + c;
#pragma unroll
      for (int j = 0; j < N; ++j) out[j] = ldv<W>(p - j * np);
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) out[j] = zrow<W>(f, y + D0 - j, c);
    }
  }
};
// x window w[0..12) = columns c - 4 .. c + 8 of a padded row (cells from
// offset 4; the zero columns stand for the cells outside the array); with
// W = 2 only w[0..10) (columns c - 4 .. c + 6) is read
template <int W>
__device__ __forceinline__ void xwin(const float *row, int c, float w[12]) {
  if constexpr (W == 4) {
    const VW<4> A = ldv<4>(row + c), B = ldv<4>(row + c + 4), D = ldv<4>(row + c + 8);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      w[q] = A.v[q];
      w[q + 4] = B.v[q];
      w[q + 8] = D.v[q];
    }
  } else {
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const VW<2> t = ldv<2>(row + c + 2 * j);
      w[2 * j] = t.v[0];
      w[2 * j + 1] = t.v[1];
    }
    w[10] = w[11] = 0.f;
  }
}

// Zero this block's shared fields (the padding columns stay zero), copy its
// rows of a state buffer (E, Hx, Hz, the four band memories) into shared
// memory (IN) or back, and the band table in.
template <bool IN>
__device__ void res_state(const Fields &st, float *sm, const ResLayout &Ly, const float *bt,
                          int s, int r0, int Rb, int ny, int64_t numel) {
  const int nx = Ly.nx, nx4 = nx >> 2, Wx = Ly.Wx, Wz = Ly.Wz, np = Ly.pitch();
  if (IN) {
    for (int64_t k = threadIdx.x; k < Ly.field(Ly.nf) / 4; k += blockDim.x)
      reinterpret_cast<float4 *>(sm)[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = threadIdx.x; k < 12 * Wx + 12 * Wz; k += blockDim.x) sm[Ly.btab() + k] = __ldg(bt + k);
    __syncthreads();
  }
  float *const g3[3] = {st.ey, st.hx, st.hz};
  for (int k = threadIdx.x; k < Rb * nx4; k += blockDim.x) {
    const int ly = k / nx4, c = (k - ly * nx4) * 4, y = r0 + ly;
    const int64_t gi = (int64_t)s * numel + (int64_t)y * nx + c;
    const int64_t li = (int64_t)ly * np + 4 + c, lz = (int64_t)ly * nx + c;
#pragma unroll
    for (int f = 0; f < 3; ++f) {
      if (IN) st4(sm + Ly.field(f) + li, lds4(g3[f] + gi));
      else st4(g3[f] + gi, lds4(sm + Ly.field(f) + li));
    }
    const int zr = zband(y, ny, Wz);
    if (zr >= 0) {
      const int64_t gz = ((int64_t)s * 2 * Wz + zr) * nx + c;
      if (IN) {
        st4(sm + Ly.zmem(0) + lz, lds4(st.mzh_node + gz));
        st4(sm + Ly.zmem(1) + lz, lds4(st.mze_node + gz));
      } else {
        st4(st.mzh_node + gz, lds4(sm + Ly.zmem(0) + lz));
        st4(st.mze_node + gz, lds4(sm + Ly.zmem(1) + lz));
      }
    }
  }
  const int w4 = Wx >> 1;  // float4 groups of a 2 Wx row
  for (int k = threadIdx.x; k < Rb * w4; k += blockDim.x) {
    const int ly = k / w4, j = (k - ly * w4) * 4;
    const int64_t gi = ((int64_t)s * ny + r0 + ly) * 2 * Wx + j;
    const int64_t li = (int64_t)ly * 2 * Wx + j;
    if (IN) {
      st4(sm + Ly.xmem(0) + li, lds4(st.mxh_node + gi));
      st4(sm + Ly.xmem(1) + li, lds4(st.mxe_node + gi));
    } else {
      st4(st.mxh_node + gi, lds4(sm + Ly.xmem(0) + li));
      st4(st.mxe_node + gi, lds4(sm + Ly.xmem(1) + li));
    }
  }
}

// The sorted entries [x, y) of a set that lie in rows [r0, r1) of shot s.
__device__ __forceinline__ int2 entry_range(const EntrySet &es, int s, int r0, int r1) {
  if (es.n == 0) return make_int2(0, 0);
  const int2 *rc = es.rcur + (int64_t)s * (es.ny + 1);
  const int *ab = es.abeg + (int64_t)s * (es.n + 1);
  return make_int2(__ldg(ab + __ldg(&rc[r0].x)), __ldg(ab + __ldg(&rc[r1].x)));
}
// The value a run head adds: its entries' values summed in index order.
__device__ __forceinline__ float head_sum(const int4 *en, const float *vs, int j, const int4 &q) {
  float v = __ldg(vs + q.z);
  for (int u = 1; u < q.w; ++u) v += __ldg(vs + __ldg(en + j + u).z);
  return v;
}

// The entries of a set in this block's rows [e.x, e.y): thread k < C takes
// entry e.x + k through a ring slot of C floats a step; the rest (if the
// block holds more than C) are handled directly, in turn by all threads.
struct REnt {
  const int4 *en;  // the shot's sorted entries
  int2 e;
  int C;
  int4 q;          // the thread's ring entry (w = -1: none)
  __device__ __forceinline__ void init(const EntrySet &es, int s, int2 e_, int C_) {
    e = e_;
    C = C_;
    en = es.n > 0 ? es.ent + (int64_t)s * es.n : nullptr;
    q = make_int4(0, 0, 0, -1);
    if (en && (int)threadIdx.x < C && e.x + (int)threadIdx.x < e.y) q = __ldg(en + e.x + threadIdx.x);
  }
  __device__ __forceinline__ bool mine() const { return q.w >= 0; }
  __device__ __forceinline__ int j() const { return e.x + (int)threadIdx.x; }
};
// Sample a padded field at the set's entries: the thread's ring entry into
// its ring slot, the others straight to out (the step's [S][n] block).
template <int NT>
__device__ __forceinline__ void res_sample(const REnt &E, float *ring_slot, float *out, int s,
                                           int n, const float *field, int r0, int np) {
  if (E.mine()) ring_slot[threadIdx.x] = field[(E.q.x - r0) * np + 4 + E.q.y];
  if (out == nullptr || E.en == nullptr) return;
  for (int j = E.e.x + E.C + (int)threadIdx.x; j < E.e.y; j += NT) {
    const int4 q = __ldg(E.en + j);
    out[(int64_t)s * n + q.z] = field[(q.x - r0) * np + 4 + q.y];
  }
}
// Add a step's values at the set's run heads: the thread's ring entry from
// its ring slot, the others from vals (the step's [S][n] block).
template <int NT>
__device__ __forceinline__ void res_inject(const REnt &E, const float *ring_slot,
                                           const float *vals, int s, int n, float *field, int r0,
                                           int np) {
  if (E.mine() && E.q.w > 0) {
    float *p = field + (E.q.x - r0) * np + 4 + E.q.y;
    *p = *p + ring_slot[threadIdx.x];
  }
  if (vals == nullptr || E.en == nullptr) return;
  for (int j = E.e.x + E.C + (int)threadIdx.x; j < E.e.y; j += NT) {
    const int4 q = __ldg(E.en + j);
    if (q.w == 0) continue;
    const float v = head_sum(E.en, vals + (int64_t)s * n, j, q);
    float *p = field + (q.x - r0) * np + 4 + q.y;
    *p = *p + v;
  }
}
// Values of the thread's ring head for up to KM steps (step i's [S][n]
// block at vals + step(i)), loaded together; written to the ring later.
template <int KM>
struct RingLoad {
  float v[KM];
  template <typename F>
  __device__ __forceinline__ void load(const REnt &E, int s, int n, int cnt, F step) {
    if (!E.mine() || E.q.w <= 0) return;
#pragma unroll
    for (int i = 0; i < KM; ++i)
      if (i < cnt) {
        const float *vs = step(i);
        v[i] = vs ? head_sum(E.en, vs + (int64_t)s * n, E.j(), E.q) : 0.f;
      }
  }
  template <typename F>
  __device__ __forceinline__ void store(const REnt &E, int cnt, F slot) const {
    if (!E.mine() || E.q.w <= 0) return;
#pragma unroll
    for (int i = 0; i < KM; ++i)
      if (i < cnt) slot(i)[threadIdx.x] = v[i];
  }
};

// Wait for the whole cluster, then leave together if an earlier wait timed
// out on this workspace (block 0 reads the word; everyone takes its answer).
__device__ __forceinline__ bool res_start(const cg::cluster_group &cl, const int *flags,
                                          int *s_stop) {
  if (threadIdx.x == 0)
    *s_stop = cl.block_rank() == 0 ? *reinterpret_cast<const volatile int *>(flags + kFlagTimeout)
                                   : 0;
  cluster_sync();
  const bool stop = *cl.map_shared_rank(s_stop, 0) != 0;
  cluster_sync();  // block 0 stays until everyone has read its word
  return stop;
}

// Snapshot store of W cells at element `elem` (the 4-cell form is
// snap_store; 2 cells: the same conversions on one pair).
template <int STORE, int W>
__device__ __forceinline__ void snap_store_w(void *base, int64_t elem, const VW<W> &v) {
  if constexpr (W == 4) {
    snap_store<STORE>(base, elem, F4{{v.v[0], v.v[1], v.v[2], v.v[3]}});
  } else if constexpr (STORE == kStoreF32) {
    *reinterpret_cast<float2 *>(reinterpret_cast<float *>(base) + elem) = make_float2(v.v[0], v.v[1]);
  } else if constexpr (STORE == kStoreBF16) {
    __nv_bfloat162 pr = __floats2bfloat162_rn(v.v[0], v.v[1]);
    *reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(base) + elem) =
        *reinterpret_cast<uint32_t *>(&pr);
  } else if constexpr (STORE == kStoreFP8) {
    const uint32_t pr =
        __nv_cvt_float2_to_fp8x2(make_float2(v.v[0], v.v[1]), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(base) + elem) = (uint16_t)pr;
  }
}
// Copy one group's staged snapshot words (W cells of the store type) from
// shared memory to the snapshot array.
template <typename T>
__device__ __forceinline__ void copy_words(const void *src, int64_t i, void *dst, int64_t j) {
  *(reinterpret_cast<T *>(dst) + j) = *(reinterpret_cast<const T *>(src) + i);
}
template <int STORE, int W>
__device__ __forceinline__ void stage_out(const void *stage, int64_t li, void *dst, int64_t so) {
  constexpr int bytes = W * (STORE == kStoreF32 ? 4 : STORE == kStoreBF16 ? 2 : 1);
  if constexpr (bytes == 16) copy_words<uint4>(stage, li / W, dst, so / W);
  else if constexpr (bytes == 8) copy_words<uint2>(stage, li / W, dst, so / W);
  else if constexpr (bytes == 4) copy_words<uint32_t>(stage, li / W, dst, so / W);
  else if constexpr (bytes == 2) copy_words<uint16_t>(stage, li / W, dst, so / W);
}
__host__ __device__ constexpr int stage_bytes(int store) {
  return store == kStoreF32 ? 4 : store == kStoreBF16 ? 2 : store == kStoreFP8 ? 1 : 0;
}

template <int P, int STORE, int NT, int G, int W>
__global__ void __launch_bounds__(NT, 1) k_res_fwd(const SmallArgs a) {
  constexpr int KM = res_kmax(G);
  using V = VW<W>;
  __shared__ int s_stop;
  const cg::cluster_group cl = cg::this_cluster();
  if (res_start(cl, a.flags, &s_stop)) return;
  const int cs = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int s = (int)(blockIdx.x / cs);
  const int ny = a.ny, nx = a.nx, nxw = nx / W, R = a.rows, K = a.kchunk, km = K - 1;
  const int r0 = rank * R, r1 = min(ny, r0 + R), Rb = r1 - r0, ng = Rb * nxw;
  const ResLayout Ly{R, nx, a.Wx, a.Wz, kResFieldsFwd, K, a.csrc, a.crec, stage_bytes(STORE),
                     STORE != kStoreNone ? K : 0};
  const int np = Ly.pitch();
  const RBlk B{r0, r1, R, ny, np};
  extern __shared__ float4 res_dyn[];
  float *sm = reinterpret_cast<float *>(res_dyn);
  float *sE = sm + Ly.field(0), *sHx = sm + Ly.field(1), *sHz = sm + Ly.field(2);
  float *sMxh = sm + Ly.xmem(0), *sMxe = sm + Ly.xmem(1);
  float *sMzh = sm + Ly.zmem(0), *sMze = sm + Ly.zmem(1);
  const float *bt = sm + Ly.btab();
  float *ringF = sm + Ly.ring_a(), *ringR = sm + Ly.ring_b();
  char *slots = reinterpret_cast<char *>(sm + Ly.slots());
  const int64_t slot_b = Ly.slot_bytes();
  const CRows fE = crows(cl, sE, rank, cs), fHx = crows(cl, sHx, rank, cs);
  const BandTab T{a.Wx, a.Wz};
  const float cqs = a.cq_arr ? 0.f : __ldg(a.cq);
  const int64_t sb = (int64_t)s * a.numel;
  // the thread's groups: row and column, and their Ca, Cb
  int gy[G], gc[G];
  V ca[G], cb[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int k = (int)threadIdx.x + g * NT;
    gy[g] = -1;
    gc[g] = 0;
    ca[g] = cb[g] = zerov<W>();
    if (k < ng) {
      const int ly = k / nxw;
      gy[g] = r0 + ly;
      gc[g] = (k - ly * nxw) * W;
      const int64_t mb = (a.batched ? sb : 0) + (int64_t)gy[g] * nx + gc[g];
      ca[g] = ldgv<W>(a.ca + mb);
      cb[g] = ldgv<W>(a.cb + mb);
    }
  }
  res_state<true>(a.st, sm, Ly, a.bt, s, r0, Rb, ny, a.numel);
  REnt src, rec;
  src.init(a.src, s, entry_range(a.src, s, r0, r1), a.csrc);
  rec.init(a.rec, s, entry_range(a.rec, s, r0, r1), a.crec);
  const int64_t fstep = (int64_t)a.S * a.src.n, rstep = (int64_t)a.S * a.rec.n;
  // steps [t0, t0 + cnt) of the rings to the snapshot arrays and the records
  auto flush = [&](int t0, int cnt) {
#pragma unroll
    for (int i = 0; i < KM; ++i) {
      if (i >= cnt) break;
      const int t = t0 + i, k = t & km;
      if constexpr (STORE != kStoreNone) {
        const char *se = slots + k * slot_b, *sc = se + slot_b / 2;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (gy[g] < 0) continue;
          const int y = gco<G>(gy[g]), c = gc[g];
          const int64_t li = (int64_t)(y - r0) * nx + c;
          const int64_t so = (int64_t)t * a.step_elems + ((int64_t)s * ny + y) * a.snap_pitch + c;
          stage_out<STORE, W>(se, li, a.snap_e, so);
          stage_out<STORE, W>(sc, li, a.snap_c, so);
        }
      }
      if (a.rec_out && rec.mine())
        a.rec_out[(int64_t)t * rstep + (int64_t)s * a.rec.n + rec.q.z] = ringR[k * a.crec + threadIdx.x];
    }
  };
  cluster_sync();
  for (int t = 0; t < a.nt; ++t) {
    // ---- H phase; first the global traffic, once a chunk: the last
    // chunk's snapshots and records out, this chunk's source values in
    if (t > 0 && a.rec_out)
      res_sample<NT>(rec, ringR + ((t - 1) & km) * a.crec, a.rec_out + (int64_t)(t - 1) * rstep, s,
                     a.rec.n, sE, r0, np);
    RingLoad<KM> fl;
    const int kc = min(K, a.nt - t);
    const bool chunk = (t & km) == 0;
    if (chunk) {
      if (t > 0) flush(t - K, K);
      if (a.f) fl.load(src, s, a.src.n, kc, [&](int i) { return a.f + (int64_t)(t + i) * fstep; });
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (gy[g] < 0) continue;
      const int y = gco<G>(gy[g]), c = gco<G>(gc[g]), ly = y - r0;
      const int64_t mb = (a.batched ? sb : 0) + (int64_t)y * nx + c;
      const V cq = a.cq_arr ? ldgv<W>(a.cq + mb) : splatv<W>(cqs);
      // the z window of E rows y - P + 1 .. y + P first: rows of the
      // neighbouring blocks take longest, and the stores below would keep
      // the compiler from hoisting their loads
      V e[2 * P];
      B.zwin<W, 2 * P, P>(fE, y, c, e);  // e[j] = E(y + P - j)
      // Hz(y, c..c+3) at the half nodes
      {
        float w[12];
        xwin<W>(sE + ly * np, c, w);
        float *hp = sHz + ly * np + 4 + c;
        const V hz_old = ldv<W>(hp);
        V hn;
        const int bc = xband(c, nx, a.Wx);
        if (bc < 0) {
#pragma unroll
          for (int q = 0; q < W; ++q) hn.v[q] = fmaf(cq.v[q], dh<P>(w, q, a.c.cx), hz_old.v[q]);
        } else {
          float *mp = sMxh + ly * 2 * a.Wx + bc;
          V mn = ldv<W>(mp);
          const V ah = ldv<W>(bt + T.x(3) + bc), bh = ldv<W>(bt + T.x(4) + bc);
          const V rk = ldv<W>(bt + T.x(5) + bc);
#pragma unroll
          for (int q = 0; q < W; ++q) {
            const float d = dh<P>(w, q, a.c.cx);
            mn.v[q] = fmaf(bh.v[q], mn.v[q], ah.v[q] * d);
            hn.v[q] = fmaf(cq.v[q], fmaf(d, rk.v[q], mn.v[q]), hz_old.v[q]);
          }
          stv<W>(mp, mn);
        }
        stv<W>(hp, hn);
      }
      // Hx(y + 1/2, c..c+3) from the z window of E
      {
        float *hp = sHx + ly * np + 4 + c;
        const V hx_old = ldv<W>(hp);
        V d;
#pragma unroll
        for (int q = 0; q < W; ++q) {
          float sacc = 0.f;
#pragma unroll
          for (int k = 1; k <= P; ++k)  // E(y + k) - E(y - k + 1)
            sacc = fmaf(a.c.cy[k - 1], e[P - k].v[q] - e[P + k - 1].v[q], sacc);
          d.v[q] = sacc;
        }
        const int zr = zband(y, ny, a.Wz);
        if (zr >= 0) {
          float *mp = sMzh + ly * nx + c;
          V mz = ldv<W>(mp);
          const float ayh = bt[T.z(3) + zr], byh = bt[T.z(4) + zr];
          const float rkyh = bt[T.z(5) + zr];
#pragma unroll
          for (int q = 0; q < W; ++q) {
            mz.v[q] = fmaf(byh, mz.v[q], ayh * d.v[q]);
            d.v[q] = fmaf(d.v[q], rkyh, mz.v[q]);
          }
          stv<W>(mp, mz);
        }
        V hn;
#pragma unroll
        for (int q = 0; q < W; ++q) hn.v[q] = fmaf(-cq.v[q], d.v[q], hx_old.v[q]);
        stv<W>(hp, hn);
      }
    }
    if (chunk && a.f) fl.store(src, kc, [&](int i) { return ringF + ((t + i) & km) * a.csrc; });
    cluster_sync();
    // ---- E phase
    char *se = slots + (t & km) * slot_b;
    void *stE = se, *stC = se + slot_b / 2;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (gy[g] < 0) continue;
      const int y = gco<G>(gy[g]), c = gco<G>(gc[g]), ly = y - r0;
      V h[2 * P];
      B.zwin<W, 2 * P, P - 1>(fHx, y, c, h);  // h[j] = Hx(y + P - 1 - j)
      float w[12];
      xwin<W>(sHz + ly * np, c, w);
      float *ep = sE + ly * np + 4 + c;
      const V e_old = ldv<W>(ep);
      V cx, cz;
#pragma unroll
      for (int q = 0; q < W; ++q) {
        cx.v[q] = di<P>(w, q, a.c.cx);
        float sacc = 0.f;
#pragma unroll
        for (int k = 1; k <= P; ++k)  // Hx(y + k - 1) - Hx(y - k)
          sacc = fmaf(a.c.cy[k - 1], h[P - k].v[q] - h[P - 1 + k].v[q], sacc);
        cz.v[q] = sacc;
      }
      const int bc = xband(c, nx, a.Wx);
      if (bc >= 0) {
        float *mp = sMxe + ly * 2 * a.Wx + bc;
        V mx = ldv<W>(mp);
        const V ax = ldv<W>(bt + T.x(0) + bc), bx = ldv<W>(bt + T.x(1) + bc);
        const V rk = ldv<W>(bt + T.x(2) + bc);
#pragma unroll
        for (int q = 0; q < W; ++q) {
          mx.v[q] = fmaf(bx.v[q], mx.v[q], ax.v[q] * cx.v[q]);
          cx.v[q] = fmaf(cx.v[q], rk.v[q], mx.v[q]);
        }
        stv<W>(mp, mx);
      }
      const int zr = zband(y, ny, a.Wz);
      if (zr >= 0) {
        float *mp = sMze + ly * nx + c;
        V mz = ldv<W>(mp);
        const float ay = bt[T.z(0) + zr], by = bt[T.z(1) + zr];
        const float rky = bt[T.z(2) + zr];
#pragma unroll
        for (int q = 0; q < W; ++q) {
          mz.v[q] = fmaf(by, mz.v[q], ay * cz.v[q]);
          cz.v[q] = fmaf(cz.v[q], rky, mz.v[q]);
        }
        stv<W>(mp, mz);
      }
      V curl, en;
#pragma unroll
      for (int q = 0; q < W; ++q) {
        curl.v[q] = cx.v[q] - cz.v[q];
        en.v[q] = fmaf(ca[g].v[q], e_old.v[q], cb[g].v[q] * curl.v[q]);
      }
      if constexpr (STORE != kStoreNone) {
        const int64_t li = (int64_t)ly * nx + c;
        snap_store_w<STORE, W>(stE, li, e_old);
        snap_store_w<STORE, W>(stC, li, curl);
      }
      stv<W>(ep, en);
    }
    // the sources of step t, added to the updated E of their cells
    if (a.f) {
      __syncthreads();
      res_inject<NT>(src, ringF + (t & km) * a.csrc, a.f + (int64_t)t * fstep, s, a.src.n, sE, r0,
                     np);
    }
    cluster_sync();
  }
  if (a.nt > 0) {
    if (a.rec_out)
      res_sample<NT>(rec, ringR + ((a.nt - 1) & km) * a.crec,
                     a.rec_out + (int64_t)(a.nt - 1) * rstep, s, a.rec.n, sE, r0, np);
    const int t0 = (a.nt - 1) & ~km;
    flush(t0, a.nt - t0);
  }
  __syncthreads();
  res_state<false>(a.st, sm, Ly, a.bt, s, r0, Rb, ny, a.numel);
}

// Snapshot words of one group (W cells) as stored (fp32, bf16 or FP8),
// loaded a step ahead and decoded at use.
template <int SNAP, int W>
struct SnapWords {
  static constexpr int kBytes = W * (SNAP == kStoreF32 ? 4 : SNAP == kStoreBF16 ? 2 : 1);
  static constexpr int kWords = (kBytes + 3) / 4;
  uint32_t w[kWords];
  // elem: the group's first cell
  __device__ __forceinline__ void load(const void *base, int64_t elem) {
    if constexpr (kBytes == 16) {
      const uint4 u = __ldg(reinterpret_cast<const uint4 *>(base) + elem / W);
      w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
    } else if constexpr (kBytes == 8) {
      const uint2 u = __ldg(reinterpret_cast<const uint2 *>(base) + elem / W);
      w[0] = u.x, w[1] = u.y;
    } else if constexpr (kBytes == 4) {
      w[0] = __ldg(reinterpret_cast<const uint32_t *>(base) + elem / W);
    } else {
      w[0] = __ldg(reinterpret_cast<const unsigned short *>(base) + elem / W);
    }
  }
  __device__ __forceinline__ VW<W> get() const {
    VW<W> r;
    if constexpr (SNAP == kStoreF32) {
#pragma unroll
      for (int q = 0; q < W; ++q) r.v[q] = __uint_as_float(w[q]);
    } else if constexpr (SNAP == kStoreBF16) {
#pragma unroll
      for (int h = 0; h < W / 2; ++h) {
        const float2 e = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[h]));
        r.v[2 * h] = e.x, r.v[2 * h + 1] = e.y;
      }
    } else {
#pragma unroll
      for (int h = 0; h < W / 2; ++h) {
        const __half2_raw pr = __nv_cvt_fp8x2_to_halfraw2(
            (__nv_fp8x2_storage_t)((w[0] >> (16 * h)) & 0xffffu), __NV_E4M3);
        const float2 f = __half22float2(__half2(pr));
        r.v[2 * h] = f.x, r.v[2 * h + 1] = f.y;
      }
    }
    return r;
  }
};

template <int P, int SNAP, int NT, int G, int W>
__global__ void __launch_bounds__(NT, 1) k_res_adj(const SmallArgs a) {
  constexpr int KM = res_kmax(G);
  using V = VW<W>;
  __shared__ int s_stop;
  const cg::cluster_group cl = cg::this_cluster();
  if (res_start(cl, a.flags, &s_stop)) return;
  const int cs = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int s = (int)(blockIdx.x / cs);
  const int ny = a.ny, nx = a.nx, nxw = nx / W, R = a.rows, K = a.kchunk, km = K - 1, nt = a.nt;
  const int r0 = rank * R, r1 = min(ny, r0 + R), Rb = r1 - r0, ng = Rb * nxw;
  const ResLayout Ly{R, nx, a.Wx, a.Wz, kResFieldsAdj, K, a.csrc, a.crec, 0, 0};
  const int np = Ly.pitch();
  const RBlk B{r0, r1, R, ny, np};
  extern __shared__ float4 res_dyn[];
  float *sm = reinterpret_cast<float *>(res_dyn);
  float *sLe = sm + Ly.field(0), *sLhx = sm + Ly.field(1), *sLhz = sm + Ly.field(2);
  float *sPx = sm + Ly.field(3), *sPz = sm + Ly.field(4), *sQx = sm + Ly.field(5),
        *sQz = sm + Ly.field(6);
  float *sMxh = sm + Ly.xmem(0), *sMxe = sm + Ly.xmem(1);
  float *sMzh = sm + Ly.zmem(0), *sMze = sm + Ly.zmem(1);
  const float *bt = sm + Ly.btab();
  float *ringG = sm + Ly.ring_a(), *ringV = sm + Ly.ring_b();
  const CRows fPz = crows(cl, sPz, rank, cs), fQz = crows(cl, sQz, rank, cs);
  const BandTab T{a.Wx, a.Wz};
  const float cqs = a.cq_arr ? 0.f : __ldg(a.cq);
  const int64_t sb = (int64_t)s * a.numel;
  int gy[G], gc[G];
  V ca[G], cb[G], gca[G], gcb[G];
  SnapWords<SNAP, W> se[G], sc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int k = (int)threadIdx.x + g * NT;
    gy[g] = -1;
    gc[g] = 0;
    ca[g] = cb[g] = gca[g] = gcb[g] = zerov<W>();
    if (k < ng) {
      const int ly = k / nxw;
      gy[g] = r0 + ly;
      gc[g] = (k - ly * nxw) * W;
      const int64_t cell = sb + (int64_t)gy[g] * nx + gc[g];
      const int64_t mb = (a.batched ? sb : 0) + (int64_t)gy[g] * nx + gc[g];
      ca[g] = ldgv<W>(a.ca + mb);
      cb[g] = ldgv<W>(a.cb + mb);
      gca[g] = ldv<W>(a.gca + cell);
      gcb[g] = ldv<W>(a.gcb + cell);
    }
  }
  auto snap_at = [&](int t, int g) -> int64_t {
    return (int64_t)t * a.step_elems + ((int64_t)s * ny + gco<G>(gy[g])) * a.snap_pitch + gc[g];
  };
  // step t's snapshots of the thread's groups, into registers
  auto fetch_snap = [&](int t) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (gy[g] < 0) continue;
      se[g].load(a.snap_e, snap_at(t, g));
      sc[g].load(a.snap_c, snap_at(t, g));
    }
  };
  res_state<true>(a.st, sm, Ly, a.bt, s, r0, Rb, ny, a.numel);
  REnt src, rec;
  src.init(a.src, s, entry_range(a.src, s, r0, r1), a.csrc);
  rec.init(a.rec, s, entry_range(a.rec, s, r0, r1), a.crec);
  const int64_t fstep = (int64_t)a.S * a.src.n, rstep = (int64_t)a.S * a.rec.n;
  // adjoint steps [u0, u0 + cnt) of the source-gradient ring out
  auto flush = [&](int u0, int cnt) {
    if (!a.grad_f || !src.mine()) return;
    for (int u = u0; u < u0 + cnt; ++u)
      a.grad_f[(int64_t)(nt - 1 - u) * fstep + (int64_t)s * a.src.n + src.q.z] =
          ringG[(u & km) * a.csrc + threadIdx.x];
  };
  if (nt > 0) {
    fetch_snap(nt - 1);
    // the residuals of the last step enter the start state; each later
    // step's are added after the lambda_E update of the step before it in
    // adjoint order
    if (a.res) {
      REnt all = rec;  // every head of the block, directly
      all.C = 0;
      all.q = make_int4(0, 0, 0, -1);
      __syncthreads();
      res_inject<NT>(all, nullptr, a.res + (int64_t)(nt - 1) * rstep, s, a.rec.n, sLe, r0, np);
    }
  }
  cluster_sync();
  for (int t = nt - 1; t >= 0; --t) {
    const int u = nt - 1 - t, k = u & km;
    // ---- E nodes: the source gradient, px and pz; first the global
    // traffic, once a chunk: the last chunk's source gradients out, this
    // chunk's residual values and (ring) the next chunk's snapshots in
    RingLoad<KM> rl;
    const int kc = min(K, nt - u);
    const bool chunk = k == 0;
    if (chunk) {
      if (u > 0) flush(u - K, K);
      if (a.res)
        rl.load(rec, s, a.rec.n, kc, [&](int i) -> const float * {
          const int tt = t - i;  // the residuals of step tt - 1 follow step tt's lambda_E
          return tt >= 1 ? a.res + (int64_t)(tt - 1) * rstep : nullptr;
        });
    }
    if (a.grad_f)
      res_sample<NT>(src, ringG + k * a.csrc, a.grad_f + (int64_t)t * fstep, s, a.src.n, sLe, r0,
                     np);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (gy[g] < 0) continue;
      const int y = gco<G>(gy[g]), c = gco<G>(gc[g]), ly = y - r0;
      const V lam = ldv<W>(sLe + ly * np + 4 + c);
      V gv;
#pragma unroll
      for (int q = 0; q < W; ++q) gv.v[q] = cb[g].v[q] * lam.v[q];
      V pz, px = gv;
#pragma unroll
      for (int q = 0; q < W; ++q) pz.v[q] = -gv.v[q];
      const int zr = zband(y, ny, a.Wz);
      if (zr >= 0) {
        float *mp = sMze + ly * nx + c;
        V M = ldv<W>(mp);
        const float ay = bt[T.z(0) + zr], by = bt[T.z(1) + zr];
        const float rky = bt[T.z(2) + zr];
#pragma unroll
        for (int q = 0; q < W; ++q) {
          M.v[q] -= gv.v[q];
          pz.v[q] = fmaf(ay, M.v[q], -gv.v[q] * rky);
          M.v[q] *= by;
        }
        stv<W>(mp, M);
      }
      const int bc = xband(c, nx, a.Wx);
      if (bc >= 0) {
        float *mp = sMxe + ly * 2 * a.Wx + bc;
        V M = ldv<W>(mp);
        const V ax = ldv<W>(bt + T.x(0) + bc), bx = ldv<W>(bt + T.x(1) + bc);
        const V rk = ldv<W>(bt + T.x(2) + bc);
#pragma unroll
        for (int q = 0; q < W; ++q) {
          M.v[q] += gv.v[q];
          px.v[q] = fmaf(ax.v[q], M.v[q], gv.v[q] * rk.v[q]);
          M.v[q] *= bx.v[q];
        }
        stv<W>(mp, M);
      }
      stv<W>(sPx + ly * np + 4 + c, px);
      stv<W>(sPz + ly * np + 4 + c, pz);
    }
    if (chunk && a.res)
      rl.store(rec, kc, [&](int i) { return ringV + ((u + i) & km) * a.crec; });
    cluster_sync();
    // ---- H nodes: lambda_Hz, qx; lambda_Hx, qz
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (gy[g] < 0) continue;
      const int y = gco<G>(gy[g]), c = gco<G>(gc[g]), ly = y - r0;
      const int64_t mb = (a.batched ? sb : 0) + (int64_t)y * nx + c;
      const V cq = a.cq_arr ? ldgv<W>(a.cq + mb) : splatv<W>(cqs);
      // the z window of pz first with one group a thread (see the forward's
      // H phase); with three, after lambda_Hz (fewer live registers)
      V p[2 * P];  // p[j] = pz(y + P - j)
      if constexpr (G == 1) B.zwin<W, 2 * P, P>(fPz, y, c, p);
      {
        float w[12];
        xwin<W>(sPx + ly * np, c, w);
        float *hp = sLhz + ly * np + 4 + c;
        const V lhz_old = ldv<W>(hp);
        V lhz, v;
#pragma unroll
        for (int q = 0; q < W; ++q) {
          lhz.v[q] = lhz_old.v[q] - dh<P>(w, q, a.c.cx);
          v.v[q] = cq.v[q] * lhz.v[q];
        }
        stv<W>(hp, lhz);
        const int bc = xband(c, nx, a.Wx);
        if (bc >= 0) {
          float *mp = sMxh + ly * 2 * a.Wx + bc;
          V M = ldv<W>(mp);
          const V ah = ldv<W>(bt + T.x(3) + bc), bh = ldv<W>(bt + T.x(4) + bc);
          const V rk = ldv<W>(bt + T.x(5) + bc);
#pragma unroll
          for (int q = 0; q < W; ++q) {
            M.v[q] += v.v[q];
            const float vq = v.v[q];
            v.v[q] = fmaf(ah.v[q], M.v[q], vq * rk.v[q]);
            M.v[q] *= bh.v[q];
          }
          stv<W>(mp, M);
        }
        stv<W>(sQx + ly * np + 4 + c, v);
      }
      {
        if constexpr (G != 1) B.zwin<W, 2 * P, P>(fPz, y, c, p);
        float *hp = sLhx + ly * np + 4 + c;
        const V lhx = ldv<W>(hp);
        V lh, qz;
#pragma unroll
        for (int q = 0; q < W; ++q) {
          float d = 0.f;
#pragma unroll
          for (int k2 = 1; k2 <= P; ++k2)  // pz(y + k) - pz(y - k + 1)
            d = fmaf(a.c.cy[k2 - 1], p[P - k2].v[q] - p[P + k2 - 1].v[q], d);
          lh.v[q] = lhx.v[q] - d;
          qz.v[q] = -cq.v[q] * lh.v[q];
        }
        stv<W>(hp, lh);
        const int zr = zband(y, ny, a.Wz);
        if (zr >= 0) {
          float *mp = sMzh + ly * nx + c;
          V M = ldv<W>(mp);
          const float ayh = bt[T.z(3) + zr], byh = bt[T.z(4) + zr];
          const float rkyh = bt[T.z(5) + zr];
#pragma unroll
          for (int q = 0; q < W; ++q) {
            const float vq = qz.v[q];
            M.v[q] += vq;
            qz.v[q] = fmaf(ayh, M.v[q], vq * rkyh);
            M.v[q] *= byh;
          }
          stv<W>(mp, M);
        }
        stv<W>(sQz + ly * np + 4 + c, qz);
      }
    }
    cluster_sync();
    // ---- lambda_E, and the gradients of step t (lam = lambda_E^{t+1})
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (gy[g] < 0) continue;
      const int y = gco<G>(gy[g]), c = gco<G>(gc[g]), ly = y - r0;
      V qv[2 * P];
      B.zwin<W, 2 * P, P - 1>(fQz, y, c, qv);  // qv[j] = qz(y + P - 1 - j)
      float w[12];
      xwin<W>(sQx + ly * np, c, w);
      float *lp = sLe + ly * np + 4 + c;
      const V lam = ldv<W>(lp);
      {
        const V ev = se[g].get(), cv = sc[g].get();
        const bool rowmask = !a.grad_mask || (y >= a.n_pml && y < ny - a.n_pml);
#pragma unroll
        for (int q = 0; q < W; ++q) {
          const bool colmask = !a.grad_mask || (c + q >= a.n_pml && c + q < nx - a.n_pml);
          if (rowmask && colmask) {
            gca[g].v[q] = fmaf(ev.v[q], lam.v[q], gca[g].v[q]);
            gcb[g].v[q] = fmaf(cv.v[q], lam.v[q], gcb[g].v[q]);
          }
        }
      }
      V en;
#pragma unroll
      for (int q = 0; q < W; ++q) {
        // Ca lam rounded on its own (never fused with the subtraction below),
        // as the stencil kernel queues it for 2P - 1 rows
        const float cla = __fmul_rn(ca[g].v[q], lam.v[q]);
        float dz = 0.f;
#pragma unroll
        for (int k2 = 1; k2 <= P; ++k2)  // qz(y + k) - qz(y - k)
          dz = fmaf(a.c.cy[k2 - 1], qv[P - k2].v[q] - qv[P - 1 + k2].v[q], dz);
        en.v[q] = cla - di<P>(w, q, a.c.cx) - dz;
      }
      stv<W>(lp, en);
    }
    // registers: the snapshots of step t - 1 (the next cluster barrier is a
    // phase away)
    if (t > 0) fetch_snap(t - 1);
    // the residuals of step t - 1 at the receivers
    if (t > 0 && a.res) {
      __syncthreads();
      res_inject<NT>(rec, ringV + k * a.crec, a.res + (int64_t)(t - 1) * rstep, s, a.rec.n, sLe,
                     r0, np);
    }
    __syncthreads();
  }
  if (nt > 0) {
    const int u0 = (nt - 1) & ~km;
    flush(u0, nt - u0);
  }
  // no block leaves while a neighbour may still read its qz rows
  cluster_sync();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (gy[g] < 0) continue;
    const int64_t cell = sb + (int64_t)gy[g] * nx + gc[g];
    stv<W>(a.gca + cell, gca[g]);
    stv<W>(a.gcb + cell, gcb[g]);
  }
  res_state<false>(a.st, sm, Ly, a.bt, s, r0, Rb, ny, a.numel);
}

// One cluster of `cs` blocks per shot, `smem` bytes of dynamic shared memory
// per block.  A cluster of more than 8 blocks is beyond the portable limit
// and needs the kernel's opt-in.
// (Set on every launch, two calls: attributes belong to the context, which
// a device reset replaces.)
template <typename K>
cudaError_t set_attrs(K kern, int cs, size_t smem) {
  if (cs > 8) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  if (smem > 48 * 1024)
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return cudaSuccess;
}
template <typename K>
cudaLaunchConfig_t cluster_cfg(K, unsigned blocks, int nt, int cs, size_t smem, cudaStream_t st,
                               cudaLaunchAttribute *attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3((unsigned)nt);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
template <typename K>
cudaError_t cluster_launch(K kern, const SmallArgs &a, int nt, int cs, size_t smem,
                           cudaStream_t st) {
  cudaError_t e = set_attrs(kern, cs, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = cluster_cfg(kern, (unsigned)(a.S * cs), nt, cs, smem, st, attr);
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}
// Whether a cluster of cs blocks of the kernel fits on the device.
template <typename K>
bool cluster_fits(K kern, int nt, int cs, size_t smem) {
  if (set_attrs(kern, cs, smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = cluster_cfg(kern, (unsigned)cs, nt, cs, smem, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return n > 0;
}

// The kernel of a launch: L2 variant with NT threads, or resident with
// (NT, G, W) = (128, 1, 4), (256, 1, 4), (512, 3, 4) or (256, 1, 2).
template <int P, int NT, int G, bool RES, int W = 4>
struct SmallKern {
  template <int STORE>
  static void *fwd_k() {
    if constexpr (RES) return (void *)k_res_fwd<P, STORE, NT, G, W>;
    else return (void *)k_small_fwd<P, STORE, NT>;
  }
  template <int SNAP>
  static void *adj_k() {
    if constexpr (RES) return (void *)k_res_adj<P, SNAP, NT, G, W>;
    else return (void *)k_small_adj<P, SNAP, NT>;
  }
  static void *fwd(int store) {
    switch (store) {
      case kStoreNone: return fwd_k<kStoreNone>();
      case kStoreF32: return fwd_k<kStoreF32>();
      case kStoreBF16: return fwd_k<kStoreBF16>();
      case kStoreFP8: return fwd_k<kStoreFP8>();
    }
    return nullptr;
  }
  static void *adj(int store) {
    switch (store) {
      case kStoreF32: return adj_k<kStoreF32>();
      case kStoreBF16: return adj_k<kStoreBF16>();
      case kStoreFP8: return adj_k<kStoreFP8>();
    }
    return nullptr;
  }
};
template <int P>
void *small_kernel(const SmallPlan &pl, bool adjoint, int store) {
  using R0 = SmallKern<P, 128, 1, true>;
  using R1 = SmallKern<P, 256, 1, true>;
  using R2 = SmallKern<P, 256, 1, true, 2>;
  using R3 = SmallKern<P, 512, 3, true>;
  using L256 = SmallKern<P, 256, 1, false>;
  using L1024 = SmallKern<P, 1024, 1, false>;
  if (pl.resident) {
    if (pl.width == 2) return adjoint ? R2::adj(store) : R2::fwd(store);
    if (pl.block == 128) return adjoint ? R0::adj(store) : R0::fwd(store);
    if (pl.block == 256) return adjoint ? R1::adj(store) : R1::fwd(store);
    return adjoint ? R3::adj(store) : R3::fwd(store);
  }
  if (pl.block == 1024) return adjoint ? L1024::adj(store) : L1024::fwd(store);
  return adjoint ? L256::adj(store) : L256::fwd(store);
}
void *kernel_of(int order, const SmallPlan &pl, bool adjoint, int store) {
  switch (order) {
    case 2: return small_kernel<1>(pl, adjoint, store);
    case 4: return small_kernel<2>(pl, adjoint, store);
    case 6: return small_kernel<3>(pl, adjoint, store);
    case 8: return small_kernel<4>(pl, adjoint, store);
  }
  return nullptr;
}

int env_int(const char *name, int dflt) {
  const char *e = getenv(name);
  return e && e[0] ? atoi(e) : dflt;
}

}  // namespace

// Resident when a block's rows of every array fit in shared memory and the
// device takes the cluster; else the L2 variant (16 blocks a shot where the
// device takes them, else the portable 8).  A resident block of one group a
// thread moves its global traffic in chunks of up to 8 steps (as many as
// shared memory holds), else one step at a time.  For tests and
// comparisons: MW_SMALL_CLUSTER caps the blocks a shot (at most 16),
// MW_SMALL_CHUNK the steps a chunk, MW_SMALL_WIDTH=4 keeps groups of 4 cells,
// and MW_SMALL_L2=1 forces the L2 variant.
bool small_plan_uncached(int order, bool adjoint, int store, int ny, int nx, int Wx, int Wz,
                         int n_src, int n_rec, SmallPlan *pl);

// (Plans are remembered per device, shape and test setting.)
bool small_plan(int order, bool adjoint, int store, int ny, int nx, int Wx, int Wz, int n_src,
                int n_rec, SmallPlan *pl) {
  using Key = std::tuple<int, int, int, int, int, int, int, int, int, int, int, int, int, int>;
  static std::mutex mu;
  static std::map<Key, std::pair<bool, SmallPlan>> plans;
  int dev = 0;
  cudaGetDevice(&dev);
  const Key key{dev, order, adjoint ? 1 : 0, store, ny, nx, Wx, Wz, n_src, n_rec,
                env_int("MW_SMALL_CLUSTER", 16), env_int("MW_SMALL_CHUNK", 8),
                env_int("MW_SMALL_WIDTH", 2) * 2 + env_int("MW_SMALL_L2", 0), 0};
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = plans.find(key);
    if (it != plans.end()) {
      *pl = it->second.second;
      return it->second.first;
    }
  }
  SmallPlan p{};
  const bool ok = small_plan_uncached(order, adjoint, store, ny, nx, Wx, Wz, n_src, n_rec, &p);
  std::lock_guard<std::mutex> lk(mu);
  plans[key] = {ok, p};
  *pl = p;
  return ok;
}

bool small_plan_uncached(int order, bool adjoint, int store, int ny, int nx, int Wx, int Wz,
                         int n_src, int n_rec, SmallPlan *pl) {
  const int P = order / 2;
  const int cap = std::max(1, std::min(16, env_int("MW_SMALL_CLUSTER", 16)));
  int kcap = 8;  // a power of two
  while (kcap > std::max(1, env_int("MW_SMALL_CHUNK", 8))) kcap /= 2;
  int optin = 0, dev = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    cudaGetLastError();
    optin = 0;
  }
  if (env_int("MW_SMALL_L2", 0) != 1) {
    for (int cmax = cap; cmax >= 1; cmax = cmax > 8 ? 8 : 0) {
      SmallPlan c{};
      c.resident = true;
      c.rows = std::max((ny + cmax - 1) / cmax, P);
      c.cluster = (ny + c.rows - 1) / c.rows;
      const int64_t groups = (int64_t)c.rows * (nx / 4);
      if (groups > 1536) break;  // fewer blocks only make it larger
      // groups of 2 cells where a 256-thread block then takes one group a
      // thread (more warps on a small block), else of 4
      c.width = (int64_t)c.rows * (nx / 2) <= 256 && env_int("MW_SMALL_WIDTH", 2) != 4 ? 2 : 4;
      c.block = c.width == 2 ? 256 : groups <= 128 ? 128 : groups <= 256 ? 256 : 512;
      const bool one = c.block <= 256;  // one group a thread
      c.csrc = std::max(0, std::min(n_src, c.block));
      c.crec = std::max(0, std::min(n_rec, c.block));
      const int eb = stage_bytes(store);
      bool fit = false;
      for (c.kchunk = one ? kcap : 1; c.kchunk >= 1; c.kchunk /= 2) {
        const int ns = adjoint ? 0 : (eb ? c.kchunk : 0);
        const ResLayout Ly{c.rows, nx, Wx, Wz, adjoint ? kResFieldsAdj : kResFieldsFwd,
                           c.kchunk, c.csrc, c.crec, eb, ns};
        c.smem = (size_t)Ly.floats() * sizeof(float);
        if ((int64_t)c.smem + 1024 <= optin) {
          fit = true;
          break;
        }
      }
      if (!fit) break;
      void *k = kernel_of(order, c, adjoint, store);
      if (k && cluster_fits(k, c.block, c.cluster, c.smem)) {
        *pl = c;
        return true;
      }
    }
  }
  SmallPlan c{};
  c.resident = false;
  c.width = 4;
  c.block = (int64_t)ny * (nx / 4) <= (int64_t)std::min(16, cap) * 256 ? 256 : 1024;
  for (int cs : {std::min(16, cap), std::min(8, cap)}) {
    c.cluster = cs;
    void *k = kernel_of(order, c, adjoint, store);
    if (k && cluster_fits(k, c.block, cs, 0)) {
      *pl = c;
      return true;
    }
  }
  return false;
}

cudaError_t launch_small(const SmallArgs &a, bool adjoint, int order, int store,
                         const SmallPlan &pl, cudaStream_t st) {
  void *k = kernel_of(order, pl, adjoint, store);
  if (!k) return cudaErrorInvalidValue;
  SmallArgs b = a;
  b.rows = pl.rows;
  b.kchunk = pl.kchunk;
  b.csrc = pl.csrc;
  b.crec = pl.crec;
  return cluster_launch(reinterpret_cast<void (*)(SmallArgs)>(k), b, pl.block, pl.cluster, pl.smem,
                        st);
}

}  // namespace mw
