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
// step.  The state stays in place in global memory (it fits in L2); each
// shot gets a thread-block cluster (16 blocks, or the portable 8), whose
// threads own float4 groups of cells (row, 4 columns), and the steps' phases
// are separated by the cluster's hardware barrier.  Reads of anything the
// launch writes bypass L1 (ld.global.cg), since L1 is not coherent between
// blocks.  Every update,
// source sum and receiver sample is the stencil kernels' operation for
// operation, so the results are bitwise those of the step-by-step launches.
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
//   workspace arrays between the phases.
#include <cuda.h>

#include "mw_device.cuh"
#include "mw_internal.cuh"

namespace mw {
namespace {
using namespace dev;

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
// same for all of them).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
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

// One cluster of `cs` blocks per shot.  A cluster of 16 is beyond the
// portable limit of 8 and needs the kernel's opt-in.
template <int NT, typename K>
cudaError_t cluster_launch(K kern, const SmallArgs &a, int cs, cudaStream_t st) {
  if (cs > 8) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.S * cs));
  cfg.blockDim = dim3((unsigned)NT);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

// Whether clusters of cs blocks of the kernel fit on the device.
template <int NT, typename K>
bool cluster_fits(K kern, int cs) {
  if (cs > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                    cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cs);
  cfg.blockDim = dim3((unsigned)NT);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return n > 0;
}

template <int P, int NT>
cudaError_t small_t(const SmallArgs &a, bool adjoint, int store, int cs, cudaStream_t st) {
  if (adjoint) {
    switch (store) {
      case kStoreF32: return cluster_launch<NT>(k_small_adj<P, kStoreF32, NT>, a, cs, st);
      case kStoreBF16: return cluster_launch<NT>(k_small_adj<P, kStoreBF16, NT>, a, cs, st);
      case kStoreFP8: return cluster_launch<NT>(k_small_adj<P, kStoreFP8, NT>, a, cs, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (store) {
    case kStoreNone: return cluster_launch<NT>(k_small_fwd<P, kStoreNone, NT>, a, cs, st);
    case kStoreF32: return cluster_launch<NT>(k_small_fwd<P, kStoreF32, NT>, a, cs, st);
    case kStoreBF16: return cluster_launch<NT>(k_small_fwd<P, kStoreBF16, NT>, a, cs, st);
    case kStoreFP8: return cluster_launch<NT>(k_small_fwd<P, kStoreFP8, NT>, a, cs, st);
  }
  return cudaErrorInvalidValue;
}

template <int P>
cudaError_t small_p(const SmallArgs &a, bool adjoint, int store, int cs, int block,
                    cudaStream_t st) {
  return block == 1024 ? small_t<P, 1024>(a, adjoint, store, cs, st)
                       : small_t<P, 256>(a, adjoint, store, cs, st);
}

template <int P>
bool fits16_t(int block) {
  return block == 1024 ? cluster_fits<1024>(k_small_adj<P, kStoreF32, 1024>, 16) &&
                             cluster_fits<1024>(k_small_fwd<P, kStoreF32, 1024>, 16)
                       : cluster_fits<256>(k_small_adj<P, kStoreF32, 256>, 16) &&
                             cluster_fits<256>(k_small_fwd<P, kStoreF32, 256>, 16);
}

}  // namespace

void small_config(int order, int64_t groups_per_shot, int *block, int *cluster) {
  // 16 blocks per shot where the device takes them (else the portable 8);
  // 256 threads a block while that gives every thread a group, else 1024
  int cs = 16;
  *block = groups_per_shot <= 16 * 256 ? 256 : 1024;
  bool ok16 = false;
  switch (order) {
    case 2: ok16 = fits16_t<1>(*block); break;
    case 4: ok16 = fits16_t<2>(*block); break;
    case 6: ok16 = fits16_t<3>(*block); break;
    default: ok16 = fits16_t<4>(*block); break;
  }
  if (!ok16) cs = 8;
  *cluster = cs;
}

cudaError_t launch_small(const SmallArgs &a, bool adjoint, int order, int store, int cluster,
                         int block, cudaStream_t st) {
  switch (order) {
    case 2: return small_p<1>(a, adjoint, store, cluster, block, st);
    case 4: return small_p<2>(a, adjoint, store, cluster, block, st);
    case 6: return small_p<3>(a, adjoint, store, cluster, block, st);
    case 8: return small_p<4>(a, adjoint, store, cluster, block, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace mw
