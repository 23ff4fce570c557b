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
// Work decomposition ("marching strips"): one warp owns a 128-column strip
// (32 lanes x float4) of one shot over a chunk of rows and walks it top to
// bottom.  Per row it reads each state value once: the y-stencil operands
// (Ey rows for Hx, Hx rows for the E update) live in register queues, the
// x-stencil operands (one Ey row, a ring of 2P Hz rows) in per-warp shared
// memory, with 8 Ey halo columns and 4 Hz halo columns recomputed at each
// strip edge.  States are ping-ponged between two buffers so halo recompute
// never races with a neighbour's writes.  CPML memories exist only in the
// bands and are touched only by warps whose rows / columns lie in them.
#include <cuda_bf16.h>

#include "mw_internal.cuh"

namespace mw {
namespace {

struct F4 {
  float v[4];
};

__device__ __forceinline__ F4 zero4() { return F4{{0.f, 0.f, 0.f, 0.f}}; }

__device__ __forceinline__ F4 ld4(const float *p) {
  float4 t = __ldg(reinterpret_cast<const float4 *>(p));
  return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ F4 ld4rw(const float *p) {
  float4 t = *reinterpret_cast<const float4 *>(p);
  return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ void st4(float *p, const F4 &a) {
  *reinterpret_cast<float4 *>(p) = make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
}
__device__ __forceinline__ float4 as_f4(const F4 &a) {
  return make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
}
__device__ __forceinline__ void win12(const float4 *p, float w[12]) {
  float4 a = p[0], b = p[1], c = p[2];
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  w[8] = c.x; w[9] = c.y; w[10] = c.z; w[11] = c.w;
}

// Snapshot row store / load (4 consecutive cells), float32 or bf16 (RNE).
template <int STORE>
__device__ __forceinline__ void snap_store(void *base, int64_t off, const F4 &v) {
  if constexpr (STORE == kStoreF32) {
    st4(reinterpret_cast<float *>(base) + off, v);
  } else if constexpr (STORE == kStoreBF16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.v[0], v.v[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.v[2], v.v[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&lo);
    pk.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(base) + off) = pk;
  }
}
template <bool BF16>
__device__ __forceinline__ F4 snap_load(const void *base, int64_t off) {
  if constexpr (!BF16) {
    return ld4(reinterpret_cast<const float *>(base) + off);
  } else {
    uint2 pk = __ldg(reinterpret_cast<const uint2 *>(
        reinterpret_cast<const __nv_bfloat16 *>(base) + off));
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&pk.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&pk.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return F4{{a.x, a.y, b.x, b.y}};
  }
}

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
  if (c < Wx) return c;
  if (c >= nx - Wx) return c - nx + 2 * Wx;
  return -1;
}
__device__ __forceinline__ int zband_row(int r, int ny, int Wz) {
  if (r < Wz) return r;
  if (r >= ny - Wz) return r - ny + 2 * Wz;
  return -1;
}

// Common per-item set-up shared by both kernels.
struct Item {
  int s, x0, ya, yb, xo;
  bool own_ok;
  int e_hslot, e_hx;  // Ey halo float4 of lanes 0..3: slots 0,1,34,35
  bool e_h;
  int h_hslot, h_hx;  // Hz halo float4 of lanes 0,1: slots 0, 33
  bool h_h;
  int64_t sb, mb, xbw, zbw;
  int bown, bhal_h, bhal_e;  // x-band column of own, Hz-halo, Ey-halo float4
};

__device__ __forceinline__ bool make_item(const Geom &g, int item, int lane, bool batched,
                                          Item &it) {
  it.s = item % g.S;
  const int rest = item / g.S;
  const int strip = rest % g.n_strips;
  const int chunk = rest / g.n_strips;
  it.x0 = strip * kStripCols;
  it.ya = chunk * g.chunk_h;
  it.yb = min(g.ny, it.ya + g.chunk_h);
  if (it.ya >= it.yb) return false;
  it.xo = it.x0 + 4 * lane;
  it.own_ok = it.xo < g.nx;
  it.e_hslot = lane < 2 ? lane : 32 + lane;
  it.e_hx = it.x0 + 4 * (it.e_hslot - 2);
  it.e_h = lane < 4 && it.e_hx >= 0 && it.e_hx < g.nx;
  it.h_hslot = lane == 0 ? 0 : 33;
  it.h_hx = it.x0 + 4 * (it.h_hslot - 1);
  it.h_h = lane < 2 && it.h_hx >= 0 && it.h_hx < g.nx;
  it.sb = (int64_t)it.s * g.numel;
  it.mb = batched ? it.sb : 0;
  it.xbw = (int64_t)it.s * g.ny * 2 * g.Wx;
  it.zbw = (int64_t)it.s * 2 * g.Wz * g.nx;
  it.bown = it.own_ok ? xband_col(it.xo, g.nx, g.Wx) : -1;
  it.bhal_h = it.h_h ? xband_col(it.h_hx, g.nx, g.Wx) : -1;
  it.bhal_e = it.e_h ? xband_col(it.e_hx, g.nx, g.Wx) : -1;
  return true;
}

// ---------------------------------------------------------------------------
// Forward: H update of one Hz float4 at half nodes xb..xb+3 (+1/2) on row r.
template <int P>
__device__ __forceinline__ F4 hz_float4(const StepArgs &a, const float4 *ewin, const F4 &hz_old,
                                        const F4 &cq, int band_col, int xb, int64_t mem_off,
                                        bool write_mem) {
  float w[12];
  win12(ewin, w);
  F4 out;
  if (band_col < 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) out.v[q] = fmaf(cq.v[q], d_half<P>(w, q, a.c.cx), hz_old.v[q]);
  } else {
    F4 m = ld4(a.in.mxh_node + mem_off);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = xb + q;
      float d = d_half<P>(w, q, a.c.cx);
      m.v[q] = fmaf(__ldg(a.pr.bxh + col), m.v[q], __ldg(a.pr.axh + col) * d);
      d = d / __ldg(a.pr.kxh + col) + m.v[q];
      out.v[q] = fmaf(cq.v[q], d, hz_old.v[q]);
    }
    if (write_mem) st4(a.out.mxh_node + mem_off, m);
  }
  return out;
}

template <int P, int STORE>
__global__ void __launch_bounds__(128) k_forward(const StepArgs a, const int batched,
                                                 const int cq_arr) {
  constexpr int NQ = 2 * P;
  extern __shared__ float4 smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  float4 *es = smem + warp * (2 * kEySlots + NQ * kHzSlots);
  float4 *hs = es + 2 * kEySlots;
  const Geom &g = a.g;
  const int nx = g.nx, ny = g.ny;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  const int stride = gridDim.x * kWarpsPerCta;
  const float cqs = cq_arr ? 0.f : __ldg(a.cq);

  for (int item = blockIdx.x * kWarpsPerCta + warp; item < n_items; item += stride) {
    Item it;
    if (!make_item(g, item, lane, batched != 0, it)) continue;
    F4 eq[NQ], hq[NQ];
#pragma unroll
    for (int k = 0; k < NQ; ++k) eq[k] = hq[k] = zero4();
    const int r0 = it.ya - (2 * P - 1);
    const int n_it = (it.yb - it.ya) + 4 * P - 2;

    for (int i0 = 0; i0 < n_it; i0 += NQ) {
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        if (i0 + u < n_it) {
          const int r = r0 + i0 + u;
          const bool r_in = r >= 0 && r < ny;
          const bool hz_row = r >= it.ya && r < it.yb;
          const int rh = r - P;
          const bool hx_need = rh >= it.ya - P && rh <= it.yb + P - 2;
          const bool hx_in = hx_need && rh >= 0 && rh < ny;
          const int y = r - 2 * P + 1;
          const bool e_row = y >= it.ya && y < it.yb;

          // ---- global loads of this row (issued together)
          F4 e_own = zero4(), e_hal = zero4();
          if (r_in && it.own_ok) e_own = ld4(a.in.ey + it.sb + (int64_t)r * nx + it.xo);
          if (r_in && it.e_h) e_hal = ld4(a.in.ey + it.sb + (int64_t)r * nx + it.e_hx);
          F4 hz_own = zero4(), hz_hal = zero4(), cqh_own, cqh_hal;
          if (hz_row) {
            if (it.own_ok) hz_own = ld4(a.in.hz + it.sb + (int64_t)r * nx + it.xo);
            if (it.h_h) hz_hal = ld4(a.in.hz + it.sb + (int64_t)r * nx + it.h_hx);
          }
          F4 hx_old = zero4(), cqx;
          if (hx_in && it.own_ok) hx_old = ld4(a.in.hx + it.sb + (int64_t)rh * nx + it.xo);
          F4 ca4 = zero4(), cb4 = zero4();
          if (e_row && it.own_ok) {
            ca4 = ld4(a.ca + it.mb + (int64_t)y * nx + it.xo);
            cb4 = ld4(a.cb + it.mb + (int64_t)y * nx + it.xo);
          }
          if (cq_arr) {
            cqh_own = (hz_row && it.own_ok) ? ld4(a.cq + it.mb + (int64_t)r * nx + it.xo) : zero4();
            cqh_hal = (hz_row && it.h_h) ? ld4(a.cq + it.mb + (int64_t)r * nx + it.h_hx) : zero4();
            cqx = (hx_in && it.own_ok) ? ld4(a.cq + it.mb + (int64_t)rh * nx + it.xo) : zero4();
          } else {
            cqh_own = cqh_hal = cqx = F4{{cqs, cqs, cqs, cqs}};
          }

          // ---- Ey row into shared memory and the register queue
          float4 *er = es + (u & 1) * kEySlots;
          er[2 + lane] = as_f4(e_own);
          if (lane < 4) er[it.e_hslot] = as_f4(e_hal);
          eq[u] = e_own;
          __syncwarp();

          // ---- Hz update, row r (own + halo float4)
          if (hz_row) {
            float4 *hr = hs + u * kHzSlots;
            const int64_t moff = it.xbw + (int64_t)r * 2 * g.Wx;
            F4 hn = hz_float4<P>(a, er + lane + 1, hz_own, cqh_own, it.bown, it.xo,
                                 moff + it.bown, true);
            if (it.own_ok) st4(a.out.hz + it.sb + (int64_t)r * nx + it.xo, hn);
            hr[1 + lane] = it.own_ok ? as_f4(hn) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane < 2) {
              F4 hh = hz_float4<P>(a, er + (lane == 0 ? 0 : 33), hz_hal, cqh_hal, it.bhal_h,
                                   it.h_hx, moff + it.bhal_h, false);
              hr[it.h_hslot] = it.h_h ? as_f4(hh) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }

          // ---- Hx update, row rh = r - P (own float4, z-stencil from the queue)
          if (hx_need) {
            F4 hn = zero4();
            if (hx_in && it.own_ok) {
              const int zr = zband_row(rh, ny, g.Wz);
              F4 m;
              int64_t moff = 0;
              if (zr >= 0) {
                moff = it.zbw + (int64_t)zr * nx + it.xo;
                m = ld4(a.in.mzh_node + moff);
              }
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float d = 0.f;
#pragma unroll
                for (int k = 1; k <= P; ++k)
                  d = fmaf(a.c.cy[k - 1],
                           eq[(u - P + k + NQ) % NQ].v[q] - eq[(u - P - k + 1 + 2 * NQ) % NQ].v[q], d);
                if (zr >= 0) {
                  m.v[q] = fmaf(__ldg(a.pr.byh + rh), m.v[q], __ldg(a.pr.ayh + rh) * d);
                  d = d / __ldg(a.pr.kyh + rh) + m.v[q];
                }
                hn.v[q] = fmaf(-cqx.v[q], d, hx_old.v[q]);
              }
              if (rh >= it.ya && rh < it.yb) {
                st4(a.out.hx + it.sb + (int64_t)rh * nx + it.xo, hn);
                if (zr >= 0) st4(a.out.mzh_node + moff, m);
              }
            }
            hq[u] = hn;
          }

          // ---- E update, row y = r - 2P + 1
          if (e_row && it.own_ok) {
            float w[12];
            win12(hs + ((u + 1) % NQ) * kHzSlots + lane, w);
            const int zr = zband_row(y, ny, g.Wz);
            F4 mx, mz;
            const int64_t mxoff = it.xbw + (int64_t)y * 2 * g.Wx + it.bown;
            const int64_t mzoff = it.zbw + (int64_t)zr * nx + it.xo;
            if (it.bown >= 0) mx = ld4(a.in.mxe_node + mxoff);
            if (zr >= 0) mz = ld4(a.in.mze_node + mzoff);
            const F4 &e_old = eq[(u + 1) % NQ];
            F4 curl, en;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float cx = d_int<P>(w, q, a.c.cx);
              float cz = 0.f;
#pragma unroll
              for (int k = 1; k <= P; ++k)
                cz = fmaf(a.c.cy[k - 1],
                          hq[(u + P + k) % NQ].v[q] - hq[(u + 1 + P - k) % NQ].v[q], cz);
              if (it.bown >= 0) {
                const int col = it.xo + q;
                mx.v[q] = fmaf(__ldg(a.pr.bx + col), mx.v[q], __ldg(a.pr.ax + col) * cx);
                cx = cx / __ldg(a.pr.kx + col) + mx.v[q];
              }
              if (zr >= 0) {
                mz.v[q] = fmaf(__ldg(a.pr.by + y), mz.v[q], __ldg(a.pr.ay + y) * cz);
                cz = cz / __ldg(a.pr.ky + y) + mz.v[q];
              }
              curl.v[q] = cx - cz;
              en.v[q] = fmaf(ca4.v[q], e_old.v[q], cb4.v[q] * curl.v[q]);
            }
            const int64_t off = it.sb + (int64_t)y * nx + it.xo;
            if constexpr (STORE != kStoreNone) {
              snap_store<STORE>(a.snap_e, off, e_old);
              snap_store<STORE>(a.snap_c, off, curl);
            }
            st4(a.out.ey + off, en);
            if (it.bown >= 0) st4(a.out.mxe_node + mxoff, mx);
            if (zr >= 0) st4(a.out.mze_node + mzoff, mz);
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Adjoint: transposed E-node CPML recursion for the x direction of one float4
// (g = Cb lam at 4 E nodes).  Returns px; updates the memory when asked.
__device__ __forceinline__ F4 px_float4(const StepArgs &a, const F4 &g, int band_col, int xb,
                                        int64_t mem_off, bool write_mem) {
  if (band_col < 0) return g;
  F4 M = ld4(a.in.mxe_node + mem_off);
  F4 p;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int col = xb + q;
    M.v[q] += g.v[q];
    p.v[q] = fmaf(__ldg(a.pr.ax + col), M.v[q], g.v[q] / __ldg(a.pr.kx + col));
    M.v[q] *= __ldg(a.pr.bx + col);
  }
  if (write_mem) st4(a.out.mxe_node + mem_off, M);
  return p;
}

// Adjoint H update of one lamHz float4 (half nodes) and its transposed CPML.
template <int P>
__device__ __forceinline__ F4 qx_float4(const StepArgs &a, const float4 *pwin, const F4 &lhz_old,
                                        const F4 &cq, int band_col, int xb, int64_t mem_off,
                                        bool own, float *lhz_out) {
  float w[12];
  win12(pwin, w);
  F4 lhz, v;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    lhz.v[q] = lhz_old.v[q] - d_half<P>(w, q, a.c.cx);
    v.v[q] = cq.v[q] * lhz.v[q];
  }
  if (own) st4(lhz_out, lhz);
  if (band_col < 0) return v;
  F4 M = ld4(a.in.mxh_node + mem_off);
  F4 qx;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int col = xb + q;
    M.v[q] += v.v[q];
    qx.v[q] = fmaf(__ldg(a.pr.axh + col), M.v[q], v.v[q] / __ldg(a.pr.kxh + col));
    M.v[q] *= __ldg(a.pr.bxh + col);
  }
  if (own) st4(a.out.mxh_node + mem_off, M);
  return qx;
}

template <int P, bool BF16>
__global__ void __launch_bounds__(128) k_adjoint(const StepArgs a, const int batched,
                                                 const int cq_arr) {
  constexpr int NQ = 2 * P;
  extern __shared__ float4 smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  float4 *es = smem + warp * (2 * kEySlots + NQ * kHzSlots);
  float4 *hs = es + 2 * kEySlots;
  const Geom &g = a.g;
  const int nx = g.nx, ny = g.ny;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  const int stride = gridDim.x * kWarpsPerCta;
  const float cqs = cq_arr ? 0.f : __ldg(a.cq);

  for (int item = blockIdx.x * kWarpsPerCta + warp; item < n_items; item += stride) {
    Item it;
    if (!make_item(g, item, lane, batched != 0, it)) continue;
    F4 pq[NQ], qq[NQ];
#pragma unroll
    for (int k = 0; k < NQ; ++k) pq[k] = qq[k] = zero4();
    const int r0 = it.ya - (2 * P - 1);
    const int n_it = (it.yb - it.ya) + 4 * P - 2;
    // gradient mask: per-column part is fixed for the item
    bool colmask[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      colmask[q] = !g.grad_mask || (it.xo + q >= g.n_pml && it.xo + q < nx - g.n_pml);

    for (int i0 = 0; i0 < n_it; i0 += NQ) {
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        if (i0 + u < n_it) {
          const int r = r0 + i0 + u;
          const bool r_in = r >= 0 && r < ny;
          const bool own_row = r >= it.ya && r < it.yb;
          const int rh = r - P;
          const bool hx_need = rh >= it.ya - P && rh <= it.yb + P - 2;
          const bool hx_in = hx_need && rh >= 0 && rh < ny;
          const int y = r - 2 * P + 1;
          const bool e_row = y >= it.ya && y < it.yb;

          // ---- loads
          F4 lam = zero4(), cbv = zero4(), lam_h = zero4(), cb_h = zero4();
          const int64_t roff = it.sb + (int64_t)r * nx;
          const int64_t rmoff = it.mb + (int64_t)r * nx;
          if (r_in && it.own_ok) {
            lam = ld4(a.in.ey + roff + it.xo);
            cbv = ld4(a.cb + rmoff + it.xo);
          }
          if (own_row && it.e_h) {
            lam_h = ld4(a.in.ey + roff + it.e_hx);
            cb_h = ld4(a.cb + rmoff + it.e_hx);
          }
          F4 lhz = zero4(), lhz_h = zero4(), cqh_own, cqh_hal;
          F4 se = zero4(), sc = zero4(), gca = zero4(), gcb = zero4();
          if (own_row) {
            if (it.own_ok) {
              lhz = ld4(a.in.hz + roff + it.xo);
              se = snap_load<BF16>(a.snap_e, roff + it.xo);
              sc = snap_load<BF16>(a.snap_c, roff + it.xo);
              gca = ld4rw(a.gca + roff + it.xo);
              gcb = ld4rw(a.gcb + roff + it.xo);
            }
            if (it.h_h) lhz_h = ld4(a.in.hz + roff + it.h_hx);
          }
          F4 lhx = zero4(), cqx;
          if (hx_in && it.own_ok) lhx = ld4(a.in.hx + it.sb + (int64_t)rh * nx + it.xo);
          F4 ca4 = zero4(), lam_y = zero4();
          if (e_row && it.own_ok) {
            ca4 = ld4(a.ca + it.mb + (int64_t)y * nx + it.xo);
            lam_y = ld4(a.in.ey + it.sb + (int64_t)y * nx + it.xo);
          }
          if (cq_arr) {
            cqh_own = (own_row && it.own_ok) ? ld4(a.cq + rmoff + it.xo) : zero4();
            cqh_hal = (own_row && it.h_h) ? ld4(a.cq + rmoff + it.h_hx) : zero4();
            cqx = (hx_in && it.own_ok) ? ld4(a.cq + it.mb + (int64_t)rh * nx + it.xo) : zero4();
          } else {
            cqh_own = cqh_hal = cqx = F4{{cqs, cqs, cqs, cqs}};
          }

          // ---- gradients (lam is lambda_E^{t+1}), own cells of own rows
          if (own_row && it.own_ok) {
            const bool rowmask = !g.grad_mask || (r >= g.n_pml && r < ny - g.n_pml);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (rowmask && colmask[q]) {
                gca.v[q] = fmaf(se.v[q], lam.v[q], gca.v[q]);
                gcb.v[q] = fmaf(sc.v[q], lam.v[q], gcb.v[q]);
              }
            }
            st4(a.gca + roff + it.xo, gca);
            st4(a.gcb + roff + it.xo, gcb);
          }

          // ---- px (x-stencil operand, own rows) and pz (queue) at E nodes
          F4 gown;
#pragma unroll
          for (int q = 0; q < 4; ++q) gown.v[q] = cbv.v[q] * lam.v[q];
          float4 *er = es + (u & 1) * kEySlots;
          if (own_row) {
            const int64_t moff = it.xbw + (int64_t)r * 2 * g.Wx;
            F4 px = px_float4(a, gown, it.bown, it.xo, moff + it.bown, true);
            er[2 + lane] = it.own_ok ? as_f4(px) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane < 4) {
              F4 gh;
#pragma unroll
              for (int q = 0; q < 4; ++q) gh.v[q] = cb_h.v[q] * lam_h.v[q];
              F4 ph = px_float4(a, gh, it.bhal_e, it.e_hx, moff + it.bhal_e, false);
              er[it.e_hslot] = it.e_h ? as_f4(ph) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
          {
            F4 pz = zero4();
            if (r_in && it.own_ok) {
              const int zr = zband_row(r, ny, g.Wz);
              if (zr < 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q) pz.v[q] = -gown.v[q];
              } else {
                const int64_t moff = it.zbw + (int64_t)zr * nx + it.xo;
                F4 M = ld4(a.in.mze_node + moff);
                const float ay = __ldg(a.pr.ay + r), by = __ldg(a.pr.by + r);
                const float ky = __ldg(a.pr.ky + r);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  M.v[q] -= gown.v[q];
                  pz.v[q] = fmaf(ay, M.v[q], -gown.v[q] / ky);
                  M.v[q] *= by;
                }
                if (own_row) st4(a.out.mze_node + moff, M);
              }
            }
            pq[u] = pz;
          }
          __syncwarp();

          // ---- lamHz, qx at row r (own + halo)
          if (own_row) {
            float4 *hr = hs + u * kHzSlots;
            const int64_t moff = it.xbw + (int64_t)r * 2 * g.Wx;
            F4 qx = qx_float4<P>(a, er + lane + 1, lhz, cqh_own, it.bown, it.xo, moff + it.bown,
                                 it.own_ok, a.out.hz + roff + it.xo);
            hr[1 + lane] = it.own_ok ? as_f4(qx) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane < 2) {
              F4 qh = qx_float4<P>(a, er + (lane == 0 ? 0 : 33), lhz_h, cqh_hal, it.bhal_h,
                                   it.h_hx, moff + it.bhal_h, false, nullptr);
              hr[it.h_hslot] = it.h_h ? as_f4(qh) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }

          // ---- lamHx, qz at row rh = r - P
          if (hx_need) {
            F4 qz = zero4();
            if (hx_in && it.own_ok) {
              const bool own_h = rh >= it.ya && rh < it.yb;
              F4 lh;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float d = 0.f;
#pragma unroll
                for (int k = 1; k <= P; ++k)
                  d = fmaf(a.c.cy[k - 1],
                           pq[(u - P + k + NQ) % NQ].v[q] - pq[(u - P - k + 1 + 2 * NQ) % NQ].v[q], d);
                lh.v[q] = lhx.v[q] - d;
                qz.v[q] = -cqx.v[q] * lh.v[q];
              }
              if (own_h) st4(a.out.hx + it.sb + (int64_t)rh * nx + it.xo, lh);
              const int zr = zband_row(rh, ny, g.Wz);
              if (zr >= 0) {
                const int64_t moff = it.zbw + (int64_t)zr * nx + it.xo;
                F4 M = ld4(a.in.mzh_node + moff);
                const float ayh = __ldg(a.pr.ayh + rh), byh = __ldg(a.pr.byh + rh);
                const float kyh = __ldg(a.pr.kyh + rh);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float v = qz.v[q];
                  M.v[q] += v;
                  qz.v[q] = fmaf(ayh, M.v[q], v / kyh);
                  M.v[q] *= byh;
                }
                if (own_h) st4(a.out.mzh_node + moff, M);
              }
            }
            qq[u] = qz;
          }

          // ---- lamE at row y = r - 2P + 1
          if (e_row && it.own_ok) {
            float w[12];
            win12(hs + ((u + 1) % NQ) * kHzSlots + lane, w);
            F4 en;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float dz = 0.f;
#pragma unroll
              for (int k = 1; k <= P; ++k)
                dz = fmaf(a.c.cy[k - 1],
                          qq[(u + P + k) % NQ].v[q] - qq[(u + 1 + P - k) % NQ].v[q], dz);
              en.v[q] = ca4.v[q] * lam_y.v[q] - d_int<P>(w, q, a.c.cx) - dz;
            }
            st4(a.out.ey + it.sb + (int64_t)y * nx + it.xo, en);
          }
        }
      }
    }
  }
}

template <int P>
constexpr size_t smem_bytes() {
  return (size_t)kWarpsPerCta * (2 * kEySlots + 2 * P * kHzSlots) * sizeof(float4);
}

template <int P, int STORE>
cudaError_t fwd_t(const StepArgs &a, bool batched, bool cq_arr, int grid, cudaStream_t st) {
  k_forward<P, STORE><<<grid, 128, smem_bytes<P>(), st>>>(a, batched ? 1 : 0, cq_arr ? 1 : 0);
  count_launches(1);
  return cudaGetLastError();
}
template <int P, bool BF16>
cudaError_t adj_t(const StepArgs &a, bool batched, bool cq_arr, int grid, cudaStream_t st) {
  k_adjoint<P, BF16><<<grid, 128, smem_bytes<P>(), st>>>(a, batched ? 1 : 0, cq_arr ? 1 : 0);
  count_launches(1);
  return cudaGetLastError();
}

template <int P>
cudaError_t fwd_store(const StepArgs &a, int store, bool batched, bool cq_arr, int grid,
                      cudaStream_t st) {
  switch (store) {
    case kStoreNone: return fwd_t<P, kStoreNone>(a, batched, cq_arr, grid, st);
    case kStoreF32: return fwd_t<P, kStoreF32>(a, batched, cq_arr, grid, st);
    case kStoreBF16: return fwd_t<P, kStoreBF16>(a, batched, cq_arr, grid, st);
  }
  return cudaErrorInvalidValue;
}

template <typename K>
int occupancy(K kern, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 128, smem) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

}  // namespace

cudaError_t launch_forward(const StepArgs &a, int order, int store, bool batched, bool cq_array,
                           int grid, cudaStream_t st) {
  switch (order) {
    case 2: return fwd_store<1>(a, store, batched, cq_array, grid, st);
    case 4: return fwd_store<2>(a, store, batched, cq_array, grid, st);
    case 6: return fwd_store<3>(a, store, batched, cq_array, grid, st);
    case 8: return fwd_store<4>(a, store, batched, cq_array, grid, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_adjoint(const StepArgs &a, int order, int snap_bf16, bool batched,
                           bool cq_array, int grid, cudaStream_t st) {
  const bool b = snap_bf16 != 0;
  switch (order) {
    case 2: return b ? adj_t<1, true>(a, batched, cq_array, grid, st)
                     : adj_t<1, false>(a, batched, cq_array, grid, st);
    case 4: return b ? adj_t<2, true>(a, batched, cq_array, grid, st)
                     : adj_t<2, false>(a, batched, cq_array, grid, st);
    case 6: return b ? adj_t<3, true>(a, batched, cq_array, grid, st)
                     : adj_t<3, false>(a, batched, cq_array, grid, st);
    case 8: return b ? adj_t<4, true>(a, batched, cq_array, grid, st)
                     : adj_t<4, false>(a, batched, cq_array, grid, st);
  }
  return cudaErrorInvalidValue;
}

// Resident warps per SM of the stencil kernel for `order` (occupancy API).
int stencil_slots_per_sm(int order, bool adjoint) {
  int blocks = 1;
  switch (order) {
    case 2: blocks = adjoint ? occupancy(k_adjoint<1, false>, smem_bytes<1>())
                             : occupancy(k_forward<1, kStoreF32>, smem_bytes<1>()); break;
    case 4: blocks = adjoint ? occupancy(k_adjoint<2, false>, smem_bytes<2>())
                             : occupancy(k_forward<2, kStoreF32>, smem_bytes<2>()); break;
    case 6: blocks = adjoint ? occupancy(k_adjoint<3, false>, smem_bytes<3>())
                             : occupancy(k_forward<3, kStoreF32>, smem_bytes<3>()); break;
    case 8: blocks = adjoint ? occupancy(k_adjoint<4, false>, smem_bytes<4>())
                             : occupancy(k_forward<4, kStoreF32>, smem_bytes<4>()); break;
  }
  return blocks * kWarpsPerCta;
}

}  // namespace mw
