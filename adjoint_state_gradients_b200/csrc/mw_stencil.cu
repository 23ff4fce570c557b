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
// outside the array; lane k issues load k) into a ring of L+1 shared-memory
// stages, L rows ahead of the row being computed, each tracked by an
// mbarrier with a bounded wait.  The y-stencil operands (Ey rows for Hx, Hx
// rows for the E update) live in register queues; the x-stencil operands
// come from the staged row and from a ring of 2P computed Hz rows.  States
// are ping-ponged between two buffers so halo recompute never races with a
// neighbour's writes.  CPML memories exist only in the bands and are fetched
// only where a row or strip lies in one.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

#include "mw_internal.cuh"

namespace mw {
namespace {

constexpr uint32_t kWaitPolls = 1u << 22;  // ~0.5 s of polling, then give up
constexpr unsigned kFull = 0xffffffffu;

// Stage layouts (float offsets, 128-byte aligned slots).
constexpr int kF_EY = 0, kF_HZ = 160, kF_HX = 288, kF_CA = 416, kF_CB = 544, kF_MZH = 672,
              kF_MZE = 800, kF_BAND = 928;
constexpr int kA_LAM = 0, kA_CB = 128, kA_LHZ = 256, kA_SE = 384, kA_SC = 512, kA_GCA = 640,
              kA_GCB = 768, kA_LHX = 896, kA_CA = 1024, kA_LAMY = 1152, kA_MZE = 1280,
              kA_MZH = 1408, kA_BAND = 1536;
constexpr int kFRing = 128;  // forward Hz ring row: 32 float4
constexpr int kAPx = 128;    // adjoint px row: 32 float4
constexpr int kARing = 120;  // adjoint qx ring row: 30 float4

template <int L>
struct Stages {
  static_assert(kWarpsPerCta * (L + 1) * 8 <= 128, "barrier area too small");
};

struct F4 {
  float v[4];
};

__device__ __forceinline__ F4 zero4() { return F4{{0.f, 0.f, 0.f, 0.f}}; }
__device__ __forceinline__ F4 lds4(const float *p) {
  float4 t = *reinterpret_cast<const float4 *>(p);
  return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ F4 ld4(const float *p) {
  float4 t = __ldg(reinterpret_cast<const float4 *>(p));
  return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ F4 splat4(float x) { return F4{{x, x, x, x}}; }
__device__ __forceinline__ void st4(float *p, const F4 &a) {
  *reinterpret_cast<float4 *>(p) = make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
}
__device__ __forceinline__ void win12(const float *p, float w[12]) {
  const float4 *q = reinterpret_cast<const float4 *>(p);
  float4 a = q[0], b = q[1], c = q[2];
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  w[8] = c.x; w[9] = c.y; w[10] = c.z; w[11] = c.w;
}

// ---- TMA / mbarrier primitives (PTX) ---------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of a stage barrier, called by all 32 lanes:
// every lane polls (acquire) and the warp votes, so the outcome is uniform.
// Returns false after the poll limit.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t k = 0; k < kWaitPolls; ++k) {
    if (__all_sync(kFull, mbar_test(bar, parity))) return true;
    if (k >= 32) __nanosleep(100);
  }
  return false;
}
__device__ __forceinline__ void tma3(float *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                     uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma4(float *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                     int c3, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar))
      : "memory");
}

// Snapshot row store (4 consecutive cells), float32 or bf16 (RNE).
template <int STORE>
__device__ __forceinline__ void snap_store(void *row, const F4 &v) {
  if constexpr (STORE == kStoreF32) {
    st4(reinterpret_cast<float *>(row), v);
  } else if constexpr (STORE == kStoreBF16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.v[0], v.v[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.v[2], v.v[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&lo);
    pk.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(row) = pk;
  }
}
// Staged snapshot values of own float4 o (float32 or bf16 in smem).
template <bool BF16>
__device__ __forceinline__ F4 snap_lds(const float *stage_row, int o) {
  if constexpr (!BF16) {
    return lds4(stage_row + 4 * o);
  } else {
    uint2 pk = *reinterpret_cast<const uint2 *>(
        reinterpret_cast<const __nv_bfloat16 *>(stage_row) + 4 * o);
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

// Rows a walk iteration touches: r (new Ey / lambda row), rh = r - P (H row
// updated in the z direction), y = r - 2P + 1 (E row updated).
template <int P>
struct Rows {
  int r, rh, y;
  bool own_r, hx_need, hx_in, e_row;
  __device__ __forceinline__ Rows(int r0, int i, int ya, int yb, int ny) {
    r = r0 + i;
    rh = r - P;
    y = r - 2 * P + 1;
    own_r = r >= ya && r < yb;
    hx_need = rh >= ya - P && rh <= yb + P - 2;
    hx_in = hx_need && rh >= 0 && rh < ny;
    e_row = y >= ya && y < yb;
  }
};

// Strip / chunk of one work item.
struct Item {
  int s, sm, x0, ya, yb, r0, n_it;
  bool xb;  // the strip (with its halo) touches an x band
};

template <int P>
__device__ __forceinline__ bool make_item(const Geom &g, int item, bool batched, Item &it) {
  it.s = item % g.S;
  const int rest = item / g.S;
  const int strip = rest % g.n_strips;
  const int chunk = rest / g.n_strips;
  it.sm = batched ? it.s : 0;
  it.x0 = strip * g.strip_cols;
  it.ya = chunk * g.chunk_h;
  it.yb = min(g.ny, it.ya + g.chunk_h);
  it.r0 = it.ya - (2 * P - 1);
  it.n_it = (it.yb - it.ya) + 4 * P - 2;
  it.xb = g.Wx > 0 && (it.x0 - 8 < g.Wx || it.x0 + g.strip_cols + 8 > g.nx - g.Wx);
  return it.ya < it.yb;
}

// ---------------------------------------------------------------------------
// forward

// Issue the TMA loads of walk iteration i into stage `st`: lane k issues load
// k (FwdLoad order; the per-lane operands are chosen with selects, not
// branches), lane 0 posts the expected byte count first.
template <int P>
__device__ __forceinline__ void fwd_issue(const FwdMaps &m, const Geom &g, const Item &it, int i,
                                          float *st, uint64_t *bar, int band_slot, int band_box,
                                          int lane) {
  const Rows<P> R(it.r0, i, it.ya, it.yb, g.ny);
  const int zh = R.hx_in ? zband_row(R.rh, g.ny, g.Wz) : -1;
  const int ze = R.e_row ? zband_row(R.y, g.ny, g.Wz) : -1;
  const bool l_ey = lane == kLdEy, l_hz = lane == kLdHz, l_hx = lane == kLdHx;
  const bool l_ca = lane == kLdCa, l_cb = lane == kLdCb, l_mxh = lane == kLdMxh;
  const bool l_mxe = lane == kLdMxe, l_mzh = lane == kLdMzh, l_mze = lane == kLdMze;
  const bool act = l_ey | (l_hz & R.own_r) | (l_hx & R.hx_in) | ((l_ca | l_cb) & R.e_row) |
                   (l_mxh & R.own_r & it.xb) | (l_mxe & R.e_row & it.xb) | (l_mzh & (zh >= 0)) |
                   (l_mze & (ze >= 0));
  const int c0 = l_ey ? it.x0 - 8 : l_hz ? it.x0 - 4 : (l_mxh | l_mxe) ? 0 : it.x0;
  const int c1 = l_hx ? R.rh : (l_ca | l_cb | l_mxe) ? R.y : l_mzh ? zh : l_mze ? ze : R.r;
  const int c2 = (l_ca | l_cb) ? it.sm : it.s;
  const int off = l_ey ? kF_EY : l_hz ? kF_HZ : l_hx ? kF_HX : l_ca ? kF_CA : l_cb ? kF_CB
                : l_mzh ? kF_MZH : l_mze ? kF_MZE : l_mxh ? kF_BAND : kF_BAND + band_slot;
  const uint32_t bytes = l_ey ? 136 * 4 : l_hz ? 128 * 4 : (l_mxh | l_mxe) ? band_box : 120 * 4;
  const uint32_t total = __reduce_add_sync(kFull, act ? bytes : 0u);
  if (lane == 0) mbar_expect_tx(bar, total);
  __syncwarp();
  if (act) {
    fence_proxy_async();
    tma3(st + off, &m.map[lane < kFwdLoads ? lane : 0], c0, c1, c2, bar);
  }
}

// Forward H update of one Hz float4 (half nodes c..c+3, +1/2) on row r;
// band_col >= 0: the float4 lies in the x band (memory row `mband`, table
// entries at band column band_col).
template <int P>
__device__ __forceinline__ F4 hz_float4(const StepArgs &a, const BandTab &T, const float *ewin,
                                        const F4 &hz_old, const F4 &cq, int band_col,
                                        const float *mband, F4 &m_new) {
  float w[12];
  win12(ewin, w);
  F4 out;
  if (band_col < 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) out.v[q] = fmaf(cq.v[q], d_half<P>(w, q, a.c.cx), hz_old.v[q]);
  } else {
    m_new = lds4(mband + band_col);
    const F4 ah = ld4(a.bt + T.x(3) + band_col), bh = ld4(a.bt + T.x(4) + band_col);
    const F4 rk = ld4(a.bt + T.x(5) + band_col);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float d = d_half<P>(w, q, a.c.cx);
      m_new.v[q] = fmaf(bh.v[q], m_new.v[q], ah.v[q] * d);
      out.v[q] = fmaf(cq.v[q], fmaf(d, rk.v[q], m_new.v[q]), hz_old.v[q]);
    }
  }
  return out;
}

template <int P, int STORE, int L>
__global__ void __launch_bounds__(128) k_forward(const __grid_constant__ FwdMaps m,
                                                 const StepArgs a, const int batched,
                                                 const int cq_arr) {
  constexpr int NQ = 2 * P;
  constexpr int NS = L + 1;
  (void)sizeof(Stages<L>);
  extern __shared__ float smem_raw[];
  float *smem = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem) + warp * NS;
  float *wb = smem + 32 + warp * a.warp_floats;
  float *hs = wb + NS * a.stage_floats;  // Hz ring: NQ rows of 32 float4
  const int band_slot = a.band_floats, band_box = a.band_box_floats * 4;
  const Geom &g = a.g;
  const int nx = g.nx, ny = g.ny;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  if (__any_sync(kFull, *reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0)) return;
  if (lane == 0) {
    for (int k = 0; k < NS; ++k) mbar_init(&bars[k], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const float cqs = cq_arr ? 0.f : __ldg(a.cq);
  const bool own_lane = lane >= 1 && lane <= 30;
  const int wl = own_lane ? lane : 1;  // window base for the E update
  const BandTab T{g.Wx, g.Wz};
  Ring ring{0, 0u};
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
    // this lane's column: Hz float4 at c; owned cells (lanes 1..30) also at c
    const int c = it.x0 - 4 + 4 * lane;
    const bool c_ok = c >= 0 && c < nx;
    const bool own = own_lane && c_ok;
    const int bcol = xband_col(c, nx, g.Wx);
    const int64_t sb = (int64_t)it.s * g.numel + c;  // + row * nx
    const int64_t mb = (int64_t)it.sm * g.numel + c;
    const int64_t xbw = (int64_t)it.s * ny * 2 * g.Wx + bcol;
    const int64_t zbw = (int64_t)it.s * 2 * g.Wz * nx + c;
    {
      Ring pr = ring;
      for (int j = 0; j < L && j < it.n_it; ++j) {
        fwd_issue<P>(m, g, it, j, wb + pr.slot * a.stage_floats, &bars[pr.slot], band_slot,
                     band_box, lane);
        pr.next(NS);
      }
    }
    F4 eq[NQ], hq[NQ];
#pragma unroll
    for (int k = 0; k < NQ; ++k) eq[k] = hq[k] = zero4();

    for (int i0 = 0; i0 < it.n_it; i0 += NQ) {
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        const int i = i0 + u;
        if (i < it.n_it) {
          if (i + L < it.n_it) {
            const int ps = ring.slot == 0 ? NS - 1 : ring.slot - 1;
            fwd_issue<P>(m, g, it, i + L, wb + ps * a.stage_floats, &bars[ps], band_slot,
                         band_box, lane);
          }
          const float *st = wb + ring.slot * a.stage_floats;
          if (!mbar_wait(&bars[ring.slot], ring.phase)) {
            // give up: flag it, let the copies in flight land, leave
            if (lane == 0) atomicOr(a.flags + kFlagTimeout, 1);
            Ring dr = ring;
            for (int j = i; j < it.n_it && j <= i + L; ++j) {
              mbar_wait(&bars[dr.slot], dr.phase);
              dr.next(NS);
            }
            return;
          }
          const Rows<P> R(it.r0, i, it.ya, it.yb, ny);
          const float *sey = st + kF_EY;
          eq[u] = lds4(sey + 4 * lane + 4);

          // ---- Hz update, row r: every lane, float4 at column c
          if (R.own_r) {
            const F4 cq = cq_arr ? (c_ok ? ld4(a.cq + mb + (int64_t)R.r * nx) : zero4()) : splat4(cqs);
            F4 mn;
            F4 hn = hz_float4<P>(a, T, sey + 4 * lane, lds4(st + kF_HZ + 4 * lane), cq, bcol,
                                 st + kF_BAND, mn);
            st4(hs + u * kFRing + 4 * lane, c_ok ? hn : zero4());
            if (own) {
              st4(a.out.hz + sb + (int64_t)R.r * nx, hn);
              if (bcol >= 0) st4(a.out.mxh_node + xbw + (int64_t)R.r * 2 * g.Wx, mn);
            }
          }

          // ---- Hx update, row rh (owned lanes; z-stencil from the Ey queue)
          if (R.hx_need) {
            F4 hn = zero4();
            if (R.hx_in) {
              const F4 hx_old = lds4(st + kF_HX + 4 * lane - 4);
              const F4 cq = cq_arr ? (own ? ld4(a.cq + mb + (int64_t)R.rh * nx) : zero4()) : splat4(cqs);
              const int zr = zband_row(R.rh, ny, g.Wz);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float d = 0.f;
#pragma unroll
                for (int k = 1; k <= P; ++k)
                  d = fmaf(a.c.cy[k - 1],
                           eq[(u - P + k + NQ) % NQ].v[q] - eq[(u - P - k + 1 + 2 * NQ) % NQ].v[q],
                           d);
                hn.v[q] = d;
              }
              if (zr >= 0) {
                F4 mz = lds4(st + kF_MZH + 4 * lane - 4);
                const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
                const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  mz.v[q] = fmaf(byh, mz.v[q], ayh * hn.v[q]);
                  hn.v[q] = fmaf(hn.v[q], rkyh, mz.v[q]);
                }
                if (own && R.rh >= it.ya && R.rh < it.yb)
                  st4(a.out.mzh_node + zbw + (int64_t)zr * nx, mz);
              }
#pragma unroll
              for (int q = 0; q < 4; ++q) hn.v[q] = fmaf(-cq.v[q], hn.v[q], hx_old.v[q]);
              if (own && R.rh >= it.ya && R.rh < it.yb) st4(a.out.hx + sb + (int64_t)R.rh * nx, hn);
            }
            hq[u] = hn;
          }

          // ---- E update, row y (owned lanes)
          if (R.e_row && own) {
            float w[12];
            win12(hs + ((u + 1) % NQ) * kFRing + 4 * wl - 4, w);
            const F4 ca4 = lds4(st + kF_CA + 4 * lane - 4);
            const F4 cb4 = lds4(st + kF_CB + 4 * lane - 4);
            const F4 &e_old = eq[(u + 1) % NQ];
            const int zr = zband_row(R.y, ny, g.Wz);
            F4 cx, cz;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              cx.v[q] = d_int<P>(w, q, a.c.cx);
              float d = 0.f;
#pragma unroll
              for (int k = 1; k <= P; ++k)
                d = fmaf(a.c.cy[k - 1], hq[(u + P + k) % NQ].v[q] - hq[(u + 1 + P - k) % NQ].v[q],
                         d);
              cz.v[q] = d;
            }
            if (bcol >= 0) {
              F4 mx = lds4(st + kF_BAND + band_slot + bcol);
              const F4 ax = ld4(a.bt + T.x(0) + bcol), bx = ld4(a.bt + T.x(1) + bcol);
              const F4 rk = ld4(a.bt + T.x(2) + bcol);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mx.v[q] = fmaf(bx.v[q], mx.v[q], ax.v[q] * cx.v[q]);
                cx.v[q] = fmaf(cx.v[q], rk.v[q], mx.v[q]);
              }
              st4(a.out.mxe_node + xbw + (int64_t)R.y * 2 * g.Wx, mx);
            }
            if (zr >= 0) {
              F4 mz = lds4(st + kF_MZE + 4 * lane - 4);
              const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
              const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                mz.v[q] = fmaf(by, mz.v[q], ay * cz.v[q]);
                cz.v[q] = fmaf(cz.v[q], rky, mz.v[q]);
              }
              st4(a.out.mze_node + zbw + (int64_t)zr * nx, mz);
            }
            F4 curl, en;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              curl.v[q] = cx.v[q] - cz.v[q];
              en.v[q] = fmaf(ca4.v[q], e_old.v[q], cb4.v[q] * curl.v[q]);
            }
            const int64_t off = sb + (int64_t)R.y * nx;
            if constexpr (STORE == kStoreF32) {
              snap_store<STORE>(reinterpret_cast<float *>(a.snap_e) + off, e_old);
              snap_store<STORE>(reinterpret_cast<float *>(a.snap_c) + off, curl);
            } else if constexpr (STORE == kStoreBF16) {
              snap_store<STORE>(reinterpret_cast<__nv_bfloat16 *>(a.snap_e) + off, e_old);
              snap_store<STORE>(reinterpret_cast<__nv_bfloat16 *>(a.snap_c) + off, curl);
            }
            st4(a.out.ey + off, en);
          }
          __syncwarp();
          ring.next(NS);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// adjoint

template <int P, bool BF16>
__device__ __forceinline__ void adj_issue(const AdjMaps &m, const StepArgs &a, const Geom &g,
                                          const Item &it, int i, float *st, uint64_t *bar,
                                          int band_slot, int band_box, int lane) {
  const Rows<P> R(it.r0, i, it.ya, it.yb, g.ny);
  const int ze = zband_row(R.r, g.ny, g.Wz);
  const int zh = R.hx_in ? zband_row(R.rh, g.ny, g.Wz) : -1;
  constexpr uint32_t snap_bytes = BF16 ? 112 * 2 : 112 * 4;
  const bool l_lam = lane == kLdLam, l_cb = lane == kLdCbA, l_lhz = lane == kLdLhz;
  const bool l_se = lane == kLdSe, l_sc = lane == kLdSc, l_gca = lane == kLdGca;
  const bool l_gcb = lane == kLdGcb, l_lhx = lane == kLdLhx, l_ca = lane == kLdCaA;
  const bool l_lamy = lane == kLdLamy, l_mxe = lane == kLdMxeA, l_mxh = lane == kLdMxhA;
  const bool l_mze = lane == kLdMzeA, l_mzh = lane == kLdMzhA;
  const bool l_own = l_lhz | l_se | l_sc | l_gca | l_gcb;
  const bool act = l_lam | l_cb | (l_own & R.own_r) | (l_lhx & R.hx_in) | ((l_ca | l_lamy) & R.e_row) |
                   ((l_mxe | l_mxh) & R.own_r & it.xb) | (l_mze & (ze >= 0)) | (l_mzh & (zh >= 0));
  const int c0 = (l_lam | l_cb) ? it.x0 - 8 : l_lhz ? it.x0 - 4 : (l_mxe | l_mxh) ? 0 : it.x0;
  const int c1 = l_lhx ? R.rh : (l_ca | l_lamy) ? R.y : l_mze ? ze : l_mzh ? zh : R.r;
  const int c2 = (l_cb | l_ca) ? it.sm : it.s;
  const int off = l_lam ? kA_LAM : l_cb ? kA_CB : l_lhz ? kA_LHZ : l_se ? kA_SE : l_sc ? kA_SC
                : l_gca ? kA_GCA : l_gcb ? kA_GCB : l_lhx ? kA_LHX : l_ca ? kA_CA
                : l_lamy ? kA_LAMY : l_mze ? kA_MZE : l_mzh ? kA_MZH : l_mxe ? kA_BAND
                : kA_BAND + band_slot;
  const uint32_t bytes = (l_lam | l_cb) ? 128 * 4 : l_lhz ? 120 * 4 : (l_se | l_sc) ? snap_bytes
                       : (l_mxe | l_mxh) ? band_box : 112 * 4;
  const uint32_t total = __reduce_add_sync(kFull, act ? bytes : 0u);
  if (lane == 0) mbar_expect_tx(bar, total);
  __syncwarp();
  if (act) {
    fence_proxy_async();
    const CUtensorMap *map = &m.map[lane < kAdjLoads ? lane : 0];
    if (l_se | l_sc)
      tma4(st + off, map, c0, c1, c2, a.snap_t, bar);
    else
      tma3(st + off, map, c0, c1, c2, bar);
  }
}

template <int P, bool BF16, int L>
__global__ void __launch_bounds__(128) k_adjoint(const __grid_constant__ AdjMaps m,
                                                 const StepArgs a, const int batched,
                                                 const int cq_arr) {
  constexpr int NQ = 2 * P;
  constexpr int NS = L + 1;
  (void)sizeof(Stages<L>);
  extern __shared__ float smem_raw[];
  float *smem = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem) + warp * NS;
  float *wb = smem + 32 + warp * a.warp_floats;
  float *prow = wb + NS * a.stage_floats;  // px row: 32 float4
  float *hs = prow + kAPx;                 // qx ring: NQ rows of 30 float4
  const int band_slot = a.band_floats, band_box = a.band_box_floats * 4;
  const Geom &g = a.g;
  const int nx = g.nx, ny = g.ny;
  const int n_items = g.S * g.n_strips * g.n_chunks;
  if (__any_sync(kFull, *reinterpret_cast<volatile int *>(a.flags + kFlagTimeout) != 0)) return;
  if (lane == 0) {
    for (int k = 0; k < NS; ++k) mbar_init(&bars[k], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const float cqs = cq_arr ? 0.f : __ldg(a.cq);
  const bool own_lane = lane >= 2 && lane <= 29;   // owned float4 o = lane - 2
  const bool q_lane = lane <= 29;                  // qx float4 at column x0 - 4 + 4 lane
  const int wq = q_lane ? lane : 0;                // px window base (lanes 30, 31 idle)
  const int wo = own_lane ? lane - 2 : 0;          // qx window base of the E update
  const BandTab T{g.Wx, g.Wz};
  Ring ring{0, 0u};
  int *ctr = a.flags + kCtrBase + a.ctr_slot;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.flags[kCtrBase + (a.ctr_slot ^ 1)] = 0;

  for (;;) {
    int item = 0;
    if (lane == 0) item = atomicAdd(ctr, 1);
    item = __shfl_sync(kFull, item, 0);
    if (item >= n_items) break;
    Item it;
    if (!make_item<P>(g, item, batched != 0, it)) continue;
    const int pc = it.x0 - 8 + 4 * lane;  // px / own float4 column
    const int qc = it.x0 - 4 + 4 * lane;  // qx float4 column
    const bool pc_ok = pc >= 0 && pc < nx;
    const bool qc_ok = q_lane && qc >= 0 && qc < nx;
    const bool own = own_lane && pc_ok;
    const bool q_own = lane >= 1 && lane <= 28 && qc_ok;  // qx float4 inside the strip
    const int pb = xband_col(pc, nx, g.Wx);
    const int qb = q_lane ? xband_col(qc, nx, g.Wx) : -1;
    const int64_t sbp = (int64_t)it.s * g.numel + pc;
    const int64_t sbq = (int64_t)it.s * g.numel + qc;
    const int64_t mbp = (int64_t)it.sm * g.numel + pc;
    const int64_t mbq = (int64_t)it.sm * g.numel + qc;
    const int64_t xw = (int64_t)it.s * ny * 2 * g.Wx;
    const int64_t zbw = (int64_t)it.s * 2 * g.Wz * nx + pc;
    bool colmask[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      colmask[q] = !g.grad_mask || (pc + q >= g.n_pml && pc + q < nx - g.n_pml);
    {
      Ring pr = ring;
      for (int j = 0; j < L && j < it.n_it; ++j) {
        adj_issue<P, BF16>(m, a, g, it, j, wb + pr.slot * a.stage_floats, &bars[pr.slot],
                           band_slot, band_box, lane);
        pr.next(NS);
      }
    }
    F4 pq[NQ], qq[NQ];
#pragma unroll
    for (int k = 0; k < NQ; ++k) pq[k] = qq[k] = zero4();

    for (int i0 = 0; i0 < it.n_it; i0 += NQ) {
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        const int i = i0 + u;
        if (i < it.n_it) {
          if (i + L < it.n_it) {
            const int ps = ring.slot == 0 ? NS - 1 : ring.slot - 1;
            adj_issue<P, BF16>(m, a, g, it, i + L, wb + ps * a.stage_floats, &bars[ps],
                               band_slot, band_box, lane);
          }
          const float *st = wb + ring.slot * a.stage_floats;
          if (!mbar_wait(&bars[ring.slot], ring.phase)) {
            if (lane == 0) atomicOr(a.flags + kFlagTimeout, 1);
            Ring dr = ring;
            for (int j = i; j < it.n_it && j <= i + L; ++j) {
              mbar_wait(&bars[dr.slot], dr.phase);
              dr.next(NS);
            }
            return;
          }
          const Rows<P> R(it.r0, i, it.ya, it.yb, ny);
          const F4 lam = lds4(st + kA_LAM + 4 * lane);
          const F4 cbv = lds4(st + kA_CB + 4 * lane);
          F4 gv;
#pragma unroll
          for (int q = 0; q < 4; ++q) gv.v[q] = cbv.v[q] * lam.v[q];

          // ---- gradients (lam = lambda_E^{t+1}) and px: own rows
          if (R.own_r) {
            const int64_t roff = (int64_t)R.r * nx;
            if (own) {
              const F4 se = snap_lds<BF16>(st + kA_SE, wo);
              const F4 sc = snap_lds<BF16>(st + kA_SC, wo);
              F4 gca = lds4(st + kA_GCA + 4 * wo), gcb = lds4(st + kA_GCB + 4 * wo);
              const bool rowmask = !g.grad_mask || (R.r >= g.n_pml && R.r < ny - g.n_pml);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                if (rowmask && colmask[q]) {
                  gca.v[q] = fmaf(se.v[q], lam.v[q], gca.v[q]);
                  gcb.v[q] = fmaf(sc.v[q], lam.v[q], gcb.v[q]);
                }
              }
              st4(a.gca + sbp + roff, gca);
              st4(a.gcb + sbp + roff, gcb);
            }
            F4 px = gv;
            if (pb >= 0) {
              F4 M = lds4(st + kA_BAND + pb);
              const F4 ax = ld4(a.bt + T.x(0) + pb), bx = ld4(a.bt + T.x(1) + pb);
              const F4 rk = ld4(a.bt + T.x(2) + pb);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                M.v[q] += gv.v[q];
                px.v[q] = fmaf(ax.v[q], M.v[q], gv.v[q] * rk.v[q]);
                M.v[q] *= bx.v[q];
              }
              if (own) st4(a.out.mxe_node + xw + (int64_t)R.r * 2 * g.Wx + pb, M);
            }
            st4(prow + 4 * lane, pc_ok ? px : zero4());
          }
          // ---- pz (queue) at E nodes, every row of the walk (owned lanes)
          {
            F4 pz;
#pragma unroll
            for (int q = 0; q < 4; ++q) pz.v[q] = -gv.v[q];
            const int zr = zband_row(R.r, ny, g.Wz);
            if (zr >= 0) {
              F4 M = lds4(st + kA_MZE + 4 * wo);
              const float ay = __ldg(a.bt + T.z(0) + zr), by = __ldg(a.bt + T.z(1) + zr);
              const float rky = __ldg(a.bt + T.z(2) + zr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                M.v[q] -= gv.v[q];
                pz.v[q] = fmaf(ay, M.v[q], -gv.v[q] * rky);
                M.v[q] *= by;
              }
              if (own && R.own_r) st4(a.out.mze_node + zbw + (int64_t)zr * nx, M);
            }
            pq[u] = pz;
          }
          __syncwarp();

          // ---- lamHz, qx at row r (lanes 0..29)
          if (R.own_r) {
            const int64_t roff = (int64_t)R.r * nx;
            float w[12];
            win12(prow + 4 * wq, w);
            const F4 lhz_old = lds4(st + kA_LHZ + 4 * wq);
            const F4 cq = cq_arr ? (qc_ok ? ld4(a.cq + mbq + roff) : zero4()) : splat4(cqs);
            F4 lhz, v;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              lhz.v[q] = lhz_old.v[q] - d_half<P>(w, q, a.c.cx);
              v.v[q] = cq.v[q] * lhz.v[q];
            }
            if (q_own) st4(a.out.hz + sbq + roff, lhz);
            if (qb >= 0) {
              F4 M = lds4(st + kA_BAND + band_slot + qb);
              const F4 ah = ld4(a.bt + T.x(3) + qb), bh = ld4(a.bt + T.x(4) + qb);
              const F4 rk = ld4(a.bt + T.x(5) + qb);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                M.v[q] += v.v[q];
                const float vq = v.v[q];
                v.v[q] = fmaf(ah.v[q], M.v[q], vq * rk.v[q]);
                M.v[q] *= bh.v[q];
              }
              if (q_own) st4(a.out.mxh_node + xw + (int64_t)R.r * 2 * g.Wx + qb, M);
            }
            if (q_lane) st4(hs + u * kARing + 4 * lane, qc_ok ? v : zero4());
          }

          // ---- lamHx, qz at row rh (owned lanes)
          if (R.hx_need) {
            F4 qz = zero4();
            if (R.hx_in) {
              const bool own_h = own && R.rh >= it.ya && R.rh < it.yb;
              const F4 lhx = lds4(st + kA_LHX + 4 * wo);
              const F4 cq = cq_arr ? (own ? ld4(a.cq + mbp + (int64_t)R.rh * nx) : zero4()) : splat4(cqs);
              F4 lh;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float d = 0.f;
#pragma unroll
                for (int k = 1; k <= P; ++k)
                  d = fmaf(a.c.cy[k - 1],
                           pq[(u - P + k + NQ) % NQ].v[q] - pq[(u - P - k + 1 + 2 * NQ) % NQ].v[q],
                           d);
                lh.v[q] = lhx.v[q] - d;
                qz.v[q] = -cq.v[q] * lh.v[q];
              }
              if (own_h) st4(a.out.hx + sbp + (int64_t)R.rh * nx, lh);
              const int zr = zband_row(R.rh, ny, g.Wz);
              if (zr >= 0) {
                F4 M = lds4(st + kA_MZH + 4 * wo);
                const float ayh = __ldg(a.bt + T.z(3) + zr), byh = __ldg(a.bt + T.z(4) + zr);
                const float rkyh = __ldg(a.bt + T.z(5) + zr);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float v = qz.v[q];
                  M.v[q] += v;
                  qz.v[q] = fmaf(ayh, M.v[q], v * rkyh);
                  M.v[q] *= byh;
                }
                if (own_h) st4(a.out.mzh_node + zbw + (int64_t)zr * nx, M);
              }
            }
            qq[u] = qz;
          }

          // ---- lamE at row y (owned lanes)
          if (R.e_row && own) {
            float w[12];
            win12(hs + ((u + 1) % NQ) * kARing + 4 * wo, w);
            const F4 ca4 = lds4(st + kA_CA + 4 * wo);
            const F4 lam_y = lds4(st + kA_LAMY + 4 * wo);
            F4 en;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float dz = 0.f;
#pragma unroll
              for (int k = 1; k <= P; ++k)
                dz = fmaf(a.c.cy[k - 1], qq[(u + P + k) % NQ].v[q] - qq[(u + 1 + P - k) % NQ].v[q],
                          dz);
              en.v[q] = ca4.v[q] * lam_y.v[q] - d_int<P>(w, q, a.c.cx) - dz;
            }
            st4(a.out.ey + sbp + (int64_t)R.y * nx, en);
          }
          __syncwarp();
          ring.next(NS);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------

constexpr int kFwdL = 1;  // forward lookahead (rows in flight)
constexpr int kAdjL = 1;  // adjoint lookahead

template <int P>
void layout_t(bool adjoint, int Wx, int *stage_floats, int *band_floats, int *warp_floats,
              size_t *smem) {
  const int bw = Wx > 0 ? ((2 * Wx + 31) / 32) * 32 : 0;
  const int sf = (adjoint ? kA_BAND : kF_BAND) + 2 * bw;
  int wf = adjoint ? (kAdjL + 1) * sf + kAPx + 2 * P * kARing : (kFwdL + 1) * sf + 2 * P * kFRing;
  wf = ((wf + 31) / 32) * 32;
  *stage_floats = sf;
  *band_floats = bw;
  *warp_floats = wf;
  *smem = (size_t)(32 + kWarpsPerCta * wf) * sizeof(float) + 128;
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
template <int P, int STORE>
std::atomic<uint64_t> &fwd_smem_flag() {
  static std::atomic<uint64_t> f{0};
  return f;
}
template <int P, bool BF16>
std::atomic<uint64_t> &adj_smem_flag() {
  static std::atomic<uint64_t> f{0};
  return f;
}

template <int P, int STORE>
cudaError_t fwd_t(const FwdMaps &m, const StepArgs &a, bool batched, bool cq_arr, int grid,
                  cudaStream_t st) {
  int sf, bw, wf;
  size_t smem;
  layout_t<P>(false, a.g.Wx, &sf, &bw, &wf, &smem);
  allow_big_smem(k_forward<P, STORE, kFwdL>, fwd_smem_flag<P, STORE>());
  k_forward<P, STORE, kFwdL><<<grid, 128, smem, st>>>(m, a, batched ? 1 : 0, cq_arr ? 1 : 0);
  count_launches(1);
  return cudaGetLastError();
}
template <int P, bool BF16>
cudaError_t adj_t(const AdjMaps &m, const StepArgs &a, bool batched, bool cq_arr, int grid,
                  cudaStream_t st) {
  int sf, bw, wf;
  size_t smem;
  layout_t<P>(true, a.g.Wx, &sf, &bw, &wf, &smem);
  allow_big_smem(k_adjoint<P, BF16, kAdjL>, adj_smem_flag<P, BF16>());
  k_adjoint<P, BF16, kAdjL><<<grid, 128, smem, st>>>(m, a, batched ? 1 : 0, cq_arr ? 1 : 0);
  count_launches(1);
  return cudaGetLastError();
}

template <int P>
cudaError_t fwd_store(const FwdMaps &m, const StepArgs &a, int store, bool batched, bool cq_arr,
                      int grid, cudaStream_t st) {
  switch (store) {
    case kStoreNone: return fwd_t<P, kStoreNone>(m, a, batched, cq_arr, grid, st);
    case kStoreF32: return fwd_t<P, kStoreF32>(m, a, batched, cq_arr, grid, st);
    case kStoreBF16: return fwd_t<P, kStoreBF16>(m, a, batched, cq_arr, grid, st);
  }
  return cudaErrorInvalidValue;
}

template <typename K>
int occupancy(K kern, size_t smem, std::atomic<uint64_t> &flag) {
  allow_big_smem(kern, flag);
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 128, smem) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

template <int P>
int slots_t(bool adjoint, int Wx) {
  int sf, bw, wf;
  size_t smem;
  layout_t<P>(adjoint, Wx, &sf, &bw, &wf, &smem);
  return (adjoint ? occupancy(k_adjoint<P, false, kAdjL>, smem, adj_smem_flag<P, false>())
                  : occupancy(k_forward<P, kStoreF32, kFwdL>, smem,
                              fwd_smem_flag<P, kStoreF32>())) *
         kWarpsPerCta;
}

}  // namespace

cudaError_t launch_forward(const FwdMaps &m, const StepArgs &a, int order, int store, bool batched,
                           bool cq_array, int grid, cudaStream_t st) {
  switch (order) {
    case 2: return fwd_store<1>(m, a, store, batched, cq_array, grid, st);
    case 4: return fwd_store<2>(m, a, store, batched, cq_array, grid, st);
    case 6: return fwd_store<3>(m, a, store, batched, cq_array, grid, st);
    case 8: return fwd_store<4>(m, a, store, batched, cq_array, grid, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_adjoint(const AdjMaps &m, const StepArgs &a, int order, int snap_bf16,
                           bool batched, bool cq_array, int grid, cudaStream_t st) {
  const bool b = snap_bf16 != 0;
  switch (order) {
    case 2: return b ? adj_t<1, true>(m, a, batched, cq_array, grid, st)
                     : adj_t<1, false>(m, a, batched, cq_array, grid, st);
    case 4: return b ? adj_t<2, true>(m, a, batched, cq_array, grid, st)
                     : adj_t<2, false>(m, a, batched, cq_array, grid, st);
    case 6: return b ? adj_t<3, true>(m, a, batched, cq_array, grid, st)
                     : adj_t<3, false>(m, a, batched, cq_array, grid, st);
    case 8: return b ? adj_t<4, true>(m, a, batched, cq_array, grid, st)
                     : adj_t<4, false>(m, a, batched, cq_array, grid, st);
  }
  return cudaErrorInvalidValue;
}

void stencil_layout(int order, bool adjoint, int Wx, int *sf, int *bw, int *wf, size_t *smem) {
  switch (order) {
    case 2: layout_t<1>(adjoint, Wx, sf, bw, wf, smem); return;
    case 4: layout_t<2>(adjoint, Wx, sf, bw, wf, smem); return;
    case 6: layout_t<3>(adjoint, Wx, sf, bw, wf, smem); return;
    default: layout_t<4>(adjoint, Wx, sf, bw, wf, smem); return;
  }
}

int stencil_slots_per_sm(int order, bool adjoint, int Wx) {
  switch (order) {
    case 2: return slots_t<1>(adjoint, Wx);
    case 4: return slots_t<2>(adjoint, Wx);
    case 6: return slots_t<3>(adjoint, Wx);
    default: return slots_t<4>(adjoint, Wx);
  }
}

}  // namespace mw
