// C ABI of the mw_tm library (declared in include/mw_tm.h): argument checks,
// workspace layout, the forward / adjoint time loops, checkpoint replay and
// per-kernel event timing.  The time loops follow the page "tide-GPR 0.0.9 ...
// tide/csrc/maxwell.cu" host drivers (forward: H, E, sources, receivers per
// step; backward: adjoint sources, source gradient, adjoint H, adjoint E with
// gradient, reversed in time) with the H and E kernels fused into one launch.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "mw_internal.cuh"

namespace mw {

static std::atomic<int64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define MW_CUDA(call)                                                                    \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(MW_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                  __FILE__, __LINE__);                                                   \
  } while (0)

// Staggered first-derivative weights (Taylor conditions on a half-integer grid).
int stencil_weights(int order, double *c) {
  c[0] = c[1] = c[2] = c[3] = 0.0;
  switch (order) {
    case 2: c[0] = 1.0; return 1;
    case 4: c[0] = 9.0 / 8.0; c[1] = -1.0 / 24.0; return 2;
    case 6: c[0] = 75.0 / 64.0; c[1] = -25.0 / 384.0; c[2] = 3.0 / 640.0; return 3;
    case 8:
      c[0] = 1225.0 / 1024.0; c[1] = -245.0 / 3072.0; c[2] = 49.0 / 5120.0;
      c[3] = -5.0 / 7168.0;
      return 4;
  }
  return 0;
}

#define MW_TRY(x)                 \
  do {                            \
    int rc_ = (x);                \
    if (rc_ != MW_OK) return rc_; \
  } while (0)

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Bands {
  int Wx, Wz;
};
Bands bands(const mw_params *p) {
  Bands b;
  b.Wx = p->n_pml > 0 ? ((p->n_pml + 1 + 3) / 4) * 4 : 0;
  b.Wz = p->n_pml > 0 ? p->n_pml + 1 : 0;
  return b;
}

size_t state_floats(const mw_params *p) {
  const Bands b = bands(p);
  const size_t S = p->n_shots, ny = p->ny, nx = p->nx;
  return S * ny * nx * 3 + S * ny * 2 * b.Wx * 2 + S * 2 * b.Wz * nx * 2;
}

// checkpoint modes: segment replay (pair store), or the E snapshot alone with
// the summation-by-parts Cb gradient
bool is_ckpt(const mw_params *p) {
  return p->snap_mode == MW_SNAP_CKPT || p->snap_mode == MW_SNAP_CKPT_EY;
}

int check_params(const mw_params *p, bool cfl) {
  if (!p) return fail(MW_ERR_ARG, "params is NULL");
  double c[4];
  if (!stencil_weights(p->order, c)) return fail(MW_ERR_ARG, "order %d not in {2,4,6,8}", p->order);
  if (p->ny < 1 || p->nx < 4) return fail(MW_ERR_ARG, "grid %d x %d too small", p->ny, p->nx);
  if (p->nx % 4 != 0) return fail(MW_ERR_ARG, "nx = %d must be a multiple of 4", p->nx);
  if (p->n_shots < 1) return fail(MW_ERR_ARG, "n_shots = %d", p->n_shots);
  if (p->n_src < 0 || p->n_rec < 0 || p->nt < 0) return fail(MW_ERR_ARG, "negative count");
  if (!(p->dt > 0) || !(p->dy > 0) || !(p->dx > 0) || !isfinite(p->dt) || !isfinite(p->dy) ||
      !isfinite(p->dx))
    return fail(MW_ERR_ARG, "dt, dy, dx must be positive and finite");
  if (p->n_pml < 0) return fail(MW_ERR_ARG, "n_pml = %d", p->n_pml);
  const Bands b = bands(p);
  if (2 * b.Wx > p->nx || 2 * b.Wz > p->ny)
    return fail(MW_ERR_ARG, "CPML band %d does not fit a %d x %d grid", p->n_pml, p->ny, p->nx);
  if (p->snap_mode < MW_SNAP_NONE || p->snap_mode > MW_SNAP_CKPT_EY)
    return fail(MW_ERR_ARG, "snap_mode = %d", p->snap_mode);
  if (p->snap_host && p->snap_mode != MW_SNAP_FP32 && p->snap_mode != MW_SNAP_BF16 &&
      p->snap_mode != MW_SNAP_FP8)
    return fail(MW_ERR_ARG, "snap_host needs snap_mode FP32, BF16 or FP8 (got %d)", p->snap_mode);
  if (is_ckpt(p) && p->ckpt_every < 1)
    return fail(MW_ERR_ARG, "ckpt_every = %d", p->ckpt_every);
  if (p->ckpt_tail < 0 || (p->ckpt_tail > 0 && !is_ckpt(p)))
    return fail(MW_ERR_ARG, "ckpt_tail = %d needs a checkpoint snap_mode", p->ckpt_tail);
  if (2 * b.Wx > 256)
    return fail(MW_ERR_UNSUPPORTED, "n_pml = %d: a band row exceeds one TMA box (n_pml <= 123)",
                p->n_pml);
  if ((int64_t)p->ny * p->nx > ((int64_t)1 << 40)) return fail(MW_ERR_ARG, "grid too large");
  if (cfl && !p->allow_unstable) {
    if (!(p->vmax > 0) || !isfinite(p->vmax))
      return fail(MW_ERR_CFL, "vmax must be positive (or set allow_unstable)");
    const double dtmax = mw_cfl_dt(p->order, p->dy, p->dx, p->vmax);
    if (p->dt > dtmax * (1.0 + 1e-12))
      return fail(MW_ERR_CFL, "dt = %.6g s exceeds the stability bound %.6g s", p->dt, dtmax);
  }
  return MW_OK;
}

// device ring slots of the pinned-host snapshot store
constexpr int kHostRing = 3;

// bytes per stored snapshot value of a full-storage mode
size_t snap_elem_bytes(int snap_mode) {
  return snap_mode == MW_SNAP_BF16 ? 2 : snap_mode == MW_SNAP_FP8 ? 1 : 4;
}
// store kind of the forward (full-storage modes) / load kind of the adjoint
int snap_store_kind(int snap_mode) {
  return snap_mode == MW_SNAP_FP32 ? kStoreF32
         : snap_mode == MW_SNAP_BF16 ? kStoreBF16
         : snap_mode == MW_SNAP_FP8 ? kStoreFP8 : kStoreNone;
}

Layout layout(const mw_params *p) {
  Layout L{};
  const size_t SN = (size_t)p->n_shots * p->ny * p->nx;
  L.state_bytes = state_floats(p) * sizeof(float);
  const size_t sb = align256(L.state_bytes);
  size_t off = 0;
  L.flags = off; off += 256;
  L.tab_src = off; off += entry_table_bytes(p->n_shots, p->n_src, p->ny);
  L.tab_rec = off; off += entry_table_bytes(p->n_shots, p->n_rec, p->ny);
  L.bandtab = off;
  {
    const Bands b = bands(p);
    off += align256(sizeof(float) * (size_t)BandTab{b.Wx, b.Wz}.floats() + 16);
  }
  L.stA = off; off += sb;
  L.stB = off; off += sb;
  L.adA = L.adB = L.rpA = L.rpB = L.snap = L.seg = 0;
  L.n_seg = 0;
  L.snap_step_bytes = 0;
  L.snap_pitch = p->nx;
  if (p->snap_mode != MW_SNAP_NONE) {
    L.adA = off; off += sb;
    L.adB = off; off += sb;
  }
  if (p->snap_mode == MW_SNAP_FP32 || p->snap_mode == MW_SNAP_BF16 ||
      p->snap_mode == MW_SNAP_FP8) {
    const size_t es = snap_elem_bytes(p->snap_mode);
    const size_t per_row = 16 / es;  // elements per 16 bytes
    L.snap_pitch = (int)(((size_t)p->nx + per_row - 1) / per_row * per_row);
    L.snap_step_bytes = (size_t)p->n_shots * p->ny * L.snap_pitch * es;
    L.snap = off;
    // device copy of every step, or with snap_host a ring of kHostRing steps
    // ([2][kHostRing] step slots) that the host copies pass through
    const size_t steps = p->snap_host ? (size_t)kHostRing : (size_t)p->nt;
    off += align256(2 * steps * L.snap_step_bytes);
  } else if (is_ckpt(p)) {
    L.n_seg = p->nt > 0 ? (p->nt + p->ckpt_every - 1) / p->ckpt_every : 0;
    L.rpA = off; off += sb;
    L.rpB = off; off += sb;
    L.snap = off; off += (size_t)L.n_seg * sb;
    L.snap_pitch = p->nx;
    L.snap_step_bytes = SN * 4;
    L.seg = off;
    off += align256(2 * (size_t)p->ckpt_every * L.snap_step_bytes);
    // the tail the forward stores itself: [E slots][curl slots], or with E
    // alone the E slots and one more for the final E (the adjoint's end term)
    L.n_tail = p->ckpt_tail < p->nt ? p->ckpt_tail : p->nt;
    L.tail = off;
    if (L.n_tail > 0) {
      const size_t slots = p->snap_mode == MW_SNAP_CKPT_EY ? (size_t)L.n_tail + 1
                                                            : 2 * (size_t)L.n_tail;
      off += align256(slots * L.snap_step_bytes);
    }
  }
  L.sbp = L.rcopy = L.acc = L.gfbuf = 0;
  if (p->snap_mode == MW_SNAP_CKPT_EY) {
    L.sbp = off; off += align256(SN * sizeof(float));
    L.rcopy = off; off += align256((size_t)p->nt * p->n_shots * p->n_rec * sizeof(float));
    // the receiver and source sums
    L.acc = off;
    off += align256((size_t)p->n_shots * (p->n_rec + (size_t)p->n_src) * sizeof(float));
    // lambda_E sampled at the sources every step, when the caller asks for
    // no grad_f (the source end term needs it)
    L.gfbuf = off;
    off += align256((size_t)p->nt * p->n_shots * p->n_src * sizeof(float));
  }
  L.total = off;
  return L;
}

Fields fields_at(const mw_params *p, float *base) {
  const Bands b = bands(p);
  const size_t SN = (size_t)p->n_shots * p->ny * p->nx;
  const size_t xb = (size_t)p->n_shots * p->ny * 2 * b.Wx;
  const size_t zb = (size_t)p->n_shots * 2 * b.Wz * p->nx;
  Fields f;
  f.ey = base;
  f.hx = base + SN;
  f.hz = base + 2 * SN;
  f.mxh_node = base + 3 * SN;
  f.mxe_node = f.mxh_node + xb;
  f.mzh_node = f.mxe_node + xb;
  f.mze_node = f.mzh_node + zb;
  return f;
}

// checkpoint k of the checkpoint modes (a full state, 256-aligned)
float *ckpt_slot(char *ws, const Layout &L, int k) {
  return (float *)(ws + L.snap + (size_t)k * align256(L.state_bytes));
}

// Pinned-host snapshot store: the caller's page-locked buffer holds step t
// as [E block][curl block] at 2 t step_bytes; a ring of kHostRing device
// slots per field stages the copies, which run on a stream of their own and
// are ordered with the compute stream by events.
int check_host_snap(const mw_params *p) {
  if (!p->snap_host) return MW_OK;
  if (!p->snap_host_ptr) return fail(MW_ERR_ARG, "snap_host_ptr is NULL");
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p->snap_host_ptr) != cudaSuccess ||
      at.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return fail(MW_ERR_ARG, "snap_host_ptr is not page-locked host memory");
  }
  return MW_OK;
}
struct HostCopies {
  cudaStream_t cs = nullptr;
  cudaEvent_t filled[kHostRing] = {}, freed[kHostRing] = {}, start = nullptr;
  int init() {
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess)
      return fail(MW_ERR_CUDA, "cannot create the snapshot copy stream");
    for (int k = 0; k < kHostRing; ++k)
      if (cudaEventCreateWithFlags(&filled[k], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&freed[k], cudaEventDisableTiming) != cudaSuccess)
        return fail(MW_ERR_CUDA, "cannot create snapshot copy events");
    if (cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess)
      return fail(MW_ERR_CUDA, "cannot create snapshot copy events");
    return MW_OK;
  }
  ~HostCopies() {  // resources are released once the queued work completes
    for (int k = 0; k < kHostRing; ++k) {
      if (filled[k]) cudaEventDestroy(filled[k]);
      if (freed[k]) cudaEventDestroy(freed[k]);
    }
    if (start) cudaEventDestroy(start);
    if (cs) cudaStreamDestroy(cs);
  }
};

// Entry tables of the sources and the receivers (built per call).
struct Tables {
  EntrySet src, rec;
};
Tables tables_at(const mw_params *p, char *ws, const Layout &L) {
  return Tables{entry_set_at(ws + L.tab_src, p->n_shots, p->n_src, p->ny),
                entry_set_at(ws + L.tab_rec, p->n_shots, p->n_rec, p->ny)};
}
// Build the table of one index set (n > 0); `out` [nt][S][n] gets zeros at
// the invalid entries.
int build_table(const mw_params *p, const int64_t *idx, int n, char *ws, size_t off, int *flags,
                float *out, cudaStream_t st) {
  if (n <= 0) return MW_OK;
  MW_CUDA(launch_entry_table(idx, p->n_shots, n, p->ny, p->nx, ws + off, flags, out, p->nt, st));
  return MW_OK;
}

// ---- launch geometry ------------------------------------------------------
int sm_count() {
  static int cached = -1;
  static int cached_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (cached < 0 || dev != cached_dev) {
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    cached = n;
    cached_dev = dev;
  }
  return cached;
}

struct Launch {
  Geom g;
  int grid;
};

// Interior rectangle of the item grid (the same edge rule as the kernels'
// make_item / make_item2): strip x0 with an xh-column margin clear of the x
// bands and the array's sides; chunk [ya, yb) whose walk rows ya - zw ..
// yb + zw - 1 stay clear of the z bands (one-step kernels: xh = 8, zw =
// 2P - 1; two-step forward: xh = halo + 4, zw = 4P - 2).  Checked to give a
// bijection of the items.
void interior_rect(Geom &g, int xh, int zw) {
  auto strip_edge = [&](int k) {
    const int x0 = k * g.strip_cols;
    return x0 - xh < g.Wx || x0 + g.strip_cols + xh > g.nx - g.Wx;
  };
  auto chunk_edge = [&](int k) {
    int ya, yb;
    chunk_rows(g, k, &ya, &yb);
    return g.Wz > 0 && (ya - zw < g.Wz || yb + zw > g.ny - g.Wz);
  };
  int a = 0, b = g.n_strips;
  while (a < b && strip_edge(a)) ++a;
  while (b > a && strip_edge(b - 1)) --b;
  int c = 0, d = g.n_chunks;
  while (c < d && chunk_edge(c)) ++c;
  while (d > c && chunk_edge(d - 1)) --d;
  for (int k = a; k < b; ++k)
    if (strip_edge(k)) a = b;  // not a single run: no interior rectangle
  for (int k = c; k < d; ++k)
    if (chunk_edge(k)) c = d;
  g.is_lo = a;
  g.is_hi = b;
  g.ic_lo = c;
  g.ic_hi = d;
  // the claim order must visit every (shot, strip, chunk) once
  const int64_t n = (int64_t)g.S * g.n_strips * g.n_chunks;
  std::vector<unsigned char> seen((size_t)n, 0);
  bool ok = true;
  for (int64_t i = 0; i < n && ok; ++i) {
    int s, st, ch;
    item_coords(g, (int)i, &s, &st, &ch);
    if (s < 0 || s >= g.S || st < 0 || st >= g.n_strips || ch < 0 || ch >= g.n_chunks) {
      ok = false;
      break;
    }
    unsigned char &f = seen[((size_t)ch * g.n_strips + st) * g.S + s];
    if (f) ok = false;
    f = 1;
  }
  if (!ok) g.is_lo = g.is_hi = g.ic_lo = g.ic_hi = 0;
}

// Choose the row-chunk height so that the warps' work items fill whole waves
// of resident warps: cost ~ waves x (rows per item + warm-up rows).
enum PlanKind { kPlanFwd = 0, kPlanAdj = 1, kPlanFwd2 = 2 };
Launch plan(const mw_params *p, int kind) {
  const bool adjoint = kind == kPlanAdj, two = kind == kPlanFwd2;
  Launch Lc{};
  Geom &g = Lc.g;
  const Bands b = bands(p);
  g.ny = p->ny;
  g.nx = p->nx;
  g.S = p->n_shots;
  g.Wx = b.Wx;
  g.Wz = b.Wz;
  g.n_pml = p->n_pml;
  g.grad_mask = p->grad_mask_pml ? 1 : 0;
  g.numel = (int64_t)p->ny * p->nx;
  const int P = p->order / 2;
  g.strip_cols = adjoint ? kAdjStripCols : two ? fwd2_width(P) : kFwdStripCols;
  g.n_strips = (p->nx + g.strip_cols - 1) / g.strip_cols;
  const int warps_sm = two ? forward2_slots_per_sm(p->order, b.Wx)
                           : stencil_slots_per_sm(p->order, adjoint, b.Wx, !p->cq_is_scalar);
  const int64_t slots = (int64_t)sm_count() * warps_sm;
  const int64_t cols_items = (int64_t)g.S * g.n_strips;
  // Items are claimed dynamically by resident warps.  Each item walks its
  // rows plus 4P - 2 warm-up rows.  Model: the claimed work spread over the
  // slots, plus the duration of the items claimed last (the tail); with n1
  // long chunks of H1 rows first and short chunks of H2 rows after them, the
  // last long items must also end in time:
  //   cost = max(W / slots + (H2 + w), W_long / slots + (H1 + w)).
  const int w = two ? 8 * P - 4 : 4 * P - 2;
  const double cols = (double)cols_items, sl = (double)slots;
  int best_h1 = p->ny, best_h2 = p->ny, best_n1 = 1;
  double best_cost = 1e300;
  for (int h1 = 8; h1 <= p->ny + 7; h1 += (h1 < 64 ? 1 : 4)) {
    const int n1_max = (p->ny + h1 - 1) / h1;
    for (int n1 = 1; n1 <= n1_max; ++n1) {
      const int rest = p->ny - n1 * h1;
      const double wl = cols * n1 * (h1 + w);
      if (rest <= 0) {  // long chunks only (the last one ragged)
        const double cost = wl / sl + (h1 + w);
        if (cost < best_cost - 1e-9) {
          best_cost = cost;
          best_h1 = h1;
          best_h2 = h1;
          best_n1 = n1;
        }
        continue;
      }
      const int h2_max = h1 - 1 < 64 ? h1 - 1 : 64;
      for (int h2 = 4; h2 <= h2_max; ++h2) {
        const int n2 = (rest + h2 - 1) / h2;
        const double W = wl + cols * n2 * (h2 + w);
        const double a = W / sl + (h2 + w), b = wl / sl + (h1 + w);
        const double cost = a > b ? a : b;
        if (cost < best_cost - 1e-9) {
          best_cost = cost;
          best_h1 = h1;
          best_h2 = h2;
          best_n1 = n1;
        }
      }
    }
  }
  g.chunk_h = best_h1;
  g.chunk_h2 = best_h2;
  g.n_big = best_n1;
  {
    const int rest = p->ny - best_n1 * best_h1;
    g.n_chunks = rest > 0 ? best_n1 + (rest + best_h2 - 1) / best_h2 : (p->ny + best_h1 - 1) / best_h1;
    if (rest <= 0) g.n_big = g.n_chunks;
  }
  if (two) interior_rect(g, fwd2_halo(P) + 4, 4 * P - 2);
  else interior_rect(g, 8, 2 * P - 1);
  const int64_t items = cols_items * g.n_chunks;
  const int wpc = adjoint ? adj_warps_per_cta(P) : kWarpsPerCta;
  int64_t grid = (items + wpc - 1) / wpc;
  const int64_t cap = slots / wpc;
  if (grid > cap) grid = cap;
  Lc.grid = (int)(grid > 0 ? grid : 1);
  return Lc;
}

Coef coef_of(const mw_params *p) {
  double c[4];
  stencil_weights(p->order, c);
  Coef k;
  for (int i = 0; i < 4; ++i) {
    k.cx[i] = (float)(c[i] / p->dx);
    k.cy[i] = (float)(c[i] / p->dy);
  }
  return k;
}

// ---- TMA tensor maps ---------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// TMA element type of a 4-, 2- or 1-byte element (float32, bf16, E4M3 bytes)
CUtensorMapDataType elem_type(int elem) {
  return elem == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
         : elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
}

// Row-box map over an array [d3][d2][d1][d0] (rank 3 or 4) of float32 (elem
// 4) or bf16 (elem 2) with dense strides, or with the given outermost stride
// (bytes, rank 4 only; 0 = dense): box = (box0, 1, 1[, box3]), zero fill
// outside.
int encode_rows(CUtensorMap *map, const void *base, int elem, int rank, uint64_t d0, uint64_t d1,
                uint64_t d2, uint64_t d3, uint32_t box0, uint32_t box3 = 1,
                uint64_t stride3 = 0) {
  EncodeTiledFn fn = encoder();
  if (!fn) return fail(MW_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * elem, d0 * d1 * elem,
                           stride3 ? stride3 : d0 * d1 * d2 * elem};
  cuuint32_t box[4] = {box0, 1, 1, box3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, elem_type(elem), (cuuint32_t)rank, const_cast<void *>(base), dims, strides,
                  box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MW_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): rank %d dims %llu %llu %llu box %u",
                (int)r, rank, (unsigned long long)d0, (unsigned long long)d1,
                (unsigned long long)d2, box0);
  return MW_OK;
}

// Map of rank 2..5 with explicit strides (bytes, rank - 1 of them) and box;
// zero fill outside.
int encode_map(CUtensorMap *map, const void *base, int elem, int rank, const uint64_t *dims,
               const uint64_t *strides, const uint32_t *box) {
  EncodeTiledFn fn = encoder();
  if (!fn) return fail(MW_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int k = 0; k < rank; ++k) {
    d[k] = dims[k];
    b[k] = box[k];
    e[k] = 1;
    if (k + 1 < rank) st[k] = strides[k];
  }
  CUresult r = fn(map, elem_type(elem), (cuuint32_t)rank, const_cast<void *>(base), d, st, b, e,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MW_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): rank %d dims %llu %llu box %u",
                (int)r, rank, (unsigned long long)dims[0], (unsigned long long)dims[1], box[0]);
  return MW_OK;
}

// Two same-shaped arrays are fetched as one pair box when they are distinct,
// non-overlapping and their distance TMA can express as a stride.
struct Pairing {
  bool pair, swap;
  uint64_t stride;
};
Pairing pairing(const void *x, const void *y, uint64_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
  Pairing r{false, false, 0};
  const uint64_t d = a < b ? b - a : a - b;
  if (d >= bytes && d % 16 == 0 && d < ((uint64_t)1 << 40)) {
    r.pair = true;
    r.swap = b < a;
    r.stride = d;
  }
  return r;
}
typedef Pairing MdPair;
MdPair md_pairing(const mw_params *p, const float *ca, const float *cb) {
  const uint64_t Sm = p->model_batched ? p->n_shots : 1;
  return pairing(ca, cb, Sm * (uint64_t)p->ny * p->nx * sizeof(float));
}
Pairing gg_pairing(const mw_params *p, const float *gca, const float *gcb) {
  return pairing(gca, gcb, (uint64_t)p->n_shots * p->ny * p->nx * sizeof(float));
}

int fwd_maps(const mw_params *p, const Fields &in, const float *ca, const float *cb,
             const float *cq, FwdMaps *m) {
  memset(m, 0, sizeof *m);
  const Bands bd = bands(p);
  const uint64_t nx = p->nx, ny = p->ny, S = p->n_shots, Sm = p->model_batched ? p->n_shots : 1;
  const uint64_t field = (uint64_t)(in.hz - in.ey) * sizeof(float);
  MW_TRY(encode_rows(&m->map[kMapEH], in.ey, 4, 4, nx, ny, S, 2, 136, 2, field));
  MW_TRY(encode_rows(&m->map[kMapHX], in.hx, 4, 3, nx, ny, S, 1, 120));
  const MdPair md = md_pairing(p, ca, cb);
  if (md.pair) {
    MW_TRY(encode_rows(&m->map[kMapMD], md.swap ? cb : ca, 4, 4, nx, ny, Sm, 2, 120, 2,
                       md.stride));
  } else {
    MW_TRY(encode_rows(&m->map[kMapMD], ca, 4, 3, nx, ny, Sm, 1, 120));
    MW_TRY(encode_rows(&m->map[kMapCB], cb, 4, 3, nx, ny, Sm, 1, 120));
  }
  if (!p->cq_is_scalar) MW_TRY(encode_rows(&m->map[kMapCQ], cq, 4, 3, nx, ny, Sm, 1, 128));
  if (bd.Wx > 0) {
    MW_TRY(encode_rows(&m->map[kMapMXH], in.mxh_node, 4, 3, 2 * bd.Wx, ny, S, 1, 2 * bd.Wx));
    MW_TRY(encode_rows(&m->map[kMapMXE], in.mxe_node, 4, 3, 2 * bd.Wx, ny, S, 1, 2 * bd.Wx));
    MW_TRY(encode_rows(&m->map[kMapMZH], in.mzh_node, 4, 3, nx, 2 * bd.Wz, S, 1, 120));
    MW_TRY(encode_rows(&m->map[kMapMZE], in.mze_node, 4, 3, nx, 2 * bd.Wz, S, 1, 120));
  }
  return MW_OK;
}

// Two-step forward: every box 128 wide (the walk's columns), Ca / Cb a pair
// box when their distance allows.
int fwd2_maps(const mw_params *p, const Fields &in, const float *ca, const float *cb,
              Fwd2Maps *m) {
  memset(m, 0, sizeof *m);
  const Bands bd = bands(p);
  const uint64_t nx = p->nx, ny = p->ny, S = p->n_shots, Sm = p->model_batched ? p->n_shots : 1;
  MW_TRY(encode_rows(&m->map[kM2E], in.ey, 4, 3, nx, ny, S, 1, 128));
  MW_TRY(encode_rows(&m->map[kM2HZ], in.hz, 4, 3, nx, ny, S, 1, 128));
  MW_TRY(encode_rows(&m->map[kM2HX], in.hx, 4, 3, nx, ny, S, 1, 128));
  const MdPair md = md_pairing(p, ca, cb);
  if (md.pair) {
    MW_TRY(encode_rows(&m->map[kM2MD], md.swap ? cb : ca, 4, 4, nx, ny, Sm, 2, 128, 2, md.stride));
  } else {
    MW_TRY(encode_rows(&m->map[kM2MD], ca, 4, 3, nx, ny, Sm, 1, 128));
    MW_TRY(encode_rows(&m->map[kM2CB], cb, 4, 3, nx, ny, Sm, 1, 128));
  }
  if (bd.Wx > 0) {
    MW_TRY(encode_rows(&m->map[kM2MXH], in.mxh_node, 4, 3, 2 * bd.Wx, ny, S, 1, 2 * bd.Wx));
    MW_TRY(encode_rows(&m->map[kM2MXE], in.mxe_node, 4, 3, 2 * bd.Wx, ny, S, 1, 2 * bd.Wx));
    MW_TRY(encode_rows(&m->map[kM2MZH], in.mzh_node, 4, 3, nx, 2 * bd.Wz, S, 1, 128));
    MW_TRY(encode_rows(&m->map[kM2MZE], in.mze_node, 4, 3, nx, 2 * bd.Wz, S, 1, 128));
  }
  return MW_OK;
}

// Born forward: dCa / dCb (pair box when their distance allows) and the
// background's snapshots (x, y, shot, step, field) as one box 144 wide.
int born_maps(const mw_params *p, const float *dca, const float *dcb, const void *se,
              const void *sc, int snap_elem, int snap_steps, int snap_pitch, FwdMaps *m) {
  const uint64_t nx = p->nx, ny = p->ny, S = p->n_shots, Sm = p->model_batched ? p->n_shots : 1;
  const MdPair bd = md_pairing(p, dca, dcb);
  if (bd.pair) {
    MW_TRY(encode_rows(&m->map[kMapBD], bd.swap ? dcb : dca, 4, 4, nx, ny, Sm, 2, 120, 2,
                       bd.stride));
  } else {
    MW_TRY(encode_rows(&m->map[kMapBD], dca, 4, 3, nx, ny, Sm, 1, 120));
    MW_TRY(encode_rows(&m->map[kMapBDB], dcb, 4, 3, nx, ny, Sm, 1, 120));
  }
  if ((const char *)sc <= (const char *)se)
    return fail(MW_ERR_ARG, "internal: snapshot fields out of order");
  const uint64_t e = (uint64_t)snap_elem, pitch = (uint64_t)snap_pitch;
  const uint64_t dims[5] = {nx, ny, S, (uint64_t)snap_steps, 2};
  const uint64_t strides[4] = {pitch * e, pitch * ny * e, pitch * ny * S * e,
                               (uint64_t)((const char *)sc - (const char *)se)};
  const uint32_t box[5] = {144, 1, 1, 1, 2};
  MW_TRY(encode_map(&m->map[kMapBS], se, snap_elem, 5, dims, strides, box));
  return MW_OK;
}

int adj_maps(const mw_params *p, const Fields &in, const float *ca, const float *cb,
             const float *cq, const float *gca, const float *gcb, const void *se, const void *sc,
             int snap_elem, int snap_steps, int snap_pitch, bool ey_only, AdjMaps *m) {
  memset(m, 0, sizeof *m);
  const Bands bd = bands(p);
  const uint64_t nx = p->nx, ny = p->ny, S = p->n_shots, Sm = p->model_batched ? p->n_shots : 1;
  MW_TRY(encode_rows(&m->map[kAMapEH], in.ey, 4, 4, nx, ny, S, 2, 128, 2,
                     (uint64_t)(in.hz - in.ey) * sizeof(float)));
  const MdPair md = md_pairing(p, ca, cb);
  if (ey_only) {  // Cb of the row fetched, Ca of the row updated
    MW_TRY(encode_rows(&m->map[kAMapCB], cb, 4, 3, nx, ny, Sm, 1, 128));
    MW_TRY(encode_rows(&m->map[kAMapCA], ca, 4, 3, nx, ny, Sm, 1, 112));
  } else if (md.pair) {
    MW_TRY(encode_rows(&m->map[kAMapMD], md.swap ? cb : ca, 4, 4, nx, ny, Sm, 2, 128, 2,
                       md.stride));
  } else {
    MW_TRY(encode_rows(&m->map[kAMapMD], ca, 4, 3, nx, ny, Sm, 1, 128));
    MW_TRY(encode_rows(&m->map[kAMapCB], cb, 4, 3, nx, ny, Sm, 1, 128));
  }
  MW_TRY(encode_rows(&m->map[kAMapHX], in.hx, 4, 3, nx, ny, S, 1, 112));
  if (ey_only) {
    // (x, y, shot, step): the E snapshots
    const uint64_t e = (uint64_t)snap_elem, pitch = (uint64_t)snap_pitch;
    const uint64_t dims[4] = {nx, ny, S, (uint64_t)snap_steps};
    const uint64_t strides[3] = {pitch * e, pitch * ny * e, pitch * ny * S * e};
    const uint32_t box[4] = {112, 1, 1, 1};
    MW_TRY(encode_map(&m->map[kAMapSS], se, snap_elem, 4, dims, strides, box));
  } else {
    // (x, y, shot, step, field): the curl snapshots follow the E snapshots
    const uint64_t e = (uint64_t)snap_elem;
    const uint64_t dims[5] = {nx, ny, S, (uint64_t)snap_steps, 2};
    const uint64_t pitch = (uint64_t)snap_pitch;
    const uint64_t strides[4] = {pitch * e, pitch * ny * e, pitch * ny * S * e,
                                 (uint64_t)((const char *)sc - (const char *)se)};
    const uint32_t box[5] = {112, 1, 1, 1, 2};
    if ((const char *)sc <= (const char *)se)
      return fail(MW_ERR_ARG, "internal: snapshot fields out of order");
    MW_TRY(encode_map(&m->map[kAMapSS], se, snap_elem, 5, dims, strides, box));
  }
  const Pairing gg = gg_pairing(p, gca, gcb);
  if (gg.pair) {
    MW_TRY(encode_rows(&m->map[kAMapGG], gg.swap ? gcb : gca, 4, 4, nx, ny, S, 2, 112, 2,
                       gg.stride));
  } else {
    MW_TRY(encode_rows(&m->map[kAMapGG], gca, 4, 3, nx, ny, S, 1, 112));
    MW_TRY(encode_rows(&m->map[kAMapGB], gcb, 4, 3, nx, ny, S, 1, 112));
  }
  if (!p->cq_is_scalar) MW_TRY(encode_rows(&m->map[kAMapCQ], cq, 4, 3, nx, ny, Sm, 1, 128));
  if (bd.Wx > 0) {
    MW_TRY(encode_rows(&m->map[kAMapMX], in.mxh_node, 4, 4, 2 * bd.Wx, ny, S, 2, 2 * bd.Wx, 2,
                       (uint64_t)(in.mxe_node - in.mxh_node) * sizeof(float)));
    MW_TRY(encode_rows(&m->map[kAMapMZE], in.mze_node, 4, 3, nx, 2 * bd.Wz, S, 1, 112));
    MW_TRY(encode_rows(&m->map[kAMapMZH], in.mzh_node, 4, 3, nx, 2 * bd.Wz, S, 1, 112));
  }
  return MW_OK;
}

// Per-call set-up shared by the forward and adjoint sweeps: the CPML band
// coefficient table and the two work-item counters.
int stencil_prologue(const mw_params *p, const float *cpml, char *ws, const Layout &L,
                     cudaStream_t st) {
  const Bands b = bands(p);
  MW_CUDA(launch_band_table(cpml, p->ny, p->nx, b.Wx, b.Wz, (float *)(ws + L.bandtab), st));
  MW_CUDA(cudaMemsetAsync(ws + L.flags + kCtrBase * sizeof(int), 0, 2 * sizeof(int), st));
  return MW_OK;
}

void set_layout(StepArgs &a, const mw_params *p, bool adjoint) {
  size_t smem;
  if (adjoint) {
    // needs a.ca / a.cb and a.gca / a.gcb (pair fetches)
    adjoint_layout(p->order, bands(p).Wx, !p->cq_is_scalar, false, &a, &smem);
    const MdPair md = md_pairing(p, a.ca, a.cb);
    a.md_pair = md.pair ? 1 : 0;
    a.md_swap = md.swap ? 1 : 0;
    const Pairing gg = gg_pairing(p, a.gca, a.gcb);
    a.gg_pair = gg.pair ? 1 : 0;
    a.gg_swap = gg.swap ? 1 : 0;
  } else {
    // forward: needs a.ca / a.cb (the Ca / Cb pair fetch)
    forward_layout(p->order, bands(p).Wx, !p->cq_is_scalar, false, &a, &smem);
    const MdPair md = md_pairing(p, a.ca, a.cb);
    a.md_pair = md.pair ? 1 : 0;
    a.md_swap = md.swap ? 1 : 0;
  }
}

// Two-step forward launches of a call: their plan, arguments (the one-step
// forward's, re-laid-out) and the maps of each input buffer they read.  Used
// only where the two-step kernel applies (orders 2-6, scalar Cq); otherwise
// `on` is false and every step runs the one-step kernel.
struct Pairs {
  bool on = false;
  Launch lc{};
  StepArgs a{};
  int init(const mw_params *p, const StepArgs &one) {
    on = forward2_supported(p->order) && p->cq_is_scalar && !pairs_disabled();
    if (!on) return MW_OK;
    lc = plan(p, kPlanFwd2);
    a = one;
    a.g = lc.g;
    size_t smem;
    forward2_layout(p->order, bands(p).Wx, &a, &smem);
    return MW_OK;
  }
  // MW_NO_TWO_STEP=1 in the environment runs every step with the one-step
  // kernel (for comparisons)
  static bool pairs_disabled() {
    const char *e = getenv("MW_NO_TWO_STEP");
    return e && e[0] == '1';
  }
};

// Step arguments shared by every stencil launch of a call.
StepArgs step_args(const mw_params *p, const Launch &lc, const float *ca, const float *cb,
                   const float *cq, int *flags, const char *ws, const Layout &L) {
  StepArgs a{};
  a.g = lc.g;
  a.c = coef_of(p);
  a.ca = ca;
  a.cb = cb;
  a.cq = cq;
  a.flags = flags;
  a.bt = (const float *)(ws + L.bandtab);
  return a;
}

// ---- per-kernel event timing ------------------------------------------------
struct Timer {
  std::mutex mu;
  bool on = false;
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Timer &timer() {
  static Timer t;
  return t;
}

template <typename F>
cudaError_t timed(int cls, cudaStream_t st, F &&launch) {
  Timer &T = timer();
  if (!T.on) return launch();
  std::lock_guard<std::mutex> lk(T.mu);
  cudaEvent_t a = T.get(), b = T.get();
  cudaEventRecord(a, st);
  cudaError_t e = launch();
  cudaEventRecord(b, st);
  T.recs.push_back({cls, {a, b}});
  return e;
}

// Small grids (at most kSmallCells cells over all shots) with every snapshot
// on the device, or none, run each sweep as one cooperative launch
// (mw_small.cu); MW_NO_SMALL=1 in the environment keeps the step-by-step
// launches (for comparisons).
constexpr int64_t kSmallCells = (int64_t)1 << 20;
bool small_path(const mw_params *p, bool adjoint, int store, SmallPlan *pl) {
  const char *e = getenv("MW_NO_SMALL");
  if (e && e[0] == '1') return false;
  if (p->snap_host || is_ckpt(p)) return false;
  if ((int64_t)p->n_shots * p->ny * p->nx > kSmallCells) return false;
  const Bands b = bands(p);
  return small_plan(p->order, adjoint, store, p->ny, p->nx, b.Wx, b.Wz, p->n_src, p->n_rec, pl);
}
SmallArgs small_args(const mw_params *p, const float *ca, const float *cb, const float *cq,
                     char *ws, const Layout &L, int *flags) {
  SmallArgs s{};
  const Bands b = bands(p);
  s.S = p->n_shots;
  s.ny = p->ny;
  s.nx = p->nx;
  s.Wx = b.Wx;
  s.Wz = b.Wz;
  s.n_pml = p->n_pml;
  s.grad_mask = p->grad_mask_pml ? 1 : 0;
  s.batched = p->model_batched ? 1 : 0;
  s.cq_arr = p->cq_is_scalar ? 0 : 1;
  s.nt = p->nt;
  s.numel = (int64_t)p->ny * p->nx;
  s.c = coef_of(p);
  s.ca = ca;
  s.cb = cb;
  s.cq = cq;
  s.bt = (const float *)(ws + L.bandtab);
  s.snap_pitch = L.snap_pitch;
  s.flags = flags;
  if (p->snap_mode != MW_SNAP_NONE) {
    s.snap_e = ws + L.snap;
    s.snap_c = ws + L.snap + (size_t)p->nt * L.snap_step_bytes;
    s.step_elems = (int64_t)(L.snap_step_bytes / snap_elem_bytes(p->snap_mode));
  }
  return s;
}
int run_small(const mw_params *p, SmallArgs &s, bool adjoint, int store, const SmallPlan &pl,
              cudaStream_t st) {
  // profile classes of whole-sweep launches: 6 / 7 / 8 resident, 9 / 10 / 11
  // state in global memory (forward, forward with snapshots, adjoint)
  const int cls = (pl.resident ? 6 : 9) + (adjoint ? 2 : (store ? 1 : 0));
  MW_CUDA(timed(cls, st, [&] { return launch_small(s, adjoint, p->order, store, pl, st); }));
  return MW_OK;
}

int check_ptr(const void *ptr, const char *name) {
  if (!ptr) return fail(MW_ERR_ARG, "%s is NULL", name);
  if (((uintptr_t)ptr) % 16 != 0) return fail(MW_ERR_ARG, "%s is not 16-byte aligned", name);
  return MW_OK;
}

// Checkpoint replay: re-runs the forward from checkpoint k (read in place)
// over its segment [k C, min((k + 1) C, t_end)) and stores each step's E and
// curl (fp32), or E alone, in the segment buffer at slot t - k C.  Used by
// the adjoint (segments newest first) and the Born forward (oldest first).
struct Replay {
  const mw_params *p = nullptr;
  char *ws = nullptr;
  Layout L{};
  cudaStream_t st = nullptr;
  const float *f = nullptr;
  EntrySet src{};
  Launch lf{};
  StepArgs fa{};
  FwdMaps fA, fB, fS;  // inputs rA, rB, the segment's checkpoint
  Pairs pr;            // two steps per launch within a segment
  Fwd2Maps f2A, f2B, f2S;
  const float *ca_ = nullptr, *cb_ = nullptr, *cq_ = nullptr;
  float *rA = nullptr, *rB = nullptr;
  int store = kStoreF32;  // the segment: E and curl, or E alone (kStoreEy)
  float *last = nullptr;  // the state after the latest replayed segment

  int init(const mw_params *p_, char *ws_, const Layout &L_, cudaStream_t st_, const float *ca,
           const float *cb, const float *cq, int *flags, const float *f_,
           const EntrySet &src_) {
    p = p_;
    ws = ws_;
    L = L_;
    st = st_;
    f = f_;
    src = src_;
    lf = plan(p, kPlanFwd);
    fa = step_args(p, lf, ca, cb, cq, flags, ws, L);
    set_layout(fa, p, false);
    fa.ea = src;  // sources injected, nothing recorded
    fa.snap_pitch = p->nx;  // the fp32 segment
    rA = (float *)(ws + L.rpA);
    rB = (float *)(ws + L.rpB);
    ca_ = ca;
    cb_ = cb;
    cq_ = cq;
    MW_TRY(fwd_maps(p, fields_at(p, rA), ca, cb, cq, &fA));
    MW_TRY(fwd_maps(p, fields_at(p, rB), ca, cb, cq, &fB));
    MW_TRY(pr.init(p, fa));
    if (pr.on) {
      MW_TRY(fwd2_maps(p, fields_at(p, rA), ca, cb, &f2A));
      MW_TRY(fwd2_maps(p, fields_at(p, rB), ca, cb, &f2B));
    }
    return MW_OK;
  }
  // replay segment k up to step t_end at most; *t0 / *t1 receive its steps
  int segment(int k, int *launch_idx, int *t0_out, int *t1_out, int t_end) {
    const int C = p->ckpt_every;
    const int t0 = k * C;
    const int t1 = (t0 + C < t_end) ? t0 + C : t_end;
    char *seg_e = ws + L.seg;
    char *seg_c = seg_e + (size_t)C * L.snap_step_bytes;
    // the first step reads the checkpoint in place
    float *rc = ckpt_slot(ws, L, k), *rn = rA;
    MW_TRY(fwd_maps(p, fields_at(p, rc), ca_, cb_, cq_, &fS));
    if (pr.on) MW_TRY(fwd2_maps(p, fields_at(p, rc), ca_, cb_, &f2S));
    for (int t = t0; t < t1;) {
      const bool pair = pr.on && t + 1 < t1;
      rn = rc == rA ? rB : rA;
      const float *f_t = f ? f + (int64_t)t * p->n_shots * p->n_src : nullptr;
      if (pair) {
        StepArgs &b = pr.a;
        b.in = fields_at(p, rc);
        b.out = fields_at(p, rn);
        b.snap_e = seg_e + (size_t)(t - t0) * L.snap_step_bytes;
        b.snap_c = seg_c + (size_t)(t - t0) * L.snap_step_bytes;
        b.snap_e2 = seg_e + (size_t)(t + 1 - t0) * L.snap_step_bytes;
        b.snap_c2 = seg_c + (size_t)(t + 1 - t0) * L.snap_step_bytes;
        b.vals_t = f_t;
        b.vals_t2 = f ? f_t + (int64_t)p->n_shots * p->n_src : nullptr;
        b.ctr_slot = ((*launch_idx)++) & 1;
        const Fwd2Maps &fm = rc == rA ? f2A : rc == rB ? f2B : f2S;
        MW_CUDA(timed(5, st, [&] {
          return launch_forward2(fm, b, p->order, store, p->model_batched != 0, pr.lc.grid, st);
        }));
        t += 2;
      } else {
        fa.in = fields_at(p, rc);
        fa.out = fields_at(p, rn);
        fa.snap_e = seg_e + (size_t)(t - t0) * L.snap_step_bytes;
        fa.snap_c = seg_c + (size_t)(t - t0) * L.snap_step_bytes;
        fa.ctr_slot = ((*launch_idx)++) & 1;
        fa.vals_t = f_t;
        const FwdMaps &fm = rc == rA ? fA : rc == rB ? fB : fS;
        MW_CUDA(timed(1, st, [&] {
          return launch_forward(fm, fa, p->order, store, kStoreNone, p->model_batched != 0,
                                !p->cq_is_scalar, lf.grid, st);
        }));
        t += 1;
      }
      rc = rn;
    }
    last = rc;
    *t0_out = t0;
    *t1_out = t1;
    return MW_OK;
  }
};

// Host -> device-ring copies of the pinned-host snapshot store: step t goes
// to ring slot t % kHostRing, on the copy stream, after the slot's previous
// reader (if any) has finished.
struct HostFetch {
  HostCopies *hc;
  const char *hbuf;
  const char *se, *sc;
  size_t step_bytes;
  int fetch(int t, bool slot_was_used) {
    const int slot = t % kHostRing;
    if (slot_was_used) MW_CUDA(cudaStreamWaitEvent(hc->cs, hc->freed[slot], 0));
    const char *h = hbuf + 2 * (size_t)t * step_bytes;
    MW_CUDA(cudaMemcpyAsync((void *)(se + (size_t)slot * step_bytes), h, step_bytes,
                            cudaMemcpyHostToDevice, hc->cs));
    MW_CUDA(cudaMemcpyAsync((void *)(sc + (size_t)slot * step_bytes), h + step_bytes, step_bytes,
                            cudaMemcpyHostToDevice, hc->cs));
    MW_CUDA(cudaEventRecord(hc->filled[slot], hc->cs));
    return MW_OK;
  }
};


}  // namespace
}  // namespace mw

using namespace mw;

extern "C" {

void mw_params_init(mw_params *p) {
  if (!p) return;
  memset(p, 0, sizeof *p);
  p->cq_is_scalar = 1;
  p->snap_mode = MW_SNAP_NONE;
}

size_t mw_state_floats(const mw_params *p) {
  if (check_params(p, false) != MW_OK) return 0;
  return state_floats(p);
}

size_t mw_snap_host_bytes(const mw_params *p) {
  if (check_params(p, false) != MW_OK || !p->snap_host) return 0;
  return 2 * (size_t)p->nt * layout(p).snap_step_bytes;
}

size_t mw_workspace_bytes(const mw_params *p) {
  if (check_params(p, false) != MW_OK) return 0;
  return layout(p).total;
}

double mw_cfl_dt(int32_t order, double dy, double dx, double vmax) {
  double c[4];
  const int P = stencil_weights(order, c);
  if (!P || !(dy > 0) || !(dx > 0) || !(vmax > 0)) return -1.0;
  double s = 0.0;
  for (int k = 0; k < P; ++k) s += fabs(c[k]);
  return 1.0 / (vmax * s * sqrt(1.0 / (dx * dx) + 1.0 / (dy * dy)));
}

int mw_validate(const mw_params *p) {
  g_err.clear();
  return check_params(p, true);
}

const char *mw_last_error(void) { return g_err.c_str(); }

int mw_model_from_eps_sigma(const mw_params *p, const float *eps_r, const float *sigma,
                            const float *mu_r, float *ca, float *cb, float *cq, void *stream) {
  g_err.clear();
  int rc = check_params(p, false);
  if (rc) return rc;
  if (!eps_r || !ca || !cb || !cq) return fail(MW_ERR_ARG, "NULL model pointer");
  if (p->cq_is_scalar && mu_r) return fail(MW_ERR_ARG, "mu_r given but cq_is_scalar = 1");
  const int64_t n = (int64_t)(p->model_batched ? p->n_shots : 1) * p->ny * p->nx;
  MW_CUDA(launch_model(n, eps_r, sigma, mu_r, p->dt, ca, cb, cq, p->cq_is_scalar ? 0 : 1,
                       (cudaStream_t)stream));
  return MW_OK;
}

int mw_cpml_profiles(const mw_params *p, double f0, double R, float *cpml, void *stream) {
  g_err.clear();
  int rc = check_params(p, false);
  if (rc) return rc;
  if (!cpml) return fail(MW_ERR_ARG, "cpml is NULL");
  if (p->n_pml > 0 && (!(p->vmax > 0) || !(f0 >= 0) || !(R > 0 && R < 1)))
    return fail(MW_ERR_ARG, "CPML needs vmax > 0, f0 >= 0, 0 < R < 1");
  MW_CUDA(launch_cpml(p->ny, p->nx, p->n_pml, p->dy, p->dx, p->dt, p->vmax, f0, R, cpml,
                      (cudaStream_t)stream));
  return MW_OK;
}

int mw_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  g_err.clear();
  if (!workspace || workspace_bytes < 256) return fail(MW_ERR_WORKSPACE, "workspace too small");
  MW_CUDA(cudaMemsetAsync(workspace, 0, 256, (cudaStream_t)stream));
  return MW_OK;
}

int mw_tm_forward(const mw_params *p, const float *ca, const float *cb, const float *cq,
                  const float *cpml, const float *f, const int64_t *src_idx,
                  const int64_t *rec_idx, float *state, float *rec, void *workspace,
                  size_t workspace_bytes, void *stream) {
  g_err.clear();
  int rc = check_params(p, true);
  if (rc) return rc;
  if ((rc = check_host_snap(p))) return rc;
  if ((rc = check_ptr(ca, "ca")) || (rc = check_ptr(cb, "cb")) || (rc = check_ptr(cpml, "cpml")))
    return rc;
  if (!cq) return fail(MW_ERR_ARG, "cq is NULL");
  if (!p->cq_is_scalar && (rc = check_ptr(cq, "cq"))) return rc;
  if (p->n_src > 0 && (!f || !src_idx)) return fail(MW_ERR_ARG, "sources need f and src_idx");
  if (p->n_rec > 0 && rec && !rec_idx) return fail(MW_ERR_ARG, "receivers need rec_idx");
  // MW_SNAP_CKPT_EY keeps its own copy of the records for the adjoint
  const bool ey_only = p->snap_mode == MW_SNAP_CKPT_EY;
  if (ey_only && p->n_rec > 0 && !rec_idx)
    return fail(MW_ERR_ARG, "snap_mode CKPT_EY: receivers need rec_idx");
  if (state && (rc = check_ptr(state, "state"))) return rc;
  if (!workspace) return fail(MW_ERR_WORKSPACE, "workspace is NULL");
  const Layout L = layout(p);
  if (workspace_bytes < L.total)
    return fail(MW_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
  if (((uintptr_t)workspace) % 256 != 0) return fail(MW_ERR_WORKSPACE, "workspace not 256-aligned");
  cudaStream_t st = (cudaStream_t)stream;
  char *ws = (char *)workspace;
  int *flags = (int *)(ws + L.flags);

  float *bufA = state ? state : (float *)(ws + L.stA);
  float *bufB = (float *)(ws + L.stB);
  if (!state) MW_CUDA(cudaMemsetAsync(bufA, 0, L.state_bytes, st));
  if (p->nt == 0) return MW_OK;

  const Launch lc = plan(p, kPlanFwd);
  StepArgs a = step_args(p, lc, ca, cb, cq, flags, ws, L);
  set_layout(a, p, false);
  a.snap_pitch = L.snap_pitch;
  MW_TRY(stencil_prologue(p, cpml, ws, L, st));
  FwdMaps mA, mB;  // input buffer A / B
  MW_TRY(fwd_maps(p, fields_at(p, bufA), ca, cb, cq, &mA));
  MW_TRY(fwd_maps(p, fields_at(p, bufB), ca, cb, cq, &mB));

  const int store = snap_store_kind(p->snap_mode);
  // checkpoint modes: the last n_tail steps store their snapshots themselves
  const int t_tail = p->nt - L.n_tail;
  const int tail_store = ey_only ? kStoreEy : kStoreF32;
  char *tail_e = ws + L.tail;
  char *tail_c = tail_e + (size_t)L.n_tail * L.snap_step_bytes;
  const int64_t SN = (int64_t)p->n_shots * p->ny * p->nx;
  const Tables tb = tables_at(p, ws, L);
  float *rec_out = ey_only ? (float *)(ws + L.rcopy) : rec;
  MW_TRY(build_table(p, src_idx, p->n_src, ws, L.tab_src, flags, nullptr, st));
  if (rec_out) MW_TRY(build_table(p, rec_idx, p->n_rec, ws, L.tab_rec, flags, rec_out, st));
  a.ea = tb.src;
  if (rec_out) a.eb = tb.rec;
  SmallPlan spl{};
  if (small_path(p, false, store, &spl)) {  // every step in one launch, the state in place
    SmallArgs sa = small_args(p, ca, cb, cq, ws, L, flags);
    sa.st = fields_at(p, bufA);
    sa.src = tb.src;
    sa.f = f;
    if (rec_out) {
      sa.rec = tb.rec;
      sa.rec_out = rec_out;
    }
    MW_TRY(run_small(p, sa, false, store, spl, st));
    if (p->check_finite) MW_CUDA(launch_check_finite(bufA, 3 * SN, flags, st));
    return MW_OK;
  }
  const bool host = p->snap_host != 0;
  const size_t ring_steps = host ? (size_t)kHostRing : (size_t)p->nt;
  char *snap_e = ws + L.snap;
  char *snap_c = ws + L.snap + ring_steps * L.snap_step_bytes;
  HostCopies hc;
  if (host) MW_TRY(hc.init());
  char *hbuf = (char *)p->snap_host_ptr;
  float *cur = bufA, *nxt = bufB;
  // checkpoint modes: checkpoint 0 is a copy of the initial state; the step
  // that produces the state of checkpoint k >= 1 writes it into the slot
  // directly and the next step reads it from there (no copies)
  const bool ck = is_ckpt(p);
  if (ck) MW_CUDA(cudaMemcpyAsync(ckpt_slot(ws, L, 0), bufA, L.state_bytes,
                                  cudaMemcpyDeviceToDevice, st));
  // the snapshot destination and store kind of step t
  auto snap_of = [&](int t, void **e, void **c) -> int {
    const int slot = host ? t % kHostRing : t;
    if (t >= t_tail && L.n_tail > 0) {
      *e = tail_e + (size_t)(t - t_tail) * L.snap_step_bytes;
      *c = tail_c + (size_t)(t - t_tail) * L.snap_step_bytes;
      return tail_store;
    }
    *e = store ? snap_e + (size_t)slot * L.snap_step_bytes : nullptr;
    *c = store ? snap_c + (size_t)slot * L.snap_step_bytes : nullptr;
    return store;
  };
  // two steps per launch where the state between them is not needed (no
  // checkpoint after the first) and both store alike; not with the host
  // snapshot ring, which copies every step out on its own
  Pairs pr;
  MW_TRY(pr.init(p, a));
  Fwd2Maps m2A, m2B, m2S;
  if (pr.on && !host) {
    MW_TRY(fwd2_maps(p, fields_at(p, bufA), ca, cb, &m2A));
    MW_TRY(fwd2_maps(p, fields_at(p, bufB), ca, cb, &m2B));
  }
  FwdMaps mS;  // input maps of a checkpoint slot
  int launch_idx = 0;
  const int C = ck ? p->ckpt_every : 0;
  for (int t = 0; t < p->nt;) {
    const bool pair = pr.on && !host && t + 1 < p->nt && !(ck && (t + 1) % C == 0) &&
                      (L.n_tail == 0 || (t >= t_tail) == (t + 1 >= t_tail));
    const int tn = pair ? t + 2 : t + 1;  // steps done after this launch
    const int k_out = ck && tn % C == 0 ? tn / C : -1;
    nxt = k_out > 0 && k_out < L.n_seg ? ckpt_slot(ws, L, k_out) : cur == bufA ? bufB : bufA;
    const int slot = host ? t % kHostRing : t;
    // the slot's previous step must have reached the host
    if (host && t >= kHostRing) MW_CUDA(cudaStreamWaitEvent(st, hc.freed[slot], 0));
    const float *f_t = f ? f + (int64_t)t * p->n_shots * p->n_src : nullptr;
    float *rec_t = rec_out ? rec_out + (int64_t)t * p->n_shots * p->n_rec : nullptr;
    if (pair) {
      StepArgs &b = pr.a;
      b.in = fields_at(p, cur);
      b.out = fields_at(p, nxt);
      const int kind = snap_of(t, &b.snap_e, &b.snap_c);
      snap_of(t + 1, &b.snap_e2, &b.snap_c2);
      b.vals_t = f_t;
      b.vals_t2 = f ? f_t + (int64_t)p->n_shots * p->n_src : nullptr;
      b.out_t = rec_t;
      b.out_t2 = rec_out ? rec_t + (int64_t)p->n_shots * p->n_rec : nullptr;
      b.ctr_slot = (launch_idx++) & 1;
      if (cur != bufA && cur != bufB) MW_TRY(fwd2_maps(p, b.in, ca, cb, &m2S));
      const Fwd2Maps &m2 = cur == bufA ? m2A : cur == bufB ? m2B : m2S;
      MW_CUDA(timed(kind ? 5 : 4, st, [&] {
        return launch_forward2(m2, b, p->order, kind, p->model_batched != 0, pr.lc.grid, st);
      }));
    } else {
      a.in = fields_at(p, cur);
      a.out = fields_at(p, nxt);
      const int kind = snap_of(t, &a.snap_e, &a.snap_c);
      if (cur != bufA && cur != bufB) MW_TRY(fwd_maps(p, a.in, ca, cb, cq, &mS));
      const FwdMaps &m = cur == bufA ? mA : cur == bufB ? mB : mS;
      a.ctr_slot = (launch_idx++) & 1;
      a.vals_t = f_t;
      a.out_t = rec_t;
      MW_CUDA(timed(kind ? 1 : 0, st, [&] {
        return launch_forward(m, a, p->order, kind, kStoreNone, p->model_batched != 0,
                              !p->cq_is_scalar, lc.grid, st);
      }));
      if (host) {  // step t: ring slot -> host, on the copy stream
        MW_CUDA(cudaEventRecord(hc.filled[slot], st));
        MW_CUDA(cudaStreamWaitEvent(hc.cs, hc.filled[slot], 0));
        char *h = hbuf + 2 * (size_t)t * L.snap_step_bytes;
        MW_CUDA(cudaMemcpyAsync(h, a.snap_e, L.snap_step_bytes, cudaMemcpyDeviceToHost, hc.cs));
        MW_CUDA(cudaMemcpyAsync(h + L.snap_step_bytes, a.snap_c, L.snap_step_bytes,
                                cudaMemcpyDeviceToHost, hc.cs));
        MW_CUDA(cudaEventRecord(hc.freed[slot], hc.cs));
      }
    }
    cur = nxt;
    t = tn;
  }
  if (ey_only && rec && p->n_rec > 0)
    MW_CUDA(cudaMemcpyAsync(rec, rec_out, (size_t)p->nt * p->n_shots * p->n_rec * sizeof(float),
                            cudaMemcpyDeviceToDevice, st));
  if (host)  // the call's stream completes only after every copy reached the host
    for (int k = 0; k < kHostRing && k < p->nt; ++k)
      MW_CUDA(cudaStreamWaitEvent(st, hc.freed[(p->nt - 1 - k) % kHostRing], 0));
  if (cur != bufA) MW_CUDA(cudaMemcpyAsync(bufA, cur, L.state_bytes, cudaMemcpyDeviceToDevice, st));
  if (ey_only && L.n_tail > 0)  // the final E, for the adjoint's end term
    MW_CUDA(cudaMemcpyAsync(tail_e + (size_t)L.n_tail * L.snap_step_bytes, bufA,
                            SN * sizeof(float), cudaMemcpyDeviceToDevice, st));
  if (p->check_finite) MW_CUDA(launch_check_finite(bufA, 3 * SN, flags, st));
  return MW_OK;
}

int mw_tm_adjoint_grad(const mw_params *p, const float *ca, const float *cb, const float *cq,
                       const float *cpml, const float *f, const int64_t *src_idx,
                       const int64_t *rec_idx, const float *res, float *gca, float *gcb,
                       float *grad_f, float *adj_state, void *workspace, size_t workspace_bytes,
                       void *stream) {
  g_err.clear();
  int rc = check_params(p, true);
  if (rc) return rc;
  if ((rc = check_host_snap(p))) return rc;
  if (p->snap_mode == MW_SNAP_NONE)
    return fail(MW_ERR_ARG, "snap_mode NONE: the forward stored nothing to differentiate");
  if ((rc = check_ptr(ca, "ca")) || (rc = check_ptr(cb, "cb")) || (rc = check_ptr(cpml, "cpml")) ||
      (rc = check_ptr(gca, "grad_ca_shot")) || (rc = check_ptr(gcb, "grad_cb_shot")))
    return rc;
  if (!cq) return fail(MW_ERR_ARG, "cq is NULL");
  if (!p->cq_is_scalar && (rc = check_ptr(cq, "cq"))) return rc;
  if (p->n_rec > 0 && (!res || !rec_idx)) return fail(MW_ERR_ARG, "receivers need res and rec_idx");
  if (p->n_src > 0 && grad_f && !src_idx) return fail(MW_ERR_ARG, "grad_f needs src_idx");
  if (is_ckpt(p) && p->n_src > 0 && (!f || !src_idx))
    return fail(MW_ERR_ARG, "checkpoint replay needs f and src_idx");
  if (adj_state && (rc = check_ptr(adj_state, "adj_state"))) return rc;
  if (!workspace) return fail(MW_ERR_WORKSPACE, "workspace is NULL");
  const Layout L = layout(p);
  if (workspace_bytes < L.total)
    return fail(MW_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
  if (((uintptr_t)workspace) % 256 != 0) return fail(MW_ERR_WORKSPACE, "workspace not 256-aligned");
  cudaStream_t st = (cudaStream_t)stream;
  char *ws = (char *)workspace;
  int *flags = (int *)(ws + L.flags);
  const int64_t numel = (int64_t)p->ny * p->nx;
  const int64_t SN = p->n_shots * numel;

  // MW_SNAP_CKPT_EY: lambda_E at the sources of every step (the source end
  // term), in grad_f or in the workspace
  const bool ey_only = p->snap_mode == MW_SNAP_CKPT_EY;
  float *gf_all = grad_f ? grad_f : ey_only ? (float *)(ws + L.gfbuf) : nullptr;
  const Tables tb = tables_at(p, ws, L);
  MW_TRY(build_table(p, rec_idx, p->n_rec, ws, L.tab_rec, flags, nullptr, st));
  // the sources: sampled (grad_f, the end term) and injected by the replay
  if (src_idx && (gf_all || is_ckpt(p)))
    MW_TRY(build_table(p, src_idx, p->n_src, ws, L.tab_src, flags, gf_all, st));
  float *adA = adj_state ? adj_state : (float *)(ws + L.adA);
  float *adB = (float *)(ws + L.adB);
  if (!adj_state) MW_CUDA(cudaMemsetAsync(adA, 0, L.state_bytes, st));
  if (p->nt == 0) return MW_OK;
  SmallPlan spl{};
  if (small_path(p, true, snap_store_kind(p->snap_mode), &spl)) {
    // every step in one launch, the adjoint state in place
    MW_TRY(stencil_prologue(p, cpml, ws, L, st));
    SmallArgs sa = small_args(p, ca, cb, cq, ws, L, flags);
    sa.st = fields_at(p, adA);
    sa.rec = tb.rec;
    sa.res = res;
    if (gf_all && src_idx) {
      sa.src = tb.src;
      sa.grad_f = gf_all;
    }
    sa.gca = gca;
    sa.gcb = gcb;
    // scratch: the second adjoint buffer's fields and the forward's spare one
    const Fields s1 = fields_at(p, adB), s2 = fields_at(p, (float *)(ws + L.stB));
    sa.px = s1.ey;
    sa.pz = s1.hx;
    sa.qx = s1.hz;
    sa.qz = s2.ey;
    MW_TRY(run_small(p, sa, true, snap_store_kind(p->snap_mode), spl, st));
    if (p->check_finite) {
      MW_CUDA(launch_check_finite(gca, SN, flags, st));
      MW_CUDA(launch_check_finite(gcb, SN, flags, st));
    }
    return MW_OK;
  }

  const Launch la = plan(p, kPlanAdj);
  // MW_SNAP_CKPT_EY: the Cb gradient accumulates E^t G^t into P (workspace)
  // and the end-term sums beside it; grad_cb_shot receives P / Cb at the end
  float *sbp = ey_only ? (float *)(ws + L.sbp) : nullptr;
  float *acc_rec = ey_only ? (float *)(ws + L.acc) : nullptr;
  float *acc_src = ey_only ? acc_rec + (size_t)p->n_shots * p->n_rec : nullptr;
  const float *rcopy = ey_only ? (const float *)(ws + L.rcopy) : nullptr;
  if (ey_only) MW_CUDA(cudaMemsetAsync(sbp, 0, SN * sizeof(float), st));
  StepArgs a = step_args(p, la, ca, cb, cq, flags, ws, L);
  a.gca = gca;
  a.gcb = ey_only ? sbp : gcb;
  set_layout(a, p, true);
  MW_TRY(stencil_prologue(p, cpml, ws, L, st));
  int launch_idx = 0;  // alternates the work counter between stencil launches

  // snapshot source of the adjoint: the full store, or the replay segment
  const bool ckpt = is_ckpt(p);
  // snapshots the adjoint reads: the full store, or the fp32 replay segment
  // (E and curl, or E alone)
  const int snap = ey_only ? kStoreEy : ckpt ? kStoreF32 : snap_store_kind(p->snap_mode);
  const int snap_elem = ckpt ? 4 : (int)snap_elem_bytes(p->snap_mode);
  const bool host = p->snap_host != 0;
  const int C = ckpt ? p->ckpt_every : host ? kHostRing : p->nt;
  const char *snap_e = ckpt ? ws + L.seg : ws + L.snap;
  const char *snap_c = snap_e + (size_t)C * L.snap_step_bytes;
  AdjMaps mA, mB;
  MW_TRY(adj_maps(p, fields_at(p, adA), ca, cb, cq, gca, a.gcb, snap_e, snap_c, snap_elem, C,
                  L.snap_pitch, ey_only, &mA));
  MW_TRY(adj_maps(p, fields_at(p, adB), ca, cb, cq, gca, a.gcb, snap_e, snap_c, snap_elem, C,
                  L.snap_pitch, ey_only, &mB));
  // checkpoint modes: the tail the forward stored, read in place
  const int t_tail = ckpt ? p->nt - L.n_tail : p->nt;
  AdjMaps tA, tB;
  if (ckpt && L.n_tail > 0) {
    const char *te = ws + L.tail, *tc = te + (size_t)L.n_tail * L.snap_step_bytes;
    MW_TRY(adj_maps(p, fields_at(p, adA), ca, cb, cq, gca, a.gcb, te, tc, snap_elem, L.n_tail,
                    L.snap_pitch, ey_only, &tA));
    MW_TRY(adj_maps(p, fields_at(p, adB), ca, cb, cq, gca, a.gcb, te, tc, snap_elem, L.n_tail,
                    L.snap_pitch, ey_only, &tB));
  }

  float *cur = adA, *nxt = adB;
  a.ea = tb.rec;  // residuals injected
  if (gf_all && src_idx) a.eb = tb.src;  // lambda_E sampled at the sources
  const bool sample_src = gf_all && src_idx;
  auto adj_step = [&](int t, int slot) -> int {
    // step t's residuals and source gradient: the step t + 1 launch applies
    // them to its output (the first step applies its own to the start state)
    if (t == p->nt - 1)
      MW_CUDA(launch_fix_field(cur, p->n_shots, p->ny, p->nx, tb.rec,
                               res ? res + (int64_t)t * p->n_shots * p->n_rec : nullptr, tb.src,
                               sample_src ? gf_all + (int64_t)t * p->n_shots * p->n_src : nullptr,
                               st));
    a.vals_t = res && t > 0 ? res + (int64_t)(t - 1) * p->n_shots * p->n_rec : nullptr;
    a.out_t = sample_src && t > 0 ? gf_all + (int64_t)(t - 1) * p->n_shots * p->n_src : nullptr;
    a.in = fields_at(p, cur);
    a.out = fields_at(p, nxt);
    a.snap_t = slot;
    a.tzero = t == 0 ? 1 : 0;
    a.ctr_slot = (launch_idx++) & 1;
    const bool in_tail = t >= t_tail;
    const AdjMaps &m = cur == adA ? (in_tail ? tA : mA) : (in_tail ? tB : mB);
    MW_CUDA(timed(2, st, [&] {
      return launch_adjoint(m, a, p->order, snap, p->model_batched != 0, !p->cq_is_scalar,
                            la.grid, st);
    }));
    std::swap(cur, nxt);
    return MW_OK;
  };

  if (host) {
    // pinned-host snapshots: prefetch step t into ring slot t % kHostRing on
    // the copy stream, kHostRing steps ahead of the adjoint that reads it
    HostCopies hc;
    MW_TRY(hc.init());
    MW_CUDA(cudaEventRecord(hc.start, st));
    MW_CUDA(cudaStreamWaitEvent(hc.cs, hc.start, 0));
    HostFetch hf{&hc, (const char *)p->snap_host_ptr, snap_e, snap_c, L.snap_step_bytes};
    for (int t = p->nt - 1; t >= 0 && t >= p->nt - kHostRing; --t) MW_TRY(hf.fetch(t, false));
    for (int t = p->nt - 1; t >= 0; --t) {
      const int slot = t % kHostRing;
      MW_CUDA(cudaStreamWaitEvent(st, hc.filled[slot], 0));
      MW_TRY(adj_step(t, slot));
      MW_CUDA(cudaEventRecord(hc.freed[slot], st));
      if (t - kHostRing >= 0) MW_TRY(hf.fetch(t - kHostRing, true));
    }
  } else if (!ckpt) {
    for (int t = p->nt - 1; t >= 0; --t) MW_TRY(adj_step(t, t));
  } else {
    // checkpoint mode: replay each segment from its checkpoint, newest first
    // the tail first (no replay), then each earlier segment replayed from its
    // checkpoint; a given adjoint start state meets the forward's final E:
    // P starts at lambda~_E^{nt} E^{nt}
    Replay rp;
    MW_TRY(rp.init(p, ws, L, st, ca, cb, cq, flags, f, tb.src));
    rp.store = ey_only ? kStoreEy : kStoreF32;
    if (L.n_tail > 0) {
      if (ey_only && adj_state)
        MW_CUDA(launch_sbp_init(sbp, adA,
                                (const float *)(ws + L.tail + (size_t)L.n_tail * L.snap_step_bytes),
                                SN, st));
      for (int t = p->nt - 1; t >= t_tail; --t) MW_TRY(adj_step(t, t - t_tail));
    }
    const int n_rep = (t_tail + p->ckpt_every - 1) / p->ckpt_every;
    for (int k = n_rep - 1; k >= 0; --k) {
      int t0, t1;
      MW_TRY(rp.segment(k, &launch_idx, &t0, &t1, t_tail));
      if (ey_only && adj_state && L.n_tail == 0 && k == n_rep - 1)
        MW_CUDA(launch_sbp_init(sbp, adA, rp.last, SN, st));
      for (int t = t1 - 1; t >= t0; --t) MW_TRY(adj_step(t, t - t0));
    }
  }
  if (cur != adA) MW_CUDA(cudaMemcpyAsync(adA, cur, L.state_bytes, cudaMemcpyDeviceToDevice, st));
  if (ey_only) {
    MW_CUDA(launch_sbp_sums(p->nt, p->n_shots, res, rcopy, p->n_rec, acc_rec,
                            src_idx ? f : nullptr, gf_all, p->n_src, acc_src, st));
    MW_CUDA(launch_sbp_scatter(sbp, numel, p->n_shots, rec_idx, acc_rec, res ? p->n_rec : 0,
                               src_idx, acc_src, f && src_idx ? p->n_src : 0, st));
    MW_CUDA(launch_sbp_finish(sbp, cb, gcb, p->n_shots, p->ny, p->nx, p->model_batched,
                              p->grad_mask_pml ? p->n_pml : 0, st));
  }
  if (p->check_finite) {
    MW_CUDA(launch_check_finite(gca, SN, flags, st));
    MW_CUDA(launch_check_finite(gcb, SN, flags, st));
  }
  return MW_OK;
}

int mw_tm_born(const mw_params *p, const float *ca, const float *cb, const float *cq,
               const float *cpml, const float *dca, const float *dcb, const float *f,
               const int64_t *src_idx, const int64_t *rec_idx, float *rec, void *workspace,
               size_t workspace_bytes, void *stream) {
  g_err.clear();
  int rc = check_params(p, true);
  if (rc) return rc;
  if ((rc = check_host_snap(p))) return rc;
  if (p->snap_mode == MW_SNAP_NONE)
    return fail(MW_ERR_ARG, "snap_mode NONE: the forward stored no background snapshots");
  if ((rc = check_ptr(ca, "ca")) || (rc = check_ptr(cb, "cb")) || (rc = check_ptr(cpml, "cpml")) ||
      (rc = check_ptr(dca, "dca")) || (rc = check_ptr(dcb, "dcb")))
    return rc;
  if (!cq) return fail(MW_ERR_ARG, "cq is NULL");
  if (!p->cq_is_scalar && (rc = check_ptr(cq, "cq"))) return rc;
  if (p->n_rec > 0 && (!rec || !rec_idx)) return fail(MW_ERR_ARG, "receivers need rec and rec_idx");
  const bool ckpt = is_ckpt(p);
  if (ckpt && p->n_src > 0 && (!f || !src_idx))
    return fail(MW_ERR_ARG, "checkpoint replay needs f and src_idx");
  if (!workspace) return fail(MW_ERR_WORKSPACE, "workspace is NULL");
  const Layout L = layout(p);
  if (workspace_bytes < L.total)
    return fail(MW_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
  if (((uintptr_t)workspace) % 256 != 0) return fail(MW_ERR_WORKSPACE, "workspace not 256-aligned");
  cudaStream_t st = (cudaStream_t)stream;
  char *ws = (char *)workspace;
  int *flags = (int *)(ws + L.flags);
  const Tables tb = tables_at(p, ws, L);
  MW_TRY(build_table(p, rec_idx, p->n_rec, ws, L.tab_rec, flags, rec, st));
  if (ckpt) MW_TRY(build_table(p, src_idx, p->n_src, ws, L.tab_src, flags, nullptr, st));
  if (p->nt == 0) return MW_OK;

  // the perturbation state lives in the adjoint's buffers, from zero
  float *dA = (float *)(ws + L.adA), *dB = (float *)(ws + L.adB);
  MW_CUDA(cudaMemsetAsync(dA, 0, L.state_bytes, st));
  const Launch lc = plan(p, kPlanFwd);
  StepArgs b = step_args(p, lc, ca, cb, cq, flags, ws, L);
  {
    size_t smem;
    forward_layout(p->order, bands(p).Wx, !p->cq_is_scalar, true, &b, &smem);
    const MdPair md = md_pairing(p, ca, cb), bd = md_pairing(p, dca, dcb);
    b.md_pair = md.pair ? 1 : 0;
    b.md_swap = md.swap ? 1 : 0;
    b.bd_pair = bd.pair ? 1 : 0;
    b.bd_swap = bd.swap ? 1 : 0;
  }
  b.eb = tb.rec;  // the perturbation's records; no sources
  MW_TRY(stencil_prologue(p, cpml, ws, L, st));

  // the background's snapshots: every step in the workspace, a 3-step ring
  // fed from pinned host memory, or a replayed checkpoint segment (fp32)
  const bool host = p->snap_host != 0;
  const int kind = ckpt ? kStoreF32 : snap_store_kind(p->snap_mode);
  const int elem = ckpt ? 4 : (int)snap_elem_bytes(p->snap_mode);
  const int steps = ckpt ? p->ckpt_every : host ? kHostRing : p->nt;
  const char *snap_e = ckpt ? ws + L.seg : ws + L.snap;
  const char *snap_c = snap_e + (size_t)steps * L.snap_step_bytes;
  FwdMaps mA, mB;
  MW_TRY(fwd_maps(p, fields_at(p, dA), ca, cb, cq, &mA));
  MW_TRY(fwd_maps(p, fields_at(p, dB), ca, cb, cq, &mB));
  MW_TRY(born_maps(p, dca, dcb, snap_e, snap_c, elem, steps, L.snap_pitch, &mA));
  MW_TRY(born_maps(p, dca, dcb, snap_e, snap_c, elem, steps, L.snap_pitch, &mB));

  int launch_idx = 0;
  float *cur = dA, *nxt = dB;
  auto born_step = [&](int t, int slot) -> int {
    b.in = fields_at(p, cur);
    b.out = fields_at(p, nxt);
    b.snap_t = slot;
    b.ctr_slot = (launch_idx++) & 1;
    b.out_t = rec ? rec + (int64_t)t * p->n_shots * p->n_rec : nullptr;
    const FwdMaps &m = cur == dA ? mA : mB;
    MW_CUDA(timed(3, st, [&] {
      return launch_forward(m, b, p->order, kStoreNone, kind, p->model_batched != 0,
                            !p->cq_is_scalar, lc.grid, st);
    }));
    std::swap(cur, nxt);
    return MW_OK;
  };

  if (host) {
    HostCopies hc;
    MW_TRY(hc.init());
    MW_CUDA(cudaEventRecord(hc.start, st));
    MW_CUDA(cudaStreamWaitEvent(hc.cs, hc.start, 0));
    HostFetch hf{&hc, (const char *)p->snap_host_ptr, snap_e, snap_c, L.snap_step_bytes};
    for (int t = 0; t < p->nt && t < kHostRing; ++t) MW_TRY(hf.fetch(t, false));
    for (int t = 0; t < p->nt; ++t) {
      const int slot = t % kHostRing;
      MW_CUDA(cudaStreamWaitEvent(st, hc.filled[slot], 0));
      MW_TRY(born_step(t, slot));
      MW_CUDA(cudaEventRecord(hc.freed[slot], st));
      if (t + kHostRing < p->nt) MW_TRY(hf.fetch(t + kHostRing, true));
    }
  } else if (!ckpt) {
    for (int t = 0; t < p->nt; ++t) MW_TRY(born_step(t, t));
  } else {
    // replay each segment of the background from its checkpoint into the fp32
    // segment buffer, then take the segment's linearised steps
    Replay rp;
    MW_TRY(rp.init(p, ws, L, st, ca, cb, cq, flags, f, tb.src));
    for (int k = 0; k < L.n_seg; ++k) {
      int t0, t1;
      MW_TRY(rp.segment(k, &launch_idx, &t0, &t1, p->nt));
      for (int t = t0; t < t1; ++t) MW_TRY(born_step(t, t - t0));
    }
  }
  return MW_OK;
}

int mw_combine_grad(const mw_params *p, const float *grad_shot, float *grad, int32_t accumulate,
                    void *stream) {
  g_err.clear();
  int rc = check_params(p, false);
  if (rc) return rc;
  if (!grad_shot || !grad) return fail(MW_ERR_ARG, "NULL gradient pointer");
  MW_CUDA(launch_combine(grad_shot, grad, p->n_shots, (int64_t)p->ny * p->nx, accumulate ? 1 : 0,
                         (cudaStream_t)stream));
  return MW_OK;
}

int mw_grad_eps_sigma(int64_t n, double dt, const float *ca, const float *cb, const float *gca,
                      const float *gcb, float *ge, float *gs, void *stream) {
  g_err.clear();
  if (n < 0 || !(dt > 0)) return fail(MW_ERR_ARG, "n < 0 or dt <= 0");
  if (!ca || !cb || !gca || !gcb) return fail(MW_ERR_ARG, "NULL input pointer");
  if (n == 0 || (!ge && !gs)) return MW_OK;
  MW_CUDA(launch_eps_sigma(n, dt, ca, cb, gca, gcb, ge, gs, (cudaStream_t)stream));
  return MW_OK;
}

int mw_residual(int64_t n, const float *d, const float *d_obs, float *res, double *J,
                void *stream) {
  g_err.clear();
  if (n < 0) return fail(MW_ERR_ARG, "n < 0");
  if (n > 0 && (!d || !d_obs || !res)) return fail(MW_ERR_ARG, "NULL pointer");
  if (n == 0) {
    if (J) MW_CUDA(cudaMemsetAsync(J, 0, sizeof(double), (cudaStream_t)stream));
    return MW_OK;
  }
  MW_CUDA(launch_residual(n, d, d_obs, res, J, (cudaStream_t)stream));
  return MW_OK;
}

int mw_sync_status(void *workspace, void *stream) {
  g_err.clear();
  cudaStream_t st = (cudaStream_t)stream;
  MW_CUDA(cudaStreamSynchronize(st));
  if (!workspace) return MW_OK;
  int h[3] = {0, 0, 0};
  MW_CUDA(cudaMemcpy(h, workspace, sizeof h, cudaMemcpyDeviceToHost));
  MW_CUDA(cudaMemset(workspace, 0, sizeof h));
  if (h[kFlagTimeout]) return fail(MW_ERR_TIMEOUT, "a stencil kernel timed out waiting for its copies");
  if (h[kFlagBadIndex]) return fail(MW_ERR_ARG, "a source or receiver index was out of range");
  if (h[kFlagNonFinite]) return fail(MW_ERR_NONFINITE, "non-finite value in a field or gradient");
  return MW_OK;
}

int64_t mw_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int mw_profile_enable(int32_t enable) {
  Timer &T = timer();
  std::lock_guard<std::mutex> lk(T.mu);
  for (auto &r : T.recs) {
    T.pool.push_back(r.second.first);
    T.pool.push_back(r.second.second);
  }
  T.recs.clear();
  T.on = enable != 0;
  return MW_OK;
}

int mw_selftest_wait_timeout(void *workspace, void *stream) {
  g_err.clear();
  if (!workspace) return fail(MW_ERR_WORKSPACE, "workspace is NULL");
  if (((uintptr_t)workspace) % 256 != 0) return fail(MW_ERR_WORKSPACE, "workspace not 256-aligned");
  MW_CUDA(launch_wait_selftest((int *)workspace, (cudaStream_t)stream));
  return MW_OK;
}

int mw_snapshot_encode(int32_t snap_mode, int64_t n, const float *x_dev, void *out_dev,
                       void *stream) {
  g_err.clear();
  if (snap_mode != MW_SNAP_BF16 && snap_mode != MW_SNAP_FP8)
    return fail(MW_ERR_ARG, "snap_mode %d has no narrow storage format", snap_mode);
  if (n < 0 || n % 4 != 0) return fail(MW_ERR_ARG, "n = %lld must be a multiple of 4", (long long)n);
  if (n == 0) return MW_OK;
  if (!x_dev || !out_dev) return fail(MW_ERR_ARG, "NULL pointer");
  const uintptr_t ax = (uintptr_t)x_dev, ao = (uintptr_t)out_dev;
  if (ax % 16 != 0 || ao % (snap_mode == MW_SNAP_BF16 ? 8 : 4) != 0)
    return fail(MW_ERR_ARG, "misaligned pointer");
  MW_CUDA(launch_snap_encode(snap_store_kind(snap_mode), n, x_dev, out_dev,
                             (cudaStream_t)stream));
  return MW_OK;
}

int mw_profile_read(int64_t *counts, double *total_ms, int32_t n_classes) {
  g_err.clear();
  Timer &T = timer();
  std::lock_guard<std::mutex> lk(T.mu);
  for (int i = 0; i < n_classes; ++i) {
    if (counts) counts[i] = 0;
    if (total_ms) total_ms[i] = 0.0;
  }
  for (auto &r : T.recs) {
    MW_CUDA(cudaEventSynchronize(r.second.second));
    float ms = 0.f;
    MW_CUDA(cudaEventElapsedTime(&ms, r.second.first, r.second.second));
    if (r.first >= 0 && r.first < n_classes) {
      if (counts) counts[r.first] += 1;
      if (total_ms) total_ms[r.first] += ms;
    }
  }
  return MW_OK;
}

// ---- forward without allocations -------------------------------------------
// The scratch of mw_tm_forward_noalloc: status words | source and receiver
// tables | CPML band table | the second state buffer of the ping-pong.  Host code must not
// use the symbol itself (it is a host-side stand-in); it takes the device
// address from cudaGetSymbolAddress with the calling device current.
}  // extern "C"

static __device__ __align__(256) unsigned char g_noalloc_scratch[MW_NOALLOC_SCRATCH_BYTES];

namespace mw {
namespace {
// The array's device address in the current device's context, looked up on
// every call: a cached address would dangle once the context is torn down
// (cudaDeviceReset) and the module is loaded again at another address.
int noalloc_scratch(char **out) {
  void *ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess || !ptr)
    return fail(MW_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed: %s",
                cudaGetErrorString(e));
  *out = (char *)ptr;
  return MW_OK;
}
}  // namespace
}  // namespace mw

extern "C" {

int mw_tm_forward_noalloc(const mw_params *p, const float *ca, const float *cb, const float *cq,
                          const float *cpml, const float *f, const int64_t *src_idx,
                          const int64_t *rec_idx, float *state, float *rec, void *stream) {
  g_err.clear();
  int rc = check_params(p, true);
  if (rc) return rc;
  if (p->snap_mode != MW_SNAP_NONE)
    return fail(MW_ERR_ARG, "the scratch-free forward keeps no snapshots: snap_mode must be NONE");
  if ((rc = check_ptr(ca, "ca")) || (rc = check_ptr(cb, "cb")) || (rc = check_ptr(cpml, "cpml")) ||
      (rc = check_ptr(state, "state")))
    return rc;
  if (!cq) return fail(MW_ERR_ARG, "cq is NULL");
  if (!p->cq_is_scalar && (rc = check_ptr(cq, "cq"))) return rc;
  if (p->n_src > 0 && (!f || !src_idx)) return fail(MW_ERR_ARG, "sources need f and src_idx");
  if (p->n_rec > 0 && rec && !rec_idx) return fail(MW_ERR_ARG, "receivers need rec_idx");

  // layout inside the built-in scratch; reject what does not fit
  const Bands bd = bands(p);
  Layout L{};
  L.flags = 0;
  L.tab_src = 256;
  L.tab_rec = L.tab_src + entry_table_bytes(p->n_shots, p->n_src, p->ny);
  L.bandtab = L.tab_rec + entry_table_bytes(p->n_shots, p->n_rec, p->ny);
  L.state_bytes = state_floats(p) * sizeof(float);
  const size_t off_state =
      L.bandtab + align256(sizeof(float) * (size_t)BandTab{bd.Wx, bd.Wz}.floats() + 16);
  const size_t need = off_state + align256(L.state_bytes);
  if (need > MW_NOALLOC_SCRATCH_BYTES)
    return fail(MW_ERR_WORKSPACE,
                "this problem needs %zu bytes of scratch but the built-in scratch holds %zu; "
                "use mw_tm_forward with a caller-provided workspace",
                need, (size_t)MW_NOALLOC_SCRATCH_BYTES);
  char *ws = nullptr;
  MW_TRY(noalloc_scratch(&ws));
  cudaStream_t st = (cudaStream_t)stream;
  int *flags = (int *)(ws + L.flags);
  // the array keeps the previous call's contents: clear the status words
  // (the band table, source / receiver tables and state buffer are fully
  // rewritten below)
  MW_CUDA(cudaMemsetAsync(ws, 0, 256, st));

  float *bufA = state;
  float *bufB = (float *)(ws + off_state);
  if (p->nt > 0) {
    const Launch lc = plan(p, kPlanFwd);
    StepArgs a = step_args(p, lc, ca, cb, cq, flags, ws, L);
    set_layout(a, p, false);
    MW_TRY(stencil_prologue(p, cpml, ws, L, st));
    FwdMaps mA, mB;
    MW_TRY(fwd_maps(p, fields_at(p, bufA), ca, cb, cq, &mA));
    MW_TRY(fwd_maps(p, fields_at(p, bufB), ca, cb, cq, &mB));
    const int64_t numel = (int64_t)p->ny * p->nx;
    const Tables tb = tables_at(p, ws, L);
    MW_TRY(build_table(p, src_idx, p->n_src, ws, L.tab_src, flags, nullptr, st));
    if (rec) MW_TRY(build_table(p, rec_idx, p->n_rec, ws, L.tab_rec, flags, rec, st));
    a.ea = tb.src;
    if (rec) a.eb = tb.rec;
    float *cur = bufA, *nxt = bufB;
    for (int t = 0; t < p->nt; ++t) {
      a.in = fields_at(p, cur);
      a.out = fields_at(p, nxt);
      a.ctr_slot = t & 1;
      a.vals_t = f ? f + (int64_t)t * p->n_shots * p->n_src : nullptr;
      a.out_t = rec ? rec + (int64_t)t * p->n_shots * p->n_rec : nullptr;
      MW_CUDA(launch_forward(cur == bufA ? mA : mB, a, p->order, kStoreNone, kStoreNone,
                             p->model_batched != 0, !p->cq_is_scalar, lc.grid, st));
      std::swap(cur, nxt);
    }
    if (cur != bufA)
      MW_CUDA(cudaMemcpyAsync(bufA, cur, L.state_bytes, cudaMemcpyDeviceToDevice, st));
    if (p->check_finite)
      MW_CUDA(launch_check_finite(bufA, 3 * (int64_t)p->n_shots * numel, flags, st));
  }
  // wait for this call's work and report its device status
  MW_CUDA(cudaStreamSynchronize(st));
  int h[3] = {0, 0, 0};
  MW_CUDA(cudaMemcpy(h, ws, sizeof h, cudaMemcpyDeviceToHost));
  if (h[kFlagTimeout]) return fail(MW_ERR_TIMEOUT, "a stencil kernel timed out waiting for its copies");
  if (h[kFlagBadIndex]) return fail(MW_ERR_ARG, "a source or receiver index was out of range");
  if (h[kFlagNonFinite]) return fail(MW_ERR_NONFINITE, "non-finite value in the final state");
  return MW_OK;
}

}  // extern "C"
