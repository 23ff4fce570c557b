// Small kernels of the mw_tm library: the sorted source / receiver tables the
// stencil kernels inject and sample from, model coefficients, CPML profiles,
// shot reduction, epsilon / sigma chain rule, residual and misfit, non-finite
// scan, the summation-by-parts end terms.
//
// Method: page "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu" -- add_sources_ey,
// record_receivers_ey, add_adjoint_sources_ey, record_adjoint_at_sources,
// combine_grad and convert_grad_ca_cb_to_eps_sigma; the model-coefficient
// forms are the ones whose derivatives that last kernel uses.
#include <cooperative_groups.h>
#include <math.h>

#include "mw_internal.cuh"

namespace mw {
namespace {

constexpr double kEps0 = 8.8541878128e-12;  // F/m (the page's EP0)
constexpr double kMu0 = 1.25663706212e-6;   // H/m (CODATA 2018)

// Entry table of one shot's index list v[0..n) (one block per shot; the
// EntrySet layout).  Pass 1 ranks every valid entry by (cell, k) and places
// it; pass 2 marks the runs of equal cells and the distinct rows.  Invalid
// entries (-1, or out of range, which also sets the bad-index flag) get no
// place; with `out` their outputs out[t][s][k] are zeroed for every step.
// O(n^2 / blockDim) per shot, once per call.
__global__ void k_entry_table(const int64_t *__restrict__ idx, int n, int ny, int nx,
                              int64_t numel, int4 *__restrict__ ent_all, int *__restrict__ arow_all,
                              int *__restrict__ abeg_all, int2 *__restrict__ rcur_all,
                              int *__restrict__ flags, float *__restrict__ out, int nt, int S) {
  const int s = blockIdx.x;
  const int64_t *v = idx + (int64_t)s * n;
  int4 *ent = ent_all + (int64_t)s * n;
  int *arow = arow_all + (int64_t)s * (n + 1);
  int *abeg = abeg_all + (int64_t)s * (n + 1);
  __shared__ int s_nv, s_nact;
  if (threadIdx.x == 0) s_nv = 0;
  __syncthreads();
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const int64_t c = v[k];
    const bool ok = c >= 0 && c < numel;
    if (!ok) {
      if (c != -1 && flags) atomicOr(flags + kFlagBadIndex, 1);
      if (out)
        for (int t = 0; t < nt; ++t) out[((int64_t)t * S + s) * n + k] = 0.f;
      continue;
    }
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const int64_t cj = v[j];
      if (cj >= 0 && cj < numel && (cj < c || (cj == c && j < k))) ++rank;
    }
    ent[rank] = make_int4((int)(c / nx), (int)(c % nx), k, 0);
    atomicAdd(&s_nv, 1);
  }
  __syncthreads();
  const int nv = s_nv;
  // runs of equal cells and the distinct rows; only the (row, column) half of
  // an entry is read here, only its run half is written
  const int2 *rc = reinterpret_cast<const int2 *>(ent);
  for (int j = threadIdx.x; j < nv; j += blockDim.x) {
    const int2 e = rc[2 * j];
    int len = 0;
    if (j == 0 || rc[2 * (j - 1)].x != e.x || rc[2 * (j - 1)].y != e.y) {
      len = 1;
      while (j + len < nv && rc[2 * (j + len)].x == e.x && rc[2 * (j + len)].y == e.y) ++len;
    }
    ent[j].w = len;
    if (j > 0 && rc[2 * (j - 1)].x == e.x) continue;
    int a = 0;  // the a-th row start: the number of row starts before j
    for (int i = 1; i <= j; ++i) a += rc[2 * i].x != rc[2 * (i - 1)].x;
    arow[a] = e.x;
    abeg[a] = j;
  }
  if (threadIdx.x == 0) {
    int na = 0;
    for (int j = 0; j < nv; ++j) na += (j == 0 || rc[2 * j].x != rc[2 * (j - 1)].x);
    s_nact = na;
  }
  __syncthreads();
  for (int a = s_nact + threadIdx.x; a <= n; a += blockDim.x) {
    arow[a] = 0x7fffffff;
    abeg[a] = nv;
  }
  __syncthreads();
  // per row: the first active row at or after it (binary search over arow)
  int2 *rcur = rcur_all + (int64_t)s * (ny + 1);
  for (int y = threadIdx.x; y <= ny; y += blockDim.x) {
    int lo = 0, hi = n;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (arow[mid] < y) lo = mid + 1;
      else hi = mid;
    }
    rcur[y] = make_int2(lo, arow[lo]);
  }
}

// Fix-ups of a whole E field [S][ny][nx] (one block per shot): add vals[s][k]
// at the entries of set `ea` (one thread per cell, duplicates added up in
// index order first), then read the field at the entries of set `eb` into
// out[s][k].  The stencil kernels make the same fix-ups row by row.
__global__ void k_fix_field(float *__restrict__ field, int64_t numel, int nx, EntrySet ea,
                            const float *__restrict__ vals, EntrySet eb, float *__restrict__ out) {
  const int s = blockIdx.x;
  float *e = field + (int64_t)s * numel;
  // programmatic dependent launch (no-ops without the launch attribute):
  // let the next stencil launch begin, then wait for the previous one
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (vals != nullptr && ea.n > 0) {
    const int nv = ea.abeg[(int64_t)s * (ea.n + 1) + ea.n];
    const int4 *en = ea.ent + (int64_t)s * ea.n;
    const float *vs = vals + (int64_t)s * ea.n;
    for (int j = threadIdx.x; j < nv; j += blockDim.x) {
      const int4 q = en[j];
      if (q.w == 0) continue;
      float v = vs[q.z];
      for (int u = 1; u < q.w; ++u) v += vs[en[j + u].z];
      e[(int64_t)q.x * nx + q.y] += v;
    }
  }
  __syncthreads();
  if (out != nullptr && eb.n > 0) {
    const int nv = eb.abeg[(int64_t)s * (eb.n + 1) + eb.n];
    const int4 *en = eb.ent + (int64_t)s * eb.n;
    for (int j = threadIdx.x; j < nv; j += blockDim.x) {
      const int4 q = en[j];
      out[(int64_t)s * eb.n + q.z] = e[(int64_t)q.x * nx + q.y];
    }
  }
}

// One thread per (shot, entry): the end-term sums in the adjoint's order.
__global__ void k_sbp_sums(int nt, int S, const float *__restrict__ res,
                           const float *__restrict__ rec, int n_rec, float *__restrict__ acc_rec,
                           const float *__restrict__ f, const float *__restrict__ lam, int n_src,
                           float *__restrict__ acc_src) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int nr = res ? S * n_rec : 0, ns = f ? S * n_src : 0;
  if (i < nr) {
    float acc = 0.f;
    for (int t = nt - 1; t >= 0; --t) acc += res[(int64_t)t * nr + i] * rec[(int64_t)t * nr + i];
    acc_rec[i] = acc;
  } else if (i < nr + ns) {
    const int j = i - nr;
    float acc = 0.f;
    for (int t = nt - 1; t >= 0; --t) acc += f[(int64_t)t * ns + j] * lam[(int64_t)t * ns + j];
    acc_src[j] = acc;
  }
}

__global__ void k_sbp_init(float *__restrict__ P, const float *__restrict__ lam,
                           const float *__restrict__ e, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    P[i] = lam[i] * e[i];
}

// One thread per shot, so that duplicate cells add in index order.
__global__ void k_sbp_scatter(float *__restrict__ P, int64_t numel, int S,
                              const int64_t *__restrict__ rec_idx,
                              const float *__restrict__ acc_rec, int n_rec,
                              const int64_t *__restrict__ src_idx,
                              const float *__restrict__ acc_src, int n_src) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  float *p = P + (int64_t)s * numel;
  for (int k = 0; k < n_rec; ++k) {
    const int64_t i = rec_idx[(int64_t)s * n_rec + k];
    if (i >= 0 && i < numel) p[i] += acc_rec[(int64_t)s * n_rec + k];
  }
  for (int k = 0; k < n_src; ++k) {
    const int64_t i = src_idx[(int64_t)s * n_src + k];
    if (i >= 0 && i < numel) p[i] -= acc_src[(int64_t)s * n_src + k];
  }
}

__global__ void k_sbp_finish(const float *__restrict__ P, const float *__restrict__ cb,
                             float *__restrict__ gcb, int S, int ny, int nx, int batched,
                             int mask_pml) {
  const int64_t numel = (int64_t)ny * nx, n = (int64_t)S * numel;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t s = i / numel, c = i - s * numel;
    const int y = (int)(c / nx), x = (int)(c - (int64_t)y * nx);
    if (mask_pml > 0 && (y < mask_pml || y >= ny - mask_pml || x < mask_pml || x >= nx - mask_pml))
      continue;
    gcb[i] += P[i] / cb[batched ? i : c];
  }
}

__global__ void k_check_finite(const float *__restrict__ x, int64_t n, int *__restrict__ flags) {
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    bad |= !isfinite(x[i]);
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags + kFlagNonFinite, 1);
}

__global__ void k_model(int64_t n, const float *__restrict__ eps_r, const float *__restrict__ sigma,
                        const float *__restrict__ mu_r, double dt, float *__restrict__ ca,
                        float *__restrict__ cb, float *__restrict__ cq, int cq_full) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double eps = kEps0 * (double)eps_r[i];
    const double s = sigma ? (double)sigma[i] : 0.0;
    const double h = 0.5 * s * dt / eps;
    ca[i] = (float)((1.0 - h) / (1.0 + h));
    cb[i] = (float)(dt / (eps + 0.5 * s * dt));
    if (cq_full) cq[i] = (float)(dt / (kMu0 * (mu_r ? (double)mu_r[i] : 1.0)));
  }
  if (!cq_full && blockIdx.x == 0 && threadIdx.x == 0) cq[0] = (float)(dt / kMu0);
}

// CPML profile entry: 12 vectors (6 along y of length ny, 6 along x of nx).
__global__ void k_cpml(int ny, int nx, int n_pml, double dy, double dx, double dt, double vmax,
                       double f0, double R, float *__restrict__ out) {
  const int64_t total = 6LL * (ny + nx);
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const bool is_y = t < 6LL * ny;
    const int n = is_y ? ny : nx;
    const int64_t loc = is_y ? t : t - 6LL * ny;
    const int which = (int)(loc / n);  // 0 a, 1 ah, 2 b, 3 bh, 4 k, 5 kh
    const int i = (int)(loc % n);
    const bool half = (which & 1) != 0;
    const double h = is_y ? dy : dx;
    double val;
    if (which >= 4) {
      val = 1.0;
    } else {
      const double pos = i + (half ? 0.5 : 0.0);
      double u = 0.0;
      if (n_pml > 0) {
        const double left = (double)n_pml - pos;
        const double right = pos - (double)(n - 1 - n_pml);
        if (left > 0.0) u = left;
        if (right > 0.0) u = right;
      }
      if (u <= 0.0) {
        val = 0.0;
      } else {
        double s = u / (double)n_pml;
        if (s > 1.0) s = 1.0;
        const double L = n_pml * h;
        const double dmax = -3.0 * vmax * log(R) / (2.0 * L);
        const double d = dmax * s * s;
        const double alpha = M_PI * f0 * (1.0 - s);
        const double b = exp(-(d + alpha) * dt);
        val = (which >= 2) ? b : (d > 0.0 ? d * (b - 1.0) / (d + alpha) : 0.0);
      }
    }
    out[t] = (float)val;
  }
}

// Band coefficient table from the 6*(ny+nx) profile floats (see BandTab).
__global__ void k_band_table(const float *__restrict__ cpml, int ny, int nx, int Wx, int Wz,
                             float *__restrict__ out) {
  const BandTab bt{Wx, Wz};
  const float *py = cpml, *px = cpml + 6 * (int64_t)ny;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < 6 * 2 * Wx + 6 * 2 * Wz;
       t += gridDim.x * blockDim.x) {
    if (t < 12 * Wx) {
      const int k = t / (2 * Wx), j = t % (2 * Wx);
      const int c = j < Wx ? j : nx - 2 * Wx + j;
      // profile vector order: a, ah, b, bh, k, kh; table order a, b, 1/k, ah, bh, 1/kh
      const int src = (k % 3) * 2 + (k >= 3 ? 1 : 0);
      const float v = px[(int64_t)src * nx + c];
      out[bt.x(k) + j] = (k % 3 == 2) ? 1.0f / v : v;
    } else {
      const int u = t - 12 * Wx;
      const int k = u / (2 * Wz), j = u % (2 * Wz);
      const int r = j < Wz ? j : ny - 2 * Wz + j;
      const int src = (k % 3) * 2 + (k >= 3 ? 1 : 0);
      const float v = py[(int64_t)src * ny + r];
      out[bt.z(k) + j] = (k % 3 == 2) ? 1.0f / v : v;
    }
  }
}

__global__ void k_combine(const float *__restrict__ gs, float *__restrict__ g, int S, int64_t n,
                          int accumulate) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += gs[(int64_t)s * n + i];
    g[i] = accumulate ? g[i] + acc : acc;
  }
}

__global__ void k_eps_sigma(int64_t n, double dt, const float *__restrict__ ca,
                            const float *__restrict__ cb, const float *__restrict__ gca,
                            const float *__restrict__ gcb, float *__restrict__ ge,
                            float *__restrict__ gs) {
  const float inv_dt = (float)(1.0 / dt);
  const float eps0 = (float)kEps0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float a = ca[i], b = cb[i], b2 = b * b;
    const float dca_de = (1.f - a) * b * inv_dt, dcb_de = -b2 * inv_dt;
    const float dca_ds = -0.5f * (1.f + a) * b, dcb_ds = -0.5f * b2;
    if (ge) ge[i] = eps0 * (gca[i] * dca_de + gcb[i] * dcb_de);
    if (gs) gs[i] = gca[i] * dca_ds + gcb[i] * dcb_ds;
  }
}

__global__ void k_residual(int64_t n, const float *__restrict__ d, const float *__restrict__ o,
                           float *__restrict__ res) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    res[i] = d[i] - o[i];
}

// Misfit 1/2 sum res^2 in one block: fixed per-thread strides and a fixed
// tree, so the value does not depend on scheduling.
// J = 1/2 sum res[i]^2 in double, in an order fixed whatever the timing,
// by one cluster of kMisfitBlocks blocks: block b sums its chunk [b C,
// b C + C) (thread t the elements t, t + 1024, ... of it, then a fixed
// tree), and block 0 adds the blocks' sums in rank order through the
// cluster's distributed shared memory.
constexpr int kMisfitBlocks = 8;
__global__ void __cluster_dims__(kMisfitBlocks, 1, 1) __launch_bounds__(1024)
    k_misfit(int64_t n, const float *__restrict__ res, double *__restrict__ J) {
  __shared__ double part[1024];
  cooperative_groups::cluster_group cl = cooperative_groups::this_cluster();
  const int b = (int)cl.block_rank();
  const int64_t C = (n + kMisfitBlocks - 1) / kMisfitBlocks;
  const int64_t lo = (int64_t)b * C, hi = lo + C < n ? lo + C : n;
  double acc = 0.0;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    const double r = res[i];
    acc += r * r;
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  cl.sync();  // every block's sum is in its part[0]
  if (b == 0 && threadIdx.x == 0) {
    double sum = 0.0;
    for (int k = 0; k < kMisfitBlocks; ++k) sum += *cl.map_shared_rank(&part[0], k);
    *J = 0.5 * sum;
  }
  cl.sync();  // no block leaves while block 0 reads its sum
}

int grid_for(int64_t n, int block) {
  int64_t g = (n + block - 1) / block;
  if (g > 148 * 16) g = 148 * 16;
  return (int)(g > 0 ? g : 1);
}

}  // namespace

size_t entry_table_bytes(int S, int n, int ny) {
  if (n <= 0) return 0;
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return a256((size_t)S * n * sizeof(int4)) + 2 * a256((size_t)S * (n + 1) * sizeof(int)) +
         a256((size_t)S * (ny + 1) * sizeof(int2));
}

EntrySet entry_set_at(void *base, int S, int n, int ny) {
  EntrySet es{nullptr, nullptr, nullptr, nullptr, 0, ny};
  if (n <= 0 || base == nullptr) return es;
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char *b = (char *)base;
  const size_t e = a256((size_t)S * n * sizeof(int4));
  const size_t r = a256((size_t)S * (n + 1) * sizeof(int));
  es.ent = (const int4 *)b;
  es.arow = (const int *)(b + e);
  es.abeg = (const int *)(b + e + r);
  es.rcur = (const int2 *)(b + e + 2 * r);
  es.n = n;
  return es;
}

cudaError_t launch_entry_table(const int64_t *idx, int S, int n, int ny, int nx, void *base,
                               int *flags, float *out, int nt, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const EntrySet es = entry_set_at(base, S, n, ny);
  k_entry_table<<<S, 256, 0, st>>>(idx, n, ny, nx, (int64_t)ny * nx, const_cast<int4 *>(es.ent),
                                   const_cast<int *>(es.arow), const_cast<int *>(es.abeg),
                                   const_cast<int2 *>(es.rcur), flags, out, nt, S);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_fix_field(float *field, int S, int ny, int nx, const EntrySet &ea,
                             const float *vals, const EntrySet &eb, float *out, cudaStream_t st) {
  if ((vals == nullptr || ea.n == 0) && (out == nullptr || eb.n == 0)) return cudaSuccess;
  const cudaError_t e = launch_dependent(k_fix_field, S, 128, 0, st, field, (int64_t)ny * nx, nx,
                                         ea, vals, eb, out);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_sbp_sums(int nt, int S, const float *res, const float *rec, int n_rec,
                            float *acc_rec, const float *f, const float *lam, int n_src,
                            float *acc_src, cudaStream_t st) {
  const int n = (res ? S * n_rec : 0) + (f ? S * n_src : 0);
  if (n <= 0) return cudaSuccess;
  k_sbp_sums<<<(n + 127) / 128, 128, 0, st>>>(nt, S, res, rec, n_rec, acc_rec, f, lam, n_src,
                                              acc_src);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_sbp_init(float *P, const float *lam, const float *e, int64_t n,
                            cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  k_sbp_init<<<grid_for(n, 256), 256, 0, st>>>(P, lam, e, n);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_sbp_scatter(float *P, int64_t numel, int S, const int64_t *rec_idx,
                               const float *acc_rec, int n_rec, const int64_t *src_idx,
                               const float *acc_src, int n_src, cudaStream_t st) {
  if (S <= 0 || (n_rec == 0 && n_src == 0)) return cudaSuccess;
  k_sbp_scatter<<<(S + 63) / 64, 64, 0, st>>>(P, numel, S, rec_idx, acc_rec, n_rec, src_idx,
                                                acc_src, n_src);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_sbp_finish(const float *P, const float *cb, float *gcb, int S, int ny, int nx,
                              int batched, int mask_pml, cudaStream_t st) {
  const int64_t n = (int64_t)S * ny * nx;
  if (n <= 0) return cudaSuccess;
  k_sbp_finish<<<grid_for(n, 256), 256, 0, st>>>(P, cb, gcb, S, ny, nx, batched, mask_pml);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_check_finite(const float *x, int64_t n, int *flags, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  k_check_finite<<<grid_for(n, 256), 256, 0, st>>>(x, n, flags);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_model(int64_t n, const float *eps_r, const float *sigma, const float *mu_r,
                         double dt, float *ca, float *cb, float *cq, int cq_full,
                         cudaStream_t st) {
  k_model<<<grid_for(n, 256), 256, 0, st>>>(n, eps_r, sigma, mu_r, dt, ca, cb, cq, cq_full);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_cpml(int ny, int nx, int n_pml, double dy, double dx, double dt, double vmax,
                        double f0, double R, float *out, cudaStream_t st) {
  k_cpml<<<grid_for(6LL * (ny + nx), 256), 256, 0, st>>>(ny, nx, n_pml, dy, dx, dt, vmax, f0, R,
                                                          out);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_band_table(const float *cpml, int ny, int nx, int Wx, int Wz, float *out,
                              cudaStream_t st) {
  if (Wx == 0 && Wz == 0) return cudaSuccess;
  k_band_table<<<grid_for(12LL * (Wx + Wz), 256), 256, 0, st>>>(cpml, ny, nx, Wx, Wz, out);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float *gs, float *g, int S, int64_t n, int accumulate,
                           cudaStream_t st) {
  k_combine<<<grid_for(n, 256), 256, 0, st>>>(gs, g, S, n, accumulate);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_eps_sigma(int64_t n, double dt, const float *ca, const float *cb,
                             const float *gca, const float *gcb, float *ge, float *gs,
                             cudaStream_t st) {
  k_eps_sigma<<<grid_for(n, 256), 256, 0, st>>>(n, dt, ca, cb, gca, gcb, ge, gs);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_residual(int64_t n, const float *d, const float *o, float *res, double *J,
                            cudaStream_t st) {
  k_residual<<<grid_for(n, 256), 256, 0, st>>>(n, d, o, res);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || J == nullptr) return e;
  k_misfit<<<kMisfitBlocks, 1024, 0, st>>>(n, res, J);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace mw
