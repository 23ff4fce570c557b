// Small kernels of the mw_tm library: source injection / receiver sampling
// and their transposes, model coefficients, CPML profiles, shot reduction,
// epsilon / sigma chain rule, residual and misfit, non-finite scan.
//
// Method: page "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu" -- add_sources_ey,
// record_receivers_ey, add_adjoint_sources_ey, record_adjoint_at_sources,
// combine_grad and convert_grad_ca_cb_to_eps_sigma; the model-coefficient
// forms are the ones whose derivatives that last kernel uses.
#include <math.h>

#include "mw_internal.cuh"

namespace mw {
namespace {

constexpr double kEps0 = 8.8541878128e-12;  // F/m (the page's EP0)
constexpr double kMu0 = 1.25663706212e-6;   // H/m (CODATA 2018)

// One block per shot.  Thread 0 applies the sources in index order (so
// duplicate cells add up deterministically), then the block samples the
// receivers.  Out-of-range indices set a status flag and are skipped.
__global__ void k_src_rec(float *__restrict__ ey, int64_t numel, const float *__restrict__ f_t,
                          const int64_t *__restrict__ src, int ns, const int64_t *__restrict__ rec,
                          int nr, float *__restrict__ r_t, int *__restrict__ flags) {
  const int s = blockIdx.x;
  float *e = ey + (int64_t)s * numel;
  if (threadIdx.x == 0 && f_t != nullptr) {
    for (int k = 0; k < ns; ++k) {
      const int64_t i = src[(int64_t)s * ns + k];
      if (i >= 0 && i < numel) {
        e[i] += f_t[(int64_t)s * ns + k];
      } else if (i != -1 && flags) {
        atomicOr(flags + kFlagBadIndex, 1);
      }
    }
  }
  __syncthreads();
  if (r_t != nullptr) {
    for (int k = threadIdx.x; k < nr; k += blockDim.x) {
      const int64_t i = rec[(int64_t)s * nr + k];
      const bool ok = i >= 0 && i < numel;
      if (!ok && i != -1 && flags) atomicOr(flags + kFlagBadIndex, 1);
      r_t[(int64_t)s * nr + k] = ok ? e[i] : 0.f;
    }
  }
}

// Transpose: lambda_E[rec] += res[t] (thread 0, index order), then
// grad_f[t] = lambda_E[src].
__global__ void k_adj_src_rec(float *__restrict__ lam, int64_t numel,
                              const float *__restrict__ res_t, const int64_t *__restrict__ rec,
                              int nr, const int64_t *__restrict__ src, int ns,
                              float *__restrict__ gf_t, int *__restrict__ flags) {
  const int s = blockIdx.x;
  float *e = lam + (int64_t)s * numel;
  if (threadIdx.x == 0 && res_t != nullptr) {
    for (int k = 0; k < nr; ++k) {
      const int64_t i = rec[(int64_t)s * nr + k];
      if (i >= 0 && i < numel) {
        e[i] += res_t[(int64_t)s * nr + k];
      } else if (i != -1 && flags) {
        atomicOr(flags + kFlagBadIndex, 1);
      }
    }
  }
  __syncthreads();
  if (gf_t != nullptr) {
    for (int k = threadIdx.x; k < ns; k += blockDim.x) {
      const int64_t i = src[(int64_t)s * ns + k];
      const bool ok = i >= 0 && i < numel;
      gf_t[(int64_t)s * ns + k] = ok ? e[i] : 0.f;
    }
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
__global__ void k_misfit(int64_t n, const float *__restrict__ res, double *__restrict__ J) {
  __shared__ double part[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const double r = res[i];
    acc += r * r;
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *J = 0.5 * part[0];
}

int grid_for(int64_t n, int block) {
  int64_t g = (n + block - 1) / block;
  if (g > 148 * 16) g = 148 * 16;
  return (int)(g > 0 ? g : 1);
}

}  // namespace

cudaError_t launch_src_rec(float *ey, int64_t numel, int S, const float *f_t, const int64_t *src,
                           int ns, const int64_t *rec, int nr, float *r_t, int *flags,
                           cudaStream_t st) {
  if ((ns == 0 || f_t == nullptr) && (nr == 0 || r_t == nullptr)) return cudaSuccess;
  k_src_rec<<<S, 128, 0, st>>>(ey, numel, ns > 0 ? f_t : nullptr, src, ns, rec, nr,
                              nr > 0 ? r_t : nullptr, flags);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_adj_src_rec(float *lam, int64_t numel, int S, const float *res_t,
                               const int64_t *rec, int nr, const int64_t *src, int ns,
                               float *gf_t, int *flags, cudaStream_t st) {
  if ((nr == 0 || res_t == nullptr) && (ns == 0 || gf_t == nullptr)) return cudaSuccess;
  k_adj_src_rec<<<S, 128, 0, st>>>(lam, numel, nr > 0 ? res_t : nullptr, rec, nr, src, ns,
                                  ns > 0 ? gf_t : nullptr, flags);
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
  k_misfit<<<1, 1024, 0, st>>>(n, res, J);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace mw
