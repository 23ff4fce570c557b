// Small tools built on the stencil kernels' device primitives: the snapshot
// storage encoder (the forward's own store conversion, for bit-exact tests)
// and the bounded-wait self-test of the failure detection.
#include "mw_device.cuh"
#include "mw_internal.cuh"

namespace mw {
namespace {
using namespace dev;

// A stage wait that nothing completes: one expected-byte count that no copy
// ever delivers.  Exercises the bounded wait every stencil kernel uses and
// the timeout report, without a fault and with no copy in flight.
__global__ void k_wait_selftest(int *flags) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(1) : "memory");
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) expect_tx_s(b, 16);
  __syncwarp();
  if (!mbar_wait_s(b, 0) && threadIdx.x == 0) atomicOr(flags + kFlagTimeout, 1);
}

// Snapshot encoding of n floats with the forward's store conversion.
template <int STORE>
__global__ void k_snap_encode(const float *__restrict__ x, void *out, int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x)
    snap_store<STORE>(out, 4 * i, ld4(x + 4 * i));
}

}  // namespace

cudaError_t launch_wait_selftest(int *flags, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(flags);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_snap_encode(int store, int64_t n, const float *x, void *out, cudaStream_t st) {
  const int64_t n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  const int grid = (int)(n4 < 148 * 32 * 256 ? (n4 + 255) / 256 : 148 * 32);
  if (store == kStoreBF16)
    k_snap_encode<kStoreBF16><<<grid, 256, 0, st>>>(x, out, n4);
  else if (store == kStoreFP8)
    k_snap_encode<kStoreFP8><<<grid, 256, 0, st>>>(x, out, n4);
  else
    return cudaErrorInvalidValue;
  count_launches(1);
  return cudaGetLastError();
}


}  // namespace mw
