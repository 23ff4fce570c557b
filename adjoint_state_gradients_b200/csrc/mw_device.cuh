// Device primitives shared by the stencil kernels and the small tools:
// float4 values, 32-bit shared-window loads and stores, mbarrier waits with
// a poll limit, TMA tile loads, programmatic-dependent-launch controls and
// the snapshot storage conversions.  Everything here is inline PTX or CUDA
// intrinsics; no arithmetic of the method.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "mw_internal.cuh"

namespace mw {
namespace dev {

constexpr uint32_t kWaitPolls = 1u << 22;  // ~0.5 s of polling, then give up
constexpr unsigned kFull = 0xffffffffu;

struct F4 {
  float v[4];
};

__device__ __forceinline__ F4 zero4() { return F4{{0.f, 0.f, 0.f, 0.f}}; }
__device__ __forceinline__ F4 ld4(const float *p) {
  float4 t = __ldg(reinterpret_cast<const float4 *>(p));
  return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ F4 splat4(float x) { return F4{{x, x, x, x}}; }
__device__ __forceinline__ void st4(float *p, const F4 &a) {
  *reinterpret_cast<float4 *>(p) = make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
}

// ---- TMA / mbarrier primitives (PTX) -------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Programmatic dependent launch: let the next kernel in the stream start
// launching (its blocks then wait in grid_dep_wait), and wait for the
// previous kernel's completion and memory before touching its results.
// Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Snapshot row store (4 consecutive cells at element `elem` of `base`):
// float32, bfloat16 (nearest even) or FP8 E4M3 (nearest even, saturating to
// the largest finite value, no scaling: the maxwell.cu page's fp8 storage).
template <int STORE>
__device__ __forceinline__ void snap_store(void *base, int64_t elem, const F4 &v) {
  if constexpr (STORE == kStoreF32 || STORE == kStoreEy) {
    st4(reinterpret_cast<float *>(base) + elem, v);
  } else if constexpr (STORE == kStoreBF16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.v[0], v.v[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.v[2], v.v[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&lo);
    pk.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(base) + elem) = pk;
  } else if constexpr (STORE == kStoreFP8) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v.v[0], v.v[1]), __NV_SATFINITE,
                                                 __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v.v[2], v.v[3]), __NV_SATFINITE,
                                                 __NV_E4M3);
    *reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(base) + elem) = lo | (hi << 16);
  }
}

// Shared-memory access by 32-bit shared-window address.
__device__ __forceinline__ F4 lds4s(uint32_t addr) {
  F4 r;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.v[0]), "=f"(r.v[1]), "=f"(r.v[2]), "=f"(r.v[3])
               : "r"(addr)
               : "memory");
  return r;
}
__device__ __forceinline__ void sts4s(uint32_t addr, const F4 &v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.v[0]), "f"(v.v[1]),
               "f"(v.v[2]), "f"(v.v[3])
               : "memory");
}
__device__ __forceinline__ void win12s(uint32_t addr, float w[12]) {
  const F4 a = lds4s(addr), b = lds4s(addr + 16), c = lds4s(addr + 32);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    w[q] = a.v[q];
    w[q + 4] = b.v[q];
    w[q + 8] = c.v[q];
  }
}
__device__ __forceinline__ void expect_tx_s(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test_s(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded, warp-uniform wait (all 32 lanes poll and vote); false after the
// poll limit.
__device__ __forceinline__ bool mbar_wait_s(uint32_t bar, uint32_t parity) {
  for (uint32_t k = 0; k < kWaitPolls; ++k) {
    if (__all_sync(kFull, mbar_test_s(bar, parity))) return true;
    if (k >= 32) __nanosleep(100);
  }
  return false;
}
__device__ __forceinline__ void tma3s(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                      uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma4s(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                      int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma5s(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                      int c3, int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(bar)
      : "memory");
}
// Staged snapshot float4 (4 cells) at byte address addr: float32, bf16 or
// FP8 E4M3 (SNAP = kStoreF32 or kStoreEy / kStoreBF16 / kStoreFP8).
template <int SNAP>
__device__ __forceinline__ F4 snap_lds_s(uint32_t addr) {
  if constexpr (SNAP == kStoreF32 || SNAP == kStoreEy) {
    return lds4s(addr);
  } else if constexpr (SNAP == kStoreBF16) {
    uint32_t lo, hi;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lo), "=r"(hi) : "r"(addr) : "memory");
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&lo);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&hi);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return F4{{fa.x, fa.y, fb.x, fb.y}};
  } else {
    uint32_t w;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(addr) : "memory");
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
    const float2 fa = __half22float2(__half2(lo)), fb = __half22float2(__half2(hi));
    return F4{{fa.x, fa.y, fb.x, fb.y}};
  }
}

// Predicated forms (no branch around them): the store or copy happens only
// where p holds; the address may be anything where it does not.
__device__ __forceinline__ void st4p(bool p, float *ptr, const F4 &v) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n"
      " @q st.global.v4.f32 [%1], {%2, %3, %4, %5};\n}\n" ::"r"((int)p),
      "l"(ptr), "f"(v.v[0]), "f"(v.v[1]), "f"(v.v[2]), "f"(v.v[3])
      : "memory");
}
__device__ __forceinline__ void sts4p(bool p, uint32_t addr, const F4 &v) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n"
      " @q st.shared.v4.f32 [%1], {%2, %3, %4, %5};\n}\n" ::"r"((int)p),
      "r"(addr), "f"(v.v[0]), "f"(v.v[1]), "f"(v.v[2]), "f"(v.v[3])
      : "memory");
}
// Snapshot row store (4 cells) where p holds.
template <int STORE>
__device__ __forceinline__ void snap_store_p(bool p, void *base, int64_t elem, const F4 &v) {
  if constexpr (STORE == kStoreF32 || STORE == kStoreEy) {
    st4p(p, reinterpret_cast<float *>(base) + elem, v);
  } else if constexpr (STORE == kStoreBF16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.v[0], v.v[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.v[2], v.v[3]);
    const uint32_t a = *reinterpret_cast<uint32_t *>(&lo), b = *reinterpret_cast<uint32_t *>(&hi);
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.global.v2.u32 [%1], {%2, %3};\n}\n" ::"r"(
            (int)p),
        "l"(reinterpret_cast<__nv_bfloat16 *>(base) + elem), "r"(a), "r"(b)
        : "memory");
  } else if constexpr (STORE == kStoreFP8) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v.v[0], v.v[1]), __NV_SATFINITE,
                                                 __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v.v[2], v.v[3]), __NV_SATFINITE,
                                                 __NV_E4M3);
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.global.u32 [%1], %2;\n}\n" ::"r"((int)p),
        "l"(reinterpret_cast<uint8_t *>(base) + elem), "r"(lo | (hi << 16))
        : "memory");
  }
}

}  // namespace dev
}  // namespace mw
