// ssm_common.cuh -- device helpers shared by the selective-scan kernels (sm_100a).
//
// Two math paths:
//  * fast (bf16 inputs): hardware approximations ex2.approx / lg2.approx / rcp.approx. The
//    relative error of ex2.approx is about 2^-22, far inside the bf16-input tolerance.
//  * precise (fp32 inputs): the CUDA math library's expf / expm1f / log1pf and IEEE division.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// ---- element conversion --------------------------------------------------------------------

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ---- hardware approximations (single MUFU instruction each) --------------------------------

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// ---- activations ---------------------------------------------------------------------------

// logistic sigmoid
template <bool PRECISE> __device__ __forceinline__ float sigmoid(float v) {
  if (PRECISE) return 1.0f / (1.0f + expf(-v));
  return rcp_approx(1.0f + ex2_approx(-v * kLog2e));
}

// softplus(v) = log1p(e^{-|v|}) + max(v, 0), the overflow-free form. The fast path evaluates
// log1p(e) for e = e^{-|v|} in (0, 1] with lg2(1 + e), except for small e where 1 + e would drop
// e's low bits; there the Taylor series e - e^2/2 + e^3/3 (truncation below e^4/4 < 2^-24 e for
// e < 2^-6) keeps the full relative precision.
template <bool PRECISE> __device__ __forceinline__ float softplus(float v) {
  if (PRECISE) return log1pf(expf(-fabsf(v))) + fmaxf(v, 0.0f);
  const float e = ex2_approx(-fabsf(v) * kLog2e);
  const float series = e * fmaf(e, fmaf(e, 1.0f / 3.0f, -0.5f), 1.0f);
  const float viaLog = lg2_approx(1.0f + e) * kLn2;
  return (e < 0.015625f ? series : viaLog) + fmaxf(v, 0.0f);
}

// ---- 16-byte async copies (Ampere-style cp.async, still the lightest way to stream small
//      per-CTA tiles into shared memory on sm_100a) --------------------------------------------

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src));
}
// Same, asking L2 to fetch the surrounding 256 bytes: rows are streamed in short slices per stage,
// so the next stages of the same row then hit in L2 instead of reopening a DRAM page.
__device__ __forceinline__ void cp_async16_l2pf(void *smem_dst, const void *gmem_src) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src));
}
// 16-byte global load with the same L2 256-byte prefetch hint (read-only data).
__device__ __forceinline__ uint4 ld_global_l2pf(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace ssm
