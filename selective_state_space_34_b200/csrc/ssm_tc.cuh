// ssm_tc.cuh -- the tcgen05 tensor-core plumbing shared by the SSD kernels on sm_100a: shared-memory
// operand descriptors, single-thread MMA issue and commit, mbarriers with bounded waits, the
// tcgen05 / async-proxy fences, row loads from tensor memory, and the byte offsets of the
// no-swizzle canonical operand layouts (8 x 16-byte core matrices).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ssm_tmem.cuh"
#include "ssm_umma.cuh"

namespace ssm {

// Shared-memory matrix descriptor of a no-swizzle operand tile (bit layout in ssm_umma.cuh).
__device__ __forceinline__ uint64_t smem_desc(const void *p, uint32_t lbo, uint32_t sbo) {
  return umma_smem_desc_bits(static_cast<uint32_t>(__cvta_generic_to_shared(p)), lbo, sbo);
}
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, int a_mn_major, int b_mn_major) {
  return umma_instr_desc_bf16_f32(M, N, a_mn_major, b_mn_major);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(a)
               : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");  // visible to the async proxy
}

// Wait for the phase with parity `phase`; gives up after max_polls polls. Returns false on timeout.
// A failed poll suspends the thread for a hardware-chosen time (about 4 us on B200, measured by
// the wait self-test), so the default bound of 2^18 polls gives up after about one second; a
// product completes in microseconds. The result is made warp-uniform by the caller before any
// warp-collective tcgen05 access.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t phase, int max_polls = 1 << 18) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
  for (int i = 0; i < max_polls; i++) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(phase)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t addr, float *v) {
  float a[16], b[16];
  tmem_ld2<16>(addr, a, addr + 16, b);
#pragma unroll
  for (int i = 0; i < 16; i++) {
    v[i] = a[i];
    v[16 + i] = b[i];
  }
}

// Byte offset of element (mn, k) in a no-swizzle operand tile with R rows along M/N; core
// matrices are laid out K-group-major: group (i, j) at (j * R/8 + i) * 128, so sbo = 128 and
// lbo = R / 8 * 128. K-major rows hold 8 consecutive k; MN-major rows hold 8 consecutive mn.
__device__ __forceinline__ uint32_t kmaj_off(int R, int mn, int k) {
  return (uint32_t)(((k >> 3) * (R >> 3) + (mn >> 3)) * 128 + (mn & 7) * 16 + (k & 7) * 2);
}
__device__ __forceinline__ uint32_t mnmaj_off(int R, int mn, int k) {
  return (uint32_t)(((k >> 3) * (R >> 3) + (mn >> 3)) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ---- TMA (cp.async.bulk.tensor) loads counted on an mbarrier ----------------------------------

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}\n" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(bar))),
               "r"(bytes)
               : "memory");
}

// One 3-D tile load (no multicast) into this CTA's shared memory; completion is counted on bar.
// The innermost coordinate times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *map, int c0, int c1, int c2, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0),
      "r"(c1), "r"(c2), "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
      : "memory");
}

}  // namespace ssm
