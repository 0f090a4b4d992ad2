// ssm_tmem.cuh -- tensor memory (TMEM) as per-thread scratch on sm_100a.
//
// Blackwell gives every SM 256 KB of tensor memory (128 lanes x 512 columns of 32 bits) next to
// the tensor cores. The scan kernels issue no MMA, so TMEM is free to hold a thread's per-block
// trajectory that would otherwise occupy registers: with the 32x32b access shape, warp w of a
// warpgroup reads and writes lanes 32w..32w+31, one lane per thread, so thread i of a 128-thread
// CTA owns lane i of the CTA's allocation and nothing is shared between threads.
//
// Protocol (PTX ISA, tcgen05 family): one warp allocates a power-of-two column count (>= 32) and
// publishes the address through shared memory; every thread reads it after a fenced barrier;
// tcgen05.st / tcgen05.ld move 32-bit registers to / from consecutive columns of the thread's
// lane and are asynchronous -- tcgen05.wait::st / tcgen05.wait::ld complete them; before exit the
// same warp frees the columns after a fenced barrier. All of these are warp-collective
// (.sync.aligned): callers keep them on warp-uniform control flow.
#pragma once

#include <cstdint>

namespace ssm {

// Allocate ncols columns by warp 0 (call from all threads); returns the CTA's base address.
__device__ __forceinline__ uint32_t tmem_alloc_cta(uint32_t *slot, uint32_t ncols) {
  if (threadIdx.x / 32 == 0) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(slot));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  return *reinterpret_cast<volatile uint32_t *>(slot);
}

// Free the CTA's columns (call from all threads, after the last TMEM access of every thread).
__device__ __forceinline__ void tmem_free_cta(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (threadIdx.x / 32 == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols));
  }
}

// This thread's lane of the allocation, column 0.
__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base) {
  return base + (static_cast<uint32_t>(threadIdx.x & ~31u) << 16);
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#define SSM_U(i) "r"(__float_as_uint(v[i]))

// Store NV consecutive columns of this thread's lane from v[0..NV).
template <int NV> __device__ __forceinline__ void tmem_st(uint32_t addr, const float *v);
template <> __device__ __forceinline__ void tmem_st<4>(uint32_t addr, const float *v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
               ::"r"(addr), SSM_U(0), SSM_U(1), SSM_U(2), SSM_U(3) : "memory");
}
template <> __device__ __forceinline__ void tmem_st<8>(uint32_t addr, const float *v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(addr), SSM_U(0), SSM_U(1), SSM_U(2), SSM_U(3), SSM_U(4), SSM_U(5), SSM_U(6),
               SSM_U(7) : "memory");
}
template <> __device__ __forceinline__ void tmem_st<16>(uint32_t addr, const float *v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, "
               "%9, %10, %11, %12, %13, %14, %15, %16};"
               ::"r"(addr), SSM_U(0), SSM_U(1), SSM_U(2), SSM_U(3), SSM_U(4), SSM_U(5), SSM_U(6),
               SSM_U(7), SSM_U(8), SSM_U(9), SSM_U(10), SSM_U(11), SSM_U(12), SSM_U(13), SSM_U(14),
               SSM_U(15) : "memory");
}
#undef SSM_U

// Load NV consecutive columns of this thread's lane from two places (a and b) and wait for both;
// the wait names the destination registers so no use of them can be scheduled before it.
#define SSM_O(x, i) "=r"(x[i])
#define SSM_W(x, i) "+r"(x[i])
template <int NV> __device__ __forceinline__ void tmem_ld2(uint32_t a, float *va, uint32_t b, float *vb);
template <> __device__ __forceinline__ void tmem_ld2<4>(uint32_t a, float *va, uint32_t b, float *vb) {
  uint32_t x[4], y[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : SSM_O(x, 0), SSM_O(x, 1), SSM_O(x, 2), SSM_O(x, 3) : "r"(a) : "memory");
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : SSM_O(y, 0), SSM_O(y, 1), SSM_O(y, 2), SSM_O(y, 3) : "r"(b) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : SSM_W(x, 0), SSM_W(x, 1), SSM_W(x, 2), SSM_W(x, 3), SSM_W(y, 0), SSM_W(y, 1),
                 SSM_W(y, 2), SSM_W(y, 3) :: "memory");
#pragma unroll
  for (int i = 0; i < 4; i++) {
    va[i] = __uint_as_float(x[i]);
    vb[i] = __uint_as_float(y[i]);
  }
}
template <> __device__ __forceinline__ void tmem_ld2<8>(uint32_t a, float *va, uint32_t b, float *vb) {
  uint32_t x[8], y[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : SSM_O(x, 0), SSM_O(x, 1), SSM_O(x, 2), SSM_O(x, 3), SSM_O(x, 4), SSM_O(x, 5),
                 SSM_O(x, 6), SSM_O(x, 7) : "r"(a) : "memory");
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : SSM_O(y, 0), SSM_O(y, 1), SSM_O(y, 2), SSM_O(y, 3), SSM_O(y, 4), SSM_O(y, 5),
                 SSM_O(y, 6), SSM_O(y, 7) : "r"(b) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : SSM_W(x, 0), SSM_W(x, 1), SSM_W(x, 2), SSM_W(x, 3), SSM_W(x, 4), SSM_W(x, 5),
                 SSM_W(x, 6), SSM_W(x, 7), SSM_W(y, 0), SSM_W(y, 1), SSM_W(y, 2), SSM_W(y, 3),
                 SSM_W(y, 4), SSM_W(y, 5), SSM_W(y, 6), SSM_W(y, 7) :: "memory");
#pragma unroll
  for (int i = 0; i < 8; i++) {
    va[i] = __uint_as_float(x[i]);
    vb[i] = __uint_as_float(y[i]);
  }
}
template <> __device__ __forceinline__ void tmem_ld2<16>(uint32_t a, float *va, uint32_t b, float *vb) {
  uint32_t x[16], y[16];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
               "%10, %11, %12, %13, %14, %15}, [%16];"
               : SSM_O(x, 0), SSM_O(x, 1), SSM_O(x, 2), SSM_O(x, 3), SSM_O(x, 4), SSM_O(x, 5),
                 SSM_O(x, 6), SSM_O(x, 7), SSM_O(x, 8), SSM_O(x, 9), SSM_O(x, 10), SSM_O(x, 11),
                 SSM_O(x, 12), SSM_O(x, 13), SSM_O(x, 14), SSM_O(x, 15) : "r"(a) : "memory");
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
               "%10, %11, %12, %13, %14, %15}, [%16];"
               : SSM_O(y, 0), SSM_O(y, 1), SSM_O(y, 2), SSM_O(y, 3), SSM_O(y, 4), SSM_O(y, 5),
                 SSM_O(y, 6), SSM_O(y, 7), SSM_O(y, 8), SSM_O(y, 9), SSM_O(y, 10), SSM_O(y, 11),
                 SSM_O(y, 12), SSM_O(y, 13), SSM_O(y, 14), SSM_O(y, 15) : "r"(b) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : SSM_W(x, 0), SSM_W(x, 1), SSM_W(x, 2), SSM_W(x, 3), SSM_W(x, 4), SSM_W(x, 5),
                 SSM_W(x, 6), SSM_W(x, 7), SSM_W(x, 8), SSM_W(x, 9), SSM_W(x, 10), SSM_W(x, 11),
                 SSM_W(x, 12), SSM_W(x, 13), SSM_W(x, 14), SSM_W(x, 15), SSM_W(y, 0), SSM_W(y, 1),
                 SSM_W(y, 2), SSM_W(y, 3), SSM_W(y, 4), SSM_W(y, 5), SSM_W(y, 6), SSM_W(y, 7),
                 SSM_W(y, 8), SSM_W(y, 9), SSM_W(y, 10), SSM_W(y, 11), SSM_W(y, 12), SSM_W(y, 13),
                 SSM_W(y, 14), SSM_W(y, 15) :: "memory");
#pragma unroll
  for (int i = 0; i < 16; i++) {
    va[i] = __uint_as_float(x[i]);
    vb[i] = __uint_as_float(y[i]);
  }
}
// Load 16 consecutive columns of this thread's lane and wait for them.
__device__ __forceinline__ void tmem_ld16(uint32_t a, float *va) {
  uint32_t x[16];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
               "%10, %11, %12, %13, %14, %15}, [%16];"
               : SSM_O(x, 0), SSM_O(x, 1), SSM_O(x, 2), SSM_O(x, 3), SSM_O(x, 4), SSM_O(x, 5),
                 SSM_O(x, 6), SSM_O(x, 7), SSM_O(x, 8), SSM_O(x, 9), SSM_O(x, 10), SSM_O(x, 11),
                 SSM_O(x, 12), SSM_O(x, 13), SSM_O(x, 14), SSM_O(x, 15) : "r"(a) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : SSM_W(x, 0), SSM_W(x, 1), SSM_W(x, 2), SSM_W(x, 3), SSM_W(x, 4), SSM_W(x, 5),
                 SSM_W(x, 6), SSM_W(x, 7), SSM_W(x, 8), SSM_W(x, 9), SSM_W(x, 10), SSM_W(x, 11),
                 SSM_W(x, 12), SSM_W(x, 13), SSM_W(x, 14), SSM_W(x, 15) :: "memory");
#pragma unroll
  for (int i = 0; i < 16; i++) va[i] = __uint_as_float(x[i]);
}
// Same for 4 or 8 columns (the 1- and 2-state lane layouts).
template <int NV> __device__ __forceinline__ void tmem_ld1(uint32_t a, float *va) {
  if constexpr (NV == 16) {
    tmem_ld16(a, va);
  } else {
    float dummy[NV];
    tmem_ld2<NV>(a, va, a, dummy);
  }
}
#undef SSM_O
#undef SSM_W

}  // namespace ssm
