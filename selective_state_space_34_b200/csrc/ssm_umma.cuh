// ssm_umma.cuh -- bit layouts of the sm_100a tensor-core (tcgen05.mma) descriptors used by the
// SSD kernels, as host/device constexpr functions so that they can be checked on the host.
//
// Shared-memory matrix descriptor (64 bits): start address >> 4 in bits [0,14), leading byte
// offset >> 4 in [16,30), stride byte offset >> 4 in [32,46), descriptor version 1 in [46,48),
// base offset [49,52) = 0, leading-offset mode bit 52 = 0, layout (swizzle) type [61,64) = 0 for
// the no-swizzle layout. In that layout a core matrix is 8 rows of 16 bytes; the stride offset
// steps between core matrices along M (or N) and the leading offset between core matrices along
// K.
// Instruction descriptor of kind::f16 (32 bits): D format [4,6) (1 = f32), A format [7,10) and B
// format [10,13) (1 = bf16), A / B major bits 15 / 16 (0 = K-major, 1 = MN-major), N >> 3 in
// [17,23), M >> 4 in [24,29).
#pragma once

#include <stdint.h>

namespace ssm {

__host__ __device__ constexpr uint64_t umma_smem_desc_bits(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

__host__ __device__ constexpr uint32_t umma_instr_desc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
         ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace ssm
