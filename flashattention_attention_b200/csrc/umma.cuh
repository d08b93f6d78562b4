// umma.cuh -- tcgen05 (5th-generation tensor core) operand descriptors.
//
// Shared-memory matrix descriptor (64 bits):
//   [0,14)  start address >> 4
//   [16,30) leading-dimension byte offset >> 4
//   [32,46) stride-dimension byte offset >> 4
//   [46,48) descriptor version, 1 on sm_100
//   [49,52) base offset (0: every operand tile here is 1024-byte aligned)
//   [52]    LBO mode (0)
//   [61,64) layout: 2 = 128-byte swizzle, 4 = 64-byte swizzle
// Operands are staged by TMA with the 128-byte swizzle, in chunks of
// [rows x 64 bf16] (128 bytes per row, 8-row / 1024-byte swizzle atoms), and
// a head size that is an odd multiple of 32 keeps its last 32 dims in a
// chunk of 64-byte rows with the 64-byte swizzle:
//   K-major (Q, K: the reduction dim contiguous): SBO = 1024 (next 8 rows),
//     LBO unused; the k-th 16-element step starts 32*k bytes further inside
//     a chunk, the next 64 elements one chunk further.
//   MN-major (V as the B operand of O += P V: the output dim contiguous):
//     LBO = byte distance between 64-column chunks, SBO = 1024 (next 8 keys);
//     a 16-key step starts 16 * 128 bytes further.
//
// Instruction descriptor for kind::f16 (32 bits):
//   [4,6) D format (1 = f32), [7,10) A format, [10,13) B format (0 f16,
//   1 bf16), [15] A major, [16] B major (0 K, 1 MN), [17,23) N >> 3,
//   [24,29) M >> 4.
#pragma once

#include <stdint.h>

namespace fa {

constexpr uint32_t kSwizzleChunkRows = 128;  // rows per TMA box in the tensor-core kernels

// layout: 2 = 128-byte swizzle, 4 = 64-byte swizzle
__device__ __forceinline__ uint64_t umma_desc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return umma_desc(smem_addr, lbo_bytes, sbo_bytes, 2u);
}
// 64-byte swizzle (rows of 32 bf16): 8-row / 512-byte atoms.  K-major: SBO =
// 512 (next 8 rows), a 16-element k-step starts 32 bytes further.  MN-major:
// SBO = 512 (next 8 K rows), a 16-row k-step starts 16 * 64 bytes further.
__device__ __forceinline__ uint64_t umma_desc_sw64(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return umma_desc(smem_addr, lbo_bytes, sbo_bytes, 4u);
}

// a_fmt/b_fmt: 0 = f16, 1 = bf16.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int m, int n, uint32_t a_fmt, uint32_t b_fmt,
                                                      bool b_mn_major) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

}  // namespace fa
