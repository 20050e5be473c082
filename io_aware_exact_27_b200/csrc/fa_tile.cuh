// Tile geometry and the tile-level steps that the forward and the backward
// kernels share: TMA loads of a 128-row tile and the S = Q K^T product issued
// on the tensor core (tcgen05, A and B from shared memory, fp32 accumulator in
// tensor memory).
#pragma once

#include "fa_common.cuh"

namespace fa {

constexpr int kBM = 128;      // query rows per tile
constexpr int kBN = 128;      // keys per block

// Loads one 128 x D tile (EB bytes per element) as D*EB/128 boxes of 128
// rows x 128 bytes (SW128).
template <int D, int EB = 2>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* m, uint32_t bar, int head, int row0) {
#pragma unroll
  for (int b = 0; b < D * EB / 128; ++b) tma_load_3d(dst + b * 16384, m, bar, b * (128 / EB), head, row0);
}

// Descriptors are built once per call; each MMA adds a compile-time byte
// offset (>> 4) to the 14-bit start-address field. Shared-memory addresses
// stay below 228 KB, so (address + offset) >> 4 never leaves the field.

// S = Q K^T over d: each MMA consumes 32 bytes of every row (16 bf16 or 32
// e4m3 elements), advancing inside the 128-byte swizzle row.
template <int D, bool F8 = false>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(kBM, kBN, false, false) : idesc_bf16_f32(kBM, kBN, false, false);
  const uint64_t qd = smem_desc(q_smem, 16, 1024, kSwizzle128B);
  const uint64_t kd = smem_desc(k_smem, 16, 1024, kSwizzle128B);
#pragma unroll
  for (int kk = 0; kk < D * (F8 ? 1 : 2) / 32; ++kk) {
    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
    if constexpr (F8)
      mma_f8_ss(s_tmem, qd + off, kd + off, idesc, kk > 0 ? 1u : 0u);
    else
      mma_f16_ss(s_tmem, qd + off, kd + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// A operand taken from TMEM where each column half of the softmax stored its
// 16-bit pairs: 16-key step kk of the first half at column 8*kk, of the
// second half at column 64 + 8*(kk-4).
__device__ __forceinline__ uint32_t split_a_col(int kk) { return kk < 4 ? 8 * kk : 64 + 8 * (kk - 4); }

}  // namespace fa
