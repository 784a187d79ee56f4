// Internal declarations shared by the host-side translation units of libsvdq.
#pragma once
#include <cstddef>
#include <cstdint>

#include "svdq.h"

namespace svdq {

// Limits of this build (checked before any launch).
constexpr int kMaxRank = 128;

inline svdq_status check_dims(svdq_format fmt, int64_t M, int64_t N, int64_t K, int rank) {
  if (fmt != SVDQ_FMT_NVFP4_G16 && fmt != SVDQ_FMT_INT4_G64 && fmt != SVDQ_FMT_MXFP4_G32 && fmt != SVDQ_FMT_W8A8)
    return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || N < 128 || K < 128) return SVDQ_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 128 != 0) return SVDQ_ERR_INVALID_ARG;
  if (rank < 0 || rank > kMaxRank || rank % 16 != 0) return SVDQ_ERR_INVALID_ARG;
  // 32-bit indexing inside the kernels and TMA coordinate limits
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 24) || K > (int64_t(1) << 24))
    return SVDQ_ERR_UNSUPPORTED;
  return SVDQ_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint16_t f32_to_bf16_rn(float f);
float bf16_to_f32(uint16_t h);
uint16_t f32_to_f16_rn_sat(float f);
float f16_to_f32(uint16_t h);
uint8_t f32_to_e4m3_rn_sat(float x);
float e4m3_to_f32(uint8_t c);
uint8_t f32_to_e2m1_rn_sat(float v);
float pow2_gscale(float amax);
bool is_pow2_positive(float g);
// Byte offset of the scale of (row, group) in the 128x4 blocked layout, groups of g elements.
size_t blocked_sf_offset(int64_t row, int64_t grp, int64_t K, int g);
// Group size of an E2M1 format (16 NVFP4, 32 MXFP4).
inline int fp4_group(svdq_format fmt) { return fmt == SVDQ_FMT_MXFP4_G32 ? 32 : 16; }
// Bytes of the codes of `rows` rows: one byte per element for W8A8, half a byte otherwise.
inline size_t code_bytes(svdq_format fmt, int64_t rows, int64_t K) {
  return static_cast<size_t>(fmt == SVDQ_FMT_W8A8 ? rows * K : rows * K / 2);
}

}  // namespace svdq
