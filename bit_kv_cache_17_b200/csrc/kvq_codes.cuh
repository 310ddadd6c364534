// kvq_codes.cuh - scalar readers of single codes from the packed K / V layouts
// (see kvq_common.cuh for the layout).  Used by the dequant kernel and the CUDA-core
// decode path; the tensor-core decode path extracts whole 32-bit words instead.
#pragma once

#include "kvq_common.cuh"

namespace kvq {

// Raw b-bit field of channel ch of a K token (tok = first code byte of the token).
template <int BITS>
__device__ __forceinline__ uint32_t k_field(const uint8_t *tok, int ch) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  const int blk = ch >> 5, e = ch & 31, jj = e >> 2, k = e & 3;
  constexpr int FL = 8 / WL;
  uint32_t f = (tok[16 * (jj / FL) + 4 * blk + k] >> ((jj % FL) * WL)) & ((1u << WL) - 1u);
  if constexpr (WH > 0) {
    constexpr int FH = 8 / WH;
    f |= ((tok[16 * WL + 16 * (jj / FH) + 4 * blk + k] >> ((jj % FH) * WH)) & ((1u << WH) - 1u)) << WL;
  }
  return f;
}

// Raw b-bit field of channel ch of token k (0..3) of a V quad (quad = first byte).
template <int BITS>
__device__ __forceinline__ uint32_t v_field(const uint8_t *quad, int k, int ch) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  const int blk = ch >> 5, e = ch & 31;
  constexpr int FL = 8 / WL;
  uint32_t f = (quad[16 * WL * blk + 4 * (e / FL) + k] >> ((e % FL) * WL)) & ((1u << WL) - 1u);
  if constexpr (WH > 0) {
    constexpr int FH = 8 / WH;
    f |= ((quad[64 * WL + 16 * WH * blk + 4 * (e / FH) + k] >> ((e % FH) * WH)) & ((1u << WH) - 1u)) << WL;
  }
  return f;
}

// Code value of a field: b-bit two's complement for symmetric / kvarn types, unsigned
// for asymmetric types.
template <int FAM, int BITS>
__device__ __forceinline__ int code_value(uint32_t f) {
  if constexpr (FAM == FAM_ASYM) return (int)f;
  return ((int)(f << (32 - BITS))) >> (32 - BITS);
}

}  // namespace kvq
