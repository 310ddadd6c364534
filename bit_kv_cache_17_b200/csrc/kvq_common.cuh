// kvq_common.cuh - device-side layout of the mixed-precision KV cache (sm_100a).
//
// Page layout (one 256-token page of one sequence, one layer):
//   for head h: [K sub-page][V sub-page]
// Sub-page of a quantized type with b-bit codes:
//   [codes: 256 * 16b bytes][d: 256 x 4 fp16][m: 256 x 4 fp16 (qb_1 only)]
//   [t: 256 fp16 (kvarn only)][c: 128 fp16 (kvarn only)]
// Codes of K are stored per token (16b bytes each); codes of V per 4-token quad
// (64b bytes each).  A b-bit code is split into a low plane of width wlo and a high
// plane of width whi (b = 2:2+0, 3:2+1, 4:4+0, 5:4+1, 6:4+2, 8:8+0).  Within a plane of
// width w (F = 8/w fields per byte):
//   K: channel 32*blk + 4*jj + k  ->  byte k of word (m = jj/F, blk) at plane byte
//      16*m + 4*blk, bits [(jj%F)*w, +w)
//   V: channel 32*blk + e of quad token k -> byte k of word m = e/F of block blk at plane
//      byte 16*w*blk + 4*m, bits [(e%F)*w, +w)
// so that a shift and a mask of one 32-bit word yields four 8-bit lanes: for K four
// consecutive channels of one token, for V one channel of four consecutive tokens.
// Symmetric codes are stored as b-bit two's complement, asymmetric codes as unsigned.
// The BF16 tail is a ring of R rows of 128 bf16 per (seq, head, K/V); token p lives in
// row p mod R.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

constexpr int D = 128;
constexpr int GROUP = 256;
constexpr int MAX_G = 8;

enum Family { FAM_BF16 = 0, FAM_SYM = 1, FAM_ASYM = 2, FAM_KVARN = 3 };

struct TypeInfo {
  int fam;
  int bits;
};

__host__ __device__ inline TypeInfo type_info(int t) {
  switch (t) {
    case 0: return {FAM_BF16, 16};
    case 1: return {FAM_SYM, 2};
    case 2: return {FAM_SYM, 3};
    case 3: return {FAM_SYM, 4};
    case 4: return {FAM_SYM, 5};
    case 5: return {FAM_SYM, 6};
    case 6: return {FAM_SYM, 8};
    case 7: return {FAM_ASYM, 4};
    case 8: return {FAM_KVARN, 2};
    case 9: return {FAM_KVARN, 3};
    case 10: return {FAM_KVARN, 4};
    case 11: return {FAM_KVARN, 5};
    case 12: return {FAM_KVARN, 6};
    case 13: return {FAM_KVARN, 8};
    case 14: return {FAM_ASYM, 2};
    case 15: return {FAM_ASYM, 3};
    case 16: return {FAM_ASYM, 5};
    case 17: return {FAM_ASYM, 6};
    default: return {-1, 0};
  }
}

__host__ __device__ constexpr int plane_lo(int bits) { return bits == 8 ? 8 : (bits >= 4 ? 4 : 2); }
__host__ __device__ constexpr int plane_hi(int bits) { return bits - plane_lo(bits); }

// bytes of one token-head in the quantized region (codes + scales, no group scales)
__host__ __device__ inline int token_bytes(int fam, int bits) {
  if (fam == FAM_BF16) return 2 * D;
  int b = 16 * bits + 8;
  if (fam == FAM_ASYM) b += 8;
  if (fam == FAM_KVARN) b += 2;
  return b;
}

struct SubLayout {
  int codes;  // offset of the code area (0)
  int d;      // offset of fp16 block scales
  int m;      // offset of fp16 block minimums (asym) or -1
  int t;      // offset of fp16 token scales (kvarn) or -1
  int c;      // offset of fp16 channel scales (kvarn) or -1
  int bytes;  // sub-page size
};

__host__ __device__ inline SubLayout sub_layout(int fam, int bits) {
  SubLayout s;
  s.codes = 0;
  s.d = GROUP * 16 * bits;
  int off = s.d + GROUP * 8;
  s.m = -1;
  s.t = -1;
  s.c = -1;
  if (fam == FAM_ASYM) {
    s.m = off;
    off += GROUP * 8;
  }
  if (fam == FAM_KVARN) {
    s.t = off;
    off += GROUP * 2;
    s.c = off;
    off += D * 2;
  }
  s.bytes = fam == FAM_BF16 ? 0 : off;
  return s;
}

// Everything a kernel needs to address one layer of a cache.
struct LayerView {
  uint8_t *pages;        // this layer's page pool
  uint8_t *ring;         // this layer's BF16 ring
  const int32_t *ptab;   // page table [n_seqs * max_pages] -> physical page
  int32_t *status;       // device status word (KVQ_STATUS_* bits)
  int64_t max_pages;
  int64_t n_phys;        // physical pages of this layer's pool (n_seqs * max_pages)
  int64_t page_bytes;
  int64_t ring_cap;      // R (rows per ring), 0 if no ring
  int32_t hkv;
  int32_t sub_k, sub_v;  // sub-page bytes of K and V
  int32_t type_k, type_v;
  int32_t tail_f16;      // the ring holds F16 rows (else BF16)
};

// Device status word bits (read and cleared by kvq_get_status): a page-table entry outside the
// layer's page pool (the access goes to physical page 0 instead, inside the caller's buffer),
// a merge ticket past the number of splits of its decode, a bounded wait of the chunk-attention
// pipeline that ran out (the CTA finished without its result).
constexpr int32_t kStatusPageTable = 1;
constexpr int32_t kStatusTicket = 2;
constexpr int32_t kStatusWait = 4;

__device__ __forceinline__ uint8_t *subpage_ptr(const LayerView &L, int seq, int64_t page, int head,
                                                int which) {
  int64_t phys = L.ptab[(int64_t)seq * L.max_pages + page];
  if ((uint64_t)phys >= (uint64_t)L.n_phys) {
    atomicOr(L.status, kStatusPageTable);
    phys = 0;
  }
  return L.pages + phys * L.page_bytes + (int64_t)head * (L.sub_k + L.sub_v) + (which ? L.sub_k : 0);
}

// ---- the tail's 16-bit format ------------------------------------------------------------
// The ring holds BF16 rows, or F16 rows for a cache with an F16 tail.  An F16 tail stores
// fp16(x) of each BF16 input x (round to nearest even, overflow to inf), and the quantizer
// reads that same value whether the token comes from the ring or straight from the input.
// (Every fp16 rounding of a BF16 value is again a BF16 value, so such a stream is the BF16
// stream of the rounded inputs.)
__device__ __forceinline__ float tail_round(float x, int f16) { return f16 ? __half2float(__float2half_rn(x)) : x; }

// two 16-bit ring elements (one 32-bit word, element 0 low) as floats
__device__ __forceinline__ float2 ring2f(uint32_t w, int f16) {
  if (f16) return __half22float2(*reinterpret_cast<const __half2 *>(&w));
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// two BF16 input elements (one word) as the ring stores them
__device__ __forceinline__ uint32_t bf16w_to_ring(uint32_t w, int f16) {
  if (!f16) return w;
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ uint4 bf16x8_to_ring(uint4 v, int f16) {
  if (!f16) return v;
  return make_uint4(bf16w_to_ring(v.x, 1), bf16w_to_ring(v.y, 1), bf16w_to_ring(v.z, 1), bf16w_to_ring(v.w, 1));
}

// ring row of a token (16-bit elements, BF16 or F16 by the cache's tail format)
__device__ __forceinline__ __nv_bfloat16 *ring_row(const LayerView &L, int seq, int head, int which,
                                                   int64_t token) {
  int64_t slot = token % L.ring_cap;
  return reinterpret_cast<__nv_bfloat16 *>(
      L.ring + ((((int64_t)seq * L.hkv + head) * 2 + which) * L.ring_cap + slot) * (2 * D));
}

// fp16 of a positive Sinkhorn scale, clamped to [2^-14, 65504]
__device__ __forceinline__ __half scale_to_half(float v) {
  unsigned short h = __half_as_ushort(__float2half_rn(v));
  if (h < 0x0400u) h = 0x0400u;
  if (h > 0x7bffu) h = 0x7bffu;
  return __ushort_as_half(h);
}

// fp16 with saturation to +-65504 (block scales and minimums)
__device__ __forceinline__ __half sat_half(float v) {
  unsigned short h = __half_as_ushort(__float2half_rn(v));
  if ((h & 0x7fffu) == 0x7c00u) h = (unsigned short)((h & 0x8000u) | 0x7bffu);
  return __ushort_as_half(h);
}

// RN_fp32(2^-3.5): the Walsh-Hadamard normalization, 1/sqrt(128) rounded to fp32
__host__ __device__ constexpr float kKappa() { return 0.0883883461356163f; }

}  // namespace kvq
