// kvq_chunk.cu - attention of a chunk of queries over [quantized prefix | BF16 tail], causal
// within the chunk (the prefill side of the pages' prefill / decode split: "Fork of beellama and
// kvarn KV quants at long context", section "Which data should accompany a speed-up claim").
//
// A decode reads every cached token once per query row; a chunk of n_q queries would read it
// n_q times.  Here each 32-token piece of the cache is read and dequantized once, into shared
// memory, for all n_q x G query rows of its KV head, and Q.K and P.V are dense f16 tensor-core
// tiles (mma.sync m16n8k16, fp32 accumulation):
//  - K-hat = code * d (+ m for qb_1 types) and V-hat = code * d (+ m) (* c for kvarn V) are
//    computed in fp32 and stored as f16 high part + f16 remainder (together exact for every
//    code width); BF16 / F16 ring rows are stored the same way (their remainder is zero);
//  - the query rows (rotated, q' = H.q.kappa, and scaled per page by the K channel scales c for
//    kvarn K) are f16 high part + remainder as well; Q.K takes hi.hi + lo.hi + hi.lo;
//  - the kvarn token scales t multiply the scores (K) and the softmax weights (V); the weights
//    are one f16 each; P.V takes p.hi + p.lo of V-hat;
//  - each CTA covers a range of chunks of one KV head (split-K); k_chunk_merge combines the
//    splits (LSE) and applies the inverse WHT to the rotated V accumulator once per row.
// Values are limited to the f16 range (|x| < 65504) in this path.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>

#include "kvq_codes.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int CH = 32;               // tokens per chunk
constexpr int NQ = 16;               // query tokens per launch (at most MAXR / G)
constexpr int RT = 16;               // rows per row tile (one consumer warp)
constexpr int NC = 5;                // consumer warps: Q.K, softmax and P.V of one row tile each
constexpr int NP = 5;                // producer warps: copies and dequantization
constexpr int MAXR = NC * RT;        // 80 rows per launch
constexpr int NW = NP + NC;          // 10 warps
constexpr int NT = 32 * NW;          // 320 threads
constexpr int NPT = 32 * NP;         // producer threads
constexpr int TS = D + 8;            // padded f16 row stride of the shared tiles (272 B)
constexpr int MAXSPL = 64;           // splits per KV head
constexpr int PSTRIDE = 4 + D;       // floats per partial record: m, l, 2 pad, acc[128]
constexpr float LOG2E = 1.4426950408889634f;

struct CArgs {
  int32_t seq, nq, G, hkv, rotk, rotv;
  int32_t nsq, nst;      // splits per KV head over the quantized prefix / the 16-bit tail
  int32_t cps_q, cps_t;  // chunks per split
  int32_t fam_k, bits_k, fam_v, bits_v;
  int64_t n, Q;          // sequence length (the chunk included), quantized tokens
  float qscale;          // softmax scale * log2(e)
  const float *q;        // [nq][hq][128]
  float *ws;             // records [qi][head][split][g][PSTRIDE]
};

// Raw bytes of one chunk (one KV head): K then V, each [codes | d | m | t | c] for a quantized
// chunk (c only on a page's first chunk) or 32 ring rows for a 16-bit chunk.
constexpr int RAW_SIDE = 32 * 2 * D;  // 8 KB: the 16-bit case is the largest
struct Raw {
  alignas(16) uint8_t k[RAW_SIDE];
  alignas(16) uint8_t v[RAW_SIDE];
};
// offsets inside one side of a quantized chunk
struct RawLay {
  int codes, d, m, t;
};
__host__ __device__ inline RawLay raw_lay(int fam, int bits) {
  RawLay r;
  r.codes = 0;
  r.d = 512 * bits;
  r.m = r.d + 256;
  r.t = r.m + (fam == FAM_ASYM ? 256 : 0);
  return r;
}

constexpr int NS = 3;  // raw chunks in the producers' ring (copies run two chunks ahead)
struct Tiles {
  __half kt[2][CH * TS];             // K-hat hi / lo, [token][channel]
  __half vt[2][CH * TS];             // V-hat hi / lo, [token][channel]
  float tk[CH], tv[CH];              // token scales of the chunk (1 for non-kvarn / 16-bit rows)
};
struct Smem {
  Raw raw[NS];                       // ring of raw chunks
  Tiles tile[2];                     // dequantized chunks, double-buffered between the roles
  __half qt[2][MAXR * TS];           // the rows' q'' hi / lo, [row][channel]
  alignas(16) float qr[MAXR * D];    // the rows' q' (rotated for quantized K, scaled by qscale)
  alignas(16) __half ck[2][D];       // K / V channel scales of a page (kvarn), by page parity: a
  alignas(16) __half cv[2][D];       // copy one chunk ahead may belong to the next page
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }

// x as an f16 high part and an f16 remainder
__device__ __forceinline__ void split_h(float x, __half &hi, __half &lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

// H.x of one 128-wide row by one warp: the lane holds x[4 lane .. 4 lane + 3]
__device__ __forceinline__ void warp_wht(float (&v)[4], int lane) {
  float a = v[0], b = v[1];
  v[0] = a + b;
  v[1] = a - b;
  a = v[2];
  b = v[3];
  v[2] = a + b;
  v[3] = a - b;
  a = v[0];
  b = v[2];
  v[0] = a + b;
  v[2] = a - b;
  a = v[1];
  b = v[3];
  v[1] = a + b;
  v[3] = a - b;
#pragma unroll
  for (int o = 1; o <= 16; o <<= 1) {
    const bool hi = lane & o;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float other = __shfl_xor_sync(FULL, v[e], o);
      v[e] = hi ? other - v[e] : v[e] + other;
    }
  }
}

// Copies chunk [i0, i0 + 32) of one KV head into `r` (all threads, 16 bytes each, one commit
// group issued by the caller).  Quantized: codes, d (and m, t) of K and V; on a page's first
// chunk, or the split's first, also the page's channel scales (kvarn) into the scale slots of
// the page's parity.
__device__ __forceinline__ void copy_chunk(const LayerView &L, const CArgs &A, int head, int64_t i0, bool first,
                                           Raw &r, Smem &S, int tid) {
  constexpr int NT = NPT;  // the producer threads issue the copies
  if (i0 < A.Q) {
    const int64_t page = i0 / GROUP;
    const int tip0 = (int)(i0 % GROUP);
    const uint8_t *sk = subpage_ptr(L, A.seq, page, head, 0);
    const uint8_t *sv = sk + L.sub_k;
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      const int fam = side ? A.fam_v : A.fam_k, bits = side ? A.bits_v : A.bits_k;
      const uint8_t *sub = side ? sv : sk;
      uint8_t *dst = side ? r.v : r.k;
      const SubLayout lay = sub_layout(fam, bits);
      const RawLay rl = raw_lay(fam, bits);
      const int ncode = 32 * bits;  // 16-byte pieces of the chunk's codes (contiguous for K and V)
      for (int p = tid; p < ncode; p += NT) cp_async16(dst + 16 * p, sub + tip0 * 16 * bits + 16 * p);
      if (tid < 16) cp_async16(dst + rl.d + 16 * tid, sub + lay.d + tip0 * 8 + 16 * tid);
      if (fam == FAM_ASYM && tid >= 16 && tid < 32)
        cp_async16(dst + rl.m + 16 * (tid - 16), sub + lay.m + tip0 * 8 + 16 * (tid - 16));
      if (fam == FAM_KVARN && tid >= 32 && tid < 36) cp_async16(dst + rl.t + 16 * (tid - 32), sub + lay.t + tip0 * 2 + 16 * (tid - 32));
      if (fam == FAM_KVARN && (tip0 == 0 || first) && tid >= 64 && tid < 80)
        cp_async16((side ? S.cv : S.ck)[page & 1] + 8 * (tid - 64), sub + lay.c + 16 * (tid - 64));
    }
  } else {
    // 16-bit ring rows: 32 rows x 256 bytes per side
    for (int p = tid; p < 2 * 32 * 16; p += NT) {
      const int side = p >> 9, row = (p >> 4) & 31, piece = p & 15;
      const int64_t tok = i0 + row;
      if (tok < A.n) {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(ring_row(L, A.seq, head, side, tok)) + 16 * piece;
        cp_async16((side ? r.v : r.k) + 256 * row + 16 * piece, src);
      }
    }
  }
}

// One side (K or V) of a quantized chunk, by single codes (any type): token i, channels
// 32 blk .. 32 blk + 31 (thread = (token, block)): value = code * d (+ m) (the kvarn channel
// scales are applied elsewhere: to the query for K, to the accumulator for V), computed in fp32
// and stored as f16 hi / lo.  A token past the split (ok false) is stored as zeros (its bytes
// are stale).
template <int WHICH, int FAM, int BITS>
__device__ __forceinline__ void dequant_q(const uint8_t *raw, const __half *cs, __half *hi, __half *lo, int tok,
                                          int blk, bool ok) {
  const RawLay rl = raw_lay(FAM, BITS);
  const float d = ok ? __half2float(reinterpret_cast<const __half *>(raw + rl.d)[tok * 4 + blk]) : 0.f;
  const float m =
      ok && FAM == FAM_ASYM ? __half2float(reinterpret_cast<const __half *>(raw + rl.m)[tok * 4 + blk]) : 0.f;
  const uint8_t *tokp = raw + tok * 16 * BITS;          // K: the token's codes
  const uint8_t *quad = raw + (tok >> 2) * 64 * BITS;   // V: the quad's codes
  __half *h = hi + tok * TS + 32 * blk, *l = lo + tok * TS + 32 * blk;
#pragma unroll 8
  for (int e = 0; e < 32; e += 2) {
    float x[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int ch = 32 * blk + e + u;
      const uint32_t f = WHICH == 0 ? k_field<BITS>(tokp, ch) : v_field<BITS>(quad, tok & 3, ch);
      x[u] = ok ? fmaf((float)code_value<FAM, BITS>(f), d, m) : 0.f;
    }
    const __half2 hh = __floats2half2_rn(x[0], x[1]);
    const float2 hf = __half22float2(hh);
    const __half2 ll = __floats2half2_rn(x[0] - hf.x, x[1] - hf.y);
    *reinterpret_cast<__half2 *>(h + e) = hh;
    *reinterpret_cast<__half2 *>(l + e) = ll;
  }
}

// ---- word-level dequantization of symmetric codes (qN_0, kvarn) ------------------------------
//
// A 32-bit word of a code plane holds four b-bit fields (one per byte, after a shift and a
// mask); xor with 2^(b-1) in every byte turns b-bit two's complement codes into c + 2^(b-1), and
// pairing each byte with 0x64 gives the f16 value 1024 + c + 2^(b-1), exactly; one f16
// subtraction leaves the code c.  hi = RN(c d) and lo = c d - hi (one fused multiply-add) are
// f16 again (exact: c d has at most 19 significant bits).

template <int W>
__device__ __forceinline__ constexpr uint32_t bytes_mask() {
  return ((1u << W) - 1u) * 0x01010101u;
}

// codes + 2^(b-1) of 4 consecutive fields as bytes -> 2 f16 pairs of the codes, times d (hi, lo)
template <int BITS>
__device__ __forceinline__ void fields_to_half(uint32_t u, __half2 d2, uint32_t &h01, uint32_t &h23, uint32_t &l01,
                                               uint32_t &l23) {
  const uint32_t v = u ^ (0x01010101u << (BITS - 1));
  const __half2 off = __float2half2_rn((float)(1024 + (1 << (BITS - 1))));
  const uint32_t a = __byte_perm(v, 0x64646464u, 0x5140), b = __byte_perm(v, 0x64646464u, 0x5342);
  const __half2 c01 = __hsub2(*reinterpret_cast<const __half2 *>(&a), off);
  const __half2 c23 = __hsub2(*reinterpret_cast<const __half2 *>(&b), off);
  const __half2 x01 = __hmul2(c01, d2), x23 = __hmul2(c23, d2);
  const __half2 r01 = __hfma2(c01, d2, __hneg2(x01)), r23 = __hfma2(c23, d2, __hneg2(x23));
  h01 = h2u(x01);
  h23 = h2u(x23);
  l01 = h2u(r01);
  l23 = h2u(r23);
}

// K: token tok, block blk (thread); channels 32 blk + 4 jj + k are byte k of word (jj / F, blk)
template <int BITS>
__device__ __forceinline__ void dequant_k_fast(const uint8_t *raw, __half *hi, __half *lo, int tok, int blk, bool ok) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  constexpr int FL = 8 / WL, FH = WH ? 8 / WH : 1;
  const RawLay rl = raw_lay(FAM_SYM, BITS);
  const __half dh = ok ? reinterpret_cast<const __half *>(raw + rl.d)[tok * 4 + blk] : __float2half(0.f);
  const __half2 d2 = __halves2half2(dh, dh);
  const uint8_t *tp = raw + tok * 16 * BITS;
  __half *h = hi + tok * TS + 32 * blk, *l = lo + tok * TS + 32 * blk;
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    const uint32_t wl = *reinterpret_cast<const uint32_t *>(tp + 16 * (jj / FL) + 4 * blk);
    uint32_t u = (wl >> ((jj % FL) * WL)) & bytes_mask<WL>();
    if constexpr (WH > 0) {
      const uint32_t wh = *reinterpret_cast<const uint32_t *>(tp + 16 * WL + 16 * (jj / FH) + 4 * blk);
      u |= ((wh >> ((jj % FH) * WH)) & bytes_mask<WH>()) << WL;
    }
    uint32_t h01, h23, l01, l23;
    fields_to_half<BITS>(u, d2, h01, h23, l01, l23);
    *reinterpret_cast<uint2 *>(h + 4 * jj) = make_uint2(h01, h23);
    *reinterpret_cast<uint2 *>(l + 4 * jj) = make_uint2(l01, l23);
  }
}

// V: quad q, block blk, 8 channels 32 blk + 8 j8 .. + 7 of the quad's 4 tokens (thread).  In a
// plane of width w the channel 32 blk + e of token k is byte k of word e / F at 16 w blk + 4 (e / F),
// bits (e % F) w: the thread's channels are the fields of words (8 j8 / F) .. (8 j8 + 7) / F.
template <int BITS>
__device__ __forceinline__ void dequant_v_fast(const uint8_t *raw, __half *hi, __half *lo, int q, int blk, int j8,
                                               int64_t tok_end) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  constexpr int FL = 8 / WL, FH = WH ? 8 / WH : 1;
  constexpr int NL = 8 / FL, NH = WH ? 8 / FH : 0;  // words of each plane holding the 8 channels
  const RawLay rl = raw_lay(FAM_SYM, BITS);
  const uint8_t *qp = raw + q * 64 * BITS;
  uint32_t wl[NL], wh[NH > 0 ? NH : 1];
#pragma unroll
  for (int i = 0; i < NL; ++i) wl[i] = *reinterpret_cast<const uint32_t *>(qp + 16 * WL * blk + 4 * (NL * j8 + i));
#pragma unroll
  for (int i = 0; i < NH; ++i) wh[i] = *reinterpret_cast<const uint32_t *>(qp + 64 * WL + 16 * WH * blk + 4 * (NH * j8 + i));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int tok = 4 * q + k;
    const bool ok = tok < tok_end;
    const __half dh = ok ? reinterpret_cast<const __half *>(raw + rl.d)[tok * 4 + blk] : __float2half(0.f);
    const __half2 d2 = __halves2half2(dh, dh);
    __half *h = hi + tok * TS + 32 * blk + 8 * j8, *l = lo + tok * TS + 32 * blk + 8 * j8;
    uint32_t u[2];  // fields of channels 0..3 and 4..7 of the group, one per byte
    if constexpr (BITS == 4) {
      // byte k of the 4 words, then low nibbles = even channels, high nibbles = odd channels
      const uint32_t sel = (uint32_t)k | ((uint32_t)(4 + k) << 4);
      const uint32_t x = __byte_perm(__byte_perm(wl[0], wl[1], sel), __byte_perm(wl[2], wl[3], sel), 0x5410);
      const uint32_t ev = x & 0x0f0f0f0fu, od = (x >> 4) & 0x0f0f0f0fu;
      u[0] = __byte_perm(ev, od, 0x5140);
      u[1] = __byte_perm(ev, od, 0x7362);
    } else {
#pragma unroll
      for (int g4 = 0; g4 < 2; ++g4) {
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = 4 * g4 + i;
          uint32_t f = (wl[e / FL] >> (8 * k + (e % FL) * WL)) & ((1u << WL) - 1u);
          if constexpr (WH > 0) f |= ((wh[e / FH] >> (8 * k + (e % FH) * WH)) & ((1u << WH) - 1u)) << WL;
          acc |= f << (8 * i);
        }
        u[g4] = acc;
      }
    }
#pragma unroll
    for (int g4 = 0; g4 < 2; ++g4) {
      uint32_t h01, h23, l01, l23;
      fields_to_half<BITS>(u[g4], d2, h01, h23, l01, l23);
      *reinterpret_cast<uint2 *>(h + 4 * g4) = make_uint2(h01, h23);
      *reinterpret_cast<uint2 *>(l + 4 * g4) = make_uint2(l01, l23);
    }
  }
}

__device__ __forceinline__ void dequant_k_sym(int bits, const uint8_t *raw, __half *hi, __half *lo, int tok, int blk,
                                              bool ok) {
  switch (bits) {
    case 2: dequant_k_fast<2>(raw, hi, lo, tok, blk, ok); break;
    case 3: dequant_k_fast<3>(raw, hi, lo, tok, blk, ok); break;
    case 4: dequant_k_fast<4>(raw, hi, lo, tok, blk, ok); break;
    case 5: dequant_k_fast<5>(raw, hi, lo, tok, blk, ok); break;
    case 6: dequant_k_fast<6>(raw, hi, lo, tok, blk, ok); break;
    default: dequant_k_fast<8>(raw, hi, lo, tok, blk, ok); break;
  }
}
__device__ __forceinline__ void dequant_v_sym(int bits, const uint8_t *raw, __half *hi, __half *lo, int q, int blk,
                                              int j8, int64_t tok_end) {
  switch (bits) {
    case 2: dequant_v_fast<2>(raw, hi, lo, q, blk, j8, tok_end); break;
    case 3: dequant_v_fast<3>(raw, hi, lo, q, blk, j8, tok_end); break;
    case 4: dequant_v_fast<4>(raw, hi, lo, q, blk, j8, tok_end); break;
    case 5: dequant_v_fast<5>(raw, hi, lo, q, blk, j8, tok_end); break;
    case 6: dequant_v_fast<6>(raw, hi, lo, q, blk, j8, tok_end); break;
    default: dequant_v_fast<8>(raw, hi, lo, q, blk, j8, tok_end); break;
  }
}

template <int WHICH>
__device__ __forceinline__ void dequant_side(int fam, int bits, const uint8_t *raw, const __half *cs, __half *hi,
                                             __half *lo, int tok, int blk, bool ok) {
#define KVQ_DQ(F, B)                                           \
  if (fam == F && bits == B) {                                 \
    dequant_q<WHICH, F, B>(raw, cs, hi, lo, tok, blk, ok);     \
    return;                                                    \
  }
  KVQ_DQ(FAM_SYM, 2) KVQ_DQ(FAM_SYM, 3) KVQ_DQ(FAM_SYM, 4) KVQ_DQ(FAM_SYM, 5) KVQ_DQ(FAM_SYM, 6) KVQ_DQ(FAM_SYM, 8)
  KVQ_DQ(FAM_ASYM, 2) KVQ_DQ(FAM_ASYM, 3) KVQ_DQ(FAM_ASYM, 4) KVQ_DQ(FAM_ASYM, 5) KVQ_DQ(FAM_ASYM, 6)
  KVQ_DQ(FAM_KVARN, 2) KVQ_DQ(FAM_KVARN, 3) KVQ_DQ(FAM_KVARN, 4) KVQ_DQ(FAM_KVARN, 5) KVQ_DQ(FAM_KVARN, 6)
  KVQ_DQ(FAM_KVARN, 8)
#undef KVQ_DQ
}

// q'' of this warp's 16 rows into the f16 tiles: q' times the page's K channel scales when ck is
// given (kvarn K); lane = 4 channels
__device__ __forceinline__ void build_q_tiles(Smem &S, const __half *ck, int warp, int lane) {
  for (int rr = 0; rr < RT; ++rr) {
    const int row = RT * warp + rr;
    const float4 qv = *reinterpret_cast<const float4 *>(&S.qr[row * D + 4 * lane]);
    float x[4] = {qv.x, qv.y, qv.z, qv.w};
    if (ck) {
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] *= __half2float(ck[4 * lane + e]);
    }
    __half h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split_h(x[e], h[e], l[e]);
    __half *ph = &S.qt[0][row * TS + 4 * lane], *pl = &S.qt[1][row * TS + 4 * lane];
    *reinterpret_cast<uint2 *>(ph) = make_uint2(h2u(__halves2half2(h[0], h[1])), h2u(__halves2half2(h[2], h[3])));
    *reinterpret_cast<uint2 *>(pl) = make_uint2(h2u(__halves2half2(l[0], l[1])), h2u(__halves2half2(l[2], l[3])));
  }
}

// named barriers between the roles: FULL[b] (producers arrive when tile buffer b holds a
// chunk, consumers wait), EMPTY[b] (consumers arrive when done with it, producers wait), and
// one among the producers
__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
constexpr int BAR_FULL = 1, BAR_EMPTY = 3, BAR_PROD = 5;

// Producer side of chunk c: dequantize the raw chunk into tile buffer T (unit u of 256:
// quantized K (token, block), quantized V (quad, block, 8 channels) or (token, block) for qb_1,
// 16-bit rows (token, 32 channels, side)).
__device__ __forceinline__ void produce_tile(const LayerView &L, const CArgs &A, const Raw &rw, Tiles &T, bool tail,
                                             int64_t i0, int64_t b, int ptid) {
  for (int u = ptid; u < 256; u += NPT) {
    if (!tail) {
      if (u < 128) {
        const int tk = u >> 2, bk = u & 3;
        const bool ok = i0 + tk < b;
        if (A.fam_k != FAM_ASYM)
          dequant_k_sym(A.bits_k, rw.k, T.kt[0], T.kt[1], tk, bk, ok);
        else
          dequant_side<0>(A.fam_k, A.bits_k, rw.k, nullptr, T.kt[0], T.kt[1], tk, bk, ok);
      } else {
        const int t = u - 128;
        if (A.fam_v != FAM_ASYM) {
          dequant_v_sym(A.bits_v, rw.v, T.vt[0], T.vt[1], t >> 4, (t >> 2) & 3, t & 3, b - i0);
        } else {
          const int tv = t >> 2, bv = t & 3;
          dequant_side<1>(A.fam_v, A.bits_v, rw.v, nullptr, T.vt[0], T.vt[1], tv, bv, i0 + tv < b);
        }
      }
    } else {
      // 16-bit rows: rows past the end are zero
      const int tok = u >> 3, blk = (u >> 1) & 3, side = u & 1;
      const bool ok = i0 + tok < b;
      const uint8_t *src = (side ? rw.v : rw.k) + 256 * tok + 64 * blk;
      __half *h = (side ? T.vt[0] : T.kt[0]) + tok * TS + 32 * blk;
      __half *l = (side ? T.vt[1] : T.kt[1]) + tok * TS + 32 * blk;
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const uint32_t w = ok ? *reinterpret_cast<const uint32_t *>(src + 2 * e) : 0u;
        float x0, x1;
        if (L.tail_f16) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w));
          x0 = f.x;
          x1 = f.y;
        } else {
          x0 = __uint_as_float(w << 16);
          x1 = __uint_as_float(w & 0xffff0000u);
        }
        const __half2 hh = __floats2half2_rn(x0, x1);
        const float2 hf = __half22float2(hh);
        *reinterpret_cast<__half2 *>(h + e) = hh;
        *reinterpret_cast<__half2 *>(l + e) = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
      }
    }
  }
  if (ptid < CH) {
    const bool ok = i0 + ptid < b;
    float tkv = ok ? 1.f : 0.f, tvv = tkv;
    if (!tail && ok && A.fam_k == FAM_KVARN)
      tkv = __half2float(reinterpret_cast<const __half *>(rw.k + raw_lay(A.fam_k, A.bits_k).t)[ptid]);
    if (!tail && ok && A.fam_v == FAM_KVARN)
      tvv = __half2float(reinterpret_cast<const __half *>(rw.v + raw_lay(A.fam_v, A.bits_v).t)[ptid]);
    T.tk[ptid] = tkv;
    T.tv[ptid] = tvv;
  }
}

__global__ void __launch_bounds__(NT, 1) k_chunk(LayerView L, CArgs A) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem &S = *reinterpret_cast<Smem *>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int nspl = A.nsq + A.nst;
  const int head = blockIdx.x / nspl, sp = blockIdx.x % nspl;
  const int G = A.G, R = A.nq * G;
  const bool tail = sp >= A.nsq;
  int64_t a, b;
  if (!tail) {
    a = (int64_t)sp * A.cps_q * CH;
    b = min(a + (int64_t)A.cps_q * CH, A.Q);
  } else {
    a = A.Q + (int64_t)(sp - A.nsq) * A.cps_t * CH;
    b = min(a + (int64_t)A.cps_t * CH, A.n);
  }
  const int nch = b > a ? (int)((b - a + CH - 1) / CH) : 0;
  const bool producer = warp < NP;

  // the producers' first NS - 1 chunks in flight (one commit group each) while q' is computed
  if (producer) {
#pragma unroll 1
    for (int j = 0; j < NS - 1; ++j) {
      if (j < nch) copy_chunk(L, A, head, a + (int64_t)j * CH, j == 0, S.raw[j], S, tid);
      cp_async_commit();
    }
  }
  // q' of every row (row = qi * G + hd; rows past R are zero), scaled by softmax scale * log2(e)
  // and, for a quantized kvarn K, rotated; warp per row
  for (int row = warp; row < MAXR; row += NW) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (row < R) {
      const int qi = row / G, hd = row % G;
      const float4 x = __ldg(reinterpret_cast<const float4 *>(A.q + ((int64_t)qi * A.hkv * G + head * G + hd) * D) + lane);
      v[0] = x.x * A.qscale;
      v[1] = x.y * A.qscale;
      v[2] = x.z * A.qscale;
      v[3] = x.w * A.qscale;
      if (A.rotk && !tail) {
        warp_wht(v, lane);
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] *= kKappa();
      }
    }
    *reinterpret_cast<float4 *>(&S.qr[row * D + 4 * lane]) = make_float4(v[0], v[1], v[2], v[3]);
  }
  __syncthreads();

  if (producer) {
    // ---- producers: copies two chunks ahead, dequantization into the tile buffers
    for (int c = 0; c < nch; ++c) {
      const int64_t i0 = a + (int64_t)c * CH;
      const int tb = c & 1;
      cp_async_wait<NS - 2>();   // this thread's copies of chunk c have landed
      bar_sync(BAR_PROD, NPT);   // ... every producer's, and every producer is done with chunk c - 1
      if (c + NS - 1 < nch) copy_chunk(L, A, head, i0 + (NS - 1) * CH, false, S.raw[(c + NS - 1) % NS], S, tid);
      cp_async_commit();
      if (c >= 2) bar_sync(BAR_EMPTY + tb, NT);  // the consumers are done with chunk c - 2
      produce_tile(L, A, S.raw[c % NS], S.tile[tb], tail, i0, b, tid);
      bar_arrive(BAR_FULL + tb, NT);
    }
    cp_async_wait<0>();
    return;
  }

  // ---- consumers: warp w' = warp - NP takes rows 16 w' .. 16 w' + 15
  const int cw = warp - NP;
  const bool kvarn_k = !tail && A.fam_k == FAM_KVARN;
  if (!kvarn_k) build_q_tiles(S, nullptr, cw, lane);  // (kvarn K: per page, below)
  const int r0 = RT * cw + g, r1 = r0 + 8;
  const int64_t lim0 = r0 < R ? A.n - A.nq + 1 + r0 / G : 0;
  const int64_t lim1 = r1 < R ? A.n - A.nq + 1 + r1 / G : 0;
  const bool active = RT * cw < R;
  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  int64_t cur_page = -1, cur_vpage = -1;
  const bool kvarn_v = !tail && A.fam_v == FAM_KVARN;

  for (int c = 0; c < nch; ++c) {
    const int64_t i0 = a + (int64_t)c * CH;
    const int tb = c & 1;
    const Tiles &T = S.tile[tb];
    bar_sync(BAR_FULL + tb, NT);  // chunk c is in tile buffer tb (and its page scales have landed)
    const int64_t page = i0 / GROUP;
    // new kvarn page: q'' of this warp's rows from the page's K channel scales
    if (kvarn_k && page != cur_page) {
      build_q_tiles(S, S.ck[page & 1], cw, lane);
      __syncwarp();
      cur_page = page;
    }
    if (active) {
      // kvarn V: the accumulator carries the channel scales of the current page; a new page
      // rescales it by c_old / c_new (V-hat holds code * d only)
      if (kvarn_v && page != cur_vpage) {
        if (cur_vpage >= 0) {
#pragma unroll
          for (int jn = 0; jn < 16; ++jn)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int ch = 8 * jn + 2 * tq + e;
              const float r = __half2float(S.cv[cur_vpage & 1][ch]) / __half2float(S.cv[page & 1][ch]);
              o[jn][e] *= r;
              o[jn][2 + e] *= r;
            }
        }
        cur_vpage = page;
      }
      // ---- S = Q.K-hat: 4 n-tiles of 8 tokens, 8 k-steps of 16 channels; hi.hi + lo.hi + hi.lo
      float s[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
      const __half *qh = &S.qt[0][(RT * cw + (lane & 15)) * TS + 8 * (lane >> 4)];
      const __half *ql = &S.qt[1][(RT * cw + (lane & 15)) * TS + 8 * (lane >> 4)];
      // B: lanes 0-7 / 8-15 / 16-23 / 24-31 address matrices (tokens 8 nt2 + 0..7, channels
      // k0 + 0..7), (same tokens, k0 + 8..15), (tokens 8 nt2 + 8.., k0), (tokens 8 nt2 + 8.., k0 + 8)
      const int brow = (lane & 7) + 8 * (lane >> 4), bcol = 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t ah[4], al[4];
        ldsm_x4(ah, qh + 16 * ks);
        ldsm_x4(al, ql + 16 * ks);
#pragma unroll
        for (int np = 0; np < 2; ++np) {  // pairs of n-tiles
          uint32_t bh[4], bl[4];
          ldsm_x4(bh, &T.kt[0][(16 * np + brow) * TS + 16 * ks + bcol]);
          ldsm_x4(bl, &T.kt[1][(16 * np + brow) * TS + 16 * ks + bcol]);
          mma16(s[2 * np], ah, bh[0], bh[1]);
          mma16(s[2 * np], al, bh[0], bh[1]);
          mma16(s[2 * np], ah, bl[0], bl[1]);
          mma16(s[2 * np + 1], ah, bh[2], bh[3]);
          mma16(s[2 * np + 1], al, bh[2], bh[3]);
          mma16(s[2 * np + 1], ah, bl[2], bl[3]);
        }
      }
      // ---- token scales, causal masks, online softmax of rows r0 (c0, c1) and r1 (c2, c3)
      float cmax0 = -INFINITY, cmax1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = 8 * nt + 2 * tq + e;
          const int64_t tokg = i0 + t;
          const float tk = T.tk[t];
          s[nt][e] = (tokg < lim0 && tokg < b) ? s[nt][e] * tk : -INFINITY;
          s[nt][2 + e] = (tokg < lim1 && tokg < b) ? s[nt][2 + e] * tk : -INFINITY;
          cmax0 = fmaxf(cmax0, s[nt][e]);
          cmax1 = fmaxf(cmax1, s[nt][2 + e]);
        }
      cmax0 = fmaxf(cmax0, __shfl_xor_sync(FULL, cmax0, 1));
      cmax0 = fmaxf(cmax0, __shfl_xor_sync(FULL, cmax0, 2));
      cmax1 = fmaxf(cmax1, __shfl_xor_sync(FULL, cmax1, 1));
      cmax1 = fmaxf(cmax1, __shfl_xor_sync(FULL, cmax1, 2));
      const float mn0 = fmaxf(m0, cmax0), mn1 = fmaxf(m1, cmax1);
      // a row with nothing valid so far keeps m = -inf, weight 0, scale 1
      const float al0 = mn0 == -INFINITY ? 1.f : exp2_fast(m0 - mn0);
      const float al1 = mn1 == -INFINITY ? 1.f : exp2_fast(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float p[4][4], ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          p[nt][e] = mn0 == -INFINITY ? 0.f : exp2_fast(s[nt][e] - mn0);
          p[nt][2 + e] = mn1 == -INFINITY ? 0.f : exp2_fast(s[nt][2 + e] - mn1);
          ps0 += p[nt][e];
          ps1 += p[nt][2 + e];
        }
      l0 = fmaf(l0, al0, ps0);
      l1 = fmaf(l1, al1, ps1);
      if (__any_sync(FULL, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          o[j][0] *= al0;
          o[j][1] *= al0;
          o[j][2] *= al1;
          o[j][3] *= al1;
        }
      }
      // ---- O += (p t_V) . V-hat: weights as one f16 each (the A fragments of two k-steps of 16
      //      tokens), V-hat hi and lo through ldmatrix.trans
      uint32_t pa[2][4];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int ta = 16 * kk + 2 * tq, tb2 = ta + 8;
        const float va0 = T.tv[ta], va1 = T.tv[ta + 1], vb0 = T.tv[tb2], vb1 = T.tv[tb2 + 1];
        pa[kk][0] = h2u(__floats2half2_rn(p[2 * kk][0] * va0, p[2 * kk][1] * va1));
        pa[kk][1] = h2u(__floats2half2_rn(p[2 * kk][2] * va0, p[2 * kk][3] * va1));
        pa[kk][2] = h2u(__floats2half2_rn(p[2 * kk + 1][0] * vb0, p[2 * kk + 1][1] * vb1));
        pa[kk][3] = h2u(__floats2half2_rn(p[2 * kk + 1][2] * vb0, p[2 * kk + 1][3] * vb1));
      }
      // B (trans): lanes 0-7 / 8-15 / 16-23 / 24-31 address rows (tokens 16 kk + 0..7, channels
      // 8 j .. 8 j + 7), (tokens 16 kk + 8.., 8 j ..), (tokens 16 kk + 0..7, 8 (j + 1) ..),
      // (tokens 16 kk + 8.., 8 (j + 1) ..)
      const int vrow = (lane & 7) + 8 * ((lane >> 3) & 1), vcol = 8 * (lane >> 4);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) {  // pairs of 8-channel n-tiles
          uint32_t vh[4], vl[4];
          ldsm_x4_t(vh, &T.vt[0][(16 * kk + vrow) * TS + 16 * jp + vcol]);
          ldsm_x4_t(vl, &T.vt[1][(16 * kk + vrow) * TS + 16 * jp + vcol]);
          mma16(o[2 * jp], pa[kk], vh[0], vh[1]);
          mma16(o[2 * jp], pa[kk], vl[0], vl[1]);
          mma16(o[2 * jp + 1], pa[kk], vh[2], vh[3]);
          mma16(o[2 * jp + 1], pa[kk], vl[2], vl[3]);
        }
      }
    }
    // done with tile buffer tb (the producers wait for it only before chunk c + 2)
    if (c + 2 < nch) bar_arrive(BAR_EMPTY + tb, NT);
  }
  if (kvarn_v && active && cur_vpage >= 0) {
#pragma unroll
    for (int jn = 0; jn < 16; ++jn)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float cj = __half2float(S.cv[cur_vpage & 1][8 * jn + 2 * tq + e]);
        o[jn][e] *= cj;
        o[jn][2 + e] *= cj;
      }
  }

  // ---- this split's record of rows r0 and r1: m, l (summed over the 4 lanes of a row), acc
  l0 += __shfl_xor_sync(FULL, l0, 1);
  l0 += __shfl_xor_sync(FULL, l0, 2);
  l1 += __shfl_xor_sync(FULL, l1, 1);
  l1 += __shfl_xor_sync(FULL, l1, 2);
  if (!active) return;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = half ? r1 : r0;
    if (row >= R) continue;
    const int qi = row / G, hd = row % G;
    float *rec = A.ws + ((((int64_t)qi * A.hkv + head) * nspl + sp) * G + hd) * PSTRIDE;
    if (tq == 0) {
      rec[0] = half ? m1 : m0;
      rec[1] = half ? l1 : l0;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      *reinterpret_cast<float2 *>(rec + 4 + 8 * j + 2 * tq) = make_float2(o[j][2 * half], o[j][2 * half + 1]);
  }
}

// One warp per (query token, query head): LSE merge of the splits of its KV head, quantized
// splits (rotated basis for kvarn V) and tail splits apart, the inverse rotation, the output.
__global__ void __launch_bounds__(256) k_chunk_merge(CArgs A, float *out) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int hq = A.hkv * A.G;
  if (wid >= (int64_t)A.nq * hq) return;
  const int qi = (int)(wid / hq), h = (int)(wid % hq);
  const int head = h / A.G, hd = h % A.G;
  const int nspl = A.nsq + A.nst;
  const float *rec0 = A.ws + (((int64_t)qi * A.hkv + head) * nspl * A.G + hd) * PSTRIDE;
  const int64_t rs = (int64_t)A.G * PSTRIDE;  // stride between splits
  float mk[2], lk[2], M = -INFINITY;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int k = lane + 32 * u;
    mk[u] = k < nspl ? rec0[k * rs] : -INFINITY;
    lk[u] = k < nspl ? rec0[k * rs + 1] : 0.f;
    M = fmaxf(M, mk[u]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o));
  float fk[2], ls = 0.f;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    fk[u] = mk[u] == -INFINITY ? 0.f : exp2_fast(mk[u] - M);
    ls = fmaf(fk[u], lk[u], ls);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(FULL, ls, o);
  // sums of f_k acc_k over the quantized splits (stored basis) and the tail splits apart
  auto wsum = [&](int kb, int ke, float (&t)[4]) {
    for (int k = kb; k < ke; ++k) {
      const float f = __shfl_sync(FULL, (k >> 5) ? fk[1] : fk[0], k & 31);
      const float4 v = *reinterpret_cast<const float4 *>(rec0 + k * rs + 4 + 4 * lane);
      t[0] = fmaf(f, v.x, t[0]);
      t[1] = fmaf(f, v.y, t[1]);
      t[2] = fmaf(f, v.z, t[2]);
      t[3] = fmaf(f, v.w, t[3]);
    }
  };
  float sr[4] = {0.f, 0.f, 0.f, 0.f}, st[4] = {0.f, 0.f, 0.f, 0.f};
  wsum(0, A.nsq, sr);
  wsum(A.nsq, nspl, st);
  if (A.rotv) {
    warp_wht(sr, lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) sr[e] *= kKappa();
  }
  const float inv = ls > 0.f ? 1.0f / ls : 0.f;
  *reinterpret_cast<float4 *>(out + ((int64_t)qi * hq + h) * D + 4 * lane) =
      make_float4((sr[0] + st[0]) * inv, (sr[1] + st[1]) * inv, (sr[2] + st[2]) * inv, (sr[3] + st[3]) * inv);
}

}  // namespace

size_t chunk_workspace_bytes(const kvq_cache *c, int n_q_tokens, int n_q_heads) {
  const int G = n_q_heads / c->p.n_kv_heads;
  return sizeof(float) * (size_t)std::min(std::max(n_q_tokens, 1), NQ) * c->p.n_kv_heads * MAXSPL * G * PSTRIDE;
}

int launch_chunk(const kvq_cache *c, int layer, int seq, int n_q, int n_q_heads, const float *q, float scale,
                 float *out, void *ws, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem)) != cudaSuccess)
      return KVQ_E_CUDA;
    attr = true;
  }
  const LayerView L = layer_view(c, layer);
  const int hkv = c->p.n_kv_heads, G = n_q_heads / hkv;
  const int64_t n = c->len[(size_t)layer * c->p.n_seqs + seq];
  const int64_t Q = quantized_len(c, n);
  const int per_launch = std::max(1, std::min(NQ, MAXR / G));  // query tokens per launch
  for (int q0 = 0; q0 < n_q; q0 += per_launch) {
    const int nq = std::min(per_launch, n_q - q0);
    CArgs A{};
    A.seq = seq;
    A.nq = nq;
    A.G = G;
    A.hkv = hkv;
    A.rotk = c->fam_k == FAM_KVARN;
    A.rotv = c->fam_v == FAM_KVARN;
    A.fam_k = c->fam_k;
    A.bits_k = c->bits_k;
    A.fam_v = c->fam_v;
    A.bits_v = c->bits_v;
    // the rows of this launch are query tokens q0 .. q0 + nq - 1 of the chunk: their context is
    // the sequence cut after the last of them
    A.n = n - (n_q - q0 - nq);
    A.Q = std::min(Q, A.n);
    A.qscale = scale * LOG2E;
    A.q = q + (size_t)q0 * n_q_heads * D;
    A.ws = static_cast<float *>(ws);
    // splits: about one CTA per SM over the KV heads, quantized and 16-bit tokens in proportion
    // to their chunks, at least one split for each part that has tokens, at most MAXSPL in all
    const int64_t chq = (A.Q + CH - 1) / CH, cht = (A.n - A.Q + CH - 1) / CH;
    const int budget = std::max(1, std::min(MAXSPL, c->num_sms / hkv));
    const int need_t = cht > 0 ? 1 : 0;
    int nsq = 0, nst = 0;
    if (chq > 0) {
      const int64_t share = (budget * chq + (chq + cht) / 2) / (chq + cht);
      nsq = (int)std::max<int64_t>(1, std::min<int64_t>({share, chq, (int64_t)(budget - need_t)}));
    }
    if (cht > 0) nst = (int)std::max<int64_t>(1, std::min<int64_t>(cht, budget - nsq));
    if (nsq + nst == 0) nst = 1;
    A.cps_q = nsq ? (int)((chq + nsq - 1) / nsq) : 1;
    A.nsq = nsq ? (int)((chq + A.cps_q - 1) / A.cps_q) : 0;
    A.cps_t = nst ? (int)((cht + nst - 1) / nst) : 1;
    A.nst = nst ? (int)((cht + A.cps_t - 1) / A.cps_t) : 0;
    if (A.nsq + A.nst == 0) A.nst = 1;
    k_chunk<<<(unsigned)(hkv * (A.nsq + A.nst)), NT, sizeof(Smem), st>>>(L, A);
    if (cudaGetLastError() != cudaSuccess) return KVQ_E_CUDA;
    const int64_t warps = (int64_t)nq * n_q_heads;
    k_chunk_merge<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(A, out + (size_t)q0 * n_q_heads * D);
    if (cudaGetLastError() != cudaSuccess) return KVQ_E_CUDA;
    note_launches(2);
  }
  return KVQ_OK;
}

}  // namespace kvq
