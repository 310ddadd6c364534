// kvq_decode.cu - split-K decode attention over [quantized prefix | BF16 tail].
//
// Pages: "Fork of beellama and kvarn KV quants at long context" (ai-manual.ru), the
// decode discussion: at long context depth decode is memory bound and the dequantization
// inside attention decides the speed; "KV Cache Precision Tail" of the BeeLLama.cpp
// v0.4.0 page: the newest tokens are read exactly from BF16.
//
// Per (sequence, KV head) the context is cut into splits; one CTA per split computes the
// online-softmax state (m, l, acc) of its G query heads, the last CTA to finish (an atomic
// ticket, no waiting) merges the splits.  For kvarn K the query is rotated once
// (q' = H.q.kappa) and scaled per 256-token page by the channel scales c, so the keys are
// never rotated back; for kvarn V the accumulator stays in the rotated basis and the
// inverse rotation is applied once per head in the merge.
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>
#include <cstddef>

#include "kvq_codes.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int CH = 32;       // tokens per chunk (one per lane)
constexpr int MAXSQ = 48;    // max splits over the quantized prefix per (seq, head)
constexpr int MAXST = 16;    // max splits over the tail per (seq, head)
constexpr int MAXSPL = MAXSQ + MAXST;
constexpr int PSTRIDE = 4 + D;  // floats per partial: m, l, 2 pad, acc[128] (16-byte records)
constexpr int PACC = 4;         // offset of acc in a partial
constexpr int MAXS = kDecodeEntriesPerLaunch;  // decode entries (query rows) per launch
constexpr float LOG2E = 1.4426950408889634f;

struct DSeq {
  int32_t seq, row;     // cache slot; row of q / out
  int32_t nsq, nst;     // splits per head over the quantized prefix / the tail
  int32_t cps_q, cps_t; // chunks per split
  int32_t cta0;         // first CTA of this sequence
  int32_t part0;        // first partial slot of this sequence
  int64_t n, Q;
  int64_t qa;           // the uniform quantized splits cover [0, qa); a last split covers [qa, Q)
  int64_t dq, dt;       // first quantized token / ring token written by the preceding kernel
};

// Waits for the kernel this one was launched behind (programmatic stream serialization) and
// for its memory writes; returns at once when the launch had no such dependency.
__device__ __forceinline__ void wait_producer() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// First chunk of a range starting at token a whose tokens reach `dirty` (chunks of CH tokens).
__device__ __forceinline__ int64_t first_dirty_chunk(int64_t a, int64_t dirty) {
  return dirty <= a ? 0 : (dirty - a) / CH;
}

// Decode modes.  M_FUSED: Q.K and P.V of one cache type in one kernel.  K and V of different
// types take two kernels over the same split plan: M_SCORES (the K type) writes the masked
// Q.K scores of the quantized prefix to the workspace, M_PVEXT (the V type) reads them back
// for the softmax and P.V (and runs the BF16 tail splits and the merge as M_FUSED does).
enum DecodeMode { M_FUSED = 0, M_SCORES = 1, M_PVEXT = 2 };

// Where one (entry, KV head) keeps its scores: head slot g at row0 + g * qcap, token i at +i.
struct ScoreRow {
  float *row0;
  int64_t qcap;
};

struct DArgs {
  int32_t nseq, G, hkv, rotk, rotv, ncta;
  float qscale;  // softmax scale * log2(e)
  const float *q;
  float *out;
  float *ws;
  uint32_t *tickets;
  float *scores;   // M_SCORES / M_PVEXT: [entry][KV head][G][qcap] fp32
  int64_t qcap;    // tokens per score row (max_ctx rounded up to a chunk)
  DSeq s[MAXS];
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

// ---- tensor-core pieces (mma.sync m16n8k32, s8 x s8 -> s32) ---------------------------
//
// Fragment layout (groupID g = lane/4, thread-in-group tq = lane%4):
//   A 16x32: a0 = (row g, k 4tq..4tq+3), a1 = (row g+8, same k), a2 = (row g, k 16+4tq..),
//            a3 = (row g+8, k 16+4tq..);  B 32x8: b0 = (k 4tq.., col g), b1 = (k 16+4tq.., col g);
//   C 16x8: c0 = (row g, col 2tq), c1 = (g, 2tq+1), c2 = (g+8, 2tq), c3 = (g+8, 2tq+1).
// Rows 0..7 carry the high int8 limb and rows 8..15 the low limb of a 16-bit fixed-point
// operand of query head g (Q for Q.K, the softmax weights for P.V); the two int32 results of
// one column combine as 256*hi + lo with one fp32 rounding.

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: two lanes per instruction, each lane
//      rounded once exactly as the scalar operation) ----------------------------------------
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pk2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ float acc_part(f32x2 v, int e) {
  float lo, hi;
  upk2(v, lo, hi);
  return e ? hi : lo;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// One block of Q.K or P.V on the tensor cores with its epilogue on packed fp32:
//   x += f * (256 * hi + lo)
// for the two columns of this lane (c0/c2 = hi/lo of column 2tq, c1/c3 = hi/lo of column
// 2tq+1).  The int32 sums (|value| < 2^22) convert to fp32 exactly.
__device__ __forceinline__ void mma_s8_fold(f32x2 &x, const uint32_t (&a)[4], uint32_t b0, uint32_t b1, f32x2 f) {
  const f32x2 k256 = 0x4380000043800000ull;  // (256, 256)
  asm("{\n"
      " .reg .b32 c0, c1, c2, c3;\n"
      " .reg .f32 h0, h1, l0, l1;\n"
      " .reg .b64 h, l;\n"
      " mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {c0,c1,c2,c3}, {%1,%2,%3,%4}, {%5,%6}, "
      "{%7,%7,%7,%7};\n"
      " cvt.rn.f32.s32 h0, c0;\n cvt.rn.f32.s32 h1, c1;\n cvt.rn.f32.s32 l0, c2;\n cvt.rn.f32.s32 l1, c3;\n"
      " mov.b64 h, {h0, h1};\n"
      " mov.b64 l, {l0, l1};\n"
      " fma.rn.f32x2 h, h, %8, l;\n"
      " fma.rn.f32x2 %0, %9, h, %0;\n"
      "}\n"
      : "+l"(x)
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0), "l"(k256), "l"(f));
}

__device__ __forceinline__ void mma_s8_fold3(f32x2 &x, const uint32_t (&a)[4], const uint32_t (&a3)[2], uint32_t b0,
                                             uint32_t b1, f32x2 f) {
  const f32x2 k256 = 0x4380000043800000ull;  // (256, 256)
  const f32x2 k254 = 0x3B8102043B810204ull;  // (1/254, 1/254) rounded to fp32
  asm("{\n"
      " .reg .b32 c0, c1, c2, c3, e0, e1, e2, e3;\n"
      " .reg .f32 h0, h1, l0, l1, m0, m1;\n"
      " .reg .b64 h, l, m;\n"
      " mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {c0,c1,c2,c3}, {%1,%2,%3,%4}, {%7,%8}, "
      "{%9,%9,%9,%9};\n"
      " mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {e0,e1,e2,e3}, {%5,%9,%6,%9}, {%7,%8}, "
      "{%9,%9,%9,%9};\n"
      " cvt.rn.f32.s32 h0, c0;\n cvt.rn.f32.s32 h1, c1;\n cvt.rn.f32.s32 l0, c2;\n cvt.rn.f32.s32 l1, c3;\n"
      " cvt.rn.f32.s32 m0, e0;\n cvt.rn.f32.s32 m1, e1;\n"
      " mov.b64 h, {h0, h1};\n"
      " mov.b64 l, {l0, l1};\n"
      " mov.b64 m, {m0, m1};\n"
      " fma.rn.f32x2 h, h, %10, l;\n"
      " fma.rn.f32x2 h, m, %12, h;\n"
      " fma.rn.f32x2 %0, %11, h, %0;\n"
      "}\n"
      : "+l"(x)
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a3[0]), "r"(a3[1]), "r"(b0), "r"(b1), "r"(0),
        "l"(k256), "l"(f), "l"(k254));
}

// field s (width W) of each byte of `word`, moved to bits [P, P+W) of the same byte
template <int W, int P>
__device__ __forceinline__ uint32_t xplane(uint32_t word, int s) {
  constexpr uint32_t M1 = ((1u << W) - 1u) << P;
  constexpr uint32_t M = M1 | (M1 << 8) | (M1 << 16) | (M1 << 24);
  return __funnelshift_l(word, word, (P - s * W) & 31) & M;
}

__device__ __forceinline__ uint32_t wsel(const uint4 &v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

__device__ __forceinline__ uint4 ld16(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }

// K codes of one token, as the B fragment of block blk: reg e holds channels
// 32 blk + 8 tq + 4 e + (0..3) as bytes code * 2^(8-b) (signed) or (u - 2^(b-1)) * 2^(8-b).
template <int FAM, int BITS>
struct KTok {
  static constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  uint4 l0, l1, h0;
  __device__ __forceinline__ void load(const uint8_t *tok, int tq) {
    if constexpr (WL == 8) {
      l0 = ld16(tok + 32 * tq);
      l1 = ld16(tok + 32 * tq + 16);
    } else if constexpr (WL == 4) {
      l0 = ld16(tok + 16 * tq);
    } else {
      l0 = ld16(tok + 16 * (tq >> 1));
    }
    if constexpr (WH == 1) h0 = ld16(tok + 16 * WL);
    if constexpr (WH == 2) h0 = ld16(tok + 16 * WL + 16 * (tq >> 1));
  }
  __device__ __forceinline__ void frag(int blk, int tq, uint32_t &b0, uint32_t &b1) const {
    constexpr int PL = 8 - BITS;
    const uint32_t w0 = wsel(l0, blk);
    if constexpr (WL == 8) {
      b0 = w0;
      b1 = wsel(l1, blk);
    } else if constexpr (WL == 4) {
      b0 = xplane<4, PL>(w0, 0);
      b1 = xplane<4, PL>(w0, 1);
    } else {
      const int s0 = (2 * tq) & 3;
      b0 = xplane<2, PL>(w0, s0);
      b1 = xplane<2, PL>(w0, s0 + 1);
    }
    if constexpr (WH > 0) {
      constexpr int PH = 8 - BITS + WL, FH = 8 / WH;
      const uint32_t wh = wsel(h0, blk);
      const int s0 = (2 * tq) % FH;
      b0 |= xplane<WH, PH>(wh, s0);
      b1 |= xplane<WH, PH>(wh, s0 + 1);
    }
    if constexpr (FAM == FAM_ASYM) {
      b0 ^= 0x80808080u;
      b1 ^= 0x80808080u;
    }
  }
};

// V codes of one quad and one block, as B fragments for channels 32 blk + 4 g + u (u = 0..3):
// byte k = quad token k.
template <int FAM, int BITS>
struct VQuad {
  static constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  uint4 l;
  uint32_t h;
  __device__ __forceinline__ void load(const uint8_t *quad, int blk, int g) {
    if constexpr (WL == 8) {
      l = ld16(quad + 128 * blk + 16 * g);
    } else if constexpr (WL == 4) {
      const uint2 t = *reinterpret_cast<const uint2 *>(quad + 64 * blk + 8 * g);
      l.x = t.x;
      l.y = t.y;
    } else {
      l.x = *reinterpret_cast<const uint32_t *>(quad + 32 * blk + 4 * g);
    }
    if constexpr (WH == 1) h = *reinterpret_cast<const uint32_t *>(quad + 64 * WL + 16 * blk + 4 * (g >> 1));
    if constexpr (WH == 2) h = *reinterpret_cast<const uint32_t *>(quad + 64 * WL + 32 * blk + 4 * g);
  }
  __device__ __forceinline__ uint32_t frag(int u, int g) const {
    constexpr int PL = 8 - BITS;
    uint32_t r;
    if constexpr (WL == 8)
      r = wsel(l, u);
    else if constexpr (WL == 4)
      r = xplane<4, PL>(u < 2 ? l.x : l.y, u & 1);
    else
      r = xplane<2, PL>(l.x, u);
    if constexpr (WH == 1) r |= xplane<1, 8 - BITS + WL>(h, 4 * (g & 1) + u);
    if constexpr (WH == 2) r |= xplane<2, 8 - BITS + WL>(h, u);
    if constexpr (FAM == FAM_ASYM) r ^= 0x80808080u;
    return r;
  }
};

__device__ __forceinline__ float h2f(const __half *p, int i) { return __half2float(p[i]); }

// 1/x by the MUFU unit (about 1 ulp): used only for fixed-point normalizers, where
// QFIX * rcp(max) keeps every scaled value within 16 bits (QFIX = 32639 leaves the margin)
__device__ __forceinline__ float rcp_fast(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max over the warp of a non-negative float (its bits order like unsigned integers)
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(v)));
}

// 16-byte global -> shared copy issued only where pred holds (no branch)
__device__ __forceinline__ void cp_async16_if(void *dst, const void *src, bool pred);

// 2^x by the MUFU unit (flushes results below 2^-126 to 0: negligible softmax weights)
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float QFIX = 32639.0f;              // 16-bit fixed point: 256*127 + 127
constexpr float MAGIC = 12582912.0f + 128.0f;  // 1.5*2^23 (+128 offset for the limb split)

// ---- staging (one pipeline per warp) ---------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy through L2 (no register staging), tracked by commit groups
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16_if(void *dst, const void *src, bool pred) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %2, 0;\n @p cp.async.cg.shared.global [%0], [%1], 16;\n}\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"((int)pred)
      : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Shared-memory image of one 32-token chunk of a quantized page (both K and V), filled by
// cp.async: codes of K, codes of V one quad per row with a 32-byte pad (so that the lanes
// of one P.V fragment load hit distinct banks), then the fp16 scales (d of K then V; m of K
// then V for qb_1; t of K then V for kvarn).
template <int FAM, int BITS>
struct Stage {
  static constexpr int QS = 64 * BITS + 32;  // padded quad stride
  static constexpr int KC = 0;
  static constexpr int VC = KC + 512 * BITS;
  static constexpr int KD = VC + 8 * QS;
  static constexpr int VD = KD + 256;
  static constexpr int KM = VD + 256;
  static constexpr int VM = KM + (FAM == FAM_ASYM ? 256 : 0);
  static constexpr int KT = VM + (FAM == FAM_ASYM ? 256 : 0);
  static constexpr int VT = KT + (FAM == FAM_KVARN ? 64 : 0);
  static constexpr int BYTES = VT + (FAM == FAM_KVARN ? 64 : 0);
  static constexpr int NST = BITS <= 3 ? 3 : 2;  // stages per warp
};

// Per-warp data of whole pages (kvarn): the channel scales c of K and V of the pages being
// copied (double-buffered by page parity: copies run at most NST - 1 chunks ahead of the
// compute, so they never reach a third page), and the V channel scales of the page being
// computed as the fp32 pairs each lane's P.V columns need.
struct PageArea {
  __half c[2][2][D];  // [page & 1][K, V][channel]
  float2 fv[4][16];   // [tq][blk * 4 + u] = (c_V[32 blk + 8 tq + u], c_V[32 blk + 8 tq + 4 + u])
};

// Source cursor of a warp's copies: the K and V sub-pages of the page being copied, looked up
// in the page table once per page.
struct PageCursor {
  int64_t page = -1;
  const uint8_t *sk = nullptr, *sv = nullptr;
  __device__ __forceinline__ bool seek(const LayerView &L, int seq, int head, int64_t p) {
    if (p == page) return false;
    page = p;
    sk = subpage_ptr(L, seq, p, head, 0);
    sv = sk + L.sub_k;
    return true;
  }
};

// Copies chunk [i0, i0+32) (K and V codes and fp16 scales; for kvarn, on the first chunk of a
// page, the page's channel scales) into the stage `st`, 16 bytes per lane and instruction, as
// one commit group.
template <int FAM, int BITS, int MODE>
__device__ __forceinline__ void copy_chunk(const LayerView &L, int seq, int head, int64_t i0, uint8_t *st, int lane,
                                           PageCursor &pc, PageArea *pa, const ScoreRow &sr, int G) {
  using S = Stage<FAM, BITS>;
  const SubLayout lay = sub_layout(FAM, BITS);
  const int64_t page = i0 / GROUP;
  // the K half (lanes 0..15 for scale pieces) is copied unless the scores come precomputed,
  // the V half (lanes 16..31) unless only scores are computed
  constexpr bool KSIDE = MODE != M_PVEXT, VSIDE = MODE != M_SCORES;
  const bool mine = lane < 16 ? KSIDE : VSIDE;
  if (pc.seek(L, seq, head, page) && FAM == FAM_KVARN)
    cp_async16_if(&pa->c[page & 1][lane >> 4][8 * (lane & 15)], (lane < 16 ? pc.sk : pc.sv) + lay.c + 16 * (lane & 15),
                  mine);
  const int tip0 = (int)(i0 % GROUP);
  constexpr int KP = 32 * BITS;  // 16-byte pieces of K codes (and of V codes)
  constexpr int QP = 4 * BITS;   // pieces per V quad
  // K and V codes of the chunk are contiguous (tip0 is a multiple of 4: V quads are whole)
  const uint8_t *kc = pc.sk + tip0 * 16 * BITS + 16 * lane;
  const uint8_t *vc = pc.sv + tip0 * 16 * BITS + 16 * lane;
  if constexpr (MODE == M_PVEXT) {
    // the chunk's scores, head slot g < G: 32 floats = 8 pieces each, into the K code area
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int p = lane + 32 * j, gg = p >> 3, pc8 = p & 7;
      cp_async16_if(st + S::KC + 128 * gg + 16 * pc8, sr.row0 + gg * sr.qcap + i0 + 4 * pc8, gg < G);
    }
  }
  if constexpr (KSIDE) {
#pragma unroll
    for (int j = 0; j < KP / 32; ++j) cp_async16(st + S::KC + 16 * lane + 512 * j, kc + 512 * j);
  }
  if constexpr (!VSIDE) {
  } else if constexpr (32 % QP == 0) {
    uint8_t *vd = st + S::VC + (lane / QP) * S::QS + 16 * (lane % QP);
#pragma unroll
    for (int j = 0; j < KP / 32; ++j) cp_async16(vd + j * (32 / QP) * S::QS, vc + 512 * j);
  } else {
#pragma unroll
    for (int j = 0; j < KP / 32; ++j) {
      const int p = lane + 32 * j, q = p / QP, o = p % QP;
      cp_async16(st + S::VC + q * S::QS + 16 * o, vc + 512 * j);
    }
  }
  // fp16 scales: d (and m for qb_1) of K in lanes 0..15, of V in lanes 16..31; t of K in lanes
  // 0..3, of V in lanes 4..7 (kvarn)
  const uint8_t *sb = (lane < 16 ? pc.sk : pc.sv) + tip0 * 8 + 16 * (lane & 15);
  cp_async16_if(st + S::KD + 16 * lane, sb + lay.d, mine);
  if constexpr (FAM == FAM_ASYM) cp_async16_if(st + S::KM + 16 * lane, sb + lay.m, mine);
  if constexpr (FAM == FAM_KVARN) {
    const bool tmine = (lane & 4) ? VSIDE : KSIDE;
    cp_async16_if(st + S::KT + 16 * (lane & 7), (lane & 4 ? pc.sv : pc.sk) + lay.t + tip0 * 2 + 16 * (lane & 3),
                  lane < 8 && tmine);
  }
}

// Per-warp scale tables of one chunk, built with one token per lane.
template <int FAM>
struct alignas(16) ChunkTabs {
  static constexpr int NM = FAM == FAM_ASYM ? CH : 1;
  // (read with 8- and 16-byte vector loads: each member starts on 16 bytes)
  alignas(16) float k[CH / 2][4][2];  // K: d * t (kvarn) or d, per token pair, block, token (0 past the end)
  alignas(16) float v[4][CH];  // V: t * d * QFIX / max over the chunk (per block) -> weights in fixed point
  alignas(16) float km[NM][4];  // qb_1 K: m + d * 2^(b-1)
  alignas(16) float vm[NM][4];  // qb_1 V: m + d * 2^(b-1)
};


// Query fragments of one page: the query of head g times the page's K channel scales c
// (kvarn), in 16-bit fixed point relative to the head's max, split into int8 limbs (hi in
// rows 0..7, lo in rows 8..15 of the MMA A operand; lane (g, tq) holds channels
// 32 blk + 8 tq + (0..7)).  sigp undoes the fixed point and the codes' byte position.
struct QFrag {
  uint32_t qa[4][4];
  uint32_t qa3[4][2];  // third limb: round(254 x the residual of the 16-bit value), rows 0..7
  float sigp;
  float qs[4];  // qb_1: the query summed over each block
};

template <int FAM, int BITS>
__device__ __forceinline__ void make_qfrag(QFrag &f, const float (*qrot)[D], const __half *ck, int g, int tq,
                                           bool hv) {
  constexpr float SCL = (float)(1 << BITS) / 256.0f / QFIX;
  float qv[32], amax = 0.f;
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    const float4 q0 = *reinterpret_cast<const float4 *>(&qrot[g][32 * blk + 8 * tq]);
    const float4 q1 = *reinterpret_cast<const float4 *>(&qrot[g][32 * blk + 8 * tq + 4]);
    const float qq[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    float cc[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
    if constexpr (FAM == FAM_KVARN) {
      const uint4 c8 = *reinterpret_cast<const uint4 *>(ck + 32 * blk + 8 * tq);
      const __half2 *c2 = reinterpret_cast<const __half2 *>(&c8);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 cf = __half22float2(c2[u]);
        cc[2 * u] = cf.x;
        cc[2 * u + 1] = cf.y;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = hv ? qq[i] * cc[i] : 0.f;
      qv[blk * 8 + i] = v;
      amax = fmaxf(amax, fabsf(v));
    }
  }
  amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
  const float inv = amax > 0.f ? QFIX * rcp_fast(amax) : 0.f;
  f.sigp = amax * SCL;
  // x * inv rounded to an integer by one FFMA with 1.5 * 2^23 + 128: the float's low bytes
  // are (qi + 128) mod 2^16, whose byte 1 is the hi limb and byte 0 (with bit 7 flipped) the lo
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w[4], z[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float xv = qv[blk * 8 + 4 * h + i];
        const float qsum = fmaf(xv, inv, MAGIC);
        w[i] = __float_as_uint(qsum);
        // residual of the rounding, |r| <= 1/2, to 8 more bits: round(254 r) in [-127, 127]
        const float r = fmaf(xv, inv, MAGIC - qsum);
        z[i] = __float_as_uint(fmaf(r, 254.0f, MAGIC));
      }
      const uint32_t x = __byte_perm(w[0], w[1], 0x5140), y = __byte_perm(w[2], w[3], 0x5140);
      f.qa[blk][2 * h] = __byte_perm(x, y, 0x7632);
      f.qa[blk][2 * h + 1] = __byte_perm(x, y, 0x5410) ^ 0x80808080u;
      f.qa3[blk][h] = __byte_perm(__byte_perm(z[0], z[1], 0x0040), __byte_perm(z[2], z[3], 0x0040), 0x5410) ^ 0x80808080u;
    }
    if constexpr (FAM == FAM_ASYM) {
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += qv[blk * 8 + i];
      sum += __shfl_xor_sync(FULL, sum, 1);
      sum += __shfl_xor_sync(FULL, sum, 2);
      f.qs[blk] = sum;
    }
  }
}

// Issues the first NST - 1 chunks of a warp's range [c0, c1) (one commit group each, empty
// groups past the end), so that their copies overlap the query prologue.
template <int FAM, int BITS, int MODE>
__device__ __forceinline__ void warp_quant_prefetch(const LayerView &L, int seq, int head, int64_t a, int c0, int c1,
                                                    int64_t cdirty, bool &waited, uint8_t *stages, int lane,
                                                    PageCursor &pc, PageArea *pa, const ScoreRow &sr, int G) {
  using S = Stage<FAM, BITS>;
#pragma unroll
  for (int j = 0; j < S::NST - 1; ++j) {
    if (c0 + j < c1) {
      if (c0 + j >= cdirty && !waited) {
        wait_producer();
        waited = true;
      }
      copy_chunk<FAM, BITS, MODE>(L, seq, head, a + (int64_t)(c0 + j) * CH, stages + j * S::BYTES, lane, pc, pa, sr,
                                  G);
    }
    cp_async_commit();
  }
}

// Q.K and P.V of one warp over its chunks [c0, c1) of a quantized split [a, b) (consecutive, so
// pages change rarely).  Writes the warp's online-softmax state (m, l and the accumulator in the
// stored basis) of its heads to shared memory.  M_SCORES stops after Q.K and writes the scores
// to sr instead; M_PVEXT reads them from sr in place of Q.K.
template <int FAM, int BITS, int MODE>
__device__ __forceinline__ void warp_quant(const LayerView &L, int seq, int head, int64_t a, int64_t b, int c0,
                                           int c1, int64_t cdirty, bool waited, int G, const float (*qrot)[D],
                                           uint8_t *stages, ChunkTabs<FAM> &T, float *mw, float *lw, float *accw,
                                           PageCursor &pc, PageArea *pa, const ScoreRow &sr) {
  using S = Stage<FAM, BITS>;
  constexpr bool KSIDE = MODE != M_PVEXT, VSIDE = MODE != M_SCORES;
  static_assert(S::KC + MAX_G * CH * 4 <= S::VC || MODE != M_PVEXT, "the K code area holds a chunk's scores");
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const bool hv = g < G;
  constexpr float CSC = (float)(1 << (BITS)) / 256.0f;  // 2^(b-8): undoes the code's byte position
  constexpr float HALF_RANGE = (float)(1 << (BITS - 1));
  constexpr float SCL = CSC / QFIX;

  f32x2 acc[16];  // index blk*4 + u <-> channels (32 blk + 8 tq + u, 32 blk + 8 tq + 4 + u)
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0ull;
  float aoff[4] = {0.f, 0.f, 0.f, 0.f};
  float m_run = -INFINITY, l_run = 0.f;
  QFrag qf;
  int cur_page = -1;

  int si = 0;  // stage of chunk c
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    {  // keep NST - 1 chunks in flight: issue chunk c + NST - 1 into the stage read last round
      const int cn = c + S::NST - 1;
      const int sn = si == 0 ? S::NST - 1 : si - 1;
      if (cn < c1) {
        if (cn >= cdirty && !waited) {
          wait_producer();
          waited = true;
        }
        copy_chunk<FAM, BITS, MODE>(L, seq, head, a + (int64_t)cn * CH, stages + sn * S::BYTES, lane, pc, pa, sr, G);
      }
      cp_async_commit();
      cp_async_wait<S::NST - 1>();  // chunk c has landed (for this lane's copies)
      __syncwarp();                 // ... and for every lane's
      uint8_t *st = stages + si * S::BYTES;
      si = si + 1 == S::NST ? 0 : si + 1;
      const int64_t i0 = a + (int64_t)c * CH;
      const int page = (int)(i0 / GROUP);
      const int nvalid = (int)((b - i0) < CH ? (b - i0) : CH);
      if (page != cur_page && (FAM == FAM_KVARN || cur_page < 0)) {
        const __half *ck = FAM == FAM_KVARN ? pa->c[page & 1][0] : nullptr;
        if constexpr (KSIDE) make_qfrag<FAM, BITS>(qf, qrot, ck, g, tq, hv);
        if constexpr (FAM == FAM_KVARN && VSIDE) {
          // lane l builds pairs 2 (l >> 2) and 2 (l >> 2) + 1 of column set tq' = l & 3
          const __half *cv = pa->c[page & 1][1];
          const int tl = lane & 3;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int idx = 2 * (lane >> 2) + e, blk = idx >> 2, u = idx & 3;
            pa->fv[tl][idx] = make_float2(__half2float(cv[32 * blk + 8 * tl + u]), __half2float(cv[32 * blk + 8 * tl + 4 + u]));
          }
          __syncwarp();
        }
        cur_page = page;
      }
      const float sigp = qf.sigp;
    // ---- scale tables: lane = token of the chunk; rows past the end of the context may hold
    //      stale bytes and get zero scales, so they never reach a sum
    float scl[4];
    {
      const bool vl = lane < nvalid;
      if constexpr (KSIDE) {
        const uint2 dkr = *reinterpret_cast<const uint2 *>(st + S::KD + 8 * lane);
        const float2 dk01 = __half22float2(*reinterpret_cast<const __half2 *>(&dkr.x));
        const float2 dk23 = __half22float2(*reinterpret_cast<const __half2 *>(&dkr.y));
        const float tkl = FAM == FAM_KVARN ? h2f(reinterpret_cast<const __half *>(st + S::KT), lane) : 1.f;
        // select (not multiply) so that NaN bit patterns in stale rows cannot leak
        const float dkt[4] = {vl ? dk01.x * tkl : 0.f, vl ? dk01.y * tkl : 0.f, vl ? dk23.x * tkl : 0.f,
                              vl ? dk23.y * tkl : 0.f};
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) T.k[lane >> 1][blk][lane & 1] = dkt[blk];
        if constexpr (FAM == FAM_ASYM) {
          const uint2 mkr = *reinterpret_cast<const uint2 *>(st + S::KM + 8 * lane);
          const float2 mk01 = __half22float2(*reinterpret_cast<const __half2 *>(&mkr.x));
          const float2 mk23 = __half22float2(*reinterpret_cast<const __half2 *>(&mkr.y));
          *reinterpret_cast<float4 *>(&T.km[lane][0]) =
              make_float4(vl ? fmaf(dk01.x, HALF_RANGE, mk01.x) : 0.f, vl ? fmaf(dk01.y, HALF_RANGE, mk01.y) : 0.f,
                          vl ? fmaf(dk23.x, HALF_RANGE, mk23.x) : 0.f, vl ? fmaf(dk23.y, HALF_RANGE, mk23.y) : 0.f);
        }
      }
      if constexpr (VSIDE) {
        const uint2 dvr = *reinterpret_cast<const uint2 *>(st + S::VD + 8 * lane);
        const float2 dv01 = __half22float2(*reinterpret_cast<const __half2 *>(&dvr.x));
        const float2 dv23 = __half22float2(*reinterpret_cast<const __half2 *>(&dvr.y));
        const float tvl = FAM == FAM_KVARN ? h2f(reinterpret_cast<const __half *>(st + S::VT), lane) : 1.f;
        float tdv[4] = {vl ? dv01.x * tvl : 0.f, vl ? dv01.y * tvl : 0.f, vl ? dv23.x * tvl : 0.f,
                        vl ? dv23.y * tvl : 0.f};
        float inv[4];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const float mx = warp_max_nonneg(tdv[blk]);  // t, d >= 0
          inv[blk] = mx > 0.f ? QFIX * rcp_fast(mx) : 0.f;
          scl[blk] = mx * SCL;
        }
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) T.v[blk][lane] = tdv[blk] * inv[blk];
        if constexpr (FAM == FAM_ASYM) {
          const uint2 mvr = *reinterpret_cast<const uint2 *>(st + S::VM + 8 * lane);
          const float2 mv01 = __half22float2(*reinterpret_cast<const __half2 *>(&mvr.x));
          const float2 mv23 = __half22float2(*reinterpret_cast<const __half2 *>(&mvr.y));
          *reinterpret_cast<float4 *>(&T.vm[lane][0]) =
              make_float4(vl ? fmaf(dv01.x, HALF_RANGE, mv01.x) : 0.f, vl ? fmaf(dv01.y, HALF_RANGE, mv01.y) : 0.f,
                          vl ? fmaf(dv23.x, HALF_RANGE, mv23.x) : 0.f, vl ? fmaf(dv23.y, HALF_RANGE, mv23.y) : 0.f);
        }
      }
      __syncwarp();
    }

    // ---- Q.K: n-tile r, column n holds token 16(r>>1) + 4(n>>1) + 2(r&1) + (n&1), so that
    //      the lane ends with the scores of tokens 4tq+(0..3) and 16+4tq+(0..3)
    float sc[8];
    if constexpr (MODE == M_PVEXT) {
      // the stored scores of head g (0 for the empty head slots), tokens 4tq+(0..3) and 16+4tq+(0..3)
      const float *sg = reinterpret_cast<const float *>(st + S::KC) + g * CH;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 s0 = hv ? *reinterpret_cast<const float4 *>(sg + 4 * tq) : z;
      const float4 s1 = hv ? *reinterpret_cast<const float4 *>(sg + 16 + 4 * tq) : z;
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) sc[k] = 16 * (k >> 2) + 4 * tq + (k & 3) < nvalid ? sv[k] : -INFINITY;
    } else {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      KTok<FAM, BITS> kt;
      kt.load(st + S::KC + (16 * (r >> 1) + 4 * (g >> 1) + 2 * (r & 1) + (g & 1)) * 16 * BITS, tq);
      const int t0 = 16 * (r >> 1) + 4 * tq + 2 * (r & 1);
      // (d of token t0, d of token t0 + 1) per block, as packed pairs
      const f32x2 *dp = reinterpret_cast<const f32x2 *>(&T.k[t0 >> 1][0][0]);
      f32x2 x = 0ull;
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t b0, b1;
        kt.frag(blk, tq, b0, b1);
        mma_s8_fold3(x, qf.qa[blk], qf.qa3[blk], b0, b1, dp[blk]);
      }
      float s0, s1;
      upk2(mul2(x, pk2(sigp, sigp)), s0, s1);
      if constexpr (FAM == FAM_ASYM) {
        const float4 mA = *reinterpret_cast<const float4 *>(&T.km[t0][0]);
        const float4 mB = *reinterpret_cast<const float4 *>(&T.km[t0 + 1][0]);
        s0 = fmaf(mA.x, qf.qs[0], fmaf(mA.y, qf.qs[1], fmaf(mA.z, qf.qs[2], fmaf(mA.w, qf.qs[3], s0))));
        s1 = fmaf(mB.x, qf.qs[0], fmaf(mB.y, qf.qs[1], fmaf(mB.z, qf.qs[2], fmaf(mB.w, qf.qs[3], s1))));
      }
      sc[2 * r] = t0 < nvalid ? s0 : -INFINITY;
      sc[2 * r + 1] = t0 + 1 < nvalid ? s1 : -INFINITY;
    }
    }
    if constexpr (MODE == M_SCORES) {
      if (hv) {
        float *dst = sr.row0 + g * sr.qcap + i0 + 4 * tq;
        *reinterpret_cast<float4 *>(dst) = make_float4(sc[0], sc[1], sc[2], sc[3]);
        *reinterpret_cast<float4 *>(dst + 16) = make_float4(sc[4], sc[5], sc[6], sc[7]);
      }
      __syncwarp();  // every lane is done with this stage before it is refilled next round
      continue;
    }

    // ---- online softmax (head g; the 4 lanes of a group hold the chunk's 32 tokens)
    float cmax = sc[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) cmax = fmaxf(cmax, sc[k]);
    cmax = fmaxf(cmax, __shfl_xor_sync(FULL, cmax, 1));
    cmax = fmaxf(cmax, __shfl_xor_sync(FULL, cmax, 2));
    // every chunk holds a valid token, so mn is finite and exp2(-inf) = 0 covers both the
    // first chunk (m_run = -inf) and the masked tokens
    const float mn = fmaxf(m_run, cmax);
    const float alpha = exp2_fast(m_run - mn);
    // the weights relative to the chunk's own largest one, pn = 2^(s - cmax) <= 1, so that
    // their 16-bit fixed point keeps its full range however far the chunk is below the
    // running max; pm = 2^(cmax - m) scales the chunk back (in l and in the P.V epilogue)
    const float pm = exp2_fast(cmax - mn);
    float p[8], psum = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      p[k] = exp2_fast(sc[k] - cmax);
      psum += p[k];
    }
    if (__any_sync(FULL, alpha != 1.f)) {
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = mul2(acc[i], pk2(alpha, alpha));
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) aoff[blk] *= alpha;
    }
    l_run = fmaf(psum, pm, l_run * alpha);
    m_run = mn;

    // ---- P.V: weights pn * (t d QFIX / max) in 16-bit fixed point, two int8 limbs
    if constexpr (FAM == FAM_ASYM) {
      float ao[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 m4 = *reinterpret_cast<const float4 *>(&T.vm[16 * (k >> 2) + 4 * tq + (k & 3)][0]);
        ao[0] = fmaf(p[k], m4.x, ao[0]);
        ao[1] = fmaf(p[k], m4.y, ao[1]);
        ao[2] = fmaf(p[k], m4.z, ao[2]);
        ao[3] = fmaf(p[k], m4.w, ao[3]);
      }
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) aoff[blk] = fmaf(pm, ao[blk], aoff[blk]);
    }
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const float4 ta = *reinterpret_cast<const float4 *>(&T.v[blk][4 * tq]);
      const float4 tb = *reinterpret_cast<const float4 *>(&T.v[blk][16 + 4 * tq]);
      const float tvk[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
      uint32_t wb[8];
#pragma unroll
      for (int k = 0; k < 8; k += 2) {
        float w0, w1;
        upk2(fma2(pk2(p[k], p[k + 1]), pk2(tvk[k], tvk[k + 1]), pk2(MAGIC, MAGIC)), w0, w1);
        wb[k] = __float_as_uint(w0);
        wb[k + 1] = __float_as_uint(w1);
      }
      uint32_t wa[4];
      {
        const uint32_t x = __byte_perm(wb[0], wb[1], 0x5140), y = __byte_perm(wb[2], wb[3], 0x5140);
        wa[0] = __byte_perm(x, y, 0x7632);
        wa[1] = __byte_perm(x, y, 0x5410) ^ 0x80808080u;
      }
      {
        const uint32_t x = __byte_perm(wb[4], wb[5], 0x5140), y = __byte_perm(wb[6], wb[7], 0x5140);
        wa[2] = __byte_perm(x, y, 0x7632);
        wa[3] = __byte_perm(x, y, 0x5410) ^ 0x80808080u;
      }
      // per-channel factor of the lane's two columns (channels 8 tq + u and 8 tq + 4 + u of
      // the block): the block's fixed-point scale times the chunk factor pm of head g, times
      // the page's V channel scale c
      const float sb = scl[blk] * pm;
      f32x2 f[4];
      if (FAM == FAM_KVARN) {
        const f32x2 *cp = reinterpret_cast<const f32x2 *>(&pa->fv[tq][4 * blk]);
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = mul2(pk2(sb, sb), cp[u]);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = pk2(sb, sb);
      }
      VQuad<FAM, BITS> v0, v1;
      v0.load(st + S::VC + tq * S::QS, blk, g);
      v1.load(st + S::VC + (4 + tq) * S::QS, blk, g);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        // column 2tq <-> channel 32 blk + 8 tq + u, column 2tq+1 <-> + 4
        mma_s8_fold(acc[blk * 4 + u], wa, v0.frag(u, g), v1.frag(u, g), f[u]);
      }
    }

    __syncwarp();  // every lane is done with this stage before it is refilled next round
    }
  }
  cp_async_wait<0>();
  __syncwarp();
  if constexpr (MODE == M_SCORES) return;
  l_run += __shfl_xor_sync(FULL, l_run, 1);
  l_run += __shfl_xor_sync(FULL, l_run, 2);
  if (FAM == FAM_ASYM) {
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      aoff[blk] += __shfl_xor_sync(FULL, aoff[blk], 1);
      aoff[blk] += __shfl_xor_sync(FULL, aoff[blk], 2);
    }
  }
  __syncwarp();
  if (hv) {
#pragma unroll
    for (int blk = 0; blk < 4; ++blk)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          accw[g * D + 32 * blk + 8 * tq + 4 * e + u] = acc_part(acc[blk * 4 + u], e) + aoff[blk];
    if (tq == 0) {
      mw[g] = m_run;
      lw[g] = l_run;
    }
  }
}

// ---- exact 16-bit rows (the tail, or a whole BF16 cache) on the tensor cores -------------
//
// mma.sync m16n8k16, bf16 x bf16 -> fp32 (f16 x f16 for a cache with an F16 tail; the
// description below says bf16 for both).  F16 high part + remainder carry about 22 bits of
// the query; values below the f16 normal range keep an absolute precision of 2^-25.  Q.K: A = the queries, rows 0..7 the bf16 high
// part of head g and rows 8..15 the bf16 remainder q - hi (together about 16 significant
// bits); B = K^T, 8 tokens per n-tile, read straight from the BF16 ring with 16-byte loads:
// within a 32-channel step s the k order is permuted so that lane (g, tq) supplies channels
// 32 s + 8 tq + 0..7 of token g; the query fragments follow the same permutation.  The
// scores of head g, tokens 2tq and 2tq+1 of the n-tile, are the sums of rows g and g+8.
// P.V: A = the softmax weights (rows g: bf16 high part, rows g+8: remainder), B = V (16
// tokens x 8 channels) built with byte permutes from four 16-byte row loads; column n of
// n-tile (j, e) is channel 8 (8 j + n) + e, so a lane's loads are whole 16-byte pieces.  The
// P.V accumulators stay in fp32 across the whole split (no per-chunk epilogue).

template <bool F16>
__device__ __forceinline__ void mma_16(float (&d)[4], const uint4 &a, uint32_t b0, uint32_t b1) {
  if constexpr (F16)
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
  else
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// (lo, hi) -> bf16x2 with lo in the low half, each rounded to nearest even
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// (x0, x1) split into a bf16x2 high part and a bf16x2 remainder
__device__ __forceinline__ void bf16_split(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  hi = bf16x2_rn(x0, x1);
  lo = bf16x2_rn(x0 - bf_lo(hi), x1 - bf_hi(hi));
}

// the same split in f16
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }
__device__ __forceinline__ void f16_split(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  hi = h2u(h);
  lo = h2u(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
}

template <bool F16>
__device__ __forceinline__ void split16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  if constexpr (F16)
    f16_split(x0, x1, hi, lo);
  else
    bf16_split(x0, x1, hi, lo);
}

// Query fragments of the BF16 path for one KV head (all warps of the CTA share them):
// qfb[ks * 32 + lane] = (a0, a1, a2, a3) of k-step ks = 2 s + h.
__device__ __forceinline__ void build_qfrag_bf16(uint4 *qfb, const float (*qraw)[D], int tid, int nthreads,
                                                 int f16) {
  for (int t = tid; t < 8 * 32; t += nthreads) {
    const int ks = t >> 5, l = t & 31, g = l >> 2, tq = l & 3;
    const int c = 32 * (ks >> 1) + 8 * tq + 4 * (ks & 1);
    uint4 f;
    if (f16) {
      f16_split(qraw[g][c], qraw[g][c + 1], f.x, f.y);
      f16_split(qraw[g][c + 2], qraw[g][c + 3], f.z, f.w);
    } else {
      bf16_split(qraw[g][c], qraw[g][c + 1], f.x, f.y);
      bf16_split(qraw[g][c + 2], qraw[g][c + 3], f.z, f.w);
    }
    qfb[t] = f;
  }
}

// Tokens [a + c0*32, a + c1*32) (clipped to b) of one warp: online-softmax state of the
// 8 head slots written to mw / lw / accw.  Ring rows past b may hold anything: their K and
// V loads are replaced by zeros and their scores by -inf.  NJ = 2 accumulates all 128
// channels in one pass over the tokens; NJ = 1 takes two passes of 64 channels (columns
// n-tile j = pass), recomputing the identical scores, with half the accumulator registers.
template <int NJ, bool F16>
__device__ __forceinline__ void warp_bf16_tc(const LayerView &L, int seq, int head, int64_t a, int64_t b, int64_t c0,
                                             int64_t c1, int64_t cdirty, const uint4 *qfb, float *mw, float *lw,
                                             float *accw) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const uint4 *kbase = reinterpret_cast<const uint4 *>(ring_row(L, seq, head, 0, 0));
  const uint4 *vbase = reinterpret_cast<const uint4 *>(ring_row(L, seq, head, 1, 0));
  // ring slots in 32 bits (a ring holds at most max_ctx < 2^31 rows)
  const int R = (int)L.ring_cap;
  const int slot_a = (int)((a + c0 * CH) % L.ring_cap);
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  bool waited = false;
#pragma unroll 1
  for (int jp = 0; jp < 2 / NJ; ++jp) {
    float acc[NJ][8][4];
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[j][e][i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    int slot0 = slot_a;
#pragma unroll 1
    for (int64_t ci = c0; ci < c1; ++ci) {
      if (!waited && ci >= cdirty) {
        wait_producer();
        waited = true;
      }
      const int64_t i0 = a + ci * CH;
      const int nvalid = (int)((b - i0) < CH ? (b - i0) : CH);
      // ---- Q.K: 4 n-tiles of 8 tokens; lane row = token 8 nt + g
      float sc[8];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int t = 8 * nt + g;
        int sl = slot0 + t;
        if (sl >= R) sl -= R;
        const uint4 *row = kbase + (size_t)sl * (2 * D / 16);
        uint4 kr[4];
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) kr[s2] = t < nvalid ? __ldg(row + 4 * s2 + tq) : zero;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) {
          mma_16<F16>(d, qfb[(2 * s2) * 32 + lane], kr[s2].x, kr[s2].y);
          mma_16<F16>(d, qfb[(2 * s2 + 1) * 32 + lane], kr[s2].z, kr[s2].w);
        }
        sc[2 * nt] = 8 * nt + 2 * tq < nvalid ? d[0] + d[2] : -INFINITY;
        sc[2 * nt + 1] = 8 * nt + 2 * tq + 1 < nvalid ? d[1] + d[3] : -INFINITY;
      }
      // ---- online softmax of head g (the 4 lanes tq of a group hold the chunk's 32 tokens)
      float cmax = sc[0];
#pragma unroll
      for (int k = 1; k < 8; ++k) cmax = fmaxf(cmax, sc[k]);
      cmax = fmaxf(cmax, __shfl_xor_sync(FULL, cmax, 1));
      cmax = fmaxf(cmax, __shfl_xor_sync(FULL, cmax, 2));
      const float mn = fmaxf(m_run, cmax);  // finite: every chunk holds a valid token
      const float alpha = exp2_fast(m_run - mn);
      float p[8], psum = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        p[k] = exp2_fast(sc[k] - mn);
        psum += p[k];
      }
      l_run = l_run * alpha + psum;
      m_run = mn;
      if (__any_sync(FULL, alpha != 1.f)) {
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
          for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[j][e][i] *= alpha;
      }
      // ---- P.V: 2 k-steps of 16 tokens
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        uint4 pa;  // rows g / g+8: weights of tokens 16 kt + 2tq + (0, 1) and 16 kt + 8 + 2tq + (0, 1)
        split16<F16>(p[4 * kt], p[4 * kt + 1], pa.x, pa.y);
        split16<F16>(p[4 * kt + 2], p[4 * kt + 3], pa.z, pa.w);
        int sl[4];
        bool vl[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = 16 * kt + 2 * tq + (r & 1) + 8 * (r >> 1);
          vl[r] = t < nvalid;
          sl[r] = slot0 + t;
          if (sl[r] >= R) sl[r] -= R;
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const int jc = NJ == 2 ? j : jp;  // channel half of these columns
          uint4 rv[4];
#pragma unroll
          for (int r = 0; r < 4; ++r)
            rv[r] = vl[r] ? __ldg(vbase + (size_t)sl[r] * (2 * D / 16) + 8 * jc + g) : zero;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int w = e >> 1;
            const unsigned sel = (e & 1) ? 0x7632u : 0x5410u;
            const uint32_t w0 = w == 0 ? rv[0].x : (w == 1 ? rv[0].y : (w == 2 ? rv[0].z : rv[0].w));
            const uint32_t w1 = w == 0 ? rv[1].x : (w == 1 ? rv[1].y : (w == 2 ? rv[1].z : rv[1].w));
            const uint32_t w2 = w == 0 ? rv[2].x : (w == 1 ? rv[2].y : (w == 2 ? rv[2].z : rv[2].w));
            const uint32_t w3 = w == 0 ? rv[3].x : (w == 1 ? rv[3].y : (w == 2 ? rv[3].z : rv[3].w));
            mma_16<F16>(acc[j][e], pa, __byte_perm(w0, w1, sel), __byte_perm(w2, w3, sel));
          }
        }
      }
      slot0 += CH;
      if (slot0 >= R) slot0 -= R;
    }
    if (jp == 2 / NJ - 1) {
      l_run += __shfl_xor_sync(FULL, l_run, 1);
      l_run += __shfl_xor_sync(FULL, l_run, 2);
      if (tq == 0) {
        mw[g] = m_run;
        lw[g] = l_run;
      }
    }
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int jc = NJ == 2 ? j : jp;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        accw[g * D + 8 * (8 * jc + 2 * tq) + e] = acc[j][e][0] + acc[j][e][2];
        accw[g * D + 8 * (8 * jc + 2 * tq + 1) + e] = acc[j][e][1] + acc[j][e][3];
      }
    }
  }
}

// H.x of one 128-wide row by one warp: the lane holds x[4 lane .. 4 lane + 3]; butterfly
// stages h = 1, 2 inside the lane, h = 4 .. 64 across lanes (xor 1 .. 16)
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

// Shared memory of the kernel (dynamic): fixed part + per-warp stage area (also used for the
// warps' accumulators once the chunks are done).
// What the end of the kernel (CTA combine, ticket, merge) needs of the launch arguments,
// computed once at the start (from the entry table, which is indexed at run time) and kept in
// shared memory, so that no register holds it across the main loop.
struct CtaMeta {
  float *rec;        // this (entry, KV head)'s split records: [split][G][PSTRIDE]
  float *out;        // this (entry, KV head)'s output rows: [G][D]
  uint32_t *ticket;  // its merge ticket
  int G, sp, nspl, nsq, rotv;
};

template <int NW, int FAM>
struct SmemFixed {
  CtaMeta meta;
  // q, q' and the merge sums are read and written with 16-byte vector accesses
  alignas(16) float qraw[MAX_G][D];
  alignas(16) float qrot[MAX_G][D];
  float mw[NW][MAX_G], lw[NW][MAX_G];
  float fw[MAXSPL][MAX_G];   // weight of each warp (CTA combine) / split (merge)
  float fm[MAXSPL][MAX_G];   // merge: m and l of the splits whose records are not staged
  float fl[MAXSPL][MAX_G];
  alignas(16) float red[MAX_G][D];  // merge: sum over the tail splits (original basis)
  float Ls[MAX_G];
  float Mc[MAX_G], Lc[MAX_G];  // this CTA's combined m and l per head
  ChunkTabs<FAM> tabs[NW];
  int is_last;
};
using SmemFixedA12 = SmemFixed<12, FAM_ASYM>;
using SmemFixedK8 = SmemFixed<8, FAM_KVARN>;
static_assert(offsetof(SmemFixedA12, qrot) % 16 == 0 && offsetof(SmemFixedK8, tabs) % 16 == 0 &&
                  offsetof(SmemFixedK8, red) % 16 == 0,
              "vector-accessed shared arrays start on 16 bytes");

template <int FAM, int BITS>
__host__ __device__ constexpr int warp_area() {
  if constexpr (FAM == FAM_BF16) {
    return 16384;  // accumulators, then (all warps together) the merge's staged partials
  } else {
    // stages, then (kvarn) the page area
    constexpr int s = Stage<FAM, BITS>::NST * Stage<FAM, BITS>::BYTES + (FAM == FAM_KVARN ? (int)sizeof(PageArea) : 0);
    return s > MAX_G * D * 4 ? s : MAX_G * D * 4;
  }
}

// the page area of a warp (kvarn): after its stages
template <int FAM, int BITS>
__device__ __forceinline__ PageArea *page_area(uint8_t *warp_base) {
  return reinterpret_cast<PageArea *>(warp_base + Stage<FAM, BITS>::NST * Stage<FAM, BITS>::BYTES);
}

// [SmemFixed][warp areas]
template <int FAM, int BITS, int NW>
__host__ __device__ constexpr size_t smem_bytes_for() {
  return ((sizeof(SmemFixed<NW, FAM>) + 127) / 128) * 128 + (size_t)NW * warp_area<FAM, BITS>();
}
constexpr size_t kSmemMax = 232448;  // dynamic shared memory per CTA on sm_100

// Warps per CTA (one CTA per SM): 12 for codes of up to 5 bits (168 registers: the 24-bit
// query limbs stay in registers; 16 warps at 128 registers measured no faster), 8 for 6- and
// 8-bit codes (about 230 registers) and for BF16 caches.
template <int FAM, int BITS>
__host__ __device__ constexpr int nwarps() {
  if constexpr (FAM == FAM_BF16 || BITS >= 6)
    return 8;
  else
    return 12;
}

template <int FAM, int BITS>
__host__ __device__ constexpr size_t smem_fixed_bytes() {
  return ((sizeof(SmemFixed<nwarps<FAM, BITS>(), FAM>) + 127) / 128) * 128;
}

template <int FAM, int BITS>
__host__ __device__ constexpr size_t smem_bytes() {
  return smem_bytes_for<FAM, BITS, nwarps<FAM, BITS>()>();
}

template <int FAM, int BITS, int MODE>
__global__ void __launch_bounds__(32 * nwarps<FAM, BITS>(), 1) k_decode(LayerView L, DArgs A) {
  static_assert(MODE == M_FUSED || FAM != FAM_BF16, "the score modes take quantized types");
  constexpr int NW = nwarps<FAM, BITS>(), DT = 32 * NW;
  extern __shared__ __align__(128) uint8_t smem[];
  SmemFixed<NW, FAM> &F = *reinterpret_cast<SmemFixed<NW, FAM> *>(smem);
  uint8_t *warp_mem = smem + smem_fixed_bytes<FAM, BITS>();
  constexpr int WA = warp_area<FAM, BITS>();

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bid = blockIdx.x;
  int si = 0;
  while (si + 1 < A.nseq && A.s[si + 1].cta0 <= bid) ++si;
  const DSeq &s = A.s[si];
  const int nspl = s.nsq + s.nst;
  const int local = bid - s.cta0;
  // CTA order within an entry: the uniform quantized splits of every head first, then the
  // light ones (the split an overlapped append rewrites, the BF16 tail splits), so that when
  // a preceding kernel still holds SMs, the CTAs left waiting for them are the light ones
  const int nreg = s.nsq - (s.qa < s.Q ? 1 : 0);
  int head, sp;
  if (local < A.hkv * nreg) {
    head = local / nreg;
    sp = local % nreg;
  } else {
    const int l2 = local - A.hkv * nreg, nlight = nspl - nreg;
    head = l2 / nlight;
    sp = nreg + l2 % nlight;
  }
  const int G = A.G;
  const bool tail = sp >= s.nsq;
  if (MODE == M_SCORES && tail) return;  // the BF16 tail splits belong to the P.V kernel
  int64_t a, b;
  int64_t nch;
  if (!tail) {
    if (s.qa < s.Q && sp == s.nsq - 1) {
      // the tokens an overlapped append rewrites, a split of their own: its warps wait for the
      // append while the other splits stream, then take one chunk each
      a = s.qa;
      b = s.Q;
    } else {
      a = (int64_t)sp * s.cps_q * CH;
      b = min(a + (int64_t)s.cps_q * CH, s.qa);
    }
  } else {
    a = s.Q + (int64_t)(sp - s.nsq) * s.cps_t * CH;
    b = min(a + (int64_t)s.cps_t * CH, s.n);
  }
  nch = b > a ? (b - a + CH - 1) / CH : 0;
  // a contiguous chunk range per warp, sizes differing by at most one
  const int64_t c0 = nch * warp / NW, c1 = nch * (warp + 1) / NW;

  // chunks at or past cdirty hold tokens the preceding (overlapped) append kernel writes
  const int64_t cdirty = first_dirty_chunk(a, (tail || FAM == FAM_BF16) ? s.dt : s.dq);
  bool waited = false;
  PageCursor pc;
  const ScoreRow sr{A.scores + (int64_t)(si * A.hkv + head) * G * A.qcap, A.qcap};
  // the query rows of this KV head are loaded first, so that they do not queue behind the
  // prefetched chunks of every CTA
  constexpr int QPER = (MAX_G * D + DT - 1) / DT;
  float qv[QPER];
#pragma unroll
  for (int u = 0; u < QPER; ++u) {
    const int idx = tid + u * DT, g = idx / D, j = idx % D;
    qv[u] = (idx < MAX_G * D && g < G) ? __ldg(&A.q[((int64_t)s.row * A.hkv * G + head * G + g) * D + j]) : 0.f;
  }
  if constexpr (FAM != FAM_BF16) {
    if (!tail)
      warp_quant_prefetch<FAM, BITS, MODE>(L, s.seq, head, a, (int)c0, (int)c1, cdirty, waited,
                                           warp_mem + (size_t)warp * WA, lane, pc,
                                           page_area<FAM, BITS>(warp_mem + (size_t)warp * WA), sr, G);
  }
  // query rows, pre-scaled by softmax_scale * log2(e); heads >= G are 0
#pragma unroll
  for (int u = 0; u < QPER; ++u) {
    const int idx = tid + u * DT;
    if (idx < MAX_G * D) F.qraw[idx / D][idx % D] = qv[u] * A.qscale;
  }
  for (int idx = tid; idx < NW * MAX_G; idx += DT) {
    F.mw[idx / MAX_G][idx % MAX_G] = -INFINITY;
    F.lw[idx / MAX_G][idx % MAX_G] = 0.f;
  }
  if (tid == 0) {
    CtaMeta m;
    m.rec = A.ws + (int64_t)(s.part0 + head * nspl) * G * PSTRIDE;
    m.out = A.out + ((int64_t)s.row * A.hkv * G + head * G) * D;
    m.ticket = &A.tickets[si * A.hkv + head];
    m.G = G;
    m.sp = sp;
    m.nspl = nspl;
    m.nsq = s.nsq;
    m.rotv = A.rotv;
    F.meta = m;
  }
  __syncthreads();
  // BF16 rows (the tail splits, or a whole BF16 cache) take the raw q as bf16 MMA fragments,
  // kept in the q' area
  const bool bf16_rows = tail || FAM == FAM_BF16;
  uint4 *qfb = reinterpret_cast<uint4 *>(&F.qrot[0][0]);
  static_assert(sizeof(F.qrot) >= 8 * 32 * sizeof(uint4), "q' area holds the BF16 query fragments");
  if (bf16_rows) {
    build_qfrag_bf16(qfb, F.qraw, tid, DT, L.tail_f16);
  } else if (MODE == M_PVEXT) {
    // the scores are given: no query on the quantized splits
  } else if (A.rotk) {
    // q' = H.q.kappa, one warp per query head
    if (warp < G) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = F.qraw[warp][4 * lane + e];
      warp_wht(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) F.qrot[warp][4 * lane + e] = v[e] * kKappa();
    }
  } else {
    for (int idx = tid; idx < MAX_G * D; idx += DT) F.qrot[idx / D][idx % D] = F.qraw[idx / D][idx % D];
  }
  __syncthreads();

  float *accw = reinterpret_cast<float *>(warp_mem + (size_t)warp * WA);  // [MAX_G][D] after the chunks
  static_assert(WA >= MAX_G * D * 4, "warp area holds the accumulator");
  if (!bf16_rows) {
    if constexpr (FAM != FAM_BF16)
      warp_quant<FAM, BITS, MODE>(L, s.seq, head, a, b, (int)c0, (int)c1, cdirty, waited, G, F.qrot,
                                  warp_mem + (size_t)warp * WA, F.tabs[warp], F.mw[warp], F.lw[warp], accw, pc,
                                  page_area<FAM, BITS>(warp_mem + (size_t)warp * WA), sr);
    if constexpr (MODE == M_SCORES) return;  // every CTA of this kernel is a quantized split
  } else {
    // quantized kernels keep their tail warps light on registers: two channel passes
    constexpr int NJ = FAM == FAM_BF16 ? 2 : 1;
    if (L.tail_f16)
      warp_bf16_tc<NJ, true>(L, s.seq, head, a, b, c0, c1, cdirty, qfb, F.mw[warp], F.lw[warp], accw);
    else
      warp_bf16_tc<NJ, false>(L, s.seq, head, a, b, c0, c1, cdirty, qfb, F.mw[warp], F.lw[warp], accw);
  }
  __syncthreads();

  const CtaMeta mt = F.meta;
  {
    const int G = mt.G;  // (shadows the launch argument: from here on only shared memory)
  // combine the warps of this CTA into its partial (m, l, acc) per query head: warp g
  // reduces head g over the warps, one lane per warp
  if (warp < G) {
    const float mw = lane < NW ? F.mw[lane][warp] : -INFINITY;
    const float M = warp_max(mw);
    const float f = (mw == -INFINITY) ? 0.f : exp2_fast(mw - M);
    if (lane < NW) F.fw[lane][warp] = f;
    const float lsum = warp_sum(lane < NW ? f * F.lw[lane][warp] : 0.f);
    if (lane == 0) {
      F.Mc[warp] = M;
      F.Lc[warp] = lsum;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += DT) {
    const int g = idx / D, c = idx % D;
    float av = 0.f;
#pragma unroll 4
    for (int w = 0; w < NW; ++w)
      av = fmaf(F.fw[w][g], reinterpret_cast<const float *>(warp_mem + (size_t)w * WA)[g * D + c], av);
    float *dst = mt.rec + (int64_t)(mt.sp * G + g) * PSTRIDE;
    dst[PACC + c] = av;
    if (c == 0) {
      dst[0] = F.Mc[g];
      dst[1] = F.Lc[g];
    }
  }

  // the last CTA of this (sequence, KV head) merges all splits (atomic ticket; no waiting).
  // The barrier orders the CTA's record stores before thread 0's fence and ticket (release);
  // in the last CTA, thread 0's second fence and the barrier order the other records before
  // every thread's reads (acquire).
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(mt.ticket, 1u);
    // a ticket past the split count means the counter was not zero when this decode began
    if (prev >= (unsigned)mt.nspl) atomicOr(L.status, kStatusTicket);
    F.is_last = prev == (unsigned)(mt.nspl - 1);
    if (F.is_last) __threadfence();
  }
  __syncthreads();
  if (!F.is_last) return;

  // The partial records (nspl * G of them, contiguous) are staged in shared memory by cp.async,
  // as many whole splits per batch as the warp areas hold; the m and l of the splits beyond
  // the first batch are read directly, so that the weights are known before any sum.
  const int nspl = mt.nspl;
  const float *part = mt.rec;
  float *stage = reinterpret_cast<float *>(warp_mem);
  constexpr int CAP = (NW * WA) / (PSTRIDE * 4);  // records that fit
  const int kper = CAP / G;                       // whole splits per batch (>= 1)
  int kb0 = 0, kb1 = min(nspl, kper);
  for (int p = tid; p < kb1 * G * (PSTRIDE / 4); p += DT) cp_async16(stage + 4 * p, part + 4 * p);
  cp_async_commit();
  for (int idx = kb1 * G + tid; idx < nspl * G; idx += DT) {
    F.fm[idx / G][idx % G] = __ldcg(part + (int64_t)idx * PSTRIDE);
    F.fl[idx / G][idx % G] = __ldcg(part + (int64_t)idx * PSTRIDE + 1);
  }
  cp_async_wait<0>();
  __syncthreads();
  // split weights: warp g, one lane per split
  if (warp < G) {
    const int g = warp;
    float mk[MAXSPL / 32], M = -INFINITY;
#pragma unroll
    for (int u = 0; u < MAXSPL / 32; ++u) {
      const int k = lane + 32 * u;
      mk[u] = k < nspl ? (k < kb1 ? stage[(k * G + g) * PSTRIDE] : F.fm[k][g]) : -INFINITY;
      M = fmaxf(M, mk[u]);
    }
    M = warp_max(M);
    float ls = 0.f;
#pragma unroll
    for (int u = 0; u < MAXSPL / 32; ++u) {
      const int k = lane + 32 * u;
      if (k < nspl) {
        const float f = (mk[u] == -INFINITY) ? 0.f : exp2_fast(mk[u] - M);
        F.fw[k][g] = f;
        ls = fmaf(f, k < kb1 ? stage[(k * G + g) * PSTRIDE + 1] : F.fl[k][g], ls);
      }
    }
    ls = warp_sum(ls);
    if (lane == 0) F.Ls[g] = ls;
  }
  __syncthreads();
  // weighted sums, one thread per (head, channel) output; quantized splits (stored basis)
  // and tail splits (original basis) are kept apart
  for (;;) {
    for (int o = tid; o < G * D; o += DT) {
      const int g = o / D, ch = o % D;
      float srot = kb0 ? F.qraw[g][ch] : 0.f, spl = kb0 ? F.red[g][ch] : 0.f;
      for (int k = kb0; k < kb1; ++k) {
        const float v = stage[((k - kb0) * G + g) * PSTRIDE + PACC + ch];
        if (k < mt.nsq)
          srot = fmaf(F.fw[k][g], v, srot);
        else
          spl = fmaf(F.fw[k][g], v, spl);
      }
      F.qraw[g][ch] = srot;
      F.red[g][ch] = spl;
    }
    if (kb1 >= nspl) break;
    __syncthreads();  // the stage is free again
    kb0 = kb1;
    kb1 = min(nspl, kb0 + kper);
    const float *src = part + (int64_t)kb0 * G * PSTRIDE;
    for (int p = tid; p < (kb1 - kb0) * G * (PSTRIDE / 4); p += DT) cp_async16(stage + 4 * p, src + 4 * p);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
  }
  __syncthreads();
  // output: (H.acc_rot.kappa + acc_plain) / L, one warp per query head
  for (int g = warp; g < G; g += NW) {
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = F.qraw[g][4 * lane + e];
    if (mt.rotv) {
      warp_wht(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] *= kKappa();
    }
    const float Lg = F.Ls[g];
    const float inv = Lg > 0.f ? 1.0f / Lg : 0.f;
    float4 o;
    o.x = (v[0] + F.red[g][4 * lane + 0]) * inv;
    o.y = (v[1] + F.red[g][4 * lane + 1]) * inv;
    o.z = (v[2] + F.red[g][4 * lane + 2]) * inv;
    o.w = (v[3] + F.red[g][4 * lane + 3]) * inv;
    *reinterpret_cast<float4 *>(mt.out + (int64_t)g * D + 4 * lane) = o;
  }
  if (tid == 0) *mt.ticket = 0u;
  }
}

template <int FAM, int BITS, int MODE>
cudaError_t run(const LayerView &L, const DArgs &A, cudaStream_t st, bool pdl) {
  constexpr size_t smem = smem_bytes<FAM, BITS>();
  static_assert(smem <= 232448, "shared memory per CTA");
  static_assert((nwarps<FAM, BITS>() * warp_area<FAM, BITS>()) / (PSTRIDE * 4) >= MAX_G, "merge stage holds a split");
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(k_decode<FAM, BITS, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)A.ncta);
  cfg.blockDim = dim3(32 * nwarps<FAM, BITS>());
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_decode<FAM, BITS, MODE>, L, A);
}

template <int MODE>
cudaError_t dispatch_q(int fam, int bits, const LayerView &L, const DArgs &A, cudaStream_t st, bool pdl) {
#define KVQ_D(F, B) \
  if (fam == F && bits == B) return run<F, B, MODE>(L, A, st, pdl);
  KVQ_D(FAM_SYM, 2) KVQ_D(FAM_SYM, 3) KVQ_D(FAM_SYM, 4) KVQ_D(FAM_SYM, 5) KVQ_D(FAM_SYM, 6) KVQ_D(FAM_SYM, 8)
  KVQ_D(FAM_ASYM, 2) KVQ_D(FAM_ASYM, 3) KVQ_D(FAM_ASYM, 4) KVQ_D(FAM_ASYM, 5) KVQ_D(FAM_ASYM, 6)
  KVQ_D(FAM_KVARN, 2) KVQ_D(FAM_KVARN, 3) KVQ_D(FAM_KVARN, 4) KVQ_D(FAM_KVARN, 5) KVQ_D(FAM_KVARN, 6)
  KVQ_D(FAM_KVARN, 8)
#undef KVQ_D
  return cudaErrorInvalidValue;
}

cudaError_t dispatch(int fam, int bits, int mode, const LayerView &L, const DArgs &A, cudaStream_t st, bool pdl) {
  if (mode == M_FUSED && fam == FAM_BF16 && bits == 16) return run<FAM_BF16, 16, M_FUSED>(L, A, st, pdl);
  if (mode == M_FUSED) return dispatch_q<M_FUSED>(fam, bits, L, A, st, pdl);
  if (mode == M_SCORES) return dispatch_q<M_SCORES>(fam, bits, L, A, st, pdl);
  if (mode == M_PVEXT) return dispatch_q<M_PVEXT>(fam, bits, L, A, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace

// The split partials; for K and V of different types also the scores of the quantized
// prefix, [entry of a launch][KV head][G][qcap] fp32 after the partials (16-byte aligned).
size_t decode_partials_bytes(const kvq_cache *c, int n_seqs, int n_q_heads) {
  const int G = n_q_heads / c->p.n_kv_heads;
  return sizeof(float) * (size_t)std::max(n_seqs, 1) * c->p.n_kv_heads * MAXSPL * G * PSTRIDE;
}
int64_t decode_score_cap(const kvq_cache *c) { return (c->p.max_ctx + CH - 1) / CH * CH; }

size_t decode_workspace_bytes(const kvq_cache *c, int n_seqs, int n_q_heads) {
  const size_t part = decode_partials_bytes(c, n_seqs, n_q_heads);
  if (c->p.type_k == c->p.type_v) return part;
  const int G = n_q_heads / c->p.n_kv_heads;
  const size_t entries = (size_t)std::min(std::max(n_seqs, 1), MAXS);
  return part + sizeof(float) * entries * c->p.n_kv_heads * G * (size_t)decode_score_cap(c);
}

int launch_decode(const kvq_cache *c, int layer, const std::vector<DecodeSeq> &seqs, int n_q_heads,
                  const float *q, float scale, float *out, void *ws, size_t ws_bytes, cudaStream_t st,
                  int budget_sms, bool pdl) {
  const int sms = budget_sms > 0 && budget_sms < c->num_sms ? budget_sms : c->num_sms;
  // K and V of different types: a Q.K kernel of the K type writes the scores, a P.V kernel of
  // the V type reads them (not overlapped with a preceding append)
  const bool mixed = c->p.type_k != c->p.type_v;
  if (mixed && (c->fam_k == FAM_BF16 || c->fam_v == FAM_BF16)) return KVQ_E_UNSUPPORTED;
  if (mixed) pdl = false;
  (void)ws_bytes;
  const LayerView L = layer_view(c, layer);
  const int hkv = c->p.n_kv_heads, G = n_q_heads / hkv;
  // relative cost of one token of a (K+V) head pair: quantized tokens by their bytes; a BF16
  // tail token (tensor-core path, 512 bytes) as about twice a quantized one
  const double tbq = (double)token_bytes(c->fam_k, c->bits_k) + token_bytes(c->fam_v, c->bits_v);
  const double tbt = 2.0 * tbq;
  // the decode overlaps the preceding append only when one launch takes every entry
  pdl = pdl && seqs.size() <= (size_t)MAXS;
  for (size_t base = 0; base < seqs.size(); base += MAXS) {
    const size_t cnt = std::min<size_t>(MAXS, seqs.size() - base);
    DArgs A{};
    A.nseq = (int)cnt;
    A.G = G;
    A.hkv = hkv;
    A.rotk = c->fam_k == FAM_KVARN;
    A.rotv = c->fam_v == FAM_KVARN;
    A.qscale = scale * LOG2E;
    A.q = q;
    A.out = out;
    A.ws = static_cast<float *>(ws);
    A.scores = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + decode_partials_bytes(c, (int)seqs.size(), n_q_heads));
    A.qcap = decode_score_cap(c);
    A.tickets = reinterpret_cast<uint32_t *>(c->base + c->off_tickets);
    // split plan (min-max greedy): every (sequence, part) with tokens starts with one split
    // per KV head; then, while a whole column of hkv CTAs still fits in one wave, the part
    // whose splits carry the most work gets one more split.  Behind an overlapped append, the
    // quantized tokens it rewrites (from the chunk holding dq on) form one more split of
    // their own, so that the wait for the append holds back only that split's few chunks.
    std::vector<int> nq(cnt), nt(cnt), nd(cnt);
    std::vector<int64_t> qa(cnt);
    int used = 0;
    for (size_t i = 0; i < cnt; ++i) {
      const DecodeSeq &d = seqs[base + i];
      qa[i] = pdl && d.dq < d.Q ? (d.dq / CH) * CH : d.Q;
      nd[i] = qa[i] < d.Q ? 1 : 0;
      nq[i] = qa[i] > 0 ? 1 : 0;
      nt[i] = d.n > d.Q ? 1 : 0;
      used += hkv * (nq[i] + nt[i] + nd[i]);
    }
    // when the entries need more than one wave anyway, plan whole waves
    const int budget = std::max(sms, ((used + sms - 1) / sms) * sms);
    while (used + hkv <= budget) {
      int best = -1;
      bool best_t = false;
      double most = 0.0;
      for (size_t i = 0; i < cnt; ++i) {
        const DecodeSeq &d = seqs[base + i];
        const int64_t nchq = (qa[i] + CH - 1) / CH, ncht = (d.n - d.Q + CH - 1) / CH;
        const double wq = nq[i] ? (double)qa[i] * tbq / nq[i] : 0.0;
        const double wt = nt[i] ? (double)(d.n - d.Q) * tbt / nt[i] : 0.0;
        if (wq > most && nq[i] + nd[i] < MAXSQ && nq[i] < nchq) { most = wq; best = (int)i; best_t = false; }
        if (wt > most && nt[i] < MAXST && nt[i] < ncht) { most = wt; best = (int)i; best_t = true; }
      }
      if (best < 0) break;
      if (best_t) ++nt[best]; else ++nq[best];
      used += hkv;
    }
    int cta = 0, part = 0;
    for (size_t i = 0; i < cnt; ++i) {
      const DecodeSeq &d = seqs[base + i];
      DSeq &s = A.s[i];
      s.seq = d.seq;
      s.row = d.row;
      s.n = d.n;
      s.Q = d.Q;
      s.qa = qa[i];
      s.dq = d.dq;
      s.dt = d.dt;
      const int64_t nchq = (qa[i] + CH - 1) / CH, ncht = (d.n - d.Q + CH - 1) / CH;
      s.cps_q = nq[i] ? (int)((nchq + nq[i] - 1) / nq[i]) : 1;
      s.nsq = (nq[i] ? (int)((nchq + s.cps_q - 1) / s.cps_q) : 0) + nd[i];
      s.cps_t = nt[i] ? (int)((ncht + nt[i] - 1) / nt[i]) : 1;
      s.nst = nt[i] ? (int)((ncht + s.cps_t - 1) / s.cps_t) : 0;
      if (s.nsq + s.nst == 0) s.nst = 1;  // empty sequence: one empty split writes zeros
      s.cta0 = cta;
      s.part0 = part;
      cta += hkv * (s.nsq + s.nst);
      part += hkv * (s.nsq + s.nst);
    }
    A.ncta = cta;
    // q / out rows are indexed by DecodeSeq::row; the workspace slots restart per launch
    // overlap only a decode of one launch: a second launch would follow the first, not the producer
    if (mixed) {
      if (dispatch(c->fam_k, c->bits_k, M_SCORES, L, A, st, false) != cudaSuccess ||
          dispatch(c->fam_v, c->bits_v, M_PVEXT, L, A, st, false) != cudaSuccess)
        return KVQ_E_CUDA;
      note_launches(2);
      continue;
    }
    if (dispatch(c->fam_k, c->bits_k, M_FUSED, L, A, st, pdl) != cudaSuccess)
      return KVQ_E_CUDA;
    note_launches(1);
  }
  return KVQ_OK;
}

}  // namespace kvq
