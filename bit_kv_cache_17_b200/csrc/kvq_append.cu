// kvq_append.cu - append path: tail ring write, spill quantization (qb_0, qb_1, kvarn).
//
// Compiled with -fmad=false and written with explicit __f*_rn intrinsics: every fp32
// operation that decides a code or a scale rounds once, in the order written, so the
// codes and fp16 scales match the CPU oracle bit for bit.
//
// Steps (pages: "KV Cache Precision Tail" and "KVarN" sections of the BeeLLama.cpp v0.4.0
// page; "How WHT and Sinkhorn save quality at 4-bit" of the Bonsai-Ternary-27B page):
//  1. tokens that leave the newest-`tail` window are quantized; for kvarn every 256-token
//     group touched by the append is rebuilt from its BF16 rows (ring or new input):
//     Walsh-Hadamard rotation -> Sinkhorn balancing -> symmetric block quantization;
//  2. the new tokens that stay 16-bit are copied into the BF16 ring.
// Step 1 reads ring rows that step 2 may overwrite, so step 2 is launched after it, unless
// no ring slot that step 2 writes can hold a row that step 1 reads (the span from the first
// row read to the last row written fits in the ring, as for one-token appends to a kvarn
// cache): then the spill kernel writes the new rows itself and one launch does both.
// Every kernel here signals its dependents as it starts (griddepcontrol.launch_dependents),
// so that a decode launched with programmatic stream serialization may overlap it.
#include <cuda_runtime.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int MAXS = 64;  // sequences per launch (kernel parameter space)

struct SeqWork {
  int32_t seq;
  int32_t pad;
  int64_t n0, n1;    // sequence length before / after the append
  int64_t in_off;    // first input row of this sequence
  int64_t a, b;      // kernel-specific range
  int64_t item0;     // first work item of this sequence
  int64_t tw;        // k_spill_kvarn: new rows [tw, n1) go to the ring in this launch
};

__device__ __forceinline__ void signal_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

struct Work {
  int32_t n;
  int32_t which;
  int64_t total;
  SeqWork s[MAXS];
};

__device__ __forceinline__ int find_seq(const Work &W, int64_t item) {
  int si = 0;
  while (si + 1 < W.n && W.s[si + 1].item0 <= item) ++si;
  return si;
}

__device__ __forceinline__ const __nv_bfloat16 *src_row(const LayerView &L, const SeqWork &s, int head,
                                                        int which, int64_t p, const __nv_bfloat16 *in) {
  if (p < s.n0) return ring_row(L, s.seq, head, which, p);
  return in + ((s.in_off + (p - s.n0)) * L.hkv + head) * D;
}

// channels 4 lane .. 4 lane + 3 of token p as the quantizer sees them: a ring row as stored,
// an input row rounded to the tail's format
__device__ __forceinline__ void load4(const LayerView &L, const SeqWork &s, int head, int which, int64_t p,
                                      const __nv_bfloat16 *in, int lane, float (&x)[4]) {
  const bool ring = p < s.n0;
  const uint2 raw = *reinterpret_cast<const uint2 *>(src_row(L, s, head, which, p, in) + 4 * lane);
  const float2 a = ring2f(raw.x, ring ? L.tail_f16 : 0), b = ring2f(raw.y, ring ? L.tail_f16 : 0);
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
  if (!ring && L.tail_f16) {
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = tail_round(x[e], 1);
  }
}

// ---- packing -------------------------------------------------------------------------

// K plane of width W: the warp's lane holds channels 4*jj..4*jj+3 of block blk (jj = lane&7).
template <int W>
__device__ __forceinline__ void pack_k_plane(const uint32_t (&v)[4], uint8_t *plane, int blk, int jj) {
  constexpr int F = 8 / W;
  constexpr uint32_t MASK = (1u << W) - 1u;
  const int m = jj / F, s = jj % F;
  uint32_t word = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) word |= (v[k] & MASK) << (8 * k + s * W);
#pragma unroll
  for (int o = 1; o < F; o <<= 1) word |= __shfl_xor_sync(FULL, word, o);
  if (s == 0) *reinterpret_cast<uint32_t *>(plane + 16 * m + 4 * blk) = word;
}

// V plane of width W for quad token k: the lane holds channels 4*j8..4*j8+3 of block blk.
template <int W>
__device__ __forceinline__ void pack_v_plane(const uint32_t (&v)[4], uint8_t *plane, int blk, int j8, int k) {
  constexpr uint32_t MASK = (1u << W) - 1u;
  uint8_t *base = plane + 16 * W * blk + k;
  if constexpr (W == 8) {
#pragma unroll
    for (int i = 0; i < 4; ++i) base[4 * (4 * j8 + i)] = (uint8_t)(v[i] & MASK);
  } else if constexpr (W == 4) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      base[4 * (2 * j8 + h)] = (uint8_t)((v[2 * h] & MASK) | ((v[2 * h + 1] & MASK) << 4));
  } else if constexpr (W == 2) {
    base[4 * j8] = (uint8_t)((v[0] & MASK) | ((v[1] & MASK) << 2) | ((v[2] & MASK) << 4) | ((v[3] & MASK) << 6));
  } else {  // W == 1: two lanes share one byte
    uint32_t nib = (v[0] & 1u) | ((v[1] & 1u) << 1) | ((v[2] & 1u) << 2) | ((v[3] & 1u) << 3);
    nib <<= 4 * (j8 & 1);
    nib |= __shfl_xor_sync(FULL, nib, 1);
    if ((j8 & 1) == 0) base[4 * (j8 >> 1)] = (uint8_t)nib;
  }
}

template <int BITS, int WHICH>
__device__ __forceinline__ void pack_codes(const int (&code)[4], uint8_t *sub, int tip, int lane) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  uint32_t lo[4], hi[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t f = (uint32_t)code[e] & ((1u << BITS) - 1u);
    lo[e] = f & ((1u << WL) - 1u);
    hi[e] = f >> WL;
  }
  const int blk = lane >> 3, j8 = lane & 7;
  if constexpr (WHICH == 0) {
    uint8_t *tok = sub + tip * 16 * BITS;
    pack_k_plane<WL>(lo, tok, blk, j8);
    if constexpr (WH > 0) pack_k_plane<WH>(hi, tok + 16 * WL, blk, j8);
  } else {
    uint8_t *quad = sub + (tip >> 2) * 64 * BITS;
    pack_v_plane<WL>(lo, quad, blk, j8, tip & 3);
    if constexpr (WH > 0) pack_v_plane<WH>(hi, quad + 64 * WL, blk, j8, tip & 3);
  }
}

// rint(RN(y / d)) (IEEE quotient, then round half to even) without a division in the common
// case.  q = RN(y * RN(1/d)) is within 2 ulp of RN(y / d); when q is more than 4 ulp away from
// the nearest half-integer both round to the same integer, otherwise the exact quotient is
// taken.  (4 ulp of q is bounded by max(|q|, 1) * 2^-20.)
__device__ __forceinline__ float rint_quotient(float y, float d, float rd) {
  const float q = __fmul_rn(y, rd);
  const float r = rintf(q);
  const float tol = fmaxf(fabsf(q), 1.0f) * 9.5367431640625e-07f;
  if (fabsf(fabsf(__fsub_rn(q, r)) - 0.5f) <= tol) return rintf(__fdiv_rn(y, d));
  return r;
}

// ---- block quantizers (one token-head per warp; lane holds channels 4*lane..+3) ------

template <int BITS, int WHICH>
__device__ __forceinline__ void quant_sym(const float (&y)[4], uint8_t *sub, const SubLayout &lay, int tip,
                                          int lane) {
  constexpr int QMAX = (1 << (BITS - 1)) - 1, QMIN = -(1 << (BITS - 1));
  float a = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
  a = fmaxf(a, __shfl_xor_sync(FULL, a, 4));
  a = fmaxf(a, __shfl_xor_sync(FULL, a, 2));
  a = fmaxf(a, __shfl_xor_sync(FULL, a, 1));
  const __half dh = sat_half(__fdiv_rn(a, (float)QMAX));
  const float df = __half2float(dh);
  const float rd = df != 0.0f ? __frcp_rn(df) : 0.0f;
  int code[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int q = 0;
    if (df != 0.0f) {
      float r = rint_quotient(y[e], df, rd);
      r = fminf(fmaxf(r, (float)QMIN), (float)QMAX);
      q = (int)r;
    }
    code[e] = q;
  }
  pack_codes<BITS, WHICH>(code, sub, tip, lane);
  if ((lane & 7) == 0) reinterpret_cast<__half *>(sub + lay.d)[tip * 4 + (lane >> 3)] = dh;
}

template <int BITS, int WHICH>
__device__ __forceinline__ void quant_asym(const float (&x)[4], uint8_t *sub, const SubLayout &lay, int tip,
                                           int lane) {
  constexpr int QMAX = (1 << BITS) - 1;
  float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
  float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
  }
  const __half dh = sat_half(__fdiv_rn(__fsub_rn(mx, mn), (float)QMAX));
  const __half mh = sat_half(mn);
  const float df = __half2float(dh), mf = __half2float(mh);
  int code[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int q = 0;
    if (df != 0.0f) {
      float r = rintf(__fdiv_rn(__fsub_rn(x[e], mf), df));
      r = fminf(fmaxf(r, 0.0f), (float)QMAX);
      q = (int)r;
    }
    code[e] = q;
  }
  pack_codes<BITS, WHICH>(code, sub, tip, lane);
  if ((lane & 7) == 0) {
    reinterpret_cast<__half *>(sub + lay.d)[tip * 4 + (lane >> 3)] = dh;
    reinterpret_cast<__half *>(sub + lay.m)[tip * 4 + (lane >> 3)] = mh;
  }
}

// ---- kernels ---------------------------------------------------------------------------

// One warp per quantized token-head of a qb_0 / qb_1 type.  Work range per sequence:
// tokens [a, b) = [Q(n0), Q(n1)), item = token * hkv + head.
template <int FAM, int BITS, int WHICH>
__global__ void __launch_bounds__(256) k_spill_qb(LayerView L, Work W, const __nv_bfloat16 *__restrict__ in) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  signal_dependents();
  if (item >= W.total) return;
  const SeqWork &s = W.s[find_seq(W, item)];
  const int64_t local = item - s.item0;
  const int head = (int)(local % L.hkv);
  const int64_t p = s.a + local / L.hkv;
  const SubLayout lay = sub_layout(FAM, BITS);
  uint8_t *sub = subpage_ptr(L, s.seq, p / GROUP, head, WHICH);
  float x[4];
  load4(L, s, head, WHICH, p, in, lane, x);
  const int tip = (int)(p % GROUP);
  if constexpr (FAM == FAM_SYM)
    quant_sym<BITS, WHICH>(x, sub, lay, tip, lane);
  else
    quant_asym<BITS, WHICH>(x, sub, lay, tip, lane);
}

constexpr int KV_THREADS = 512;  // 16 warps: two threads per row / token, 8 x 8 Sinkhorn tiles
constexpr int XS = D + 1;  // padded row stride of the fp32 tile in shared memory

struct KvarnSmem {
  float X[GROUP * XS];  // rotated rows x (fp32), padded rows
  float uS[32][8];      // 1/t^2 of token l + 32 k at [l][k]
  float tS[GROUP];      // token scales t
  float cS[D];          // channel scales c
  float wS[D];          // 1/c^2
  float part[16][GROUP];  // token-sum partials of the 16 runs of 8 channels
  float rc[D];          // 1/fp16(c)
  float rt[GROUP];      // 1/fp16(t)
  uint32_t img[GROUP * 16 * 8 / 4];  // packed code area of the sub-page (up to 8-bit codes)
};

// d = a*b + c on two fp32 lanes, each rounded once (the same result as two fmaf)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  memcpy(&ra, &a, 8);
  memcpy(&rb, &b, 8);
  memcpy(&rc, &c, 8);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  memcpy(&d, &rd, 8);
  return d;
}

// Packed fp32 pairs in one 64-bit register (sm_100 f32x2 arithmetic): each lane is rounded
// once, exactly as the scalar operation with the same operands.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// rint(RN(y / d)) for the codes of one block, by the reciprocal.  With rd = RN(1/d) and
// q = RN(y * rd), |q - RN(y / d)| <= 2^-15.4 for |q| <= 128 (two roundings of 2^-24 relative
// each, plus the quotient's own).  q + 1.5 * 2^23 rounds q to the nearest integer, ties to
// even, and its low bits are that integer in two's complement (the code, before masking);
// subtracting the constant back gives r = rint(q) exactly and t = q - r exactly.  Where
// |t| <= 0.5 - 2^-13 no half-integer lies between q and RN(y / d), so both round to r; where
// any |t| of the block is larger, the caller takes the exact quotients instead.
constexpr float kRintMagic = 12582912.0f;   // 1.5 * 2^23
constexpr float kTieBound = 0.4998779296875f;  // 0.5 - 2^-13

// Quantization of a balanced group (see k_spill_kvarn, step 4): warp w takes tokens
// 32 (w >> 1) + lane and blocks 2 (w & 1), 2 (w & 1) + 1, so that the lanes of a warp read
// distinct rows of the tile (conflict-free).  The block loop is kept rolled: its instruction
// footprint, not its arithmetic, sets the pace.
template <int BITS, int WHICH>
__device__ __forceinline__ void quant_rows(KvarnSmem &S, uint8_t *sub, const SubLayout &lay, int ng, int tid) {
  constexpr int QMAX = (1 << (BITS - 1)) - 1, QMIN = -(1 << (BITS - 1));
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  uint8_t *img = reinterpret_cast<uint8_t *>(S.img);
  const int tok = 32 * (tid >> 6) + (tid & 31), bhalf = (tid >> 5) & 1;
  if (tok < ng) {
    const float rti = S.rt[tok];
    const float *xr = &S.X[tok * XS];
    uint32_t dpair = 0u;  // fp16 d of the two blocks
#pragma unroll 1
    for (int bb = 0; bb < 2; ++bb) {
      const int blk = 2 * bhalf + bb;
      // y = (x * rc_j) * rt_i, two roundings, on channel pairs
      f32x2 yp[16];
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const f32x2 rcp = *reinterpret_cast<const f32x2 *>(&S.rc[32 * blk + 2 * i]);
        yp[i] = mul2(mul2(pk2(xr[32 * blk + 2 * i], xr[32 * blk + 2 * i + 1]), rcp), pk2(rti, rti));
        float y0, y1;
        upk2(yp[i], y0, y1);
        amax = max3(amax, fabsf(y0), fabsf(y1));
      }
      const __half dh = sat_half(__fdiv_rn(amax, (float)QMAX));
      const float df = __half2float(dh);
      const unsigned short dbits = __half_as_ushort(dh) & 0x7fffu;
      dpair |= (uint32_t)__half_as_ushort(dh) << (16 * bb);
      uint32_t f[32];  // low BITS bits: the code in two's complement
      // a normal, unsaturated d keeps |y / d| <= QMAX (1 + 2^-11): no clamp needed
      const bool plain = dbits >= 0x0400u && dbits != 0x7bffu;
      bool tie = !plain;
      if (plain) {
        const float rd = __frcp_rn(df);
        const f32x2 rd2 = pk2(rd, rd), mg = pk2(kRintMagic, kRintMagic);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const f32x2 q = mul2(yp[i], rd2);
          const f32x2 m = add2(q, mg);
          float t0, t1, m0, m1;
          upk2(sub2(q, sub2(m, mg)), t0, t1);
          upk2(m, m0, m1);
          tie |= fabsf(t0) > kTieBound;
          tie |= fabsf(t1) > kTieBound;
          f[2 * i] = __float_as_uint(m0);
          f[2 * i + 1] = __float_as_uint(m1);
        }
      }
      if (tie) {  // exact quotients (rare), clamped; d = 0 gives zero codes
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float y[2];
          upk2(yp[i], y[0], y[1]);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float rr = df != 0.0f ? fminf(fmaxf(rintf(__fdiv_rn(y[e], df)), (float)QMIN), (float)QMAX) : 0.0f;
            f[2 * i + e] = (uint32_t)(int)rr;
          }
        }
      }
#pragma unroll
      for (int pl = 0; pl < 2; ++pl) {
        const int w = pl == 0 ? WL : WH;
        if (w == 0) continue;
        const int shift_in = pl == 0 ? 0 : WL;
        const uint32_t wm = (1u << w) - 1u;
        const int F = 8 / w;
        if (WHICH == 0) {
          // K: channel 32 blk + 4 jj + k -> byte k of word (jj / F, blk), bits (jj % F) w
          uint8_t *plane = img + tok * 16 * BITS + (pl == 0 ? 0 : 16 * WL);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            if (m >= w) break;
            uint32_t word = 0;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              if (jj / F != m) continue;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                word |= ((f[4 * jj + kk] >> shift_in) & wm) << (8 * kk + (jj % F) * w);
            }
            *reinterpret_cast<uint32_t *>(plane + 16 * m + 4 * blk) = word;
          }
        } else {
          // V: channel 32 blk + e of quad token k -> byte k of word e / F of block blk,
          // bits (e % F) w
          uint8_t *plane = img + (tok >> 2) * 64 * BITS + (pl == 0 ? 0 : 64 * WL) + 16 * w * blk + (tok & 3);
#pragma unroll
          for (int m = 0; m < 32; ++m) {
            if (m >= 4 * w) break;
            uint32_t byte = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e / F != m) continue;
              byte |= ((f[e] >> shift_in) & wm) << ((e % F) * w);
            }
            plane[4 * m] = (uint8_t)byte;
          }
        }
      }
    }
    *reinterpret_cast<uint32_t *>(sub + lay.d + tok * 8 + 4 * bhalf) = dpair;
  }
  __syncthreads();
  const int nbytes = WHICH == 0 ? ng * 16 * BITS : ((ng + 3) / 4) * 64 * BITS;
  for (int p = tid; p < nbytes / 16; p += KV_THREADS)
    reinterpret_cast<uint4 *>(sub)[p] = reinterpret_cast<const uint4 *>(img)[p];
}

// One CTA (512 threads) per (kvarn group, head, K or V).  Per sequence, s.a is the first
// group the append touches (it may be a partial group that grows) and s.b the quantized
// length Q(n1) after the append; items enumerate (which, group, head) with which = 0 for the
// first W.total/2 items when K and V are processed by one launch (W.which == 2).
// TF16: the cache's tail is F16 (a separate instance, so that the BF16 instance is free of
// the conversions).
template <int BITS, int TF16>
__global__ void __launch_bounds__(KV_THREADS, 1)
    k_spill_kvarn(LayerView L, Work W, const __nv_bfloat16 *__restrict__ in_k, const __nv_bfloat16 *__restrict__ in_v,
                  int iters) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  KvarnSmem &S = *reinterpret_cast<KvarnSmem *>(smem_raw);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t item = blockIdx.x;
  int which = W.which;
  if (which == 2) {
    const int64_t half = W.total / 2;
    which = item >= half ? 1 : 0;
    if (which) item -= half;
  }
  const __nv_bfloat16 *in = which ? in_v : in_k;
  const SeqWork &s = W.s[find_seq(W, item)];
  const int64_t local = item - s.item0;
  const int head = (int)(local % L.hkv);
  const int64_t g = s.a + local / L.hkv;
  const int64_t g0 = g * GROUP;
  const int64_t Q1 = s.b;
  const int ng = (int)((Q1 - g0) < GROUP ? (Q1 - g0) : GROUP);
  const SubLayout lay = sub_layout(FAM_KVARN, BITS);
  uint8_t *sub = subpage_ptr(L, s.seq, g, head, which);
  signal_dependents();

  // 0. fused ring write: the CTA of the stream's last group copies the new rows that stay
  //    16-bit (16 threads per 256-byte row); no row it writes shares a slot with a row read here
  if (g0 + GROUP >= Q1) {
    for (int64_t p = s.tw + tid / 16; p < s.n1; p += KV_THREADS / 16) {
      const uint4 *src = reinterpret_cast<const uint4 *>(in + ((s.in_off + (p - s.n0)) * L.hkv + head) * D);
      reinterpret_cast<uint4 *>(ring_row(L, s.seq, head, which, p))[tid & 15] = bf16x8_to_ring(src[tid & 15], TF16);
    }
  }

  // 1. two threads per row rotate it: thread parity h keeps channels 2i + h.  Stage h = 1 pairs
  //    (2i, 2i+1), which both threads read from the whole row, and every later stage pairs
  //    channels of one parity (2i + h, 2(i + d) + h), so each thread runs it alone, two
  //    butterflies per packed add / sub; then x kappa.
  {
    const int row = tid >> 1, h = tid & 1;
    if (row < ng) {
      const uint4 *src = reinterpret_cast<const uint4 *>(src_row(L, s, head, which, g0 + row, in));
      // a ring row as stored; an input row rounded to the tail's format (F16 tails)
      const bool ring = g0 + row < s.n0;
      const int f16r = ring ? TF16 : 0, rnd = ring ? 0 : TF16;
      float r[D / 2];  // r[i] = channel 2i + h
      if (f16r | rnd) {
#pragma unroll
        for (int j8 = 0; j8 < D / 8; ++j8) {
          const uint4 raw = src[j8];
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 xf = ring2f(w[u], f16r);
            const float x0 = tail_round(xf.x, rnd), x1 = tail_round(xf.y, rnd);
            r[4 * j8 + u] = h ? __fsub_rn(x0, x1) : __fadd_rn(x0, x1);
          }
        }
      } else {
#pragma unroll
        for (int j8 = 0; j8 < D / 8; ++j8) {
          const uint4 raw = src[j8];
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float x0 = __uint_as_float(w[u] << 16), x1 = __uint_as_float(w[u] & 0xffff0000u);
            r[4 * j8 + u] = h ? __fsub_rn(x0, x1) : __fadd_rn(x0, x1);
          }
        }
      }
      f32x2 rp[D / 4];  // (r[2m], r[2m+1])
#pragma unroll
      for (int m = 0; m < D / 4; ++m) rp[m] = pk2(r[2 * m], r[2 * m + 1]);
      // stage d = 2 (r index distance 1) on scalars
#pragma unroll
      for (int m = 0; m < D / 4; ++m) {
        float a0, a1;
        upk2(rp[m], a0, a1);
        rp[m] = pk2(__fadd_rn(a0, a1), __fsub_rn(a0, a1));
      }
      // stages d = 4 .. 64 (distance dp = 1 .. 16 in pairs)
#pragma unroll
      for (int dp = 1; dp < D / 4; dp <<= 1) {
#pragma unroll
        for (int m = 0; m < D / 4; ++m) {
          if (m & dp) continue;
          const f32x2 a0 = rp[m], a1 = rp[m + dp];
          rp[m] = add2(a0, a1);
          rp[m + dp] = sub2(a0, a1);
        }
      }
      const f32x2 kk = pk2(kKappa(), kKappa());
#pragma unroll
      for (int m = 0; m < D / 4; ++m) {
        float a0, a1;
        upk2(mul2(rp[m], kk), a0, a1);
        S.X[row * XS + 4 * m + h] = a0;
        S.X[row * XS + 4 * m + 2 + h] = a1;
      }
    }
  }
  if (tid < GROUP) S.uS[tid & 31][tid >> 5] = 1.0f;  // first iteration: t = 1
  __syncthreads();

  // 2. Sinkhorn on the squared tile held in registers: thread (warp w, lane l) covers channels
  //    8w..8w+7 and tokens l + 32k (k = 0..7); rows past the group end square to 0.
  //    x2p[kp][c] holds tokens (l + 64 kp, l + 64 kp + 32) of channel 8w + c.
  float2 x2p[4][8];
#pragma unroll
  for (int kp = 0; kp < 4; ++kp)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i0 = lane + 64 * kp, i1 = i0 + 32;
      const float x0 = i0 < ng ? S.X[i0 * XS + 8 * warp + c] : 0.0f;
      const float x1 = i1 < ng ? S.X[i1 * XS + 8 * warp + c] : 0.0f;
      x2p[kp][c] = make_float2(__fmul_rn(x0, x0), __fmul_rn(x1, x1));
    }
  const float fng = (float)ng;
  // S / ng for a full group (ng = 256) is the exact product with 2^-8: the same rounded value
  // as the division, at the cost of one multiply
  const bool full = ng == GROUP;
  // channel index (within the warp's 8) this lane ends with after the recursive halving
  const int cidx = 4 * ((lane >> 4) & 1) + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);
  for (int it = 0; it < iters; ++it) {
    // channel step: S_j = sum_i x2_ij u_i.  Each lane chains its even-stride tokens
    // (l + 64 m) and its odd-stride tokens (l + 64 m + 32) separately, two chains per packed
    // FMA, adds the two, then the butterfly 16, 8, 4, 2, 1 across lanes (recursive halving)
    float2 u2[4];  // (u of token l + 64 kp, u of token l + 64 kp + 32)
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) u2[kp] = *reinterpret_cast<const float2 *>(&S.uS[lane][2 * kp]);
    float v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) acc = ffma2(x2p[kp][c], u2[kp], acc);
      v[c] = __fadd_rn(acc.x, acc.y);
    }
    {  // level 16: keep channels [4 b16, 4 b16 + 4)
      const bool hi = lane & 16;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float send = hi ? v[c] : v[c + 4];
        const float keep = hi ? v[c + 4] : v[c];
        v[c] = __fadd_rn(keep, __shfl_xor_sync(FULL, send, 16));
      }
    }
    {  // level 8
      const bool hi = lane & 8;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float send = hi ? v[c] : v[c + 2];
        const float keep = hi ? v[c + 2] : v[c];
        v[c] = __fadd_rn(keep, __shfl_xor_sync(FULL, send, 8));
      }
    }
    {  // level 4
      const bool hi = lane & 4;
      const float send = hi ? v[0] : v[1];
      const float keep = hi ? v[1] : v[0];
      v[0] = __fadd_rn(keep, __shfl_xor_sync(FULL, send, 4));
    }
    v[0] = __fadd_rn(v[0], __shfl_xor_sync(FULL, v[0], 2));  // level 2
    v[0] = __fadd_rn(v[0], __shfl_xor_sync(FULL, v[0], 1));  // level 1
    if ((lane & 3) == 0) {
      // the iterations carry w_j = 1 / c_j^2 = n / S_j; the scale itself comes from the last S
      S.cS[8 * warp + cidx] = v[0];
      S.wS[8 * warp + cidx] = v[0] > 0.0f ? __fdiv_rn(fng, v[0]) : 1.0f;
    }
    __syncwarp();
    // token step: R_i = sum_j x2_ij w_j; this warp's partial is the chain over its 8 channels
    // in order, two tokens per packed FMA
    float w[8];
    {
      const float4 wa = *reinterpret_cast<const float4 *>(&S.wS[8 * warp]);
      const float4 wb = *reinterpret_cast<const float4 *>(&S.wS[8 * warp + 4]);
      w[0] = wa.x; w[1] = wa.y; w[2] = wa.z; w[3] = wa.w;
      w[4] = wb.x; w[5] = wb.y; w[6] = wb.z; w[7] = wb.w;
    }
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc = ffma2(x2p[kp][c], make_float2(w[c], w[c]), acc);
      S.part[warp][lane + 64 * kp] = acc.x;
      S.part[warp][lane + 64 * kp + 32] = acc.y;
    }
    __syncthreads();
    if (tid < ng) {
      // the 16 run partials by the xor butterfly 8, 4, 2, 1
      float p[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) p[r] = S.part[r][tid];
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
        for (int r = 0; r < off; ++r) p[r] = __fadd_rn(p[r], p[r + off]);
      const float R = p[0];
      S.tS[tid] = R;  // u_i = 1 / t_i^2 = 128 / R_i; the scale itself comes from the last R
      S.uS[tid & 31][tid >> 5] = R > 0.0f ? __fdiv_rn(128.0f, R) : 1.0f;
    }
    __syncthreads();
  }

  // 3. scales from the last sums, c_j = sqrt(S_j / n) and t_i = sqrt(R_i / 128) (S_j / 256 and
  //    R_i / 128 are exact products), rounded to fp16; normalization uses the stored values
  if (tid < D) {
    const float Sj = S.cS[tid];
    const float c = (iters > 0 && Sj > 0.0f) ? __fsqrt_rn(full ? __fmul_rn(Sj, 1.0f / GROUP) : __fdiv_rn(Sj, fng)) : 1.0f;
    const __half h = scale_to_half(c);
    reinterpret_cast<__half *>(sub + lay.c)[tid] = h;
    S.rc[tid] = __frcp_rn(__half2float(h));
  }
  if (tid < ng) {
    const float Ri = S.tS[tid];
    const float t = (iters > 0 && Ri > 0.0f) ? __fsqrt_rn(__fmul_rn(Ri, 1.0f / D)) : 1.0f;
    const __half h = scale_to_half(t);
    reinterpret_cast<__half *>(sub + lay.t)[tid] = h;
    S.rt[tid] = __frcp_rn(__half2float(h));
  }
  __syncthreads();

  // 4. thread i quantizes token i: y = (x * rc_j) * rt_i, symmetric b-bit blocks of 32; the
  //    packed codes go to an image of the sub-page's code area in shared memory (it reuses
  //    the tile), which the CTA then copies out with 16-byte stores
  if (which == 0)
    quant_rows<BITS, 0>(S, sub, lay, ng, tid);
  else
    quant_rows<BITS, 1>(S, sub, lay, ng, tid);
}

// Copies new rows that stay 16-bit into the ring: range per sequence [a, n1), rows
// enumerated as (token, head), 16 threads per 256-byte row.
__global__ void __launch_bounds__(256) k_tail_write(LayerView L, Work W, const __nv_bfloat16 *__restrict__ in_k,
                                                    const __nv_bfloat16 *__restrict__ in_v) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t item = t >> 4;
  const int part = (int)(t & 15);
  signal_dependents();
  if (item >= W.total) return;
  int which = W.which;
  if (which == 2) {  // K and V in one launch: the first half of the items is K
    const int64_t half = W.total / 2;
    which = item >= half ? 1 : 0;
    if (which) item -= half;
  }
  const __nv_bfloat16 *in = which ? in_v : in_k;
  const SeqWork &s = W.s[find_seq(W, item)];
  const int64_t local = item - s.item0;
  const int head = (int)(local % L.hkv);
  const int64_t p = s.a + local / L.hkv;
  const uint4 *src = reinterpret_cast<const uint4 *>(in + ((s.in_off + (p - s.n0)) * L.hkv + head) * D);
  uint4 *dst = reinterpret_cast<uint4 *>(ring_row(L, s.seq, head, which, p));
  dst[part] = bf16x8_to_ring(src[part], L.tail_f16);
}

// ---- dispatch ----------------------------------------------------------------------------

template <int WHICH>
cudaError_t spill_qb(int fam, int bits, const LayerView &L, const Work &W, const __nv_bfloat16 *in,
                     cudaStream_t st) {
  const unsigned grid = (unsigned)((W.total + 7) / 8);
#define KVQ_QB(F, B) \
  if (fam == F && bits == B) { k_spill_qb<F, B, WHICH><<<grid, 256, 0, st>>>(L, W, in); return cudaGetLastError(); }
  KVQ_QB(FAM_SYM, 2) KVQ_QB(FAM_SYM, 3) KVQ_QB(FAM_SYM, 4) KVQ_QB(FAM_SYM, 5) KVQ_QB(FAM_SYM, 6)
  KVQ_QB(FAM_SYM, 8) KVQ_QB(FAM_ASYM, 2) KVQ_QB(FAM_ASYM, 3) KVQ_QB(FAM_ASYM, 4) KVQ_QB(FAM_ASYM, 5)
  KVQ_QB(FAM_ASYM, 6)
#undef KVQ_QB
  return cudaErrorInvalidValue;
}

template <int BITS, int TF16>
cudaError_t launch_kvarn_tf(const LayerView &L, const Work &W, const __nv_bfloat16 *in_k, const __nv_bfloat16 *in_v,
                            int iters, cudaStream_t st) {
  static bool attr_set = false;  // per template instance; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_spill_kvarn<BITS, TF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(KvarnSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  k_spill_kvarn<BITS, TF16><<<(unsigned)W.total, KV_THREADS, sizeof(KvarnSmem), st>>>(L, W, in_k, in_v, iters);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_kvarn_t(const LayerView &L, const Work &W, const __nv_bfloat16 *in_k, const __nv_bfloat16 *in_v,
                           int iters, cudaStream_t st) {
  return L.tail_f16 ? launch_kvarn_tf<BITS, 1>(L, W, in_k, in_v, iters, st)
                    : launch_kvarn_tf<BITS, 0>(L, W, in_k, in_v, iters, st);
}

cudaError_t spill_kvarn(int bits, const LayerView &L, const Work &W, const __nv_bfloat16 *in_k,
                        const __nv_bfloat16 *in_v, int iters, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_kvarn_t<2>(L, W, in_k, in_v, iters, st);
    case 3: return launch_kvarn_t<3>(L, W, in_k, in_v, iters, st);
    case 4: return launch_kvarn_t<4>(L, W, in_k, in_v, iters, st);
    case 5: return launch_kvarn_t<5>(L, W, in_k, in_v, iters, st);
    case 6: return launch_kvarn_t<6>(L, W, in_k, in_v, iters, st);
    case 8: return launch_kvarn_t<8>(L, W, in_k, in_v, iters, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int launch_append(const kvq_cache *c, int layer, const std::vector<AppendSeq> &seqs, const void *k,
                  const void *v, cudaStream_t st, AppendInfo *info) {
  AppendInfo local;
  AppendInfo &I = info ? *info : local;
  I = AppendInfo{};
  const LayerView L = layer_view(c, layer);
  const __nv_bfloat16 *in[2] = {static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v)};
  const int fam[2] = {c->fam_k, c->fam_v}, bits[2] = {c->bits_k, c->bits_v};
  const int64_t hkv = c->p.n_kv_heads;

  for (size_t base = 0; base < seqs.size(); base += MAXS) {
    const size_t cnt = std::min<size_t>(MAXS, seqs.size() - base);
    // 1. spill quantization: K and V in one launch when they share a kvarn type; that launch
    //    also writes the new ring rows when every sequence spills and, for each, the rows from
    //    the first one the spill reads to the last one written span at most the ring
    const bool fused = c->p.type_k == c->p.type_v && fam[0] == FAM_KVARN;
    bool ring_fused = fused;
    for (size_t i = 0; i < cnt && ring_fused; ++i) {
      const AppendSeq &a = seqs[base + i];
      const int64_t n1 = a.n0 + a.n_new;
      const int64_t Q0 = quantized_len(c, a.n0), Q1 = quantized_len(c, n1);
      if (Q1 <= Q0 || n1 - (Q0 / GROUP) * GROUP > c->ring_cap) ring_fused = false;
    }
    for (int which = 0; which < 2; ++which) {
      if (fam[which] == FAM_BF16) continue;
      if (fused && which == 1) continue;
      Work W{};
      W.which = fused ? 2 : which;
      int64_t total = 0;
      for (size_t i = 0; i < cnt; ++i) {
        const AppendSeq &a = seqs[base + i];
        SeqWork &s = W.s[W.n];
        s.seq = a.seq;
        s.n0 = a.n0;
        s.n1 = a.n0 + a.n_new;
        s.in_off = a.in_off;
        const int64_t ks = keep_start(c, fam[which], s.n1);
        s.tw = ring_fused ? (ks > s.n0 ? ks : s.n0) : s.n1;
        const int64_t Q0 = quantized_len(c, s.n0), Q1 = quantized_len(c, s.n1);
        if (Q1 <= Q0) continue;
        int64_t items;
        if (fam[which] == FAM_KVARN) {
          s.a = Q0 / GROUP;               // first group touched (may be partial)
          s.b = Q1;                       // quantized length after the append
          items = ((Q1 - 1) / GROUP - s.a + 1) * hkv;
        } else {
          s.a = Q0;
          s.b = Q1;
          items = (Q1 - Q0) * hkv;
        }
        s.item0 = total;
        total += items;
        ++W.n;
      }
      W.total = fused ? 2 * total : total;
      if (total == 0) continue;
      cudaError_t e = fam[which] == FAM_KVARN
                          ? spill_kvarn(bits[which], L, W, in[0], in[1], c->p.sinkhorn_iters, st)
                          : (which == 0 ? spill_qb<0>(fam[which], bits[which], L, W, in[which], st)
                                        : spill_qb<1>(fam[which], bits[which], L, W, in[which], st));
      if (e != cudaSuccess) return KVQ_E_CUDA;
      note_launches(1);
      ++I.launches;
    }
    if (ring_fused) continue;
    // 2. ring write of the new rows that stay 16-bit (K and V in one launch when their
    //    types keep the same rows)
    const bool same_keep = fam[0] == fam[1];
    for (int which = 0; which < 2; ++which) {
      if (same_keep && which == 1) continue;
      Work W{};
      W.which = same_keep ? 2 : which;
      int64_t total = 0;
      for (size_t i = 0; i < cnt; ++i) {
        const AppendSeq &a = seqs[base + i];
        SeqWork &s = W.s[W.n];
        s.seq = a.seq;
        s.n0 = a.n0;
        s.n1 = a.n0 + a.n_new;
        s.in_off = a.in_off;
        const int64_t ks = keep_start(c, fam[which], s.n1);
        s.a = ks > s.n0 ? ks : s.n0;
        s.b = s.n1;
        if (s.b <= s.a) continue;
        s.item0 = total;
        total += (s.b - s.a) * hkv;
        ++W.n;
      }
      W.total = same_keep ? 2 * total : total;
      if (total == 0) continue;
      const int64_t threads = W.total * 16;
      k_tail_write<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(L, W, in[0], in[1]);
      if (cudaGetLastError() != cudaSuccess) return KVQ_E_CUDA;
      note_launches(1);
      ++I.launches;
    }
  }
  return KVQ_OK;
}

}  // namespace kvq
