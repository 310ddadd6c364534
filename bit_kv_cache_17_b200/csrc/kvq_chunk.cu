// kvq_chunk.cu - attention of a chunk of queries over [quantized prefix | BF16 tail], causal
// within the chunk (the prefill side of the pages' prefill / decode split: "Fork of beellama and
// kvarn KV quants at long context", section "Which data should accompany a speed-up claim").
//
// A decode reads every cached token once per query row; a chunk of n_q queries would read it
// n_q times.  Here each 64-token tile of the cache is read and rebuilt once, into shared memory,
// for all n_q x G query rows of its KV head (up to 80 rows), and both products run on the
// fifth-generation tensor cores (tcgen05.mma, kind::f16, M = 128 rows, fp32 accumulators in
// tensor memory).  Warp roles:
//  - a copy warp moves the raw bytes of the next tiles (codes and scales) into a two-slot ring
//    with cp.async, its completion counted on an mbarrier;
//  - eight producer warps rebuild each tile: K-hat = code * d * t * c and V-hat = code * d * t * c
//    for kvarn, code * d for the symmetric formats (f16 pair arithmetic, each product split
//    exactly into a rounded part and its remainder), code * d + m for qb_1 (fp32), the 16-bit
//    rows as they are, stored as an f16 high part plus an f16 remainder (together about 22
//    significant bits) in the tensor core's no-swizzle canonical layouts (8 x 16-byte core
//    matrices);
//  - the query rows q' (times the softmax scale and log2 e; rotated, q' = H.q.kappa, for a
//    quantized kvarn K) are f16 high part + remainder too; one thread issues S = Q.K-hat^T as
//    hi.hi + lo.hi + hi.lo (24 MMAs of N = 64 per tile) into one of two S buffers in tensor
//    memory, and O += P.V-hat as p.hi + p.lo (8 MMAs of N = 128);
//  - four softmax warps own one query row per thread (the row's tensor-memory lane): they read
//    the row's 64 scores, keep the running maximum lazily (the weights 2^(s - m) stay below 2^4;
//    the accumulator is rescaled, in tensor memory, only when a score passes m + 4), and write
//    the weights as f16;
//  - mbarriers (tcgen05.commit for the tensor side) hand the raw, K, V, score and weight buffers
//    between the roles; every wait is bounded;
//  - each CTA covers a range of tiles of one KV head (split-K); k_chunk_merge combines the splits
//    (LSE) and applies the inverse WHT to the rotated V accumulator once per row.
// Values are limited to the f16 range (|x| < 65504) in this path.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int TT = 64;               // tokens per tile
constexpr int NQ = 16;               // query tokens per launch (at most MAXR / G)
constexpr int MAXR = 80;             // query rows per launch (of the MMA's 128; the rest unused)
constexpr int NSW = 4;               // softmax warps (row = thread = tensor-memory lane)
constexpr int MMA_WARP = 4;          // issues the MMAs, owns the tensor-memory allocation
constexpr int COPY_WARP = 5;         // copies the raw tiles (cp.async, completion on an mbarrier)
constexpr int NPW = 8;               // producer warps: tile rebuilding
constexpr int PW0 = 6;               // first producer warp
constexpr int NW = PW0 + NPW;        // 14 warps
constexpr int NT = 32 * NW;          // 448 threads
constexpr int NPT = 32 * NPW;        // 256 producer threads
constexpr int MAXSPL = 64;           // splits per KV head
constexpr int PSTRIDE = 4 + D;       // floats per partial record: m, l, 2 pad, acc[128]
constexpr float LOG2E = 1.4426950408889634f;
constexpr float TAU = 4.f;           // lazy rescale margin (log2 units)
constexpr uint32_t TMEM_COLS = 256;  // S buffers at columns 0 and 64, O at 128
constexpr uint32_t SUSPEND_NS = 100000;      // longest suspension of one mbarrier test (100 us)
constexpr long long WAIT_CYCLES = 1ll << 31;  // a wait gives up after about a second

// ---- shared memory map (bytes from a 1024-aligned base) ---------------------------------------
// Q: rows 0..79 of q' hi at 0 and lo at QLO, core matrix (r / 8, k / 8) at (r / 8) 2048 + (k / 8) 128;
//    an M = 128 MMA also reads rows 80..127 (past the hi rows into the lo rows, past the lo rows
//    into the K tiles): those rows of S are never used.
// K tiles (2): [hi | lo], each 64 tokens x 128 channels K-major, core (t / 8, k / 8) at
//    (t / 8) 2048 + (k / 8) 128.
// V tiles (2): [hi | lo], each MN-major (N = channel, K = token), core (c / 8, t / 8) at
//    (c / 8) 1024 + (t / 8) 128, a core row = one token's 8 channels.
// P: 128 rows x 64 tokens K-major, core (r / 8, t / 8) at (r / 8) 1024 + (t / 8) 128.
// raw tiles (2): the copied bytes of a quantized tile, K side then V side.
constexpr int OFF_Q = 0;
constexpr int QLO = 20480;
constexpr int OFF_K = 40960;
constexpr int TILE_B = 32768;  // one K or V tile, hi + lo
constexpr int HALF_B = 16384;
constexpr int OFF_V = OFF_K + 2 * TILE_B;
constexpr int OFF_P = OFF_V + 2 * TILE_B;
constexpr int OFF_RAW = OFF_P + 16384;

struct Ctl {
  uint64_t raw_full[2];   // copy warp (its 32 threads' cp.async completions) -> producers
  uint64_t raw_free[2];   // producers (one arrival per warp) -> copy warp
  uint64_t k_full[2];     // producers (one arrival per warp) -> MMA
  uint64_t v_full[2];     // producers (one arrival per warp) -> MMA
  uint64_t k_free[2];     // MMA commit after Q.K of the tile -> producers
  uint64_t v_free[2];     // MMA commit after P.V of the tile -> producers
  uint64_t s_full[2];     // MMA commit after Q.K -> softmax
  uint64_t s_free[2];     // softmax (one arrival per warp) -> MMA
  uint64_t p_full;        // softmax (one arrival per warp) -> MMA
  uint64_t pv_done;       // MMA commit after P.V -> softmax
  uint64_t last;          // MMA commit after its last MMA -> MMA warp (before the release)
  uint32_t tmem;
  int32_t abort;
};

struct CArgs {
  int32_t seq, nq, G, hkv, rotk, rotv;
  int32_t nsq, nst;      // splits per KV head over the quantized prefix / the 16-bit tail
  int32_t cps_q, cps_t;  // tiles per split
  int32_t fam_k, bits_k, fam_v, bits_v;
  int32_t raw_k;         // bytes of the K side of a raw tile (the V side follows)
  int32_t raw_b;         // bytes of a raw tile
  int64_t n, Q;          // sequence length (the chunk included), quantized tokens
  float qscale;          // softmax scale * log2(e)
  const float *q;        // [nq][hq][128]
  float *ws;             // records [qi][head][split][g][PSTRIDE]
};

// one side of a raw quantized tile: [codes][d 512][m 512 (qb_1)][t 128 (kvarn)][c 256 (kvarn)]; the
// codes of a K token (16 b bytes) or a V quad (64 b bytes) start every `stride` bytes, an odd number
// of 16-byte pieces, so that the 8 tokens (quads) a warp reads at once fall in 8 different banks
struct RawSide {
  int stride, d, m, t, c, bytes;
};
__host__ __device__ inline RawSide raw_side(int fam, int bits, int which) {
  RawSide r;
  r.stride = which ? 64 * bits + 16 : 16 * bits + ((bits & 1) ? 32 : 16);
  r.d = (which ? 16 : 64) * r.stride;
  int off = r.d + 512;
  r.m = off;
  if (fam == FAM_ASYM) off += 512;
  r.t = off;
  r.c = off + 128;
  if (fam == FAM_KVARN) off += 128 + 256;
  r.bytes = off;
  return r;
}

// ---- PTX wrappers -----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
// the mbarrier receives one arrival once all of this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// one arrival for the whole warp, after every lane's earlier shared-memory writes (the barrier
// counts warps)
__device__ __forceinline__ void mbar_arrive_warp(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
// tests the phase; the thread is suspended (not polling) until it completes or SUSPEND_NS pass
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(SUSPEND_NS)
      : "memory");
  return ok != 0;
}
// Waits for the phase of the given parity to complete.  Gives up after about a second (the
// CTA's abort flag set, the status word marked); once the flag is set every wait returns at
// once, so a CTA whose pipeline broke still runs to its end and releases its tensor memory
// (follow_abort false: the wait for the tensor core's own completion, which needs no other role,
// before the tensor memory is released)
__device__ __forceinline__ void mbar_wait(uint32_t bar, uint32_t parity, volatile int32_t *abort, int32_t *status,
                                          bool follow_abort = true) {
  if (mbar_try(bar, parity)) return;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try(bar, parity)) return;
    if (follow_abort && *abort) return;
    if (clock64() - t0 > WAIT_CYCLES) {
      *abort = 1;
      atomicOr(status, kStatusWait);
      return;
    }
  }
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// shared-memory matrix descriptor, no swizzle: start, leading (K-direction core matrix) and
// stride (M/N-direction core matrix) byte offsets, descriptor version 1
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
// instruction descriptor of kind::f16: f16 A and B, fp32 D, A K-major, B K- or MN-major
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn) {
  return (1u << 4) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
      "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
      "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }

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

template <int W>
__device__ __forceinline__ constexpr uint32_t bytes_mask() {
  return ((1u << W) - 1u) * 0x01010101u;
}

// four b-bit fields, one per byte of u, as floats: two's complement codes (sym / kvarn) or
// unsigned (qb_1).  Byte e of u (offset by 2^(b-1) for signed codes) becomes the low byte of the
// fp32 number 2^23 + byte, exactly; one subtraction leaves the code (no conversion instruction)
template <int FAM, int BITS>
__device__ __forceinline__ void fields_to_float(uint32_t u, float *c) {
  constexpr uint32_t bias = FAM == FAM_ASYM ? 0u : (1u << (BITS - 1));
  const uint32_t v = u ^ (bias * 0x01010101u);
  constexpr float off = 8388608.f + (float)bias;
#pragma unroll
  for (int e = 0; e < 4; ++e) c[e] = __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7440u + e)) - off;
}

// 8 fp32 values as f16 high parts and f16 remainders, stored as one 16-byte row each: the high
// part is x with its significand rounded to 11 bits (integer rounding of the fp32 pattern, then
// exact in f16 for values in the f16 range), the remainder x - hi is exact in fp32 and rounded once
__device__ __forceinline__ void store_hilo8(uint8_t *hi, uint8_t *lo, const float (&x)[8]) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float h0 = __uint_as_float((__float_as_uint(x[2 * i]) + 0x1000u) & 0xFFFFE000u);
    const float h1 = __uint_as_float((__float_as_uint(x[2 * i + 1]) + 0x1000u) & 0xFFFFE000u);
    h[i] = h2u(__floats2half2_rn(h0, h1));
    l[i] = h2u(__floats2half2_rn(x[2 * i] - h0, x[2 * i + 1] - h1));
  }
  *reinterpret_cast<uint4 *>(hi) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4 *>(lo) = make_uint4(l[0], l[1], l[2], l[3]);
}

// What a unit (one token, 8 channels) reads: its code fields (one per byte, two words) and the raw
// f16 scales: d (and t for kvarn, m for qb_1) of its (token, block), the 8 channel scales (kvarn)
struct UnitIn {
  uint32_t u0, u1;
  __half d, t, m;
  uint4 cw;
};

template <int FAM>
__device__ __forceinline__ void unit_scales(const uint8_t *side, const RawSide &r, int tok, int c8, bool ok,
                                            UnitIn &in) {
  const int blk = c8 >> 2;
  const __half zero = __ushort_as_half((unsigned short)0);
  in.d = ok ? reinterpret_cast<const __half *>(side + r.d)[tok * 4 + blk] : zero;
  in.m = (FAM == FAM_ASYM && ok) ? reinterpret_cast<const __half *>(side + r.m)[tok * 4 + blk] : zero;
  in.t = (FAM == FAM_KVARN && ok) ? reinterpret_cast<const __half *>(side + r.t)[tok] : zero;
  if (FAM == FAM_KVARN) in.cw = *reinterpret_cast<const uint4 *>(side + r.c + 16 * c8);
}

// four b-bit fields, one per byte of u, as two f16 pairs of the codes (exact): the byte (offset by
// 2^(b-1) for signed codes) is the low byte of the f16 number 1024 + byte
template <int FAM, int BITS>
__device__ __forceinline__ void fields_to_h2(uint32_t u, __half2 &c01, __half2 &c23) {
  constexpr uint32_t bias = FAM == FAM_ASYM ? 0u : (1u << (BITS - 1));
  const uint32_t v = u ^ (bias * 0x01010101u);
  const __half2 off = __float2half2_rn((float)(1024 + (int)bias));
  const uint32_t a = __byte_perm(v, 0x64646464u, 0x5140), b = __byte_perm(v, 0x64646464u, 0x5342);
  c01 = __hsub2(*reinterpret_cast<const __half2 *>(&a), off);
  c23 = __hsub2(*reinterpret_cast<const __half2 *>(&b), off);
}

// x = code * s (s = d, or d * t * c[ch] for kvarn) of the unit's 8 channels as f16 hi / lo rows, in
// f16 pair arithmetic: with a product a * b = p + e split exactly (p = RN(a b), e = fma(a, b, -p)),
// the per-channel scale s = s_hi + s_lo is formed first (|s| <= |x| for a nonzero code, so no step
// leaves the range of x), then hi = RN(code * s_hi) and lo = RN(code * s_lo + (code * s_hi - hi));
// for the block formats s = d is one f16 and hi + lo = code * d exactly.
template <int FAM, int BITS>
__device__ __forceinline__ void unit_store_h(const UnitIn &in, uint8_t *hi, uint8_t *lo) {
  __half2 c[4];
  fields_to_h2<FAM, BITS>(in.u0, c[0], c[1]);
  fields_to_h2<FAM, BITS>(in.u1, c[2], c[3]);
  __half2 sh = __half2half2(in.d), sl = __float2half2_rn(0.f);
  if constexpr (FAM == FAM_KVARN) {
    const __half2 t2 = __half2half2(in.t);
    const __half2 p = __hmul2(sh, t2);
    sl = __hfma2(sh, t2, __hneg2(p));
    sh = p;
  }
  const uint32_t cws[4] = {in.cw.x, in.cw.y, in.cw.z, in.cw.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 ah = sh, al = sl;
    if constexpr (FAM == FAM_KVARN) {
      const __half2 c2 = *reinterpret_cast<const __half2 *>(&cws[i]);
      ah = __hmul2(sh, c2);
      al = __hfma2(sl, c2, __hfma2(sh, c2, __hneg2(ah)));
    }
    const __half2 xh = __hmul2(c[i], ah);
    const __half2 xl = __hfma2(c[i], al, __hfma2(c[i], ah, __hneg2(xh)));
    h[i] = h2u(xh);
    l[i] = h2u(xl);
  }
  *reinterpret_cast<uint4 *>(hi) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4 *>(lo) = make_uint4(l[0], l[1], l[2], l[3]);
}

// qb_1: x = code * d + m in fp32, stored as f16 hi / lo rows
template <int FAM, int BITS>
__device__ __forceinline__ void unit_store_f(const UnitIn &in, uint8_t *hi, uint8_t *lo) {
  float c[8], x[8];
  fields_to_float<FAM, BITS>(in.u0, c);
  fields_to_float<FAM, BITS>(in.u1, c + 4);
  const float d = __half2float(in.d), m = __half2float(in.m);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = fmaf(c[e], d, m);
  store_hilo8(hi, lo, x);
}

template <int FAM, int BITS>
__device__ __forceinline__ void unit_store(const UnitIn &in, uint8_t *hi, uint8_t *lo) {
  if constexpr (FAM == FAM_ASYM)
    unit_store_f<FAM, BITS>(in, hi, lo);
  else
    unit_store_h<FAM, BITS>(in, hi, lo);
}

// K unit: token tok, channels 8 c8 .. 8 c8 + 7 (K layout: channel 32 blk + 4 jj + k is byte k of
// plane word (jj / F, blk))
template <int FAM, int BITS>
__device__ __forceinline__ UnitIn k_load(const uint8_t *side, const RawSide &r, int tok, int c8, bool ok) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  constexpr int FL = 8 / WL, FH = WH ? 8 / WH : 1;
  const int blk = c8 >> 2, jj0 = 2 * (c8 & 3);
  const uint8_t *tp = side + tok * r.stride;
  const uint32_t w0 = *reinterpret_cast<const uint32_t *>(tp + 16 * (jj0 / FL) + 4 * blk);
  const uint32_t w1 = FL >= 2 ? w0 : *reinterpret_cast<const uint32_t *>(tp + 16 * ((jj0 + 1) / FL) + 4 * blk);
  UnitIn in;
  in.u0 = (w0 >> ((jj0 % FL) * WL)) & bytes_mask<WL>();
  in.u1 = (w1 >> (((jj0 + 1) % FL) * WL)) & bytes_mask<WL>();
  if constexpr (WH > 0) {
    const uint32_t h = *reinterpret_cast<const uint32_t *>(tp + 16 * WL + 16 * (jj0 / FH) + 4 * blk);
    in.u0 |= ((h >> ((jj0 % FH) * WH)) & bytes_mask<WH>()) << WL;
    in.u1 |= ((h >> (((jj0 + 1) % FH) * WH)) & bytes_mask<WH>()) << WL;
  }
  unit_scales<FAM>(side, r, tok, c8, ok, in);
  return in;
}

// V unit: token tok (byte tok % 4 of its quad's words), channels 8 c8 .. 8 c8 + 7 (V layout:
// channel 32 blk + e of quad token k is byte k of plane word e / F of block blk)
template <int FAM, int BITS>
__device__ __forceinline__ UnitIn v_load(const uint8_t *side, const RawSide &r, int tok, int c8, bool ok) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  constexpr int FL = 8 / WL, FH = WH ? 8 / WH : 1;
  constexpr int NL = 8 / FL, NH = WH ? 8 / FH : 0;  // plane words holding the 8 channels
  const int blk = c8 >> 2, e0 = 8 * (c8 & 3), k = tok & 3;
  const uint8_t *qp = side + (tok >> 2) * r.stride;
  uint32_t wl[NL], wh[NH > 0 ? NH : 1];
#pragma unroll
  for (int i = 0; i < NL; ++i) wl[i] = *reinterpret_cast<const uint32_t *>(qp + 16 * WL * blk + 4 * (e0 / FL + i));
#pragma unroll
  for (int i = 0; i < NH; ++i)
    wh[i] = *reinterpret_cast<const uint32_t *>(qp + 64 * WL + 16 * WH * blk + 4 * (e0 / FH + i));
  UnitIn in;
  uint32_t u[2] = {0u, 0u};
  if constexpr (BITS == 4) {
    // byte k of the 4 words (channels e0 + 2 i, e0 + 2 i + 1 in its nibbles), then even / odd nibbles
    const uint32_t sel = (uint32_t)k | ((uint32_t)(4 + k) << 4);
    const uint32_t x = __byte_perm(__byte_perm(wl[0], wl[1], sel), __byte_perm(wl[2], wl[3], sel), 0x5410);
    const uint32_t ev = x & 0x0f0f0f0fu, od = (x >> 4) & 0x0f0f0f0fu;
    u[0] = __byte_perm(ev, od, 0x5140);
    u[1] = __byte_perm(ev, od, 0x7362);
  } else
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    uint32_t f = (wl[e / FL] >> (8 * k + (e % FL) * WL)) & ((1u << WL) - 1u);
    if constexpr (WH > 0) f |= ((wh[e / FH] >> (8 * k + (e % FH) * WH)) & ((1u << WH) - 1u)) << WL;
    u[e >> 2] |= f << (8 * (e & 3));
  }
  in.u0 = u[0];
  in.u1 = u[1];
  unit_scales<FAM>(side, r, tok, c8, ok, in);
  return in;
}

// The K (V) tile of a quantized raw tile: 1024 units, one at a time per producer thread (a
// smaller loop body measured faster than two units in flight); a warp's 32 units fill four
// core matrices (conflict-free 16-byte stores, 8 lanes per core matrix) and read 8 tokens
// (quads) of the padded raw rows, 8 banks apart.  K: unit u = (token 8 (u / 128) + u % 8,
// c8 = 4 ((u / 8) % 4) + (u / 32) % 4), the lanes of a warp spanning the 4 blocks;
// V: (token 8 ((u / 8) % 8) + u % 8, c8 = u / 64).
template <int FAM, int BITS>
__device__ __forceinline__ void rebuild_k(const uint8_t *side, uint8_t *kt, int nvalid, int pt) {
  const RawSide r = raw_side(FAM, BITS, 0);
#pragma unroll 1
  for (int u = pt; u < 1024; u += NPT) {
    const int tok = 8 * (u >> 7) + (u & 7), c8 = 4 * ((u >> 3) & 3) + ((u >> 5) & 3);
    const UnitIn in = k_load<FAM, BITS>(side, r, tok, c8, tok < nvalid);
    uint8_t *dst = kt + (tok >> 3) * 2048 + c8 * 128 + (tok & 7) * 16;
    unit_store<FAM, BITS>(in, dst, dst + HALF_B);
  }
}
template <int FAM, int BITS>
__device__ __forceinline__ void rebuild_v(const uint8_t *side, uint8_t *vt, int nvalid, int pt) {
  const RawSide r = raw_side(FAM, BITS, 1);
#pragma unroll 1
  for (int u = pt; u < 1024; u += NPT) {
    const int tok = 8 * ((u >> 3) & 7) + (u & 7), c8 = u >> 6;
    const UnitIn in = v_load<FAM, BITS>(side, r, tok, c8, tok < nvalid);
    uint8_t *dst = vt + c8 * 1024 + (tok >> 3) * 128 + (tok & 7) * 16;
    unit_store<FAM, BITS>(in, dst, dst + HALF_B);
  }
}

#define KVQ_EACH_QTYPE(X)                                                                               \
  X(FAM_SYM, 2) X(FAM_SYM, 3) X(FAM_SYM, 4) X(FAM_SYM, 5) X(FAM_SYM, 6) X(FAM_SYM, 8) X(FAM_ASYM, 2)     \
  X(FAM_ASYM, 3) X(FAM_ASYM, 4) X(FAM_ASYM, 5) X(FAM_ASYM, 6) X(FAM_KVARN, 2) X(FAM_KVARN, 3)           \
  X(FAM_KVARN, 4) X(FAM_KVARN, 5) X(FAM_KVARN, 6) X(FAM_KVARN, 8)

__device__ __forceinline__ void rebuild_k_dispatch(int fam, int bits, const uint8_t *side, uint8_t *kt, int nvalid, int pt) {
#define KVQ_RK(F, B)                              \
  if (fam == F && bits == B) {                    \
    rebuild_k<F, B>(side, kt, nvalid, pt);   \
    return;                                       \
  }
  KVQ_EACH_QTYPE(KVQ_RK)
#undef KVQ_RK
}
__device__ __forceinline__ void rebuild_v_dispatch(int fam, int bits, const uint8_t *side, uint8_t *vt, int nvalid, int pt) {
#define KVQ_RV(F, B)                              \
  if (fam == F && bits == B) {                    \
    rebuild_v<F, B>(side, vt, nvalid, pt);   \
    return;                                       \
  }
  KVQ_EACH_QTYPE(KVQ_RV)
#undef KVQ_RV
}
#undef KVQ_EACH_QTYPE

// One side of a tail tile: 16-bit rows (BF16 or F16 ring) straight from global memory, four rows
// pieces per thread loaded before any is stored; rows past the end are zero
__device__ __forceinline__ void rebuild_ring(const LayerView &L, int seq, int head, int side, int64_t i0, int nvalid,
                                             uint8_t *t, int pt) {
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int u = pt + NPT * i;
    const int tok = side ? 8 * ((u >> 3) & 7) + (u & 7) : 8 * (u >> 7) + (u & 7);
    const int c8 = side ? (u >> 6) & 15 : (u >> 3) & 15;
    v[i] = u < 1024 && tok < nvalid
               ? *reinterpret_cast<const uint4 *>(ring_row(L, seq, head, side, i0 + tok) + 8 * c8)
               : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int u = pt + NPT * i;
    if (u >= 1024) break;
    const int tok = side ? 8 * ((u >> 3) & 7) + (u & 7) : 8 * (u >> 7) + (u & 7);
    const int c8 = side ? u >> 6 : (u >> 3) & 15;
    const float2 a = ring2f(v[i].x, L.tail_f16), b = ring2f(v[i].y, L.tail_f16), c = ring2f(v[i].z, L.tail_f16),
                 d = ring2f(v[i].w, L.tail_f16);
    const float x[8] = {a.x, a.y, b.x, b.y, c.x, c.y, d.x, d.y};
    uint8_t *dst = side ? t + c8 * 1024 + (tok >> 3) * 128 + (tok & 7) * 16 : t + (tok >> 3) * 2048 + c8 * 128 + (tok & 7) * 16;
    store_hilo8(dst, dst + HALF_B, x);
  }
}

// Copies quantized tile [i0, i0 + 64) of one KV head (inside one page) into a raw slot: codes,
// d (and m, t, c) of K then V; 16 bytes per copy, by the 32 lanes of the copy warp.
__device__ __forceinline__ void copy_tile(const LayerView &L, const CArgs &A, int head, int64_t i0, uint32_t slot,
                                          int lane) {
  const int64_t page = i0 / GROUP;
  const int tip0 = (int)(i0 % GROUP);
  const uint8_t *sk = subpage_ptr(L, A.seq, page, head, 0);
#pragma unroll
  for (int side = 0; side < 2; ++side) {
    const int fam = side ? A.fam_v : A.fam_k, bits = side ? A.bits_v : A.bits_k;
    const uint8_t *sub = side ? sk + L.sub_k : sk;
    const uint32_t dst = slot + (side ? A.raw_k : 0);
    const SubLayout lay = sub_layout(fam, bits);
    const RawSide r = raw_side(fam, bits, side);
    // the tile's codes: 64 tokens (16 quads) contiguous in the page, 16-byte pieces, each token's
    // (quad's) pieces at the padded row stride
    const int ncode = 64 * bits, per = side ? 4 * bits : bits;
    for (int p = lane; p < ncode; p += 32) {
      const int row = p / per;
      cp_async16(dst + row * r.stride + 16 * (p - row * per), sub + tip0 * 16 * bits + 16 * p);
    }
    cp_async16(dst + r.d + 16 * lane, sub + lay.d + tip0 * 8 + 16 * lane);  // d: 32 pieces
    if (fam == FAM_ASYM) cp_async16(dst + r.m + 16 * lane, sub + lay.m + tip0 * 8 + 16 * lane);
    if (fam == FAM_KVARN && lane < 8) cp_async16(dst + r.t + 16 * lane, sub + lay.t + tip0 * 2 + 16 * lane);
    if (fam == FAM_KVARN && lane < 16) cp_async16(dst + r.c + 16 * lane, sub + lay.c + 16 * lane);
  }
}

__global__ void __launch_bounds__(NT, 1) k_chunk(LayerView L, CArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t *S = smem_raw + pad;
  const uint32_t base = raw_base + pad;
  Ctl &C = *reinterpret_cast<Ctl *>(S + OFF_RAW + 2 * A.raw_b);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nspl = A.nsq + A.nst;
  const int head = blockIdx.x / nspl, sp = blockIdx.x % nspl;
  const int G = A.G, R = A.nq * G;
  const bool tail = sp >= A.nsq;
  int64_t a, b;
  if (!tail) {
    a = (int64_t)sp * A.cps_q * TT;
    b = min(a + (int64_t)A.cps_q * TT, A.Q);
  } else {
    a = A.Q + (int64_t)(sp - A.nsq) * A.cps_t * TT;
    b = min(a + (int64_t)A.cps_t * TT, A.n);
  }
  const int ntile = b > a ? (int)((b - a + TT - 1) / TT) : 0;
  const uint32_t cb = smem_u32(&C);
  const uint32_t bar_raw_full = cb + (uint32_t)offsetof(Ctl, raw_full), bar_raw_free = cb + (uint32_t)offsetof(Ctl, raw_free);
  const uint32_t bar_k_full = cb + (uint32_t)offsetof(Ctl, k_full), bar_v_full = cb + (uint32_t)offsetof(Ctl, v_full);
  const uint32_t bar_k_free = cb + (uint32_t)offsetof(Ctl, k_free), bar_v_free = cb + (uint32_t)offsetof(Ctl, v_free);
  const uint32_t bar_s_full = cb + (uint32_t)offsetof(Ctl, s_full), bar_s_free = cb + (uint32_t)offsetof(Ctl, s_free);
  const uint32_t bar_p_full = cb + (uint32_t)offsetof(Ctl, p_full), bar_pv_done = cb + (uint32_t)offsetof(Ctl, pv_done);
  const uint32_t bar_last = cb + (uint32_t)offsetof(Ctl, last);
  volatile int32_t *abort = &C.abort;

  if (warp == COPY_WARP) {
    // the raw-tile barriers, then the first two tiles in flight while q' is computed
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar_raw_full + 8 * i, 32);
        mbar_init(bar_raw_free + 8 * i, NPW);
      }
    }
    __syncwarp();
    if (!tail) {
#pragma unroll 1
      for (int t = 0; t < 2 && t < ntile; ++t) {
        copy_tile(L, A, head, a + (int64_t)t * TT, base + OFF_RAW + t * A.raw_b, lane);
        cp_async_mbar_arrive(bar_raw_full + 8 * t);
      }
    }
  } else if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_k_full + 8 * i, NPW);
      mbar_init(bar_v_full + 8 * i, NPW);
      mbar_init(bar_k_free + 8 * i, 1);
      mbar_init(bar_v_free + 8 * i, 1);
      mbar_init(bar_s_full + 8 * i, 1);
      mbar_init(bar_s_free + 8 * i, NSW);
    }
    mbar_init(bar_p_full, NSW);
    mbar_init(bar_pv_done, 1);
    mbar_init(bar_last, 1);
    C.abort = 0;
  }
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(cb + (uint32_t)offsetof(Ctl, tmem)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // q' of rows 0..79 (row = qi * G + hd; rows past R are zero), scaled by softmax scale * log2(e)
  // and, for a quantized kvarn K, rotated; warp per row (all warps but the copy warp), lane = 4
  // channels; f16 hi / lo
  if (warp != COPY_WARP) {
    const int qw = warp < COPY_WARP ? warp : warp - 1;
    for (int row = qw; row < MAXR; row += NW - 1) {
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (row < R) {
        const int qi = row / G, hd = row % G;
        const float4 x =
            __ldg(reinterpret_cast<const float4 *>(A.q + ((int64_t)qi * A.hkv * G + head * G + hd) * D) + lane);
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
      const __half2 h01 = __floats2half2_rn(v[0], v[1]), h23 = __floats2half2_rn(v[2], v[3]);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      const __half2 l01 = __floats2half2_rn(v[0] - f01.x, v[1] - f01.y);
      const __half2 l23 = __floats2half2_rn(v[2] - f23.x, v[3] - f23.y);
      uint8_t *dst = S + OFF_Q + (row >> 3) * 2048 + (lane >> 1) * 128 + (row & 7) * 16 + (lane & 1) * 8;
      *reinterpret_cast<uint2 *>(dst) = make_uint2(h2u(h01), h2u(h23));
      *reinterpret_cast<uint2 *>(dst + QLO) = make_uint2(h2u(l01), h2u(l23));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = C.tmem;

  if (warp == COPY_WARP) {
    // ---- copy warp: raw tile t into slot t % 2 once the producers are done with tile t - 2
    if (!tail) {
#pragma unroll 1
      for (int t = 2; t < ntile; ++t) {
        const int tb = t & 1;
        mbar_wait(bar_raw_free + 8 * tb, ((t - 2) >> 1) & 1, abort, L.status);
        copy_tile(L, A, head, a + (int64_t)t * TT, base + OFF_RAW + tb * A.raw_b, lane);
        cp_async_mbar_arrive(bar_raw_full + 8 * tb);
      }
    }
    cp_async_wait<0>();
  } else if (warp >= PW0) {
    // ---- producers: the K tile, then the V tile, of each tile of the split
    const int pt = tid - 32 * PW0;
#pragma unroll 1
    for (int t = 0; t < ntile; ++t) {
      const int tb = t & 1;
      const int64_t i0 = a + (int64_t)t * TT;
      const int nvalid = (int)min((int64_t)TT, b - i0);
      const uint8_t *raw = S + OFF_RAW + tb * A.raw_b;
      if (!tail) mbar_wait(bar_raw_full + 8 * tb, (t >> 1) & 1, abort, L.status);
      if (t >= 2) mbar_wait(bar_k_free + 8 * tb, ((t - 2) >> 1) & 1, abort, L.status);
      uint8_t *kt = S + OFF_K + tb * TILE_B;
      if (!tail)
        rebuild_k_dispatch(A.fam_k, A.bits_k, raw, kt, nvalid, pt);
      else
        rebuild_ring(L, A.seq, head, 0, i0, nvalid, kt, pt);
      fence_async_smem();
      mbar_arrive_warp(bar_k_full + 8 * tb);
      if (t >= 2) mbar_wait(bar_v_free + 8 * tb, ((t - 2) >> 1) & 1, abort, L.status);
      uint8_t *vt = S + OFF_V + tb * TILE_B;
      if (!tail)
        rebuild_v_dispatch(A.fam_v, A.bits_v, raw + A.raw_k, vt, nvalid, pt);
      else
        rebuild_ring(L, A.seq, head, 1, i0, nvalid, vt, pt);
      fence_async_smem();
      mbar_arrive_warp(bar_v_full + 8 * tb);
      if (!tail) mbar_arrive_warp(bar_raw_free + 8 * tb);
    }
  } else if (warp == MMA_WARP) {
    // ---- one thread issues S = Q.K^T (tile t) and O += P.V (tile t - 1)
    if (lane == 0 && ntile > 0) {
      const uint32_t idS = idesc_f16(128, TT, 0), idO = idesc_f16(128, D, 1);
      const uint64_t qh = smem_desc(base + OFF_Q, 128, 2048), ql = smem_desc(base + OFF_Q + QLO, 128, 2048);
      const uint64_t pd = smem_desc(base + OFF_P, 128, 1024);
      auto pv = [&](int u) {
        mbar_wait(bar_p_full, u & 1, abort, L.status);
        mbar_wait(bar_v_full + 8 * (u & 1), (u >> 1) & 1, abort, L.status);
        tc_fence_after();
        const uint32_t vbase = base + OFF_V + (u & 1) * TILE_B;
        const uint64_t vh = smem_desc(vbase, 128, 1024), vl = smem_desc(vbase + HALF_B, 128, 1024);
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk) {
          const uint64_t o = (uint64_t)(kk * 16);  // 256 bytes: two core matrices along the tokens
          umma(tm + 128, pd + o, vh + o, idO, (u > 0 || kk > 0) ? 1u : 0u);
          umma(tm + 128, pd + o, vl + o, idO, 1u);
        }
        umma_commit(bar_v_free + 8 * (u & 1));
        umma_commit(bar_pv_done);
      };
#pragma unroll 1
      for (int t = 0; t < ntile; ++t) {
        const int tb = t & 1;
        mbar_wait(bar_k_full + 8 * tb, (t >> 1) & 1, abort, L.status);
        if (t >= 2) mbar_wait(bar_s_free + 8 * tb, ((t - 2) >> 1) & 1, abort, L.status);
        tc_fence_after();
        const uint32_t kb = base + OFF_K + tb * TILE_B;
        const uint64_t kh = smem_desc(kb, 128, 2048), kl = smem_desc(kb + HALF_B, 128, 2048);
        const uint32_t d = tm + TT * tb;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t o = (uint64_t)(ks * 16);  // 256 bytes: two core matrices along the channels
          umma(d, qh + o, kh + o, idS, ks > 0 ? 1u : 0u);
          umma(d, ql + o, kh + o, idS, 1u);
          umma(d, qh + o, kl + o, idS, 1u);
        }
        umma_commit(bar_s_full + 8 * tb);
        umma_commit(bar_k_free + 8 * tb);
        if (t >= 1) pv(t - 1);
      }
      pv(ntile - 1);
      umma_commit(bar_last);
      mbar_wait(bar_last, 0, abort, L.status, false);
    }
    __syncwarp();
  } else {
    // ---- softmax warps: row = tid, tensor-memory lane = tid
    const int row = tid;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const bool active = row < R;
    const int64_t lim = active ? min(b, A.n - A.nq + 1 + row / G) : a;  // tokens < lim are visible
    float m_used = -INFINITY, l = 0.f;
    uint8_t *prow = S + OFF_P + (row >> 3) * 1024 + (row & 7) * 16;
#pragma unroll 1
    for (int t = 0; t < ntile; ++t) {
      const int tb = t & 1;
      const int64_t i0 = a + (int64_t)t * TT;
      mbar_wait(bar_s_full + 8 * tb, (t >> 1) & 1, abort, L.status);
      tc_fence_after();
      float s[TT];
      tmem_ld32(tm + lane_base + TT * tb, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(tm + lane_base + TT * tb + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_warp(bar_s_free + 8 * tb);
      // causal / range mask; rows past R see nothing
      if (i0 + TT > lim) {
#pragma unroll
        for (int j = 0; j < TT; ++j)
          if (i0 + j >= lim) s[j] = -INFINITY;
      }
      float cmax = s[0];
#pragma unroll
      for (int j = 1; j < TT; ++j) cmax = fmaxf(cmax, s[j]);
      float al = 1.f;
      if (cmax > m_used + TAU) {  // also the first visible score (m_used = -inf)
        al = exp2_fast(m_used - cmax);
        m_used = cmax;
        l *= al;
      }
      // the weight buffer and the accumulator are free once P.V of tile t - 1 is done
      if (t >= 1) {
        mbar_wait(bar_pv_done, (t - 1) & 1, abort, L.status);
        tc_fence_after();
        if (__any_sync(FULL, al != 1.f)) {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            float o[32];
            tmem_ld32(tm + lane_base + 128 + 32 * c4, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] *= al;
            tmem_st32(tm + lane_base + 128 + 32 * c4, o);
          }
          tmem_wait_st();
        }
      }
      float ps = 0.f;
      uint32_t pw[TT / 2];
#pragma unroll
      for (int j = 0; j < TT; j += 2) {
        const float p0 = m_used == -INFINITY ? 0.f : exp2_fast(s[j] - m_used);
        const float p1 = m_used == -INFINITY ? 0.f : exp2_fast(s[j + 1] - m_used);
        ps += p0 + p1;
        pw[j / 2] = h2u(__floats2half2_rn(p0, p1));
      }
      l += ps;
#pragma unroll
      for (int t8 = 0; t8 < TT / 8; ++t8)
        *reinterpret_cast<uint4 *>(prow + t8 * 128) = make_uint4(pw[4 * t8], pw[4 * t8 + 1], pw[4 * t8 + 2], pw[4 * t8 + 3]);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive_warp(bar_p_full);
    }
    // ---- this split's record of the row: m, l, acc (rotated basis for a quantized kvarn V)
    if (ntile > 0) {
      mbar_wait(bar_pv_done, (ntile - 1) & 1, abort, L.status);
      tc_fence_after();
    }
    const int qi = active ? row / G : 0, hd = active ? row % G : 0;
    float *rec = A.ws + ((((int64_t)qi * A.hkv + head) * nspl + sp) * G + hd) * PSTRIDE;
#pragma unroll 1
    for (int c4 = 0; c4 < 4; ++c4) {
      float o[32];
      if (ntile > 0) {
        tmem_ld32(tm + lane_base + 128 + 32 * c4, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0.f;
      }
      if (active) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4 *>(rec + 4 + 32 * c4 + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
      }
    }
    if (active) {
      rec[0] = m_used;
      rec[1] = l;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(TMEM_COLS));
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

// dynamic shared memory of a launch: the fixed buffers, two raw tiles, the control block, the
// alignment slack
size_t chunk_smem_bytes(int raw_b) { return (size_t)OFF_RAW + 2 * (size_t)raw_b + sizeof(Ctl) + 1024; }

}  // namespace

size_t chunk_workspace_bytes(const kvq_cache *c, int n_q_tokens, int n_q_heads) {
  const int G = n_q_heads / c->p.n_kv_heads;
  return sizeof(float) * (size_t)std::min(std::max(n_q_tokens, 1), NQ) * c->p.n_kv_heads * MAXSPL * G * PSTRIDE;
}

int launch_chunk(const kvq_cache *c, int layer, int seq, int n_q, int n_q_heads, const float *q, float scale,
                 float *out, void *ws, cudaStream_t st) {
  static size_t attr_bytes = 0;
  const LayerView L = layer_view(c, layer);
  const int hkv = c->p.n_kv_heads, G = n_q_heads / hkv;
  const int64_t n = c->len[(size_t)layer * c->p.n_seqs + seq];
  const int64_t Q = quantized_len(c, n);
  const int raw_k = c->fam_k == FAM_BF16 ? 0 : raw_side(c->fam_k, c->bits_k, 0).bytes;
  const int raw_v = c->fam_v == FAM_BF16 ? 0 : raw_side(c->fam_v, c->bits_v, 1).bytes;
  const int raw_b = ((raw_k + raw_v + 15) / 16) * 16;
  const size_t smem = chunk_smem_bytes(raw_b);
  if (smem > attr_bytes) {
    if (cudaFuncSetAttribute(k_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return KVQ_E_CUDA;
    attr_bytes = smem;
  }
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
    A.raw_k = raw_k;
    A.raw_b = raw_b;
    // the rows of this launch are query tokens q0 .. q0 + nq - 1 of the chunk: their context is
    // the sequence cut after the last of them
    A.n = n - (n_q - q0 - nq);
    A.Q = std::min(Q, A.n);
    A.qscale = scale * LOG2E;
    A.q = q + (size_t)q0 * n_q_heads * D;
    A.ws = static_cast<float *>(ws);
    // splits: about one CTA per SM over the KV heads, quantized and 16-bit tokens in proportion
    // to their tiles, at least one split for each part that has tokens, at most MAXSPL in all
    const int64_t chq = (A.Q + TT - 1) / TT, cht = (A.n - A.Q + TT - 1) / TT;
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
    k_chunk<<<(unsigned)(hkv * (A.nsq + A.nst)), NT, smem, st>>>(L, A);
    if (cudaGetLastError() != cudaSuccess) return KVQ_E_CUDA;
    const int64_t warps = (int64_t)nq * n_q_heads;
    k_chunk_merge<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(A, out + (size_t)q0 * n_q_heads * D);
    if (cudaGetLastError() != cudaSuccess) return KVQ_E_CUDA;
    note_launches(2);
  }
  return KVQ_OK;
}

}  // namespace kvq
