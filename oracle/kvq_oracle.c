/*
 * kvq_oracle.c - the CPU oracle.  TEST INFRASTRUCTURE ONLY (see kvq_oracle.h).
 *
 * Built with gcc -O2 -ffp-contract=off -fno-fast-math: every fp32 expression below is
 * evaluated exactly as written (one IEEE round per operation, fmaf only where named).
 *
 * What pins each part (tests/test_oracle_*.py):
 *   number formats   - exhaustive/bit-pattern checks against numpy's own fp16 cast and
 *                      the bf16 definition (truncate + round-to-nearest-even).
 *   kvqo_wht128      - e_k maps to column k of the Sylvester matrix H_ij = (-1)^popcount(i&j)
 *                      times kappa; H.H^T = 128 I in integers; rotate->rotate returns the
 *                      input within the fp32 error bound; matches an fp64 matrix product.
 *   kvqo_sinkhorn    - agrees with the literal fp64 form (kvqo_sinkhorn_literal) and with a
 *                      numpy restatement of the literal form; token RMS == 1 after the last
 *                      token step; rank-1 magnitudes converge in one iteration.
 *   quantizers       - round-trip error <= d/2, brute-force nearest-code check, zero
 *                      block -> zero codes, idempotence.
 *   packing          - independent bit-loop unpacker in the test, plus a hand-written
 *                      golden byte image (tests/golden/).
 *   stream state     - chunking invariance is a property of the definition; the tail
 *                      rule and group boundaries are checked against the definition.
 *   decode           - pure-BF16 case equals a numpy textbook softmax attention to 1e-12,
 *                      one-hot and constant-V special cases, GQA independence.
 *   calculator       - the pages' worked arithmetic (tests/golden/calculator_pins.txt).
 */
#include "kvq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define D 128
#define GROUP 256

/* ------------------------------------------------------------------------------------ */
/* types                                                                                */
/* ------------------------------------------------------------------------------------ */

/* [p2] "Extended palette": q2_0..q6_1 next to upstream q4_0/q4_1/q5_0/q5_1/q8_0;
 * [p5] KLD table: kvarn2, kvarn3, kvarn4, kvarn5, kvarn6, kvarn8. */
static const int FAMILY[KVQO_NTYPES] = {0, 1, 1, 1, 1, 1, 1, 2, 3, 3, 3, 3, 3, 3, 2, 2, 2, 2};
static const int BITS[KVQO_NTYPES] = {16, 2, 3, 4, 5, 6, 8, 4, 2, 3, 4, 5, 6, 8, 2, 3, 5, 6};

int kvqo_type_family(int type) { return (type >= 0 && type < KVQO_NTYPES) ? FAMILY[type] : -1; }
int kvqo_type_bits(int type) { return (type >= 0 && type < KVQO_NTYPES) ? BITS[type] : -1; }

int kvqo_token_bytes(int type) {
  int f = kvqo_type_family(type);
  if (f < 0) return -1;
  if (f == 0) return 2 * D;
  int b = BITS[type];
  int bytes = 16 * b + 8;          /* 128 b-bit codes + four fp16 block scales d */
  if (f == 2) bytes += 8;          /* four fp16 block minimums m */
  if (f == 3) bytes += 2;          /* one fp16 token scale t */
  return bytes;
}

int kvqo_subpage_bytes(int type) {
  int f = kvqo_type_family(type);
  if (f <= 0) return -1;
  int bytes = GROUP * kvqo_token_bytes(type);
  if (f == 3) bytes += 2 * D;      /* fp16 channel scales c of the group */
  return bytes;
}

/* ------------------------------------------------------------------------------------ */
/* number formats                                                                       */
/* ------------------------------------------------------------------------------------ */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

uint16_t kvqo_f32_to_bf16(float f) {
  uint32_t u = f2u(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

float kvqo_bf16_to_f32(uint16_t h) { return u2f((uint32_t)h << 16); }

uint16_t kvqo_f32_to_f16(float f) {
  uint32_t u = f2u(f);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  uint32_t a = u & 0x7fffffffu;
  if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);     /* NaN */
  if (a == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);    /* inf */
  int e = (int)(a >> 23) - 127;                                /* unbiased exponent */
  if (e >= 16) return (uint16_t)(sign | 0x7c00u);              /* >= 65536 */
  if (e >= -14) {                                              /* normal half range */
    uint32_t m = a & 0x7fffffu;
    uint32_t h = ((uint32_t)(e + 15) << 10) | (m >> 13);
    uint32_t rem = m & 0x1fffu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;  /* may carry to inf */
    return (uint16_t)(sign | h);
  }
  if (a < 0x00800000u) return sign;                            /* fp32 subnormal -> 0 */
  /* half subnormal: value = M * 2^(e-23), result k = RNE(value / 2^-24) = RNE(M >> sh) */
  uint32_t M = (a & 0x7fffffu) | 0x800000u;
  int sh = -e - 1;                                             /* = 23 - (e + 24) */
  if (sh >= 32) return sign;
  uint32_t k = M >> sh;
  uint32_t rem = M & ((1u << sh) - 1u);
  uint32_t half = 1u << (sh - 1);
  if (rem > half || (rem == half && (k & 1u))) k += 1u;
  return (uint16_t)(sign | k);
}

float kvqo_f16_to_f32(uint16_t h) {
  uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
  uint32_t e = ((uint32_t)h >> 10) & 0x1fu;
  uint32_t m = (uint32_t)h & 0x3ffu;
  if (e == 0x1fu) return u2f(sign | 0x7f800000u | (m << 13));
  if (e == 0) {
    float v = (float)m * u2f(0x33800000u);                     /* m * 2^-24, exact */
    return sign ? -v : v;
  }
  return u2f(sign | ((e + 112u) << 23) | (m << 13));
}

/* fp16 with saturation to the largest finite half (block scales, block minimums) */
static uint16_t f16_sat(float f) {
  uint16_t h = kvqo_f32_to_f16(f);
  if ((h & 0x7fffu) == 0x7c00u) return (uint16_t)((h & 0x8000u) | 0x7bffu);
  return h;
}

/* fp16 of a positive scale, clamped to [2^-14, 65504] */
static uint16_t f16_scale(float f) {
  uint16_t h = kvqo_f32_to_f16(f);
  if (h < 0x0400u) h = 0x0400u;
  if (h > 0x7bffu) h = 0x7bffu;
  return h;
}

/* ------------------------------------------------------------------------------------ */
/* Walsh-Hadamard rotation   [p4] "How WHT and Sinkhorn save quality at 4-bit"         */
/* ------------------------------------------------------------------------------------ */

void kvqo_wht128(float *v) {
  for (int h = 1; h < D; h <<= 1) {
    for (int i = 0; i < D; ++i) {
      if (i & h) continue;
      float a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
  const float kappa = u2f(0x3DB504F3u);                        /* RN_fp32(2^-3.5) */
  for (int i = 0; i < D; ++i) v[i] = v[i] * kappa;
}

void kvqo_wht128_f64(double *v) {
  for (int h = 1; h < D; h <<= 1) {
    for (int i = 0; i < D; ++i) {
      if (i & h) continue;
      double a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
  const double s = 1.0 / sqrt(128.0);
  for (int i = 0; i < D; ++i) v[i] = v[i] * s;
}

/* ------------------------------------------------------------------------------------ */
/* Sinkhorn balancing   [p4] "after the WHT ... Sinkhorn picks a scale per dimension"   */
/* ------------------------------------------------------------------------------------ */

/* Canonical sum of the n products a[i]*u[i] over the group's tokens: 32 partial sums.
 * Partial l is the sum of two chains, each fmaf in ascending order from 0.0f: one over the
 * tokens l, l+64, l+128, l+192 and one over l+32, l+96, l+160, l+224 (absent tokens of a
 * partial group are skipped); the 32 partials are combined by an xor butterfly with
 * offsets 16, 8, 4, 2, 1. */
static float sum_over_tokens(const float *x2, int n, int j, const float *u) {
  float p[32], q[32];
  for (int l = 0; l < 32; ++l) {
    float acc[2] = {0.0f, 0.0f};
    for (int e = 0; e < 2; ++e)
      for (int i = l + 32 * e; i < n; i += 64) acc[e] = fmaf(x2[(size_t)i * D + j], u[i], acc[e]);
    p[l] = acc[0] + acc[1];
  }
  for (int off = 16; off >= 1; off >>= 1) {
    for (int l = 0; l < 32; ++l) q[l] = p[l] + p[l ^ off];
    memcpy(p, q, sizeof p);
  }
  return p[0];
}

/* Canonical sum of the 128 products row[j]*w[j] of one token: 16 partial sums, partial r
 * chains fmaf over channels 8r .. 8r+7 in ascending order from 0.0f; the 16 partials are
 * combined by an xor butterfly with offsets 8, 4, 2, 1. */
static float sum_over_channels(const float *row2, const float *w) {
  float p[16], q[16];
  for (int r = 0; r < 16; ++r) {
    float acc = 0.0f;
    for (int j = 8 * r; j < 8 * r + 8; ++j) acc = fmaf(row2[j], w[j], acc);
    p[r] = acc;
  }
  for (int off = 8; off >= 1; off >>= 1) {
    for (int r = 0; r < 16; ++r) q[r] = p[r] + p[r ^ off];
    memcpy(p, q, sizeof p);
  }
  return p[0];
}

/* Scale-only form.  With Y = X / (c_j t_i), the channel step sets
 * c_j = sqrt(mean_i X_ij^2 / t_i^2) and the token step t_i = sqrt(mean_j X_ij^2 / c_j^2);
 * one iteration is a channel step followed by a token step.  The iterations carry only the
 * squared reciprocals u_i = 1/t_i^2 = 128 / R_i and w_j = 1/c_j^2 = n / S_j (one division
 * each, from the sums S_j = sum_i X_ij^2 u_i and R_i = sum_j X_ij^2 w_j); the scales are
 * taken from the last sums, c_j = sqrt(S_j / n) and t_i = sqrt(R_i / 128).  A zero sum
 * gives 1 (for the scale and for its reciprocal). */
void kvqo_sinkhorn(const float *x, int n, int iters, float *c, float *t) {
  float *x2 = (float *)malloc(sizeof(float) * (size_t)n * D);
  float u[GROUP], w[D], S[D], R[GROUP];
  for (int i = 0; i < n * D; ++i) x2[i] = x[i] * x[i];
  for (int i = 0; i < n; ++i) u[i] = 1.0f;
  const float fn = (float)n;
  for (int j = 0; j < D; ++j) S[j] = 0.0f;
  for (int i = 0; i < n; ++i) R[i] = 0.0f;
  for (int it = 0; it < iters; ++it) {
    for (int j = 0; j < D; ++j) {
      S[j] = sum_over_tokens(x2, n, j, u);
      w[j] = S[j] > 0.0f ? fn / S[j] : 1.0f;
    }
    for (int i = 0; i < n; ++i) {
      R[i] = sum_over_channels(x2 + (size_t)i * D, w);
      u[i] = R[i] > 0.0f ? 128.0f / R[i] : 1.0f;
    }
  }
  for (int j = 0; j < D; ++j) c[j] = (iters > 0 && S[j] > 0.0f) ? sqrtf(S[j] / fn) : 1.0f;
  for (int i = 0; i < n; ++i) t[i] = (iters > 0 && R[i] > 0.0f) ? sqrtf(R[i] / 128.0f) : 1.0f;
  free(x2);
}

void kvqo_sinkhorn_literal(const double *x, int n, int iters, double *c, double *t) {
  double *y = (double *)malloc(sizeof(double) * (size_t)n * D);
  memcpy(y, x, sizeof(double) * (size_t)n * D);
  for (int j = 0; j < D; ++j) c[j] = 1.0;
  for (int i = 0; i < n; ++i) t[i] = 1.0;
  for (int it = 0; it < iters; ++it) {
    for (int j = 0; j < D; ++j) {                     /* divide each channel by its RMS */
      double s = 0.0;
      for (int i = 0; i < n; ++i) s += y[(size_t)i * D + j] * y[(size_t)i * D + j];
      double r = s > 0.0 ? sqrt(s / n) : 1.0;
      for (int i = 0; i < n; ++i) y[(size_t)i * D + j] /= r;
      c[j] *= r;
    }
    for (int i = 0; i < n; ++i) {                     /* divide each token by its RMS */
      double s = 0.0;
      for (int j = 0; j < D; ++j) s += y[(size_t)i * D + j] * y[(size_t)i * D + j];
      double r = s > 0.0 ? sqrt(s / D) : 1.0;
      for (int j = 0; j < D; ++j) y[(size_t)i * D + j] /= r;
      t[i] *= r;
    }
  }
  free(y);
}

/* ------------------------------------------------------------------------------------ */
/* block quantizers   [p2] "Extended palette"; block 32 with fp16 scale (and min)      */
/* ------------------------------------------------------------------------------------ */

void kvqo_quant_sym(const float *y, int bits, uint16_t *d16, int16_t *codes) {
  const int qmax = (1 << (bits - 1)) - 1, qmin = -(1 << (bits - 1));
  float amax = 0.0f;
  for (int j = 0; j < 32; ++j) {
    float a = fabsf(y[j]);
    if (a > amax) amax = a;
  }
  float d = amax / (float)qmax;
  uint16_t h = f16_sat(d);
  float df = kvqo_f16_to_f32(h);
  *d16 = h;
  for (int j = 0; j < 32; ++j) {
    int q = 0;
    if (df != 0.0f) {
      float r = rintf(y[j] / df);
      if (r > (float)qmax) r = (float)qmax;
      if (r < (float)qmin) r = (float)qmin;
      q = (int)r;
    }
    codes[j] = (int16_t)q;
  }
}

void kvqo_quant_asym(const float *x, int bits, uint16_t *d16, uint16_t *m16, int16_t *codes) {
  const int qmax = (1 << bits) - 1;
  float mn = x[0], mx = x[0];
  for (int j = 1; j < 32; ++j) {
    if (x[j] < mn) mn = x[j];
    if (x[j] > mx) mx = x[j];
  }
  float d = (mx - mn) / (float)qmax;
  uint16_t h = f16_sat(d);
  uint16_t hm = f16_sat(mn);
  float df = kvqo_f16_to_f32(h), mf = kvqo_f16_to_f32(hm);
  *d16 = h;
  *m16 = hm;
  for (int j = 0; j < 32; ++j) {
    int q = 0;
    if (df != 0.0f) {
      float r = rintf((x[j] - mf) / df);
      if (r > (float)qmax) r = (float)qmax;
      if (r < 0.0f) r = 0.0f;
      q = (int)r;
    }
    codes[j] = (int16_t)q;
  }
}

/* ------------------------------------------------------------------------------------ */
/* stream state   [p2] "KV Cache Precision Tail": the newest N tokens stay 16-bit, the */
/* rest is stored in the low-bit type; [p1] "How selective differs": when to quantize  */
/* ------------------------------------------------------------------------------------ */

int64_t kvqo_stream_state(int type, const uint16_t *xb, int64_t n, int64_t tail, int iters,
                          int16_t *codes, uint16_t *d16, uint16_t *m16, uint16_t *t16,
                          uint16_t *c16) {
  int fam = kvqo_type_family(type);
  if (fam < 0 || n < 0 || tail < 0 || iters < 0) return -1;
  int64_t keep = n < tail ? n : tail;
  int64_t Q = n - keep;
  if (fam == 0) return 0;
  int bits = BITS[type];
  float x[D];
  if (fam == 1 || fam == 2) {
    for (int64_t i = 0; i < Q; ++i) {
      for (int j = 0; j < D; ++j) x[j] = kvqo_bf16_to_f32(xb[i * D + j]);
      for (int b = 0; b < 4; ++b) {
        if (fam == 1)
          kvqo_quant_sym(x + 32 * b, bits, &d16[i * 4 + b], &codes[i * D + 32 * b]);
        else
          kvqo_quant_asym(x + 32 * b, bits, &d16[i * 4 + b], &m16[i * 4 + b], &codes[i * D + 32 * b]);
      }
    }
    return Q;
  }
  /* kvarn: tokens [256 g, min(256 g + 256, Q)) form group g; each group is rotated,
   * balanced and quantized as a unit (a partial last group included). */
  float *xr = (float *)malloc(sizeof(float) * GROUP * D);
  float c[D], t[GROUP], rc[D], y[32];
  for (int64_t g0 = 0; g0 < Q; g0 += GROUP) {
    int ng = (int)((Q - g0) < GROUP ? (Q - g0) : GROUP);
    for (int i = 0; i < ng; ++i) {
      for (int j = 0; j < D; ++j) xr[i * D + j] = kvqo_bf16_to_f32(xb[(g0 + i) * D + j]);
      kvqo_wht128(xr + i * D);
    }
    kvqo_sinkhorn(xr, ng, iters, c, t);
    int64_t g = g0 / GROUP;
    for (int j = 0; j < D; ++j) {
      uint16_t h = f16_scale(c[j]);
      if (c16) c16[g * D + j] = h;
      rc[j] = 1.0f / kvqo_f16_to_f32(h);
    }
    for (int i = 0; i < ng; ++i) {
      uint16_t ht = f16_scale(t[i]);
      t16[g0 + i] = ht;
      float rt = 1.0f / kvqo_f16_to_f32(ht);
      for (int b = 0; b < 4; ++b) {
        for (int e = 0; e < 32; ++e) {
          int j = 32 * b + e;
          y[e] = (xr[i * D + j] * rc[j]) * rt;
        }
        kvqo_quant_sym(y, bits, &d16[(g0 + i) * 4 + b], &codes[(g0 + i) * D + 32 * b]);
      }
    }
  }
  free(xr);
  return Q;
}

/* ------------------------------------------------------------------------------------ */
/* packing (the pages fix no bit layout; the layout below is the definition used)      */
/* ------------------------------------------------------------------------------------ */

/* b-bit codes are split into a low plane of width wlo and a high plane of width whi. */
static void planes(int bits, int *wlo, int *whi) {
  switch (bits) {
    case 2: *wlo = 2; *whi = 0; break;
    case 3: *wlo = 2; *whi = 1; break;
    case 4: *wlo = 4; *whi = 0; break;
    case 5: *wlo = 4; *whi = 1; break;
    case 6: *wlo = 4; *whi = 2; break;
    default: *wlo = 8; *whi = 0; break;
  }
}

/* K layout of one token (16*bits bytes).  In a plane of width w (F = 8/w fields per
 * byte), channel 32*blk + e with e = 4*jj + k is stored in byte k of the 32-bit word
 * (m = jj / F, blk) at byte offset 16*m + 4*blk of the plane, in bits [s*w, s*w+w) with
 * s = jj % F. */
static void put_k(uint8_t *tok, int bits, const uint32_t *field) {
  int wlo, whi;
  planes(bits, &wlo, &whi);
  int ws[2] = {wlo, whi};
  int off = 0;
  for (int p = 0; p < 2; ++p) {
    int w = ws[p];
    if (w == 0) continue;
    int F = 8 / w;
    int shift_in = p == 0 ? 0 : wlo;
    for (int blk = 0; blk < 4; ++blk)
      for (int e = 0; e < 32; ++e) {
        int jj = e / 4, k = e % 4, m = jj / F, s = jj % F;
        uint32_t v = (field[32 * blk + e] >> shift_in) & ((1u << w) - 1u);
        tok[off + 16 * m + 4 * blk + k] |= (uint8_t)(v << (s * w));
      }
    off += 16 * w;
  }
}

/* V layout of one 4-token quad (64*bits bytes).  In a plane of width w, channel
 * 32*blk + e of quad token k is stored in byte k of word m = e / F of block blk, at byte
 * offset 16*w*blk + 4*m of the plane, in bits [s*w, s*w+w) with s = e % F. */
static void put_v(uint8_t *quad, int k, int bits, const uint32_t *field) {
  int wlo, whi;
  planes(bits, &wlo, &whi);
  int ws[2] = {wlo, whi};
  int off = 0;
  for (int p = 0; p < 2; ++p) {
    int w = ws[p];
    if (w == 0) continue;
    int F = 8 / w;
    int shift_in = p == 0 ? 0 : wlo;
    for (int blk = 0; blk < 4; ++blk)
      for (int e = 0; e < 32; ++e) {
        int m = e / F, s = e % F;
        uint32_t v = (field[32 * blk + e] >> shift_in) & ((1u << w) - 1u);
        quad[off + 16 * w * blk + 4 * m + k] |= (uint8_t)(v << (s * w));
      }
    off += 64 * w;
  }
}

static void put_u16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)(v & 0xff); p[1] = (uint8_t)(v >> 8); }

/* Sub-page: [codes 256*16b B][d 256*8 B][m 256*8 B (asym)][t 256*2 B (kvarn)][c 128*2 B (kvarn)]
 * token i's d (m) at 8*i + 2*blk of its area, t at 2*i, channel scale j at 2*j. */
int kvqo_pack_subpage(int type, int which, int n_valid, const int16_t *codes, const uint16_t *d16,
                      const uint16_t *m16, const uint16_t *t16, const uint16_t *c16,
                      uint8_t *img, uint8_t *mask) {
  int fam = kvqo_type_family(type);
  if (fam <= 0 || n_valid < 0 || n_valid > GROUP) return -1;
  int bits = BITS[type];
  int bytes = kvqo_subpage_bytes(type);
  memset(img, 0, (size_t)bytes);
  memset(mask, 0, (size_t)bytes);
  const uint32_t fmask = (1u << bits) - 1u;
  uint32_t field[D];
  const int cbytes = 16 * bits;
  for (int i = 0; i < n_valid; ++i) {
    for (int j = 0; j < D; ++j) field[j] = ((uint32_t)(int32_t)codes[i * D + j]) & fmask;
    if (which == 0) {
      put_k(img + (size_t)i * cbytes, bits, field);
      memset(mask + (size_t)i * cbytes, 1, (size_t)cbytes);
    } else {
      int q = i / 4, k = i % 4;
      put_v(img + (size_t)q * 4 * cbytes, k, bits, field);
      /* the bytes of token k are byte k of every 32-bit word of the quad */
      for (int o = k; o < 4 * cbytes; o += 4) mask[(size_t)q * 4 * cbytes + o] = 1;
    }
  }
  int off_d = GROUP * cbytes;
  int off_m = off_d + GROUP * 8;
  int off_t = off_d + GROUP * 8 + (fam == 2 ? GROUP * 8 : 0);
  int off_c = off_t + GROUP * 2;
  for (int i = 0; i < n_valid; ++i) {
    for (int b = 0; b < 4; ++b) {
      put_u16(img + off_d + 8 * i + 2 * b, d16[i * 4 + b]);
      mask[off_d + 8 * i + 2 * b] = mask[off_d + 8 * i + 2 * b + 1] = 1;
      if (fam == 2) {
        put_u16(img + off_m + 8 * i + 2 * b, m16[i * 4 + b]);
        mask[off_m + 8 * i + 2 * b] = mask[off_m + 8 * i + 2 * b + 1] = 1;
      }
    }
    if (fam == 3) {
      put_u16(img + off_t + 2 * i, t16[i]);
      mask[off_t + 2 * i] = mask[off_t + 2 * i + 1] = 1;
    }
  }
  if (fam == 3 && n_valid > 0) {
    for (int j = 0; j < D; ++j) {
      put_u16(img + off_c + 2 * j, c16[j]);
      mask[off_c + 2 * j] = mask[off_c + 2 * j + 1] = 1;
    }
  }
  return bytes;
}

/* ------------------------------------------------------------------------------------ */
/* dequantization and attention (fp64)                                                   */
/* ------------------------------------------------------------------------------------ */

int kvqo_dequant(int type, int64_t Q, const int16_t *codes, const uint16_t *d16, const uint16_t *m16,
                 const uint16_t *t16, const uint16_t *c16, int basis, double *out) {
  int fam = kvqo_type_family(type);
  if (fam <= 0 || Q < 0) return -1;
  for (int64_t i = 0; i < Q; ++i) {
    double *o = out + i * D;
    for (int j = 0; j < D; ++j) {
      int b = j / 32;
      double v = (double)codes[i * D + j] * (double)kvqo_f16_to_f32(d16[i * 4 + b]);
      if (fam == 2) v += (double)kvqo_f16_to_f32(m16[i * 4 + b]);
      if (fam == 3)
        v *= (double)kvqo_f16_to_f32(t16[i]) * (double)kvqo_f16_to_f32(c16[(i / GROUP) * D + j]);
      o[j] = v;
    }
    if (fam == 3 && basis == 0) kvqo_wht128_f64(o);
  }
  return 0;
}

void kvqo_attend(const double *q, int G, const double *k, const double *v, int64_t n,
                 double scale, double *out) {
  double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int h = 0; h < G; ++h) {
    const double *qh = q + (size_t)h * D;
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
      double acc = 0.0;
      for (int j = 0; j < D; ++j) acc += qh[j] * k[i * D + j];
      s[i] = acc * scale;
      if (s[i] > mx) mx = s[i];
    }
    double l = 0.0;
    double *o = out + (size_t)h * D;
    for (int j = 0; j < D; ++j) o[j] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
      double p = exp(s[i] - mx);
      l += p;
      for (int j = 0; j < D; ++j) o[j] += p * v[i * D + j];
    }
    for (int j = 0; j < D; ++j) o[j] = n > 0 ? o[j] / l : 0.0;
  }
  free(s);
}

static int stream_rows(int type, const uint16_t *xb, int64_t n, int64_t tail, int iters, double *rows) {
  int fam = kvqo_type_family(type);
  if (fam < 0) return -1;
  int64_t keep = n < tail ? n : tail;
  int64_t Q = fam == 0 ? 0 : n - keep;
  if (fam == 0) keep = n;
  if (Q > 0) {
    int64_t ng = (Q + GROUP - 1) / GROUP;
    int16_t *codes = (int16_t *)malloc(sizeof(int16_t) * (size_t)Q * D);
    uint16_t *d16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)Q * 4);
    uint16_t *m16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)Q * 4);
    uint16_t *t16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)Q);
    uint16_t *c16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)ng * D);
    kvqo_stream_state(type, xb, n, tail, iters, codes, d16, m16, t16, c16);
    kvqo_dequant(type, Q, codes, d16, m16, t16, c16, 0, rows);
    free(codes); free(d16); free(m16); free(t16); free(c16);
  }
  for (int64_t i = Q; i < n; ++i)
    for (int j = 0; j < D; ++j) rows[i * D + j] = (double)kvqo_bf16_to_f32(xb[i * D + j]);
  return 0;
}

int kvqo_decode_head(int type_k, int type_v, const uint16_t *xk, const uint16_t *xv,
                     int64_t n, int64_t tail, int iters, const float *q, int G, double scale,
                     double *out) {
  if (n < 0 || G <= 0) return -1;
  double *k = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
  double *v = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
  double *qd = (double *)malloc(sizeof(double) * (size_t)G * D);
  int rc = stream_rows(type_k, xk, n, tail, iters, k);
  if (rc == 0) rc = stream_rows(type_v, xv, n, tail, iters, v);
  if (rc == 0) {
    for (int i = 0; i < G * D; ++i) qd[i] = (double)q[i];
    kvqo_attend(qd, G, k, v, n, scale, out);
  }
  free(k); free(v); free(qd);
  return rc;
}

/* Chunk (prefill) reference for one KV head: the stream state of the full n-row history,
 * then query token i of the chunk (its n_q newest tokens) attends with its G heads to rows
 * [0, n - n_q + 1 + i) of that state (causal within the chunk). */
int kvqo_prefill_head(int type_k, int type_v, const uint16_t *xk, const uint16_t *xv, int64_t n, int64_t tail,
                      int iters, const float *q, int n_q, int G, double scale, double *out) {
  if (n < 0 || G <= 0 || n_q < 0 || n_q > n) return -1;
  double *k = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
  double *v = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
  double *qd = (double *)malloc(sizeof(double) * (size_t)G * D);
  int rc = stream_rows(type_k, xk, n, tail, iters, k);
  if (rc == 0) rc = stream_rows(type_v, xv, n, tail, iters, v);
  for (int i = 0; rc == 0 && i < n_q; ++i) {
    for (int j = 0; j < G * D; ++j) qd[j] = (double)q[(size_t)i * G * D + j];
    kvqo_attend(qd, G, k, v, n - n_q + 1 + i, scale, out + (size_t)i * G * D);
  }
  free(k); free(v); free(qd);
  return rc;
}

/* ------------------------------------------------------------------------------------ */
/* size calculator   [p1] "Why the KV cache becomes the bottleneck", "What if the tail  */
/* grows to 20k"; [p2] "How it works: hybrid storage", "Extended palette"               */
/* ------------------------------------------------------------------------------------ */

double kvqo_payload_bytes(int type, int raw_bits, int64_t n_layers, int64_t n_kv_heads,
                          int64_t head_dim, int64_t n, int64_t tail) {
  int fam = kvqo_type_family(type);
  if (fam < 0) return -1.0;
  int64_t keep = n < tail ? n : tail;
  if (fam == 0) keep = n;
  int64_t Q = n - keep;
  double per_stream = (double)keep * (double)head_dim * 2.0;
  if (raw_bits > 0) {
    per_stream += (double)Q * (double)head_dim * raw_bits / 8.0;
  } else if (Q > 0) {
    per_stream += (double)Q * (double)kvqo_token_bytes(type) * ((double)head_dim / D);
    if (fam == 3) per_stream += (double)((Q + GROUP - 1) / GROUP) * 2.0 * (double)head_dim;
  }
  return per_stream * 2.0 * (double)n_layers * (double)n_kv_heads;
}

/* ------------------------------------------------------------------------------------ */
/* array forms of the number formats (for the Python wrapper)                           */
/* ------------------------------------------------------------------------------------ */

void kvqo_f32_to_bf16_n(const float *x, uint16_t *y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = kvqo_f32_to_bf16(x[i]);
}
void kvqo_f32_to_f16_n(const float *x, uint16_t *y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = kvqo_f32_to_f16(x[i]);
}
void kvqo_f16_to_f32_n(const uint16_t *x, float *y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = kvqo_f16_to_f32(x[i]);
}
