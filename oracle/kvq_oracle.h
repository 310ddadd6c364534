/*
 * kvq_oracle.h - plain, slow, scalar CPU oracle for the mixed-precision KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code, header,
 * table or constant with the CUDA library, and it never calls it.
 *
 * Sources (the method is described in prose on these pages):
 *   [p1] ai-manual.ru, "Beellama and Beellama-kvarn: selective KV-cache quantization"
 *        - section "Why the KV cache becomes the bottleneck" (per-token byte arithmetic),
 *        - section "What if the tail grows to 20k" (4-bit / tail arithmetic).
 *   [p2] ai-manual.ru, "Experimental KV-cache quantization methods in BeeLLama.cpp v0.4.0:
 *        KVarN and precision tail" - sections "KVarN", "KV Cache Precision Tail",
 *        "Extended palette from q2_0 to q6_1".
 *   [p4] ai-manual.ru, "Bonsai-Ternary-27B on 120k tokens" - section "How the
 *        Walsh-Hadamard transform and Sinkhorn save quality at 4-bit".
 *   [p5] molayo1419.me, "BeeLLama.cpp v0.4.0: KVarN, precision tail, q2_0-q3_1"
 *        - KLD table (cache types kvarn2..kvarn8).
 * The pages give KVarN only qualitatively.  Its steps are fixed here as: Sylvester
 * Hadamard rotation in a fixed fp32 butterfly order, 8 Sinkhorn iterations into fp16
 * per-channel and per-token scales, symmetric blocks of 32 with an fp16 scale d.  Where
 * the pages leave a step open, the comment at the step states the reading taken.
 *
 * Parity status per function (see the header of kvq_oracle.c for the pins):
 *   every exported function below is pinned by at least one test in
 *   tests/test_oracle_*.py; none is "parity unpinned".
 *
 * Precision: the quantizer runs in IEEE fp32 with no contraction (the codes are
 * integers decided by fp32 arithmetic, so the oracle takes those decisions in the
 * kernel's precision); dequantization and attention run in fp64.
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Cache types.  The numbering is the oracle's own; tests map names to numbers. */
enum {
  KVQO_BF16 = 0,
  KVQO_Q2_0, KVQO_Q3_0, KVQO_Q4_0, KVQO_Q5_0, KVQO_Q6_0, KVQO_Q8_0,
  KVQO_Q4_1,
  KVQO_KVARN2, KVQO_KVARN3, KVQO_KVARN4, KVQO_KVARN5, KVQO_KVARN6, KVQO_KVARN8,
  KVQO_Q2_1, KVQO_Q3_1, KVQO_Q5_1, KVQO_Q6_1,
  KVQO_NTYPES
};

/* family: 0 = bf16 (no quantization), 1 = symmetric qb_0, 2 = asymmetric qb_1, 3 = kvarn */
int kvqo_type_family(int type);
int kvqo_type_bits(int type);
/* bytes one token of one head of K (or V) occupies in the quantized region
 * (codes + fp16 block scales [+ fp16 mins] [+ fp16 token scale]); the kvarn per-group
 * channel scales (256 B per 256 tokens) are not included. */
int kvqo_token_bytes(int type);
/* bytes of one 256-token sub-page (one head, one of K/V) */
int kvqo_subpage_bytes(int type);

/* ---- number formats (round to nearest, ties to even) ---- */
uint16_t kvqo_f32_to_bf16(float f);
float    kvqo_bf16_to_f32(uint16_t h);
uint16_t kvqo_f32_to_f16(float f);
float    kvqo_f16_to_f32(uint16_t h);
void     kvqo_f32_to_bf16_n(const float *x, uint16_t *y, int64_t n);
void     kvqo_f32_to_f16_n(const float *x, uint16_t *y, int64_t n);
void     kvqo_f16_to_f32_n(const uint16_t *x, float *y, int64_t n);

/* ---- KVarN steps ---- */
/* In-place 128-point Walsh-Hadamard rotation, fp32: butterfly stages h = 1,2,...,64
 * (ascending), then every element times kappa = RN_fp32(2^-3.5). */
void kvqo_wht128(float *v);
/* Same butterfly in fp64 followed by a multiply by 1/sqrt(128) (the exact inverse
 * rotation used by the fp64 decode reference). */
void kvqo_wht128_f64(double *v);
/* Sinkhorn balancing, scale-only form, fp32, canonical summation order.
 * x: n x 128 rotated rows (n <= 256).  Outputs fp32 c[128], t[n]. */
void kvqo_sinkhorn(const float *x, int n, int iters, float *c, float *t);
/* Literal form: repeatedly divides a copy of the tile by channel RMS then token
 * RMS, in fp64, accumulating the scales.  Cross-check only. */
void kvqo_sinkhorn_literal(const double *x, int n, int iters, double *c, double *t);

/* ---- block quantizers (32 values) ---- */
/* symmetric b-bit: d = fp16(absmax / (2^(b-1)-1)), code = clamp(rint(y/d)) */
void kvqo_quant_sym(const float *y, int bits, uint16_t *d16, int16_t *codes);
/* asymmetric b-bit: d = fp16((max-min)/(2^b-1)), m = fp16(min), code = clamp(rint((x-m)/d)) */
void kvqo_quant_asym(const float *x, int bits, uint16_t *d16, uint16_t *m16, int16_t *codes);

/* ---- whole-stream state ----
 * One stream = one (layer, sequence, KV head, K-or-V).  Given the stream's n
 * appended BF16 head vectors (n x 128) and the tail length, computes the state of
 * its quantized region [0, Q) with Q = n - min(n, tail):
 *   codes[Q*128], d16[Q*4], m16[Q*4] (asym only), t16[Q] (kvarn only),
 *   c16[ceil(Q/256)*128] (kvarn only).  Unused outputs may be NULL.
 * Returns Q, or -1 on a bad argument. */
int64_t kvqo_stream_state(int type, const uint16_t *x_bf16, int64_t n, int64_t tail, int iters,
                          int16_t *codes, uint16_t *d16, uint16_t *m16, uint16_t *t16,
                          uint16_t *c16);

/* Packs the state of tokens [0, n_valid) of one 256-token page into the sub-page byte
 * image (kvqo_subpage_bytes(type) bytes).  which: 0 = K layout, 1 = V layout.
 * mask[i] = 1 for every byte that holds data of a valid token (0 elsewhere). */
int kvqo_pack_subpage(int type, int which, int n_valid, const int16_t *codes, const uint16_t *d16,
                      const uint16_t *m16, const uint16_t *t16, const uint16_t *c16,
                      uint8_t *img, uint8_t *mask);

/* fp64 dequantization of Q quantized tokens (original basis when basis == 0, rotated
 * basis when basis == 1; the rotated basis only differs for kvarn types). */
int kvqo_dequant(int type, int64_t Q, const int16_t *codes, const uint16_t *d16, const uint16_t *m16,
                 const uint16_t *t16, const uint16_t *c16, int basis, double *out);

/* fp64 softmax attention of G query rows over n keys/values (row-major, 128 wide). */
void kvqo_attend(const double *q, int G, const double *k, const double *v, int64_t n,
                 double scale, double *out);

/* Decode reference for one KV head: dequantizes the stream state, appends the BF16
 * tail rows, and attends with G query heads (fp64 throughout).  q: G x 128 fp32.
 * x_k_bf16 / x_v_bf16: the full n-row histories (the tail rows are read from them). */
int kvqo_decode_head(int type_k, int type_v, const uint16_t *x_k_bf16, const uint16_t *x_v_bf16,
                     int64_t n, int64_t tail, int iters, const float *q, int G, double scale,
                     double *out);

/* Chunk (prefill) reference for one KV head: the state of the full n-row history, then query
 * token i of the chunk (the n_q newest tokens) attends with its G heads to rows
 * [0, n - n_q + 1 + i) of that state.  q: n_q x G x 128 fp32; out: n_q x G x 128 fp64. */
int kvqo_prefill_head(int type_k, int type_v, const uint16_t *x_k_bf16, const uint16_t *x_v_bf16,
                      int64_t n, int64_t tail, int iters, const float *q, int n_q, int G, double scale,
                      double *out);

/* ---- size calculator ----
 * Payload bytes of a cache of n_layers x n_kv_heads x (K and V) streams of n tokens of
 * head_dim 128 with the newest min(n, tail) tokens kept as 16-bit values.
 * If raw_bits > 0 the quantized tokens are counted at raw_bits per value with no
 * block or scale overhead (the pages' back-of-envelope form); else at the type's
 * token size.  kvarn channel scales (256 B per full or partial 256-token group) are
 * counted when raw_bits == 0. */
double kvqo_payload_bytes(int type, int raw_bits, int64_t n_layers, int64_t n_kv_heads,
                          int64_t head_dim, int64_t n, int64_t tail);

#ifdef __cplusplus
}
#endif
#endif
