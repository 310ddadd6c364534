/*
 * kvq.h - C ABI of libkvq.so: a mixed-precision KV cache with a BF16 precision tail
 * and decode attention over it, for NVIDIA B200 (sm_100a).
 *
 * What the library computes, by page and section:
 *  - "Experimental KV-cache quantization methods in BeeLLama.cpp v0.4.0: KVarN and
 *    precision tail" (ai-manual.ru), section "KV Cache Precision Tail" / "How it works":
 *    the newest N tokens of every K/V stream stay 16-bit (BF16 here), older ones are
 *    stored in a low-bit cache type; section "Extended palette": the q2_0..q6_1 block
 *    types; section "KVarN": variance normalization applied once, at cache write.
 *  - "Bonsai-Ternary-27B on 120k tokens" (ai-manual.ru), section "How the Walsh-Hadamard
 *    transform and Sinkhorn save quality at 4-bit": KVarN = Walsh-Hadamard rotation of
 *    each head vector, then Sinkhorn per-dimension variance balancing, then quantization.
 *  - "BeeLLama.cpp v0.4.0 ..." (molayo1419.me), KLD table: the kvarn2..kvarn8 types.
 *  - "Fork of beellama and kvarn KV quants at long context" (ai-manual.ru), section on
 *    decode: at long context decode attention is memory bound; the dequantization
 *    inside the attention kernel decides whether the smaller cache pays off.
 * The steps the pages leave open are fixed as follows (one reading each):
 *  - head_dim is 128; blocks of 32 channels; fp16 block scale d = absmax/(2^(b-1)-1)
 *    (symmetric types) or d = (max-min)/(2^b-1) with fp16 min m (asymmetric types);
 *  - kvarn: each 256-token group of a stream is rotated x -> H.x.RN(2^-3.5) (Sylvester
 *    H, butterfly stages h = 1..64 ascending, fp32), balanced by 8 Sinkhorn iterations
 *    (channel step then token step) into fp16 per-channel scales c (per group) and fp16
 *    per-token scales t, then y = (x/c)/t is quantized in symmetric b-bit blocks;
 *  - a stream of n tokens keeps its newest min(n, tail) tokens in BF16; the older ones
 *    are quantized as they leave the tail; a kvarn group that is still filling is
 *    re-quantized from its BF16 rows each time it grows, so the cache state depends
 *    only on the tokens appended, not on how the appends were chunked.
 *
 * Conventions (all entry points):
 *  - Return value: KVQ_OK (0) or a negative KVQ_E_* code; kvq_strerror() names it.
 *    Arguments are validated on the host before anything is launched; a failed call
 *    changes no state.
 *  - Device work runs on the caller's stream, in stream order; nothing synchronizes
 *    except kvq_get_status().  Host metadata (sequence lengths) is updated when the call
 *    returns, so calls on one cache must be issued from one host thread in order.
 *  - Ownership: the caller allocates every device buffer (cache storage, workspace,
 *    inputs, outputs).  The library never allocates device memory.  kvq_cache_destroy
 *    frees only host metadata.
 *  - Pointers marked "device" must be device memory of the current device, 16-byte
 *    aligned (KVQ_E_ALIGN otherwise).  Every entry point that touches the device checks,
 *    before it launches anything, that the calling thread's current device is the one the
 *    cache was created on: another one gives KVQ_E_INVAL.
 *  - head_dim must be 128; page_tokens and group must be 256 (KVQ_E_UNSUPPORTED).
 *  - GQA: query head h reads KV head h / (n_q_heads / n_kv_heads).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvq_stream_t; /* a cudaStream_t; NULL = legacy default stream */

/* Cache types.  BF16 keeps every token 16-bit (the tail covers the whole context). */
typedef enum kvq_type {
  KVQ_BF16 = 0,
  KVQ_Q2_0 = 1, KVQ_Q3_0 = 2, KVQ_Q4_0 = 3, KVQ_Q5_0 = 4, KVQ_Q6_0 = 5, KVQ_Q8_0 = 6,
  KVQ_Q4_1 = 7,
  KVQ_KVARN2 = 8, KVQ_KVARN3 = 9, KVQ_KVARN4 = 10, KVQ_KVARN5 = 11, KVQ_KVARN6 = 12,
  KVQ_KVARN8 = 13,
  KVQ_Q2_1 = 14, KVQ_Q3_1 = 15, KVQ_Q5_1 = 16, KVQ_Q6_1 = 17,
  KVQ_TYPE_COUNT = 18
} kvq_type;

enum {
  KVQ_OK = 0,
  KVQ_E_INVAL = -1,       /* bad argument (NULL, out of range, duplicate sequence id) */
  KVQ_E_UNSUPPORTED = -2, /* head_dim != 128, group/page != 256, unknown type, G > 8 */
  KVQ_E_CAPACITY = -3,    /* append would exceed max_ctx */
  KVQ_E_ALIGN = -4,       /* a device pointer is not 16-byte aligned */
  KVQ_E_CUDA = -5,        /* a CUDA launch or runtime call failed */
  KVQ_E_DEVICE = -6,      /* the device-side status word reports an error */
  KVQ_E_SIZE = -7         /* a caller buffer (cache storage or workspace) is too small */
};

/* Cache geometry.  Mirrors the pages' CLI: --cache-type-k / --cache-type-v (separate K
 * and V types), --cache-precision-tail N ("Configuring the KV cache" section). */
typedef struct kvq_params {
  int32_t n_layers;       /* >= 1 */
  int32_t n_seqs;         /* sequence slots, >= 1 */
  int32_t n_kv_heads;     /* >= 1 */
  int32_t head_dim;       /* must be 128 */
  int64_t max_ctx;        /* tokens per sequence, >= 1 */
  int32_t type_k, type_v; /* kvq_type, chosen independently; BF16 must be used for both
                           * or neither (KVQ_E_UNSUPPORTED) */
  int32_t tail;           /* newest tokens kept in BF16, >= 0 */
  int32_t group;          /* kvarn group length, must be 256 */
  int32_t sinkhorn_iters; /* Sinkhorn iterations, 1..64 (8 by default) */
  int32_t page_tokens;    /* tokens per page, must be 256 */
  int32_t var_norm;       /* 0 or 1: KVarN variance normalization on the qN_0 types, the
                           * pages' --cache-var-norm switch ("KVarN" section of the BeeLLama.cpp
                           * v0.4.0 page): qN_0 with it is stored as kvarnN (rotation, Sinkhorn,
                           * then the same symmetric quantizer); kvarn types are unchanged; BF16
                           * and the qN_1 types with it are KVQ_E_UNSUPPORTED */
  int32_t tail_f16;       /* 0: the 16-bit tail (and a BF16 cache) holds BF16 rows; 1: F16
                           * rows (the pages' "last N tokens in BF16/F16", "KV Cache
                           * Precision Tail").  An F16 tail stores fp16(x) of each BF16
                           * input x (round to nearest even; beyond +-65504 it overflows to
                           * inf, as any F16 cache), and tokens are quantized from that same
                           * value.  Other values: KVQ_E_INVAL */
} kvq_params;

typedef struct kvq_cache kvq_cache;

/* Default parameters (head_dim 128, group 256, page 256, 8 iterations, tail 1024, no var_norm,
 * BF16 tail). */
void kvq_default_params(kvq_params *p);

/* Bytes of device memory a cache with these parameters needs (host-only arithmetic).
 * Also the size calculator: the quantized payload per token-head is 16*b + 8 bytes for
 * qb_0 types, 16*b + 16 for qb_1, 16*b + 10 (+256 per group) for kvarn, 256 for BF16. */
int kvq_cache_bytes(const kvq_params *p, size_t *bytes);

/* Pure payload arithmetic (no layout padding): bytes of n_layers x n_kv_heads x (K+V)
 * streams of n tokens of head_dim 128 keeping min(n, tail) tokens 16-bit.  raw_bits > 0
 * counts quantized values at raw_bits each with no scale overhead (the pages' form:
 * "Why the KV cache becomes the bottleneck" and "What if the tail grows to 20k" sections
 * of the Beellama selective-quantization page). */
int kvq_payload_bytes(int32_t type, int32_t raw_bits, int64_t n_layers, int64_t n_kv_heads,
                      int64_t n, int64_t tail, double *bytes);

/* Creates a cache inside the caller's device buffer dev_buf (bytes >= kvq_cache_bytes).
 * The metadata part of dev_buf (page table, merge tickets, status word) is initialized by
 * one kernel enqueued on the current device's legacy default stream (no host copy, no wait):
 * work on streams that do not synchronize with it (cudaStreamNonBlocking) must be ordered
 * after it by the caller.  All sequences start empty.  *out receives a host handle. */
int kvq_cache_create(const kvq_params *p, void *dev_buf, size_t bytes, kvq_cache **out);

/* Frees the host handle only; dev_buf stays owned by the caller. */
void kvq_cache_destroy(kvq_cache *c);

/* Appends n_new[i] tokens to sequence seq_ids[i] (i < n_seqs, ids distinct) of one layer.
 * k_bf16, v_bf16: device, [sum(n_new), n_kv_heads, 128] BF16, the rows of seq_ids[0]
 * first.  Tokens that leave the tail are quantized (kvarn groups re-balanced), and the
 * new tokens that stay in the tail are copied to the BF16 ring.  KVQ_E_CAPACITY if a
 * sequence would exceed max_ctx.  The input buffers may be reused once the stream has
 * passed the call. */
int kvq_append(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
               const int32_t *n_new, const void *k_bf16, const void *v_bf16, kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn needs for n_seqs sequences and n_q_heads heads: the
 * split-K partials, and, when type_k != type_v, also the Q.K scores of the quantized prefix
 * (4 bytes x min(n_seqs, 64) x n_q_heads x max_ctx rounded up to 32). */
int kvq_workspace_bytes(const kvq_cache *c, int32_t n_seqs, int32_t n_q_heads, size_t *bytes);

/* Decode attention of one query token per sequence over [quantized prefix | BF16 tail].
 * q: device fp32 [n_seqs, n_q_heads, 128]; out: device fp32 [n_seqs, n_q_heads, 128];
 * softmax_scale <= 0 selects 1/sqrt(128).  n_q_heads must be a multiple of n_kv_heads
 * with n_q_heads / n_kv_heads <= 8.  Split-K over the context; the last block of each
 * (sequence, KV head) merges the splits.  workspace: device, >= kvq_workspace_bytes.
 * K and V of one type run as one kernel; different types (the pages' separate
 * --cache-type-k / --cache-type-v) as two over the same split plan: Q.K of the K type
 * writes the scores of the quantized prefix to the workspace, then softmax and P.V of
 * the V type, the BF16 tail and the merge read them.
 * A sequence with no tokens gives zeros.  Decodes of one cache must not overlap on the
 * GPU (they share per-cache merge counters). */
int kvq_decode_attn(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
                    int32_t n_q_heads, const float *q, float softmax_scale, float *out,
                    void *workspace, size_t ws_bytes, kvq_stream_t stream);

/* Attention of a chunk of n_q_tokens queries over the cache of one sequence, causal
 * within the chunk: query row i attends to the first n - n_q_tokens + 1 + i tokens, n being
 * the sequence's current length (the chunk's own tokens already appended, as in a prefill
 * step that writes the chunk's K/V and then attends; the pages' prefill / decode split of
 * "Fork of beellama and kvarn KV quants at long context").  Every query sees the tokens of
 * the cache as they are stored now (quantized or BF16 by the current length).
 * q: device fp32 [n_q_tokens, n_q_heads, 128]; out: device fp32, same shape; softmax_scale
 * <= 0 selects 1/sqrt(128); workspace: device, >= kvq_workspace_bytes(c, n_q_tokens,
 * n_q_heads).  KVQ_E_INVAL if n_q_tokens exceeds the sequence length.  Each 64-token tile of
 * the cache is read and rebuilt once (into shared memory: the values with all their scales,
 * as f16 high part + f16 remainder) for all query rows of its KV head, up to 16 query tokens
 * (80 query rows) per launch, and Q.K and P.V run on the tcgen05 tensor cores (f16 operands,
 * fp32 accumulators in tensor memory); cached values, the rebuilt ones and, for kvarn, the
 * products d * t of block and token scales must lie within the f16 range (|x| < 65504).  A
 * wait between the kernel's roles that runs out sets the status word (kvq_get_status). */
int kvq_prefill_attn(kvq_cache *c, int32_t layer, int32_t seq, int32_t n_q_tokens, int32_t n_q_heads,
                     const float *q, float softmax_scale, float *out, void *workspace, size_t ws_bytes,
                     kvq_stream_t stream);

/* One decode step of a layer: kvq_append (n_new[i] tokens to seq_ids[i]) followed by
 * kvq_decode_attn of the same sequences (q / out row i belongs to seq_ids[i]), with the
 * same arguments, layouts and results as the two calls.  The pages ("KV Cache Precision
 * Tail": the newest tokens are written 16-bit, the oldest tail token spills into its
 * quantized group; the long-context decode discussion: decode attention reads the whole
 * cache) make these the two halves of every generated token.
 * The decode is launched with programmatic stream serialization behind the append's last
 * kernel: its warps start on pages the append does not touch while the append runs, and
 * wait for it (griddepcontrol.wait) only before the pages and ring rows it rewrites, which
 * form splits of their own.  The decode launches its light CTAs (those splits and the BF16
 * tail) last, so that the ones left waiting for SMs a one-token spill still holds are
 * these.  With type_k != type_v the decode follows the append in plain stream order
 * instead.  Requirements beyond the two calls': q must be complete before this call
 * is issued (it is read while the append runs), and nothing else may be enqueued on `stream`
 * in between (there is nothing in between: this is one call).  Errors: those of the two
 * calls, all checked before anything is launched. */
int kvq_append_decode(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
                      const int32_t *n_new, const void *k_bf16, const void *v_bf16, int32_t n_q_heads,
                      const float *q, float softmax_scale, float *out, void *workspace, size_t ws_bytes,
                      kvq_stream_t stream);

/* Dequantizes tokens [t0, t1) of K (which = 0) or V (which = 1) of one sequence into
 * out: device fp32 [t1 - t0, n_kv_heads, 128].  basis 0 = original basis (kvarn values
 * are rotated back with the same fp32 butterfly), basis 1 = the stored rotated basis.
 * Tail tokens are returned exactly (BF16 -> fp32). */
int kvq_dequant(kvq_cache *c, int32_t layer, int32_t seq, int32_t which, int64_t t0, int64_t t1,
                int32_t basis, float *out, kvq_stream_t stream);

/* Current length of a sequence in a layer (host metadata, no device access). */
int kvq_seq_len(const kvq_cache *c, int32_t layer, int32_t seq, int64_t *len);

/* Empties a sequence in every layer (host metadata; the old bytes are overwritten by
 * later appends). */
int kvq_seq_reset(kvq_cache *c, int32_t seq);

/* Byte offset inside dev_buf of the 256-token sub-page (layer, seq, page, head, which),
 * of the BF16 ring row holding token `token`, of the page-table entry of (seq, page), or
 * of a decode merge ticket, for tests and tools.  kind 0 = sub-page (token ignored),
 * kind 1 = ring row (page ignored), kind 2 = page-table entry, an int32 physical page
 * index shared by all layers, kind 3 = the uint32 merge ticket of KV head `head` of the
 * decode entry `seq` (the position of a sequence in a decode call's list).  Arguments a
 * kind does not use are only range-checked.  *bytes receives the region size. */
int kvq_locate(const kvq_cache *c, int32_t kind, int32_t layer, int32_t seq, int64_t page,
               int32_t head, int32_t which, int64_t token, size_t *offset, size_t *bytes);

/* Synchronizes `stream`, then reads and clears the device status word: KVQ_OK, or
 * KVQ_E_DEVICE if a kernel recorded an inconsistency in the cache buffer since the last
 * call.  Kernels record (and never trap on):
 *  - a page-table entry outside the layer's page pool: the access goes to physical page 0
 *    instead, so nothing outside dev_buf is read or written (the results of that call are
 *    wrong, the cache buffer having been corrupted);
 *  - a decode merge ticket that was not zero when the decode began (a corrupted ticket, or
 *    two decodes of one cache overlapping on the GPU): that decode's output may be stale;
 *  - a wait between the roles of the chunk-attention kernel that ran out (each is bounded):
 *    that call's output is wrong; the kernel still finishes and frees what it holds. */
int kvq_get_status(kvq_cache *c, kvq_stream_t stream);

/* Human-readable description of the cache (types, tail, bytes); valid until the next
 * call on this cache. */
const char *kvq_describe(kvq_cache *c);

const char *kvq_strerror(int code);

/* Decode attention that allocates nothing: the same computation and arguments as
 * kvq_decode_attn, without the workspace.  The pages have no counterpart of this entry
 * point; it exists for callers that cannot allocate device memory: a plugin running inside
 * a host runtime that owns all device memory and offers it no allocator, or a serving loop
 * that must not allocate (a possible stall or failure) once it runs.
 *  - The split-K partial results go to one library-owned static device array of
 *    KVQ_NOALLOC_SCRATCH_BYTES (4 MiB) per GPU, held by every GPU that loads the library
 *    until the process exits.  A call that needs more than the array (kvq_workspace_bytes
 *    for the same n_seqs / n_q_heads) returns KVQ_E_SIZE and launches nothing.  The need is
 *    33 792 x n_seqs x n_kv_heads x G bytes of partials (G = n_q_heads / n_kv_heads), plus,
 *    when type_k != type_v, 4 x n_seqs x n_kv_heads x G x max_ctx (rounded up to 32) bytes
 *    of scores.  With 8 KV heads and G = 5 that admits 3 sequences of one type, or one
 *    sequence of a mixed K/V cache with max_ctx <= 17 760.
 *  - Every call looks the array's device address up with the cache's device current (the
 *    call is rejected with KVQ_E_INVAL when another device is current); the first call on
 *    a device may load the library's device code, so make it before any stream capture.
 *  - Every call shares the array and it keeps the last call's contents; nothing in it needs
 *    to start at zero (every partial is written before it is read).  Calls that overlap on
 *    the GPU, on any stream or cache, race on the array: issue them in stream order.
 *  - Never calls cudaMalloc, cudaFree or any allocating routine. */
#define KVQ_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
int kvq_decode_attn_noalloc(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
                            int32_t n_q_heads, const float *q, float softmax_scale, float *out,
                            kvq_stream_t stream);

/* Diagnostic: number of kernels this library has launched (or recorded into a CUDA graph
 * under stream capture) in this process, across all caches. */
int kvq_launch_count(uint64_t *count);

#ifdef __cplusplus
}
#endif
#endif
