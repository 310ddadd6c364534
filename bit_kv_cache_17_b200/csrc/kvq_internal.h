// kvq_internal.h - host-side cache handle and the launchers behind the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/kvq.h"
#include "kvq_common.cuh"

struct kvq_cache {
  kvq_params p;
  uint8_t *base = nullptr;
  size_t bytes = 0;
  int fam_k = 0, bits_k = 0, fam_v = 0, bits_v = 0;
  kvq::SubLayout lk{}, lv{};
  int64_t max_pages = 0;     // pages per sequence
  int64_t page_bytes = 0;    // bytes of one page (all heads, K and V)
  int64_t ring_cap = 0;      // BF16 ring rows per (seq, head, K/V)
  size_t layer_pages_bytes = 0, layer_ring_bytes = 0;
  size_t off_pages = 0, off_ring = 0, off_ptab = 0, off_tickets = 0, off_status = 0;
  size_t total = 0;
  std::vector<int64_t> len;  // [n_layers * n_seqs] host-side sequence lengths
  int num_sms = 148;
  int device = 0;
  std::string desc;
};

namespace kvq {

// Decode entries (query rows, each with its own context length) per decode launch; the merge
// tickets are indexed by (entry within its launch, KV head), so a cache holds this many
// tickets per head (or n_seqs, if more).
constexpr int kDecodeEntriesPerLaunch = 64;

// Counts kernel launches (kvq_launch_count).
void note_launches(int n);

// KVQ_OK when the calling thread's current device is the one the cache was created on,
// KVQ_E_INVAL when it is another, KVQ_E_CUDA when the runtime cannot tell.
int check_device(const kvq_cache *c);

// Tokens of a stream kept in the BF16 ring after it holds n tokens: [keep_start, n).
// qb types keep the tail; kvarn also keeps the rows of its open (partial) group.
inline int64_t quantized_len(const kvq_cache *c, int64_t n) {
  if (c->fam_k == FAM_BF16) return 0;
  int64_t keep = n < c->p.tail ? n : c->p.tail;
  return n - keep;
}
inline int64_t keep_start(const kvq_cache *c, int fam, int64_t n) {
  if (fam == FAM_BF16) return 0;
  int64_t Q = quantized_len(c, n);
  return fam == FAM_KVARN ? (Q / GROUP) * GROUP : Q;
}

LayerView layer_view(const kvq_cache *c, int layer);

struct AppendSeq {
  int32_t seq;
  int32_t n_new;
  int64_t n0;      // length before the append
  int64_t in_off;  // first input row of this sequence
};

// What an append left in flight, for a decode launched right behind it.
struct AppendInfo {
  int launches = 0;  // kernels launched by the append
};

// Launchers; return KVQ_OK or a KVQ_E_* code.  Every append kernel signals its dependents
// (griddepcontrol.launch_dependents) as it starts, so that a decode launched with
// programmatic stream serialization behind it may begin early.
int launch_append(const kvq_cache *c, int layer, const std::vector<AppendSeq> &seqs,
                  const void *k, const void *v, cudaStream_t st, AppendInfo *info = nullptr);

constexpr int64_t kNeverDirty = INT64_MAX;
struct DecodeSeq {
  int32_t seq;      // sequence slot in the cache
  int32_t row;      // row of q/out for this sequence
  int64_t n;        // tokens
  int64_t Q;        // quantized tokens
  // Tokens written by the kernel(s) right before this decode in the stream (an overlapped
  // append): quantized tokens >= dq and BF16 ring rows of tokens >= dt.  A warp waits for
  // those kernels (griddepcontrol.wait) before it reads such a token.
  int64_t dq = kNeverDirty, dt = kNeverDirty;
};
// budget_sms: SMs the split plan may fill (0 = all; every caller passes 0); pdl: launch with
// programmatic stream serialization (the previous kernel in the stream must be an append
// kernel of this library and every token it wrote must be covered by the sequences' dq / dt).
int launch_decode(const kvq_cache *c, int layer, const std::vector<DecodeSeq> &seqs, int n_q_heads,
                  const float *q, float scale, float *out, void *ws, size_t ws_bytes, cudaStream_t st,
                  int budget_sms = 0, bool pdl = false);
size_t decode_workspace_bytes(const kvq_cache *c, int n_seqs, int n_q_heads);

// Chunk attention (kvq_prefill_attn): n_q query tokens of one sequence, causal within the
// chunk, up to 16 query tokens (80 query rows) per launch; the workspace holds
// chunk_workspace_bytes.
int launch_chunk(const kvq_cache *c, int layer, int seq, int n_q, int n_q_heads, const float *q, float scale,
                 float *out, void *ws, cudaStream_t st);
size_t chunk_workspace_bytes(const kvq_cache *c, int n_q_tokens, int n_q_heads);

int launch_dequant(const kvq_cache *c, int layer, int seq, int which, int64_t t0, int64_t t1,
                   int basis, float *out, cudaStream_t st);

}  // namespace kvq
