// kvq_abi.cu - the extern "C" entry points of libkvq.so (host code only).
//
// Validation happens here, before any launch; the launchers in kvq_append.cu,
// kvq_decode.cu and kvq_dequant.cu only see consistent arguments.
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <new>
#include <string>
#include <vector>

#include "kvq_internal.h"

using namespace kvq;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

const char *type_name(int t) {
  static const char *names[KVQ_TYPE_COUNT] = {
      "bf16", "q2_0", "q3_0", "q4_0", "q5_0", "q6_0", "q8_0", "q4_1", "kvarn2", "kvarn3",
      "kvarn4", "kvarn5", "kvarn6", "kvarn8", "q2_1", "q3_1", "q5_1", "q6_1"};
  return (t >= 0 && t < KVQ_TYPE_COUNT) ? names[t] : "?";
}

// var_norm: a qb_0 type with the KVarN variance normalization is the kvarn type of the same
// width (rotation, Sinkhorn, then the symmetric block quantizer); kvarn types already have it.
int resolve_type(int type, int var_norm, int *out) {
  const TypeInfo ti = type_info(type);
  if (ti.fam < 0) return KVQ_E_UNSUPPORTED;
  *out = type;
  if (!var_norm || ti.fam == FAM_KVARN) return KVQ_OK;
  if (ti.fam != FAM_SYM) return KVQ_E_UNSUPPORTED;  // BF16 and the qb_1 types have no such form
  static const int kvarn_of_bits[9] = {-1, -1, KVQ_KVARN2, KVQ_KVARN3, KVQ_KVARN4, KVQ_KVARN5, KVQ_KVARN6, -1,
                                       KVQ_KVARN8};
  *out = kvarn_of_bits[ti.bits];
  return KVQ_OK;
}

// Parameters with var_norm applied to the types (the form the cache is planned and built in).
int resolve_params(const kvq_params *p, kvq_params *r) {
  if (!p) return KVQ_E_INVAL;
  if (p->var_norm != 0 && p->var_norm != 1) return KVQ_E_INVAL;
  *r = *p;
  int rc = resolve_type(p->type_k, p->var_norm, &r->type_k);
  if (rc == KVQ_OK) rc = resolve_type(p->type_v, p->var_norm, &r->type_v);
  r->var_norm = 0;
  return rc;
}

int check_params(const kvq_params *p) {
  if (!p) return KVQ_E_INVAL;
  if (p->n_layers < 1 || p->n_seqs < 1 || p->n_kv_heads < 1 || p->max_ctx < 1 || p->tail < 0)
    return KVQ_E_INVAL;
  if (p->head_dim != D || p->group != GROUP || p->page_tokens != GROUP) return KVQ_E_UNSUPPORTED;
  if (p->sinkhorn_iters < 1 || p->sinkhorn_iters > 64) return KVQ_E_INVAL;
  if (p->tail_f16 != 0 && p->tail_f16 != 1) return KVQ_E_INVAL;
  TypeInfo tk = type_info(p->type_k), tv = type_info(p->type_v);
  if (tk.fam < 0 || tv.fam < 0) return KVQ_E_UNSUPPORTED;
  if ((tk.fam == FAM_BF16) != (tv.fam == FAM_BF16)) return KVQ_E_UNSUPPORTED;
  return KVQ_OK;
}

// Fills the derived geometry of a cache; returns the device bytes it needs.
size_t plan(kvq_cache *c) {
  const kvq_params &p = c->p;
  TypeInfo tk = type_info(p.type_k), tv = type_info(p.type_v);
  c->fam_k = tk.fam;
  c->bits_k = tk.bits;
  c->fam_v = tv.fam;
  c->bits_v = tv.bits;
  c->lk = sub_layout(tk.fam, tk.bits);
  c->lv = sub_layout(tv.fam, tv.bits);
  const bool bf16 = tk.fam == FAM_BF16;
  c->max_pages = bf16 ? 0 : (p.max_ctx + GROUP - 1) / GROUP;
  c->page_bytes = (int64_t)p.n_kv_heads * (c->lk.bytes + c->lv.bytes);
  const bool any_kvarn = tk.fam == FAM_KVARN || tv.fam == FAM_KVARN;
  c->ring_cap = bf16 ? p.max_ctx : (int64_t)p.tail + (any_kvarn ? GROUP : 0);
  c->layer_pages_bytes = align_up((size_t)p.n_seqs * c->max_pages * c->page_bytes);
  c->layer_ring_bytes = align_up((size_t)p.n_seqs * p.n_kv_heads * 2 * c->ring_cap * 2 * D);
  size_t off = 0;
  c->off_pages = off;
  off += c->layer_pages_bytes * p.n_layers;
  c->off_ring = off;
  off += c->layer_ring_bytes * p.n_layers;
  c->off_ptab = off;
  off += align_up(sizeof(int32_t) * std::max<int64_t>(1, (int64_t)p.n_seqs * c->max_pages));
  c->off_tickets = off;
  off += align_up(sizeof(uint32_t) * (size_t)std::max<int64_t>(p.n_seqs, kDecodeEntriesPerLaunch) * p.n_kv_heads);
  c->off_status = off;
  off += kAlign;
  c->total = off;
  return off;
}

// the cache's metadata at creation: the identity page table and zeroed tickets / status word
__global__ void k_init_meta(int32_t *ptab, int64_t n_ptab, uint8_t *meta, int64_t n_meta) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_ptab; i += stride) ptab[i] = (int32_t)i;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_meta; i += stride) meta[i] = 0;
}

}  // namespace

namespace kvq {
static std::atomic<uint64_t> g_launches{0};

int check_device(const kvq_cache *c) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_E_CUDA;
  return dev == c->device ? KVQ_OK : KVQ_E_INVAL;
}

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

LayerView layer_view(const kvq_cache *c, int layer) {
  LayerView L;
  L.pages = c->base + c->off_pages + c->layer_pages_bytes * layer;
  L.ring = c->base + c->off_ring + c->layer_ring_bytes * layer;
  L.ptab = reinterpret_cast<const int32_t *>(c->base + c->off_ptab);
  L.status = reinterpret_cast<int32_t *>(c->base + c->off_status);
  L.max_pages = c->max_pages;
  L.n_phys = (int64_t)c->p.n_seqs * c->max_pages;
  L.page_bytes = c->page_bytes;
  L.ring_cap = c->ring_cap;
  L.hkv = c->p.n_kv_heads;
  L.sub_k = c->lk.bytes;
  L.sub_v = c->lv.bytes;
  L.type_k = c->p.type_k;
  L.type_v = c->p.type_v;
  L.tail_f16 = c->p.tail_f16;
  return L;
}
}  // namespace kvq

extern "C" {

void kvq_default_params(kvq_params *p) {
  if (!p) return;
  memset(p, 0, sizeof *p);
  p->n_layers = 1;
  p->n_seqs = 1;
  p->n_kv_heads = 8;
  p->head_dim = D;
  p->max_ctx = 65536;
  p->type_k = KVQ_KVARN4;
  p->type_v = KVQ_KVARN4;
  p->tail = 1024;
  p->group = GROUP;
  p->sinkhorn_iters = 8;
  p->page_tokens = GROUP;
}

int kvq_cache_bytes(const kvq_params *pin, size_t *bytes) {
  kvq_params rp;
  int rc = resolve_params(pin, &rp);
  if (rc) return rc;
  const kvq_params *p = &rp;
  rc = check_params(p);
  if (rc) return rc;
  if (!bytes) return KVQ_E_INVAL;
  kvq_cache tmp;
  tmp.p = *p;
  *bytes = plan(&tmp);
  return KVQ_OK;
}

int kvq_payload_bytes(int32_t type, int32_t raw_bits, int64_t n_layers, int64_t n_kv_heads,
                      int64_t n, int64_t tail, double *bytes) {
  TypeInfo ti = type_info(type);
  if (ti.fam < 0 || !bytes || n < 0 || tail < 0 || n_layers < 0 || n_kv_heads < 0 || raw_bits < 0)
    return KVQ_E_INVAL;
  int64_t keep = ti.fam == FAM_BF16 ? n : std::min(n, tail);
  int64_t Q = n - keep;
  double per = (double)keep * D * 2.0;
  if (raw_bits > 0)
    per += (double)Q * D * raw_bits / 8.0;
  else if (Q > 0) {
    per += (double)Q * token_bytes(ti.fam, ti.bits);
    if (ti.fam == FAM_KVARN) per += (double)((Q + GROUP - 1) / GROUP) * 2.0 * D;
  }
  *bytes = per * 2.0 * (double)n_layers * (double)n_kv_heads;
  return KVQ_OK;
}

int kvq_cache_create(const kvq_params *pin, void *dev_buf, size_t bytes, kvq_cache **out) {
  kvq_params rp;
  int rc = resolve_params(pin, &rp);
  if (rc) return rc;
  const kvq_params *p = &rp;
  rc = check_params(p);
  if (rc) return rc;
  if (!dev_buf || !out) return KVQ_E_INVAL;
  if (!aligned16(dev_buf)) return KVQ_E_ALIGN;
  kvq_cache *c = new (std::nothrow) kvq_cache;
  if (!c) return KVQ_E_INVAL;
  c->p = *p;
  size_t need = plan(c);
  if (bytes < need) {
    delete c;
    return KVQ_E_SIZE;
  }
  c->base = static_cast<uint8_t *>(dev_buf);
  c->bytes = bytes;
  c->len.assign((size_t)p->n_layers * p->n_seqs, 0);
  if (cudaGetDevice(&c->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
    delete c;
    return KVQ_E_CUDA;
  }
  // the metadata, by one kernel on the legacy default stream (no host copy, no wait): the
  // static page table (sequence s, logical page j -> physical page s * max_pages + j), the
  // merge tickets and the status word at zero
  const int64_t n_ptab = (int64_t)p->n_seqs * c->max_pages;
  const int64_t n_meta = (int64_t)(c->total - c->off_tickets);
  k_init_meta<<<(unsigned)std::max<int64_t>(1, std::min<int64_t>(4 * c->num_sms, (std::max(n_ptab, n_meta) + 255) / 256)),
                256>>>(reinterpret_cast<int32_t *>(c->base + c->off_ptab), n_ptab, c->base + c->off_tickets, n_meta);
  if (cudaGetLastError() != cudaSuccess) {
    delete c;
    return KVQ_E_CUDA;
  }
  kvq::note_launches(1);
  *out = c;
  return KVQ_OK;
}

void kvq_cache_destroy(kvq_cache *c) { delete c; }

int kvq_append(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
               const int32_t *n_new, const void *k_bf16, const void *v_bf16, kvq_stream_t stream) {
  if (!c || layer < 0 || layer >= c->p.n_layers || n_seqs < 0) return KVQ_E_INVAL;
  if (n_seqs > 0 && (!seq_ids || !n_new)) return KVQ_E_INVAL;
  std::vector<char> seen(c->p.n_seqs, 0);
  std::vector<AppendSeq> seqs;
  int64_t rows = 0;
  for (int i = 0; i < n_seqs; ++i) {
    int s = seq_ids[i];
    if (s < 0 || s >= c->p.n_seqs || seen[s] || n_new[i] < 0) return KVQ_E_INVAL;
    seen[s] = 1;
    int64_t n0 = c->len[(size_t)layer * c->p.n_seqs + s];
    if (n0 + n_new[i] > c->p.max_ctx) return KVQ_E_CAPACITY;
    if (n_new[i] > 0) seqs.push_back({s, n_new[i], n0, rows});
    rows += n_new[i];
  }
  if (rows == 0) return KVQ_OK;
  if (!k_bf16 || !v_bf16) return KVQ_E_INVAL;
  if (!aligned16(k_bf16) || !aligned16(v_bf16)) return KVQ_E_ALIGN;
  int rc = check_device(c);
  if (rc) return rc;
  rc = launch_append(c, layer, seqs, k_bf16, v_bf16, reinterpret_cast<cudaStream_t>(stream));
  if (rc) return rc;
  for (const AppendSeq &a : seqs) c->len[(size_t)layer * c->p.n_seqs + a.seq] = a.n0 + a.n_new;
  return KVQ_OK;
}

int kvq_workspace_bytes(const kvq_cache *c, int32_t n_seqs, int32_t n_q_heads, size_t *bytes) {
  if (!c || !bytes || n_seqs < 0 || n_q_heads < 1) return KVQ_E_INVAL;
  if (n_q_heads % c->p.n_kv_heads) return KVQ_E_INVAL;
  if (n_q_heads / c->p.n_kv_heads > MAX_G) return KVQ_E_UNSUPPORTED;
  *bytes = decode_workspace_bytes(c, n_seqs, n_q_heads);
  return KVQ_OK;
}

int kvq_append_decode(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
                      const int32_t *n_new, const void *k_bf16, const void *v_bf16, int32_t n_q_heads,
                      const float *q, float softmax_scale, float *out, void *workspace, size_t ws_bytes,
                      kvq_stream_t stream) {
  // every argument is checked before anything is launched, so a failed call changes nothing
  if (!c || layer < 0 || layer >= c->p.n_layers || n_seqs < 0) return KVQ_E_INVAL;
  if (n_seqs == 0) return KVQ_OK;
  if (!seq_ids || !n_new || !q || !out || !workspace || n_q_heads < 1) return KVQ_E_INVAL;
  if (n_q_heads % c->p.n_kv_heads) return KVQ_E_INVAL;
  if (n_q_heads / c->p.n_kv_heads > MAX_G) return KVQ_E_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_E_ALIGN;
  if (ws_bytes < decode_workspace_bytes(c, n_seqs, n_q_heads)) return KVQ_E_SIZE;
  std::vector<char> seen(c->p.n_seqs, 0);
  std::vector<AppendSeq> app;
  std::vector<DecodeSeq> dec;
  int64_t rows = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    if (s < 0 || s >= c->p.n_seqs || seen[s] || n_new[i] < 0) return KVQ_E_INVAL;
    seen[s] = 1;
    const int64_t n0 = c->len[(size_t)layer * c->p.n_seqs + s];
    if (n0 + n_new[i] > c->p.max_ctx) return KVQ_E_CAPACITY;
    if (n_new[i] > 0) app.push_back({s, n_new[i], n0, rows});
    rows += n_new[i];
    const int64_t n1 = n0 + n_new[i];
    DecodeSeq d{s, i, n1, quantized_len(c, n1)};
    if (n_new[i] > 0) {
      // what this append rewrites: the quantized tokens from the first group (kvarn) or token
      // (q types) it touches, and the ring rows of the new tokens
      const int64_t Q0 = quantized_len(c, n0);
      d.dq = c->fam_k == FAM_KVARN ? (Q0 / GROUP) * GROUP : Q0;
      d.dt = n0;
    }
    dec.push_back(d);
  }
  if (rows > 0 && (!k_bf16 || !v_bf16)) return KVQ_E_INVAL;
  if (rows > 0 && (!aligned16(k_bf16) || !aligned16(v_bf16))) return KVQ_E_ALIGN;
  if (const int rc = check_device(c)) return rc;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  AppendInfo info;
  if (rows > 0) {
    const int rc = launch_append(c, layer, app, k_bf16, v_bf16, st, &info);
    if (rc) return rc;
    for (const AppendSeq &a : app) c->len[(size_t)layer * c->p.n_seqs + a.seq] = a.n0 + a.n_new;
  }
  // the decode overlaps the append's last kernel and plans for every SM: the CTAs that wait
  // for the SMs a small spill still holds are the decode's light ones (its launch order)
  const bool pdl = info.launches > 0;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)D);
  return launch_decode(c, layer, dec, n_q_heads, q, scale, out, workspace, ws_bytes, st, /*budget_sms=*/0, pdl);
}

int kvq_prefill_attn(kvq_cache *c, int32_t layer, int32_t seq, int32_t n_q_tokens, int32_t n_q_heads,
                     const float *q, float softmax_scale, float *out, void *workspace, size_t ws_bytes,
                     kvq_stream_t stream) {
  if (!c || layer < 0 || layer >= c->p.n_layers || seq < 0 || seq >= c->p.n_seqs || n_q_tokens < 0)
    return KVQ_E_INVAL;
  if (n_q_tokens == 0) return KVQ_OK;
  if (!q || !out || !workspace || n_q_heads < 1) return KVQ_E_INVAL;
  if (n_q_heads % c->p.n_kv_heads) return KVQ_E_INVAL;
  if (n_q_heads / c->p.n_kv_heads > MAX_G) return KVQ_E_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_E_ALIGN;
  if (ws_bytes < decode_workspace_bytes(c, n_q_tokens, n_q_heads)) return KVQ_E_SIZE;
  const int64_t n = c->len[(size_t)layer * c->p.n_seqs + seq];
  if (n_q_tokens > n) return KVQ_E_INVAL;
  if (const int rc = check_device(c)) return rc;
  // query i attends to the first n - n_q_tokens + 1 + i tokens of the cache as it is now
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)D);
  return launch_chunk(c, layer, seq, n_q_tokens, n_q_heads, q, scale, out, workspace,
                      reinterpret_cast<cudaStream_t>(stream));
}

int kvq_decode_attn(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
                    int32_t n_q_heads, const float *q, float softmax_scale, float *out, void *workspace,
                    size_t ws_bytes, kvq_stream_t stream) {
  if (!c || layer < 0 || layer >= c->p.n_layers || n_seqs < 0) return KVQ_E_INVAL;
  if (n_seqs == 0) return KVQ_OK;
  if (!seq_ids || !q || !out || !workspace || n_q_heads < 1) return KVQ_E_INVAL;
  if (n_q_heads % c->p.n_kv_heads) return KVQ_E_INVAL;
  if (n_q_heads / c->p.n_kv_heads > MAX_G) return KVQ_E_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_E_ALIGN;
  if (ws_bytes < decode_workspace_bytes(c, n_seqs, n_q_heads)) return KVQ_E_SIZE;
  std::vector<char> seen(c->p.n_seqs, 0);
  std::vector<DecodeSeq> seqs;
  for (int i = 0; i < n_seqs; ++i) {
    int s = seq_ids[i];
    if (s < 0 || s >= c->p.n_seqs || seen[s]) return KVQ_E_INVAL;
    seen[s] = 1;
    int64_t n = c->len[(size_t)layer * c->p.n_seqs + s];
    seqs.push_back({s, i, n, quantized_len(c, n)});
  }
  if (const int rc = check_device(c)) return rc;
  float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)D);
  return launch_decode(c, layer, seqs, n_q_heads, q, scale, out, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int kvq_dequant(kvq_cache *c, int32_t layer, int32_t seq, int32_t which, int64_t t0, int64_t t1,
                int32_t basis, float *out, kvq_stream_t stream) {
  if (!c || layer < 0 || layer >= c->p.n_layers || seq < 0 || seq >= c->p.n_seqs) return KVQ_E_INVAL;
  if (which < 0 || which > 1 || basis < 0 || basis > 1) return KVQ_E_INVAL;
  int64_t n = c->len[(size_t)layer * c->p.n_seqs + seq];
  if (t0 < 0 || t1 < t0 || t1 > n) return KVQ_E_INVAL;
  if (t1 == t0) return KVQ_OK;
  if (!out) return KVQ_E_INVAL;
  if (!aligned16(out)) return KVQ_E_ALIGN;
  if (const int rc = check_device(c)) return rc;
  return launch_dequant(c, layer, seq, which, t0, t1, basis, out, reinterpret_cast<cudaStream_t>(stream));
}

int kvq_seq_len(const kvq_cache *c, int32_t layer, int32_t seq, int64_t *len) {
  if (!c || !len || layer < 0 || layer >= c->p.n_layers || seq < 0 || seq >= c->p.n_seqs)
    return KVQ_E_INVAL;
  *len = c->len[(size_t)layer * c->p.n_seqs + seq];
  return KVQ_OK;
}

int kvq_seq_reset(kvq_cache *c, int32_t seq) {
  if (!c || seq < 0 || seq >= c->p.n_seqs) return KVQ_E_INVAL;
  for (int l = 0; l < c->p.n_layers; ++l) c->len[(size_t)l * c->p.n_seqs + seq] = 0;
  return KVQ_OK;
}

int kvq_locate(const kvq_cache *c, int32_t kind, int32_t layer, int32_t seq, int64_t page, int32_t head,
               int32_t which, int64_t token, size_t *offset, size_t *bytes) {
  if (!c || !offset || !bytes || layer < 0 || layer >= c->p.n_layers || seq < 0 || seq >= c->p.n_seqs ||
      head < 0 || head >= c->p.n_kv_heads || which < 0 || which > 1)
    return KVQ_E_INVAL;
  if (kind == 0) {
    if (page < 0 || page >= c->max_pages) return KVQ_E_INVAL;
    int64_t phys = (int64_t)seq * c->max_pages + page;
    *offset = c->off_pages + c->layer_pages_bytes * layer + phys * c->page_bytes +
              (size_t)head * (c->lk.bytes + c->lv.bytes) + (which ? c->lk.bytes : 0);
    *bytes = which ? c->lv.bytes : c->lk.bytes;
    return KVQ_OK;
  }
  if (kind == 3) {
    // tickets are indexed by (entry of a decode launch, KV head); `seq` is the entry here
    if (seq >= std::max<int32_t>(c->p.n_seqs, kDecodeEntriesPerLaunch)) return KVQ_E_INVAL;
    *offset = c->off_tickets + sizeof(uint32_t) * ((size_t)seq * c->p.n_kv_heads + head);
    *bytes = sizeof(uint32_t);
    return KVQ_OK;
  }
  if (kind == 2) {
    if (page < 0 || page >= c->max_pages) return KVQ_E_INVAL;
    *offset = c->off_ptab + sizeof(int32_t) * ((size_t)seq * c->max_pages + page);
    *bytes = sizeof(int32_t);
    return KVQ_OK;
  }
  if (kind == 1) {
    if (c->ring_cap == 0 || token < 0) return KVQ_E_INVAL;
    *offset = c->off_ring + c->layer_ring_bytes * layer +
              ((((size_t)seq * c->p.n_kv_heads + head) * 2 + which) * c->ring_cap + token % c->ring_cap) *
                  (2 * D);
    *bytes = 2 * D;
    return KVQ_OK;
  }
  return KVQ_E_INVAL;
}

int kvq_get_status(kvq_cache *c, kvq_stream_t stream) {
  if (!c) return KVQ_E_INVAL;
  if (const int rc = check_device(c)) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return KVQ_E_CUDA;
  int32_t st = 0;
  if (cudaMemcpy(&st, c->base + c->off_status, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess)
    return KVQ_E_CUDA;
  if (st != 0) {
    cudaMemset(c->base + c->off_status, 0, sizeof st);
    return KVQ_E_DEVICE;
  }
  return KVQ_OK;
}

const char *kvq_describe(kvq_cache *c) {
  if (!c) return "";
  char buf[512];
  snprintf(buf, sizeof buf,
           "kvq cache: K %s, V %s, tail %d (%s), %d layers x %d seqs x %d KV heads x %d, max_ctx %lld, "
           "sinkhorn_iters %d, %zu bytes (pages %zu/layer, ring %zu/layer)",
           type_name(c->p.type_k), type_name(c->p.type_v), c->p.tail, c->p.tail_f16 ? "F16" : "BF16", c->p.n_layers,
           c->p.n_seqs,
           c->p.n_kv_heads, c->p.head_dim, (long long)c->p.max_ctx, c->p.sinkhorn_iters, c->total,
           c->layer_pages_bytes, c->layer_ring_bytes);
  c->desc = buf;
  return c->desc.c_str();
}

int kvq_launch_count(uint64_t *count) {
  if (!count) return KVQ_E_INVAL;
  *count = g_launches.load(std::memory_order_relaxed);
  return KVQ_OK;
}

const char *kvq_strerror(int code) {
  switch (code) {
    case KVQ_OK: return "ok";
    case KVQ_E_INVAL: return "invalid argument";
    case KVQ_E_UNSUPPORTED: return "unsupported geometry or type";
    case KVQ_E_CAPACITY: return "sequence capacity (max_ctx) exceeded";
    case KVQ_E_ALIGN: return "device pointer not 16-byte aligned";
    case KVQ_E_CUDA: return "CUDA error";
    case KVQ_E_DEVICE: return "device status word reports an error";
    case KVQ_E_SIZE: return "caller buffer too small";
    default: return "unknown error";
  }
}

}  // extern "C"
